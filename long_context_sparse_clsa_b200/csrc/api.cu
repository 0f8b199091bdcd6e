// C ABI of libclsa.so: argument validation, workspace layout and launch order.
// The operations are defined in include/clsa.h; every step of the path runs in
// the kernels of this directory.
#include <algorithm>
#include <cmath>
#include <cstdlib>
#include <cstring>

#include "common.cuh"
#include "kernels.h"

namespace clsa {

const DeviceInfo& device_info() {
  static thread_local int cached_dev = -1;
  static thread_local DeviceInfo info;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) dev = 0;
  if (dev != cached_dev) {
    cudaDeviceGetAttribute(&info.sm_count, cudaDevAttrMultiProcessorCount, dev);
    cudaDeviceGetAttribute(&info.max_smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    cached_dev = dev;
  }
  return info;
}

namespace {
thread_local int g_launches = 0;
thread_local int g_last_launches = 0;
// launch timing: events armed for the next call (pending), and those of the running call
thread_local cudaEvent_t const* g_ev_pending = nullptr;
thread_local int g_ev_pending_max = 0;
thread_local cudaEvent_t const* g_ev = nullptr;
thread_local int g_ev_max = 0, g_ev_n = 0;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }
bool dims_ok(int d) { return d == 64 || d == 128; }
bool dtype_ok(clsa_dtype dt) { return dt == CLSA_F32 || dt == CLSA_BF16; }

clsa_status from_cuda(cudaError_t e) { return e == cudaSuccess ? CLSA_OK : CLSA_ERR_CUDA; }

// attention shape checks shared by clsa_sparse_attn and clsa_decode_step
// kmax: 4096 for the selection paths; clsa_sparse_attn reads K_S/V_S rows directly and
// takes any k up to kMaxDirectK (a whole cache: dense attention)
constexpr int kMaxSelectK = 4096;
constexpr int kMaxDirectK = 1 << 24;
clsa_status check_attn(int B, int k, int L, int Hq, int Hkv, int d, clsa_dtype dt, int kmax = kMaxSelectK) {
  if (B < 1 || k < 1 || L < 1 || Hq < 1 || Hkv < 1) return CLSA_ERR_INVALID_ARG;
  if (!dtype_ok(dt)) return CLSA_ERR_INVALID_ARG;
  if (!dims_ok(d) || Hq % Hkv != 0 || k > kmax) return CLSA_ERR_UNSUPPORTED;
  const int G = Hq / Hkv;
  if (G > (dt == CLSA_BF16 ? 128 : 32)) return CLSA_ERR_UNSUPPORTED;
  return CLSA_OK;
}

struct DecodeLayout {
  bool fused = false;
  size_t scores = 0, topk = 0, attn = 0, total = 0;
};

// CLSA_DECODE_PLAN=unfused forces the four-kernel path (scan, top-k, attention, combine)
bool fused_allowed() {
  const char* v = std::getenv("CLSA_DECODE_PLAN");
  return !(v && std::strcmp(v, "unfused") == 0);
}

DecodeLayout decode_layout(const clsa_decode_args* a) {
  DecodeLayout l;
  if (fused_allowed() && fused_decode_supported(a)) {
    l.fused = true;
    l.total = kWsHeader + fused_decode_ws_bytes(a);
    return l;
  }
  size_t off = kWsHeader;
  if (!a->scores) {
    l.scores = off;
    off += align_up((size_t)a->B * a->n_max * sizeof(float), 256);
  }
  l.topk = off;
  off += topk_ws_bytes(a->B, a->n_max, a->k);
  AttnShape sh{a->B, a->k, a->L, a->Hq, a->Hkv, a->d, a->dtype, a->K_S == nullptr, a->n_max, a->n_max};
  l.attn = off;
  off += attn_ws_bytes(sh);
  l.total = off;
  return l;
}

clsa_status check_decode(const clsa_decode_args* a) {
  if (!a) return CLSA_ERR_INVALID_ARG;
  clsa_status st = check_attn(a->B, a->k, a->L, a->Hq, a->Hkv, a->d, a->dtype);
  if (st != CLSA_OK) return st;
  if (a->n_max < 1) return CLSA_ERR_INVALID_ARG;
  if (!dims_ok(a->d_idx)) return CLSA_ERR_UNSUPPORTED;
  if (!a->q_idx || !a->k_idx || !a->K || !a->V || !a->Q || !a->seq_lens || !a->O || !a->idx || !a->count)
    return CLSA_ERR_INVALID_ARG;
  if ((a->K_S == nullptr) != (a->V_S == nullptr)) return CLSA_ERR_INVALID_ARG;
  for (const void* p : {a->q_idx, a->k_idx, a->K, a->V, a->Q, (const void*)a->O, (const void*)a->K_S,
                        (const void*)a->V_S})
    if (p && !aligned16(p)) return CLSA_ERR_INVALID_ARG;
  for (const void* p : {(const void*)a->seq_lens, (const void*)a->idx, (const void*)a->count,
                        (const void*)a->scores, (const void*)a->lse})
    if (p && !aligned4(p)) return CLSA_ERR_INVALID_ARG;
  return CLSA_OK;
}

float resolve_scale(float scale, int d) { return scale > 0.f ? scale : 1.0f / std::sqrt((float)d); }

}  // namespace

CallScope::CallScope(void* stream) {
  g_launches = 0;
  g_ev = nullptr;
  if (g_ev_pending) {  // an armed call: event 0 before its first launch
    g_ev = g_ev_pending;
    g_ev_max = g_ev_pending_max;
    g_ev_pending = nullptr;
    g_ev_n = 0;
    if (g_ev_max > 0) {
      if (cudaEventRecord(g_ev[0], static_cast<cudaStream_t>(stream)) == cudaSuccess) {
        g_ev_n = 1;
      } else {  // not a valid event: record nothing, and leave no error behind for the launches
        (void)cudaGetLastError();
        g_ev = nullptr;
      }
    }
  }
}
CallScope::~CallScope() {
  g_last_launches = g_launches;
  g_ev = nullptr;
}

void launches_reset() { g_launches = 0; }
void launches_add(int n, cudaStream_t s) {
  g_launches += n;
  if (g_ev && g_ev_n < g_ev_max) {
    if (cudaEventRecord(g_ev[g_ev_n], s) == cudaSuccess) {
      ++g_ev_n;
    } else {
      (void)cudaGetLastError();
      g_ev = nullptr;
    }
  }
}
int launches_get() { return g_launches; }

}  // namespace clsa

using namespace clsa;

extern "C" {

int clsa_version(void) { return 100; }  // 0.1.0

int clsa_last_launch_count(void) { return clsa::g_last_launches; }

clsa_status clsa_time_next_call(void* const* events, int max_events) {
  if (max_events < 0 || (max_events > 0 && !events)) return CLSA_ERR_INVALID_ARG;
  clsa::g_ev_pending = max_events > 0 ? reinterpret_cast<cudaEvent_t const*>(events) : nullptr;
  clsa::g_ev_pending_max = max_events;
  return CLSA_OK;
}

int clsa_timed_event_count(void) { return clsa::g_ev_n; }

const char* clsa_status_string(clsa_status s) {
  switch (s) {
    case CLSA_OK: return "CLSA_OK";
    case CLSA_ERR_INVALID_ARG: return "CLSA_ERR_INVALID_ARG";
    case CLSA_ERR_UNSUPPORTED: return "CLSA_ERR_UNSUPPORTED";
    case CLSA_ERR_WORKSPACE: return "CLSA_ERR_WORKSPACE";
    case CLSA_ERR_CUDA: return "CLSA_ERR_CUDA";
    case CLSA_ERR_TIMEOUT: return "CLSA_ERR_TIMEOUT";
    case CLSA_ERR_BAD_INDEX: return "CLSA_ERR_BAD_INDEX";
  }
  return "CLSA_ERR_UNKNOWN";
}

size_t clsa_workspace_size(int op, const void* args) {
  if (!args) return 0;
  switch (op) {
    case CLSA_OP_DECODE_STEP: return clsa_decode_workspace_size(static_cast<const clsa_decode_args*>(args));
    case CLSA_OP_PREFILL_CHUNK: return clsa_prefill_workspace_size(static_cast<const clsa_prefill_args*>(args));
    default: return 0;
  }
}

clsa_status clsa_workspace_init(void* ws, size_t bytes, void* stream) {
  if (!ws || bytes < kWsHeader) return CLSA_ERR_INVALID_ARG;
  return from_cuda(cudaMemsetAsync(ws, 0, bytes, static_cast<cudaStream_t>(stream)));
}

clsa_status clsa_selftest_timeout(int which, void* ws, size_t ws_bytes, void* stream) {
  CallScope scope(stream);
  if (which != 0 && which != 1) return CLSA_ERR_INVALID_ARG;
  if (!ws || ws_bytes < kWsHeader + 256 || !aligned16(ws)) return CLSA_ERR_WORKSPACE;
  char* w = static_cast<char*>(ws);
  return from_cuda(launch_selftest_timeout(which, w, w + kWsHeader, static_cast<cudaStream_t>(stream)));
}

clsa_status clsa_read_device_status(void* ws, void* stream, int64_t* detail) {
  if (!ws) return CLSA_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  struct {
    uint32_t code, pad;
    int64_t detail;
  } h{};
  if (cudaMemcpyAsync(&h, ws, sizeof(h), cudaMemcpyDeviceToHost, s) != cudaSuccess) return CLSA_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return CLSA_ERR_CUDA;
  if (h.code != 0) {
    if (cudaMemsetAsync(ws, 0, 16, s) != cudaSuccess) return CLSA_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return CLSA_ERR_CUDA;
  }
  if (detail) *detail = h.detail;
  return static_cast<clsa_status>(h.code);
}

clsa_status clsa_index_scores(const void* q_idx, const void* k_idx, const int32_t* seq_lens, int B, int n_max,
                              int d_idx, clsa_dtype dt, float* scores, void* stream) {
  CallScope scope(stream);
  if (!q_idx || !k_idx || !seq_lens || !scores || B < 1 || n_max < 1 || !dtype_ok(dt))
    return CLSA_ERR_INVALID_ARG;
  if (!dims_ok(d_idx)) return CLSA_ERR_UNSUPPORTED;
  if (!aligned16(q_idx) || !aligned16(k_idx) || !aligned4(seq_lens) || !aligned4(scores))
    return CLSA_ERR_INVALID_ARG;
  return from_cuda(launch_index_scores(q_idx, k_idx, seq_lens, B, n_max, d_idx, dt, scores, nullptr,
                                       static_cast<cudaStream_t>(stream)));
}

size_t clsa_topk_workspace_size(int B, int n_max, int k) {
  if (B < 1 || n_max < 1 || k < 1) return 0;
  return kWsHeader + topk_ws_bytes(B, n_max, k);
}

clsa_status clsa_topk(const float* scores, const int32_t* seq_lens, int B, int n_max, int k, int32_t* idx,
                      int32_t* count, void* ws, size_t ws_bytes, void* stream) {
  CallScope scope(stream);
  if (!scores || !seq_lens || !idx || !count || B < 1 || n_max < 1 || k < 1) return CLSA_ERR_INVALID_ARG;
  if (k > 4096) return CLSA_ERR_UNSUPPORTED;
  for (const void* p : {(const void*)scores, (const void*)seq_lens, (const void*)idx, (const void*)count})
    if (!aligned4(p)) return CLSA_ERR_INVALID_ARG;
  if (!ws || ws_bytes < clsa_topk_workspace_size(B, n_max, k) || !aligned16(ws)) return CLSA_ERR_WORKSPACE;
  char* w = static_cast<char*>(ws);
  return from_cuda(launch_topk(scores, seq_lens, B, n_max, k, idx, count, w, w + kWsHeader,
                               static_cast<cudaStream_t>(stream)));
}

size_t clsa_gather_kv_workspace_size(void) { return kWsHeader; }

clsa_status clsa_gather_kv(const void* K, const void* V, const int32_t* idx, const int32_t* count, int B,
                           int n_max, int k, int Hkv, int d, clsa_dtype dt, void* K_S, void* V_S, void* ws,
                           size_t ws_bytes, void* stream) {
  CallScope scope(stream);
  if (!K || !V || !idx || !count || !K_S || !V_S || B < 1 || n_max < 1 || k < 1 || Hkv < 1 || !dtype_ok(dt))
    return CLSA_ERR_INVALID_ARG;
  if (!dims_ok(d) || k > 4096) return CLSA_ERR_UNSUPPORTED;
  for (const void* p : {K, V, (const void*)K_S, (const void*)V_S})
    if (!aligned16(p)) return CLSA_ERR_INVALID_ARG;
  if (!aligned4(idx) || !aligned4(count)) return CLSA_ERR_INVALID_ARG;
  if (!ws || ws_bytes < kWsHeader || !aligned16(ws)) return CLSA_ERR_WORKSPACE;
  return from_cuda(launch_gather_kv(K, V, idx, count, B, n_max, k, Hkv, d, dt, K_S, V_S, ws,
                                    static_cast<cudaStream_t>(stream)));
}

size_t clsa_sparse_attn_workspace_size(int B, int k, int L, int Hq, int Hkv, int d) {
  if (check_attn(B, k, L, Hq, Hkv, d, CLSA_BF16, kMaxDirectK) != CLSA_OK) return 0;
  // the larger of the bf16 and fp32 plans, so one size serves both dtypes
  AttnShape a{B, k, L, Hq, Hkv, d, CLSA_BF16, false, 0, 0};
  AttnShape f{B, k, L, Hq, Hkv, d, CLSA_F32, false, 0, 0};
  return kWsHeader + std::max(attn_ws_bytes(a), attn_ws_bytes(f));
}

clsa_status clsa_sparse_attn(const void* Q, const void* K_S, const void* V_S, const int32_t* count, int B, int k,
                             int L, int Hq, int Hkv, int d, float scale, clsa_dtype dt, void* O, float* lse,
                             void* ws, size_t ws_bytes, void* stream) {
  CallScope scope(stream);
  clsa_status st = check_attn(B, k, L, Hq, Hkv, d, dt, kMaxDirectK);
  if (st != CLSA_OK) return st;
  if (!Q || !K_S || !V_S || !count || !O) return CLSA_ERR_INVALID_ARG;
  for (const void* p : {Q, K_S, V_S, (const void*)O})
    if (!aligned16(p)) return CLSA_ERR_INVALID_ARG;
  if (!aligned4(count) || (lse && !aligned4(lse))) return CLSA_ERR_INVALID_ARG;
  if (!ws || ws_bytes < clsa_sparse_attn_workspace_size(B, k, L, Hq, Hkv, d) || !aligned16(ws))
    return CLSA_ERR_WORKSPACE;
  AttnShape sh{B, k, L, Hq, Hkv, d, dt, false, 0, 0};
  char* w = static_cast<char*>(ws);
  return from_cuda(launch_sparse_attn(sh, Q, K_S, V_S, nullptr, count, resolve_scale(scale, d), O, lse, w,
                                      w + kWsHeader, static_cast<cudaStream_t>(stream)));
}

size_t clsa_distill_workspace_size(int B, int n_max, int L, int Hq, int Hkv, int d) {
  if (check_attn(B, n_max, L, Hq, Hkv, d, CLSA_BF16, kMaxDirectK) != CLSA_OK) return 0;
  return kWsHeader + std::max(distill_ws_bytes(B, n_max, L, Hq, Hkv, d, CLSA_BF16),
                              distill_ws_bytes(B, n_max, L, Hq, Hkv, d, CLSA_F32));
}

clsa_status clsa_distill_target(const void* Q, const void* K, const float* scores, const int32_t* seq_lens, int B,
                                int n_max, int L, int Hq, int Hkv, int d, float scale, clsa_dtype dt, float* abar,
                                float* kl, void* ws, size_t ws_bytes, void* stream) {
  CallScope scope(stream);
  clsa_status st = check_attn(B, n_max, L, Hq, Hkv, d, dt, kMaxDirectK);
  if (st != CLSA_OK) return st;
  if (!Q || !K || !scores || !seq_lens || !kl) return CLSA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned4(scores) || !aligned4(seq_lens) || !aligned4(kl) ||
      (abar && !aligned4(abar)))
    return CLSA_ERR_INVALID_ARG;
  if (!ws || ws_bytes < clsa_distill_workspace_size(B, n_max, L, Hq, Hkv, d) || !aligned16(ws))
    return CLSA_ERR_WORKSPACE;
  char* w = static_cast<char*>(ws);
  return from_cuda(launch_distill(Q, K, scores, seq_lens, B, n_max, L, Hq, Hkv, d, resolve_scale(scale, d), dt, abar,
                                  kl, w, w + kWsHeader, static_cast<cudaStream_t>(stream)));
}

size_t clsa_attention_mass_workspace_size(int B, int n_max, int L, int Hq, int Hkv, int d) {
  if (check_attn(B, n_max, L, Hq, Hkv, d, CLSA_BF16, kMaxDirectK) != CLSA_OK) return 0;
  return kWsHeader + std::max(attention_mass_ws_bytes(B, n_max, L, Hq, Hkv, d, CLSA_BF16),
                              attention_mass_ws_bytes(B, n_max, L, Hq, Hkv, d, CLSA_F32));
}

clsa_status clsa_attention_mass(const void* Q, const void* K, const float* lse_sparse, const int32_t* seq_lens, int B,
                                int n_max, int L, int Hq, int Hkv, int d, float scale, clsa_dtype dt, float* mass,
                                float* lse_all, void* ws, size_t ws_bytes, void* stream) {
  CallScope scope(stream);
  clsa_status st = check_attn(B, n_max, L, Hq, Hkv, d, dt, kMaxDirectK);
  if (st != CLSA_OK) return st;
  if (!Q || !K || !lse_sparse || !seq_lens || !mass) return CLSA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned4(lse_sparse) || !aligned4(seq_lens) || !aligned4(mass) ||
      (lse_all && !aligned4(lse_all)))
    return CLSA_ERR_INVALID_ARG;
  if (!ws || ws_bytes < clsa_attention_mass_workspace_size(B, n_max, L, Hq, Hkv, d) || !aligned16(ws))
    return CLSA_ERR_WORKSPACE;
  char* w = static_cast<char*>(ws);
  return from_cuda(launch_attention_mass(Q, K, lse_sparse, seq_lens, B, n_max, L, Hq, Hkv, d, resolve_scale(scale, d),
                                         dt, mass, lse_all, w, w + kWsHeader, static_cast<cudaStream_t>(stream)));
}

size_t clsa_decode_workspace_size(const clsa_decode_args* a) {
  if (check_decode(a) != CLSA_OK) return 0;
  return decode_layout(a).total;
}

clsa_status clsa_decode_step(const clsa_decode_args* a, void* ws, size_t ws_bytes, void* stream) {
  CallScope scope(stream);
  clsa_status st = check_decode(a);
  if (st != CLSA_OK) return st;
  const DecodeLayout lay = decode_layout(a);
  if (!ws || ws_bytes < lay.total || !aligned16(ws)) return CLSA_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  char* w = static_cast<char*>(ws);
  if (lay.fused) return from_cuda(launch_decode_fused(a, resolve_scale(a->scale, a->d), w, w + kWsHeader, s));
  float* scores = a->scores ? a->scores : reinterpret_cast<float*>(w + lay.scores);
  cudaError_t e = launch_index_scores(a->q_idx, a->k_idx, a->seq_lens, a->B, a->n_max, a->d_idx, a->dtype,
                                      scores, w, s);
  if (e != cudaSuccess) return CLSA_ERR_CUDA;
  e = launch_topk(scores, a->seq_lens, a->B, a->n_max, a->k, a->idx, a->count, w, w + lay.topk, s);
  if (e != cudaSuccess) return CLSA_ERR_CUDA;
  const float scale = resolve_scale(a->scale, a->d);
  if (a->K_S) {
    e = launch_gather_kv(a->K, a->V, a->idx, a->count, a->B, a->n_max, a->k, a->Hkv, a->d, a->dtype, a->K_S,
                         a->V_S, w, s);
    if (e != cudaSuccess) return CLSA_ERR_CUDA;
    AttnShape sh{a->B, a->k, a->L, a->Hq, a->Hkv, a->d, a->dtype, false, a->n_max, a->n_max};
    e = launch_sparse_attn(sh, a->Q, a->K_S, a->V_S, nullptr, a->count, scale, a->O, a->lse, w, w + lay.attn, s);
  } else {
    AttnShape sh{a->B, a->k, a->L, a->Hq, a->Hkv, a->d, a->dtype, true, a->n_max, a->n_max};
    e = launch_sparse_attn(sh, a->Q, a->K, a->V, a->idx, a->count, scale, a->O, a->lse, w, w + lay.attn, s);
  }
  return from_cuda(e);
}

size_t clsa_prefill_workspace_size(const clsa_prefill_args* a) {
  if (!a) return 0;
  const size_t body = prefill_ws_bytes(a);
  return body ? kWsHeader + body : 0;
}

clsa_status clsa_prefill_chunk(const clsa_prefill_args* a, void* ws, size_t ws_bytes, void* stream) {
  CallScope scope(stream);
  if (!a) return CLSA_ERR_INVALID_ARG;
  clsa_status st = check_attn(a->T, a->k, a->L, a->Hq, a->Hkv, a->d, a->dtype);
  if (st != CLSA_OK) return st;
  if (a->dtype != CLSA_BF16) return CLSA_ERR_UNSUPPORTED;
  if (a->n < 1 || a->T < 1 || a->T > a->n) return CLSA_ERR_INVALID_ARG;
  if (!dims_ok(a->d_idx)) return CLSA_ERR_UNSUPPORTED;
  if (!a->q_idx || !a->k_idx || !a->K || !a->V || !a->Q || !a->O || !a->idx || !a->count)
    return CLSA_ERR_INVALID_ARG;
  for (const void* p : {a->q_idx, a->k_idx, a->K, a->V, a->Q, (const void*)a->O})
    if (!aligned16(p)) return CLSA_ERR_INVALID_ARG;
  if (!aligned4(a->idx) || !aligned4(a->count) || (a->lse && !aligned4(a->lse))) return CLSA_ERR_INVALID_ARG;
  const size_t need = clsa_prefill_workspace_size(a);
  if (!ws || need == 0 || ws_bytes < need || !aligned16(ws)) return CLSA_ERR_WORKSPACE;
  char* w = static_cast<char*>(ws);
  return run_prefill(a, w, w + kWsHeader, static_cast<cudaStream_t>(stream));
}

clsa_status clsa_prefill_attention(const clsa_prefill_args* a, int mode, void* ws, size_t ws_bytes, void* stream) {
  CallScope scope(stream);
  if (!a || (mode != 0 && mode != 1)) return CLSA_ERR_INVALID_ARG;
  clsa_status st = check_attn(a->T, a->k, a->L, a->Hq, a->Hkv, a->d, a->dtype);
  if (st != CLSA_OK) return st;
  if (a->dtype != CLSA_BF16) return CLSA_ERR_UNSUPPORTED;
  if (a->n < 1 || a->T < 1 || a->T > a->n) return CLSA_ERR_INVALID_ARG;
  if (!dims_ok(a->d_idx)) return CLSA_ERR_UNSUPPORTED;
  if (!a->K || !a->V || !a->Q || !a->O || !a->idx || !a->count) return CLSA_ERR_INVALID_ARG;
  for (const void* p : {a->K, a->V, a->Q, (const void*)a->O})
    if (!aligned16(p)) return CLSA_ERR_INVALID_ARG;
  if (!aligned4(a->idx) || !aligned4(a->count) || (a->lse && !aligned4(a->lse))) return CLSA_ERR_INVALID_ARG;
  if (mode == 1 && !prefill_attn_pair_supported(a)) return CLSA_ERR_UNSUPPORTED;
  const size_t need = clsa_prefill_workspace_size(a);
  if (!ws || need == 0 || ws_bytes < need || !aligned16(ws)) return CLSA_ERR_WORKSPACE;
  char* w = static_cast<char*>(ws);
  return run_prefill_attention(a, mode, w, w + kWsHeader, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
