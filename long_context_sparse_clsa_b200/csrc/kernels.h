// Internal launchers used by the C ABI layer (api.cu).  Host code only.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/clsa.h"

namespace clsa {

struct DeviceInfo {
  int sm_count = 0;
  int max_smem_optin = 0;
};
const DeviceInfo& device_info();

// per-host-thread count of kernel launches in the current API call; an entry point
// holds a CallScope (with its stream) for its duration, so clsa_last_launch_count()
// reports its launches, and a call armed by clsa_time_next_call records its events
struct CallScope {
  explicit CallScope(void* stream = nullptr);
  ~CallScope();
};
void launches_reset();
// after each kernel launch (or group of n launches) on stream s
void launches_add(int n, cudaStream_t s);
int launches_get();

// ----- indexer scan (routing equation, scores) ------------------------------
// ws_header: the call's error word (a bounded wait that runs out records CLSA_ERR_TIMEOUT), or null
cudaError_t launch_index_scores(const void* q_idx, const void* k_idx, const int32_t* seq_lens, int B,
                                int n_max, int d_idx, clsa_dtype dt, float* scores, void* ws_header,
                                cudaStream_t s);

// ----- exact radix top-k -----------------------------------------------------
size_t topk_ws_bytes(int B, int n_max, int k);
// causal_base >= 0: row b has length causal_base + b + 1 and seq_lens is ignored.
// row_skip: rows with row_skip[b] == skip_val are left untouched.  idx_map: the row's
// selected positions j are written as idx_map[b * ld_map + j] (positions are ascending,
// so ascending maps stay ascending).
cudaError_t launch_topk(const float* scores, const int32_t* seq_lens, int B, int n_max, int k,
                        int32_t* idx, int32_t* count, void* ws_header, void* topk_ws, cudaStream_t s,
                        int causal_base = -1, const int32_t* row_skip = nullptr, int skip_val = 0,
                        const int32_t* idx_map = nullptr, int ld_map = 0);

// ----- selector gather --------------------------------------------------------
cudaError_t launch_gather_kv(const void* K, const void* V, const int32_t* idx, const int32_t* count, int B,
                             int n_max, int k, int Hkv, int d, clsa_dtype dt, void* K_S, void* V_S,
                             void* ws_header, cudaStream_t s);

// ----- sparse attention (split-k flash decoding) ----------------------------
struct AttnShape {
  int B, k, L, Hq, Hkv, d;
  clsa_dtype dt;
  // gather mode: rows come from the full cache through idx
  bool gather;
  int n_max;
  // cache rows per sequence in gather mode (n_max; 0 = one cache shared by every b)
  long long kv_bstride;
};
struct AttnPlan {
  int Lg;       // layers per CTA row-group
  int nlg;      // layer groups
  int rows;     // Lg * G rows per CTA
  int nsplit;   // token splits per (b, kv head, layer group)
  int chunk;    // tokens per split (multiple of 64)
};
AttnPlan plan_attention(const AttnShape& sh);
size_t attn_ws_bytes(const AttnShape& sh);
cudaError_t launch_sparse_attn(const AttnShape& sh, const void* Q, const void* Kc, const void* Vc,
                               const int32_t* idx, const int32_t* count, float scale, void* O, float* lse,
                               void* ws_header, void* attn_ws, cudaStream_t s);
// few rows per KV head (bf16, L * G <= 16, d = 64 or 128): CUDA cores, splits merged in-kernel;
// false if the shape is outside it.  The plan it fills is the one plan_attention returns.
bool sparse_attn_rows_plan(const AttnShape& sh, int sm_count, AttnPlan* pl);
cudaError_t launch_sparse_attn_rows(const AttnShape& sh, const AttnPlan& pl, const void* Q, const void* Kc,
                                    const void* Vc, const int32_t* idx, const int32_t* count, float scale_log2,
                                    void* O, float* lse, float* Op, float* Mp, float* Lp, uint32_t* counter,
                                    void* ws_header, cudaStream_t s);
// the same attention on tcgen05 (bf16, d = 128, rows <= 128); partials as the split-k path's
bool sparse_attn_tc_supported(const AttnShape& sh, const AttnPlan& pl, const void* Q, const void* K, const void* V,
                              const void* O);
cudaError_t launch_sparse_attn_tc(const AttnShape& sh, const AttnPlan& pl, const void* Q, const void* Kc,
                                  const void* Vc, const int32_t* idx, const int32_t* count, float scale_log2, void* O,
                                  float* lse, float* Op, float* Mp, float* Lp, void* ws_header, cudaStream_t s);

// ----- distillation target (forward): Abar and KL(Abar || softmax(I)) ----------------
size_t distill_ws_bytes(int B, int n_max, int L, int Hq, int Hkv, int d, clsa_dtype dt);
cudaError_t launch_distill(const void* Q, const void* K, const float* scores, const int32_t* lens, int B, int n_max,
                           int L, int Hq, int Hkv, int d, float scale, clsa_dtype dt, float* abar, float* kl,
                           void* ws_header, void* ws, cudaStream_t s);
// tcgen05 path (bf16, d = 128, G <= 128): two streaming passes over the cache
bool distill_tc_supported(int B, int n_max, int L, int Hq, int Hkv, int d, clsa_dtype dt);
size_t distill_tc_ws_bytes(int B, int n_max, int L, int Hq, int Hkv);
cudaError_t launch_distill_tc(const void* Q, const void* K, const float* scores, const int32_t* lens, int B, int n_max,
                              int L, int Hq, int Hkv, float scale, float* abar, float* kl, void* ws_header, void* ws,
                              cudaStream_t s);

// ----- attention-mass coverage: exp(lse_S - lse_all) per (layer, sequence, query head) -----
size_t attention_mass_ws_bytes(int B, int n_max, int L, int Hq, int Hkv, int d, clsa_dtype dt);
cudaError_t launch_attention_mass(const void* Q, const void* K, const float* lse_sparse, const int32_t* lens, int B,
                                  int n_max, int L, int Hq, int Hkv, int d, float scale, clsa_dtype dt, float* mass,
                                  float* lse_all, void* ws_header, void* ws, cudaStream_t s);
size_t attention_mass_tc_ws_bytes(int B, int n_max, int L, int Hq, int Hkv);
cudaError_t launch_attention_mass_tc(const void* Q, const void* K, const float* lse_sparse, const int32_t* lens, int B,
                                     int n_max, int L, int Hq, int Hkv, float scale, float* mass, float* lse_all,
                                     void* ws_header, void* ws, cudaStream_t s);

// ----- failure-detection self-test (a wait that runs out and reports) ------------
cudaError_t launch_selftest_timeout(int which, void* ws_header, void* ws_body, cudaStream_t s);

// ----- fused decode step (one cooperative launch) -------------------------------
bool fused_decode_supported(const clsa_decode_args* a);
size_t fused_decode_ws_bytes(const clsa_decode_args* a);
cudaError_t launch_decode_fused(const clsa_decode_args* a, float scale, void* ws_header, void* ws_body,
                                cudaStream_t s);

// ----- prefill ------------------------------------------------------------------
struct PrefillRouteBufs {
  uint32_t* dval;     // [T][ldd] dense candidate scores (fp32 bits)
  int32_t* dtok;      // [T][ldd] their token indices (ascending per row)
  int32_t* dlen;      // [T] candidates per row (0 for a flagged row)
  int32_t* flag;      // [T] 1: the row needs the exact fallback
  uint32_t* any_flag; // some row is flagged
  int ldd;
};
bool prefill_route_supported(const clsa_prefill_args* a);
int prefill_route_ldd(const clsa_prefill_args* a);  // dense candidate row length
size_t prefill_route_ws_bytes(const clsa_prefill_args* a);
cudaError_t launch_prefill_route(const clsa_prefill_args* a, void* ws_header, void* ws, cudaStream_t s,
                                 PrefillRouteBufs* out);
// per-row sparse attention of a prefill chunk on tcgen05 (bf16, d = 128); else the split-k kernel
bool prefill_attn_tc_supported(const clsa_prefill_args* a);
cudaError_t launch_prefill_attn_tc(const clsa_prefill_args* a, float scale, void* ws_header, cudaStream_t s);
// key-centric prefill attention: pairs of new rows over the union of their selections (tcgen05)
bool prefill_attn_pair_supported(const clsa_prefill_args* a);
cudaError_t launch_prefill_attn_pair(const clsa_prefill_args* a, float scale, void* ws_header, cudaStream_t s);
size_t prefill_ws_bytes(const clsa_prefill_args* a);
clsa_status run_prefill(const clsa_prefill_args* a, void* ws_header, void* ws_body, cudaStream_t s);
// the attention stage alone over a->idx / a->count: mode 0 per row, mode 1 key-centric row pairs
clsa_status run_prefill_attention(const clsa_prefill_args* a, int mode, void* ws_header, void* ws_body,
                                  cudaStream_t s);

}  // namespace clsa
