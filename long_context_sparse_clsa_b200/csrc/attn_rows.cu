// Token-sparse GQA attention for few rows per KV head (L*G <= 16: one layer's heads, the
// model-faithful per-layer decode call), bf16, d = 64 or 128:
//   O^(l)[b, h] = softmax(Q^(l)[b, h] K_S^T * scale) V_S
// (picx.dev CLSA summary, Methodology > Architecture Overview, per-layer equation).
//
// With 4 query rows per KV head the products are a few hundred thousand multiply-adds per
// CTA, too small to keep a tensor-core pipeline busy; the time is the latency of moving
// K_S/V_S in and the result out.  So the kernel runs on the CUDA cores and is built to take
// few dependent round trips:
//   1. one CTA per (token split, KV head, sequence): its Q rows and its <= 128 selected K/V
//      rows land in shared memory in one wave of 16-byte async copies;
//   2. scores (one thread per token and four rows), the split's row max and sum, P V
//      (one thread per four columns and two rows), all from shared memory;
//   3. the split's unnormalised output, max and sum go to the split partials; the CTA that
//      arrives last at its (sequence, head) counter merges the splits with the log-sum-exp
//      rule, writes O and the LSE, and returns the counter to zero.
// No second kernel, no grid barrier.  Index checks and counters as in the other paths.
#include <algorithm>
#include <cmath>

#include "common.cuh"
#include "kernels.h"

namespace clsa {

namespace {

constexpr int kThreadsR = 256;
constexpr int kMaxRowsR = 16;
constexpr int kMaxTokR = 128;  // tokens per CTA
constexpr int kMaxSplitR = 64;
constexpr float kLn2R = 0.6931471805599453f;

struct RowsParams {
  const __nv_bfloat16* Q;   // [L][B][Hq][D]
  const __nv_bfloat16* K;   // token r of sequence b, head g: row ((b * kv_bstride + r) * Hkv + g)
  const __nv_bfloat16* V;
  const int32_t* idx;       // [B][k] or null (compact: position i is row i)
  const int32_t* count;     // [B]
  __nv_bfloat16* O;         // [L][B][Hq][D]
  float* lse;               // [L][B][Hq] or null
  float* Op;                // [B][Hkv][nsplit][rows][D]
  float* Mp;                // [B][Hkv][nsplit][rows]  (log2 units)
  float* Lp;
  uint32_t* counter;        // [B][Hkv], zero between calls
  void* ws_header;
  long long kv_bstride;
  int B, k, L, Hq, Hkv, G, rows, n_max, nsplit, chunk;
  float scale_log2;
};

template <int D>
struct RowsSmem {
  static constexpr int KSTR = D + 8;  // padded K row (elements): conflict-free row-per-lane reads
  __nv_bfloat16 K[kMaxTokR][KSTR];
  __nv_bfloat16 V[kMaxTokR][D];
  __nv_bfloat16 Q[kMaxRowsR][D];
  float S[kMaxRowsR][kMaxTokR];     // scores, then P
  float m[kMaxRowsR], l[kMaxRowsR];
  float w[kMaxSplitR][kMaxRowsR];   // merge weights
  float inv[kMaxRowsR];
  int tok[kMaxTokR];
  int last;
};

template <int D>
__global__ void __launch_bounds__(kThreadsR) attn_rows_kernel(const RowsParams p) {
  pdl_enter();  // launched programmatically: the previous kernel's writes first
  extern __shared__ __align__(16) unsigned char smem_raw[];
  RowsSmem<D>& sm = *reinterpret_cast<RowsSmem<D>*>(smem_raw);
  constexpr int VPR = D / 8;  // 16-byte vectors per row
  const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int R = p.rows;
  const int cnt = max(0, min(p.count[b], p.k));
  const int t0 = split * p.chunk;
  const int ntok = max(0, min(cnt, t0 + p.chunk) - t0);

  // ---- 1. the split's token rows, Q rows, K/V rows ---------------------------------------
  for (int i = tid; i < ntok; i += kThreadsR) {
    const int tk = p.idx ? __ldg(p.idx + (size_t)b * p.k + t0 + i) : t0 + i;
    const bool ok = (unsigned)tk < (unsigned)p.n_max;
    if (!ok) record_error(p.ws_header, CLSA_ERR_BAD_INDEX, ((long long)b << 32) | (unsigned)(t0 + i));
    sm.tok[i] = ok ? tk : -1;
  }
  for (int v = tid; v < R * VPR; v += kThreadsR) {  // row r = (layer r / G, head g * G + r % G)
    const int r = v / VPR, c = v % VPR;
    const int l = r / p.G, h = g * p.G + r % p.G;
    cp_async_16(&sm.Q[r][c * 8], p.Q + (((size_t)l * p.B + b) * p.Hq + h) * D + c * 8, 16);
  }
  __syncthreads();  // tokens visible
  const size_t gstride = (size_t)p.Hkv * D;
  const size_t gbase = (size_t)b * (size_t)p.kv_bstride * gstride + (size_t)g * D;
  for (int v = tid; v < ntok * VPR; v += kThreadsR) {
    const int i = v / VPR, c = v % VPR;
    const int tk = sm.tok[i];
    const size_t off = tk >= 0 ? gbase + (size_t)tk * gstride + c * 8 : 0;
    cp_async_16(&sm.K[i][c * 8], p.K + off, tk >= 0 ? 16 : 0);
    cp_async_16(&sm.V[i][c * 8], p.V + off, tk >= 0 ? 16 : 0);
  }
  cp_async_commit();
  cp_async_wait<0>();
  __syncthreads();

  // ---- 2a. scores: thread = (token t, rows rg, rg + 4, rg + 8, rg + 12) --------------------
  {
    const int t = tid & 63;   // 64 tokens per pass
    const int rg = tid >> 6;                   // 0..3
#pragma unroll 1
    for (int tb = 0; tb < ntok; tb += 64) {
      const int tt = tb + t;
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
      if (tt < ntok) {
#pragma unroll 4
        for (int c = 0; c < VPR; ++c) {
          const uint4 kv = *reinterpret_cast<const uint4*>(&sm.K[tt][c * 8]);
          float kf[8];
          unpack_bf16x2(kv.x, kf[0], kf[1]);
          unpack_bf16x2(kv.y, kf[2], kf[3]);
          unpack_bf16x2(kv.z, kf[4], kf[5]);
          unpack_bf16x2(kv.w, kf[6], kf[7]);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int r = rg + 4 * j;
            if (r < R) {
              const uint4 qv = *reinterpret_cast<const uint4*>(&sm.Q[r][c * 8]);  // broadcast
              float qf[8];
              unpack_bf16x2(qv.x, qf[0], qf[1]);
              unpack_bf16x2(qv.y, qf[2], qf[3]);
              unpack_bf16x2(qv.z, qf[4], qf[5]);
              unpack_bf16x2(qv.w, qf[6], qf[7]);
#pragma unroll
              for (int e = 0; e < 8; ++e) acc[j] = fmaf(qf[e], kf[e], acc[j]);
            }
          }
        }
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int r = rg + 4 * j;
        if (r < R && tt < kMaxTokR) sm.S[r][tt] = tt < ntok ? acc[j] * p.scale_log2 : -INFINITY;
      }
    }
  }
  __syncthreads();

  // ---- 2b. row max / exponentials / sum: warp w takes rows w and w + 8 ---------------------
  for (int r = warp; r < R; r += kThreadsR / 32) {
    float mx = -INFINITY;
    for (int t = lane; t < ntok; t += 32) mx = fmaxf(mx, sm.S[r][t]);
    mx = warp_max(mx);
    float s = 0.f;
    for (int t = lane; t < ntok; t += 32) {
      const float e = exp2f(sm.S[r][t] - mx);
      sm.S[r][t] = e;
      s += e;
    }
    s = warp_sum(s);
    if (lane == 0) {
      sm.m[r] = ntok > 0 ? mx : -INFINITY;
      sm.l[r] = s;
    }
  }
  __syncthreads();

  // ---- 2c. P V: thread = (4 columns cq, rows rr and rr + 8) --------------------------------
  constexpr int NQ = D / 4;               // column quads: 32 (D = 128) or 16 (D = 64)
  constexpr int RPT = kThreadsR / NQ;     // row slots per pass: 8 or 16
  const int cq = tid % NQ, rr = tid / NQ;
  float o[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll 4
  for (int t = 0; t < ntok; ++t) {
    const uint2 vv = *reinterpret_cast<const uint2*>(&sm.V[t][cq * 4]);
    float vf[4];
    unpack_bf16x2(vv.x, vf[0], vf[1]);
    unpack_bf16x2(vv.y, vf[2], vf[3]);
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int r = rr + RPT * j;
      if (r < R) {
        const float pr = sm.S[r][t];
#pragma unroll
        for (int e = 0; e < 4; ++e) o[j][e] = fmaf(pr, vf[e], o[j][e]);
      }
    }
  }

  auto store_out = [&](int r, const float* v4, float scale) {  // O row r, columns cq * 4 ..
    const int l = r / p.G, h = g * p.G + r % p.G;
    __nv_bfloat16* dst = p.O + (((size_t)l * p.B + b) * p.Hq + h) * D + cq * 4;
    *reinterpret_cast<uint2*>(dst) = make_uint2(pack_bf16x2(v4[0] * scale, v4[1] * scale),
                                                pack_bf16x2(v4[2] * scale, v4[3] * scale));
  };
  auto store_lse = [&](int r, float m2, float s) {
    if (!p.lse) return;
    const int l = r / p.G, h = g * p.G + r % p.G;
    p.lse[((size_t)l * p.B + b) * p.Hq + h] = s > 0.f ? (m2 + log2f(s)) * kLn2R : -INFINITY;
  };

  if (p.nsplit == 1) {  // the CTA holds the whole selection: final rows
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int r = rr + RPT * j;
      if (r < R) store_out(r, o[j], sm.l[r] > 0.f ? 1.f / sm.l[r] : 0.f);
    }
    if (tid < R) store_lse(tid, sm.m[tid], sm.l[tid]);
    return;
  }

  // ---- 3. split partials, then the last CTA of (b, g) merges -------------------------------
  const size_t ub = ((size_t)b * p.Hkv + g) * p.nsplit;  // this (b, g)'s first split
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const int r = rr + RPT * j;
    if (r < R)
      __stcg(reinterpret_cast<float4*>(p.Op + ((ub + split) * R + r) * D + cq * 4),
             make_float4(o[j][0], o[j][1], o[j][2], o[j][3]));
  }
  if (tid < R) {
    __stcg(p.Mp + (ub + split) * R + tid, sm.m[tid]);
    __stcg(p.Lp + (ub + split) * R + tid, sm.l[tid]);
  }
  __threadfence();  // this thread's partial stores are visible at GPU scope ...
  __syncthreads();  // ... for every thread of the CTA before the arrival
  if (tid == 0) {
    const uint32_t prev = atomicAdd(p.counter + (size_t)b * p.Hkv + g, 1u);
    sm.last = prev == (uint32_t)p.nsplit - 1u;
  }
  __syncthreads();
  if (!sm.last) return;
  __threadfence();  // the other splits' partials, published before their arrivals

  // merge weights: M_r = max_s m_s, w_s = 2^(m_s - M_r), den_r = sum_s w_s l_s.  Warp r takes
  // row r: lane s holds splits s and s + 32 (one round trip for every split's max and sum)
  for (int r = warp; r < R; r += kThreadsR / 32) {
    float ms[2], ls[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int s = lane + 32 * j;
      ms[j] = s < p.nsplit ? __ldcg(p.Mp + (ub + s) * R + r) : -INFINITY;
      ls[j] = s < p.nsplit ? __ldcg(p.Lp + (ub + s) * R + r) : 0.f;
    }
    const float M = warp_max(fmaxf(ms[0], ms[1]));
    float den = 0.f;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int s = lane + 32 * j;
      const float wv = M == -INFINITY ? 0.f : exp2f(ms[j] - M);
      if (s < p.nsplit) sm.w[s][r] = wv;
      den = fmaf(wv, ls[j], den);
    }
    den = warp_sum(den);
    if (lane == 0) {
      sm.inv[r] = den > 0.f ? 1.f / den : 0.f;
      store_lse(r, M, den);
    }
  }
  __syncthreads();  // sm.w, sm.inv
  // every output quad: the splits in batches of 16 loads issued together
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const int r = rr + RPT * j;
    if (r >= R) continue;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int s0 = 0; s0 < p.nsplit; s0 += 16) {
      float4 x[16];
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const int s = min(s0 + u, p.nsplit - 1);
        x[u] = __ldcg(reinterpret_cast<const float4*>(p.Op + ((ub + s) * R + r) * D + cq * 4));
      }
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const float wv = s0 + u < p.nsplit ? sm.w[s0 + u][r] : 0.f;
        acc[0] = fmaf(wv, x[u].x, acc[0]);
        acc[1] = fmaf(wv, x[u].y, acc[1]);
        acc[2] = fmaf(wv, x[u].z, acc[2]);
        acc[3] = fmaf(wv, x[u].w, acc[3]);
      }
    }
    o[j][0] = acc[0];
    o[j][1] = acc[1];
    o[j][2] = acc[2];
    o[j][3] = acc[3];
  }
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const int r = rr + RPT * j;
    if (r < R) store_out(r, o[j], sm.inv[r]);
  }
  if (tid == 0) p.counter[(size_t)b * p.Hkv + g] = 0u;  // clean for the next call
}

}  // namespace

bool sparse_attn_rows_plan(const AttnShape& sh, int sm_count, AttnPlan* pl) {
  if (sh.dt != CLSA_BF16 || (sh.d != 64 && sh.d != 128) || sh.Hq % sh.Hkv != 0) return false;
  const int G = sh.Hq / sh.Hkv;
  if (sh.L * G > kMaxRowsR) return false;
  const long long units = (long long)sh.B * sh.Hkv;
  const long long target = 2LL * std::max(sm_count, 1);
  const int ns0 = (int)std::max(1LL, (target + units - 1) / units);
  int chunk = (sh.k + ns0 - 1) / ns0;
  chunk = std::min(kMaxTokR, (chunk + 63) / 64 * 64);
  const int nsplit = (sh.k + chunk - 1) / chunk;
  if (nsplit > kMaxSplitR) return false;
  pl->Lg = sh.L;
  pl->nlg = 1;
  pl->rows = sh.L * G;
  pl->nsplit = nsplit;
  pl->chunk = chunk;
  return true;
}

size_t attn_rows_smem_bytes(int d) {
  return d == 128 ? sizeof(RowsSmem<128>) : sizeof(RowsSmem<64>);
}

cudaError_t launch_sparse_attn_rows(const AttnShape& sh, const AttnPlan& pl, const void* Q, const void* Kc,
                                    const void* Vc, const int32_t* idx, const int32_t* count, float scale_log2,
                                    void* O, float* lse, float* Op, float* Mp, float* Lp, uint32_t* counter,
                                    void* ws_header, cudaStream_t s) {
  RowsParams p{};
  p.Q = static_cast<const __nv_bfloat16*>(Q);
  p.K = static_cast<const __nv_bfloat16*>(Kc);
  p.V = static_cast<const __nv_bfloat16*>(Vc);
  p.count = count;
  p.O = static_cast<__nv_bfloat16*>(O);
  p.lse = lse;
  p.Op = Op;
  p.Mp = Mp;
  p.Lp = Lp;
  p.counter = counter;
  p.ws_header = ws_header;
  if (sh.gather) {
    p.idx = idx;
    p.n_max = sh.n_max;
    p.kv_bstride = sh.kv_bstride;
  } else {
    p.idx = nullptr;
    p.n_max = sh.k;
    p.kv_bstride = sh.k;
  }
  p.B = sh.B;
  p.k = sh.k;
  p.L = sh.L;
  p.Hq = sh.Hq;
  p.Hkv = sh.Hkv;
  p.G = sh.Hq / sh.Hkv;
  p.rows = pl.rows;
  p.nsplit = pl.nsplit;
  p.chunk = pl.chunk;
  p.scale_log2 = scale_log2;
  const dim3 grid(pl.nsplit, sh.Hkv, sh.B);
  const size_t smem = attn_rows_smem_bytes(sh.d);
  cudaError_t e;
  if (sh.d == 128) {
    e = cudaFuncSetAttribute(attn_rows_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess) e = launch_pdl(attn_rows_kernel<128>, grid, dim3(kThreadsR), smem, s, p);
  } else {
    e = cudaFuncSetAttribute(attn_rows_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess) e = launch_pdl(attn_rows_kernel<64>, grid, dim3(kThreadsR), smem, s, p);
  }
  launches_add(1, s);
  return e;
}

}  // namespace clsa
