// Distillation target of the shared indexer, forward only (picx.dev CLSA summary,
// Methodology > Architecture Overview, multi-layer distillation).  bf16 with d = 128 runs
// the tcgen05 path of distill_tc.cu; this file is the path for the other shapes:
//   Abar_b = 1/(L Hq) sum_{l,h} softmax(Q^(l)[b,h] K[b]^T * scale)   over the len_b rows
//   kl[b]  = KL(Abar_b || softmax(I_b))
// with query head h reading KV head h / G, the attention scale of the layers, and no scale
// on the indexer scores I.
//
// 1. The lse of every (layer, query head) row over the whole cache comes from the dense
//    split-k attention of sparse_attn.cu (the cache as K_S; the output rows are discarded).
// 2. lse_kernel: the lse of each sequence's scores I.
// 3. abar_kernel: one CTA per (64-token tile, sequence).  For every KV head g it stages the
//    tile's K rows (fp32, rows padded to D + 1 words: conflict-free column reads) and the
//    group's query rows 32 at a time; thread (token j, row lane q) sums exp(s scale - lse)
//    over rows q, q + 4, ...; the four row lanes meet in shared memory.  Abar is written
//    for the tile and its KL terms Abar (log Abar - (I - lse_I)) are summed into one
//    partial per tile.
// 4. kl_kernel: each sequence's tile partials in tile order (deterministic).
#include <algorithm>
#include <cmath>

#include "common.cuh"
#include "kernels.h"

namespace clsa {

namespace {

constexpr int kTileTok = 64;
constexpr int kRowLanes = 4;                 // 256 threads = 64 tokens x 4 row lanes
constexpr int kRowBatch = 32;                // query rows staged at once
constexpr int kDistillThreads = kTileTok * kRowLanes;

__device__ __forceinline__ float load_f(const __nv_bfloat16* p) { return __bfloat162float(*p); }
__device__ __forceinline__ float load_f(const float* p) { return *p; }

// lse_I[b] = log sum_{j < len_b} exp(I[b, j])  (-inf for an empty sequence)
__global__ void __launch_bounds__(256) lse_kernel(const float* __restrict__ scores, const int32_t* __restrict__ lens,
                                                  int n_max, float* __restrict__ lse_I) {
  __shared__ float red[8];
  const int b = blockIdx.x;
  const int n = max(0, min(lens[b], n_max));
  const float* I = scores + (size_t)b * n_max;
  float m = -INFINITY;
  for (int j = threadIdx.x; j < n; j += 256) m = fmaxf(m, I[j]);
  m = warp_max(m);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  m = red[0];
#pragma unroll
  for (int w = 1; w < 8; ++w) m = fmaxf(m, red[w]);
  __syncthreads();
  float s = 0.f;
  if (m != -INFINITY)
    for (int j = threadIdx.x; j < n; j += 256) s += expf(I[j] - m);
  s = warp_sum(s);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = 0.f;
    for (int w = 0; w < 8; ++w) t += red[w];
    lse_I[b] = t > 0.f ? m + logf(t) : -INFINITY;
  }
}

struct DistillParams {
  const void* Q;        // [L][B][Hq][d]
  const void* K;        // [B][n_max][Hkv][d]
  const float* scores;  // [B][n_max]
  const int32_t* lens;  // [B]
  const float* lse_row; // [L][B][Hq] natural-log lse of the scaled scores of every row
  const float* lse_I;   // [B]
  float* abar;          // [B][n_max] or null
  float* partial;       // [B][ntiles]
  int B, n_max, L, Hq, Hkv, G, ntiles;
  float scale;
};

template <typename T, int D>
__global__ void __launch_bounds__(kDistillThreads) abar_kernel(const DistillParams p) {
  extern __shared__ float sm[];
  float* sK = sm;                                  // [kTileTok][D + 1]
  float* sQ = sK + kTileTok * (D + 1);             // [kRowBatch][D]
  float* sL = sQ + kRowBatch * D;                  // [kRowBatch] row lse
  float* sCol = sL + kRowBatch;                    // [kRowLanes][kTileTok] column sums
  float* sRed = sCol + kRowLanes * kTileTok;       // [8] block reduction
  const int tile = blockIdx.x, b = blockIdx.y;
  const int j0 = tile * kTileTok;
  const int n = max(0, min(p.lens[b], p.n_max));
  const int tj = threadIdx.x % kTileTok, rq = threadIdx.x / kTileTok;
  const T* Q = static_cast<const T*>(p.Q);
  const T* K = static_cast<const T*>(p.K);
  const int rows = p.L * p.G;  // rows of one KV head group
  float col = 0.f;             // this thread's share of column tj
  if (j0 < n) {
#pragma unroll 1
    for (int g = 0; g < p.Hkv; ++g) {
      __syncthreads();  // the previous group's tiles are read
      for (int v = threadIdx.x; v < kTileTok * D; v += kDistillThreads) {
        const int r = v / D, c = v % D;
        const int j = j0 + r;
        sK[r * (D + 1) + c] = j < n ? load_f(K + (((size_t)b * p.n_max + j) * p.Hkv + g) * D + c) : 0.f;
      }
#pragma unroll 1
      for (int r0 = 0; r0 < rows; r0 += kRowBatch) {
        __syncthreads();  // sK visible; the previous row batch is read
        for (int v = threadIdx.x; v < kRowBatch * D; v += kDistillThreads) {
          const int r = v / D, c = v % D;
          const int rr = r0 + r;
          float x = 0.f;
          if (rr < rows) {
            const int l = rr / p.G, h = g * p.G + rr % p.G;
            x = load_f(Q + (((size_t)l * p.B + b) * p.Hq + h) * D + c);
          }
          sQ[r * D + c] = x;
        }
        if (threadIdx.x < kRowBatch) {
          const int rr = r0 + threadIdx.x;
          float lse = INFINITY;  // a missing row contributes exp(-inf) = 0
          if (rr < rows) {
            const int l = rr / p.G, h = g * p.G + rr % p.G;
            lse = p.lse_row[((size_t)l * p.B + b) * p.Hq + h];
          }
          sL[threadIdx.x] = lse;
        }
        __syncthreads();
        if (j0 + tj < n) {
          const float* kr = sK + tj * (D + 1);
#pragma unroll 1
          for (int r = rq; r < kRowBatch; r += kRowLanes) {
            const float* qr = sQ + r * D;
            float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
#pragma unroll 8
            for (int c = 0; c < D; c += 4) {
              s0 = fmaf(qr[c], kr[c], s0);
              s1 = fmaf(qr[c + 1], kr[c + 1], s1);
              s2 = fmaf(qr[c + 2], kr[c + 2], s2);
              s3 = fmaf(qr[c + 3], kr[c + 3], s3);
            }
            col += expf(((s0 + s1) + (s2 + s3)) * p.scale - sL[r]);
          }
        }
      }
    }
  }
  sCol[rq * kTileTok + tj] = col;
  __syncthreads();
  float kl_term = 0.f;
  if (threadIdx.x < kTileTok) {
    const int j = j0 + threadIdx.x;
    float a = 0.f;
    if (j < n) {
      a = ((sCol[threadIdx.x] + sCol[kTileTok + threadIdx.x]) +
           (sCol[2 * kTileTok + threadIdx.x] + sCol[3 * kTileTok + threadIdx.x])) /
          (float)(p.L * p.Hq);
      if (a > 0.f) kl_term = a * (logf(a) - (p.scores[(size_t)b * p.n_max + j] - p.lse_I[b]));
    }
    if (p.abar && j < p.n_max) p.abar[(size_t)b * p.n_max + j] = a;
  }
  // tile partial (threads 64.. hold 0)
  kl_term = warp_sum(kl_term);
  if ((threadIdx.x & 31) == 0) sRed[threadIdx.x >> 5] = kl_term;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = 0.f;
    for (int w = 0; w < kDistillThreads / 32; ++w) t += sRed[w];
    p.partial[(size_t)b * p.ntiles + tile] = t;
  }
}

// kl[b] = sum of the tile partials in tile order (one warp per sequence)
__global__ void __launch_bounds__(32) kl_kernel(const float* __restrict__ partial, int ntiles,
                                                float* __restrict__ kl) {
  const int b = blockIdx.x;
  float s = 0.f;
  for (int t = threadIdx.x; t < ntiles; t += 32) s += partial[(size_t)b * ntiles + t];
  s = warp_sum(s);
  if (threadIdx.x == 0) kl[b] = s;
}

size_t dsmem_bytes(int D) {
  return (size_t)(kTileTok * (D + 1) + kRowBatch * D + kRowBatch + kRowLanes * kTileTok + 8) * sizeof(float);
}

}  // namespace

size_t distill_ws_bytes(int B, int n_max, int L, int Hq, int Hkv, int d, clsa_dtype dt) {
  const int ntiles = (n_max + kTileTok - 1) / kTileTok;
  AttnShape sh{B, n_max, L, Hq, Hkv, d, dt, false, n_max, 0};
  size_t off = 0;
  off += align_up((size_t)L * B * Hq * d * (dt == CLSA_BF16 ? 2 : 4), 256);  // discarded attention output
  off += align_up((size_t)L * B * Hq * 4, 256);                              // row lse
  off += align_up((size_t)B * 4, 256);                                       // lse of I
  off += align_up((size_t)B * ntiles * 4, 256);                              // tile partials
  off += attn_ws_bytes(sh);
  if (distill_tc_supported(B, n_max, L, Hq, Hkv, d, dt)) off = std::max(off, distill_tc_ws_bytes(B, n_max, L, Hq, Hkv));
  return off;
}

cudaError_t launch_distill(const void* Q, const void* K, const float* scores, const int32_t* lens, int B, int n_max,
                           int L, int Hq, int Hkv, int d, float scale, clsa_dtype dt, float* abar, float* kl,
                           void* ws_header, void* ws, cudaStream_t s) {
  if (distill_tc_supported(B, n_max, L, Hq, Hkv, d, dt))
    return launch_distill_tc(Q, K, scores, lens, B, n_max, L, Hq, Hkv, scale, abar, kl, ws_header, ws, s);
  const int ntiles = (n_max + kTileTok - 1) / kTileTok;
  char* w = static_cast<char*>(ws);
  void* O = w;
  w += align_up((size_t)L * B * Hq * d * (dt == CLSA_BF16 ? 2 : 4), 256);
  float* lse_row = reinterpret_cast<float*>(w);
  w += align_up((size_t)L * B * Hq * 4, 256);
  float* lse_I = reinterpret_cast<float*>(w);
  w += align_up((size_t)B * 4, 256);
  float* partial = reinterpret_cast<float*>(w);
  w += align_up((size_t)B * ntiles * 4, 256);
  // 1. row lse: dense attention over each sequence's cache (K stands in for V: lse does not use V)
  AttnShape sh{B, n_max, L, Hq, Hkv, d, dt, false, n_max, 0};
  cudaError_t e = launch_sparse_attn(sh, Q, K, K, nullptr, lens, scale, O, lse_row, ws_header, w, s);
  if (e != cudaSuccess) return e;
  // 2. lse of the scores
  lse_kernel<<<B, 256, 0, s>>>(scores, lens, n_max, lse_I);
  launches_add(1, s);
  // 3. Abar and the tile partials of the KL
  DistillParams p{Q, K, scores, lens, lse_row, lse_I, abar, partial, B, n_max, L, Hq, Hkv, Hq / Hkv, ntiles, scale};
  const dim3 grid(ntiles, B);
  const size_t smem = dsmem_bytes(d);
#define CLSA_DISTILL(T, D)                                                                            \
  do {                                                                                                \
    e = cudaFuncSetAttribute(abar_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem); \
    if (e == cudaSuccess) abar_kernel<T, D><<<grid, kDistillThreads, smem, s>>>(p);                    \
  } while (0)
  if (dt == CLSA_BF16) {
    if (d == 128) CLSA_DISTILL(__nv_bfloat16, 128);
    else CLSA_DISTILL(__nv_bfloat16, 64);
  } else {
    if (d == 128) CLSA_DISTILL(float, 128);
    else CLSA_DISTILL(float, 64);
  }
#undef CLSA_DISTILL
  launches_add(1, s);
  if (e != cudaSuccess) return e;
  // 4. per-sequence KL
  kl_kernel<<<B, 32, 0, s>>>(partial, ntiles, kl);
  launches_add(1, s);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Attention-mass coverage for the shapes the tensor-core pass does not take (fp32, d = 64):
// the row lse over each sequence's cache from the split-k attention kernel (K stands in for
// V: the lse does not use V; the output is discarded), then mass = exp(lse_S - lse_all).
// ---------------------------------------------------------------------------
namespace {
__global__ void mass_from_lse_kernel(const float* __restrict__ lse_sparse, const float* __restrict__ lse_all, int n,
                                     float* __restrict__ mass) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const float ls = lse_sparse[i], la = lse_all[i];
  mass[i] = (la == -INFINITY || ls == -INFINITY) ? 0.f : expf(ls - la);
}
}  // namespace

size_t attention_mass_ws_bytes(int B, int n_max, int L, int Hq, int Hkv, int d, clsa_dtype dt) {
  if (distill_tc_supported(B, n_max, L, Hq, Hkv, d, dt)) return attention_mass_tc_ws_bytes(B, n_max, L, Hq, Hkv);
  AttnShape sh{B, n_max, L, Hq, Hkv, d, dt, false, n_max, 0};
  size_t off = 0;
  off += align_up((size_t)L * B * Hq * d * (dt == CLSA_BF16 ? 2 : 4), 256);  // discarded attention output
  off += align_up((size_t)L * B * Hq * 4, 256);                              // row lse
  off += attn_ws_bytes(sh);
  return off;
}

cudaError_t launch_attention_mass(const void* Q, const void* K, const float* lse_sparse, const int32_t* lens, int B,
                                  int n_max, int L, int Hq, int Hkv, int d, float scale, clsa_dtype dt, float* mass,
                                  float* lse_all, void* ws_header, void* ws, cudaStream_t s) {
  if (distill_tc_supported(B, n_max, L, Hq, Hkv, d, dt))
    return launch_attention_mass_tc(Q, K, lse_sparse, lens, B, n_max, L, Hq, Hkv, scale, mass, lse_all, ws_header, ws, s);
  char* w = static_cast<char*>(ws);
  void* O = w;
  w += align_up((size_t)L * B * Hq * d * (dt == CLSA_BF16 ? 2 : 4), 256);
  float* lse_row = lse_all ? lse_all : reinterpret_cast<float*>(w);
  w += align_up((size_t)L * B * Hq * 4, 256);
  AttnShape sh{B, n_max, L, Hq, Hkv, d, dt, false, n_max, 0};
  cudaError_t e = launch_sparse_attn(sh, Q, K, K, nullptr, lens, scale, O, lse_row, ws_header, w, s);
  if (e != cudaSuccess) return e;
  const int n = L * B * Hq;
  mass_from_lse_kernel<<<(n + 255) / 256, 256, 0, s>>>(lse_sparse, lse_row, n, mass);
  launches_add(1, s);
  return cudaGetLastError();
}

}  // namespace clsa
