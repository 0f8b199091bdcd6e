// Prefill chunk: the routing equation and the per-layer equation of the CLSA
// summary (picx.dev, Methodology > Architecture Overview) for T new rows at
// cache positions t = n - T + i, causal (row t scores only tokens j <= t), with
// k_eff = min(k, t + 1).
//
// Stages:
//   1. index scores  I[i, j] = q_idx[i] . k_idx[j]   (dense contraction, bf16
//      tensor cores, fp32 accumulate; tiles wholly above the diagonal skipped)
//   2. per-row exact radix TopK (the decode top-k kernel with causal lengths)
//   3. per-row sparse attention of every layer (the decode attention kernel in
//      gather mode, each row its own sequence over the one shared cache)
#include "common.cuh"
#include "kernels.h"

namespace clsa {

namespace {

constexpr int kTM = 64;   // query rows per CTA
constexpr int kTN = 128;  // keys per CTA

// S tile = Q_idx[64 rows] . K_idx[128 keys]^T with mma.sync m16n8k16; 4 warps x 16 rows.
template <int DI>
__global__ void __launch_bounds__(128) prefill_scores_kernel(const __nv_bfloat16* __restrict__ q_idx,
                                                             const __nv_bfloat16* __restrict__ k_idx, int n,
                                                             int T, float* __restrict__ scores) {
  constexpr int STR = DI + 8;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  __nv_bfloat16* sA = reinterpret_cast<__nv_bfloat16*>(smem_raw);  // [kTM][STR]
  __nv_bfloat16* sB = sA + kTM * STR;                               // [kTN][STR]
  const int j0 = blockIdx.x * kTN;
  const int i0 = blockIdx.y * kTM;
  const int base = n - T;
  // rows i0..i0+63 see keys j <= base + i; skip tiles with every key beyond every row
  if (j0 > base + min(i0 + kTM - 1, T - 1)) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gid = lane >> 2, tig = lane & 3;
  constexpr int VPR = DI * 2 / 16;
  for (int v = threadIdx.x; v < kTM * VPR; v += blockDim.x) {
    const int r = v / VPR, c = v % VPR;
    const int i = i0 + r;
    cp_async_16(sA + r * STR + c * 8, i < T ? q_idx + (size_t)i * DI + c * 8 : q_idx, i < T ? 16 : 0);
  }
  for (int v = threadIdx.x; v < kTN * VPR; v += blockDim.x) {
    const int r = v / VPR, c = v % VPR;
    const int j = j0 + r;
    cp_async_16(sB + r * STR + c * 8, j < n ? k_idx + (size_t)j * DI + c * 8 : k_idx, j < n ? 16 : 0);
  }
  cp_async_commit();
  cp_async_wait<0>();
  __syncthreads();

  float acc[kTN / 8][4];
#pragma unroll
  for (int t = 0; t < kTN / 8; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;
#pragma unroll
  for (int ks = 0; ks < DI / 16; ++ks) {
    uint32_t a[4];
    {
      const int mi = lane >> 3;
      const int row = warp * 16 + (lane & 7) + 8 * (mi & 1);
      const int col = ks * 16 + 8 * (mi >> 1);
      ldmatrix_x4(a[0], a[1], a[2], a[3], sA + row * STR + col);
    }
#pragma unroll
    for (int nt2 = 0; nt2 < kTN / 16; ++nt2) {
      const int mi = lane >> 3;
      const int tok = nt2 * 16 + 8 * (mi >> 1) + (lane & 7);
      const int col = ks * 16 + 8 * (mi & 1);
      uint32_t r0, r1, r2, r3;
      ldmatrix_x4(r0, r1, r2, r3, sB + tok * STR + col);
      mma_bf16_16816(acc[2 * nt2], a, r0, r1);
      mma_bf16_16816(acc[2 * nt2 + 1], a, r2, r3);
    }
  }
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int i = i0 + warp * 16 + gid + 8 * half;
    if (i >= T) continue;
    const int t = base + i;
    float* row = scores + (size_t)i * n;
#pragma unroll
    for (int nt = 0; nt < kTN / 8; ++nt) {
      const int j = j0 + nt * 8 + 2 * tig;
      if (j < n) row[j] = j <= t ? acc[nt][2 * half] : -INFINITY;
      if (j + 1 < n) row[j + 1] = j + 1 <= t ? acc[nt][2 * half + 1] : -INFINITY;
    }
  }
}

struct PrefillLayout {
  size_t scores = 0, topk = 0, attn = 0, total = 0;
};

PrefillLayout prefill_layout(const clsa_prefill_args* a) {
  PrefillLayout l;
  size_t off = 0;
  l.scores = off;
  off += align_up((size_t)a->T * a->n * sizeof(float), 256);
  l.topk = off;
  off += topk_ws_bytes(a->T, a->n, a->k);
  AttnShape sh{a->T, a->k, a->L, a->Hq, a->Hkv, a->d, a->dtype, true, a->n, 0};
  l.attn = off;
  off += attn_ws_bytes(sh);
  l.total = off;
  return l;
}

}  // namespace

size_t prefill_ws_bytes(const clsa_prefill_args* a) {
  if (!a || a->n < 1 || a->T < 1 || a->T > a->n || a->k < 1 || a->Hkv < 1 || a->Hq < 1) return 0;
  return prefill_layout(a).total;
}

clsa_status run_prefill(const clsa_prefill_args* a, void* ws_header, void* ws_body, cudaStream_t s) {
  const PrefillLayout lay = prefill_layout(a);
  char* w = static_cast<char*>(ws_body);
  float* scores = reinterpret_cast<float*>(w + lay.scores);
  dim3 grid((a->n + kTN - 1) / kTN, (a->T + kTM - 1) / kTM);
  const auto* q = static_cast<const __nv_bfloat16*>(a->q_idx);
  const auto* kx = static_cast<const __nv_bfloat16*>(a->k_idx);
  const int smem = (kTM + kTN) * (a->d_idx + 8) * 2;
  if (a->d_idx == 128) {
    cudaFuncSetAttribute(prefill_scores_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    prefill_scores_kernel<128><<<grid, 128, smem, s>>>(q, kx, a->n, a->T, scores);
  } else {
    cudaFuncSetAttribute(prefill_scores_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    prefill_scores_kernel<64><<<grid, 128, smem, s>>>(q, kx, a->n, a->T, scores);
  }
  launches_add(1);
  if (cudaGetLastError() != cudaSuccess) return CLSA_ERR_CUDA;
  cudaError_t e = launch_topk(scores, nullptr, a->T, a->n, a->k, a->idx, a->count, ws_header, w + lay.topk, s,
                              a->n - a->T);
  if (e != cudaSuccess) return CLSA_ERR_CUDA;
  const float scale = a->scale > 0.f ? a->scale : 1.0f / sqrtf((float)a->d);
  AttnShape sh{a->T, a->k, a->L, a->Hq, a->Hkv, a->d, a->dtype, true, a->n, 0};
  e = launch_sparse_attn(sh, a->Q, a->K, a->V, a->idx, a->count, scale, a->O, a->lse, ws_header, w + lay.attn, s);
  return e == cudaSuccess ? CLSA_OK : CLSA_ERR_CUDA;
}

}  // namespace clsa
