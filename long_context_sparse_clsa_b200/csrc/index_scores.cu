// Indexer scan: I[b, j] = q_idx[b] . k_idx[b, j]
// (routing equation of the picx.dev CLSA summary, Methodology > Architecture
// Overview; single indexer head, bare product).
//
// HBM-bound GEMV.  Each K_idx row (d_idx * elem bytes = 128..512 B) is read by a
// group of LPR lanes with 16-byte non-allocating loads; every thread keeps its
// 16-byte slice of q in registers, multiplies exactly (bf16 products fit fp32),
// accumulates in fp32 and the group reduces with shuffles.  UNROLL independent
// row loads per thread are issued before any arithmetic so that enough bytes
// are in flight per SM to cover HBM latency.
#include "common.cuh"
#include "kernels.h"

namespace clsa {

namespace {

template <typename T, int DIDX, int UNROLL>
__global__ void __launch_bounds__(256) index_scores_kernel(const T* __restrict__ q_idx,
                                                           const T* __restrict__ k_idx,
                                                           const int32_t* __restrict__ seq_lens,
                                                           int n_max, float* __restrict__ scores) {
  constexpr int EPT = 16 / sizeof(T);  // elements per 16-byte load
  constexpr int LPR = DIDX / EPT;      // lanes per row
  constexpr int RPW = 32 / LPR;        // rows per warp per load
  static_assert(LPR <= 32 && 32 % LPR == 0, "row must fit a warp");

  const int b = blockIdx.y;
  const int len = max(0, min(seq_lens[b], n_max));
  const int lane = threadIdx.x & 31;
  const int sub = lane % LPR;
  const int rsub = lane / LPR;

  float q[EPT];
  {
    const uint4 qv = *reinterpret_cast<const uint4*>(q_idx + (size_t)b * DIDX + sub * EPT);
    if constexpr (sizeof(T) == 2) {
      unpack_bf16x2(qv.x, q[0], q[1]);
      unpack_bf16x2(qv.y, q[2], q[3]);
      unpack_bf16x2(qv.z, q[4], q[5]);
      unpack_bf16x2(qv.w, q[6], q[7]);
    } else {
      q[0] = __uint_as_float(qv.x);
      q[1] = __uint_as_float(qv.y);
      q[2] = __uint_as_float(qv.z);
      q[3] = __uint_as_float(qv.w);
    }
  }

  const T* kb = k_idx + (size_t)b * n_max * DIDX;
  float* sb = scores + (size_t)b * n_max;
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int nwarps = (gridDim.x * blockDim.x) >> 5;
  constexpr int STEP = RPW * UNROLL;

  for (int base = warp * STEP; base < n_max; base += nwarps * STEP) {
    uint4 v[UNROLL];
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      const int j = base + u * RPW + rsub;
      if (j < len) v[u] = ld_stream_v4(kb + (size_t)j * DIDX + sub * EPT);
      else v[u] = make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      const int j = base + u * RPW + rsub;
      float acc;
      if constexpr (sizeof(T) == 2) {
        float a0, a1, a2, a3, a4, a5, a6, a7;
        unpack_bf16x2(v[u].x, a0, a1);
        unpack_bf16x2(v[u].y, a2, a3);
        unpack_bf16x2(v[u].z, a4, a5);
        unpack_bf16x2(v[u].w, a6, a7);
        acc = q[0] * a0;
        acc = fmaf(q[1], a1, acc);
        acc = fmaf(q[2], a2, acc);
        acc = fmaf(q[3], a3, acc);
        acc = fmaf(q[4], a4, acc);
        acc = fmaf(q[5], a5, acc);
        acc = fmaf(q[6], a6, acc);
        acc = fmaf(q[7], a7, acc);
      } else {
        acc = q[0] * __uint_as_float(v[u].x);
        acc = fmaf(q[1], __uint_as_float(v[u].y), acc);
        acc = fmaf(q[2], __uint_as_float(v[u].z), acc);
        acc = fmaf(q[3], __uint_as_float(v[u].w), acc);
      }
#pragma unroll
      for (int o = LPR / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      if (sub == 0 && j < n_max) sb[j] = (j < len) ? acc : -INFINITY;
    }
  }
}

template <typename T, int DIDX>
cudaError_t launch_t(const void* q, const void* kx, const int32_t* lens, int B, int n_max, float* scores,
                     cudaStream_t s) {
  constexpr int UNROLL = 8;
  constexpr int EPT = 16 / sizeof(T);
  constexpr int RPW = 32 / (DIDX / EPT);
  const int rows_per_cta = 8 * RPW * UNROLL;  // 8 warps per CTA
  const int want = device_info().sm_count * 4;  // ~4 CTAs per SM in total
  int gx = (n_max + rows_per_cta - 1) / rows_per_cta;
  const int cap = (want + B - 1) / B;
  if (gx > cap) gx = cap;
  if (gx < 1) gx = 1;
  dim3 grid(gx, B);
  index_scores_kernel<T, DIDX, UNROLL><<<grid, 256, 0, s>>>(
      static_cast<const T*>(q), static_cast<const T*>(kx), lens, n_max, scores);
  launches_add(1, s);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_index_scores(const void* q_idx, const void* k_idx, const int32_t* seq_lens, int B,
                                int n_max, int d_idx, clsa_dtype dt, float* scores, cudaStream_t s) {
  if (dt == CLSA_BF16) {
    if (d_idx == 128) return launch_t<__nv_bfloat16, 128>(q_idx, k_idx, seq_lens, B, n_max, scores, s);
    return launch_t<__nv_bfloat16, 64>(q_idx, k_idx, seq_lens, B, n_max, scores, s);
  }
  if (d_idx == 128) return launch_t<float, 128>(q_idx, k_idx, seq_lens, B, n_max, scores, s);
  return launch_t<float, 64>(q_idx, k_idx, seq_lens, B, n_max, scores, s);
}

}  // namespace clsa
