// Indexer scan: I[b, j] = q_idx[b] . k_idx[b, j]
// (routing equation of the picx.dev CLSA summary, Methodology > Architecture
// Overview; single indexer head, bare product).
//
// HBM-bound GEMV.  K_idx streams through shared memory in 16 KiB tiles of whole rows
// (one 1-D bulk copy each, completing on an mbarrier), kStages tiles in flight per CTA
// and two CTAs per SM: 128 KiB requested per SM at any time, enough to cover HBM latency
// with one issuing thread.  In a tile, each row (d_idx * elem bytes = 128..512 B) is read
// by a group of LPR lanes, 16 bytes each; every thread keeps its 16-byte slice of q in
// registers, multiplies exactly (bf16 products fit fp32), accumulates in fp32 and the
// group reduces with shuffles.  The CTAs of a sequence take its tiles round-robin.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace clsa {

namespace {

constexpr int kThr = 256;
constexpr int kTileBytes = 16384;  // one bulk copy: 64 bf16 rows of d_idx = 128
constexpr int kStages = 4;         // tiles in flight per CTA

template <typename T, int DIDX>
__global__ void __launch_bounds__(kThr) index_scores_kernel(const T* __restrict__ q_idx, const T* __restrict__ k_idx,
                                                            const int32_t* __restrict__ seq_lens, int n_max,
                                                            float* __restrict__ scores, void* ws_header) {
  constexpr int kRowBytes = DIDX * (int)sizeof(T);
  constexpr int kTile = kTileBytes / kRowBytes;  // rows per tile
  constexpr int EPT = 16 / sizeof(T);            // elements per 16-byte chunk
  constexpr int LPR = DIDX / EPT;                // lanes per row
  constexpr int RPP = kThr / LPR;                // rows per pass over a tile
  static_assert(LPR <= 32 && 32 % LPR == 0 && kTile % RPP == 0, "row must fit a warp");
  extern __shared__ __align__(128) unsigned char ring[];  // [kStages][kTileBytes]
  __shared__ uint64_t full[kStages];

  const int b = blockIdx.y;
  const int len = max(0, min(seq_lens[b], n_max));
  const int sub = threadIdx.x % LPR;
  const int rsub = threadIdx.x / LPR;
  const T* kb = k_idx + (size_t)b * n_max * DIDX;
  float* sb = scores + (size_t)b * n_max;
  // this CTA's tiles: blockIdx.x, + gridDim.x, ...; the first nload of them hold rows < len
  const int ntiles = (n_max + kTile - 1) / kTile;
  const int first = blockIdx.x, step = gridDim.x;
  const int nmine = first < ntiles ? (ntiles - 1 - first) / step + 1 : 0;
  const int tiles_len = (len + kTile - 1) / kTile;
  const int nload = first < tiles_len ? (tiles_len - 1 - first) / step + 1 : 0;
  auto issue = [&](int j) {  // my j-th tile into stage j % kStages
    const int r0 = (first + j * step) * kTile;
    const int nr = min(len - r0, kTile);
    uint64_t* bar = &full[j % kStages];
    mbar_arrive_expect_tx(bar, (uint32_t)(nr * kRowBytes));
    bulk_g2s(ring + (j % kStages) * kTileBytes, kb + (size_t)r0 * DIDX, (uint32_t)(nr * kRowBytes), bar);
  };
  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) mbar_init(&full[i], 1);
    fence_mbar_init();
    for (int j = 0; j < min(kStages, nload); ++j) issue(j);
  }
  // this thread's 16-byte slice of q, exact in fp32
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
  __syncthreads();  // barriers initialised

  for (int j = 0; j < nload; ++j) {
    const int r0 = (first + j * step) * kTile;
    const int nr = min(len - r0, kTile);
    if (!mbar_wait(&full[j % kStages], (uint32_t)(j / kStages) & 1u)) {
      if (ws_header) record_error(ws_header, CLSA_ERR_TIMEOUT, 60);
      return;
    }
    const unsigned char* tile = ring + (j % kStages) * kTileBytes;
#pragma unroll 4
    for (int p = 0; p < kTile / RPP; ++p) {
      const int r = p * RPP + rsub;
      const uint4 v = *reinterpret_cast<const uint4*>(tile + r * kRowBytes + sub * 16);
      float acc;
      if constexpr (sizeof(T) == 2) {
        float a0, a1, a2, a3, a4, a5, a6, a7;
        unpack_bf16x2(v.x, a0, a1);
        unpack_bf16x2(v.y, a2, a3);
        unpack_bf16x2(v.z, a4, a5);
        unpack_bf16x2(v.w, a6, a7);
        acc = q[0] * a0;
        acc = fmaf(q[1], a1, acc);
        acc = fmaf(q[2], a2, acc);
        acc = fmaf(q[3], a3, acc);
        acc = fmaf(q[4], a4, acc);
        acc = fmaf(q[5], a5, acc);
        acc = fmaf(q[6], a6, acc);
        acc = fmaf(q[7], a7, acc);
      } else {
        acc = q[0] * __uint_as_float(v.x);
        acc = fmaf(q[1], __uint_as_float(v.y), acc);
        acc = fmaf(q[2], __uint_as_float(v.z), acc);
        acc = fmaf(q[3], __uint_as_float(v.w), acc);
      }
#pragma unroll
      for (int o = LPR / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      // rows of the tile past len (the tile that straddles it) read stale bytes: -inf
      if (sub == 0 && r0 + r < n_max) sb[r0 + r] = r < nr ? acc : -INFINITY;
    }
    __syncthreads();  // every thread is done with this stage
    if (threadIdx.x == 0 && j + kStages < nload) issue(j + kStages);
  }
  // tiles wholly past len: -inf
  for (int j = nload; j < nmine; ++j) {
    const int r0 = (first + j * step) * kTile;
    for (int r = threadIdx.x; r < kTile && r0 + r < n_max; r += kThr) sb[r0 + r] = -INFINITY;
  }
}

template <typename T, int DIDX>
cudaError_t launch_t(const void* q, const void* kx, const int32_t* lens, int B, int n_max, float* scores,
                     void* ws_header, cudaStream_t s) {
  constexpr int kTile = kTileBytes / (DIDX * (int)sizeof(T));
  const int ntiles = (n_max + kTile - 1) / kTile;
  const int want = device_info().sm_count * 2;  // two CTAs (2 x 64 KiB in flight) per SM
  int gx = std::min(ntiles, std::max(1, (want + B - 1) / B));
  dim3 grid(gx, B);
  const int smem = kStages * kTileBytes;
  cudaError_t e = cudaFuncSetAttribute(index_scores_kernel<T, DIDX>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  index_scores_kernel<T, DIDX><<<grid, kThr, smem, s>>>(static_cast<const T*>(q), static_cast<const T*>(kx), lens,
                                                         n_max, scores, ws_header);
  launches_add(1, s);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_index_scores(const void* q_idx, const void* k_idx, const int32_t* seq_lens, int B,
                                int n_max, int d_idx, clsa_dtype dt, float* scores, void* ws_header, cudaStream_t s) {
  if (dt == CLSA_BF16) {
    if (d_idx == 128) return launch_t<__nv_bfloat16, 128>(q_idx, k_idx, seq_lens, B, n_max, scores, ws_header, s);
    return launch_t<__nv_bfloat16, 64>(q_idx, k_idx, seq_lens, B, n_max, scores, ws_header, s);
  }
  if (d_idx == 128) return launch_t<float, 128>(q_idx, k_idx, seq_lens, B, n_max, scores, ws_header, s);
  return launch_t<float, 64>(q_idx, k_idx, seq_lens, B, n_max, scores, ws_header, s);
}

}  // namespace clsa
