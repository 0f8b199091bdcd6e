// Prefill chunk: the routing equation and the per-layer equation of the CLSA
// summary (picx.dev, Methodology > Architecture Overview) for T new rows at
// cache positions t = n - T + i, causal (row t scores only tokens j <= t), with
// k_eff = min(k, t + 1).
//
// Stages:
//   1. index scores  I[i, j] = q_idx[i] . k_idx[j]   (dense contraction on the
//      tcgen05 tensor cores, fp32 accumulate in TMEM; tiles wholly above the diagonal
//      skipped)
//   2. per-row exact radix TopK (the decode top-k kernel with causal lengths)
//   3. per-row sparse attention of every layer (the decode attention kernel in
//      gather mode, each row its own sequence over the one shared cache)
#include <algorithm>

#include "common.cuh"
#include "kernels.h"
#include "tcgen05.cuh"

namespace clsa {

namespace {

constexpr int kTcM = 128;  // query rows per tile (TMEM lanes)
constexpr int kTcN = 256;  // keys per tile (TMEM columns, fp32)

// Score tiles I[i0:i0+128, j0:j0+256] = Q_idx[rows] . K_idx[keys]^T on the 5th-generation
// tensor cores.  Operands are staged with 16-byte cp.async into 128B-swizzled K-major
// tiles; one thread issues DI/16 tcgen05.mma (M=128, N=256, K=16, bf16 -> fp32) into a
// 256-column TMEM accumulator and commits to an mbarrier; the four warps read their 32
// TMEM lanes (one query row per thread), apply the causal mask and store the row.
// Tiles whose keys all lie beyond every row's position are skipped.  Persistent: each
// CTA walks tiles blockIdx.x, blockIdx.x + gridDim.x, ...
template <int DI>
__global__ void __launch_bounds__(128) prefill_scores_tc_kernel(const __nv_bfloat16* __restrict__ q_idx,
                                                                const __nv_bfloat16* __restrict__ k_idx, int n,
                                                                int T, float* __restrict__ scores,
                                                                void* ws_header,
                                                                const int32_t* __restrict__ only_rows,
                                                                const uint32_t* __restrict__ any_flag) {
  constexpr int KAT = DI / 64;                 // 128-byte K atoms
  constexpr uint32_t A_ATOM = kTcM * 128;      // bytes of one K atom of the A tile
  constexpr uint32_t B_ATOM = kTcN * 128;
  constexpr int CPR = DI / 8;                  // 16-byte chunks per row
  extern __shared__ __align__(1024) unsigned char smem[];
  unsigned char* sA = smem;
  unsigned char* sB = smem + KAT * A_ATOM;
  __shared__ uint64_t mbar;
  __shared__ uint32_t tmem_base;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (any_flag && *any_flag == 0u) return;  // fallback use: nothing to recompute
  if (warp == 0) {
    tc::tmem_alloc(&tmem_base, kTcN);
    tc::tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(&mbar, 1);
    fence_mbar_init();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = tmem_base;
  const int base = n - T;
  const int nqb = (T + kTcM - 1) / kTcM, nkt = (n + kTcN - 1) / kTcN;
  constexpr uint32_t idesc = tc::idesc_bf16_f32(kTcM, kTcN);
  uint32_t phase = 0;
  for (int item = blockIdx.x; item < nqb * nkt; item += gridDim.x) {
    const int qb = item / nkt, kt = item % nkt;
    const int i0 = qb * kTcM, j0 = kt * kTcN;
    if (j0 > base + min(i0 + kTcM - 1, T - 1)) continue;  // every key beyond every row
    if (only_rows) {  // fallback use: only row blocks holding a flagged row
      const int r = i0 + tid;
      if (!__syncthreads_or(r < T && only_rows[r] != 0)) continue;
    }
    for (int v = tid; v < kTcM * CPR; v += 128) {
      const int r = v / CPR, c = v % CPR;
      const bool in = i0 + r < T;
      cp_async_16(sA + (c >> 3) * A_ATOM + tc::sw128_offset(r, c & 7),
                  in ? q_idx + (size_t)(i0 + r) * DI + c * 8 : q_idx, in ? 16 : 0);
    }
    for (int v = tid; v < kTcN * CPR; v += 128) {
      const int r = v / CPR, c = v % CPR;
      const bool in = j0 + r < n;
      cp_async_16(sB + (c >> 3) * B_ATOM + tc::sw128_offset(r, c & 7),
                  in ? k_idx + (size_t)(j0 + r) * DI + c * 8 : k_idx, in ? 16 : 0);
    }
    cp_async_commit();
    cp_async_wait<0>();
    fence_proxy_async_smem();  // generic-proxy writes -> visible to the tensor core's reads
    __syncthreads();
    tc::fence_after_sync();
    if (tid == 0) {
#pragma unroll
      for (int ks = 0; ks < DI / 16; ++ks) {
        const uint32_t koff = (uint32_t)(ks & 3) * 32u;
        const uint64_t a = tc::sw128_desc(smem_u32(sA) + (ks >> 2) * A_ATOM + koff);
        const uint64_t b = tc::sw128_desc(smem_u32(sB) + (ks >> 2) * B_ATOM + koff);
        tc::mma_bf16(tmem, a, b, idesc, ks > 0);
      }
      tc::mma_commit(&mbar);
    }
    const bool ok = __syncthreads_and(mbar_wait(&mbar, phase));
    phase ^= 1u;
    if (!ok) {
      if (tid == 0) record_error(ws_header, CLSA_ERR_TIMEOUT, 300);
      break;
    }
    tc::fence_after_sync();
    // Epilogue: each thread pulls its row's next 32 columns from TMEM (its lane) and
    // parks them in the free B tile; then each warp writes its 32 rows as 128-byte
    // row segments (lane = column), causal mask applied on the way out.
    float* stage = reinterpret_cast<float*>(sB) + warp * 32 * 33;  // [32 rows][33] per warp
#pragma unroll 1
    for (int cb = 0; cb < kTcN; cb += 32) {
      uint32_t v[32];
      tc::ld_32x32b_x32(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)cb, v);
      tc::ld_wait();
#pragma unroll
      for (int q = 0; q < 32; ++q) stage[lane * 33 + q] = __uint_as_float(v[q]);
      __syncwarp();
      const int j = j0 + cb + lane;
#pragma unroll 4
      for (int rr = 0; rr < 32; ++rr) {
        const int i = i0 + warp * 32 + rr;
        if (i < T && j < n) scores[(size_t)i * n + j] = j <= base + i ? stage[rr * 33 + lane] : -INFINITY;
      }
      __syncwarp();
    }
    tc::fence_before_sync();
    __syncthreads();  // TMEM and the operand tiles are reused by the next tile
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tmem, kTcN);
}

struct PrefillLayout {
  bool route = false;
  size_t scores = 0, topk = 0, attn = 0, route_ws = 0, total = 0;
};

PrefillLayout prefill_layout(const clsa_prefill_args* a) {
  PrefillLayout l;
  l.route = prefill_route_supported(a);
  size_t off = 0;
  l.scores = off;  // fp32 scores of the exact path (the fallback when routing is on)
  off += align_up((size_t)a->T * a->n * sizeof(float), 256);
  l.topk = off;  // shared by the top-k over score rows and over dense candidate rows
  off += std::max(topk_ws_bytes(a->T, a->n, a->k),
                  l.route ? topk_ws_bytes(a->T, prefill_route_ldd(a), a->k) : (size_t)0);
  AttnShape sh{a->T, a->k, a->L, a->Hq, a->Hkv, a->d, a->dtype, true, a->n, 0};
  l.attn = off;
  off += attn_ws_bytes(sh);
  if (l.route) {
    l.route_ws = off;
    off += prefill_route_ws_bytes(a);
  }
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
  const int nsm = std::max(1, device_info().sm_count);
  const auto* q = static_cast<const __nv_bfloat16*>(a->q_idx);
  const auto* kx = static_cast<const __nv_bfloat16*>(a->k_idx);
  // Each CTA holds 256 TMEM columns of the SM's 512, so at most two may share an SM: the
  // d_idx = 64 tiles (49 KB) are padded to 80 KB of shared memory, which lets no third
  // CTA in (a third would wait in tcgen05.alloc until one of the two finished).
  const int smem = std::max((a->d_idx / 64) * (kTcM + kTcN) * 128, 80 * 1024);
  auto scores_kernel = [&](const int32_t* only_rows, const uint32_t* any_flag) {
    if (a->d_idx == 128) {
      cudaFuncSetAttribute(prefill_scores_tc_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      prefill_scores_tc_kernel<128><<<2 * nsm, 128, smem, s>>>(q, kx, a->n, a->T, scores, ws_header, only_rows,
                                                                 any_flag);
    } else {
      cudaFuncSetAttribute(prefill_scores_tc_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      prefill_scores_tc_kernel<64><<<2 * nsm, 128, smem, s>>>(q, kx, a->n, a->T, scores, ws_header, only_rows,
                                                                any_flag);
    }
    launches_add(1, s);
    return cudaGetLastError();
  };
  cudaError_t e;
  if (lay.route) {
    // routing from on-chip candidates, then the exact path for any flagged row
    PrefillRouteBufs rb{};
    e = launch_prefill_route(a, ws_header, w + lay.route_ws, s, &rb);
    if (e != cudaSuccess) return CLSA_ERR_CUDA;
    e = launch_topk(reinterpret_cast<const float*>(rb.dval), rb.dlen, a->T, rb.ldd, a->k, a->idx, a->count,
                    ws_header, w + lay.topk, s, -1, rb.flag, 1, rb.dtok, rb.ldd);
    if (e != cudaSuccess) return CLSA_ERR_CUDA;
    if (scores_kernel(rb.flag, rb.any_flag) != cudaSuccess) return CLSA_ERR_CUDA;
    e = launch_topk(scores, nullptr, a->T, a->n, a->k, a->idx, a->count, ws_header, w + lay.topk, s, a->n - a->T,
                    rb.flag, 0);
    if (e != cudaSuccess) return CLSA_ERR_CUDA;
  } else {
    if (scores_kernel(nullptr, nullptr) != cudaSuccess) return CLSA_ERR_CUDA;
    e = launch_topk(scores, nullptr, a->T, a->n, a->k, a->idx, a->count, ws_header, w + lay.topk, s, a->n - a->T);
    if (e != cudaSuccess) return CLSA_ERR_CUDA;
  }
  return run_prefill_attention(a, 0, ws_header, ws_body, s);
}

clsa_status run_prefill_attention(const clsa_prefill_args* a, int mode, void* ws_header, void* ws_body,
                                  cudaStream_t s) {
  const PrefillLayout lay = prefill_layout(a);
  char* w = static_cast<char*>(ws_body);
  const float scale = a->scale > 0.f ? a->scale : 1.0f / sqrtf((float)a->d);
  cudaError_t e;
  if (mode == 1) {
    if (!prefill_attn_pair_supported(a)) return CLSA_ERR_UNSUPPORTED;
    e = launch_prefill_attn_pair(a, scale, ws_header, s);
  } else if (prefill_attn_tc_supported(a)) {
    e = launch_prefill_attn_tc(a, scale, ws_header, s);
  } else {
    AttnShape sh{a->T, a->k, a->L, a->Hq, a->Hkv, a->d, a->dtype, true, a->n, 0};
    e = launch_sparse_attn(sh, a->Q, a->K, a->V, a->idx, a->count, scale, a->O, a->lse, ws_header, w + lay.attn, s);
  }
  return e == cudaSuccess ? CLSA_OK : CLSA_ERR_CUDA;
}

}  // namespace clsa
