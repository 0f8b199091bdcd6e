// Per-layer token-sparse GQA attention over the shared selection,
//   O_t^(l) = softmax(Q_t^(l) K_S^T * scale) V_S            for every layer l
// (picx.dev CLSA summary, Methodology > Architecture Overview, per-layer
// equation; scale 1/sqrt(d_k) from the zhichai.net post, Background).
//
// Split-k flash decoding.  A CTA owns one (sequence b, KV head g, layer group,
// token split).  Its rows are every (layer, query head) pair of that KV head in
// the layer group -- L*G rows share the same K_S/V_S rows, so the selected K/V
// rows of a split are read from memory once for all layers ("compute S_t once,
// reuse it in every layer").  Tokens stream through shared memory in blocks of
// 64 with an online softmax in the exp2 domain; splits are merged by a second
// kernel with the log-sum-exp rule.  In gather mode the rows are fetched
// straight from the [n][Hkv][d] cache through the index list, which fuses the
// Selector's gather into the attention.
//
// bf16: mma.sync m16n8k16 (fp32 accumulate), one warp per 16 rows, operands via
// ldmatrix from padded shared tiles; a ring of kStages token blocks keeps the gathered
// rows of the next blocks in flight while one is reduced.  fp32: FFMA, one lane per token for the
// scores and one lane per column for the output.
#include <cmath>

#include "common.cuh"
#include "kernels.h"

namespace clsa {

namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr int kBlk = 64;  // tokens per shared-memory block (bf16 path)
constexpr int kStages = 4;  // K/V blocks in flight (bf16 path): gathered rows have HBM latency

struct AttnParams {
  const void* Q;
  const void* K;
  const void* V;
  const int32_t* idx;
  const int32_t* count;
  int B, k, L, Hq, Hkv, G, n_max;
  long long kv_bstride;
  int Lg, nlg, rows, nsplit, chunk;
  float scale_log2;
  void* O;
  float* lse;
  float* Op;
  float* Mp;
  float* Lp;
  void* ws_header;
};

// address of token i's head-g row: compact [B][k][Hkv][D] or gathered from [B][n_max][Hkv][D]
template <typename T, int D, bool GATHER>
__device__ __forceinline__ const T* kv_row(const AttnParams& p, const T* base, int b, int g, int i, bool& ok) {
  if constexpr (GATHER) {
    const int t = __ldg(p.idx + (size_t)b * p.k + i);
    ok = (unsigned)t < (unsigned)p.n_max;
    if (!ok) {
      record_error(p.ws_header, CLSA_ERR_BAD_INDEX, ((long long)b << 32) | (unsigned)i);
      return base;
    }
    return base + (((size_t)b * p.kv_bstride + t) * p.Hkv + g) * D;
  } else {
    ok = true;
    return base + (((size_t)b * p.k + i) * p.Hkv + g) * D;
  }
}

// token t's head-g row of the [B][kv][Hkv][D] cache (t already read from the index list)
template <typename T, int D>
__device__ __forceinline__ const T* kv_row_tok(const AttnParams& p, const T* base, int b, int g, int i, int t,
                                               bool& ok) {
  ok = (unsigned)t < (unsigned)p.n_max;
  if (!ok) {
    record_error(p.ws_header, CLSA_ERR_BAD_INDEX, ((long long)b << 32) | (unsigned)i);
    return base;
  }
  return base + (((size_t)b * p.kv_bstride + t) * p.Hkv + g) * D;
}

// (layer, head) of CTA-local row r in layer group lgrp; false if r is padding
__device__ __forceinline__ bool row_coords(const AttnParams& p, int lgrp, int g, int r, int& l, int& h) {
  if (r >= p.rows) return false;
  l = lgrp * p.Lg + r / p.G;
  h = g * p.G + r % p.G;
  return l < p.L;
}

// ---------------------------------------------------------------------------
// bf16 tensor-core path
// ---------------------------------------------------------------------------
// MINB = 1: up to 8 warps, kStages-deep ring, Q fragments held in registers.
// MINB = 2: up to 6 warps and two CTAs per SM (their loads overlap each other's math):
// a 2-deep ring per CTA and Q fragments re-read from shared memory at each k-step.
template <int D, bool GATHER, int MINB>
__global__ void __launch_bounds__(MINB == 2 ? 192 : 256, MINB) attn_bf16_kernel(const AttnParams p) {
  constexpr int NST = MINB == 2 ? 2 : kStages;
  constexpr int STR = D + 8;  // padded row (elements): 16-byte aligned, ldmatrix conflict-free
  extern __shared__ __align__(16) unsigned char smem_raw[];
  __nv_bfloat16* sQ = reinterpret_cast<__nv_bfloat16*>(smem_raw);
  const int NW = blockDim.x >> 5;
  __nv_bfloat16* sK = sQ + NW * 16 * STR;            // [kStages][kBlk][STR]
  __nv_bfloat16* sV = sK + NST * kBlk * STR;     // [kStages][kBlk][STR]
  int* sIdx = reinterpret_cast<int*>(sV + NST * kBlk * STR);  // [chunk] this split's token indices

  const int split = blockIdx.x, g = blockIdx.y;
  const int b = blockIdx.z / p.nlg, lgrp = blockIdx.z % p.nlg;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gid = lane >> 2, tig = lane & 3;
  const int cnt = max(0, min(p.count[b], p.k));
  const int t0 = split * p.chunk;
  const int t1 = min(cnt, t0 + p.chunk);

  const __nv_bfloat16* Qg = static_cast<const __nv_bfloat16*>(p.Q);
  const __nv_bfloat16* Kg = static_cast<const __nv_bfloat16*>(p.K);
  const __nv_bfloat16* Vg = static_cast<const __nv_bfloat16*>(p.V);
  // the split's token indices, read once (coalesced): the gathers below then depend only on
  // shared memory, not on a global load per row
  if constexpr (GATHER)
    for (int j = threadIdx.x; j < t1 - t0; j += blockDim.x) sIdx[j] = __ldg(p.idx + (size_t)b * p.k + t0 + j);

  // ---- Q tile -> shared (zero rows for padding)
  {
    constexpr int VPR = D * 2 / 16;  // 16-byte vectors per row
    for (int v = threadIdx.x; v < NW * 16 * VPR; v += blockDim.x) {
      const int r = v / VPR, c = v % VPR;
      int l, h;
      uint4 val = make_uint4(0, 0, 0, 0);
      if (row_coords(p, lgrp, g, r, l, h))
        val = *reinterpret_cast<const uint4*>(Qg + (((size_t)l * p.B + b) * p.Hq + h) * D + c * 8);
      *reinterpret_cast<uint4*>(sQ + r * STR + c * 8) = val;
    }
  }

  auto load_block = [&](int stage, int blk0) {
    constexpr int VPR = D * 2 / 16;
    __nv_bfloat16* dk = sK + stage * kBlk * STR;
    __nv_bfloat16* dv = sV + stage * kBlk * STR;
    for (int v = threadIdx.x; v < kBlk * VPR; v += blockDim.x) {
      const int r = v / VPR, c = v % VPR;
      const int i = blk0 + r;
      const __nv_bfloat16* srck = Kg;
      const __nv_bfloat16* srcv = Vg;
      int bytes = 0;
      if (i < t1) {
        bool ok;
        if constexpr (GATHER) {
          const int tk = sIdx[i - t0];
          srck = kv_row_tok<__nv_bfloat16, D>(p, Kg, b, g, i, tk, ok);
          srcv = kv_row_tok<__nv_bfloat16, D>(p, Vg, b, g, i, tk, ok);
        } else {
          srck = kv_row<__nv_bfloat16, D, GATHER>(p, Kg, b, g, i, ok);
          srcv = kv_row<__nv_bfloat16, D, GATHER>(p, Vg, b, g, i, ok);
        }
        if (ok) {
          srck += c * 8;
          srcv += c * 8;
          bytes = 16;
        } else {
          srck = Kg;
          srcv = Vg;
        }
      }
      cp_async_16(dk + r * STR + c * 8, srck, bytes);
      cp_async_16(dv + r * STR + c * 8, srcv, bytes);
    }
    cp_async_commit();
  };

  const int nblk = t1 > t0 ? (t1 - t0 + kBlk - 1) / kBlk : 0;
  if constexpr (GATHER) __syncthreads();  // sIdx is visible to every thread
  for (int j = 0; j < NST - 1; ++j) {  // blocks 0 .. NST-2 in flight (one group each)
    if (j < nblk) load_block(j, t0 + j * kBlk);
    else cp_async_commit();
  }
  __syncthreads();

  constexpr int QR = MINB == 2 ? 1 : D / 16;  // Q fragments kept in registers
  uint32_t qa[QR][4];
  auto load_qa = [&](int ks, uint32_t (&f)[4]) {
    const int mi = lane >> 3;
    const int row = warp * 16 + (lane & 7) + 8 * (mi & 1);
    const int col = ks * 16 + 8 * (mi >> 1);
    ldmatrix_x4(f[0], f[1], f[2], f[3], sQ + row * STR + col);
  };
  if constexpr (MINB == 1) {
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) load_qa(ks, qa[ks]);
  }

  float o[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;

  for (int bi = 0; bi < nblk; ++bi) {
    const int stage = bi % NST;
    const int blk0 = t0 + bi * kBlk;
    {  // block bi + NST - 1 into the stage block bi - 1 used (released by its trailing sync)
      const int nb = bi + NST - 1;
      if (nb < nblk) load_block(nb % NST, t0 + nb * kBlk);
      else cp_async_commit();
    }
    cp_async_wait<NST - 1>();  // block bi has landed
    __syncthreads();
    const __nv_bfloat16* tk = sK + stage * kBlk * STR;
    const __nv_bfloat16* tv = sV + stage * kBlk * STR;

    // S = Q K^T for 64 tokens (8 n-tiles of 8)
    float s[kBlk / 8][4];
#pragma unroll
    for (int i = 0; i < kBlk / 8; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      uint32_t qf[4];
      if constexpr (MINB == 2) load_qa(ks, qf);
      const uint32_t(&qk)[4] = MINB == 2 ? qf : qa[MINB == 2 ? 0 : ks];
#pragma unroll
      for (int nt2 = 0; nt2 < kBlk / 16; ++nt2) {
        const int mi = lane >> 3;
        const int tok = nt2 * 16 + 8 * (mi >> 1) + (lane & 7);
        const int col = ks * 16 + 8 * (mi & 1);
        uint32_t r0, r1, r2, r3;
        ldmatrix_x4(r0, r1, r2, r3, tk + tok * STR + col);
        mma_bf16_16816(s[2 * nt2], qk, r0, r1);
        mma_bf16_16816(s[2 * nt2 + 1], qk, r2, r3);
      }
    }
    // scale, mask, row max
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < kBlk / 8; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int tok = blk0 + nt * 8 + 2 * tig + (e & 1);
        s[nt][e] = tok < t1 ? s[nt][e] * p.scale_log2 : -INFINITY;
      }
      mx0 = fmaxf(mx0, fmaxf(s[nt][0], s[nt][1]));
      mx1 = fmaxf(mx1, fmaxf(s[nt][2], s[nt][3]));
    }
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
    const float ref0 = mn0 == -INFINITY ? 0.f : mn0;
    const float ref1 = mn1 == -INFINITY ? 0.f : mn1;
    const float c0 = exp2f(m0 - ref0), c1 = exp2f(m1 - ref1);
    m0 = mn0;
    m1 = mn1;
    float rs0 = 0.f, rs1 = 0.f;
#pragma unroll
    for (int nt = 0; nt < kBlk / 8; ++nt) {
      s[nt][0] = exp2f(s[nt][0] - ref0);
      s[nt][1] = exp2f(s[nt][1] - ref0);
      s[nt][2] = exp2f(s[nt][2] - ref1);
      s[nt][3] = exp2f(s[nt][3] - ref1);
      rs0 += s[nt][0] + s[nt][1];
      rs1 += s[nt][2] + s[nt][3];
    }
    l0 = l0 * c0 + rs0;
    l1 = l1 * c1 + rs1;
#pragma unroll
    for (int nd = 0; nd < D / 8; ++nd) {
      o[nd][0] *= c0;
      o[nd][1] *= c0;
      o[nd][2] *= c1;
      o[nd][3] *= c1;
    }
    // O += P V
#pragma unroll
    for (int kk = 0; kk < kBlk / 16; ++kk) {
      uint32_t pa[4];
      pa[0] = pack_bf16x2(s[2 * kk][0], s[2 * kk][1]);
      pa[1] = pack_bf16x2(s[2 * kk][2], s[2 * kk][3]);
      pa[2] = pack_bf16x2(s[2 * kk + 1][0], s[2 * kk + 1][1]);
      pa[3] = pack_bf16x2(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
      for (int nd2 = 0; nd2 < D / 16; ++nd2) {
        const int mi = lane >> 3;
        const int tok = kk * 16 + 8 * (mi & 1) + (lane & 7);
        const int col = nd2 * 16 + 8 * (mi >> 1);
        uint32_t r0, r1, r2, r3;
        ldmatrix_x4_trans(r0, r1, r2, r3, tv + tok * STR + col);
        mma_bf16_16816(o[2 * nd2], pa, r0, r1);
        mma_bf16_16816(o[2 * nd2 + 1], pa, r2, r3);
      }
    }
    __syncthreads();
  }

  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);

#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int r = warp * 16 + gid + 8 * half;
    int l, h;
    if (!row_coords(p, lgrp, g, r, l, h)) continue;
    const float m = half ? m1 : m0;
    const float lsum = half ? l1 : l0;
    if (p.nsplit == 1) {
      const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
      __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.O) + (((size_t)l * p.B + b) * p.Hq + h) * D;
#pragma unroll
      for (int nd = 0; nd < D / 8; ++nd) {
        const uint32_t w = pack_bf16x2(o[nd][2 * half] * inv, o[nd][2 * half + 1] * inv);
        *reinterpret_cast<uint32_t*>(out + nd * 8 + 2 * tig) = w;
      }
      if (p.lse && tig == 0)
        p.lse[((size_t)l * p.B + b) * p.Hq + h] = lsum > 0.f ? (m + log2f(lsum)) * kLn2 : -INFINITY;
    } else {
      const size_t pi = ((((size_t)b * p.Hkv + g) * p.nlg + lgrp) * p.nsplit + split) * p.rows + r;
      float* op = p.Op + pi * D;
#pragma unroll
      for (int nd = 0; nd < D / 8; ++nd)
        *reinterpret_cast<float2*>(op + nd * 8 + 2 * tig) = make_float2(o[nd][2 * half], o[nd][2 * half + 1]);
      if (tig == 0) {
        p.Mp[pi] = m;
        p.Lp[pi] = lsum;
      }
    }
  }
}

// ---------------------------------------------------------------------------
// fp32 FFMA path (4 warps, up to 32 rows per CTA, 32-token blocks)
// ---------------------------------------------------------------------------
template <int D, bool GATHER>
__global__ void __launch_bounds__(128) attn_f32_kernel(const AttnParams p) {
  constexpr int TB = 32;
  constexpr int MAXR = 8;  // rows per warp
  constexpr int CPL = D / 32;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  float* sQ = reinterpret_cast<float*>(smem_raw);  // [32][D]
  float* sK = sQ + 32 * D;                          // [TB][D+1]
  float* sV = sK + TB * (D + 1);                    // [TB][D]

  const int split = blockIdx.x, g = blockIdx.y;
  const int b = blockIdx.z / p.nlg, lgrp = blockIdx.z % p.nlg;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cnt = max(0, min(p.count[b], p.k));
  const int t0 = split * p.chunk;
  const int t1 = min(cnt, t0 + p.chunk);
  const float* Qg = static_cast<const float*>(p.Q);
  const float* Kg = static_cast<const float*>(p.K);
  const float* Vg = static_cast<const float*>(p.V);

  for (int v = threadIdx.x; v < 32 * D; v += blockDim.x) {
    const int r = v / D, c = v % D;
    int l, h;
    sQ[v] = row_coords(p, lgrp, g, r, l, h) ? Qg[(((size_t)l * p.B + b) * p.Hq + h) * D + c] : 0.f;
  }

  float m[MAXR], lsum[MAXR], o[MAXR][CPL];
#pragma unroll
  for (int j = 0; j < MAXR; ++j) {
    m[j] = -INFINITY;
    lsum[j] = 0.f;
#pragma unroll
    for (int c = 0; c < CPL; ++c) o[j][c] = 0.f;
  }

  for (int blk0 = t0; blk0 < t1; blk0 += TB) {
    __syncthreads();
    for (int v = threadIdx.x; v < TB * D; v += blockDim.x) {
      const int r = v / D, c = v % D;
      const int i = blk0 + r;
      float kv = 0.f, vv = 0.f;
      if (i < t1) {
        bool ok;
        const float* rk = kv_row<float, D, GATHER>(p, Kg, b, g, i, ok);
        const float* rv = kv_row<float, D, GATHER>(p, Vg, b, g, i, ok);
        if (ok) {
          kv = rk[c];
          vv = rv[c];
        }
      }
      sK[r * (D + 1) + c] = kv;
      sV[r * D + c] = vv;
    }
    __syncthreads();
    const int tok = blk0 + lane;
#pragma unroll
    for (int j = 0; j < MAXR; ++j) {
      const int r = warp + 4 * j;
      if (r >= p.rows) break;
      float s = 0.f;
#pragma unroll 8
      for (int c = 0; c < D; ++c) s = fmaf(sQ[r * D + c], sK[lane * (D + 1) + c], s);
      s = tok < t1 ? s * p.scale_log2 : -INFINITY;
      const float mn = fmaxf(m[j], warp_max(s));
      const float ref = mn == -INFINITY ? 0.f : mn;
      const float corr = exp2f(m[j] - ref);
      const float pr = exp2f(s - ref);
      m[j] = mn;
      lsum[j] = lsum[j] * corr + warp_sum(pr);
#pragma unroll
      for (int c = 0; c < CPL; ++c) o[j][c] *= corr;
#pragma unroll 4
      for (int i = 0; i < TB; ++i) {
        const float pi = __shfl_sync(0xffffffffu, pr, i);
#pragma unroll
        for (int c = 0; c < CPL; ++c) o[j][c] = fmaf(pi, sV[i * D + lane + 32 * c], o[j][c]);
      }
    }
  }

#pragma unroll
  for (int j = 0; j < MAXR; ++j) {
    const int r = warp + 4 * j;
    int l, h;
    if (!row_coords(p, lgrp, g, r, l, h)) continue;
    if (p.nsplit == 1) {
      const float inv = lsum[j] > 0.f ? 1.f / lsum[j] : 0.f;
      float* out = static_cast<float*>(p.O) + (((size_t)l * p.B + b) * p.Hq + h) * D;
#pragma unroll
      for (int c = 0; c < CPL; ++c) out[lane + 32 * c] = o[j][c] * inv;
      if (p.lse && lane == 0)
        p.lse[((size_t)l * p.B + b) * p.Hq + h] = lsum[j] > 0.f ? (m[j] + log2f(lsum[j])) * kLn2 : -INFINITY;
    } else {
      const size_t pi = ((((size_t)b * p.Hkv + g) * p.nlg + lgrp) * p.nsplit + split) * p.rows + r;
#pragma unroll
      for (int c = 0; c < CPL; ++c) p.Op[pi * D + lane + 32 * c] = o[j][c];
      if (lane == 0) {
        p.Mp[pi] = m[j];
        p.Lp[pi] = lsum[j];
      }
    }
  }
}

// ---------------------------------------------------------------------------
// split combine: O = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s
// ---------------------------------------------------------------------------
template <typename T, int D>
__global__ void __launch_bounds__(256) attn_combine_kernel(const AttnParams p) {
  // one warp per output row.  Every load of a group of 32 splits is issued before any is
  // used: lane s reads split s's max and row sum, and every lane its columns of all the
  // group's partial outputs, so a row costs one L2 round trip per 32 splits (the reductions
  // over the lanes follow in registers).
  constexpr int CPL = D / 32;  // output columns per lane: 4 (D = 128) or 2 (D = 64)
  pdl_enter();  // launched programmatically behind the attention kernel: its partials first
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= p.L * p.B * p.Hq) return;
  const int h = row % p.Hq;
  const int b = (row / p.Hq) % p.B;
  const int l = row / (p.Hq * p.B);
  const int g = h / p.G, lgrp = l / p.Lg;
  const int r = (l % p.Lg) * p.G + h % p.G;
  const size_t base = (((size_t)b * p.Hkv + g) * p.nlg + lgrp) * p.nsplit * p.rows + r;
  float acc[CPL];
#pragma unroll
  for (int c = 0; c < CPL; ++c) acc[c] = 0.f;
  float M = -INFINITY, den = 0.f;
  for (int s0 = 0; s0 < p.nsplit; s0 += 32) {
    const int ns = min(32, p.nsplit - s0);
    float ml = -INFINITY, ll = 0.f;  // split s0 + lane
    if (lane < ns) {
      const size_t pi = base + (size_t)(s0 + lane) * p.rows;
      ml = __ldcg(p.Mp + pi);
      ll = __ldcg(p.Lp + pi);
    }
    float o[32][CPL];
#pragma unroll
    for (int u = 0; u < 32; ++u) {
      const float* src = p.Op + (base + (size_t)(s0 + min(u, ns - 1)) * p.rows) * D + lane * CPL;
      if constexpr (CPL == 4) {
        const float4 v = __ldcg(reinterpret_cast<const float4*>(src));
        o[u][0] = v.x;
        o[u][1] = v.y;
        o[u][2] = v.z;
        o[u][3] = v.w;
      } else {
        const float2 v = __ldcg(reinterpret_cast<const float2*>(src));
        o[u][0] = v.x;
        o[u][1] = v.y;
      }
    }
    // merge this group into the running (M, den, acc)
    const float Mg = warp_max(ml);
    const float Mn = fmaxf(M, Mg);
    if (Mn != -INFINITY) {
      const float a = exp2f(M - Mn);  // 0 on the first group with a finite max
      const float wl = exp2f(ml - Mn);
      den = den * a + warp_sum(wl * ll);
#pragma unroll
      for (int c = 0; c < CPL; ++c) acc[c] *= a;
#pragma unroll
      for (int u = 0; u < 32; ++u) {
        float w = __shfl_sync(0xffffffffu, wl, u);
        w = u < ns ? w : 0.f;  // past the last split: the clamped reload counts 0
#pragma unroll
        for (int c = 0; c < CPL; ++c) acc[c] = fmaf(w, o[u][c], acc[c]);
      }
      M = Mn;
    }
  }
  const float inv = den > 0.f ? 1.f / den : 0.f;
  T* out = static_cast<T*>(p.O) + (((size_t)l * p.B + b) * p.Hq + h) * D;
#pragma unroll
  for (int c = 0; c < CPL; ++c) out[lane * CPL + c] = Elem<T>::from_f(acc[c] * inv);
  if (p.lse && lane == 0)
    p.lse[((size_t)l * p.B + b) * p.Hq + h] = den > 0.f ? (M + log2f(den)) * kLn2 : -INFINITY;
}

bool aligned16_(const void* a) { return reinterpret_cast<uintptr_t>(a) % 16 == 0; }

template <typename K>
cudaError_t set_smem(K kernel, int bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

}  // namespace

AttnPlan plan_attention(const AttnShape& sh) {
  AttnPlan pl{};
  if (sparse_attn_rows_plan(sh, device_info().sm_count, &pl)) return pl;
  const int G = sh.Hq / sh.Hkv;
  const int max_rows = sh.dt == CLSA_BF16 ? 128 : 32;
  int Lg = std::max(1, std::min(sh.L, max_rows / G));
  pl.nlg = (sh.L + Lg - 1) / Lg;
  pl.Lg = (sh.L + pl.nlg - 1) / pl.nlg;
  pl.rows = pl.Lg * G;
  const int units = sh.B * sh.Hkv * pl.nlg;
  const int blk = sh.dt == CLSA_BF16 ? 64 : 32;
  const int target = 2 * std::max(device_info().sm_count, 1);
  int nsplit = std::max(1, (target + units - 1) / units);
  const int max_split = (sh.k + blk - 1) / blk;
  nsplit = std::min(nsplit, max_split);
  int chunk = (sh.k + nsplit - 1) / nsplit;
  chunk = (chunk + blk - 1) / blk * blk;
  pl.chunk = chunk;
  pl.nsplit = (sh.k + chunk - 1) / chunk;
  return pl;
}

size_t attn_counter_bytes(const AttnShape& sh) { return align_up((size_t)sh.B * sh.Hkv * sizeof(uint32_t), 256); }

size_t attn_ws_bytes(const AttnShape& sh) {
  const AttnPlan pl = plan_attention(sh);
  if (pl.nsplit == 1) return 0;
  const size_t n = (size_t)sh.B * sh.Hkv * pl.nlg * pl.nsplit * pl.rows;
  // one arrival counter per (b, KV head) first, at an offset no plan changes (so calls of other
  // shapes on the same workspace never write over them), then the split partials (output, max,
  // sum)
  return attn_counter_bytes(sh) + align_up(n * sh.d * sizeof(float), 256) + 2 * align_up(n * sizeof(float), 256);
}

cudaError_t launch_sparse_attn(const AttnShape& sh, const void* Q, const void* Kc, const void* Vc,
                               const int32_t* idx, const int32_t* count, float scale, void* O, float* lse,
                               void* ws_header, void* attn_ws, cudaStream_t s) {
  const AttnPlan pl = plan_attention(sh);
  AttnParams p{};
  p.Q = Q;
  p.K = Kc;
  p.V = Vc;
  p.idx = idx;
  p.count = count;
  p.B = sh.B;
  p.k = sh.k;
  p.L = sh.L;
  p.Hq = sh.Hq;
  p.Hkv = sh.Hkv;
  p.G = sh.Hq / sh.Hkv;
  p.n_max = sh.n_max;
  p.kv_bstride = sh.kv_bstride;
  p.Lg = pl.Lg;
  p.nlg = pl.nlg;
  p.rows = pl.rows;
  p.nsplit = pl.nsplit;
  p.chunk = pl.chunk;
  p.scale_log2 = scale * kLog2e;
  p.O = O;
  p.lse = lse;
  p.ws_header = ws_header;
  uint32_t* counter = nullptr;
  if (pl.nsplit > 1) {
    const size_t n = (size_t)sh.B * sh.Hkv * pl.nlg * pl.nsplit * pl.rows;
    char* w = static_cast<char*>(attn_ws);
    counter = reinterpret_cast<uint32_t*>(w);
    w += attn_counter_bytes(sh);
    p.Op = reinterpret_cast<float*>(w);
    w += align_up(n * sh.d * sizeof(float), 256);
    p.Mp = reinterpret_cast<float*>(w);
    w += align_up(n * sizeof(float), 256);
    p.Lp = reinterpret_cast<float*>(w);
  }
  AttnPlan rp{};
  if (sparse_attn_rows_plan(sh, device_info().sm_count, &rp) && aligned16_(Q) && aligned16_(Kc) && aligned16_(Vc) &&
      aligned16_(O))
    return launch_sparse_attn_rows(sh, pl, Q, Kc, Vc, idx, count, p.scale_log2, O, lse, p.Op, p.Mp, p.Lp, counter,
                                   ws_header, s);
  dim3 grid(pl.nsplit, sh.Hkv, sh.B * pl.nlg);
  cudaError_t e = cudaSuccess;
  const bool tc5 = sparse_attn_tc_supported(sh, pl, Q, Kc, Vc, O);
  if (tc5) {  // counts its own launch
    e = launch_sparse_attn_tc(sh, pl, Q, Kc, Vc, idx, count, p.scale_log2, O, lse, p.Op, p.Mp, p.Lp, ws_header, s);
  } else if (sh.dt == CLSA_BF16) {
    const int NW = (pl.rows + 15) / 16;
    const bool two = NW <= 6;  // two CTAs per SM fit
    // the split's token list lives in shared memory only when gathering by index
    auto smem = [&](int D, int nst) { return (NW * 16 + 2 * nst * kBlk) * (D + 8) * 2 + (sh.gather ? pl.chunk * 4 : 0); };
#define CLSA_ATTN_BF16(D, GA)                                                           \
  do {                                                                                  \
    if (two) {                                                                          \
      auto kern = attn_bf16_kernel<D, GA, 2>;                                           \
      e = set_smem(kern, smem(D, 2));                                                   \
      if (e == cudaSuccess) kern<<<grid, NW * 32, smem(D, 2), s>>>(p);                 \
    } else {                                                                            \
      auto kern = attn_bf16_kernel<D, GA, 1>;                                           \
      e = set_smem(kern, smem(D, kStages));                                             \
      if (e == cudaSuccess) kern<<<grid, NW * 32, smem(D, kStages), s>>>(p);           \
    }                                                                                   \
  } while (0)
    if (sh.d == 128) {
      if (sh.gather) CLSA_ATTN_BF16(128, true);
      else CLSA_ATTN_BF16(128, false);
    } else {
      if (sh.gather) CLSA_ATTN_BF16(64, true);
      else CLSA_ATTN_BF16(64, false);
    }
#undef CLSA_ATTN_BF16
  } else {
    auto smem = [&](int D) { return (32 * D + 32 * (D + 1) + 32 * D) * 4; };
#define CLSA_ATTN_F32(D, GA)                                                   \
  do {                                                                         \
    auto kern = attn_f32_kernel<D, GA>;                                        \
    e = set_smem(kern, smem(D));                                               \
    if (e == cudaSuccess) kern<<<grid, 128, smem(D), s>>>(p);                  \
  } while (0)
    if (sh.d == 128) {
      if (sh.gather) CLSA_ATTN_F32(128, true);
      else CLSA_ATTN_F32(128, false);
    } else {
      if (sh.gather) CLSA_ATTN_F32(64, true);
      else CLSA_ATTN_F32(64, false);
    }
#undef CLSA_ATTN_F32
  }
  if (!tc5) launches_add(1, s);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess || pl.nsplit == 1) return e;
  const int rows_total = sh.L * sh.B * sh.Hq;
  dim3 cg((rows_total + 7) / 8);
  if (sh.dt == CLSA_BF16) {
    if (sh.d == 128) e = launch_pdl(attn_combine_kernel<__nv_bfloat16, 128>, cg, dim3(256), 0, s, p);
    else e = launch_pdl(attn_combine_kernel<__nv_bfloat16, 64>, cg, dim3(256), 0, s, p);
  } else {
    if (sh.d == 128) e = launch_pdl(attn_combine_kernel<float, 128>, cg, dim3(256), 0, s, p);
    else e = launch_pdl(attn_combine_kernel<float, 64>, cg, dim3(256), 0, s, p);
  }
  launches_add(1, s);
  return e;
}

}  // namespace clsa
