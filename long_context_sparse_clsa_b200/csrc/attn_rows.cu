// Token-sparse GQA attention for few rows per KV head (L*G <= 16: one layer's heads, the
// model-faithful per-layer decode call), bf16, d = 64 or 128:
//   O^(l)[b, h] = softmax(Q^(l)[b, h] K_S^T * scale) V_S
// (picx.dev CLSA summary, Methodology > Architecture Overview, per-layer equation).
//
// With 4 query rows per KV head the products are a handful of 16 x 8 x 16 tiles per CTA: a
// tcgen05 pipeline (TMEM allocation, 128-row tiles, commit round trips) would only add
// latency, and the time is the latency of moving K_S/V_S in and the result out.  So the
// tiles run on warp-level mma.sync (bf16 in, fp32 out, operands by ldmatrix) and the kernel
// is built to take few dependent round trips:
//   1. one CTA per (token split, KV head, sequence): its Q rows (zero-padded to 16) and its
//      <= 128 selected K/V rows land in shared memory in one wave of 16-byte async copies;
//   2. warp w: S for tokens [16 w, 16 w + 16); the split's row max and row sum through
//      shared memory; P as bf16 in shared memory;
//   3. warp w: P V for output columns [16 w, 16 w + 16) over all the split's tokens;
//   4. the split's unnormalised output, max and sum go to the split partials; the CTA that
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
  static constexpr int STR = D + 8;   // padded bf16 row: conflict-free ldmatrix
  static constexpr int PSTR = kMaxTokR + 8;
  __nv_bfloat16 K[kMaxTokR][STR];
  __nv_bfloat16 V[kMaxTokR][STR];
  __nv_bfloat16 Q[kMaxRowsR][STR];  // rows >= R are zero
  __nv_bfloat16 P[kMaxRowsR][PSTR];
  float red_m[kThreadsR / 32][kMaxRowsR], red_l[kThreadsR / 32][kMaxRowsR];
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
  for (int v = tid; v < kMaxRowsR * VPR; v += kThreadsR) {  // row r = (layer r / G, head g * G + r % G)
    const int r = v / VPR, c = v % VPR;
    if (r < R) {
      const int l = r / p.G, h = g * p.G + r % p.G;
      cp_async_16(&sm.Q[r][c * 8], p.Q + (((size_t)l * p.B + b) * p.Hq + h) * D + c * 8, 16);
    } else {
      *reinterpret_cast<uint4*>(&sm.Q[r][c * 8]) = make_uint4(0u, 0u, 0u, 0u);  // padding rows: S = 0
    }
  }
  __syncthreads();  // tokens visible
  const int nt16 = (ntok + 15) & ~15;  // the MMAs read whole 16-token tiles: the rest zero-filled
  const size_t gstride = (size_t)p.Hkv * D;
  const size_t gbase = (size_t)b * (size_t)p.kv_bstride * gstride + (size_t)g * D;
  for (int v = tid; v < nt16 * VPR; v += kThreadsR) {
    const int i = v / VPR, c = v % VPR;
    const int tk = i < ntok ? sm.tok[i] : -1;
    const size_t off = tk >= 0 ? gbase + (size_t)tk * gstride + c * 8 : 0;
    cp_async_16(&sm.K[i][c * 8], p.K + off, tk >= 0 ? 16 : 0);
    cp_async_16(&sm.V[i][c * 8], p.V + off, tk >= 0 ? 16 : 0);
  }
  cp_async_commit();
  cp_async_wait<0>();
  __syncthreads();

  // ---- 2. S = Q K^T: warp w takes tokens [16 w, 16 w + 16) (mma.sync m16n8k16, fp32) ------
  const int gid = lane >> 2, tig = lane & 3, mi = lane >> 3;
  float sc[2][4];  // rows gid, gid + 8; tokens 16 w + 8 nt + 2 tig + (e & 1)
#pragma unroll
  for (int nt = 0; nt < 2; ++nt) sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
  if (16 * warp < nt16) {
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      uint32_t qa[4], k0, k1, k2, k3;
      ldmatrix_x4(qa[0], qa[1], qa[2], qa[3], &sm.Q[(lane & 7) + 8 * (mi & 1)][ks * 16 + 8 * (mi >> 1)]);
      ldmatrix_x4(k0, k1, k2, k3, &sm.K[16 * warp + 8 * (mi >> 1) + (lane & 7)][ks * 16 + 8 * (mi & 1)]);
      mma_bf16_16816(sc[0], qa, k0, k1);
      mma_bf16_16816(sc[1], qa, k2, k3);
    }
  }
  float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
  for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int t = 16 * warp + 8 * nt + 2 * tig + (e & 1);
      sc[nt][e] = t < ntok ? sc[nt][e] * p.scale_log2 : -INFINITY;
    }
    mx0 = fmaxf(mx0, fmaxf(sc[nt][0], sc[nt][1]));
    mx1 = fmaxf(mx1, fmaxf(sc[nt][2], sc[nt][3]));
  }
  mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
  mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
  mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
  mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
  if (tig == 0) {
    sm.red_m[warp][gid] = mx0;
    sm.red_m[warp][gid + 8] = mx1;
  }
  __syncthreads();
  float M0 = -INFINITY, M1 = -INFINITY;  // the split's row maxima (log2 units)
#pragma unroll
  for (int w2 = 0; w2 < kThreadsR / 32; ++w2) {
    M0 = fmaxf(M0, sm.red_m[w2][gid]);
    M1 = fmaxf(M1, sm.red_m[w2][gid + 8]);
  }
  const float r0 = M0 == -INFINITY ? 0.f : M0, r1 = M1 == -INFINITY ? 0.f : M1;
  float l0 = 0.f, l1 = 0.f;
#pragma unroll
  for (int nt = 0; nt < 2; ++nt) {
    const float a0 = exp2f(sc[nt][0] - r0), a1 = exp2f(sc[nt][1] - r0);
    const float b0 = exp2f(sc[nt][2] - r1), b1 = exp2f(sc[nt][3] - r1);
    l0 += a0 + a1;
    l1 += b0 + b1;
    const int t = 16 * warp + 8 * nt + 2 * tig;
    if (t < kMaxTokR) {
      *reinterpret_cast<uint32_t*>(&sm.P[gid][t]) = pack_bf16x2(a0, a1);
      *reinterpret_cast<uint32_t*>(&sm.P[gid + 8][t]) = pack_bf16x2(b0, b1);
    }
  }
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  if (tig == 0) {
    sm.red_l[warp][gid] = l0;
    sm.red_l[warp][gid + 8] = l1;
  }
  __syncthreads();  // P and the partial row sums complete

  // ---- 3. O = P V: warp w takes output columns [16 w, 16 w + 16) over all tokens ----------
  float o[2][4];
#pragma unroll
  for (int nd = 0; nd < 2; ++nd) o[nd][0] = o[nd][1] = o[nd][2] = o[nd][3] = 0.f;
  const bool pv = 16 * warp < D;
  if (pv) {
#pragma unroll 1
    for (int kk = 0; kk < nt16 / 16; ++kk) {
      uint32_t pa[4], v0, v1, v2, v3;
      ldmatrix_x4(pa[0], pa[1], pa[2], pa[3], &sm.P[(lane & 7) + 8 * (mi & 1)][kk * 16 + 8 * (mi >> 1)]);
      ldmatrix_x4_trans(v0, v1, v2, v3, &sm.V[kk * 16 + 8 * (mi & 1) + (lane & 7)][16 * warp + 8 * (mi >> 1)]);
      mma_bf16_16816(o[0], pa, v0, v1);
      mma_bf16_16816(o[1], pa, v2, v3);
    }
  }
  float L0 = 0.f, L1 = 0.f;  // the split's row sums
#pragma unroll
  for (int w2 = 0; w2 < kThreadsR / 32; ++w2) {
    L0 += sm.red_l[w2][gid];
    L1 += sm.red_l[w2][gid + 8];
  }
  // this thread's outputs: rows gid (e < 2) and gid + 8, columns 16 w + 8 nd + 2 tig + (e & 1)
  auto out_row = [&](int r) -> __nv_bfloat16* {
    const int l = r / p.G, h = g * p.G + r % p.G;
    return p.O + (((size_t)l * p.B + b) * p.Hq + h) * D;
  };
  auto store_lse = [&](int r, float m2, float s2) {
    if (!p.lse) return;
    const int l = r / p.G, h = g * p.G + r % p.G;
    p.lse[((size_t)l * p.B + b) * p.Hq + h] = s2 > 0.f ? (m2 + log2f(s2)) * kLn2R : -INFINITY;
  };

  if (p.nsplit == 1) {  // the CTA holds the whole selection: final rows
    if (pv) {
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const int r = gid + 8 * hf;
        if (r >= R) continue;
        const float Ls = hf ? L1 : L0;
        const float inv = Ls > 0.f ? 1.f / Ls : 0.f;
        __nv_bfloat16* dst = out_row(r);
#pragma unroll
        for (int nd = 0; nd < 2; ++nd)
          *reinterpret_cast<uint32_t*>(dst + 16 * warp + 8 * nd + 2 * tig) =
              pack_bf16x2(o[nd][2 * hf] * inv, o[nd][2 * hf + 1] * inv);
      }
    }
    if (warp == 0 && tig == 0) {
      if (gid < R) store_lse(gid, M0, L0);
      if (gid + 8 < R) store_lse(gid + 8, M1, L1);
    }
    return;
  }

  // ---- 4. split partials, then the last CTA of (b, g) merges -------------------------------
  const size_t ub = ((size_t)b * p.Hkv + g) * p.nsplit;  // this (b, g)'s first split
  if (pv) {
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      const int r = gid + 8 * hf;
      if (r >= R) continue;
      float* dst = p.Op + ((ub + split) * R + r) * D + 16 * warp + 2 * tig;
#pragma unroll
      for (int nd = 0; nd < 2; ++nd) __stcg(reinterpret_cast<float2*>(dst + 8 * nd), make_float2(o[nd][2 * hf], o[nd][2 * hf + 1]));
    }
  }
  if (warp == 0 && tig == 0) {
    const float mm0 = ntok > 0 ? M0 : -INFINITY, mm1 = ntok > 0 ? M1 : -INFINITY;
    if (gid < R) {
      __stcg(p.Mp + (ub + split) * R + gid, mm0);
      __stcg(p.Lp + (ub + split) * R + gid, L0);
    }
    if (gid + 8 < R) {
      __stcg(p.Mp + (ub + split) * R + gid + 8, mm1);
      __stcg(p.Lp + (ub + split) * R + gid + 8, L1);
    }
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
  constexpr int NQ = D / 4;            // column quads: 32 (D = 128) or 16 (D = 64)
  constexpr int RPT = kThreadsR / NQ;  // row slots per pass: 8 or 16
  const int cq = tid % NQ, rr = tid / NQ;
  auto store_out = [&](int r, const float* v4, float scale) {  // O row r, columns cq * 4 ..
    *reinterpret_cast<uint2*>(out_row(r) + cq * 4) = make_uint2(pack_bf16x2(v4[0] * scale, v4[1] * scale),
                                                                pack_bf16x2(v4[2] * scale, v4[3] * scale));
  };

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
  // about one CTA per SM: splits of up to 128 tokens (fewer splits to merge beat more CTAs
  // in flight: 7.7 vs 9.2 us per one-layer call at 128K)
  const long long target = std::max(sm_count, 1);
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
