// Token-sparse GQA attention on the 5th-generation tensor cores (bf16, d = 128).
//
// Per-layer equation (picx.dev CLSA summary, Methodology > Architecture Overview):
//   O^(l)[b, h] = softmax(Q^(l)[b, h] K_S^T * scale) V_S,   S = the selected token list of b
// with query head h reading KV head h / G.  One kernel serves two callers:
//   * clsa_sparse_attn: B sequences, each with its selection (or an already-gathered compact
//     K_S/V_S), every layer of a layer group reading the same selected rows;
//   * the prefill chunk: every new row t is its own "sequence" b = t with its own S_t over
//     the one shared cache (sequence stride 0 into K/V).
//
// One CTA per unit (KV head g, layer group, sequence b, token split).  Units run head-major,
// so the CTAs in flight share one head's K/V rows in L2.  The unit's M rows are the (layer,
// query head) pairs of head g (L*G = 96 at the 24-layer, 32/8-head shape; G = 4 for one
// layer), the A operand of every chunk.  The split's tokens go in chunks of 64:
//   S = Q K_c^T      tcgen05.mma M128 N64 (K = d, 8 steps) -> TMEM, double-buffered
//   softmax          8 warps: one row (TMEM lane) and 32 of the chunk's columns per
//                    thread; the chunk's row max is exchanged through shared memory
//   O += P_c V_c     P_c bf16 in shared memory (A, K-major), V_c as the MN-major B operand
//                    from its row-major [token][d] tile: M128 N128 (K = 64), accumulated in
//                    TMEM.  P is taken against a reference max that moves only when a row
//                    max grows by more than 2^8: then O and the row sum are rescaled once,
//                    by TMEM load / multiply / store.
// The S MMAs of chunk c + 1 go out right behind P V of chunk c.  K/V chunks are gathered
// by 16-byte async copies into the 128-byte-swizzle layout, one chunk ahead (2 stages).
// At most about 111 KiB of shared memory and 256 TMEM columns per CTA: two CTAs share an
// SM, so one CTA's softmax overlaps the other's MMAs and gathers.
//
// With one split the unit's rows are final (O = acc / l, lse = m + log2 l in natural
// units).  With several, the unit writes the unnormalised accumulator, its reference max
// (log2 units) and its row sum to the split partials, which the log-sum-exp combine of the
// split-k path merges.
//
// Only the Q and P rows that exist are stored (rows rounded up to 8); the MMAs read the
// 128-row tiles on into the next shared-memory region.  Those extra rows only produce
// TMEM rows that no thread reads.  Every wait is bounded (kWaitLimitNs).
#include <algorithm>
#include <cmath>

#include "common.cuh"
#include "kernels.h"
#include "tcgen05.cuh"

namespace clsa {

namespace {

constexpr int kW = 8;                               // warps: 4 lane quarters x 2 column groups
constexpr int kThreadsTC = kW * 32;
constexpr int kTok = 64;                            // tokens per chunk
constexpr int kD = 128;                             // head dim
constexpr int kM = 128;                             // MMA rows
constexpr int kNpt = kTok / 2;                      // S columns per thread
constexpr int kOpt = kD / 2;                        // output columns per thread
constexpr uint32_t kKVAtom = kTok * 128;            // 64 rows x 128 bytes
constexpr uint32_t kKVTile = 2 * kKVAtom;           // K or V chunk: both 64-column atoms
constexpr uint32_t kStageBytes = 2 * kKVTile;       // K and V
constexpr uint32_t kTmemCols = 256;                 // S at [0, 128) (two buffers), O at [128, 256)
constexpr uint32_t kIdescQK = tc::idesc_bf16_f32(kM, kTok);
constexpr uint32_t kIdescPV = tc::idesc_bf16_f32(kM, kD) | (1u << 16);  // B (V) MN-major
constexpr float kLn2 = 0.6931471805599453f;

static_assert(kThreadsTC == 256 && kTok == 64, "the gather maps 256 threads onto 64 rows x 16 columns");

struct TCParams {
  const __nv_bfloat16* Q;   // [L][B][Hq][d]
  const __nv_bfloat16* K;   // token r of sequence b, head g: row ((b * kv_bstride + r) * Hkv + g)
  const __nv_bfloat16* V;
  const int32_t* idx;       // [B][k] selected tokens, or null: position i is row i (compact K_S/V_S)
  const int32_t* count;     // [B]
  __nv_bfloat16* O;         // [L][B][Hq][d]
  float* lse;               // [L][B][Hq] or null
  float* Op;                // split partials (nsplit > 1), attn_combine layout
  float* Mp;
  float* Lp;
  void* ws_header;
  long long kv_bstride;
  int B, k, L, Hq, Hkv, G, Lg, nlg, rows, n_max, nsplit, chunk;
  float scale_log2;
};

// shared-memory carve-up (offsets from a 1024-aligned base)
struct TCLayout {
  uint32_t q_atom, q, kv, p, tok, cm, cl, bars, total;
};
__host__ __device__ inline TCLayout tc_layout(int rows, int chunk) {
  TCLayout s;
  const uint32_t rows8 = (uint32_t)((rows + 7) & ~7);
  s.q_atom = rows8 * 128;                        // one 64-column atom of the rows that exist
  s.q = 0;
  s.kv = 2 * s.q_atom;                           // [2 stages][K, V]
  s.p = s.kv + 2 * kStageBytes;                  // P: rows8 x 64 tokens
  s.tok = s.p + s.q_atom;                        // [chunk] the split's selected tokens
  s.cm = s.tok + (uint32_t)(((chunk * 4) + 15) & ~15);  // [2][128] row-max exchange
  s.cl = s.cm + 2 * kM * 4;                      // [2][128] row-sum exchange
  s.bars = s.cl + 2 * kM * 4;                    // bar_s, bar_o, tmem address
  s.total = s.bars + 32;
  // the MMAs read 128-row tiles: keep the reads past Q atom 1 and past P inside the carve-up
  const uint32_t tail = s.p + (uint32_t)kM * 128 + 128;  // + the K-step offset of the last read
  if (s.total < tail) s.total = tail;
  return s;
}

__global__ void __launch_bounds__(kThreadsTC, 2) attn_tc_kernel(const TCParams p) {
  pdl_enter();  // launched programmatically: the previous kernel's writes first
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const TCLayout lay = tc_layout(p.rows, p.chunk);
  unsigned char* sQ = base + lay.q;
  unsigned char* kv = base + lay.kv;
  unsigned char* sP = base + lay.p;
  int32_t* stok = reinterpret_cast<int32_t*>(base + lay.tok);
  float* cm = reinterpret_cast<float*>(base + lay.cm);
  float* cl = reinterpret_cast<float*>(base + lay.cl);
  uint64_t* bar_s = reinterpret_cast<uint64_t*>(base + lay.bars);
  uint64_t* bar_o = bar_s + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_s + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q4 = warp & 3, cg = warp >> 2;
  const int row = q4 * 32 + lane;
  // unit order: (g, layer group, b, split), split fastest
  int u = blockIdx.x;
  const int split = u % p.nsplit;
  u /= p.nsplit;
  const int b = u % p.B;
  u /= p.B;
  const int lgrp = u % p.nlg;
  const int g = u / p.nlg;
  const int cnt = max(0, min(p.count[b], p.k));
  const int t0 = split * p.chunk;
  const int ntok = max(0, min(cnt, t0 + p.chunk) - t0);  // tokens of this split
  const int nch = (ntok + kTok - 1) / kTok;

  if (warp == 0) {
    tc::tmem_alloc(tmem_slot, kTmemCols);
    tc::tmem_relinquish();
  }
  if (threadIdx.x == 0) {
    mbar_init(bar_s, 1);
    mbar_init(bar_o, 1);
    fence_mbar_init();
  }
  // the split's token rows (coalesced), checked once
  for (int i = threadIdx.x; i < ntok; i += kThreadsTC) {
    const int tk = p.idx ? __ldg(p.idx + (size_t)b * p.k + t0 + i) : t0 + i;
    if ((unsigned)tk >= (unsigned)p.n_max)
      record_error(p.ws_header, CLSA_ERR_BAD_INDEX, ((long long)b << 32) | (unsigned)(t0 + i));
    stok[i] = (unsigned)tk < (unsigned)p.n_max ? tk : -1;
  }
  // Q rows of this unit: row r = (layer lgrp * Lg + r / G, head g * G + r % G)
  const int rows8 = (p.rows + 7) & ~7;
  for (int v = threadIdx.x; v < rows8 * 16; v += kThreadsTC) {
    const int r = v >> 4, c = v & 15;
    unsigned char* dst = sQ + (c >> 3) * lay.q_atom + tc::sw128_offset(r, c & 7);
    const int l = lgrp * p.Lg + r / p.G;
    if (r < p.rows && l < p.L) {
      const int h = g * p.G + r % p.G;
      cp_async_16(dst, p.Q + (((size_t)l * p.B + b) * p.Hq + h) * kD + c * 8, 16);
    } else {
      *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
    }
  }
  cp_async_commit();
  tc::fence_before_sync();
  __syncthreads();  // tokens visible; TMEM address and barriers ready
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  // the gather: thread x copies 16-byte column j = x % 16 of chunk rows x / 16 + 16 i
  // (i = 0..3); the swizzled destinations of those rows are 2 KiB apart
  const int gj = threadIdx.x & 15, gr0 = threadIdx.x >> 4;
  const uint32_t go0 = (uint32_t)(gj >> 3) * kKVAtom + tc::sw128_offset(gr0, gj & 7);
  const size_t gstride = (size_t)p.Hkv * kD;
  const size_t gcol = (size_t)b * (size_t)p.kv_bstride * gstride + (size_t)g * kD + gj * 8;
  auto load_chunk = [&](int c) {  // chunk c into stage c % 2
    unsigned char* dk = kv + (c & 1) * kStageBytes + go0;
    unsigned char* dv = dk + kKVTile;
#pragma unroll
    for (int it = 0; it < kTok / 16; ++it) {
      const int i = c * kTok + gr0 + 16 * it;
      const int tk = i < ntok ? stok[i] : -1;
      const bool ok = tk >= 0;
      const size_t off = ok ? gcol + (size_t)tk * gstride : 0;
      cp_async_16(dk + 2048 * it, p.K + off, ok ? 16 : 0);
      cp_async_16(dv + 2048 * it, p.V + off, ok ? 16 : 0);
    }
  };
  auto issue_qk = [&](int c) {  // S of chunk c into TMEM columns [64 (c & 1), +64)
    const uint32_t kb = smem_u32(kv + (c & 1) * kStageBytes);
#pragma unroll
    for (int ks = 0; ks < kD / 16; ++ks)
      tc::mma_bf16(tmem + (uint32_t)(kTok * (c & 1)), tc::sw128_desc(smem_u32(sQ) + (ks >> 2) * lay.q_atom + (ks & 3) * 32),
                   tc::sw128_desc(kb + (ks >> 2) * kKVAtom + (ks & 3) * 32), kIdescQK, ks > 0);
    tc::mma_commit(bar_s);
  };

  if (nch > 0) load_chunk(0);
  cp_async_commit();
  if (nch > 1) load_chunk(1);
  cp_async_commit();

  const uint32_t tl = tmem + ((uint32_t)(q4 * 32) << 16);
  const uint32_t to = tl + 128u + (uint32_t)(kOpt * cg);  // this thread's 64 output columns in TMEM
  const bool live = q4 * 32 < p.rows;  // warp-uniform
  // P is taken against a reference max m that moves only when a chunk's row max exceeds it
  // by more than 2^kTau: then the TMEM output and the row sum are scaled by 2^(m_old - m_new)
  // once (rare after the first chunks); P stays below 2^kTau, well inside bf16 and fp32.
  constexpr float kTau = 8.f;
  float m = -INFINITY, lp = 0.f;
  bool dead = false;
  if (nch > 0) {
    cp_async_wait<1>();  // Q and chunk 0 landed
    fence_proxy_async_smem();
    tc::fence_before_sync();
    __syncthreads();
    if (threadIdx.x == 0) {
      tc::fence_after_sync();
      issue_qk(0);
    }
  }

#pragma unroll 1
  for (int c = 0; c < nch; ++c) {
    const uint32_t ph = (uint32_t)c & 1u;
    if (!dead && !mbar_wait_warp(bar_s, ph)) {
      if (lane == 0) record_error(p.ws_header, CLSA_ERR_TIMEOUT, 40);
      dead = true;
    }
    tc::fence_after_sync();
    const uint32_t ts = tl + (uint32_t)(kTok * (c & 1) + kNpt * cg);
    const int nv = ntok - (c * kTok + kNpt * cg);  // valid columns of this thread
    const bool full = nv >= kNpt;  // warp-uniform: every column of this thread is a token
    uint32_t v[kNpt];  // the scores, held until P is final
    float lmx = -INFINITY;  // this thread's max of its columns (log2 units)
    if (live) {
      if (!dead) {
        tc::ld_32x32b_x32(ts, v);
        tc::ld_wait();
        float cmx = -INFINITY;
        if (full) {
#pragma unroll
          for (int j = 0; j < kNpt; j += 2) cmx = fmaxf(cmx, fmaxf(__uint_as_float(v[j]), __uint_as_float(v[j + 1])));
        } else {
#pragma unroll
          for (int j = 0; j < kNpt; ++j)
            if (j < nv) cmx = fmaxf(cmx, __uint_as_float(v[j]));
        }
        lmx = cmx * p.scale_log2;  // scale > 0: the max commutes
      } else {
#pragma unroll
        for (int j = 0; j < kNpt; ++j) v[j] = 0xff800000u;  // -inf: P = 0
      }
    }
    const int lim = full ? kNpt : nv;  // columns at or past lim are not tokens: P = 0
    // P of this thread's columns against the row's reference max m, into shared memory; the
    // row sum of those columns is returned
    auto write_p = [&]() -> float {
      float rs = 0.f;
#pragma unroll
      for (int q = 0; q < kNpt / 8; ++q) {
        uint32_t pw[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int j0 = 8 * q + 2 * j;
          float a = fast_exp2(fmaf(__uint_as_float(v[j0]), p.scale_log2, -m));
          float e = fast_exp2(fmaf(__uint_as_float(v[j0 + 1]), p.scale_log2, -m));
          if (!full) {
            a = j0 < lim ? a : 0.f;
            e = j0 + 1 < lim ? e : 0.f;
          }
          rs += a + e;
          pw[j] = pack_bf16x2(a, e);
        }
        // P holds only the rows8 stored rows (the next region follows): no row past them
        if (row < rows8)
          *reinterpret_cast<uint4*>(sP + tc::sw128_offset(row, (kNpt * cg) / 8 + q)) = make_uint4(pw[0], pw[1], pw[2], pw[3]);
      }
      return rs;
    };
    // Common case: no column of the thread lies more than 2^kTau above its row's reference max,
    // and P goes out against that max with no exchange.  The first chunk (no max yet) and a
    // column above the bound anywhere in the CTA take the exchange below (both threads of a row
    // then agree on the row's new max and rewrite their P); the vote rides on the barrier that
    // precedes the MMA issue anyway.
    const bool need = live && (c == 0 || lmx > m + kTau);
    float rs = 0.f;
    if (live && !need) rs = write_p();
    if (c + 1 < nch) cp_async_wait<0>();  // chunk c + 1 landed
    fence_proxy_async_smem();
    tc::fence_before_sync();
    if (__syncthreads_or(need)) {
      if (live) cm[cg * kM + row] = lmx;
      __syncthreads();
      if (live) {
        const float mn = fmaxf(cm[row], cm[kM + row]);
        const bool up = c == 0 || mn > m + kTau;  // the same in both threads of the row
        if (c > 0 && __any_sync(0xffffffffu, up)) {
          // TMEM load / store are .sync.aligned: every lane of the warp (alpha = 1 if not up)
          const float alpha = up ? fast_exp2(m - mn) : 1.f;
          if (!dead) {  // P V of the previous chunk has completed (waited below)
#pragma unroll 1
            for (int h2 = 0; h2 < 2; ++h2) {
              uint32_t w[32];
              tc::ld_32x32b_x32(to + (uint32_t)(32 * h2), w);
              tc::ld_wait();
#pragma unroll
              for (int j = 0; j < 32; ++j) w[j] = __float_as_uint(__uint_as_float(w[j]) * alpha);
              tc::st_32x32b_x32(to + (uint32_t)(32 * h2), w);
            }
            tc::st_wait();
          }
          if (up) lp *= alpha;
        }
        if (up) {
          m = mn;
          rs = write_p();
        }
      }
      fence_proxy_async_smem();
      tc::fence_before_sync();
      __syncthreads();
    }
    lp += rs;
    if (threadIdx.x == 0) {
      tc::fence_after_sync();
      const uint32_t vb = smem_u32(kv + (c & 1) * kStageBytes + kKVTile);
#pragma unroll
      for (int ks = 0; ks < kTok / 16; ++ks)
        tc::mma_bf16(tmem + 128u, tc::sw128_desc(smem_u32(sP) + ks * 32), tc::sw128_desc_mn(vb + ks * 16 * 128, kKVAtom),
                     kIdescPV, c > 0 || ks > 0);
      tc::mma_commit(bar_o);
      if (c + 1 < nch) issue_qk(c + 1);
    }
    // P V of this chunk completes before P, this K/V stage and (on a rescale) the output are reused
    if (!dead && !mbar_wait_warp(bar_o, ph)) {
      if (lane == 0) record_error(p.ws_header, CLSA_ERR_TIMEOUT, 41);
      dead = true;
    }
    tc::fence_after_sync();
    // chunk c + 2 into this chunk's stage: its S and P V MMAs have completed
    if (c + 2 < nch) load_chunk(c + 2);
    cp_async_commit();
  }
  cp_async_wait<0>();

  // row sum over the two column groups, then the output rows from TMEM
  cl[cg * kM + row] = lp;
  __syncthreads();
  const float ls = cl[row] + cl[kM + row];
  const int l = lgrp * p.Lg + row / p.G;
  const bool mine = row < p.rows && l < p.L;  // this lane's row is an output row
  const bool has = nch > 0 && !dead;          // warp-uniform; else an empty result
  // the TMEM loads are .sync.aligned: every lane of a live warp runs them, only `mine` stores
  if (live) {
    const int h = g * p.G + row % p.G;
    if (p.nsplit == 1) {
      uint4* out = reinterpret_cast<uint4*>(p.O + (((size_t)l * p.B + b) * p.Hq + h) * kD + kOpt * cg);
      if (has) {
        const float inv = ls > 0.f ? 1.f / ls : 0.f;
#pragma unroll 1
        for (int h2 = 0; h2 < 2; ++h2) {
          uint32_t w[32];
          tc::ld_32x32b_x32(to + (uint32_t)(32 * h2), w);
          tc::ld_wait();
          if (mine) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const float* f = reinterpret_cast<const float*>(w) + 8 * j;
              out[4 * h2 + j] = make_uint4(pack_bf16x2(f[0] * inv, f[1] * inv), pack_bf16x2(f[2] * inv, f[3] * inv),
                                           pack_bf16x2(f[4] * inv, f[5] * inv), pack_bf16x2(f[6] * inv, f[7] * inv));
            }
          }
        }
      } else if (mine) {
#pragma unroll
        for (int j = 0; j < kOpt / 8; ++j) out[j] = make_uint4(0u, 0u, 0u, 0u);
      }
      if (mine && p.lse && cg == 0)
        p.lse[((size_t)l * p.B + b) * p.Hq + h] = has && ls > 0.f ? (m + log2f(ls)) * kLn2 : -INFINITY;
    } else {
      const size_t pi = ((((size_t)b * p.Hkv + g) * p.nlg + lgrp) * p.nsplit + split) * p.rows + row;
      float4* op = reinterpret_cast<float4*>(p.Op + pi * kD + kOpt * cg);
      if (has) {
#pragma unroll 1
        for (int h2 = 0; h2 < 2; ++h2) {
          uint32_t w[32];
          tc::ld_32x32b_x32(to + (uint32_t)(32 * h2), w);
          tc::ld_wait();
          if (mine) {
#pragma unroll
            for (int j = 0; j < 8; ++j)
              op[8 * h2 + j] = make_float4(__uint_as_float(w[4 * j]), __uint_as_float(w[4 * j + 1]),
                                           __uint_as_float(w[4 * j + 2]), __uint_as_float(w[4 * j + 3]));
          }
        }
      } else if (mine) {
#pragma unroll
        for (int j = 0; j < kOpt / 4; ++j) op[j] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
      if (mine && cg == 0) {
        p.Mp[pi] = has ? m : -INFINITY;
        p.Lp[pi] = has ? ls : 0.f;
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tmem, kTmemCols);
}

bool aligned16(const void* a) { return reinterpret_cast<uintptr_t>(a) % 16 == 0; }

cudaError_t launch_tc(const TCParams& p, cudaStream_t s) {
  const TCLayout lay = tc_layout(p.rows, p.chunk);
  const int smem = (int)lay.total + 1024;  // + alignment of the carve-up base
  cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const long long units = (long long)p.Hkv * p.nlg * p.B * p.nsplit;
  e = launch_pdl(attn_tc_kernel, dim3((unsigned)units), dim3(kThreadsTC), (size_t)smem, s, p);
  launches_add(1, s);
  return e;
}

}  // namespace

// ----- clsa_sparse_attn / the unfused decode step -------------------------------------
bool sparse_attn_tc_supported(const AttnShape& sh, const AttnPlan& pl, const void* Q, const void* K, const void* V,
                              const void* O) {
  if (sh.dt != CLSA_BF16 || sh.d != kD || sh.Hq % sh.Hkv != 0 || pl.rows > kM) return false;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O)) return false;
  return (int)tc_layout(pl.rows, pl.chunk).total + 1024 <= device_info().max_smem_optin;
}

cudaError_t launch_sparse_attn_tc(const AttnShape& sh, const AttnPlan& pl, const void* Q, const void* Kc,
                                  const void* Vc, const int32_t* idx, const int32_t* count, float scale_log2, void* O,
                                  float* lse, float* Op, float* Mp, float* Lp, void* ws_header, cudaStream_t s) {
  TCParams p{};
  p.Q = static_cast<const __nv_bfloat16*>(Q);
  p.K = static_cast<const __nv_bfloat16*>(Kc);
  p.V = static_cast<const __nv_bfloat16*>(Vc);
  p.count = count;
  p.O = static_cast<__nv_bfloat16*>(O);
  p.lse = lse;
  p.Op = Op;
  p.Mp = Mp;
  p.Lp = Lp;
  p.ws_header = ws_header;
  if (sh.gather) {  // rows come from the full cache through the index list
    p.idx = idx;
    p.n_max = sh.n_max;
    p.kv_bstride = sh.kv_bstride;
  } else {  // compact [B][k][Hkv][d]: position i of sequence b is row b * k + i
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
  p.Lg = pl.Lg;
  p.nlg = pl.nlg;
  p.rows = pl.rows;
  p.nsplit = pl.nsplit;
  p.chunk = pl.chunk;
  p.scale_log2 = scale_log2;
  return launch_tc(p, s);
}

// ----- prefill: one unit per (KV head, layer group, new row t), no split -----------------
bool prefill_attn_tc_supported(const clsa_prefill_args* a) {
  if (a->dtype != CLSA_BF16 || a->d != kD || a->Hq % a->Hkv != 0) return false;
  if (!aligned16(a->Q) || !aligned16(a->K) || !aligned16(a->V) || !aligned16(a->O)) return false;
  const int G = a->Hq / a->Hkv;
  if (G > kM) return false;
  const int Lg = std::max(1, std::min(a->L, kM / G));
  return (int)tc_layout(Lg * G, a->k).total + 1024 <= device_info().max_smem_optin;
}

cudaError_t launch_prefill_attn_tc(const clsa_prefill_args* a, float scale, void* ws_header, cudaStream_t s) {
  TCParams p{};
  p.Q = static_cast<const __nv_bfloat16*>(a->Q);
  p.K = static_cast<const __nv_bfloat16*>(a->K);
  p.V = static_cast<const __nv_bfloat16*>(a->V);
  p.idx = a->idx;
  p.count = a->count;
  p.O = static_cast<__nv_bfloat16*>(a->O);
  p.lse = a->lse;
  p.ws_header = ws_header;
  p.kv_bstride = 0;  // every row reads the one shared cache
  p.B = a->T;
  p.k = a->k;
  p.L = a->L;
  p.Hq = a->Hq;
  p.Hkv = a->Hkv;
  p.G = a->Hq / a->Hkv;
  p.Lg = std::max(1, std::min(a->L, kM / p.G));
  p.nlg = (a->L + p.Lg - 1) / p.Lg;
  p.Lg = (a->L + p.nlg - 1) / p.nlg;  // balanced layer groups
  p.rows = p.Lg * p.G;
  p.n_max = a->n;
  p.nsplit = 1;
  p.chunk = a->k;
  p.scale_log2 = scale * 1.4426950408889634f;
  return launch_tc(p, s);
}

}  // namespace clsa
