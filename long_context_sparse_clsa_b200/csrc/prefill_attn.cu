// Prefill sparse attention on the 5th-generation tensor cores.
//
// Per-layer equation for every new row t and layer l (picx.dev CLSA summary,
// Methodology > Architecture Overview; each prefill row attends over its own S_t):
//   O^(l)[t, h] = softmax(Q^(l)[t, h] K_{S_t}^T * scale) V_{S_t},   S_t = idx[t][0..count[t])
// with query head h reading KV head h / G of the one shared cache.
//
// One CTA per unit (KV head g, layer group, row t); units run head-major, so the CTAs in
// flight share one head's K/V rows (64 MiB at n = 128K) in L2.  The unit's M rows are the
// (layer, query head) pairs of head g at row t (L*G = 96 at the benchmark shape), the A
// operand for every chunk; row t's selected tokens go in chunks of 64:
//   S = Q K_c^T      tcgen05.mma M128 N64 (K = d, 8 steps) -> TMEM, double-buffered
//   softmax          8 warps: one row (TMEM lane) and 32 of the chunk's columns per
//                    thread; the chunk's row max is exchanged through shared memory
//   O_c = P_c V_c    P_c bf16 in shared memory (A, K-major), V_c as the MN-major B operand
//                    from its row-major [token][d] tile: M128 N128 (K = 64) -> TMEM
//   o = o 2^(m_old - m) + O_c   in registers, 64 of the d columns per thread
// The S MMAs of chunk c + 1 go out right behind P V of chunk c.  K/V chunks are gathered
// by 16-byte async copies into the 128-byte-swizzle layout, one chunk ahead (2 stages).
// About 111 KiB of shared memory and 256 TMEM columns per CTA: two CTAs share an SM, so
// one CTA's softmax overlaps the other's MMAs and gathers.  A unit has no split: its
// output rows are final (no partials, no combine).
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
constexpr int kThreadsPA = kW * 32;
constexpr int kTok = 64;                            // tokens per chunk
constexpr int kD = 128;                             // head dim
constexpr int kM = 128;                             // MMA rows
constexpr int kNpt = kTok / 2;                      // S columns per thread
constexpr int kOpt = kD / 2;                        // output columns per thread
constexpr uint32_t kKVAtom = kTok * 128;            // 64 rows x 128 bytes
constexpr uint32_t kKVTile = 2 * kKVAtom;           // K or V chunk: both 64-column atoms
constexpr uint32_t kStageBytes = 2 * kKVTile;       // K and V
constexpr uint32_t kTmemCols = 256;                 // S at [0, 128) (two buffers), O_c at [128, 256)
constexpr uint32_t kIdescQK = tc::idesc_bf16_f32(kM, kTok);
constexpr uint32_t kIdescPV = tc::idesc_bf16_f32(kM, kD) | (1u << 16);  // B (V) MN-major

static_assert(kThreadsPA == 256 && kTok == 64, "the gather maps 256 threads onto 64 rows x 16 columns");

struct PAParams {
  const __nv_bfloat16* Q;   // [L][T][Hq][d]
  const __nv_bfloat16* K;   // [n][Hkv][d]
  const __nv_bfloat16* V;
  const int32_t* idx;       // [T][k]
  const int32_t* count;     // [T]
  __nv_bfloat16* O;         // [L][T][Hq][d]
  float* lse;               // [L][T][Hq] or null
  void* ws_header;
  int T, k, L, Hq, Hkv, G, Lg, nlg, rows, n;
  float scale_log2;
};

// shared-memory carve-up (offsets from a 1024-aligned base)
struct PALayout {
  uint32_t q_atom, q, kv, p, tok, cm, cl, bars, total;
};
__host__ __device__ inline PALayout pa_layout(int rows, int k) {
  PALayout s;
  const uint32_t rows8 = (uint32_t)((rows + 7) & ~7);
  s.q_atom = rows8 * 128;                        // one 64-column atom of the rows that exist
  s.q = 0;
  s.kv = 2 * s.q_atom;                           // [2 stages][K, V]
  s.p = s.kv + 2 * kStageBytes;                  // P: rows8 x 64 tokens
  s.tok = s.p + s.q_atom;                        // [k] row t's selected tokens
  s.cm = s.tok + (uint32_t)(((k * 4) + 15) & ~15);  // [2][128] row-max exchange
  s.cl = s.cm + 2 * kM * 4;                      // [2][128] row-sum exchange
  s.bars = s.cl + 2 * kM * 4;                    // bar_s, bar_o, tmem address
  s.total = s.bars + 32;
  // the MMAs read 128-row tiles: keep the reads past Q atom 1 and past P inside the carve-up
  const uint32_t tail = s.p + (uint32_t)kM * 128 + 128;  // + the K-step offset of the last read
  if (s.total < tail) s.total = tail;
  return s;
}

__global__ void __launch_bounds__(kThreadsPA, 2) prefill_attn_tc_kernel(const PAParams p) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const PALayout lay = pa_layout(p.rows, p.k);
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
  const int u = blockIdx.x;
  const int g = u / (p.nlg * p.T);
  const int rem = u % (p.nlg * p.T);
  const int lgrp = rem / p.T, t = rem % p.T;
  const int cnt = max(0, min(p.count[t], p.k));
  const int nch = (cnt + kTok - 1) / kTok;

  if (warp == 0) {
    tc::tmem_alloc(tmem_slot, kTmemCols);
    tc::tmem_relinquish();
  }
  if (threadIdx.x == 0) {
    mbar_init(bar_s, 1);
    mbar_init(bar_o, 1);
    fence_mbar_init();
  }
  // row t's selection (coalesced), checked once
  for (int i = threadIdx.x; i < cnt; i += kThreadsPA) {
    const int tk = __ldg(p.idx + (size_t)t * p.k + i);
    if ((unsigned)tk >= (unsigned)p.n) record_error(p.ws_header, CLSA_ERR_BAD_INDEX, ((long long)t << 32) | (unsigned)i);
    stok[i] = (unsigned)tk < (unsigned)p.n ? tk : -1;
  }
  // Q rows of this unit: row r = (layer lgrp * Lg + r / G, head g * G + r % G)
  const int rows8 = (p.rows + 7) & ~7;
  for (int v = threadIdx.x; v < rows8 * 16; v += kThreadsPA) {
    const int r = v >> 4, c = v & 15;
    unsigned char* dst = sQ + (c >> 3) * lay.q_atom + tc::sw128_offset(r, c & 7);
    const int l = lgrp * p.Lg + r / p.G;
    if (r < p.rows && l < p.L) {
      const int h = g * p.G + r % p.G;
      cp_async_16(dst, p.Q + (((size_t)l * p.T + t) * p.Hq + h) * kD + c * 8, 16);
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
  const size_t gcol = (size_t)g * kD + gj * 8;
  const size_t gstride = (size_t)p.Hkv * kD;
  auto load_chunk = [&](int c) {  // chunk c into stage c % 2
    unsigned char* dk = kv + (c & 1) * kStageBytes + go0;
    unsigned char* dv = dk + kKVTile;
#pragma unroll
    for (int it = 0; it < kTok / 16; ++it) {
      const int i = c * kTok + gr0 + 16 * it;
      const int tk = i < cnt ? stok[i] : -1;
      const bool ok = (unsigned)tk < (unsigned)p.n;
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
  const bool live = q4 * 32 < p.rows;  // warp-uniform
  float o[kOpt];
#pragma unroll
  for (int j = 0; j < kOpt; ++j) o[j] = 0.f;
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
    const int nv = cnt - (c * kTok + kNpt * cg);  // valid columns of this thread
    const bool full = nv >= kNpt;  // warp-uniform: every column of this thread is a token
    if (live) {
      float cmx = -INFINITY;
      if (!dead) {
        uint32_t v[kNpt];
        tc::ld_32x32b_x32(ts, v);
        tc::ld_wait();
        if (full) {
#pragma unroll
          for (int j = 0; j < kNpt; j += 2) cmx = fmaxf(cmx, fmaxf(__uint_as_float(v[j]), __uint_as_float(v[j + 1])));
        } else {
#pragma unroll
          for (int j = 0; j < kNpt; ++j)
            if (j < nv) cmx = fmaxf(cmx, __uint_as_float(v[j]));
        }
      }
      cm[cg * kM + row] = cmx * p.scale_log2;  // scale > 0: the max commutes
    }
    __syncthreads();
    float alpha = 1.f;
    if (live) {
      const float mn = fmaxf(m, fmaxf(cm[row], cm[kM + row]));
      alpha = fast_exp2(m - mn);  // m = -inf on the first chunk: 0
      m = mn;
      uint32_t v[kNpt];
      if (!dead) {
        tc::ld_32x32b_x32(ts, v);
        tc::ld_wait();
      } else {
#pragma unroll
        for (int j = 0; j < kNpt; ++j) v[j] = 0xff800000u;
      }
      float rs = 0.f;
      const int lim = full ? kNpt : nv;  // columns at or past lim are not tokens: P = 0
#pragma unroll
      for (int q = 0; q < kNpt / 8; ++q) {
        uint32_t pw[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int j0 = 8 * q + 2 * j;
          float a = fast_exp2(fmaf(__uint_as_float(v[j0]), p.scale_log2, -mn));
          float e = fast_exp2(fmaf(__uint_as_float(v[j0 + 1]), p.scale_log2, -mn));
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
      lp = lp * alpha + rs;
    }
    if (c + 1 < nch) cp_async_wait<0>();  // chunk c + 1 landed
    fence_proxy_async_smem();
    tc::fence_before_sync();
    __syncthreads();
    if (threadIdx.x == 0) {
      tc::fence_after_sync();
      const uint32_t vb = smem_u32(kv + (c & 1) * kStageBytes + kKVTile);
#pragma unroll
      for (int ks = 0; ks < kTok / 16; ++ks)
        tc::mma_bf16(tmem + 128u, tc::sw128_desc(smem_u32(sP) + ks * 32), tc::sw128_desc_mn(vb + ks * 16 * 128, kKVAtom),
                     kIdescPV, ks > 0);
      tc::mma_commit(bar_o);
      if (c + 1 < nch) issue_qk(c + 1);
    }
    if (!dead && !mbar_wait_warp(bar_o, ph)) {
      if (lane == 0) record_error(p.ws_header, CLSA_ERR_TIMEOUT, 41);
      dead = true;
    }
    tc::fence_after_sync();
    if (live && !dead) {
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        uint32_t v[32];
        tc::ld_32x32b_x32(tl + 128u + (uint32_t)(kOpt * cg + 32 * h2), v);
        tc::ld_wait();
#pragma unroll
        for (int j = 0; j < 32; ++j) o[32 * h2 + j] = fmaf(o[32 * h2 + j], alpha, __uint_as_float(v[j]));
      }
    }
    tc::fence_before_sync();  // O_c is read before the next P V overwrites it
    // chunk c + 2 into this chunk's stage: its S and P V MMAs have completed
    if (c + 2 < nch) load_chunk(c + 2);
    cp_async_commit();
  }
  cp_async_wait<0>();

  // row sum over the two column groups, then the output rows
  cl[cg * kM + row] = lp;
  __syncthreads();
  const float ls = cl[row] + cl[kM + row];
  if (row < p.rows) {
    const int l = lgrp * p.Lg + row / p.G;
    if (l < p.L) {
      const int h = g * p.G + row % p.G;
      const float inv = ls > 0.f ? 1.f / ls : 0.f;
      uint4* out = reinterpret_cast<uint4*>(p.O + (((size_t)l * p.T + t) * p.Hq + h) * kD + kOpt * cg);
#pragma unroll
      for (int j = 0; j < kOpt / 8; ++j)
        out[j] = make_uint4(pack_bf16x2(o[8 * j] * inv, o[8 * j + 1] * inv), pack_bf16x2(o[8 * j + 2] * inv, o[8 * j + 3] * inv),
                            pack_bf16x2(o[8 * j + 4] * inv, o[8 * j + 5] * inv), pack_bf16x2(o[8 * j + 6] * inv, o[8 * j + 7] * inv));
      if (p.lse && cg == 0) p.lse[((size_t)l * p.T + t) * p.Hq + h] = ls > 0.f ? (m + log2f(ls)) * 0.6931471805599453f : -INFINITY;
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tmem, kTmemCols);
}

}  // namespace

bool prefill_attn_tc_supported(const clsa_prefill_args* a) {
  if (a->dtype != CLSA_BF16 || a->d != kD || a->Hq % a->Hkv != 0) return false;
  if ((reinterpret_cast<uintptr_t>(a->Q) | reinterpret_cast<uintptr_t>(a->K) | reinterpret_cast<uintptr_t>(a->V) |
       reinterpret_cast<uintptr_t>(a->O)) % 16 != 0)
    return false;
  const int G = a->Hq / a->Hkv;
  if (G > kM) return false;
  const int Lg = std::max(1, std::min(a->L, kM / G));
  const PALayout lay = pa_layout(Lg * G, a->k);
  return (int)lay.total + 1024 <= device_info().max_smem_optin;
}

cudaError_t launch_prefill_attn_tc(const clsa_prefill_args* a, float scale, void* ws_header, cudaStream_t s) {
  PAParams p{};
  p.Q = static_cast<const __nv_bfloat16*>(a->Q);
  p.K = static_cast<const __nv_bfloat16*>(a->K);
  p.V = static_cast<const __nv_bfloat16*>(a->V);
  p.idx = a->idx;
  p.count = a->count;
  p.O = static_cast<__nv_bfloat16*>(a->O);
  p.lse = a->lse;
  p.ws_header = ws_header;
  p.T = a->T;
  p.k = a->k;
  p.L = a->L;
  p.Hq = a->Hq;
  p.Hkv = a->Hkv;
  p.G = a->Hq / a->Hkv;
  p.Lg = std::max(1, std::min(a->L, kM / p.G));
  p.nlg = (a->L + p.Lg - 1) / p.Lg;
  p.Lg = (a->L + p.nlg - 1) / p.nlg;  // balanced layer groups
  p.rows = p.Lg * p.G;
  p.n = a->n;
  p.scale_log2 = scale * 1.4426950408889634f;
  const PALayout lay = pa_layout(p.rows, p.k);
  const int smem = (int)lay.total + 1024;  // + alignment of the carve-up base
  cudaError_t e = cudaFuncSetAttribute(prefill_attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const long long units = (long long)a->Hkv * p.nlg * a->T;
  prefill_attn_tc_kernel<<<(unsigned)units, kThreadsPA, smem, s>>>(p);
  launches_add(1, s);
  return cudaGetLastError();
}

}  // namespace clsa
