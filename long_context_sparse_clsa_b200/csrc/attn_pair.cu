// Key-centric prefill attention: two new rows per CTA, over the union of their selections.
//
// Per-layer equation for rows t and t' of a prefill chunk (picx.dev CLSA summary,
// Methodology > Architecture Overview; each row attends over its own S_t):
//   O^(l)[t, h] = softmax(Q^(l)[t, h] K_{S_t}^T * scale) V_{S_t}
// Neighbouring rows of a chunk often select many of the same tokens.  Here a CTA owns a pair
// of rows (t, t + 1) for one KV head and layer group, builds U = S_t U S_t+1 (S_t's tokens,
// then those of S_t+1 that S_t lacks), and streams U through shared memory once: each K/V
// row of U is fetched once for both rows.  Each row keeps its own 128-row tile (its (layer,
// query head) pairs, 96 at 24 layers x 4 heads): per 64-token chunk of U,
//   S_x = Q_x K_c^T   (tcgen05, both tiles against the same K chunk)
//   softmax_x         over the columns of U that row x selected (a membership bit per column)
//   O_x += P_x V_c    (accumulated in TMEM, lazy rescale as in the per-row kernel)
// so a tile's work grows with |U| / |S_x| while the gather shrinks with |S_t| + |S_t+1| over
// |U|.  It pays only when the tiles' softmax is not what bounds the kernel; the per-row
// kernel (attn_tc.cu) stays the default and this one is an option of the attention entry.
// One CTA per SM: 16 warps (8 per tile), 512 TMEM columns, ~160 KiB of shared memory.
// Every wait is bounded (kWaitLimitNs).
#include <algorithm>
#include <cmath>

#include "common.cuh"
#include "kernels.h"
#include "tcgen05.cuh"

namespace clsa {

namespace {

constexpr int kTiles = 2;
constexpr int kWarpsPerTile = 8;                    // 4 lane quarters x 2 column groups
constexpr int kThreadsKP = kTiles * kWarpsPerTile * 32;
constexpr int kTok = 64;                            // union tokens per chunk
constexpr int kD = 128;
constexpr int kM = 128;
constexpr int kNpt = kTok / 2;                      // S columns per thread
constexpr int kOpt = kD / 2;                        // output columns per thread
constexpr uint32_t kKVAtom = kTok * 128;
constexpr uint32_t kKVTile = 2 * kKVAtom;
constexpr uint32_t kStageBytes = 2 * kKVTile;
constexpr uint32_t kTmemCols = 512;                 // tile x: S [256x, +128) (two buffers), O [256x + 128, +128)
constexpr uint32_t kIdescQK = tc::idesc_bf16_f32(kM, kTok);
constexpr uint32_t kIdescPV = tc::idesc_bf16_f32(kM, kD) | (1u << 16);  // B (V) MN-major
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kTau = 8.f;

static_assert(kThreadsKP == 512 && kTok == 64, "the gather maps 512 threads onto 64 rows x 16 columns, twice");

struct KPParams {
  const __nv_bfloat16* Q;   // [L][T][Hq][d]
  const __nv_bfloat16* K;   // [n][Hkv][d]
  const __nv_bfloat16* V;
  const int32_t* idx;       // [T][k], ascending token order per row
  const int32_t* count;     // [T]
  __nv_bfloat16* O;         // [L][T][Hq][d]
  float* lse;               // [L][T][Hq] or null
  void* ws_header;
  int T, k, L, Hq, Hkv, G, Lg, nlg, rows, n, npairs;
  float scale_log2;
};

// membership words per tile: two per 64-token chunk of a union of up to 2k tokens
__host__ __device__ inline int kp_mask_words(int k) { return (2 * k + kTok - 1) / kTok * 2; }

struct KPLayout {
  uint32_t q_atom, q, kv, p, u, mask, cm, cl, bars, total;
};
__host__ __device__ inline KPLayout kp_layout(int rows, int k) {
  KPLayout s;
  const uint32_t rows8 = (uint32_t)((rows + 7) & ~7);
  s.q_atom = rows8 * 128;
  s.q = 0;                                      // tile x: two atoms at q + 2 x q_atom
  s.kv = 4 * s.q_atom;                          // [2 stages][K, V]; the union build's scratch first
  s.p = s.kv + 2 * kStageBytes;                 // tile x: P at p + x q_atom
  s.u = s.p + 2 * s.q_atom;                     // [2k] union tokens
  s.mask = s.u + (uint32_t)(2 * k * 4);         // [2 tiles][kp_mask_words(k)] membership words
  s.cm = s.mask + (uint32_t)(2 * kp_mask_words(k) * 4 + 15) / 16 * 16;  // [2 tiles][2][128]
  s.cl = s.cm + 2 * 2 * kM * 4;
  s.bars = s.cl + 2 * 2 * kM * 4;               // bar_s, bar_o, tmem slot, counts
  s.total = s.bars + 64;
  const uint32_t tail = s.p + s.q_atom + (uint32_t)kM * 128 + 128;  // tile 1's P read as a 128-row tile
  if (s.total < tail) s.total = tail;
  return s;
}

__device__ __forceinline__ bool bsearch_sorted(const int32_t* a, int n, int x) {
  int lo = 0, hi = n;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (a[mid] < x) lo = mid + 1;
    else hi = mid;
  }
  return lo < n && a[lo] == x;
}

__global__ void __launch_bounds__(kThreadsKP, 1) attn_pair_kernel(const KPParams p) {
  pdl_enter();
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const KPLayout lay = kp_layout(p.rows, p.k);
  unsigned char* kv = base + lay.kv;
  int32_t* su = reinterpret_cast<int32_t*>(base + lay.u);
  uint32_t* smask = reinterpret_cast<uint32_t*>(base + lay.mask);
  float* cm_all = reinterpret_cast<float*>(base + lay.cm);
  float* cl_all = reinterpret_cast<float*>(base + lay.cl);
  uint64_t* bar_s = reinterpret_cast<uint64_t*>(base + lay.bars);
  uint64_t* bar_o = bar_s + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_s + 2);
  int* s_nbonly = reinterpret_cast<int*>(bar_s + 3);
  const int mwords = kp_mask_words(p.k);  // membership words per tile

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int x = warp / kWarpsPerTile;      // tile: row t0 + x
  const int wt = warp % kWarpsPerTile;
  const int q4 = wt & 3, cg = wt >> 2;
  const int row = q4 * 32 + lane;
  // unit order: (g, layer group, pair), pair fastest
  int u = blockIdx.x;
  const int pair = u % p.npairs;
  u /= p.npairs;
  const int lgrp = u % p.nlg;
  const int g = u / p.nlg;
  const int t0 = 2 * pair;
  const bool has_b = t0 + 1 < p.T;
  const int cntA = max(0, min(p.count[t0], p.k));
  const int cntB = has_b ? max(0, min(p.count[t0 + 1], p.k)) : 0;

  if (warp == 0) {
    tc::tmem_alloc(tmem_slot, kTmemCols);
    tc::tmem_relinquish();
  }
  if (threadIdx.x == 0) {
    mbar_init(bar_s, 1);
    mbar_init(bar_o, 1);
    fence_mbar_init();
  }

  // ---- the union: S_t's tokens, then S_t+1's that S_t lacks (scratch in the K/V stages) ----
  int32_t* la = reinterpret_cast<int32_t*>(kv);
  int32_t* lb = la + p.k;
  uint8_t* in_b = reinterpret_cast<uint8_t*>(lb + p.k);  // [k] S_t's token i is in S_t+1
  uint8_t* b_only = in_b + p.k;                          // [k] S_t+1's token j is not in S_t
  int* wtot = reinterpret_cast<int*>(cm_all);            // block-scan warp totals (cm is free here)
  for (int i = threadIdx.x; i < cntA + cntB; i += kThreadsKP) {
    const bool a = i < cntA;
    const int r = a ? t0 : t0 + 1, j = a ? i : i - cntA;
    const int tk = __ldg(p.idx + (size_t)r * p.k + j);
    if ((unsigned)tk >= (unsigned)p.n) record_error(p.ws_header, CLSA_ERR_BAD_INDEX, ((long long)r << 32) | (unsigned)j);
    (a ? la : lb)[j] = (unsigned)tk < (unsigned)p.n ? tk : -1;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < cntA; i += kThreadsKP) in_b[i] = bsearch_sorted(lb, cntB, la[i]) ? 1 : 0;
  for (int j = threadIdx.x; j < cntB; j += kThreadsKP) b_only[j] = bsearch_sorted(la, cntA, lb[j]) ? 0 : 1;
  __syncthreads();
  {  // S_t+1's own tokens go after S_t's, in token order: contiguous runs + a block scan
    const int per = (cntB + kThreadsKP - 1) / kThreadsKP;
    const int j0 = threadIdx.x * per, j1 = min(cntB, j0 + per);
    int mine = 0;
    for (int j = j0; j < j1; ++j) mine += b_only[j];
    int incl = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) wtot[warp] = incl;
    __syncthreads();
    int before = 0;
    for (int w2 = 0; w2 < warp; ++w2) before += wtot[w2];
    int pos = cntA + before + incl - mine;
    for (int j = j0; j < j1; ++j)
      if (b_only[j]) su[pos++] = lb[j];
    if (threadIdx.x == kThreadsKP - 1) *s_nbonly = before + incl;
    for (int i = threadIdx.x; i < cntA; i += kThreadsKP) su[i] = la[i];
  }
  __syncthreads();
  const int nU = cntA + *s_nbonly;
  // membership words: tile 0 takes U[0, cntA); tile 1 takes the S_t tokens it shares and all of
  // U[cntA, nU)
  for (int w2 = threadIdx.x; w2 < 2 * mwords; w2 += kThreadsKP) {
    const int tile = w2 / mwords, w = w2 % mwords;
    uint32_t bits = 0u;
    for (int e = 0; e < 32; ++e) {
      const int i = 32 * w + e;
      const bool m = tile == 0 ? i < cntA : (i < cntA ? in_b[i] != 0 : i < nU);
      bits |= (m ? 1u : 0u) << e;
    }
    smask[w2] = bits;
  }

  // Q rows of both tiles: row r = (layer lgrp * Lg + r / G, head g * G + r % G)
  const int rows8 = (p.rows + 7) & ~7;
  for (int v = threadIdx.x; v < kTiles * rows8 * 16; v += kThreadsKP) {
    const int tile = v / (rows8 * 16), rv = v % (rows8 * 16);
    const int r = rv >> 4, c = rv & 15;
    unsigned char* dst = base + lay.q + (2 * tile + (c >> 3)) * lay.q_atom + tc::sw128_offset(r, c & 7);
    const int l = lgrp * p.Lg + r / p.G;
    const int t = t0 + tile;
    if (r < p.rows && l < p.L && t < p.T) {
      const int h = g * p.G + r % p.G;
      cp_async_16(dst, p.Q + (((size_t)l * p.T + t) * p.Hq + h) * kD + c * 8, 16);
    } else {
      *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
    }
  }
  cp_async_commit();
  tc::fence_before_sync();
  __syncthreads();  // union and masks visible (its scratch in the stages is dead); TMEM ready
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const int nch = (nU + kTok - 1) / kTok;

  // the gather: thread v copies 16-byte column j = v % 16 of chunk rows v / 16 + 32 i (i = 0, 1)
  const int gj = threadIdx.x & 15, gr0 = threadIdx.x >> 4;
  const uint32_t go0 = (uint32_t)(gj >> 3) * kKVAtom + tc::sw128_offset(gr0, gj & 7);
  const size_t gstride = (size_t)p.Hkv * kD;
  const size_t gcol = (size_t)g * kD + gj * 8;
  auto load_chunk = [&](int c) {  // chunk c of U into stage c % 2
    unsigned char* dk = kv + (c & 1) * kStageBytes + go0;
    unsigned char* dv = dk + kKVTile;
#pragma unroll
    for (int it = 0; it < 2; ++it) {
      const int i = c * kTok + gr0 + 32 * it;
      const int tk = i < nU ? su[i] : -1;
      const bool ok = tk >= 0;
      const size_t off = ok ? gcol + (size_t)tk * gstride : 0;
      cp_async_16(dk + 4096 * it, p.K + off, ok ? 16 : 0);  // 32 rows = 4 swizzle atoms further
      cp_async_16(dv + 4096 * it, p.V + off, ok ? 16 : 0);
    }
  };
  auto issue_qk = [&](int c) {  // S of chunk c for both tiles
    const uint32_t kb = smem_u32(kv + (c & 1) * kStageBytes);
#pragma unroll
    for (int tile = 0; tile < kTiles; ++tile) {
      const uint32_t qb = smem_u32(base + lay.q) + 2 * tile * lay.q_atom;
#pragma unroll
      for (int ks = 0; ks < kD / 16; ++ks)
        tc::mma_bf16(tmem + 256u * tile + (uint32_t)(kTok * (c & 1)),
                     tc::sw128_desc(qb + (ks >> 2) * lay.q_atom + (ks & 3) * 32),
                     tc::sw128_desc(kb + (ks >> 2) * kKVAtom + (ks & 3) * 32), kIdescQK, ks > 0);
    }
    tc::mma_commit(bar_s);
  };

  if (nch > 0) load_chunk(0);
  cp_async_commit();
  if (nch > 1) load_chunk(1);
  cp_async_commit();

  unsigned char* sP = base + lay.p + x * lay.q_atom;
  float* cm = cm_all + x * 2 * kM;
  float* cl = cl_all + x * 2 * kM;
  const uint32_t* mk = smask + x * mwords;
  const uint32_t tl = tmem + ((uint32_t)(q4 * 32) << 16) + 256u * x;
  const uint32_t to = tl + 128u + (uint32_t)(kOpt * cg);
  const bool live = q4 * 32 < p.rows && t0 + x < p.T;  // warp-uniform
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
      if (lane == 0) record_error(p.ws_header, CLSA_ERR_TIMEOUT, 50);
      dead = true;
    }
    tc::fence_after_sync();
    const uint32_t bits = mk[(c * kTok + kNpt * cg) >> 5];  // this thread's 32 columns of U
    uint32_t v[kNpt];
    float lmx = -INFINITY;
    if (live) {
      if (!dead) {
        tc::ld_32x32b_x32(tl + (uint32_t)(kTok * (c & 1) + kNpt * cg), v);
        tc::ld_wait();
        float cmx = -INFINITY;
#pragma unroll
        for (int j = 0; j < kNpt; ++j)
          if ((bits >> j) & 1u) cmx = fmaxf(cmx, __uint_as_float(v[j]));
        lmx = cmx * p.scale_log2;
      } else {
#pragma unroll
        for (int j = 0; j < kNpt; ++j) v[j] = 0xff800000u;
      }
    }
    auto write_p = [&]() -> float {
      float rs = 0.f;
#pragma unroll
      for (int q = 0; q < kNpt / 8; ++q) {
        uint32_t pw[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int j0 = 8 * q + 2 * j;
          const float a = (bits >> j0) & 1u ? fast_exp2(fmaf(__uint_as_float(v[j0]), p.scale_log2, -m)) : 0.f;
          const float e = (bits >> (j0 + 1)) & 1u ? fast_exp2(fmaf(__uint_as_float(v[j0 + 1]), p.scale_log2, -m)) : 0.f;
          rs += a + e;
          pw[j] = pack_bf16x2(a, e);
        }
        if (row < rows8)
          *reinterpret_cast<uint4*>(sP + tc::sw128_offset(row, (kNpt * cg) / 8 + q)) = make_uint4(pw[0], pw[1], pw[2], pw[3]);
      }
      return rs;
    };
    // as in the per-row kernel: P at once against the row's reference max unless a selected
    // column lies more than 2^kTau above it (or no max exists yet); the exchange is voted
    const bool need = live && (m == -INFINITY ? lmx != -INFINITY || c == 0 : lmx > m + kTau);
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
        const bool up = m == -INFINITY ? true : mn > m + kTau;  // the same in both threads of the row
        if (__any_sync(0xffffffffu, up && m != -INFINITY)) {
          // a row's first selected columns find O = 0 and lp = 0: nothing to rescale there
          const float alpha = up && m != -INFINITY ? fast_exp2(m - mn) : 1.f;
          if (!dead && c > 0) {  // P V of the previous chunk has completed (waited below)
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
          lp *= alpha;
        }
        if (up) {
          m = mn;  // stays -inf while the row has selected nothing yet: P = 0 below
          rs = m == -INFINITY ? 0.f : write_p();
          if (m == -INFINITY && row < rows8)  // no selected column yet: P = 0
#pragma unroll
            for (int q = 0; q < kNpt / 8; ++q)
              *reinterpret_cast<uint4*>(sP + tc::sw128_offset(row, (kNpt * cg) / 8 + q)) = make_uint4(0u, 0u, 0u, 0u);
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
      for (int tile = 0; tile < kTiles; ++tile) {
        const uint32_t pb = smem_u32(base + lay.p + tile * lay.q_atom);
#pragma unroll
        for (int ks = 0; ks < kTok / 16; ++ks)
          tc::mma_bf16(tmem + 256u * tile + 128u, tc::sw128_desc(pb + ks * 32),
                       tc::sw128_desc_mn(vb + ks * 16 * 128, kKVAtom), kIdescPV, c > 0 || ks > 0);
      }
      tc::mma_commit(bar_o);
      if (c + 1 < nch) issue_qk(c + 1);
    }
    if (!dead && !mbar_wait_warp(bar_o, ph)) {
      if (lane == 0) record_error(p.ws_header, CLSA_ERR_TIMEOUT, 51);
      dead = true;
    }
    tc::fence_after_sync();
    if (c + 2 < nch) load_chunk(c + 2);
    cp_async_commit();
  }
  cp_async_wait<0>();

  // row sums over the two column groups of each tile, then the output rows from TMEM
  cl[cg * kM + row] = lp;
  __syncthreads();
  const float ls = cl[row] + cl[kM + row];
  const int l = lgrp * p.Lg + row / p.G;
  const int t = t0 + x;
  const bool mine = row < p.rows && l < p.L && t < p.T;
  const bool has = nch > 0 && !dead;
  if (q4 * 32 < p.rows) {  // warp-uniform (the tile's rows); the TMEM loads are .sync.aligned
    const int h = g * p.G + row % p.G;
    uint4* out = reinterpret_cast<uint4*>(p.O + (((size_t)l * p.T + t) * p.Hq + h) * kD + kOpt * cg);
    if (has) {
      const float inv = ls > 0.f ? 1.f / ls : 0.f;  // a row with no selected token: O = 0
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
      p.lse[((size_t)l * p.T + t) * p.Hq + h] = has && ls > 0.f ? (m + log2f(ls)) * kLn2 : -INFINITY;
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tmem, kTmemCols);
}

}  // namespace

bool prefill_attn_pair_supported(const clsa_prefill_args* a) {
  if (a->dtype != CLSA_BF16 || a->d != kD || a->Hq % a->Hkv != 0 || a->k > 4096) return false;
  if ((reinterpret_cast<uintptr_t>(a->Q) | reinterpret_cast<uintptr_t>(a->K) | reinterpret_cast<uintptr_t>(a->V) |
       reinterpret_cast<uintptr_t>(a->O)) % 16 != 0)
    return false;
  const int G = a->Hq / a->Hkv;
  if (G > kM) return false;
  const int Lg = std::max(1, std::min(a->L, kM / G));
  return (int)kp_layout(Lg * G, a->k).total + 1024 <= device_info().max_smem_optin;
}

cudaError_t launch_prefill_attn_pair(const clsa_prefill_args* a, float scale, void* ws_header, cudaStream_t s) {
  KPParams p{};
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
  p.Lg = (a->L + p.nlg - 1) / p.nlg;
  p.rows = p.Lg * p.G;
  p.n = a->n;
  p.npairs = (a->T + 1) / 2;
  p.scale_log2 = scale * 1.4426950408889634f;
  const int smem = (int)kp_layout(p.rows, p.k).total + 1024;
  cudaError_t e = cudaFuncSetAttribute(attn_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const long long units = (long long)a->Hkv * p.nlg * p.npairs;
  e = launch_pdl(attn_pair_kernel, dim3((unsigned)units), dim3(kThreadsKP), (size_t)smem, s, p);
  launches_add(1, s);
  return e;
}

}  // namespace clsa
