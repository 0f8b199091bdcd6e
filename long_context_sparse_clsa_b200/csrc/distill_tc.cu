// Distillation target of the shared indexer on the 5th-generation tensor cores
// (bf16, d = 128).  Forward only (picx.dev CLSA summary, Methodology > Architecture
// Overview, multi-layer distillation):
//   Abar_b = 1/(L Hq) sum_{l,h} softmax(Q^(l)[b,h] K[b]^T * scale)   over the len_b rows
//   kl[b]  = KL(Abar_b || softmax(I_b)) = sum_j a_j log a_j - sum_j a_j I_j + lse(I_b) sum_j a_j
// with query head h reading KV head h / G and no scale on the indexer scores I.
//
// Two streaming passes over the cache, each one launch of distill_tc_kernel:
//   unit = (sequence b, KV head g, layer group, token split).  The unit's rows are every
//   (layer, query head) pair of head g in the layer group (L_g * G <= 128); they stay in
//   shared memory for the whole unit, while the split's K rows of head g stream through a
//   two-stage ring of 128-token tiles (TMA, 128-byte swizzle).  Warp 8 loads, warp 9
//   issues the MMAs into one of two TMEM buffers, and warps 0-7 (two groups of four that
//   take alternate tiles) read TMEM.
//   pass 1 (row lse)  S = Q K_tile^T (M = 128 rows, N = 128 tokens): a thread owns one
//                     row and keeps an online max and sum of 2^(s scale log2 e) over its
//                     group's tiles; the groups merge, and the unit writes one (max, sum)
//                     pair per row.
//   pass 2 (Abar)     S^T = K_tile Q^T (M = 128 tokens, N = rows rounded up to 16): the
//                     prologue merges pass 1's pairs of the unit's rows over every split
//                     (in split order) into lse2_r; a thread owns one token and sums
//                     2^(s scale log2 e - lse2_r) over the rows.  One fp32 partial per
//                     (sequence, KV head, layer group, token).
// distill_final_kernel: per token, Abar_j = its partials summed in (head, group) order
//   / (L Hq); per 256-token tile, sum a log a - a I, sum a, and (max, sum exp) of I.
// distill_kl_kernel: merges the tile partials in tile order (deterministic).
//
// Reads the cache twice (pass 1, pass 2): 2 n Hkv d bytes per pass.  Every wait is
// bounded (kWaitLimitNs); a timeout records CLSA_ERR_TIMEOUT and the CTA drains its
// copies and MMAs before it frees TMEM and returns.
#include <algorithm>
#include <cmath>

#include "common.cuh"
#include "kernels.h"
#include "tcgen05.cuh"
#include "tma.h"

namespace clsa {

namespace {

constexpr int kTokT = 128;                       // tokens per K tile
constexpr int kHd = 128;                         // head dim
constexpr int kRing = 2;                         // K tiles in flight per CTA (two CTAs per SM)
constexpr int kEpiW = 8;                         // epilogue warps: 2 groups x 4 lane quarters
constexpr int kEpiT = kEpiW * 32;
constexpr int kDThreads = kEpiT + 64;            // + TMA warp + MMA warp
constexpr uint32_t kAtomB = 128 * 128;           // 128 rows x 128 bytes (64 bf16)
constexpr uint32_t kTileB = 2 * kAtomB;          // 128 rows x 128 bf16
constexpr int kUnitsTarget = 2 * 148;            // one wave at two CTAs per SM
constexpr int kMaxSplitTiles = 64;               // at most 8192 tokens per unit
constexpr int kFinalT = 256;                     // tokens per final-kernel tile

struct DTSmem {
  uint64_t full[kRing], empty[kRing], tfull[2], tempty[2], done;
  uint32_t tmem;
  int abort;
  float nl2[128];            // pass 2: -lse2 of each row (-inf past the unit's rows)
  float cm[128], cl[128];    // pass 1: group 1's (max, sum) per row
};

constexpr size_t kDTSmemBytes = 1024 + kTileB * (1 + kRing) + sizeof(DTSmem);

struct DTParams {
  const __nv_bfloat16* Q;    // [L][B][Hq][d]
  const int32_t* lens;       // [B]
  float* pm;                 // [units][128] pass-1 row max (log2 units)
  float* pl;                 // [units][128] pass-1 row sum
  float* tokpart;            // [B][Hkv * nlg][n_max]
  void* ws_header;
  int B, n_max, L, Hq, Hkv, G, Lg, nlg, nsplit, chunk;
  float scale_log2;
};

__device__ __forceinline__ void epi_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kEpiT) : "memory"); }

template <int PASS>
__global__ void __launch_bounds__(kDThreads, 2)
    distill_tc_kernel(const __grid_constant__ CUtensorMap tk, const DTParams p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* base = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                         ~uintptr_t(1023));
  unsigned char* sQ = base;                     // [2 atoms][128 rows][128 B]
  unsigned char* sK = base + kTileB;            // [kRing][2 atoms][128 tokens][128 B]
  DTSmem& sm = *reinterpret_cast<DTSmem*>(sK + kRing * kTileB);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_enter();

  // unit -> (b, g, layer group, split)
  int u = blockIdx.x;
  const int s = u % p.nsplit;
  u /= p.nsplit;
  const int lg = u % p.nlg;
  u /= p.nlg;
  const int g = u % p.Hkv, b = u / p.Hkv;
  const int rows = min(p.Lg, p.L - lg * p.Lg) * p.G;
  const int n = max(0, min(p.lens[b], p.n_max));
  const int t_begin = s * p.chunk;
  const int ntile = max(0, min(p.chunk, (n + kTokT - 1) / kTokT - t_begin));
  const size_t group_unit = ((size_t)b * p.Hkv + g) * p.nlg + lg;  // pass-1 partials of the group

  if (threadIdx.x == 0) {
    for (int i = 0; i < kRing; ++i) {
      mbar_init(&sm.full[i], 1);
      mbar_init(&sm.empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.tfull[i], 1);
      mbar_init(&sm.tempty[i], 4);
    }
    mbar_init(&sm.done, 1);
    sm.abort = 0;
    fence_mbar_init();
  }
  if (warp == kEpiW + 1) {
    tc::tmem_alloc(&sm.tmem, 256);
    tc::tmem_relinquish();
  }
  if (threadIdx.x < kEpiT) {
    // the unit's rows r = (layer lg * Lg + r / G, head g * G + r % G); zeros past `rows`
    for (int v = threadIdx.x; v < 128 * 16; v += kEpiT) {
      const int r = v >> 4, c = v & 15;
      unsigned char* dst = sQ + (c >> 3) * kAtomB + tc::sw128_offset(r, c & 7);
      if (r < rows && ntile > 0) {
        const int l = lg * p.Lg + r / p.G, h = g * p.G + r % p.G;
        cp_async_16(dst, p.Q + (((size_t)l * p.B + b) * p.Hq + h) * kHd + c * 8, 16);
      } else {
        *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
      }
    }
    cp_async_commit();
    if (PASS == 2 && threadIdx.x < 128) {
      // lse2 of row r: pass 1's (max, sum) pairs merged over the splits in split order
      const int r = threadIdx.x;
      float nl = -INFINITY;
      if (r < rows && ntile > 0) {
        const float* pm = p.pm + group_unit * p.nsplit * 128 + r;
        const float* pl = p.pl + group_unit * p.nsplit * 128 + r;
        float M = -INFINITY;
#pragma unroll 4
        for (int x = 0; x < p.nsplit; ++x) M = fmaxf(M, pm[(size_t)x * 128]);
        float S = 0.f;
        if (M != -INFINITY) {
#pragma unroll 4
          for (int x = 0; x < p.nsplit; ++x) S += pl[(size_t)x * 128] * exp2f(pm[(size_t)x * 128] - M);
        }
        nl = S > 0.f ? -(M + log2f(S)) : -INFINITY;
      }
      sm.nl2[r] = nl;
    }
    cp_async_wait<0>();
    fence_proxy_async_smem();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = sm.tmem;

  if (warp == kEpiW) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const int y0 = b * p.n_max + t_begin * kTokT;
      int issued = 0;
      for (int i = 0; i < ntile && !*(volatile int*)&sm.abort; ++i) {
        const int st = i % kRing;
        const uint32_t ph = (uint32_t)(i / kRing) & 1u;
        if (!mbar_wait(&sm.empty[st], ph ^ 1u)) {
          record_error(p.ws_header, CLSA_ERR_TIMEOUT, 700);
          sm.abort = 1;
          break;
        }
        mbar_arrive_expect_tx(&sm.full[st], kTileB);
        unsigned char* dst = sK + st * kTileB;
        tma_load_2d(dst, &tk, g * kHd, y0 + i * kTokT, &sm.full[st]);
        tma_load_2d(dst + kAtomB, &tk, g * kHd + 64, y0 + i * kTokT, &sm.full[st]);
        issued = i + 1;
      }
      // drain: the newest load of each stage has landed (returns at once when consumed)
      for (int i = max(0, issued - kRing); i < issued; ++i)
        if (!mbar_wait(&sm.full[i % kRing], (uint32_t)(i / kRing) & 1u)) record_error(p.ws_header, CLSA_ERR_TIMEOUT, 701);
    }
  } else if (warp == kEpiW + 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const int n2 = max(16, (rows + 15) & ~15);
      const uint32_t idesc = PASS == 1 ? tc::idesc_bf16_f32(128, kTokT) : tc::idesc_bf16_f32(128, n2);
      const uint32_t q_addr = smem_u32(sQ);
      for (int i = 0; i < ntile && !*(volatile int*)&sm.abort; ++i) {
        const int st = i % kRing, buf = i & 1;
        if (!mbar_wait(&sm.full[st], (uint32_t)(i / kRing) & 1u) ||
            !mbar_wait(&sm.tempty[buf], ((uint32_t)(i >> 1) & 1u) ^ 1u)) {
          record_error(p.ws_header, CLSA_ERR_TIMEOUT, 710);
          sm.abort = 1;
          break;
        }
        tc::fence_after_sync();
        const uint32_t k_addr = smem_u32(sK + st * kTileB);
        const uint32_t a_addr = PASS == 1 ? q_addr : k_addr;
        const uint32_t b_addr = PASS == 1 ? k_addr : q_addr;
#pragma unroll
        for (int ks = 0; ks < kHd / 16; ++ks) {
          const uint32_t off = (uint32_t)(ks >> 2) * kAtomB + (uint32_t)(ks & 3) * 32u;
          tc::mma_bf16(tmem + (uint32_t)(buf * 128), tc::sw128_desc(a_addr + off), tc::sw128_desc(b_addr + off), idesc,
                       ks > 0);
        }
        tc::mma_commit(&sm.empty[st]);
        tc::mma_commit(&sm.tfull[buf]);
      }
      tc::mma_commit(&sm.done);  // every MMA issued above has completed when this arrives
      if (!mbar_wait(&sm.done, 0)) record_error(p.ws_header, CLSA_ERR_TIMEOUT, 711);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int grp = warp >> 2, q = warp & 3;
    const uint32_t tl = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(grp * 128);
    const float sl2 = p.scale_log2;
    if (PASS == 1) {
      const int row = q * 32 + lane;
      const bool quarter_live = q * 32 < rows;  // warp-uniform
      float m = -INFINITY, l = 0.f;
      for (int i = grp; i < ntile; i += 2) {
        if (!mbar_wait_warp(&sm.tfull[grp], (uint32_t)(i >> 1) & 1u)) {
          if (lane == 0) {
            record_error(p.ws_header, CLSA_ERR_TIMEOUT, 720);
            sm.abort = 1;
          }
          break;
        }
        tc::fence_after_sync();
        if (quarter_live) {
          const int nv = n - (t_begin + i) * kTokT;  // valid tokens in this tile (>= 1)
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            uint32_t v[64];
            tc::ld_32x32b_x64(tl + (uint32_t)(h * 64), v);
            tc::ld_wait();
            if (nv < 128) {
#pragma unroll
              for (int x = 0; x < 64; ++x)
                if (h * 64 + x >= nv) v[x] = __float_as_uint(-INFINITY);
            }
            float mx = -INFINITY;
#pragma unroll
            for (int x = 0; x < 64; ++x) mx = fmaxf(mx, __uint_as_float(v[x]));
            const float mn = fmaxf(m, mx * sl2);
            if (mn != -INFINITY) {
              float a0 = 0.f, a1 = 0.f;
#pragma unroll
              for (int x = 0; x < 64; x += 2) {
                a0 += fast_exp2(fmaf(__uint_as_float(v[x]), sl2, -mn));
                a1 += fast_exp2(fmaf(__uint_as_float(v[x + 1]), sl2, -mn));
              }
              l = l * fast_exp2(m - mn) + (a0 + a1);
              m = mn;
            }
          }
        }
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.tempty[grp]);
      }
      if (grp == 1) {
        sm.cm[row] = m;
        sm.cl[row] = l;
      }
      epi_sync();
      if (grp == 0) {
        const float m1 = sm.cm[row], l1 = sm.cl[row];
        const float M = fmaxf(m, m1);
        float L = 0.f;
        if (M != -INFINITY) L = l * fast_exp2(m - M) + l1 * fast_exp2(m1 - M);
        const size_t o = (size_t)blockIdx.x * 128 + row;
        p.pm[o] = row < rows ? M : -INFINITY;
        p.pl[o] = row < rows ? L : 0.f;
      }
    } else {
      const int n2 = max(16, (rows + 15) & ~15);
      float* out = p.tokpart + group_unit * p.n_max;
      for (int i = grp; i < ntile; i += 2) {
        if (!mbar_wait_warp(&sm.tfull[grp], (uint32_t)(i >> 1) & 1u)) {
          if (lane == 0) {
            record_error(p.ws_header, CLSA_ERR_TIMEOUT, 730);
            sm.abort = 1;
          }
          break;
        }
        tc::fence_after_sync();
        float a0 = 0.f, a1 = 0.f;
        int c0 = 0;
        for (; c0 + 32 <= n2; c0 += 32) {
          uint32_t v[32];
          tc::ld_32x32b_x32(tl + (uint32_t)c0, v);
          tc::ld_wait();
#pragma unroll
          for (int x = 0; x < 32; x += 4) {
            const float4 nl = *reinterpret_cast<const float4*>(&sm.nl2[c0 + x]);
            a0 += fast_exp2(fmaf(__uint_as_float(v[x]), sl2, nl.x));
            a1 += fast_exp2(fmaf(__uint_as_float(v[x + 1]), sl2, nl.y));
            a0 += fast_exp2(fmaf(__uint_as_float(v[x + 2]), sl2, nl.z));
            a1 += fast_exp2(fmaf(__uint_as_float(v[x + 3]), sl2, nl.w));
          }
        }
        if (c0 < n2) {  // a last 16 columns
          uint32_t v[16];
          tc::ld_32x32b_x16(tl + (uint32_t)c0, v);
          tc::ld_wait();
#pragma unroll
          for (int x = 0; x < 16; x += 4) {
            const float4 nl = *reinterpret_cast<const float4*>(&sm.nl2[c0 + x]);
            a0 += fast_exp2(fmaf(__uint_as_float(v[x]), sl2, nl.x));
            a1 += fast_exp2(fmaf(__uint_as_float(v[x + 1]), sl2, nl.y));
            a0 += fast_exp2(fmaf(__uint_as_float(v[x + 2]), sl2, nl.z));
            a1 += fast_exp2(fmaf(__uint_as_float(v[x + 3]), sl2, nl.w));
          }
        }
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.tempty[grp]);
        const int tok = (t_begin + i) * kTokT + q * 32 + lane;
        if (tok < n) out[tok] = a0 + a1;
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == kEpiW + 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, 256);
  }
}

// Abar and the tile partials: [0] sum a log a - a I, [1] sum a, [2] max I, [3] sum exp(I - max I)
__global__ void __launch_bounds__(kFinalT) distill_final_kernel(const float* __restrict__ tokpart,
                                                                const float* __restrict__ scores,
                                                                const int32_t* __restrict__ lens, int n_max, int HG,
                                                                float inv_rows, float* __restrict__ abar,
                                                                float* __restrict__ tpart, int nt) {
  __shared__ float red[3][kFinalT / 32];
  __shared__ float smax;
  pdl_enter();
  const int b = blockIdx.y, t = blockIdx.x;
  const int j = t * kFinalT + threadIdx.x;
  const int n = max(0, min(lens[b], n_max));
  float a = 0.f, I = -INFINITY, x = 0.f;
  if (j < n) {
    const float* tp = tokpart + (size_t)b * HG * n_max + j;
    float sum = 0.f;
    for (int q = 0; q < HG; ++q) sum += tp[(size_t)q * n_max];
    a = sum * inv_rows;
    I = scores[(size_t)b * n_max + j];
    x = (a > 0.f ? a * logf(a) : 0.f) - a * I;
  }
  if (abar && j < n_max) abar[(size_t)b * n_max + j] = a;
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float xs = warp_sum(x), as = warp_sum(a), im = warp_max(I);
  if (lane == 0) {
    red[0][w] = xs;
    red[1][w] = as;
    red[2][w] = im;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float mm = -INFINITY;
    for (int k = 0; k < kFinalT / 32; ++k) mm = fmaxf(mm, red[2][k]);
    smax = mm;
  }
  __syncthreads();
  const float mI = smax;
  float e = (j < n && mI != -INFINITY) ? expf(I - mI) : 0.f;
  e = warp_sum(e);
  __syncthreads();  // red[2] read by thread 0 above
  if (lane == 0) red[2][w] = e;
  __syncthreads();
  if (threadIdx.x == 0) {
    float X = 0.f, S = 0.f, E = 0.f;
    for (int k = 0; k < kFinalT / 32; ++k) {
      X += red[0][k];
      S += red[1][k];
      E += red[2][k];
    }
    float* o = tpart + ((size_t)b * nt + t) * 4;
    o[0] = X;
    o[1] = S;
    o[2] = mI;
    o[3] = E;
  }
}

// kl[b] = sum X + lse(I) sum S over the tile partials: one block per sequence, each thread
// a strided run of tiles, then the warps and the block in a fixed order (deterministic)
constexpr int kKlT = 256;
__global__ void __launch_bounds__(kKlT) distill_kl_kernel(const float* __restrict__ tpart, int nt,
                                                         float* __restrict__ kl) {
  __shared__ float red[4][kKlT / 32];
  pdl_enter();
  const int b = blockIdx.x, lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  float X = 0.f, S = 0.f, m = -INFINITY, e = 0.f;
  for (int t = threadIdx.x; t < nt; t += kKlT) {
    const float4 o = *reinterpret_cast<const float4*>(tpart + ((size_t)b * nt + t) * 4);
    X += o.x;
    S += o.y;
    const float mn = fmaxf(m, o.z);
    if (mn != -INFINITY) {
      e = e * expf(m - mn) + o.w * expf(o.z - mn);
      m = mn;
    }
  }
  X = warp_sum(X);
  S = warp_sum(S);
  float M = warp_max(m);
  e = warp_sum(M != -INFINITY ? e * expf(m - M) : 0.f);
  if (lane == 0) {
    red[0][w] = X;
    red[1][w] = S;
    red[2][w] = M;
    red[3][w] = e;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    X = 0.f, S = 0.f, M = -INFINITY;
    for (int k = 0; k < kKlT / 32; ++k) {
      X += red[0][k];
      S += red[1][k];
      M = fmaxf(M, red[2][k]);
    }
    float E = 0.f;
    if (M != -INFINITY)
      for (int k = 0; k < kKlT / 32; ++k) E += red[3][k] * expf(red[2][k] - M);
    kl[b] = (S > 0.f && E > 0.f) ? X + (M + logf(E)) * S : 0.f;
  }
}

struct DTPlan {
  int G, Lg, nlg, nsplit, chunk, units, HG, nt;
};

DTPlan dt_plan(int B, int n_max, int L, int Hq, int Hkv) {
  DTPlan pl;
  pl.G = Hq / Hkv;
  pl.Lg = std::max(1, std::min(L, 128 / pl.G));
  pl.nlg = (L + pl.Lg - 1) / pl.Lg;
  const int ntiles = std::max(1, (n_max + kTokT - 1) / kTokT);
  const long long base = (long long)B * Hkv * pl.nlg;
  long long ns = std::max<long long>((kUnitsTarget + base - 1) / base, (ntiles + kMaxSplitTiles - 1) / kMaxSplitTiles);
  ns = std::max<long long>(1, std::min<long long>(ns, ntiles));
  pl.chunk = (int)((ntiles + ns - 1) / ns);
  pl.nsplit = (ntiles + pl.chunk - 1) / pl.chunk;
  pl.units = (int)(base * pl.nsplit);
  pl.HG = Hkv * pl.nlg;
  pl.nt = (n_max + kFinalT - 1) / kFinalT;
  return pl;
}

}  // namespace

bool distill_tc_supported(int B, int n_max, int L, int Hq, int Hkv, int d, clsa_dtype dt) {
  if (dt != CLSA_BF16 || d != kHd || Hkv < 1 || Hq % Hkv != 0 || Hq / Hkv > 128) return false;
  if ((long long)B * n_max + kTokT > 0x7fffffffLL) return false;  // TMA row coordinate
  const DTPlan pl = dt_plan(B, n_max, L, Hq, Hkv);
  return (long long)B * Hkv * pl.nlg * pl.nsplit < 0x7fffffffLL;
}

size_t distill_tc_ws_bytes(int B, int n_max, int L, int Hq, int Hkv) {
  const DTPlan pl = dt_plan(B, n_max, L, Hq, Hkv);
  size_t off = 0;
  off += 2 * align_up((size_t)pl.units * 128 * 4, 256);             // pass-1 (max, sum) per unit row
  off += align_up((size_t)B * pl.HG * n_max * 4, 256);              // per-token partials
  off += align_up((size_t)B * pl.nt * 4 * 4, 256);                  // final-kernel tile partials
  return off;
}

cudaError_t launch_distill_tc(const void* Q, const void* K, const float* scores, const int32_t* lens, int B, int n_max,
                              int L, int Hq, int Hkv, float scale, float* abar, float* kl, void* ws_header, void* ws,
                              cudaStream_t s) {
  const DTPlan pl = dt_plan(B, n_max, L, Hq, Hkv);
  char* w = static_cast<char*>(ws);
  float* pm = reinterpret_cast<float*>(w);
  w += align_up((size_t)pl.units * 128 * 4, 256);
  float* plsum = reinterpret_cast<float*>(w);
  w += align_up((size_t)pl.units * 128 * 4, 256);
  float* tokpart = reinterpret_cast<float*>(w);
  w += align_up((size_t)B * pl.HG * n_max * 4, 256);
  float* tpart = reinterpret_cast<float*>(w);

  CUtensorMap tk;
  if (!make_tmap_bf16_2d(&tk, K, (uint64_t)B * n_max, (uint64_t)Hkv * kHd, (uint64_t)Hkv * kHd * 2, kTokT, 64))
    return cudaErrorInvalidValue;
  DTParams p{static_cast<const __nv_bfloat16*>(Q), lens, pm, plsum, tokpart, ws_header, B, n_max, L, Hq, Hkv,
             pl.G, pl.Lg, pl.nlg, pl.nsplit, pl.chunk, scale * 1.4426950408889634f};
  cudaError_t e = cudaFuncSetAttribute(distill_tc_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kDTSmemBytes);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(distill_tc_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kDTSmemBytes);
  if (e != cudaSuccess) return e;
  // each kernel waits at entry for the one before it (pdl_enter): launches overlap, work does not
  e = launch_pdl(distill_tc_kernel<1>, dim3(pl.units), dim3(kDThreads), kDTSmemBytes, s, tk, p);
  if (e == cudaSuccess) e = launch_pdl(distill_tc_kernel<2>, dim3(pl.units), dim3(kDThreads), kDTSmemBytes, s, tk, p);
  if (e == cudaSuccess)
    e = launch_pdl(distill_final_kernel, dim3(pl.nt, B), dim3(kFinalT), 0, s, (const float*)tokpart, scores, lens,
                   n_max, pl.HG, 1.f / (float)(L * Hq), abar, tpart, pl.nt);
  if (e == cudaSuccess) e = launch_pdl(distill_kl_kernel, dim3(B), dim3(kKlT), 0, s, (const float*)tpart, pl.nt, kl);
  if (e != cudaSuccess) return e;
  launches_add(4, s);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Attention-mass coverage: the share of each row's dense softmax mass that the selection S
// holds, mass = sum_{j in S} softmax_j = exp(lse_S - lse_all).  lse_all over the whole
// cache is pass 1 of the distillation kernel (per unit row: max and sum of 2^(s scale
// log2 e) over its token split); this kernel merges the splits in split order and takes
// lse_S from the decode step's lse output.
// ---------------------------------------------------------------------------
namespace {

__global__ void __launch_bounds__(128) attn_mass_kernel(const float* __restrict__ pm, const float* __restrict__ pl,
                                                        const float* __restrict__ lse_sparse, int B, int L, int Hq,
                                                        int Hkv, int G, int Lg, int nlg, int nsplit,
                                                        float* __restrict__ mass, float* __restrict__ lse_all) {
  pdl_enter();
  int u = blockIdx.x;  // (b, g, layer group), the order of distill_tc_kernel's units / nsplit
  const int lg = u % nlg;
  u /= nlg;
  const int g = u % Hkv, b = u / Hkv;
  const int r = threadIdx.x;
  const int rows = min(Lg, L - lg * Lg) * G;
  if (r >= rows) return;
  const size_t unit0 = ((size_t)blockIdx.x * nsplit) * 128 + r;
  float M = -INFINITY;
  for (int x = 0; x < nsplit; ++x) M = fmaxf(M, pm[unit0 + (size_t)x * 128]);
  float S = 0.f;
  if (M != -INFINITY)
    for (int x = 0; x < nsplit; ++x) S += pl[unit0 + (size_t)x * 128] * exp2f(pm[unit0 + (size_t)x * 128] - M);
  const float la = S > 0.f ? (M + log2f(S)) * 0.6931471805599453f : -INFINITY;  // natural log
  const int l = lg * Lg + r / G, h = g * G + r % G;
  const size_t o = ((size_t)l * B + b) * Hq + h;
  const float ls = lse_sparse[o];
  mass[o] = (la == -INFINITY || ls == -INFINITY) ? 0.f : expf(ls - la);
  if (lse_all) lse_all[o] = la;
}

}  // namespace

size_t attention_mass_tc_ws_bytes(int B, int n_max, int L, int Hq, int Hkv) {
  const DTPlan pl = dt_plan(B, n_max, L, Hq, Hkv);
  return 2 * align_up((size_t)pl.units * 128 * 4, 256);
}

cudaError_t launch_attention_mass_tc(const void* Q, const void* K, const float* lse_sparse, const int32_t* lens, int B,
                                     int n_max, int L, int Hq, int Hkv, float scale, float* mass, float* lse_all,
                                     void* ws_header, void* ws, cudaStream_t s) {
  const DTPlan pl = dt_plan(B, n_max, L, Hq, Hkv);
  char* w = static_cast<char*>(ws);
  float* pm = reinterpret_cast<float*>(w);
  w += align_up((size_t)pl.units * 128 * 4, 256);
  float* plsum = reinterpret_cast<float*>(w);
  CUtensorMap tk;
  if (!make_tmap_bf16_2d(&tk, K, (uint64_t)B * n_max, (uint64_t)Hkv * kHd, (uint64_t)Hkv * kHd * 2, kTokT, 64))
    return cudaErrorInvalidValue;
  DTParams p{static_cast<const __nv_bfloat16*>(Q), lens, pm, plsum, nullptr, ws_header, B, n_max, L, Hq, Hkv,
             pl.G, pl.Lg, pl.nlg, pl.nsplit, pl.chunk, scale * 1.4426950408889634f};
  cudaError_t e = cudaFuncSetAttribute(distill_tc_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kDTSmemBytes);
  if (e != cudaSuccess) return e;
  e = launch_pdl(distill_tc_kernel<1>, dim3(pl.units), dim3(kDThreads), kDTSmemBytes, s, tk, p);
  if (e == cudaSuccess)
    e = launch_pdl(attn_mass_kernel, dim3(B * Hkv * pl.nlg), dim3(128), 0, s, (const float*)pm, (const float*)plsum,
                   lse_sparse, B, L, Hq, Hkv, pl.G, pl.Lg, pl.nlg, pl.nsplit, mass, lse_all);
  if (e != cudaSuccess) return e;
  launches_add(2, s);
  return cudaGetLastError();
}

}  // namespace clsa
