// Prefill routing without materialising the T x n score matrix.
//
// Routing equation for T new rows at cache positions t = n - T + i (picx.dev CLSA
// summary, Methodology > Architecture Overview): I[i, j] = q_idx[i] . K_idx[j] for
// j <= t, S_t = TopK(I_t, min(k, t + 1)).
//
// prefill_route_kernel: persistent, one CTA per SM, warp-specialised tcgen05 GEMM.
//   unit     = two 128-row query blocks x one slice of the key range (so every CTA has
//              work; the two blocks share each K_idx tile, halving its L2 traffic)
//   warp 0   TMA producer: the unit's two Q_idx blocks once, then 128-key K_idx tiles
//            into a 3-stage ring (128-byte swizzle, the UMMA K-major layout)
//   warp 1   MMA issuer: per tile, 2 x 8 tcgen05.mma (M=128, N=128, K=16) into one of
//            two TMEM buffers; commits free the ring stage and publish the buffer
//   warps 2-9 epilogue, one query row per thread (TMEM lane): tcgen05.ld 32 scores at a
//            time, causal mask, then
//              warm-up tiles: a 32-bin histogram of the row's scores over
//                             [mean, mean + 1.25 (max - mean)] of its first visible tile,
//                             in a thread-private shared-memory column;
//              threshold:     tau = the lower edge of the bin where the count from the
//                             top reaches m, m chosen so that ~2 k_eff tokens of the
//                             whole row score >= tau;
//              every tile:    a bit mask of the 32 scores >= tau, the scores staged in a
//                             private shared-memory row, and one (score, token) store per
//                             set bit into the row's slice buffer, in token order.
//   The warm-up tiles are spread over the slice and scored a second time in the main
//   pass (8 extra tiles per ~110).
// prefill_densify_kernel: per row, concatenate the slice buffers (token order) into a
//   dense candidate row.  The row is exact iff at least k_eff candidates score >= the
//   largest tau any of its slices used: every dropped token then scores strictly below
//   the k_eff-th candidate, so it cannot be selected (ties included).  A row failing
//   that, or with an overflowed slice buffer, is flagged for the exact fallback (score
//   the whole row, select).
// The exact TopK over each dense candidate row is the radix-select kernel of topk.cu.
#include <cmath>
#include <cstdio>
#include <cstdlib>

#include "common.cuh"
#include "kernels.h"
#include "tcgen05.cuh"
#include "tma.h"

namespace clsa {

bool make_tmap_bf16_2d(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint64_t pitch_bytes,
                       uint32_t box_rows, uint32_t box_cols) {
  using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
  static EncodeFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !p)
      return false;
    fn = reinterpret_cast<EncodeFn>(p);
  }
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {pitch_bytes};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

namespace {

constexpr int kRM = 128;         // rows per query block (TMEM lanes)
constexpr int kRN = 128;         // keys per tile: two 64-key halves
constexpr int kRH = 64;          // keys per half
constexpr int kRStages = 2;      // K tile ring
constexpr int kEpiWarps = 16;    // 4 lane quarters x 2 query blocks x 2 key halves
constexpr int kEpiThreads = kEpiWarps * 32;
constexpr int kRThreads = 64 + kEpiThreads;  // + producer warp + MMA warp
constexpr int kWarm = 8;         // warm-up tiles per unit
constexpr int kBins = 32;        // warm-up histogram bins per row
constexpr int kStagePitch = 36;  // words per staged row
constexpr int kTraceSlots = 40;  // producer issue, MMA operands ready, MMA issued, epilogue warps done, started
constexpr int kMinSample = 8;    // fewer expected sample scores above the boundary: no bound
constexpr uint32_t kABlock = kRM * 128 * 2;  // one query block, both 64-column atoms: 32 KiB
constexpr uint32_t kBTile = kRN * 128 * 2;   // one key tile, both atoms: 32 KiB
constexpr uint32_t kAtomA = kRM * 128;       // 16 KiB
constexpr uint32_t kAtomB = kRN * 128;
constexpr uint32_t kHalfB = kRH * 128;       // one half of one atom of the key tile: 8 KiB

struct RouteParams {
  int n, T, k, S, cap, nunits;
  uint2* cand;         // [T][S][2][cap/2] candidates: (score fp32 bits, token), per key half
  int32_t* cand_cnt;   // [T][S][2]  (> cap/2: overflow)
  float* cand_tau;     // [T][S]  the bound the slice used (-inf: every token kept)
  uint32_t* any_flag;  // set by the densify step when some row needs the exact fallback
  unsigned long long* trace;  // CTA 0 per-step stamps [512][kTraceSlots] or null
  void* ws_header;
};

struct RouteSmem {
  // per epilogue thread, private: its warm-up histogram (column et of hist), then, in the
  // main pass, its 32 staged scores (row et of stage, padded so that eight 16-byte
  // stores of a quarter-warp hit distinct banks)
  union {
    uint32_t hist[kBins][kEpiThreads];
    uint32_t stage[kEpiThreads][kStagePitch];
  } u;
  float xmax[kEpiThreads], xsum[kEpiThreads];  // range exchange between the two halves of a row
  int xcnt[kEpiThreads], xseen[kEpiThreads];
  uint64_t full[kRStages], empty[kRStages];
  uint64_t tfull[2], tempty[2];
  uint64_t afull, aempty;
  uint32_t tmem;
  int abort_flag;
};
constexpr size_t kRouteSmem = 1024 /*align slack*/ + 2 * kABlock + kRStages * kBTile + sizeof(RouteSmem);
static_assert(kRouteSmem <= 227 * 1024, "shared memory");

// warm-up histogram bin of a score: round(sat(score * hs + hb) * (kBins - 1)), the
// rounding done by adding 1.5 * 2^23 (the sum's low mantissa bits are the integer)
__device__ __forceinline__ int hist_bin(uint32_t bits, float hs, float hb) {
  const float x = __saturatef(fmaf(__uint_as_float(bits), hs, hb));
  return __float_as_int(fmaf(x, (float)(kBins - 1), 12582912.f)) - 0x4B400000;
}

// shared-memory increment by shared-window address (a generic atomic is slower)
__device__ __forceinline__ void red_shared_inc(uint32_t addr) {
  asm volatile("red.shared.add.u32 [%0], 1;" ::"r"(addr) : "memory");
}

// The main-pass test of a pair of scores against the row bound tau, in two instructions:
// both scores rounded toward zero to bf16 in one conversion, then one packed compare with
// rz(tau), 0xffff in each half that passes.  Rounding toward zero is monotone, so every
// score >= tau passes (a superset test); a score that passes below tau lies within one
// bf16 step of it and is only an extra candidate: exactness is decided later on the fp32
// scores (ties and all), and a dropped score has rz(score) < rz(tau), hence score < tau.
// tau = -inf (every token kept) passes every finite score.
__device__ __forceinline__ uint32_t rz_bf16x2(float hi, float lo) {
  uint32_t d;
  asm("cvt.rz.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
  return d;
}
__device__ __forceinline__ uint32_t ge_bf16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("set.ge.u32.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

__device__ __forceinline__ uint32_t ld_shared_u32(uint32_t addr) {
  uint32_t x;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(x) : "r"(addr) : "memory");
  return x;
}

// 16-byte shared store, done only when `pred` is non-zero (no branch)
__device__ __forceinline__ void st_shared_v4_if(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d,
                                                uint32_t pred) {
  asm volatile("{\n .reg .pred q;\n setp.ne.u32 q, %5, 0;\n @q st.shared.v4.u32 [%0], {%1, %2, %3, %4};\n}" ::"r"(addr),
               "r"(a), "r"(b), "r"(c), "r"(d), "r"(pred)
               : "memory");
}

// predicated 8-byte global store (no branch)
__device__ __forceinline__ void st_global_v2_if(uint2* p, uint32_t a, uint32_t b, bool pred) {
  asm volatile("{\n .reg .pred q;\n setp.ne.u32 q, %3, 0;\n @q st.global.v2.u32 [%0], {%1, %2};\n}" ::"l"(p), "r"(a),
               "r"(b), "r"((uint32_t)pred));
}

// barrier among the epilogue warps only (named barrier 1)
__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 1, %0;" ::"n"(kEpiThreads) : "memory"); }

// A unit's key slice, in 64-key blocks [b_lo, b_hi), is cut into two contiguous halves
// [b_lo, b_mid) and [b_mid, b_hi); step tau loads block b_lo + tau of the first half and
// b_mid + tau of the second (absent past b_hi).  Main pass: tau = 0 .. L-1; warm-up:
// nwarm steps spread over the same range.
struct UnitTiles {
  int r0, b_lo, b_mid, b_hi, L, nwarm;
  __device__ int count() const { return nwarm + L; }
  __device__ int tau(int it) const {
    if (it < nwarm) return (int)(((long long)it * L) / nwarm);
    return it - nwarm;
  }
  __device__ int block(int it, int half) const { return (half ? b_mid : b_lo) + tau(it); }
  __device__ bool valid(int it, int half) const { return block(it, half) < (half ? b_hi : b_mid); }
};

__device__ __forceinline__ UnitTiles unit_tiles(const RouteParams& p, int u) {
  UnitTiles ut;
  const int pair = u / p.S, s = u % p.S;
  ut.r0 = pair * 2 * kRM;
  const int tmax = p.n - p.T + min(ut.r0 + 2 * kRM, p.T) - 1;  // largest position of the pair
  const int nblk = tmax / kRH + 1;
  ut.b_lo = (int)(((long long)s * nblk) / p.S);
  ut.b_hi = (int)(((long long)(s + 1) * nblk) / p.S);
  ut.L = (ut.b_hi - ut.b_lo + 1) / 2;
  ut.b_mid = ut.b_lo + ut.L;
  ut.nwarm = min(kWarm, ut.L);
  return ut;
}

__global__ void __launch_bounds__(kRThreads, 1)
    prefill_route_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                         const RouteParams p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                         ~uintptr_t(1023));
  unsigned char* sA = smem;                    // [2 blocks][2 atoms][128 rows][128 B]
  unsigned char* sB = smem + 2 * kABlock;      // [stage][2 atoms][2 halves x 64 keys][128 B]
  RouteSmem& sm = *reinterpret_cast<RouteSmem*>(sB + kRStages * kBTile);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kRStages; ++i) {
      mbar_init(&sm.full[i], 1);
      mbar_init(&sm.empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.tfull[i], 1);
      mbar_init(&sm.tempty[i], kEpiWarps);
    }
    mbar_init(&sm.afull, 1);
    mbar_init(&sm.aempty, 1);
    sm.abort_flag = 0;
    fence_mbar_init();
    if (blockIdx.x == 0) *p.any_flag = 0u;  // the densify step runs after this kernel
  }
  if (warp == 1) {
    tc::tmem_alloc(&sm.tmem, 512);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = sm.tmem;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t ph_empty = 1, ph_aempty = 1;
      for (int u = blockIdx.x; u < p.nunits && !*(volatile int*)&sm.abort_flag; u += gridDim.x) {
        const UnitTiles ut = unit_tiles(p, u);
        if (!mbar_wait_sleep(&sm.aempty, ph_aempty)) { record_error(p.ws_header, CLSA_ERR_TIMEOUT, 400); sm.abort_flag = 1; break; }
        ph_aempty ^= 1u;
        mbar_arrive_expect_tx(&sm.afull, 2 * kABlock);
        for (int h = 0; h < 2; ++h)
          for (int a = 0; a < 2; ++a)
            tma_load_2d(sA + h * kABlock + a * kAtomA, &tq, a * 64, ut.r0 + h * kRM, &sm.afull);
        for (int it = 0; it < ut.count(); ++it) {
          if (!mbar_wait_sleep(&sm.empty[stage], ph_empty)) { record_error(p.ws_header, CLSA_ERR_TIMEOUT, 401); sm.abort_flag = 1; break; }
          if (p.trace && blockIdx.x == 0 && it < 512) p.trace[it * kTraceSlots] = globaltimer_ns();
          mbar_arrive_expect_tx(&sm.full[stage], kBTile);
          // key rows 0..63 of the tile: block of the first half; 64..127: of the second
          // (past the slice, or past n: loaded, masked by the epilogue / zero-filled)
          for (int hf = 0; hf < 2; ++hf)
            for (int a = 0; a < 2; ++a)
              tma_load_2d(sB + stage * kBTile + a * kAtomB + hf * kHalfB, &tk, a * 64, ut.block(it, hf) * kRH,
                          &sm.full[stage]);
          if (++stage == kRStages) { stage = 0; ph_empty ^= 1u; }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = tc::idesc_bf16_f32(kRM, kRN);
      int stage = 0, buf = 0;
      uint32_t ph_full = 0, ph_tempty = 1, ph_afull = 0;
      for (int u = blockIdx.x; u < p.nunits && !*(volatile int*)&sm.abort_flag; u += gridDim.x) {
        const UnitTiles ut = unit_tiles(p, u);
        if (!mbar_wait_sleep(&sm.afull, ph_afull)) { record_error(p.ws_header, CLSA_ERR_TIMEOUT, 410); sm.abort_flag = 1; break; }
        ph_afull ^= 1u;
        for (int it = 0; it < ut.count(); ++it) {
          const bool got_full = mbar_wait_sleep(&sm.full[stage], ph_full);
          if (p.trace && blockIdx.x == 0 && it < 512) p.trace[it * kTraceSlots + 1] = globaltimer_ns();
          if (!got_full || !mbar_wait_sleep(&sm.tempty[buf], ph_tempty)) {
            record_error(p.ws_header, CLSA_ERR_TIMEOUT, 411);
            sm.abort_flag = 1;
            break;
          }
          tc::fence_after_sync();
          const uint32_t b_base = smem_u32(sB + stage * kBTile);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const uint32_t a_base = smem_u32(sA + h * kABlock);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
              const uint32_t koff = (uint32_t)(ks & 3) * 32u;
              tc::mma_bf16(tmem + (uint32_t)(buf * 256 + h * kRN),
                           tc::sw128_desc(a_base + (ks >> 2) * kAtomA + koff),
                           tc::sw128_desc(b_base + (ks >> 2) * kAtomB + koff), idesc, ks > 0);
            }
          }
          tc::mma_commit(&sm.empty[stage]);
          tc::mma_commit(&sm.tfull[buf]);
          if (p.trace && blockIdx.x == 0 && it < 512) p.trace[it * kTraceSlots + 2] = globaltimer_ns();
          if (++stage == kRStages) { stage = 0; ph_full ^= 1u; }
          if (++buf == 2) { buf = 0; ph_tempty ^= 1u; }
        }
        tc::mma_commit(&sm.aempty);  // the A blocks are free once this unit's MMAs finish
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (one row half per thread)
    const int w = warp - 2;
    const int q = warp & 3;                    // TMEM lane quarter this warp may read
    const int g4 = w >> 2;
    const int blk = g4 & 1, hc = g4 >> 1;      // query block, key half
    const int et = w * 32 + lane;              // epilogue thread 0..511: its private smem column / row
    const int pt = et ^ (kEpiThreads / 2);     // the thread holding the other half of the same row
    const uint32_t hist_col = smem_u32(&sm.u.hist[0][et]);  // bin b at + b * 4 * kEpiThreads bytes
    const uint32_t stage_addr = smem_u32(sm.u.stage[et] + 4);  // scores at words 4..35; word 3 is read for an empty mask
    const int caph = p.cap / 2;
    int buf = 0;
    uint32_t ph_tfull = 0;
    bool dead = false;
    // Every epilogue warp runs the same units and steps, so the named barriers below
    // match even after a timeout (a dead warp keeps stepping without touching TMEM).
    for (int u = blockIdx.x; u < p.nunits; u += gridDim.x) {
      epi_bar();  // the previous unit's staging rows are free for this unit's histograms
      const UnitTiles ut = unit_tiles(p, u);
      const int s = u % p.S;
      const int i = ut.r0 + blk * kRM + q * 32 + lane;  // query row
      const bool row_ok = i < p.T;
      const int t = p.n - p.T + i;                      // its cache position
      const int keff = min(p.k, t + 1);
#pragma unroll
      for (int y = 0; y < kBins; ++y) sm.u.hist[y][et] = 0u;
      bool have = false;  // histogram range fixed
      float hs = 0.f, hb = 0.f, lo = 0.f, span = 0.f;  // bin map: sat(score * hs + hb) * (kBins - 1)
      int seen = 0, cnt = 0;
      float tau = -INFINITY;
      uint32_t tau2 = rz_bf16x2(-INFINITY, -INFINITY);  // rz(tau) in both halves (set with tau)
      uint2* const dst = p.cand + ((size_t)((row_ok ? i : 0) * p.S + s) * 2 + hc) * caph;
      for (int it = 0; it < ut.count(); ++it) {
        if (!dead && !mbar_wait_warp(&sm.tfull[buf], ph_tfull)) {
          if (lane == 0) record_error(p.ws_header, CLSA_ERR_TIMEOUT, 420);
          sm.abort_flag = 1;
          dead = true;
        }
        dead = __any_sync(0xffffffffu, dead || *(volatile int*)&sm.abort_flag);
        if (p.trace && blockIdx.x == 0 && lane == 0 && it < 512) p.trace[it * kTraceSlots + 3 + kEpiWarps + w] = globaltimer_ns();
        tc::fence_after_sync();
        const bool warm = it < ut.nwarm;
        const int j0 = ut.block(it, hc) * kRH;
        const int nvis = (row_ok && ut.valid(it, hc)) ? max(0, min(kRH, t - j0 + 1)) : 0;  // visible keys
        const uint32_t tbase = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(buf * 256 + blk * kRN + hc * kRH);
        if (warm && it == 0) {
          // histogram range of the row from this first tile, both halves:
          // [mean, mean + 1.25 (max - mean)]; larger scores count in the top bin
          float mx = -INFINITY, s0 = 0.f, s1 = 0.f;
          if (!dead) {
#pragma unroll 1
            for (int ch = 0; ch < 2; ++ch) {
              uint32_t v[32];
              tc::ld_32x32b_x32(tbase + (uint32_t)(32 * ch), v);
              tc::ld_wait();
#pragma unroll
              for (int c = 0; c < 32; c += 2) {
                if (32 * ch + c < nvis) {
                  mx = fmaxf(mx, __uint_as_float(v[c]));
                  s0 += __uint_as_float(v[c]);
                }
                if (32 * ch + c + 1 < nvis) {
                  mx = fmaxf(mx, __uint_as_float(v[c + 1]));
                  s1 += __uint_as_float(v[c + 1]);
                }
              }
            }
          }
          sm.xmax[et] = mx;
          sm.xsum[et] = s0 + s1;
          sm.xcnt[et] = nvis;
          epi_bar();
          const float mx2 = fmaxf(mx, sm.xmax[pt]);
          const int c2 = nvis + sm.xcnt[pt];
          if (row_ok && c2 > 0) {
            // the pair sums in the same order on both threads: the same range
            lo = (hc == 0 ? (s0 + s1) + sm.xsum[pt] : sm.xsum[pt] + (s0 + s1)) / (float)c2;
            span = 1.25f * (mx2 - lo);
            if (span > 0.f && span < INFINITY) {
              hs = 1.f / span;
              hb = -lo * hs;
              have = true;
            }
          }
        }
        if (!dead && (!warm || __any_sync(0xffffffffu, have))) {
          if (warm && have) seen += nvis;
#pragma unroll 1
          for (int ch = 0; ch < 2; ++ch) {
            uint32_t v[32];
            tc::ld_32x32b_x32(tbase + (uint32_t)(32 * ch), v);
            tc::ld_wait();
            const int nv = nvis - 32 * ch;  // visible columns of this chunk (may be <= 0 or > 32)
            if (warm) {
              if (have) {
                if (nv >= 32) {
#pragma unroll
                  for (int c = 0; c < 32; ++c)
                    red_shared_inc(hist_col + (uint32_t)hist_bin(v[c], hs, hb) * (4u * kEpiThreads));
                } else {
#pragma unroll
                  for (int c = 0; c < 32; ++c)
                    if (c < nv) red_shared_inc(hist_col + (uint32_t)hist_bin(v[c], hs, hb) * (4u * kEpiThreads));
                }
              }
            } else {
              // bit c of the mask: column c passes (columns c and c + 16 share one
              // conversion and one packed compare; two accumulators halve the OR chain)
              uint32_t ma = 0u, mb = 0u;
#pragma unroll
              for (int c = 0; c < 16; c += 2) {
                ma |= ge_bf16x2(rz_bf16x2(__uint_as_float(v[16 + c]), __uint_as_float(v[c])), tau2) & (0x10001u << c);
                mb |= ge_bf16x2(rz_bf16x2(__uint_as_float(v[17 + c]), __uint_as_float(v[c + 1])), tau2) &
                      (0x20002u << c);
              }
              uint32_t mm = ma | mb;
              if (nv < 32) mm &= nv <= 0 ? 0u : (0xffffffffu >> (32 - nv));
              // stage the scores of every 4-column group that holds a candidate in this
              // thread's smem row, then one (score, token) store per set bit, in column order
              if (__any_sync(0xffffffffu, mm != 0u)) {
#pragma unroll
                for (int g = 0; g < 8; ++g)
                  st_shared_v4_if(stage_addr + 16u * g, v[4 * g], v[4 * g + 1], v[4 * g + 2], v[4 * g + 3],
                                  mm & (0xfu << (4 * g)));
                const uint32_t jb = (uint32_t)(j0 + 32 * ch);
                const int pc = __popc(mm);
                if (cnt + pc <= caph) {
                  uint2* const out = dst + cnt;
#pragma unroll
                  for (int e = 0; e < 4; ++e) {
                    const uint32_t lsb = mm & (0u - mm);
                    const int c = 31 - __clz(lsb);  // -1 when mm == 0: reads the pad word, store off
                    st_global_v2_if(out + e, ld_shared_u32(stage_addr + 4 * c), jb + (uint32_t)c, mm != 0u);
                    mm ^= lsb;
                  }
                  if (__any_sync(0xffffffffu, mm != 0u)) {
                    int e = 4;
                    while (mm) {
                      const int c = __ffs(mm) - 1;
                      out[e++] = make_uint2(ld_shared_u32(stage_addr + 4 * c), jb + (uint32_t)c);
                      mm &= mm - 1u;
                    }
                  }
                } else {
                  // overflow: keep counting (the row is flagged), stop writing past the buffer
                  int e = 0;
                  while (mm) {
                    const int c = __ffs(mm) - 1;
                    if (cnt + e < caph) dst[cnt + e] = make_uint2(ld_shared_u32(stage_addr + 4 * c), jb + (uint32_t)c);
                    ++e;
                    mm &= mm - 1u;
                  }
                }
                cnt += pc;
              }
            }
          }
        }
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.tempty[buf]);
        if (p.trace && blockIdx.x == 0 && lane == 0 && it < 512) p.trace[it * kTraceSlots + 3 + w] = globaltimer_ns();
        if (++buf == 2) { buf = 0; ph_tfull ^= 1u; }
        if (it + 1 == ut.nwarm) {
          // lower edge of the highest bin at which the sample count (both halves) from the
          // top reaches m = twice the expected count of the sample above the k_eff
          // boundary; no bound (tau = -inf, every token a candidate) when all tokens are
          // selected or the sample is too small.  The bound is a guess: the densify step
          // verifies it.  Both threads of a row compute the same tau.
          sm.xseen[et] = seen;
          epi_bar();  // both halves' histograms are complete
          const int seen2 = seen + sm.xseen[pt];
          tau = -INFINITY;
          if (have && keff < t + 1) {
            const int m = (int)ceilf(2.0f * (float)keff * (float)seen2 / (float)(t + 1));
            if (m >= kMinSample && seen2 >= m) {
              int cum = 0;
              for (int y = kBins - 1; y >= 1; --y) {  // bin 0 also holds every lower score
                cum += (int)(sm.u.hist[y][et] + sm.u.hist[y][pt]);
                if (cum >= m) {
                  tau = lo + ((float)y - 0.5f) * span / (float)(kBins - 1);
                  break;
                }
              }
            }
          }
          tau2 = rz_bf16x2(tau, tau);
          epi_bar();  // every histogram is read: the staging rows may overwrite them
        }
      }
      if (row_ok) {
        p.cand_cnt[((size_t)i * p.S + s) * 2 + hc] = cnt;
        if (hc == 0) p.cand_tau[(size_t)i * p.S + s] = ut.count() > 0 ? tau : -INFINITY;
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) tc::tmem_dealloc(tmem, 512);
}

// One CTA per row: concatenate the row's buffers (slices in key order, each slice's two
// halves in key order, tokens ascending inside a buffer) into a dense candidate row, or
// flag the row for the exact fallback when a buffer overflowed or the candidates number
// fewer than k_eff.
__global__ void __launch_bounds__(256) prefill_densify_kernel(const RouteParams p, uint32_t* __restrict__ dval,
                                                              int32_t* __restrict__ dtok,
                                                              int32_t* __restrict__ dlen,
                                                              int32_t* __restrict__ flag, int ldd) {
  __shared__ int off[2 * 64 + 1];
  __shared__ int bad;
  __shared__ float tmax;
  __shared__ int above;
  const int i = blockIdx.x;
  const int t = p.n - p.T + i;
  const int keff = min(p.k, t + 1);
  if (threadIdx.x == 0) {
    const int caph = p.cap / 2;
    int acc = 0, over = 0;
    float tm = -INFINITY;
    for (int b2 = 0; b2 < 2 * p.S; ++b2) {
      const int c = p.cand_cnt[(size_t)i * p.S * 2 + b2];
      off[b2] = acc;
      over |= c > caph;
      acc += min(c, caph);
    }
    for (int s2 = 0; s2 < p.S; ++s2) tm = fmaxf(tm, p.cand_tau[(size_t)i * p.S + s2]);
    off[2 * p.S] = acc;
    bad = over || acc < keff;
    tmax = tm;
    above = 0;
  }
  __syncthreads();
  if (!bad) {
    int mine = 0;
    for (int b2 = 0; b2 < 2 * p.S; ++b2) {
      const int o = off[b2], c = off[b2 + 1] - o;
      const size_t src = ((size_t)i * p.S * 2 + b2) * (p.cap / 2);
      for (int e = threadIdx.x; e < c; e += blockDim.x) {
        const uint2 cv = p.cand[src + e];
        dval[(size_t)i * ldd + o + e] = cv.x;
        dtok[(size_t)i * ldd + o + e] = (int32_t)cv.y;
        mine += __uint_as_float(cv.x) >= tmax;
      }
    }
    if (mine) atomicAdd(&above, mine);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    if (!bad && above < keff) bad = 1;  // some slice's bound may have dropped a selected token
    flag[i] = bad;
    dlen[i] = bad ? 0 : off[2 * p.S];
    if (bad) atomicOr(p.any_flag, 1u);
  }
}

struct RoutePlan {
  int S, cap, nunits, grid, ldd;
};

RoutePlan route_plan(int n, int T, int k) {
  RoutePlan rp{};
  const int sms = std::max(1, device_info().sm_count);
  const int npairs = (T + 2 * kRM - 1) / (2 * kRM);
  rp.S = std::max(1, std::min(64, sms / npairs));
  rp.nunits = npairs * rp.S;
  rp.grid = std::min(rp.nunits, sms);
  const int expect = (int)std::ceil(2.0 * std::min(k, n) / rp.S);
  rp.cap = std::max(256, std::min(16384, (4 * expect + 63) / 64 * 64));
  rp.ldd = rp.S * rp.cap;
  return rp;
}

}  // namespace

int prefill_route_ldd(const clsa_prefill_args* a) { return route_plan(a->n, a->T, a->k).ldd; }

bool prefill_route_supported(const clsa_prefill_args* a) {
  return a->d_idx == 128 && device_info().max_smem_optin >= (int)kRouteSmem && a->T >= 1;
}

size_t prefill_route_ws_bytes(const clsa_prefill_args* a) {
  const RoutePlan rp = route_plan(a->n, a->T, a->k);
  const size_t T = (size_t)a->T;
  size_t off = 0;
  off += align_up(T * rp.S * rp.cap * 8, 256);      // slice buffers (score, token)
  off += align_up(T * rp.S * 2 * 4, 256);           // buffer counts (slice x half)
  off += align_up(T * rp.S * 4, 256);               // slice bounds
  off += 2 * align_up(T * rp.ldd * 4, 256);         // dense candidate rows
  off += 2 * align_up(T * 4, 256);                  // dense lengths, fallback flags
  off += 256;                                       // any-flag word
  off += 512 * kTraceSlots * 8;                     // step stamps (CLSA_TRACE=1)
  return off;
}

cudaError_t launch_prefill_route(const clsa_prefill_args* a, void* ws_header, void* ws, cudaStream_t s,
                                 PrefillRouteBufs* out) {
  const RoutePlan rp = route_plan(a->n, a->T, a->k);
  const size_t T = (size_t)a->T;
  char* w = static_cast<char*>(ws);
  RouteParams p{};
  p.n = a->n;
  p.T = a->T;
  p.k = a->k;
  p.S = rp.S;
  p.cap = rp.cap;
  p.nunits = rp.nunits;
  p.ws_header = ws_header;
  p.cand = reinterpret_cast<uint2*>(w);
  w += align_up(T * rp.S * rp.cap * 8, 256);
  p.cand_cnt = reinterpret_cast<int32_t*>(w);
  w += align_up(T * rp.S * 2 * 4, 256);
  p.cand_tau = reinterpret_cast<float*>(w);
  w += align_up(T * rp.S * 4, 256);
  out->dval = reinterpret_cast<uint32_t*>(w);
  w += align_up(T * rp.ldd * 4, 256);
  out->dtok = reinterpret_cast<int32_t*>(w);
  w += align_up(T * rp.ldd * 4, 256);
  out->dlen = reinterpret_cast<int32_t*>(w);
  w += align_up(T * 4, 256);
  out->flag = reinterpret_cast<int32_t*>(w);
  w += align_up(T * 4, 256);
  out->any_flag = reinterpret_cast<uint32_t*>(w);
  w += 256;
  const char* tr = std::getenv("CLSA_TRACE");
  p.trace = (tr && tr[0] == '1') ? reinterpret_cast<unsigned long long*>(w) : nullptr;
  out->ldd = rp.ldd;
  p.any_flag = out->any_flag;

  CUtensorMap tq, tk;
  if (!make_tmap_bf16_2d(&tq, a->q_idx, (uint64_t)a->T, 128, 256, kRM, 64) ||
      !make_tmap_bf16_2d(&tk, a->k_idx, (uint64_t)a->n, 128, 256, kRH, 64))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(prefill_route_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kRouteSmem);
  if (e != cudaSuccess) return e;
  prefill_route_kernel<<<rp.grid, kRThreads, kRouteSmem, s>>>(tq, tk, p);
  launches_add(1, s);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  prefill_densify_kernel<<<a->T, 256, 0, s>>>(p, out->dval, out->dtok, out->dlen, out->flag, rp.ldd);
  launches_add(1, s);
  return cudaGetLastError();
}

}  // namespace clsa
