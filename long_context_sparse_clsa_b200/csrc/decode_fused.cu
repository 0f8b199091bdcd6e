// Fused CLSA decode step: one persistent cooperative launch that scores, selects,
// gathers and attends.
//
//   routing equation   I = q_idx . K_idx^T ,  S = TopK(I, k)      (once per token)
//   per-layer equation O^(l) = softmax(Q^(l) K_S^T / sqrt(d)) V_S  (every layer)
// (picx.dev CLSA summary, Methodology > Architecture Overview; scale from the
// zhichai.net post, Background; gather by the shared index from its "Selector").
//
// One CTA per SM.  Each sequence b gets a group of C_b CTAs, in proportion to its
// length; CTA c of the group owns the contiguous token slice [r0, r1).
//
//  1. Scan.  16 lanes per 256-byte K_idx row, 16-byte non-allocating loads with
//     8 rows in flight per lane group, fp32 dot product, shuffle reduce.  (Measured
//     on B200: deep plain loads stream a 32 MiB slice set faster than a 1-D bulk-copy
//     ring with one CTA per SM.)  Scores stay on chip and go to global memory
//     (L2-resident), and feed a 12-bit key histogram of the slice.
//  2. Candidates.  From its own histogram a CTA picks the bound E: the lowest bin edge
//     with at most win of its tokens at or above it.  It writes those tokens, in token
//     order, to its window of the candidate list, and adds its histogram bins at or
//     above E into the group's coarse histogram in global memory (L2 reductions), with
//     E and its largest key folded into group maxima.  No CTA waits for another before
//     this point.
//  3. One barrier for the group.  Every CTA then reads the coarse histogram between the
//     largest bound E_max and the largest key.  It counts every token of those bins (each
//     CTA added all its bins at or above its own E <= E_max), so it gives the boundary
//     bin of the k_eff-th key and the count above it; only the candidates of that bin are
//     histogrammed again (12 more key bits), and the few keys of the boundary sub-bin
//     are ranked exactly (ties to the earlier list position = lower token index).  If
//     fewer than k_eff tokens lie at or above E_max, or the sub-bin holds heavy ties,
//     the same selection runs digit by digit over the whole row of scores.  Selected
//     tokens are ranked in ascending token order from per-window counts; each CTA
//     writes its own window's share of idx and keeps the tokens of its attention unit.
//  4. Attention.  A unit is (KV head g, split s of the selected ranks); its rows
//     are all L*G (layer, query head) pairs of head g, so every selected K/V row is
//     read once for all layers.  tcgen05.mma bf16 -> fp32 in TMEM over 64-token
//     chunks (S = Q K^T, then P V with V as an MN-major operand), online softmax in
//     exp2 with the output accumulated in TMEM (rescaled only when the max jumps).
//  5. Each split publishes its partial with a flag; the splits of one head merge each
//     other's partials (log-sum-exp rule) as their flags appear.
//
// Every wait is bounded (kWaitLimitNs); running out records CLSA_ERR_TIMEOUT.
#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstdlib>

#include "common.cuh"
#include "kernels.h"
#include "tcgen05.cuh"

namespace clsa {

namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kBins = 4096;          // digit histograms of the selection
constexpr int kTauBits = 12;          // key bits of the candidate-bound histogram
constexpr int kTauBins = 1 << kTauBits;
constexpr int kScanU = 4;             // rows per lane group per scan stage (the reduction assumes 4)
constexpr int kScanS = 4;             // scan stages in flight (the whole of `big`)
constexpr int kMaxRows = 128;         // L*G rows per unit (8 m-tiles x 2 token sets = 16 warps)
constexpr int kD = 128;               // head dim of the fused path
constexpr int kSTR = kD + 8;          // padded bf16 row in shared memory
constexpr int kMaxUnitTok = 4096;     // tokens one unit can hold (k <= 4096); also slice scores kept on chip
constexpr int kCandCap = 16384;       // candidate slots kept in shared memory (key + index)
constexpr int kMaxGroups = 256;       // CTAs per launch
constexpr int kMaxDevices = 64;       // host-side per-device state
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// per-row global state (u32 words).  The group histogram of 16-bit key bins has two
// copies: launch e of a row uses copy e & 1 and the bin-range words of slot e & 3; at its
// start it clears the bins copy (e - 1) & 1 had touched (range slot (e - 1) & 3) and zeroes
// slot (e + 1) & 3, so no CTA clears shared state at the end of a launch.  e is the row's
// own counter (the last CTA of the launch adds one for every row it processed).
constexpr int kH16Bits = 16;
constexpr int kH16Bins = 1 << kH16Bits;
constexpr int kRowEpoch = 0;                      // the row's launch counter
constexpr int kRowRange = 4;                      // [4][4] per epoch slot: E_max, key max, (kH16Bins - 1 - lowest bin), -
constexpr int kRowBar = 32;                       // row-group barrier state [2]
constexpr int kRowFlag = 256;                     // [kMaxGroups] per CTA of the group: its split partial
                                                  // is written (the row's launch counter + 1)
constexpr int kRowH16 = 512;                      // [2][kH16Bins] group histograms of the 16-bit key bins
constexpr int kRowWords = kRowH16 + 2 * kH16Bins;

struct FusedParams {
  const __nv_bfloat16* q_idx;
  const __nv_bfloat16* k_idx;
  const __nv_bfloat16* K;
  const __nv_bfloat16* V;
  const __nv_bfloat16* Q;
  const int32_t* seq_lens;
  __nv_bfloat16* O;
  int32_t* idx;
  int32_t* count;
  float* lse;
  float* scores;       // [B][n_max]
  uint32_t* row_ws;    // [B][kRowWords]
  uint32_t* leave;     // CTAs of this launch past their last count barrier
  uint32_t* cand_key;  // [B][kCandCap]  candidate keys, the group's windows back to back (0 = empty slot)
  int32_t* cand_tok;   // [B][kCandCap]
  __nv_bfloat16* Op;   // [gridDim][rows][D]  split partials (unnormalised), one slot per CTA
  float* Ml;           // [gridDim][rows][4]  (m, l, -, -): one 16-byte slot per row
  void* ws_header;
  unsigned long long* trace;  // [gridDim][16] globaltimer stamps per phase, or null
  int B, n_max, k, L, Hq, Hkv, G, rows, nsplit_max;
  float scale_log2;
  float pf_mult;       // K/V rows of a CTA's likely-selected tokens are prefetched into L2:
  uint32_t pf_add;     // its top pf_mult * e + pf_add tokens (to the key-bin granularity)
};

constexpr int kTraceSlots = 64;
__device__ __forceinline__ void stamp(const FusedParams& p, int phase) {
  if (p.trace && threadIdx.x == 0) {
    p.trace[blockIdx.x * kTraceSlots + phase] = globaltimer_ns();
    if (phase == 1) p.trace[blockIdx.x * kTraceSlots + 29] = clock64();  // SM clock calibration
    if (phase == 9) p.trace[blockIdx.x * kTraceSlots + 30] = clock64();
  }
}

struct Plan {
  int b, c, Cb, start;   // sequence, index in its group, group size, group's first CTA (b < 0: idle)
  int len, keff, r0, r1;
  int nsplit;            // token splits per KV head in this group
  int unit_g0, unit_step, nunits_here;  // heads this CTA attends: g0, g0+step, ... (count)
  int split;             // split index of this CTA's units
  int tok0, tok1;        // selected-rank range of the unit
  int win;               // candidate window per CTA (slots, a multiple of 4)
};

struct Smem {
  Plan plan;
  uint64_t bar_s, bar_o;  // attention: S and O_c MMAs complete
  uint32_t tmem_base;
  int abort_flag;
  uint32_t tau_key;
  uint32_t theta, ties_needed;
  int sel_bin;
  uint32_t sel_above;
  uint32_t warp_tot[kWarps];
  uint32_t warp_tot2[kWarps + 1];
  int seg_off[kMaxGroups + 1];
  int seg_cnt[kMaxGroups];
  uint32_t b16, above16, m16;
  int sel_ok;
  int leave_last;
  uint32_t live_rows[4];                // rows with tokens (the fused path takes B <= 128)
  __align__(16) uint32_t row_hdr[20];   // the row's epoch and range slots (async copy at entry)
  uint32_t grp_emax, grp_kmax;
  __align__(16) uint32_t hist[kBins];
  uint32_t red_max[kWarps];
  uint32_t theta_key, theta_pos;
  int list_n;
  uint32_t slice_max, pf_key;
  union {                          // slice scores until the candidates are out, then the
    float score[kMaxUnitTok];      // boundary-bin list of the selection, then unit tokens
    int unit_tok[kMaxUnitTok];
    struct {
      uint32_t list_key[1024];
      int list_pos[1024];
    };
  };
  float cm[512], cl[512];          // split-combine staging (m, l per row x split)
};
// dynamic shared memory: [Smem][sQ: kMaxRows x kSTR bf16][big: 128 KiB, reused by phase]
constexpr size_t kSmemQ = (size_t)kMaxRows * kSTR * 2;
constexpr size_t kSmemBig = 128 * 1024;
constexpr size_t smem_bytes() { return align_up(sizeof(Smem), 128) + kSmemQ + kSmemBig; }
static_assert(kScanS * kScanU * kThreads * 16 <= (int)kSmemBig, "scan ring exceeds big");
static_assert(kScanU == 4, "the scan reduction handles 4 rows per lane group");
static_assert(kTauBins <= kBins, "the slice histogram lives in Smem::hist");

// ---------------------------------------------------------------------------
// small block-wide helpers (512 threads)
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t block_scan(uint32_t v, uint32_t* warp_tot, uint32_t* total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_tot[w] = x;
  __syncthreads();
  if (w == 0) {
    uint32_t t = lane < kWarps ? warp_tot[lane] : 0u;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += y;
    }
    if (lane < kWarps) warp_tot[lane] = t;
  }
  __syncthreads();
  const uint32_t before = (w > 0 ? warp_tot[w - 1] : 0u) + x - v;
  *total = warp_tot[kWarps - 1];
  __syncthreads();
  return before;
}

// bin T with sum(hist[>T]) < need <= sum(hist[>=T]); sm.sel_bin = -1 if the total is below need
__device__ void select_bin(Smem& sm, int nbins, uint32_t need) {
  const int per = (nbins + kThreads - 1) / kThreads;
  const int hi = nbins - threadIdx.x * per;
  const int lo = max(hi - per, 0);
  uint32_t local = 0;
  for (int i = lo; i < hi; ++i) local += sm.hist[i];
  if (threadIdx.x == 0) sm.sel_bin = -1;
  uint32_t total;
  const uint32_t before = block_scan(hi > 0 ? local : 0u, sm.warp_tot, &total);
  if (hi > 0 && before < need && need <= before + local) {
    uint32_t acc = before;
    for (int i = hi - 1; i >= lo; --i) {
      const uint32_t c = sm.hist[i];
      if (acc + c >= need) {
        sm.sel_bin = i;
        sm.sel_above = acc;
        break;
      }
      acc += c;
    }
  }
  __syncthreads();
}

// exclusive prefix of a 0/1 flag in thread order (ballots); *total = block total
__device__ __forceinline__ uint32_t block_flag_scan(bool flag, uint32_t* warp_tot, uint32_t* total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const uint32_t bal = __ballot_sync(0xffffffffu, flag);
  if (lane == 0) warp_tot[w] = __popc(bal);
  __syncthreads();
  if (w == 0) {
    const uint32_t t = lane < kWarps ? warp_tot[lane] : 0u;
    uint32_t x = t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane < kWarps) warp_tot[lane] = x - t;
    if (lane == 31) warp_tot[kWarps] = x;
  }
  __syncthreads();
  const uint32_t before = warp_tot[w] + __popc(bal & ((1u << lane) - 1u));
  *total = warp_tot[kWarps];
  __syncthreads();
  return before;
}

// Exclusive prefix of v over the block in thread order with a single barrier: every warp
// reads the 16 warp totals itself (redux).  wt [kWarps] must not be written again until a
// later barrier has passed (alternate two arrays between back-to-back calls).
__device__ __forceinline__ uint32_t block_excl_scan1(uint32_t v, uint32_t* wt, uint32_t* total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  uint32_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) wt[w] = incl;
  __syncthreads();
  const uint32_t t = lane < kWarps ? wt[lane] : 0u;
  *total = __reduce_add_sync(0xffffffffu, t);
  return __reduce_add_sync(0xffffffffu, lane < w ? t : 0u) + incl - v;
}

// histogram increment (plain shared atomics measured ~9x faster here than warp aggregation)
__device__ __forceinline__ void hist_add(uint32_t* hist, uint32_t bin) { atomicAdd(&hist[bin], 1u); }

// Find bin T with sum(hist[>T]) < need <= sum(hist[>=T]) over hist[0, nbins), nbins a
// multiple of 2048.  Warp w covers a contiguous range from the top, each lane a run of
// nbins/512 bins read with 16-byte loads; two block syncs.  Writes sm.sel_bin (-1 if
// the total is below need) and sm.sel_above.
// With scale > 0 the target is max(1, floor(need * total * scale)), total = the histogram sum.
__device__ void select_bin_wide(Smem& sm, const uint32_t* hist, int nbins, uint32_t need, float scale = 0.f) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int per_lane = nbins / kThreads;
  const int hi = nbins - (w * 32 + lane) * per_lane;
  uint32_t local = 0;
  for (int q = 0; q < per_lane; q += 4) {
    const uint4 x = *reinterpret_cast<const uint4*>(hist + hi - per_lane + q);
    local += x.x + x.y + x.z + x.w;
  }
  uint32_t incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) sm.warp_tot[w] = incl;
  if (threadIdx.x == 0) sm.sel_bin = -1;
  __syncthreads();
  uint32_t before = incl - local;
  {
    const uint32_t wt = lane < kWarps ? sm.warp_tot[lane] : 0u;
    uint32_t pre = lane < w ? wt : 0u, total = wt;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      pre += __shfl_xor_sync(0xffffffffu, pre, o);
      total += __shfl_xor_sync(0xffffffffu, total, o);
    }
    before += pre;
    if (scale > 0.f) need = max(1u, (uint32_t)((float)need * (float)total * scale));
  }
  if (before < need && need <= before + local) {
    uint32_t acc = before;
    for (int i = hi - 1; i >= hi - per_lane; --i) {
      const uint32_t c = hist[i];
      if (acc + c >= need) {
        sm.sel_bin = i;
        sm.sel_above = acc;
        break;
      }
      acc += c;
    }
  }
  __syncthreads();
}

// ---------------------------------------------------------------------------
// work partition (computed identically by every CTA from seq_lens)
// ---------------------------------------------------------------------------
// live: bit b set for every row with tokens (rows < 128)
__device__ void make_plan(const FusedParams& p, Plan& pl, uint32_t* live) {
  const int ncta = gridDim.x;
  long long total = 0;
  int nb = 0;
#pragma unroll 1
  for (int w = 0; w < 4; ++w) live[w] = 0u;
#pragma unroll 1
  for (int b = 0; b < p.B; ++b) {
    const int len = max(0, min(p.seq_lens[b], p.n_max));
    total += len;
    nb += len > 0;
    if (len > 0) live[b >> 5] |= 1u << (b & 31);
  }
  pl.b = -1;
  if (nb == 0) return;
  // A sequence's CTAs scan its slice (work in proportion to its length) and then attend: Hkv
  // head units of k_eff tokens whatever its length.  With fewer than Hkv CTAs a CTA runs
  // several head units one after the other.  So with several sequences (when the grid has
  // Hkv CTAs for each) a sequence whose length share of the grid falls below Hkv CTAs is
  // pinned at Hkv, and the others share the remaining CTAs in proportion to their lengths
  // (re-split while new sequences pin: each pass pins one or more, or stops); then every
  // unpinned share is at least Hkv.  Otherwise CTAs go one per sequence plus the rest in
  // proportion to length; a lone sequence takes the whole grid.
  const bool grouped = nb >= 2 && ncta >= p.Hkv * nb;
  uint64_t pin0 = 0u, pin1 = 0u;  // pinned sequences (bit b of pin0, or b - 64 of pin1)
  auto pinned = [&](int b) { return ((b < 64 ? pin0 >> b : pin1 >> (b - 64)) & 1u) != 0u; };
  long long tot2 = total;  // length of the unpinned sequences
  int rem = ncta;          // CTAs they share
  if (grouped) {
#pragma unroll 1
    for (int round = 0; round < nb; ++round) {
      bool changed = false;
#pragma unroll 1
      for (int b = 0; b < p.B; ++b) {
        const int len = max(0, min(p.seq_lens[b], p.n_max));
        if (len == 0 || pinned(b)) continue;
        if ((long long)rem * len < (long long)p.Hkv * tot2) {
          if (b < 64) pin0 |= 1ull << b;
          else pin1 |= 1ull << (b - 64);
          rem -= p.Hkv;
          tot2 -= len;
          changed = true;
        }
      }
      if (!changed) break;
    }
  }
  const int spare = ncta - nb;
  int start = 0;
#pragma unroll 1
  for (int b = 0; b < p.B; ++b) {
    const int len = max(0, min(p.seq_lens[b], p.n_max));
    if (len == 0) continue;
    const int Cb = !grouped ? 1 + (int)((long long)spare * len / total)
                   : pinned(b) ? p.Hkv
                                                      : (int)((long long)rem * len / tot2);
    if ((int)blockIdx.x < start + Cb) {
      pl.b = b;
      pl.start = start;
      pl.c = blockIdx.x - start;
      pl.Cb = Cb;
      pl.len = len;
      pl.keff = min(p.k, len);
      const int chunk = (len + Cb - 1) / Cb;
      pl.r0 = min(len, pl.c * chunk);
      pl.r1 = min(len, pl.r0 + chunk);
      // window: 1.5 e + 4 sqrt(e) + 4 slots for the expected share e = k_eff / C_b of the
      // TopK per CTA (a CTA holding more TopK tokens than its window sends the group to
      // the whole-row path); all windows of the group fit kCandCap
      const float e = (float)pl.keff / (float)Cb;
      const int wn = ((int)ceilf(1.5f * e + 4.f * sqrtf(e) + 4.f) + 3) & ~3;
      pl.win = max(4, min(wn, (kCandCap / Cb) & ~3));
      break;
    }
    start += Cb;
  }
  if (pl.b < 0) return;
  if (pl.Cb >= p.Hkv) {
    pl.nsplit = pl.Cb / p.Hkv;
    const bool active = pl.c < p.Hkv * pl.nsplit;
    pl.unit_g0 = active ? pl.c / pl.nsplit : 0;
    pl.unit_step = p.Hkv;
    pl.nunits_here = active ? 1 : 0;
    pl.split = active ? pl.c % pl.nsplit : 0;
  } else {
    pl.nsplit = 1;
    pl.unit_g0 = pl.c;
    pl.unit_step = pl.Cb;
    pl.nunits_here = (p.Hkv - pl.c + pl.Cb - 1) / pl.Cb;
    pl.split = 0;
  }
  const int per = (pl.keff + pl.nsplit - 1) / pl.nsplit;
  pl.tok0 = min(pl.keff, pl.split * per);
  pl.tok1 = min(pl.keff, pl.tok0 + per);
}

// The count-barrier words are zeroed by the last CTA to leave them: every CTA counts
// itself in p.leave right after its last count barrier and its last read of the group
// state (leave_issue) and reads the old count only at its end (leave_finish), so no
// barrier waits on that atomic.  The
// CTA that saw gridDim.x - 1 runs after every CTA has stopped polling, and the next
// launch starts from zeroed words.
// A relaxed add: the CTA does not wait for it (an acquire here would hold the whole CTA for
// an L2 round trip); its old value is read only at the end, in leave_finish.
__device__ __forceinline__ uint32_t leave_issue(const FusedParams& p) {
  return threadIdx.x == 0 ? atomicAdd(p.leave, 1u) : 0u;
}
__device__ __forceinline__ void red_max_gpu(uint32_t* p, uint32_t v) {
  asm volatile("red.relaxed.gpu.global.max.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ void red_add_gpu(uint32_t* p, uint32_t v) {
  asm volatile("red.relaxed.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Called by every thread of the CTA.  The last CTA to leave returns the barrier words to
// zero and advances the launch counter of every row it processed (a row with tokens).
__device__ void leave_finish(const FusedParams& p, Smem& sm, uint32_t old) {
  if (threadIdx.x == 0) sm.leave_last = old == gridDim.x - 1;
  __syncthreads();
  if (!sm.leave_last) return;
  for (int b = threadIdx.x; b < p.B; b += kThreads) {
    uint32_t* rw = p.row_ws + (size_t)b * kRowWords;
    rw[kRowBar] = 0u;
    if ((sm.live_rows[b >> 5] >> (b & 31)) & 1u) red_add_gpu(rw + kRowEpoch, 1u);
  }
  if (threadIdx.x == 0) *p.leave = 0u;
}

// The row's header (launch counter and range slots) into shared memory by async copies
// (5 x 16 bytes), issued with the first copies of the launch; read after the scan.
__device__ __forceinline__ void load_row_header(const FusedParams& p, Smem& sm, int b) {
  if (threadIdx.x < 5) cp_async_16(sm.row_hdr + 4 * threadIdx.x, p.row_ws + (size_t)b * kRowWords + 4 * threadIdx.x, 16);
  cp_async_commit();
}

// Launch e of a row: clear the bins launch e - 1 touched in the other histogram copy (the
// group's CTAs share the range), and zero the range slot of launch e + 1.
__device__ void clear_previous_copy(const FusedParams& p, const Smem& sm, const Plan& pl) {
  uint32_t* rw = p.row_ws + (size_t)pl.b * kRowWords;
  const uint32_t e = sm.row_hdr[kRowEpoch];
  const uint32_t* pr = sm.row_hdr + kRowRange + ((e - 1u) & 3u) * 4;
  const int lo = kH16Bins - 1 - (int)pr[2], hi = (int)(pr[1] >> (32 - kH16Bits));
  uint32_t* old = rw + kRowH16 + ((e - 1u) & 1u) * kH16Bins;
  for (int i = lo + pl.c * kThreads + (int)threadIdx.x; i <= hi; i += pl.Cb * kThreads) old[i] = 0u;
  if (pl.c == 0 && threadIdx.x < 4) rw[kRowRange + ((e + 1u) & 3u) * 4 + threadIdx.x] = 0u;
}

template <int DIDX>
__device__ __forceinline__ float row_dot(const uint4 v, const float (&q)[8]) {
  float a0, a1, a2, a3, a4, a5, a6, a7;
  unpack_bf16x2(v.x, a0, a1);
  unpack_bf16x2(v.y, a2, a3);
  unpack_bf16x2(v.z, a4, a5);
  unpack_bf16x2(v.w, a6, a7);
  float acc = q[0] * a0;
  acc = fmaf(q[1], a1, acc);
  acc = fmaf(q[2], a2, acc);
  acc = fmaf(q[3], a3, acc);
  acc = fmaf(q[4], a4, acc);
  acc = fmaf(q[5], a5, acc);
  acc = fmaf(q[6], a6, acc);
  acc = fmaf(q[7], a7, acc);
  return acc;
}

// Rows [j0, j1) of the slice, streamed through a ring of S stages of U rows per lane
// group in shared memory (16-byte cp.async, L2 only).  Every thread reads back only the
// chunks it copied, so no barrier is needed: S - 1 stages stay in flight while one is
// reduced.
// stage st of the ring: rows base0 + grp + u * GROUPS (u < kScanU) of [.., j1)
template <int DIDX>
__device__ __forceinline__ void scan_issue(uint4* ring, const __nv_bfloat16* src, int st, int base0, int j1) {
  constexpr int LPR = DIDX / 8;
  constexpr int GROUPS = kThreads / LPR;
  const int grp = threadIdx.x / LPR, sub = threadIdx.x % LPR;
#pragma unroll
  for (int u = 0; u < kScanU; ++u) {
    const int j = base0 + grp + u * GROUPS;
    if (j < j1) cp_async_16(ring + (st * kScanU + u) * kThreads + threadIdx.x, src + (size_t)j * DIDX + sub * 8, 16);
  }
  cp_async_commit();  // one group per stage, empty or not
}
// the ring's first kScanS stages: the stream starts as soon as the slice is known
template <int DIDX>
__device__ __forceinline__ void scan_start(uint4* ring, const __nv_bfloat16* src, int j0, int j1) {
  constexpr int ROWS = kThreads / (DIDX / 8) * kScanU;
  const int nst = (j1 - j0 + ROWS - 1) / ROWS;
#pragma unroll
  for (int st = 0; st < kScanS; ++st) {
    if (st < nst) scan_issue<DIDX>(ring, src, st, j0 + st * ROWS, j1);
    else cp_async_commit();
  }
}
// reduce the stream begun by scan_start (no other async copy committed since), refilling
// each stage as it is read
template <int DIDX>
__device__ __forceinline__ void scan_rows(const FusedParams& p, Smem& sm, uint32_t* th, uint4* ring,
                                          const __nv_bfloat16* src, float* sc, const float (&q)[8], int j0, int j1,
                                          int nrows, bool hist) {
  constexpr int LPR = DIDX / 8;                 // lanes per row (16-byte chunks)
  constexpr int GROUPS = kThreads / LPR;        // row groups per CTA
  const int grp = threadIdx.x / LPR, sub = threadIdx.x % LPR;
  constexpr int ROWS = GROUPS * kScanU;         // rows per stage
  auto issue = [&](int st, int base0) { scan_issue<DIDX>(ring, src, st, base0, j1); };
  const int nst = (j1 - j0 + ROWS - 1) / ROWS;  // the same for every thread (whole-warp shuffles below)
  for (int it = 0; it < nst; ++it) {
    cp_async_wait<kScanS - 1>();  // stage it has landed
    const int st = it % kScanS;
    const int base0 = j0 + it * ROWS;
    // the stage's 4 rows per lane group: 4 independent partial dot products per lane, then
    // one transposed reduction over the group's LPR lanes (each level sends the half of
    // the rows the partner keeps): 2 + 1 + log2(LPR / 4) shuffles for all 4 rows
    float acc[kScanU];
#pragma unroll
    for (int u = 0; u < kScanU; ++u) {
      const int j = base0 + grp + u * GROUPS;
      const uint4 v = j < j1 ? ring[(st * kScanU + u) * kThreads + threadIdx.x] : make_uint4(0, 0, 0, 0);
      acc[u] = row_dot<DIDX>(v, q);
    }
    const bool hi_a = (sub & (LPR / 2)) != 0, hi_b = (sub & (LPR / 4)) != 0;
    float k0 = hi_a ? acc[2] : acc[0], k1 = hi_a ? acc[3] : acc[1];
    k0 += __shfl_xor_sync(0xffffffffu, hi_a ? acc[0] : acc[2], LPR / 2);
    k1 += __shfl_xor_sync(0xffffffffu, hi_a ? acc[1] : acc[3], LPR / 2);
    float tot = hi_b ? k1 : k0;
    tot += __shfl_xor_sync(0xffffffffu, hi_b ? k0 : k1, LPR / 4);
#pragma unroll
    for (int o = LPR / 8; o > 0; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
    {
      const int u = (hi_a ? 2 : 0) + (hi_b ? 1 : 0);  // the row this lane now holds in full
      const int j = base0 + grp + u * GROUPS;
      if ((sub & (LPR / 4 - 1)) == 0 && j < j1) {  // the stream is HBM-bound: store here
        if (nrows <= kMaxUnitTok) sm.score[j] = tot;
        __stcg(sc + j, tot);
        if (hist) atomicAdd(&th[float_key(tot) >> (32 - kTauBits)], 1u);
      }
    }
    if (it + kScanS < nst) issue(st, j0 + (it + kScanS) * ROWS);  // refill the slot just read
    else cp_async_commit();
  }
  cp_async_wait<0>();
}

__device__ __forceinline__ void load_q_tile(const FusedParams& p, int b, int g, unsigned char* sQa);

// this thread's 16-byte chunk of q_idx[b] (the chunk its scan lane multiplies)
template <int DIDX>
__device__ __forceinline__ uint4 load_q_chunk(const FusedParams& p, int b) {
  return *reinterpret_cast<const uint4*>(p.q_idx + (size_t)b * DIDX + (threadIdx.x % (DIDX / 8)) * 8);
}

// started: the stream was begun by scan_start at entry, and qv holds load_q_chunk of the
// sequence (both issued before the plan, so their latency overlaps it)
template <int DIDX>
// sQa: the attention unit's Q tile is loaded right behind the first stages of the stream
// (null: this CTA attends nothing)
__device__ bool scan_slice(const FusedParams& p, Smem& sm, uint32_t* th, unsigned char* ring, bool hist,
                           bool started, uint4 qv, unsigned char* sQa) {
  const Plan pl = sm.plan;  // a copy: loops below store to shared memory
  const int nrows = pl.r1 - pl.r0;
  const __nv_bfloat16* src = p.k_idx + ((size_t)pl.b * p.n_max + pl.r0) * DIDX;
  float* sc = p.scores + (size_t)pl.b * p.n_max + pl.r0;
  float q[8];
  {
    if (!started) qv = load_q_chunk<DIDX>(p, pl.b);
    unpack_bf16x2(qv.x, q[0], q[1]);
    unpack_bf16x2(qv.y, q[2], q[3]);
    unpack_bf16x2(qv.z, q[4], q[5]);
    unpack_bf16x2(qv.w, q[6], q[7]);
  }
  if (!started) {
    load_row_header(p, sm, pl.b);
    scan_start<DIDX>(reinterpret_cast<uint4*>(ring), src, 0, nrows);
  }
  if (sQa) load_q_tile(p, pl.b, pl.unit_g0, sQa);
  stamp(p, 24);
  for (int i = threadIdx.x; i < kTauBins; i += kThreads) th[i] = 0;
  __syncthreads();
  stamp(p, 14);
  scan_rows<DIDX>(p, sm, th, reinterpret_cast<uint4*>(ring), src, sc, q, 0, nrows, nrows, hist);
  stamp(p, 16);
  __syncthreads();
  return true;
}

// ---------------------------------------------------------------------------
// phase 2: candidate bound tau from the group histogram, candidate segment
// ---------------------------------------------------------------------------
constexpr int kCandRun = 8;  // tokens per thread per pass of the candidate writer (4096 per pass)

__device__ void write_candidates(const FusedParams& p, Smem& sm, const uint32_t* th) {
  const Plan pl = sm.plan;  // a copy: loops below store to shared memory
  uint32_t* rw = p.row_ws + (size_t)pl.b * kRowWords;
  const uint32_t epoch = sm.row_hdr[kRowEpoch];
  uint32_t* h16 = rw + kRowH16 + (epoch & 1u) * kH16Bins;
  uint32_t* rng = rw + kRowRange + (epoch & 3u) * 4;
  // The local bound E: the lower edge of the lowest 12-bit key bin such that the slice
  // holds at most win tokens at or above it (E = 0: every token).  Thread t holds the
  // eight bins 4088 - 8t .. 4095 - 8t; one scan from the top finds the bin.
  const int hi = kTauBins - 8 * threadIdx.x;  // this thread's bins: [hi - 8, hi)
  uint32_t h[8], local = 0;
  {
    const uint4 x0 = *reinterpret_cast<const uint4*>(th + hi - 8), x1 = *reinterpret_cast<const uint4*>(th + hi - 4);
    h[0] = x0.x, h[1] = x0.y, h[2] = x0.z, h[3] = x0.w, h[4] = x1.x, h[5] = x1.y, h[6] = x1.z, h[7] = x1.w;
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) local += h[i];
  {
    uint32_t top = 0;  // 1 + the highest non-empty bin of this thread's run (0: none)
#pragma unroll
    for (int i = 0; i < 8; ++i)
      if (h[i] != 0u) top = (uint32_t)(hi - 8 + i + 1);
    top = __reduce_max_sync(0xffffffffu, top);
    if ((threadIdx.x & 31) == 0) sm.red_max[threadIdx.x >> 5] = top;
    uint32_t total;
    const uint32_t before = block_excl_scan1(local, sm.warp_tot, &total);  // tokens in higher bins
    stamp(p, 42);
    if (threadIdx.x < 32) {  // warp 0: the slice's highest non-empty bin (redux over the warp maxima)
      const uint32_t m = __reduce_max_sync(0xffffffffu, threadIdx.x < kWarps ? sm.red_max[threadIdx.x] : 0u);
      // the upper edge of the highest non-empty bin bounds every key of the slice
      if (threadIdx.x == 0)
        sm.slice_max = m == 0 ? 0u : (m >= (uint32_t)kTauBins ? 0xFFFFFFFFu : (m << (32 - kTauBits)) - 1u);
    }
    const uint32_t win = (uint32_t)pl.win;
    if (threadIdx.x == 0 && total <= win) sm.tau_key = 0u;
    if (before <= win && before + local > win) {
      uint32_t acc = before;
#pragma unroll
      for (int i = 7; i >= 0; --i) {
        if (acc + h[i] > win) {  // bin hi - 8 + i would overflow: E is its upper edge
          const int bin = hi - 8 + i;  // the top bin alone overflowing: publish nothing
          sm.tau_key = bin + 1 < kTauBins ? ((uint32_t)(bin + 1)) << (32 - kTauBits) : 0xFFFFFFFFu;
          break;
        }
        acc += h[i];
      }
    }
    // the prefetch bound: the same rule for the likely selected tokens
    const uint32_t w2 = min(win, (uint32_t)ceilf(p.pf_mult * (float)pl.keff / (float)pl.Cb) + p.pf_add);
    if (threadIdx.x == 0 && total <= w2) sm.pf_key = 0u;
    if (before <= w2 && before + local > w2) {
      uint32_t acc = before;
#pragma unroll
      for (int i = 7; i >= 0; --i) {
        if (acc + h[i] > w2) {
          const int bin = hi - 8 + i;
          sm.pf_key = bin + 1 < kTauBins ? ((uint32_t)(bin + 1)) << (32 - kTauBits) : 0xFFFFFFFFu;
          break;
        }
        acc += h[i];
      }
    }
  }
  __syncthreads();
  stamp(p, 43);
  const uint32_t tau = sm.tau_key, pf = sm.pf_key;
  // This CTA's tokens with key >= tau, in token order, to its window of win slots; each one
  // adds 1 to its 16-bit bin of the group histogram.  Thread t takes a contiguous run of
  // the pass's tokens (all its keys loaded before any store), one block scan places them.
  const float* gsc = p.scores + (size_t)pl.b * p.n_max + pl.r0;
  const int n = pl.r1 - pl.r0;
  const bool on_chip = n <= kMaxUnitTok;
  uint32_t* ck = p.cand_key + (size_t)pl.b * kCandCap + (size_t)pl.c * pl.win;
  int32_t* ct = p.cand_tok + (size_t)pl.b * kCandCap + (size_t)pl.c * pl.win;
  uint32_t written = 0;
  int pass = 0;
#pragma unroll 1
  for (int base = 0; base < n; base += kThreads * kCandRun, ++pass) {
    const int nb = min(n - base, kThreads * kCandRun);
    const int run = (nb + kThreads - 1) / kThreads;
    const int j0 = base + (int)threadIdx.x * run, j1 = min(j0 + run, base + nb);
    uint32_t m = 0;  // bit u: token j0 + u is a candidate
#pragma unroll 1
    for (int j = j0; j < j1; ++j)
      m |= (uint32_t)(float_key(on_chip ? sm.score[j] : __ldcg(gsc + j)) >= tau) << (j - j0);
    uint32_t tot;
    const uint32_t pos0 = written + block_excl_scan1((uint32_t)__popc(m), (pass & 1) ? sm.warp_tot : sm.warp_tot2, &tot);
    stamp(p, 44);
    uint32_t pos = pos0;
#pragma unroll 1
    while (m != 0u) {
      const int j = j0 + __ffs(m) - 1;
      m &= m - 1u;
      if (pos < (uint32_t)pl.win) {
        const uint32_t key = float_key(on_chip ? sm.score[j] : __ldcg(gsc + j));
        const int tok = pl.r0 + j;
        __stcg(ck + pos, key);
        __stcg(ct + pos, tok);
        red_add_gpu(h16 + (key >> (32 - kH16Bits)), 1u);
        if (key >= pf) {  // a likely TopK token: its K and V rows (all heads) into L2 now
          const size_t row = ((size_t)pl.b * p.n_max + tok) * p.Hkv * kD;
          bulk_prefetch_l2(p.K + row, (uint32_t)(p.Hkv * kD * 2));
          bulk_prefetch_l2(p.V + row, (uint32_t)(p.Hkv * kD * 2));
        }
      }
      ++pos;
    }
    written += tot;
  }
  for (int i = (int)written + threadIdx.x; i < pl.win; i += kThreads) __stcg(ck + i, 0u);  // empty slots
  if (threadIdx.x == 0) {  // E and the key bound into the group maxima, the lowest bin touched
    red_max_gpu(rng + 0, tau);
    red_max_gpu(rng + 1, sm.slice_max);
    if (tau != 0xFFFFFFFFu) red_max_gpu(rng + 2, (uint32_t)(kH16Bins - 1 - (int)(tau >> (32 - kH16Bits))));
  }
}

// ---------------------------------------------------------------------------
// phase 3: exact TopK over the candidate positions p in [0, P)
//   fast: keys/tokens in shared memory (concatenated segments, token order)
//   slow: the whole row of scores (position = token)
// ---------------------------------------------------------------------------
struct CandSrc {
  const uint32_t* skey;
  const int32_t* stok;
  const float* row_scores;
  bool fast;
  __device__ __forceinline__ uint32_t key(int i) const {
    return fast ? skey[i] : float_key(__ldcg(row_scores + i));
  }
  __device__ __forceinline__ int tok(int i) const { return fast ? stok[i] : i; }
};

// digit histograms; leaves theta and ties_needed in sm
__device__ void resolve_theta(Smem& sm, const CandSrc& src, int P, uint32_t keff, void* ws_header) {
  for (int i = threadIdx.x; i < kBins; i += kThreads) sm.hist[i] = 0;
  __syncthreads();
  for (int i = threadIdx.x; i < P; i += kThreads) hist_add(sm.hist, src.key(i) >> 20);
  __syncthreads();
  select_bin_wide(sm, sm.hist, kBins, keff);
  if (sm.sel_bin < 0) {  // fewer candidates than k_eff: cannot happen for a clean workspace
    if (threadIdx.x == 0) {
      record_error(ws_header, CLSA_ERR_BAD_INDEX, -1);
      sm.theta = 0xFFFFFFFFu;
      sm.ties_needed = 0;
    }
    __syncthreads();
    return;
  }
  const uint32_t t1 = (uint32_t)sm.sel_bin;
  uint32_t need = keff - sm.sel_above;
  __syncthreads();
  for (int i = threadIdx.x; i < kBins; i += kThreads) sm.hist[i] = 0;
  __syncthreads();
  for (int i = threadIdx.x; i < P; i += kThreads) {
    const uint32_t k = src.key(i);
    if ((k >> 20) == t1) hist_add(sm.hist, (k >> 8) & 0xFFFu);
  }
  __syncthreads();
  select_bin_wide(sm, sm.hist, kBins, need);
  const uint32_t p2 = (t1 << 12) | (uint32_t)sm.sel_bin;
  need -= sm.sel_above;
  __syncthreads();
  for (int i = threadIdx.x; i < 256; i += kThreads) sm.hist[i] = 0;
  __syncthreads();
  for (int i = threadIdx.x; i < P; i += kThreads) {
    const uint32_t k = src.key(i);
    if ((k >> 8) == p2) hist_add(sm.hist, k & 0xFFu);
  }
  __syncthreads();
  select_bin(sm, 256, need);
  if (threadIdx.x == 0) {
    sm.theta = (p2 << 8) | (uint32_t)sm.sel_bin;
    sm.ties_needed = need - sm.sel_above;
  }
  __syncthreads();
}

// rank the selected positions in order; keep the unit's tokens, write this CTA's share of idx
__device__ void compact_selected(const FusedParams& p, Smem& sm, const CandSrc& src, int P) {
  const Plan pl = sm.plan;  // a copy: loops below store to shared memory
  const uint32_t theta = sm.theta, ties = sm.ties_needed;
  int32_t* out = p.idx + (size_t)pl.b * p.k;
  uint32_t eq_seen = 0, sel_seen = 0;
  for (int base = 0; base < P; base += kThreads) {
    const int i = base + threadIdx.x;
    const bool valid = i < P;
    const uint32_t k = valid ? src.key(i) : 0u;
    const bool gt = valid && k > theta, eq = valid && k == theta;
    uint32_t eq_tot, s_tot;
    const uint32_t er = eq_seen + block_flag_scan(eq, sm.warp_tot2, &eq_tot);
    const bool s = gt || (eq && er < ties);
    const uint32_t rank = sel_seen + block_flag_scan(s, sm.warp_tot2, &s_tot);
    if (s) {
      const int t = src.tok(i);
      if ((int)rank >= pl.tok0 && (int)rank < pl.tok1) sm.unit_tok[rank - pl.tok0] = t;
      if (t >= pl.r0 && t < pl.r1 && (int)rank < pl.keff) out[rank] = t;
    }
    eq_seen += eq_tot;
    sel_seen += s_tot;
  }
  __syncthreads();
}

// ---------------------------------------------------------------------------
// phase 3 (fast path): the candidate windows of the group are landing in shared memory
// (skey: keys back to back in CTA order, each window in token order, empty slots key 0).
//   a. E_max, the key bound and the group histogram of 16-bit key bins between them (one
//      round trip: the 512 bins above this CTA's own bound, which hold that range unless
//      it is wider) give the bin B holding the k_eff-th key and the count above it;
//   b. thread t holds a contiguous run of slots in registers; the keys of bin B are listed;
//   c. each listed key is ranked exactly (key descending, slot ascending = token
//      ascending): theta is the (key, slot) of the k_eff-th;
//   d. the selected slots are ranked in slot order = ascending token order by one block
//      scan of the per-thread counts; the CTA keeps its unit's tokens and writes idx for
//      its own window.
// Returns false when the windows cannot decide (fewer than k_eff tokens at or above
// E_max, or more than 1024 keys in bin B): the whole-row path runs.
// ---------------------------------------------------------------------------
__device__ bool select_windows(const FusedParams& p, Smem& sm, const uint32_t* rw, const uint32_t* skey,
                               const int32_t* stok, int P) {
  const Plan pl = sm.plan;  // a copy: loops below store to shared memory
  const uint32_t keff = (uint32_t)pl.keff;
  const uint32_t epoch = sm.row_hdr[kRowEpoch];
  const uint32_t* h16 = rw + kRowH16 + (epoch & 1u) * kH16Bins;
  const uint32_t* rng = rw + kRowRange + (epoch & 3u) * 4;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    sm.sel_ok = 0;
    sm.list_n = 0;
  }
  const uint32_t emax = __ldcg(rng), kmax = __ldcg(rng + 1);
  int top = (int)(sm.tau_key >> (32 - kH16Bits)) + kThreads - 1;  // this CTA's bound <= E_max
  int bin = top - (int)threadIdx.x;
  uint32_t v = bin < kH16Bins ? __ldcg(h16 + bin) : 0u;
  if (emax == 0xFFFFFFFFu || kmax < emax) {
    cp_async_wait<1>();
    __syncthreads();
    return false;
  }
  const int lo = (int)(emax >> (32 - kH16Bits)), hi = (int)(kmax >> (32 - kH16Bits));
  uint32_t acc = 0;  // keys in the bins above the current run of 512
  int pass = 0;
  if (hi > top) {  // a range wider than the speculative run: runs of 512 from the top
    top = hi;
    bin = top - (int)threadIdx.x;
    v = __ldcg(h16 + bin);
  }
#pragma unroll 1
  for (;; ++pass) {
    const uint32_t x = bin >= lo && bin <= hi ? v : 0u;
    uint32_t tot;
    const uint32_t before = acc + block_excl_scan1(x, (pass & 1) ? sm.warp_tot2 : sm.warp_tot, &tot);
    if (before < keff && keff <= before + x) {
      sm.b16 = (uint32_t)bin;
      sm.above16 = before;
      sm.m16 = x;
      sm.sel_ok = 1;
    }
    if (pass == 0) cp_async_wait<1>();  // the window keys (the tokens may still be in flight)
    __syncthreads();
    if (sm.sel_ok || top - kThreads < lo) break;
    acc += tot;
    top -= kThreads;
    bin = top - (int)threadIdx.x;
    v = bin >= 0 ? __ldcg(h16 + bin) : 0u;
  }
  stamp(p, 4);
  if (!sm.sel_ok || sm.m16 > 1024u) return false;  // too few keys at or above E_max / heavy ties
  const uint32_t b16 = sm.b16, need = keff - sm.above16, m = sm.m16;
  // b. thread t takes the contiguous slots [t seg, t seg + seg) of the concatenated windows,
  //    four at a time (16-byte loads, a rolled loop: few instructions per slot); the keys of
  //    bin B go to the list.  Empty slots (key 0) never fall in bin B: B >= the bin of E_max,
  //    and every finite score has a key above 0x007FFFFF.
  const int seg = ((P + kThreads - 1) / kThreads + 3) & ~3;
  const int s0 = (int)threadIdx.x * seg, s1 = min(s0 + seg, P);
  uint32_t inb = 0;   // bit u: slot s0 + u is in bin B (seg <= 32)
  uint32_t above = 0; // slots of this thread in bins above B (all of them selected)
  {
#pragma unroll 1
    for (int u = 0; s0 + u < s1; u += 4) {
      const uint4 x = *reinterpret_cast<const uint4*>(skey + s0 + u);
      const uint32_t b0 = x.x >> (32 - kH16Bits), b1 = x.y >> (32 - kH16Bits), b2 = x.z >> (32 - kH16Bits),
                     b3 = x.w >> (32 - kH16Bits);
      inb |= (uint32_t)(b0 == b16) << u | (uint32_t)(b1 == b16) << (u + 1) | (uint32_t)(b2 == b16) << (u + 2) |
             (uint32_t)(b3 == b16) << (u + 3);
      above += (uint32_t)(b0 > b16) + (uint32_t)(b1 > b16) + (uint32_t)(b2 > b16) + (uint32_t)(b3 > b16);
    }
    const uint32_t n = (uint32_t)__popc(inb);
    if (__any_sync(0xffffffffu, n != 0u)) {  // warp-aggregated: one list reservation per warp
      uint32_t pre = n;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, pre, o);
        if (lane >= o) pre += y;
      }
      int base = 0;
      if (lane == 31) base = atomicAdd(&sm.list_n, (int)pre);
      base = __shfl_sync(0xffffffffu, base, 31) + (int)(pre - n);
      uint32_t mm = inb;
#pragma unroll 1
      while (mm != 0u) {
        const int u = __ffs(mm) - 1;
        mm &= mm - 1u;
        if (base < 1024) {
          sm.list_key[base] = skey[s0 + u];
          sm.list_pos[base] = s0 + u;
        }
        ++base;
      }
    }
  }
  __syncthreads();
  stamp(p, 19);
  if ((uint32_t)sm.list_n != m) {  // the windows disagree with the group histogram: cannot happen
    if (threadIdx.x == 0) record_error(p.ws_header, CLSA_ERR_BAD_INDEX, -3);
    return false;
  }
  // c. exact rank inside bin B: eight threads per listed key, each comparing it with every
  //    eighth key, then a three-step shuffle sum
#pragma unroll 1
  for (int e0 = 0; e0 < (int)m; e0 += kThreads / 8) {
    const int e = e0 + (threadIdx.x >> 3), part = threadIdx.x & 7;
    const bool live = e < (int)m;
    const uint32_t ke = live ? sm.list_key[e] : 0u;
    const int pe = live ? sm.list_pos[e] : 0;
    uint32_t r = 0;
#pragma unroll 1
    for (int f = part; f < (int)m; f += 8) {
      const uint32_t kf = sm.list_key[f];
      const int pf = sm.list_pos[f];
      r += kf > ke || (kf == ke && pf < pe);
    }
    r += __shfl_xor_sync(0xffffffffu, r, 1);
    r += __shfl_xor_sync(0xffffffffu, r, 2);
    r += __shfl_xor_sync(0xffffffffu, r, 4);
    if (live && part == 0 && r == need - 1) {
      sm.theta_key = ke;
      sm.theta_pos = (uint32_t)pe;
    }
  }
  __syncthreads();
  stamp(p, 20);
  // d. rank the selected slots (key > theta_key, or key == theta_key at a slot <= theta_pos) in
  //    slot order = ascending token order: one block scan over the per-thread counts (the
  //    slots above bin B, plus this thread's selected slots of bin B)
  const uint32_t tk = sm.theta_key, tp = sm.theta_pos;
  uint32_t cnt = above;
  {
    uint32_t mm = inb;
#pragma unroll 1
    while (mm != 0u) {
      const int u = __ffs(mm) - 1;
      mm &= mm - 1u;
      const uint32_t k = skey[s0 + u];
      cnt += k > tk || (k == tk && (uint32_t)(s0 + u) <= tp);
    }
  }
  uint32_t tot;
  stamp(p, 32);
  cp_async_wait<0>();  // the window tokens (visible to all after the scan's barrier)
  int r = (int)block_excl_scan1(cnt, sm.warp_tot2, &tot);
  stamp(p, 33);
  if (threadIdx.x == 0 && tot != keff) record_error(p.ws_header, CLSA_ERR_BAD_INDEX, -2);
  // e. the unit's tokens (ranks [tok0, tok1)) and idx for this CTA's own window: only the
  //    threads whose ranks meet the unit's range or whose slots meet the own window
  const int own0 = pl.c * pl.win, own1 = own0 + pl.win;
  int32_t* out = p.idx + (size_t)pl.b * p.k;
  const bool in_unit = r < pl.tok1 && r + (int)cnt > pl.tok0, in_own = s0 < own1 && s1 > own0;
  if (cnt != 0u && (in_unit || in_own)) {
#pragma unroll 1
    for (int u = 0; s0 + u < s1; u += 4) {
      const uint4 x = *reinterpret_cast<const uint4*>(skey + s0 + u);
      const int sl = s0 + u;
      uint32_t m4 = (uint32_t)(x.x > tk || (x.x == tk && (uint32_t)sl <= tp)) |
                    (uint32_t)(x.y > tk || (x.y == tk && (uint32_t)(sl + 1) <= tp)) << 1 |
                    (uint32_t)(x.z > tk || (x.z == tk && (uint32_t)(sl + 2) <= tp)) << 2 |
                    (uint32_t)(x.w > tk || (x.w == tk && (uint32_t)(sl + 3) <= tp)) << 3;
#pragma unroll 1
      while (m4 != 0u) {
        const int q = sl + __ffs(m4) - 1;
        m4 &= m4 - 1u;
        const int t = stok[q];
        if (r >= pl.tok0 && r < pl.tok1) sm.unit_tok[r - pl.tok0] = t;
        if (q >= own0 && q < own1 && r < pl.keff) out[r] = t;
        ++r;
      }
    }
  }
  stamp(p, 34);
  __syncthreads();
  return true;
}

// ---------------------------------------------------------------------------
// phase 4: attention of one unit (head g, tokens sm.unit_tok[0..ntok)), on the 5th
// generation tensor cores.  The unit's M = 128 rows (the L*G (layer, query head) rows of
// head g, zero above p.rows) stay in shared memory as the A operand; the tokens go in
// chunks of TOK (128 when the unit fits one chunk, else 64 in a 3-stage ring):
//   S = Q K_c^T        tcgen05.mma M128 N=TOK (K = d, 8 steps) -> TMEM
//   softmax            every warp: one row (its TMEM lane), TOK/4 of the chunk's columns;
//                      the chunk's row max is exchanged through shared memory, so the four
//                      warps of a row share one running max m
//   O_c = P_c V_c      P_c (bf16) in shared memory (A, K-major), V_c as the MN-major B
//                      operand straight from its row-major [token][d] tile;
//                      M128 N128 (K = TOK tokens) -> TMEM columns [128, 256)
//   O += P_c V_c in TMEM; O and l are rescaled by 2^(m_old - m) only when m jumps
// The S MMAs of chunk c + 1 are issued right behind the P V MMAs of chunk c (S is
// double-buffered in TMEM).  K/V chunks are gathered by 16-byte async copies into the
// 128-byte-swizzle layout, two chunks ahead.  Each tcgen05.mma costs tens of cycles to
// issue whatever its N, so the wide chunk halves the instruction count of a short unit.
// ---------------------------------------------------------------------------
constexpr uint32_t kQAtom = kMaxRows * 128;          // 16 KiB
constexpr uint32_t kTmemCols = 256;                  // S at [0, 128), O_c at [128, 256)
constexpr int kOPitch = kD + 8;                      // staged partial row, bf16 (272 bytes)
constexpr uint32_t kIdescPV = tc::idesc_bf16_f32(kMaxRows, kD) | (1u << 16);  // B (V) MN-major
static_assert(2 * kQAtom + 1024 <= kSmemQ, "Q tile exceeds its region");
static_assert(kMaxRows * kOPitch * 2 + 1024 <= kSmemBig, "partial staging exceeds big");

template <int TOK>
struct AttnShape {
  static constexpr int kStages = TOK == 64 ? 3 : 1;         // the wide chunk runs alone
  static constexpr uint32_t kKVAtom = TOK * 128;            // TOK rows x 128 bytes
  static constexpr uint32_t kKVTile = 2 * kKVAtom;          // K or V chunk, both 64-column atoms
  static constexpr uint32_t kPAtom = kMaxRows * 128;        // 64 tokens of P
  static constexpr int kPerThread = TOK / 4;                // S columns per thread
  static constexpr uint32_t kIdescQK = tc::idesc_bf16_f32(kMaxRows, TOK);
  static_assert(kStages * 2 * kKVTile + (TOK / 64) * kPAtom + 1024 <= kSmemBig, "attention tiles exceed big");
  static_assert(TOK * (TOK == 64 ? 2 : 1) <= 128, "S buffers overlap O");
};

__device__ __forceinline__ unsigned char* align1024(unsigned char* q) {
  return q + ((1024u - (smem_u32(q) & 1023u)) & 1023u);
}

// Q rows of head g in the 128-byte-swizzle K-major layout (two 64-column atoms)
__device__ __forceinline__ void load_q_tile(const FusedParams& p, int b, int g, unsigned char* sQa) {
  const float invG = 1.f / (float)p.G;  // floor((r + 0.5) / G) in fp32 is exact for r < 2^12
#pragma unroll
  for (int v = threadIdx.x; v < kMaxRows * 16; v += kThreads) {
    const int r = v >> 4, c = v & 15;
    unsigned char* dst = sQa + (c >> 3) * kQAtom + tc::sw128_offset(r, c & 7);
    if (r < p.rows) {
      const int l = (int)(((float)r + 0.5f) * invG), h = g * p.G + (r - l * p.G);
      cp_async_16(dst, p.Q + (((size_t)l * p.B + b) * p.Hq + h) * kD + c * 8, 16);
    } else {
      *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
    }
  }
  cp_async_commit();
}

// K and V rows of tokens [TOK c, TOK c + TOK) of the unit, same layout (rows past ntok: zero)
template <int TOK>
__device__ __forceinline__ void load_kv_chunk(const FusedParams& p, const Smem& sm, int b, int g, int len, int c,
                                              int ntok, unsigned char* dk, unsigned char* dv) {
#pragma unroll 1
  for (int v = threadIdx.x; v < TOK * 16; v += kThreads) {
    const int r = v >> 4, j = v & 15;
    const int i = c * TOK + r;
    const __nv_bfloat16* sk = p.K;
    const __nv_bfloat16* sv = p.V;
    int bytes = 0;
    if (i < ntok) {
      const int t = sm.unit_tok[i];
      if ((unsigned)t < (unsigned)len) {
        const size_t off = (((size_t)b * p.n_max + t) * p.Hkv + g) * kD + j * 8;
        sk += off;
        sv += off;
        bytes = 16;
      } else if (j == 0) {
        record_error(p.ws_header, CLSA_ERR_BAD_INDEX, ((long long)b << 32) | (unsigned)i);
      }
    }
    const uint32_t o = (uint32_t)(j >> 3) * AttnShape<TOK>::kKVAtom + tc::sw128_offset(r, j & 7);
    cp_async_16(dk + o, sk, bytes);
    cp_async_16(dv + o, sv, bytes);
  }
}

template <int N>
__device__ __forceinline__ void tmem_ld_row(uint32_t taddr, uint32_t (&v)[N]) {
  if constexpr (N == 16) tc::ld_32x32b_x16(taddr, v);
  else tc::ld_32x32b_x32(taddr, v);
}

// `it` counts the chunks this CTA has run (the phase of both MMA barriers).  TOK = 128
// only for a unit of at most 128 tokens (one chunk).
template <int TOK>
__device__ void attend_unit(const FusedParams& p, Smem& sm, unsigned char* sQa, unsigned char* kv, int g, int ntok,
                            bool q_loaded, bool kv0_issued, uint32_t tmem, uint32_t& it) {
  using SH = AttnShape<TOK>;
  constexpr int NPT = SH::kPerThread;
  const Plan pl = sm.plan;  // a copy: loops below store to shared memory
  const int b = pl.b;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q4 = warp & 3, cg = warp >> 2;  // TMEM lane quarter; column group
  const int row = q4 * 32 + lane;
  unsigned char* sP = kv + SH::kStages * 2 * SH::kKVTile;
  if (!q_loaded) load_q_tile(p, b, g, sQa);
  const int nch = (ntok + TOK - 1) / TOK;
#pragma unroll 1
  for (int c = 0; c < 2; ++c) {
    if (c == 0 && kv0_issued) continue;  // the caller issued chunk 0 as its own group
    if (c < nch && c < SH::kStages)
      load_kv_chunk<TOK>(p, sm, b, g, pl.len, c, ntok, kv + c * 2 * SH::kKVTile, kv + c * 2 * SH::kKVTile + SH::kKVTile);
    cp_async_commit();
  }
  stamp(p, 35);
  const uint32_t tl = tmem + ((uint32_t)(q4 * 32) << 16);
  const bool live = q4 * 32 < p.rows;  // warp-uniform: rows of this lane quarter exist
  float m = -INFINITY, lp = 0.f;
  bool dead = false;
  // S = Q K_c^T into TMEM columns [TOK (c & 1), +TOK); issued by thread 0
  auto issue_qk = [&](int c) {
    const uint32_t kb = smem_u32(kv + (c % SH::kStages) * 2 * SH::kKVTile);
#pragma unroll
    for (int ks = 0; ks < kD / 16; ++ks)
      tc::mma_bf16(tmem + (uint32_t)(TOK * (c & 1)),
                   tc::sw128_desc(smem_u32(sQa) + (ks >> 2) * kQAtom + (ks & 3) * 32),
                   tc::sw128_desc(kb + (ks >> 2) * SH::kKVAtom + (ks & 3) * 32), SH::kIdescQK, ks > 0);
    tc::mma_commit(&sm.bar_s);
  };
  if (nch > 0) {
    cp_async_wait<1>();  // chunk 0 (and the Q tile) landed
    fence_proxy_async_smem();
    tc::fence_before_sync();
    __syncthreads();
    stamp(p, 10);
    if (threadIdx.x == 0) {
      tc::fence_after_sync();
      issue_qk(0);
    }
  }

#pragma unroll 1
  for (int c = 0; c < nch; ++c) {
    unsigned char* sV = kv + (c % SH::kStages) * 2 * SH::kKVTile + SH::kKVTile;
    // chunk c + 2 into the stage of chunk c - 1, whose MMAs have completed
    if (SH::kStages == 3 && c + 2 < nch) {
      unsigned char* nk = kv + ((c + 2) % SH::kStages) * 2 * SH::kKVTile;
      load_kv_chunk<TOK>(p, sm, b, g, pl.len, c + 2, ntok, nk, nk + SH::kKVTile);
    }
    cp_async_commit();

    if (!dead && !mbar_spin_warp(&sm.bar_s, it & 1u)) {
      if (lane == 0) record_error(p.ws_header, CLSA_ERR_TIMEOUT, 30);
      dead = true;
    }
    if (c == 0) stamp(p, 36);
    tc::fence_after_sync();
    const uint32_t ts = tl + (uint32_t)(TOK * (c & 1) + NPT * cg);
    const int t0 = c * TOK + NPT * cg;
    const int nv = ntok - t0;  // valid columns of this thread (may be <= 0 or > NPT)
    uint32_t v[NPT];           // the scores, held until P is final
    float lmx = -INFINITY;     // this thread's max of its columns (log2 units)
    if (live) {
      if (!dead) {
        tmem_ld_row<NPT>(ts, v);
        tc::ld_wait();
        float cmx = -INFINITY;
#pragma unroll
        for (int j = 0; j < NPT; ++j)
          if (j < nv) cmx = fmaxf(cmx, __uint_as_float(v[j]));
        lmx = cmx * p.scale_log2;  // scale > 0: the max commutes
      } else {
#pragma unroll
        for (int j = 0; j < NPT; ++j) v[j] = 0xff800000u;  // -inf: P = 0
      }
    }
    // P of this thread's columns against the row's reference max m, into shared memory; the
    // sum of those columns is returned
    auto write_p = [&]() -> float {
      float rs = 0.f;
#pragma unroll
      for (int q = 0; q < NPT / 8; ++q) {  // 8 tokens = one 16-byte chunk of the P row
        uint32_t pw[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int j0 = 8 * q + 2 * j;
          const float a = j0 < nv ? fast_exp2(fmaf(__uint_as_float(v[j0]), p.scale_log2, -m)) : 0.f;
          const float e = j0 + 1 < nv ? fast_exp2(fmaf(__uint_as_float(v[j0 + 1]), p.scale_log2, -m)) : 0.f;
          rs += a + e;
          pw[j] = pack_bf16x2(a, e);
        }
        const int ch = (NPT * cg) / 8 + q;  // 16-byte chunk of the row: atom ch / 8, chunk ch % 8
        *reinterpret_cast<uint4*>(sP + (ch >> 3) * SH::kPAtom + tc::sw128_offset(row, ch & 7)) =
            make_uint4(pw[0], pw[1], pw[2], pw[3]);
      }
      return rs;
    };
    // The output accumulates in TMEM (P V with accumulate).  P is taken against a reference max
    // m that moves only when a column exceeds it by more than 2^kTau: then the row's TMEM output
    // and sum are scaled by 2^(m_old - m_new) once.  In the common case a thread writes its P at
    // once; the first chunk, or a column above the bound anywhere in the CTA, takes the row-max
    // exchange (voted on the barrier that precedes the MMA issue anyway), after which the
    // threads of a row whose max moved rewrite their P.
    constexpr float kTau = 8.f;
    const bool need = live && (c == 0 || lmx > m + kTau);
    float rs = 0.f;
    if (live && !need) rs = write_p();
    if (SH::kStages == 3 && c + 1 < nch) cp_async_wait<1>();  // chunk c + 1 landed (c + 2 may be in flight)
    fence_proxy_async_smem();
    tc::fence_before_sync();
    if (__syncthreads_or(need)) {
      if (live) sm.cm[cg * kMaxRows + row] = lmx;
      __syncthreads();
      if (c == 0) stamp(p, 37);
      if (live) {
        const float mn = fmaxf(fmaxf(sm.cm[row], sm.cm[kMaxRows + row]),
                               fmaxf(sm.cm[2 * kMaxRows + row], sm.cm[3 * kMaxRows + row]));
        const bool up = c == 0 || mn > m + kTau;  // the same in the four threads of the row
        if (c > 0 && __any_sync(0xffffffffu, up)) {
          // TMEM load / store are .sync.aligned: every lane of the warp (alpha = 1 if not up);
          // P V of the previous chunk has completed (waited below)
          const float alpha = up ? fast_exp2(m - mn) : 1.f;
          if (!dead) {
            uint32_t w[32];
            tc::ld_32x32b_x32(tl + 128u + (uint32_t)(32 * cg), w);
            tc::ld_wait();
#pragma unroll
            for (int j = 0; j < 32; ++j) w[j] = __float_as_uint(__uint_as_float(w[j]) * alpha);
            tc::st_32x32b_x32(tl + 128u + (uint32_t)(32 * cg), w);
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
    if (c == 0) stamp(p, 38);
    if (threadIdx.x == 0) {
      // O += P_c V_c, then S of the next chunk into the other S buffer
      tc::fence_after_sync();
#pragma unroll
      for (int ks = 0; ks < TOK / 16; ++ks)
        tc::mma_bf16(tmem + 128u, tc::sw128_desc(smem_u32(sP) + (ks >> 2) * SH::kPAtom + (ks & 3) * 32),
                     tc::sw128_desc_mn(smem_u32(sV) + ks * 16 * 128, SH::kKVAtom), kIdescPV, c > 0 || ks > 0);
      tc::mma_commit(&sm.bar_o);
      if (c + 1 < nch) issue_qk(c + 1);
    }
    if (!dead && !mbar_spin_warp(&sm.bar_o, it & 1u)) {
      if (lane == 0) record_error(p.ws_header, CLSA_ERR_TIMEOUT, 31);
      dead = true;
    }
    if (c == 0) stamp(p, 39);
    tc::fence_after_sync();
    ++it;
  }
  // the unit's output rows from TMEM (every lane of a live warp: the load is .sync.aligned)
  float o[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) o[j] = 0.f;
  if (live && !dead && nch > 0) {
    uint32_t w[32];
    tc::ld_32x32b_x32(tl + 128u + (uint32_t)(32 * cg), w);
    tc::ld_wait();
#pragma unroll
    for (int j = 0; j < 32; ++j) o[j] = __uint_as_float(w[j]);
  }
  tc::fence_before_sync();  // the TMEM output is read before the next unit's first P V overwrites it
  cp_async_wait<0>();  // no copy of this unit outlives it (the trailing groups are empty)
  stamp(p, 11);

  // row sum over the four column groups, in a fixed order
  sm.cl[cg * kMaxRows + row] = lp;
  __syncthreads();
  const float ls = (sm.cl[row] + sm.cl[kMaxRows + row]) + (sm.cl[2 * kMaxRows + row] + sm.cl[3 * kMaxRows + row]);
  stamp(p, 13);
  if (row < p.rows) {
    const int l = row / p.G, h = g * p.G + row % p.G;
    if (pl.nsplit == 1) {
      const float inv = ls > 0.f ? 1.f / ls : 0.f;
      uint4* out = reinterpret_cast<uint4*>(p.O + (((size_t)l * p.B + b) * p.Hq + h) * kD + 32 * cg);
#pragma unroll
      for (int j = 0; j < 4; ++j)
        out[j] = make_uint4(pack_bf16x2(o[8 * j] * inv, o[8 * j + 1] * inv),
                            pack_bf16x2(o[8 * j + 2] * inv, o[8 * j + 3] * inv),
                            pack_bf16x2(o[8 * j + 4] * inv, o[8 * j + 5] * inv),
                            pack_bf16x2(o[8 * j + 6] * inv, o[8 * j + 7] * inv));
      if (p.lse && cg == 0)
        p.lse[((size_t)l * p.B + b) * p.Hq + h] = ls > 0.f ? (m + log2f(ls)) * kLn2 : -INFINITY;
    }
  }
  if (pl.nsplit > 1) {
    // this CTA's partial rows are one contiguous block of p.Op, in bf16 (the merge sums them
    // in fp32; a partial's rounding is 2^-9 of its own size): stage them in shared memory
    // (row pitch kOPitch bf16: conflict-free 16-byte stores down a column), then write the
    // block with whole-line stores
    __nv_bfloat16* stg = reinterpret_cast<__nv_bfloat16*>(kv);
    uint4* srow = reinterpret_cast<uint4*>(stg + row * kOPitch + 32 * cg);
#pragma unroll
    for (int j = 0; j < 4; ++j)
      srow[j] = make_uint4(pack_bf16x2(o[8 * j], o[8 * j + 1]), pack_bf16x2(o[8 * j + 2], o[8 * j + 3]),
                           pack_bf16x2(o[8 * j + 4], o[8 * j + 5]), pack_bf16x2(o[8 * j + 6], o[8 * j + 7]));
    if (cg == 0 && row < p.rows)
      __stcg(reinterpret_cast<float4*>(p.Ml + ((size_t)blockIdx.x * p.rows + row) * 4), make_float4(m, ls, 0.f, 0.f));
    __syncthreads();
    uint4* op = reinterpret_cast<uint4*>(p.Op + (size_t)blockIdx.x * p.rows * kD);
#pragma unroll 1
    for (int i = threadIdx.x; i < p.rows * (kD / 8); i += kThreads)
      __stcg(op + i, *reinterpret_cast<const uint4*>(stg + (i / (kD / 8)) * kOPitch + 8 * (i % (kD / 8))));
    // the partial is complete: the CTA's barrier orders every thread's stores before the
    // release that publishes its flag (the row's launch counter + 1)
    __syncthreads();
    if (threadIdx.x == 0)
      st_release_gpu(p.row_ws + (size_t)b * kRowWords + kRowFlag + pl.c, sm.row_hdr[kRowEpoch] + 1u);
  }
  stamp(p, 12);
  __syncthreads();  // cm / cl and the tiles are free for the next unit
}

// ---------------------------------------------------------------------------
// phase 5: merge the nsplit partials of head g for rows r = split, split + nsplit, ...
// Warp w waits for the flag of split w (w + 16, ...) and at once issues the async copies
// of that split's partial rows and (m, l) pairs, then goes on to its next flag, so the
// copies of the early splits overlap the wait for the late ones.  Then one warp per row
// takes M = max m and den = sum 2^(m - M) l over the splits and sums the split rows in
// split order (the same order every call: the result is deterministic).  The code is
// rolled: it runs once per launch, so its size is instruction fetches on the critical path.
// ---------------------------------------------------------------------------
__device__ void combine_head(const FusedParams& p, Smem& sm, unsigned char* big, const Plan pl, int g) {
  stamp(p, 18);
  const int ns = pl.nsplit;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nr = (p.rows - pl.split + ns - 1) / ns;
  if (nr <= 0) return;
  const size_t cta0 = (size_t)pl.start + (size_t)g * ns;  // CTA holding split 0 of head g
  const uint32_t* flags = p.row_ws + (size_t)pl.b * kRowWords + kRowFlag + (size_t)g * ns;
  const uint32_t tag = sm.row_hdr[kRowEpoch] + 1u;
  // Every (row, split) pair of the head is staged at once: nr * ns <= rows + ns - 1.
  constexpr int kMaxPairs = kMaxRows + kMaxGroups - 1;
  static_assert(kMaxPairs * kD * 2 + kMaxPairs * 16 <= (int)kSmemBig, "merge staging exceeds big");
  static_assert(kMaxPairs <= 512, "split weights exceed sm.cm");
  __nv_bfloat16* stg = reinterpret_cast<__nv_bfloat16*>(big);  // [split][row][kD]
  float4* mls = reinterpret_cast<float4*>(big + (size_t)kMaxPairs * kD * sizeof(__nv_bfloat16));  // [row][split]
  bool dead = false;
  auto wait_flag = [&](int s2) {  // warp-wide; false on timeout
    uint32_t ok = 1;
    if (lane == 0) {
      const unsigned long long t0 = globaltimer_ns();
      while (ld_acquire_gpu(flags + s2) != tag) {
        if (globaltimer_ns() - t0 > kWaitLimitNs) {
          record_error(p.ws_header, CLSA_ERR_TIMEOUT, 2);
          ok = 0;
          break;
        }
      }
    }
    __syncwarp();  // lane 0's acquire orders the warp's loads below
    return __shfl_sync(0xffffffffu, ok, 0) != 0u;
  };
#pragma unroll 1
  for (int s2 = warp; s2 < ns; s2 += kWarps) {
    if (!wait_flag(s2)) {
      dead = true;
      continue;
    }
    const size_t src_row = (cta0 + s2) * p.rows + pl.split;  // row ri of the split: src_row + ri * ns
#pragma unroll 1
    for (int e = lane; e < nr * 16; e += 32) {  // 16 lanes per 256-byte row
      const int ri = e >> 4, q = e & 15;
      cp_async_16(stg + (s2 * nr + ri) * kD + q * 8, p.Op + (src_row + (size_t)ri * ns) * kD + q * 8, 16);
    }
#pragma unroll 1
    for (int ri = lane; ri < nr; ri += 32) cp_async_16(mls + ri * ns + s2, p.Ml + (src_row + (size_t)ri * ns) * 4, 16);
  }
  cp_async_commit();
  cp_async_wait<0>();  // no copy outlives an abort below
  if (dead) sm.abort_flag = 1;
  __syncthreads();
  stamp(p, 17);
  if (sm.abort_flag) return;
#pragma unroll 1
  for (int ri = warp; ri < nr; ri += kWarps) {
    float M = -INFINITY, den = 0.f;
#pragma unroll 1
    for (int s2 = lane; s2 < ns; s2 += 32) M = fmaxf(M, mls[ri * ns + s2].x);
    M = warp_max(M);
#pragma unroll 1
    for (int s2 = lane; s2 < ns; s2 += 32) {
      const float4 ml = mls[ri * ns + s2];
      const float wgt = M == -INFINITY ? 0.f : exp2f(ml.x - M);
      den = fmaf(wgt, ml.y, den);
      sm.cm[ri * ns + s2] = wgt;
    }
    den = warp_sum(den);
    __syncwarp();  // the row's weights are visible to the whole warp
    // lane: 4 of the 128 columns
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 2
    for (int s2 = 0; s2 < ns; ++s2) {
      const float w = sm.cm[ri * ns + s2];
      const uint2 vv = *reinterpret_cast<const uint2*>(stg + (s2 * nr + ri) * kD + lane * 4);
      float v0, v1, v2, v3;
      unpack_bf16x2(vv.x, v0, v1);
      unpack_bf16x2(vv.y, v2, v3);
      a.x = fmaf(w, v0, a.x);
      a.y = fmaf(w, v1, a.y);
      a.z = fmaf(w, v2, a.z);
      a.w = fmaf(w, v3, a.w);
    }
    const int r = pl.split + ri * ns;
    const float inv = den > 0.f ? 1.f / den : 0.f;
    const int l = r / p.G, h = g * p.G + r % p.G;
    __nv_bfloat16* out = p.O + (((size_t)l * p.B + pl.b) * p.Hq + h) * kD + lane * 4;
    uint2 wv;
    wv.x = pack_bf16x2(a.x * inv, a.y * inv);
    wv.y = pack_bf16x2(a.z * inv, a.w * inv);
    *reinterpret_cast<uint2*>(out) = wv;
    if (p.lse && lane == 0)
      p.lse[((size_t)l * p.B + pl.b) * p.Hq + h] = den > 0.f ? (M + log2f(den)) * kLn2 : -INFINITY;
  }
  stamp(p, 46);
}

// ---------------------------------------------------------------------------
// the kernel
// ---------------------------------------------------------------------------
template <int DIDX>
__global__ void __launch_bounds__(kThreads, 1) decode_fused_kernel(const FusedParams p) {
  extern __shared__ __align__(128) unsigned char smem[];
  Smem& sm = *reinterpret_cast<Smem*>(smem);
  __nv_bfloat16* sQ = reinterpret_cast<__nv_bfloat16*>(smem + align_up(sizeof(Smem), 128));
  unsigned char* big = smem + align_up(sizeof(Smem), 128) + kSmemQ;

  // launched with programmatic stream serialization: wait until the previous grid on the
  // stream has completed and its memory is visible (a no-op otherwise), then let the next
  // one be scheduled
  pdl_enter();
  stamp(p, 0);
  // One sequence: CTA c's slice is [c chunk, c chunk + chunk) with chunk = ceil(len /
  // gridDim.x) (what make_plan gives for B = 1), so every thread starts the K_idx stream
  // before the plan exists; the plan is checked against it below.
  int pre_r0 = 0, pre_r1 = 0;
  bool pre = false;
  uint4 pre_q = make_uint4(0, 0, 0, 0);
  if (p.B == 1) {
    const int len = max(0, min(p.seq_lens[0], p.n_max));
    if (len > 0) {
      const int chunk = (len + (int)gridDim.x - 1) / (int)gridDim.x;
      pre_r0 = min(len, (int)blockIdx.x * chunk);
      pre_r1 = min(len, pre_r0 + chunk);
      pre_q = load_q_chunk<DIDX>(p, 0);  // ahead of the K_idx stream (it would queue behind it)
      load_row_header(p, sm, 0);
      scan_start<DIDX>(reinterpret_cast<uint4*>(big), p.k_idx + (size_t)pre_r0 * DIDX, 0, pre_r1 - pre_r0);
      pre = true;
    }
  }
  if (threadIdx.x == 0) {
    make_plan(p, sm.plan, sm.live_rows);
    sm.abort_flag = 0;
  }
  __syncthreads();
  stamp(p, 15);
  const Plan pl = sm.plan;
  if (blockIdx.x == 0) {  // sequences with no tokens: count 0, idx -1, O = 0, lse = -inf
#pragma unroll 1
    for (int b = 0; b < p.B; ++b) {
      if (max(0, min(p.seq_lens[b], p.n_max)) > 0) continue;
      for (int i = threadIdx.x; i < p.k; i += kThreads) p.idx[(size_t)b * p.k + i] = -1;
      if (threadIdx.x == 0) p.count[b] = 0;
      for (int i = threadIdx.x; i < p.L * p.Hq * kD; i += kThreads) {
        const int l = i / (p.Hq * kD), rem = i % (p.Hq * kD);
        p.O[((size_t)l * p.B + b) * p.Hq * kD + rem] = __float2bfloat16_rn(0.f);
      }
      if (p.lse)
        for (int i = threadIdx.x; i < p.L * p.Hq; i += kThreads)
          p.lse[((size_t)(i / p.Hq) * p.B + b) * p.Hq + i % p.Hq] = -INFINITY;
    }
  }
  if (pl.b < 0) {
    leave_finish(p, sm, leave_issue(p));
    return;
  }
  const bool merge = pl.nsplit > 1 && pl.nunits_here > 0;  // this CTA merges split partials of its head
  uint32_t left = 0;
  if (pl.c == 0) {
    for (int i = pl.keff + threadIdx.x; i < p.k; i += kThreads) p.idx[(size_t)pl.b * p.k + i] = -1;
    if (threadIdx.x == 0) p.count[pl.b] = pl.keff;
  }
  if (pl.c == pl.Cb - 1)  // score tail beyond the sequence
    for (int j = pl.len + threadIdx.x; j < p.n_max; j += kThreads) p.scores[(size_t)pl.b * p.n_max + j] = -INFINITY;
  unsigned char* sQa = align1024(reinterpret_cast<unsigned char*>(sQ));
  if (pre && (pl.b != 0 || pl.r0 != pre_r0 || pl.r1 != pre_r1)) {  // cannot happen: the plan's own slice
    record_error(p.ws_header, CLSA_ERR_INVALID_ARG, 50);
    cp_async_wait<0>();
    pre = false;
  }

  const bool all_sel = pl.keff == pl.len;
  stamp(p, 23);
  if (!scan_slice<DIDX>(p, sm, sm.hist, big, !all_sel, pre, pre_q, pl.nunits_here > 0 ? sQa : nullptr)) return;
  clear_previous_copy(p, sm, pl);
  stamp(p, 1);

  if (all_sel) {  // every token is selected: rank = token index
    left = leave_issue(p);
    int32_t* out = p.idx + (size_t)pl.b * p.k;
    for (int j = pl.r0 + threadIdx.x; j < pl.r1; j += kThreads) out[j] = j;
    for (int i = threadIdx.x; i < pl.tok1 - pl.tok0; i += kThreads) sm.unit_tok[i] = pl.tok0 + i;
    __syncthreads();
  } else {
    write_candidates(p, sm, sm.hist);
    stamp(p, 2);
    uint32_t* rw = p.row_ws + (size_t)pl.b * kRowWords;
    if (!count_barrier(rw + kRowBar, pl.Cb, p.ws_header, 1)) return;
    stamp(p, 3);
    // the group's windows (back to back, token order, empty slots key 0) to shared
    // memory in 16-byte copies: keys first, then tokens (needed only for the ranking)
    uint32_t* skey = reinterpret_cast<uint32_t*>(big);
    int32_t* stok = reinterpret_cast<int32_t*>(big + kCandCap * 4);
    const int nslot = pl.Cb * pl.win;  // a multiple of 4
    {
      const uint4* gk = reinterpret_cast<const uint4*>(p.cand_key + (size_t)pl.b * kCandCap);
      const uint4* gt = reinterpret_cast<const uint4*>(p.cand_tok + (size_t)pl.b * kCandCap);
      for (int i = threadIdx.x; i < nslot / 4; i += kThreads) cp_async_16(skey + 4 * i, gk + i, 16);
      cp_async_commit();
      for (int i = threadIdx.x; i < nslot / 4; i += kThreads) cp_async_16(stok + 4 * i, gt + i, 16);
      cp_async_commit();
    }
    const bool done = select_windows(p, sm, rw, skey, stok, nslot);
    // past the row barrier: the last CTA to leave may reset its word
    left = leave_issue(p);
    stamp(p, 5);
    if (!done) {  // too few candidates at or above E_max, or a boundary sub-bin of heavy ties:
              // digit-by-digit select over the whole row
      cp_async_wait<0>();
      __syncthreads();
      CandSrc src{skey, stok, p.scores + (size_t)pl.b * p.n_max, false};
      resolve_theta(sm, src, pl.len, (uint32_t)pl.keff, p.ws_header);
      compact_selected(p, sm, src, pl.len);
    }
    if (p.trace && threadIdx.x == 0) p.trace[blockIdx.x * kTraceSlots + 31] = (unsigned long long)nslot | ((unsigned long long)done << 32);
  }
  stamp(p, 6);

  // ---- attention units (TMEM held only for this phase: no return path in between)
  if (pl.nunits_here > 0) {
    const int ntok = pl.tok1 - pl.tok0;
    unsigned char* kv = align1024(big);  // the windows are dead past the ranking
    // the first unit's first K/V chunk goes out now, so that its gather overlaps the TMEM
    // allocation and the barrier below (attend_unit then skips it)
    if (ntok > 0) {
      if (ntok <= 128) load_kv_chunk<128>(p, sm, pl.b, pl.unit_g0, pl.len, 0, ntok, kv, kv + AttnShape<128>::kKVTile);
      else load_kv_chunk<64>(p, sm, pl.b, pl.unit_g0, pl.len, 0, ntok, kv, kv + AttnShape<64>::kKVTile);
    }
    cp_async_commit();
    if (threadIdx.x < 32) {
      tc::tmem_alloc(&sm.tmem_base, kTmemCols);
      tc::tmem_relinquish();
    }
    if (threadIdx.x == 0) {
      mbar_init(&sm.bar_s, 1);
      mbar_init(&sm.bar_o, 1);
      fence_mbar_init();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = sm.tmem_base;
    uint32_t it = 0;
    for (int u = 0; u < pl.nunits_here; ++u) {
      const int g = pl.unit_g0 + u * pl.unit_step;
      if (ntok <= 128) attend_unit<128>(p, sm, sQa, kv, g, ntok, u == 0, u == 0, tmem, it);
      else attend_unit<64>(p, sm, sQa, kv, g, ntok, u == 0, u == 0, tmem, it);
    }
    tc::fence_before_sync();
    __syncthreads();
    if (threadIdx.x < 32) tc::tmem_dealloc(tmem, kTmemCols);
  }
  stamp(p, 7);
  if (merge) {
    stamp(p, 8);
    combine_head(p, sm, big, pl, pl.unit_g0);
  }
  leave_finish(p, sm, left);
  stamp(p, 9);
}

struct FusedCfg {
  int ncta = 0;
  bool ok = false;
};

// computed from the current device's attributes on every call (device_info() caches
// them per host thread and device), so mixed devices and host threads get their own
FusedCfg fused_cfg() {
  FusedCfg cfg;
  const DeviceInfo& di = device_info();
  if (di.sm_count > 0 && (size_t)di.max_smem_optin >= smem_bytes()) {
    cfg.ncta = std::min(di.sm_count, kMaxGroups);
    cfg.ok = true;
  }
  return cfg;
}

}  // namespace

bool fused_decode_supported(const clsa_decode_args* a) {
  if (a->dtype != CLSA_BF16 || a->d != kD || (a->d_idx != 64 && a->d_idx != 128)) return false;
  if (a->K_S != nullptr) return false;
  // 16-byte copies and L2 bulk prefetches of K_idx, K and V rows; 16-byte Q copies and O stores
  if ((reinterpret_cast<uintptr_t>(a->k_idx) | reinterpret_cast<uintptr_t>(a->K) |
       reinterpret_cast<uintptr_t>(a->V) | reinterpret_cast<uintptr_t>(a->Q) | reinterpret_cast<uintptr_t>(a->O)) %
          16 !=
      0)
    return false;
  if (a->Hkv > 64 || a->L * (a->Hq / a->Hkv) > kMaxRows || a->k > kMaxUnitTok) return false;
  const FusedCfg cfg = fused_cfg();
  if (!cfg.ok || a->B > cfg.ncta / 2) return false;
  return true;
}

size_t fused_decode_ws_bytes(const clsa_decode_args* a) {
  const FusedCfg cfg = fused_cfg();
  const size_t rows = (size_t)a->L * (a->Hq / a->Hkv);
  size_t off = 0;
  off += (size_t)kMaxGroups * kTraceSlots * 8;                  // phase stamps (CLSA_TRACE=1)
  off += align_up((size_t)a->B * a->n_max * 4, 256);           // scores (when not an output)
  off += align_up(((size_t)a->B * kRowWords + 1) * 4, 256);    // row state, leave count
  off += 2 * align_up((size_t)a->B * kCandCap * 4, 256);  // candidate windows
  off += align_up((size_t)cfg.ncta * rows * kD * 4, 256);      // split partials
  off += align_up((size_t)cfg.ncta * rows * 4 * 4, 256);     // split (m, l), 16-byte slots
  return off;
}

// Cooperative launch with programmatic stream serialization: the launch of the next step
// may be processed while this one runs (its CTAs wait at griddepcontrol.wait before any
// work), which hides the launch latency between back-to-back steps.  Falls back to the
// plain cooperative launch where the runtime refuses the pair of attributes.
template <int DIDX>
cudaError_t launch_fused(const FusedParams& p, int ncta, size_t smem, cudaStream_t s) {
  cudaError_t e = cudaFuncSetAttribute(decode_fused_kernel<DIDX>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  // per device: whether the runtime took the pair of launch attributes there
  static std::atomic<int> pdl_refused[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) dev = 0;
  if (pdl_refused[dev].load(std::memory_order_relaxed) == 0) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(ncta);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute at[2];
    at[0].id = cudaLaunchAttributeCooperative;
    at[0].val.cooperative = 1;
    at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 2;
    e = cudaLaunchKernelEx(&cfg, decode_fused_kernel<DIDX>, p);
    if (e != cudaErrorNotSupported && e != cudaErrorInvalidValue) return e;
    (void)cudaGetLastError();
    pdl_refused[dev].store(1, std::memory_order_relaxed);
  }
  void* args[] = {(void*)&p};
  return cudaLaunchCooperativeKernel((const void*)decode_fused_kernel<DIDX>, dim3(ncta), dim3(kThreads), args, smem, s);
}

cudaError_t launch_decode_fused(const clsa_decode_args* a, float scale, void* ws_header, void* ws_body,
                                cudaStream_t s) {
  const FusedCfg cfg = fused_cfg();
  FusedParams p{};
  p.q_idx = static_cast<const __nv_bfloat16*>(a->q_idx);
  p.k_idx = static_cast<const __nv_bfloat16*>(a->k_idx);
  p.K = static_cast<const __nv_bfloat16*>(a->K);
  p.V = static_cast<const __nv_bfloat16*>(a->V);
  p.Q = static_cast<const __nv_bfloat16*>(a->Q);
  p.seq_lens = a->seq_lens;
  p.O = static_cast<__nv_bfloat16*>(a->O);
  p.idx = a->idx;
  p.count = a->count;
  p.lse = a->lse;
  p.B = a->B;
  p.n_max = a->n_max;
  p.k = a->k;
  p.L = a->L;
  p.Hq = a->Hq;
  p.Hkv = a->Hkv;
  p.G = a->Hq / a->Hkv;
  p.rows = a->L * p.G;
  p.nsplit_max = std::max(1, cfg.ncta / a->Hkv);
  p.scale_log2 = scale * kLog2e;
  p.pf_mult = 1.5f;
  p.pf_add = 8u;
  if (const char* pf = std::getenv("CLSA_PREFETCH")) {  // "mult,add" (tuning)
    float m = 0.f;
    unsigned ad = 0;
    if (std::sscanf(pf, "%f,%u", &m, &ad) == 2) {
      p.pf_mult = m;
      p.pf_add = ad;
    }
  }
  p.ws_header = ws_header;
  char* w = static_cast<char*>(ws_body);
  const char* tr = std::getenv("CLSA_TRACE");
  p.trace = (tr && tr[0] == '1') ? reinterpret_cast<unsigned long long*>(w) : nullptr;
  w += (size_t)kMaxGroups * kTraceSlots * 8;
  float* ws_scores = reinterpret_cast<float*>(w);
  w += align_up((size_t)a->B * a->n_max * 4, 256);
  p.scores = a->scores ? a->scores : ws_scores;
  p.row_ws = reinterpret_cast<uint32_t*>(w);
  p.leave = p.row_ws + (size_t)a->B * kRowWords;
  w += align_up(((size_t)a->B * kRowWords + 1) * 4, 256);
  p.cand_key = reinterpret_cast<uint32_t*>(w);
  w += align_up((size_t)a->B * kCandCap * 4, 256);
  p.cand_tok = reinterpret_cast<int32_t*>(w);
  w += align_up((size_t)a->B * kCandCap * 4, 256);
  p.Op = reinterpret_cast<__nv_bfloat16*>(w);
  w += align_up((size_t)cfg.ncta * p.rows * kD * 4, 256);
  p.Ml = reinterpret_cast<float*>(w);
  const size_t smem = smem_bytes();
  const cudaError_t e = a->d_idx == 128 ? launch_fused<128>(p, cfg.ncta, smem, s) : launch_fused<64>(p, cfg.ncta, smem, s);
  launches_add(1, s);
  return e;
}

}  // namespace clsa
