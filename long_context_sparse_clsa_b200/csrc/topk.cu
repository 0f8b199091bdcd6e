// Exact TopK of the routing equation, S_b = TopK(I_b, k) (picx.dev CLSA summary,
// Methodology > Architecture Overview), as a multi-CTA radix select.
//
// Order: larger score first, equal scores to the lower token index, -0.0 == +0.0.
// Scores are mapped to order-preserving 32-bit keys.  The k_eff-th largest key
// theta is found digit by digit (12 + 12 + 8 bits), each digit from a histogram
// that the C CTAs of a row build over their slices and merge in global memory.
// Every key > theta is selected, and of the keys == theta the lowest-index
// (k_eff - #greater) ones.  Output positions come from per-CTA counts, so the
// index list is written in ascending token order without a sort.
//
// With C > 1 CTAs per row, the first digit's histogram is merged in global memory and
// its boundary bin t1 found after one barrier.  When t1 holds at most kCandMax keys (the
// usual case: about 1% of a 128K row), every CTA publishes its keys of bin t1 (key and
// token) and its count of keys above t1; after a second barrier each CTA reads the short
// candidate list and resolves the remaining 20 bits on chip, so a row costs two barriers.
// A heavier boundary bin (many equal keys) takes the digit-by-digit path with four.
// group_barrier: bounded wait, reusable state.  C > 1 requires a cooperative launch;
// C == 1 rows need none.
#include <atomic>
#include "common.cuh"
#include "kernels.h"

namespace clsa {

namespace {

constexpr int kThreads = 512;
constexpr int kMaxCtasPerRow = 512;
constexpr int kBins1 = 4096, kBins2 = 4096, kBins3 = 256;
// per-row workspace, in u32 words
constexpr int kOffH1 = 0;
constexpr int kOffH2 = kOffH1 + kBins1;
constexpr int kOffH3 = kOffH2 + kBins2;
constexpr int kOffBar = kOffH3 + kBins3;          // 2 words used, 32 reserved
constexpr int kOffCandN = kOffBar + 2;            // candidates published so far
constexpr int kOffCnt = kOffBar + 32;             // 2 words per CTA
constexpr int kCandMax = 4096;                    // boundary-bin keys resolved on chip
constexpr int kOffCand = kOffCnt + 2 * kMaxCtasPerRow;  // [kCandMax] keys, [kCandMax] tokens
constexpr int kRowWords = kOffCand + 2 * kCandMax;
constexpr int kHistWords = kBins1 + kBins2 + kBins3;
// dynamic shared memory of a C > 1 launch: this CTA's digit-1 histogram, the candidates
constexpr int kDynWords = kBins1 + 2 * kCandMax;

struct TopkSmem {
  uint32_t hist[kBins1];
  uint32_t warp_tot[kThreads / 32];
  uint32_t warp_tot2[kThreads / 32];
  int sel_bin;
  uint32_t sel_above;
  uint32_t red_gt, red_eq;
  uint32_t take, out_off;
  uint32_t cand_n, cand_base;
};

// Block-wide exclusive prefix sum of v (thread order).  Returns the exclusive
// prefix; *total receives the block total.  Uses sm.warp_tot.
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t* warp_tot, uint32_t* total) {
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
    constexpr int NW = kThreads / 32;
    uint32_t t = lane < NW ? warp_tot[lane] : 0u;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += y;
    }
    if (lane < NW) warp_tot[lane] = t;  // inclusive
  }
  __syncthreads();
  const uint32_t before = (w > 0 ? warp_tot[w - 1] : 0u) + x - v;
  *total = warp_tot[kThreads / 32 - 1];
  __syncthreads();
  return before;
}

// Find bin T with  sum(hist[i], i > T) < need <= sum(hist[i], i >= T).
// Writes sm.sel_bin and sm.sel_above (= sum over i > T).
__device__ void select_bin(TopkSmem& sm, int nbins, uint32_t need) {
  const int per = (nbins + kThreads - 1) / kThreads;
  // thread t owns bins [hi - per, hi) counted from the top
  const int hi = nbins - threadIdx.x * per;
  const int lo = max(hi - per, 0);
  uint32_t local = 0;
  for (int i = lo; i < hi; ++i) local += sm.hist[i];
  uint32_t total;
  const uint32_t before = block_excl_scan(hi > 0 ? local : 0u, sm.warp_tot, &total);
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

__device__ __forceinline__ void merge_hist(TopkSmem& sm, uint32_t* g, int nbins, int C) {
  // add this CTA's bins to the row's global histogram
  if (C > 1) {
    for (int i = threadIdx.x; i < nbins; i += kThreads) {
      const uint32_t c = sm.hist[i];
      if (c) atomicAdd(g + i, c);
    }
  }
}

__device__ __forceinline__ void load_hist(TopkSmem& sm, const uint32_t* g, int nbins, int C) {
  if (C > 1) {
    for (int i = threadIdx.x; i < nbins; i += kThreads) sm.hist[i] = __ldcg(g + i);
  }
  __syncthreads();
}

// Block-wide sum of v (every thread gets it).  Uses warp_tot.
__device__ __forceinline__ uint32_t block_sum(uint32_t v, uint32_t* warp_tot) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if (lane == 0) warp_tot[w] = v;
  __syncthreads();
  uint32_t t = 0;
#pragma unroll
  for (int i = 0; i < kThreads / 32; ++i) t += warp_tot[i];
  __syncthreads();
  return t;
}

// Write this slice's selected token indices in ascending order from position off: every
// key > theta, and the first `take` keys == theta of the slice (token order).
__device__ void write_selected(TopkSmem& sm, const float* sc, int lo, int hi, uint32_t theta, uint32_t take,
                               uint32_t off, int keff, int32_t* out, const int32_t* map, void* ws_header, int b) {
  uint32_t ties_seen = 0, written = 0;
  for (int base = lo; base < hi; base += kThreads) {
    const int j = base + threadIdx.x;
    uint32_t key = 0;
    const bool in = j < hi;
    if (in) key = float_key(sc[j]);
    const uint32_t is_eq = in && key == theta;
    uint32_t tile_eq;
    const uint32_t eq_rank = ties_seen + block_excl_scan(is_eq, sm.warp_tot, &tile_eq);
    const uint32_t sel = in && (key > theta || (is_eq && eq_rank < take));
    uint32_t tile_sel;
    const uint32_t pos = written + block_excl_scan(sel, sm.warp_tot, &tile_sel);
    if (sel) {
      if (off + pos < (uint32_t)keff) out[off + pos] = map ? map[j] : j;
      else record_error(ws_header, CLSA_ERR_BAD_INDEX, ((long long)b << 32) | (off + pos));
    }
    ties_seen += tile_eq;
    written += tile_sel;
  }
}

// The two-barrier path of a C > 1 row whose digit-1 boundary bin t1 holds cand_total <=
// kCandMax keys.  `need` keys of bin t1 are taken (all keys above t1 are).
//  1. publish: this CTA's count of keys above t1 (from its own digit-1 histogram) and its
//     keys of bin t1 with their tokens, at a position reserved with one atomic;
//  2. barrier; every CTA loads the cand_total candidates into shared memory and finds the
//     need-th largest (key bits 19..8, then 7..0) with a shared-memory histogram each;
//  3. this slice's output offset = keys above t1 in the CTAs before it + candidates taken
//     from tokens before lo (those > theta, and min(ties before lo, ties needed) == theta).
__device__ void candidate_select(TopkSmem& sm, uint32_t* dynw, uint32_t* row_ws, uint32_t* bar,
                                 const float* sc, int lo, int hi, int c, int C, uint32_t t1, uint32_t need,
                                 uint32_t cand_total, int keff, int32_t* out, const int32_t* map, void* ws_header,
                                 int b) {
  const uint32_t* lhist = dynw;  // this CTA's digit-1 histogram
  uint32_t* ckey = dynw + kBins1;
  int32_t* ctok = reinterpret_cast<int32_t*>(dynw + kBins1 + kCandMax);
  uint32_t* gkey = row_ws + kOffCand;
  int32_t* gtok = reinterpret_cast<int32_t*>(row_ws + kOffCand + kCandMax);
  uint32_t* cnt = row_ws + kOffCnt;

  // ---- 1. publish
  uint32_t above = 0;
  for (int i = (int)t1 + 1 + threadIdx.x; i < kBins1; i += kThreads) above += lhist[i];
  above = block_sum(above, sm.warp_tot);
  if (threadIdx.x == 0) {
    __stcg(cnt + 2 * c, above);
    sm.cand_n = 0;
    sm.cand_base = lhist[t1] ? atomicAdd(row_ws + kOffCandN, lhist[t1]) : 0u;
  }
  __syncthreads();
  const uint32_t base = sm.cand_base;
  for (int j = lo + threadIdx.x; j < hi; j += kThreads) {
    const uint32_t key = float_key(sc[j]);
    if ((key >> 20) == t1) {
      const uint32_t q = base + atomicAdd(&sm.cand_n, 1u);  // order is free: ranks use (key, token)
      if (q < (uint32_t)kCandMax) {
        __stcg(gkey + q, key);
        __stcg(gtok + q, j);
      }
    }
  }
  if (!group_barrier(bar, C, ws_header, 5)) return;

  // ---- 2. every CTA: the candidates, then the need-th largest of them
  for (int i = threadIdx.x; i < (int)cand_total; i += kThreads) {
    ckey[i] = __ldcg(gkey + i);
    ctok[i] = __ldcg(gtok + i);
  }
  // digit-1 histogram words were read by every CTA before the barrier: clear this CTA's share;
  // the candidate count goes back to zero for the next call
  {
    const int per = (kBins1 + C - 1) / C;
    const int h0 = c * per, h1 = min(kBins1, h0 + per);
    for (int i = h0 + threadIdx.x; i < h1; i += kThreads) row_ws[kOffH1 + i] = 0u;
    if (c == 0 && threadIdx.x == 0) row_ws[kOffCandN] = 0u;
  }
  for (int i = threadIdx.x; i < kBins2; i += kThreads) sm.hist[i] = 0;
  __syncthreads();
  for (int i = threadIdx.x; i < (int)cand_total; i += kThreads) atomicAdd(&sm.hist[(ckey[i] >> 8) & 0xFFFu], 1u);
  __syncthreads();
  select_bin(sm, kBins2, need);
  const uint32_t p2 = (t1 << 12) | (uint32_t)sm.sel_bin;
  need -= sm.sel_above;
  __syncthreads();
  for (int i = threadIdx.x; i < kBins3; i += kThreads) sm.hist[i] = 0;
  __syncthreads();
  for (int i = threadIdx.x; i < (int)cand_total; i += kThreads)
    if ((ckey[i] >> 8) == p2) atomicAdd(&sm.hist[ckey[i] & 0xFFu], 1u);
  __syncthreads();
  select_bin(sm, kBins3, need);
  const uint32_t theta = (p2 << 8) | (uint32_t)sm.sel_bin;
  const uint32_t ties_needed = need - sm.sel_above;  // >= 1 candidates equal to theta are taken
  __syncthreads();

  // ---- 3. this slice's offset and its share of the ties
  uint32_t gt_lo = 0, eq_lo = 0, eq_in = 0;
  for (int i = threadIdx.x; i < (int)cand_total; i += kThreads) {
    const uint32_t key = ckey[i];
    const int tk = ctok[i];
    gt_lo += key > theta && tk < lo;
    eq_lo += key == theta && tk < lo;
    eq_in += key == theta && tk >= lo && tk < hi;
  }
  uint32_t above_before = 0;
  for (int cc = threadIdx.x; cc < c; cc += kThreads) above_before += __ldcg(cnt + 2 * cc);
  gt_lo = block_sum(gt_lo, sm.warp_tot);
  eq_lo = block_sum(eq_lo, sm.warp_tot);
  eq_in = block_sum(eq_in, sm.warp_tot);
  above_before = block_sum(above_before, sm.warp_tot);
  const uint32_t ties_before = min(eq_lo, ties_needed);
  const uint32_t take = min(eq_in, ties_needed - ties_before);
  write_selected(sm, sc, lo, hi, theta, take, above_before + gt_lo + ties_before, keff, out, map, ws_header, b);
}

__global__ void __launch_bounds__(kThreads) topk_kernel(const float* __restrict__ scores,
                                                        const int32_t* __restrict__ seq_lens, int n_max,
                                                        int k, int C, int chunk, int32_t* __restrict__ idx,
                                                        int32_t* __restrict__ count, void* ws_header,
                                                        uint32_t* __restrict__ row_ws_all, int causal_base,
                                                        const int32_t* __restrict__ row_skip, int skip_val,
                                                        const int32_t* __restrict__ idx_map, int ld_map) {
  __shared__ TopkSmem sm;
  extern __shared__ uint32_t dyn[];  // C > 1 only: [kBins1] local digit-1 histogram, candidates
  const int b = blockIdx.y;
  const int c = blockIdx.x;
  if (row_skip && row_skip[b] == skip_val) return;  // uniform for the row's CTAs
  const int len = max(0, min(causal_base >= 0 ? causal_base + b + 1 : seq_lens[b], n_max));
  const int keff = min(k, len);
  uint32_t* row_ws = row_ws_all + (size_t)b * kRowWords;
  uint32_t* bar = row_ws + kOffBar;
  const float* sc = scores + (size_t)b * n_max;
  int32_t* out = idx + (size_t)b * k;

  // -1 padding after the k_eff selected entries, and the count
  if (c == 0) {
    for (int i = keff + threadIdx.x; i < k; i += kThreads) out[i] = -1;
    if (threadIdx.x == 0) count[b] = keff;
  }
  if (keff == 0) return;
  const int lo = c * chunk;
  const int hi = min(len, lo + chunk);
  const int32_t* map = idx_map ? idx_map + (size_t)b * ld_map : nullptr;
  if (keff == len) {  // every token is selected
    for (int j = lo + threadIdx.x; j < hi; j += kThreads) out[j] = map ? map[j] : j;
    return;
  }

  // ---- digit 1: key bits 31..20 -------------------------------------------
  for (int i = threadIdx.x; i < kBins1; i += kThreads) sm.hist[i] = 0;
  __syncthreads();
  for (int j = lo + threadIdx.x; j < hi; j += kThreads) atomicAdd(&sm.hist[float_key(sc[j]) >> 20], 1u);
  __syncthreads();
  uint32_t* lhist = dyn;
  if (C > 1)
    for (int i = threadIdx.x; i < kBins1; i += kThreads) lhist[i] = sm.hist[i];
  merge_hist(sm, row_ws + kOffH1, kBins1, C);
  if (C > 1 && !group_barrier(bar, C, ws_header, 1)) return;
  load_hist(sm, row_ws + kOffH1, kBins1, C);
  select_bin(sm, kBins1, (uint32_t)keff);
  const uint32_t t1 = (uint32_t)sm.sel_bin;
  uint32_t need = (uint32_t)keff - sm.sel_above;
  const uint32_t cand_total = sm.hist[t1];  // the same in every CTA of the row
  __syncthreads();

  if (C > 1 && cand_total <= (uint32_t)kCandMax) {
    candidate_select(sm, dyn, row_ws, bar, sc, lo, hi, c, C, t1, need, cand_total, keff, out, map, ws_header, b);
    return;
  }

  // ---- digit 2: key bits 19..8 within bin t1 --------------------------------
  for (int i = threadIdx.x; i < kBins2; i += kThreads) sm.hist[i] = 0;
  __syncthreads();
  for (int j = lo + threadIdx.x; j < hi; j += kThreads) {
    const uint32_t key = float_key(sc[j]);
    if ((key >> 20) == t1) atomicAdd(&sm.hist[(key >> 8) & 0xFFFu], 1u);
  }
  __syncthreads();
  merge_hist(sm, row_ws + kOffH2, kBins2, C);
  if (C > 1 && !group_barrier(bar, C, ws_header, 2)) return;
  load_hist(sm, row_ws + kOffH2, kBins2, C);
  select_bin(sm, kBins2, need);
  const uint32_t p2 = (t1 << 12) | (uint32_t)sm.sel_bin;  // key bits 31..8
  need -= sm.sel_above;
  __syncthreads();

  // ---- digit 3: key bits 7..0 within prefix p2 --------------------------------
  for (int i = threadIdx.x; i < kBins3; i += kThreads) sm.hist[i] = 0;
  __syncthreads();
  for (int j = lo + threadIdx.x; j < hi; j += kThreads) {
    const uint32_t key = float_key(sc[j]);
    if ((key >> 8) == p2) atomicAdd(&sm.hist[key & 0xFFu], 1u);
  }
  __syncthreads();
  merge_hist(sm, row_ws + kOffH3, kBins3, C);
  if (C > 1 && !group_barrier(bar, C, ws_header, 3)) return;
  load_hist(sm, row_ws + kOffH3, kBins3, C);
  select_bin(sm, kBins3, need);
  const uint32_t theta = (p2 << 8) | (uint32_t)sm.sel_bin;
  const uint32_t ties_needed = need - sm.sel_above;  // >= 1 keys equal to theta are taken
  __syncthreads();

  // ---- per-CTA counts of keys > theta and == theta ----------------------------
  uint32_t gt = 0, eq = 0;
  for (int j = lo + threadIdx.x; j < hi; j += kThreads) {
    const uint32_t key = float_key(sc[j]);
    gt += key > theta;
    eq += key == theta;
  }
  {
    uint32_t tot_gt, tot_eq;
    block_excl_scan(gt, sm.warp_tot, &tot_gt);
    block_excl_scan(eq, sm.warp_tot, &tot_eq);
    gt = tot_gt;
    eq = tot_eq;
  }
  uint32_t take = 0, off = 0;
  if (C > 1) {
    uint32_t* cnt = row_ws + kOffCnt;
    if (threadIdx.x == 0) {
      __stcg(cnt + 2 * c, gt);
      __stcg(cnt + 2 * c + 1, eq);
    }
    if (!group_barrier(bar, C, ws_header, 4)) return;
    // prefix over the CTAs before this one (in token order)
    uint32_t my_gt = 0, my_eq = 0;
    for (int cc = threadIdx.x; cc < c; cc += kThreads) {
      my_gt += __ldcg(cnt + 2 * cc);
      my_eq += __ldcg(cnt + 2 * cc + 1);
    }
    uint32_t gt_before, eq_before;
    block_excl_scan(my_gt, sm.warp_tot, &gt_before);
    block_excl_scan(my_eq, sm.warp_tot, &eq_before);
    // ties are taken in token order: CTAs before this one took min(eq_before, ties_needed)
    const uint32_t ties_before = min(eq_before, ties_needed);
    take = min(eq, ties_needed - ties_before);
    off = gt_before + ties_before;
    // every CTA of the row is past its last read of the histograms: clear this
    // CTA's share so the workspace is clean for the next call
    const int per = (kHistWords + C - 1) / C;
    const int h0 = c * per, h1 = min(kHistWords, h0 + per);
    for (int i = h0 + threadIdx.x; i < h1; i += kThreads) row_ws[i] = 0u;
  } else {
    take = ties_needed;
    off = 0;
  }

  write_selected(sm, sc, lo, hi, theta, take, off, keff, out, map, ws_header, b);
}

struct TopkLaunchCfg {
  int C, chunk;
};

TopkLaunchCfg topk_cfg(int B, int n_max) {
  // resident CTAs per SM, per device (0: not yet queried; a benign race stores the same value)
  constexpr int kMaxDevices = 64;
  static std::atomic<int> per_sm_dev[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) dev = 0;
  int per_sm = per_sm_dev[dev].load(std::memory_order_relaxed);
  if (per_sm == 0) {
    // with the dynamic shared memory of a multi-CTA row (the bound the cooperative launch needs)
    int v = 0;
    if (cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kDynWords * 4) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&v, topk_kernel, kThreads, kDynWords * 4) != cudaSuccess || v < 1)
      v = 1;
    per_sm = v;
    per_sm_dev[dev].store(v, std::memory_order_relaxed);
  }
  const int resident = per_sm * device_info().sm_count;
  int C = (n_max + 1023) / 1024;
  C = std::min(C, kMaxCtasPerRow);
  C = std::min(C, std::max(1, resident / std::max(B, 1)));
  if (C < 1) C = 1;
  const int chunk = (n_max + C - 1) / C;
  return {C, chunk};
}

}  // namespace

size_t topk_ws_bytes(int B, int n_max, int /*k*/) {
  if (topk_cfg(B, n_max).C == 1) return 0;  // one CTA per row: histograms stay in shared memory
  return align_up((size_t)B * kRowWords * sizeof(uint32_t), 256);
}

cudaError_t launch_topk(const float* scores, const int32_t* seq_lens, int B, int n_max, int k,
                        int32_t* idx, int32_t* count, void* ws_header, void* topk_ws, cudaStream_t s,
                        int causal_base, const int32_t* row_skip, int skip_val, const int32_t* idx_map,
                        int ld_map) {
  const TopkLaunchCfg cfg = topk_cfg(B, n_max);
  dim3 grid(cfg.C, B);
  int C = cfg.C, chunk = cfg.chunk;
  uint32_t* rw = static_cast<uint32_t*>(topk_ws);
  void* args[] = {(void*)&scores, (void*)&seq_lens, (void*)&n_max, (void*)&k, (void*)&C, (void*)&chunk,
                  (void*)&idx, (void*)&count, (void*)&ws_header, (void*)&rw, (void*)&causal_base,
                  (void*)&row_skip, (void*)&skip_val, (void*)&idx_map, (void*)&ld_map};
  cudaError_t e;
  if (C > 1) {
    e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kDynWords * 4);
    if (e == cudaSuccess)
      e = cudaLaunchCooperativeKernel((const void*)topk_kernel, grid, dim3(kThreads), args, kDynWords * 4, s);
  } else {
    e = cudaLaunchKernel((const void*)topk_kernel, grid, dim3(kThreads), args, 0, s);
  }
  launches_add(1, s);
  return e;
}

}  // namespace clsa
