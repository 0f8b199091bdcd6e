/*
 * clsa.h -- C ABI of libclsa.so, the B200 (sm_100a) implementation of the
 * Cross-Layer Sparse Attention (CLSA) shared-routing hot path.
 *
 * The method ("You Only Index Once: Cross-Layer Sparse Attention with Shared
 * Routing"; picx.dev summary, Methodology > Architecture Overview):
 *   routing equation    I = Q_idx K_idx^T ,  S_t = TopK(I_t, k)     -- once per token
 *   per-layer equation  O_t^(l) = Attn(Q_t^(l), K_{S_t}, V_{S_t})    -- every layer l
 * with Attn(Q, K, V) = softmax(Q K^T / sqrt(d_k)) V (zhichai.net post "CLSA
 * Explained", Background: Attention and Its Limits), K/V one shared (YOCO) cache,
 * and the selected rows gathered by the shared index ("Selector", zhichai.net
 * post, CLSA: Sharing the Index Across Layers).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Pointers.    Every tensor pointer is a DEVICE pointer (cudaMalloc'd or
 *              equivalent) unless stated otherwise, 16-byte aligned, dense,
 *              row-major in the layout given.  The caller owns every buffer;
 *              the library never allocates device memory and keeps no state
 *              between calls other than what lives in the caller's workspace.
 * Streams.     `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *              stream).  Every call is asynchronous on that stream.
 * dtype.       CLSA_F32 or CLSA_BF16 for every floating input of one call;
 *              outputs O are written in the same dtype (bf16 rounded to nearest
 *              even from fp32); scores and lse are always fp32.  All scoring,
 *              softmax and accumulation are fp32.
 * Shapes.      d, d_idx in {64, 128}; Hq % Hkv == 0; 1 <= k <= 4096
 *              (clsa_sparse_attn: 1 <= k <= 2^24, the rows are read directly);
 *              B >= 1; 0 <= seq_lens[b] <= n_max (seq_lens is device int32).
 *              Other shapes return CLSA_ERR_UNSUPPORTED before any launch.
 * scale.       Attention scale; a value <= 0 selects 1/sqrt(d).
 * TopK order.  Largest score first; equal scores go to the lower token index;
 *              -0.0 equals +0.0.  The selected indices of a row are written in
 *              ascending token order, k_eff = min(k, len) of them, and the rest
 *              of the row is -1.  count[b] = k_eff.  Scores must not be NaN.
 * GQA.         Query head h reads KV head h / (Hq / Hkv).
 * Workspace.   `ws` is a caller-owned device buffer of at least the size the
 *              matching *_workspace_size function returns.  It must be zeroed
 *              once before first use (clsa_workspace_init) and again after any
 *              call reported CLSA_ERR_TIMEOUT; the kernels leave it clean after
 *              a successful call.  Clean means clean for the entry point and
 *              sizes that last used it: before handing a workspace to another
 *              entry point or other sizes, zero it again.  One workspace must not
 *              be used by two calls that can run at the same time.
 * Errors.      Argument errors return before anything is launched.  Errors the
 *              kernels detect (an out-of-range index, a wait that ran out)
 *              are recorded in the workspace and read with
 *              clsa_read_device_status.  A failed launch returns CLSA_ERR_CUDA.
 *              No kernel traps or asserts.
 */
#ifndef CLSA_H_
#define CLSA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define CLSA_API __attribute__((visibility("default")))
#else
#define CLSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum clsa_status {
  CLSA_OK = 0,
  CLSA_ERR_INVALID_ARG = 1,  /* null pointer, bad size, misaligned pointer     */
  CLSA_ERR_UNSUPPORTED = 2,  /* shape outside the supported set               */
  CLSA_ERR_WORKSPACE = 3,    /* workspace missing or smaller than required     */
  CLSA_ERR_CUDA = 4,         /* a CUDA launch or copy failed                   */
  CLSA_ERR_TIMEOUT = 5,      /* an inter-CTA wait ran out (device-detected)    */
  CLSA_ERR_BAD_INDEX = 6     /* a gather index outside [0, n_max) (device)     */
} clsa_status;

typedef enum clsa_dtype { CLSA_F32 = 0, CLSA_BF16 = 1 } clsa_dtype;

/* ------------------------------------------------------------------------ */
/* Routing equation, scores: I[b, j] = q_idx[b] . k_idx[b, j]                */
/* ------------------------------------------------------------------------ */
/* q_idx [B][d_idx], k_idx [B][n_max][d_idx] (dtype dt); scores [B][n_max]
 * fp32 out: entries j < seq_lens[b] hold the dot product (fp32 accumulation of
 * exact products), entries j >= seq_lens[b] are -inf.  No scale or activation
 * (the indexer is a single head with a bare product).  Needs no workspace. */
CLSA_API clsa_status clsa_index_scores(const void* q_idx, const void* k_idx, const int32_t* seq_lens,
                              int B, int n_max, int d_idx, clsa_dtype dt, float* scores,
                              void* stream);

/* ------------------------------------------------------------------------ */
/* Routing equation, selection: S_b = TopK(I_b, k)  (exact radix select)     */
/* ------------------------------------------------------------------------ */
/* scores [B][n_max] fp32 (only j < seq_lens[b] are read); idx [B][k] int32 and
 * count [B] int32 out, ordered as in "TopK order" above.  The result is exact:
 * bit-identical to a stable sort of the same fp32 scores. */
CLSA_API size_t clsa_topk_workspace_size(int B, int n_max, int k);
CLSA_API clsa_status clsa_topk(const float* scores, const int32_t* seq_lens, int B, int n_max, int k,
                      int32_t* idx, int32_t* count, void* ws, size_t ws_bytes, void* stream);

/* Allocation-free TopK.  The paper has no counterpart for this entry point; it
 * exists for callers that cannot call cudaMalloc: code that runs inside another
 * runtime's memory pool and gets no allocator handle, or a path that must not
 * risk the device synchronisation cudaMalloc/cudaFree can cause.  It computes
 * exactly what clsa_topk computes (same kernel, same result) but takes no
 * workspace: its scratch is a fixed 2 MiB array inside the library, held on
 * every GPU that loads the library until the process exits.
 *   - The first call on a device looks up that array's device address; make
 *     that first call before any stream capture.
 *   - Each call clears the part of the array it uses on `stream` before the
 *     kernel runs.  Calls that overlap on the GPU (other streams, other host
 *     threads) share the array and race: serialise them.
 *   - A size is refused with CLSA_ERR_UNSUPPORTED exactly when
 *     clsa_topk_workspace_size(B, n_max, k) exceeds 2 MiB (at n_max = 128K that
 *     is a middle range of B, where each row still gets several CTAs).
 *   - The array's address belongs to the device's primary context: after
 *     cudaDeviceReset on a device, do not call this entry point there again.
 *   - Errors the kernel records on the device are not reported (there is no
 *     caller workspace to hold them); argument errors are returned as usual.
 * Allocates nothing: no cudaMalloc, cudaFree or allocating library call. */
CLSA_API clsa_status clsa_topk_noalloc(const float* scores, const int32_t* seq_lens, int B, int n_max,
                                       int k, int32_t* idx, int32_t* count, void* stream);

/* ------------------------------------------------------------------------ */
/* Selector: gather the selected K/V rows once into a compact buffer          */
/* ------------------------------------------------------------------------ */
/* K, V [B][n_max][Hkv][d]; idx [B][k], count [B] as written by clsa_topk.
 * K_S, V_S [B][k][Hkv][d] out: row i < count[b] is the cache row idx[b][i];
 * rows i >= count[b] are left untouched.  An index outside [0, n_max) is not
 * read: its row is zero-filled and CLSA_ERR_BAD_INDEX is recorded in ws. */
CLSA_API size_t clsa_gather_kv_workspace_size(void);
CLSA_API clsa_status clsa_gather_kv(const void* K, const void* V, const int32_t* idx, const int32_t* count,
                           int B, int n_max, int k, int Hkv, int d, clsa_dtype dt,
                           void* K_S, void* V_S, void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------ */
/* Per-layer equation: O^(l) = softmax(Q^(l) K_S^T * scale) V_S               */
/* ------------------------------------------------------------------------ */
/* Q [L][B][Hq][d]: the queries of L >= 1 layers that share one selection (L = 1
 * is the per-layer call a model makes layer by layer).  K_S, V_S [B][k][Hkv][d]
 * compact rows, count [B] valid rows per sequence.  O [L][B][Hq][d] out;
 * lse [L][B][Hq] fp32 out (natural-log sum of exp of the scaled scores), may
 * be NULL.  A sequence with count 0 gets O = 0 and lse = -inf.  k may exceed
 * the selection limit (up to 2^24): passing the whole cache as K_S/V_S with
 * count = seq_lens is dense attention over it.
 * Split-k flash decoding with an online softmax; fp32 accumulation. */
CLSA_API size_t clsa_sparse_attn_workspace_size(int B, int k, int L, int Hq, int Hkv, int d);
CLSA_API clsa_status clsa_sparse_attn(const void* Q, const void* K_S, const void* V_S, const int32_t* count,
                             int B, int k, int L, int Hq, int Hkv, int d, float scale,
                             clsa_dtype dt, void* O, float* lse, void* ws, size_t ws_bytes,
                             void* stream);

/* ------------------------------------------------------------------------ */
/* Attention-mass coverage of the shared selection                            */
/* ------------------------------------------------------------------------ */
/* picx.dev CLSA summary, Attention Sparsity Analysis: the share of each layer's
 * dense softmax mass that the selected tokens hold,
 *   mass[l][b][h] = sum_{j in S_b} softmax_j(Q^(l)[b,h] K[b]^T * scale)
 *                 = exp(lse_S[l][b][h] - lse_all[l][b][h]),
 * with lse_S the lse the decode step returned for the selection (clsa_decode_step's
 * `lse` output) and lse_all the lse over every one of the len_b cached rows.
 * Q [L][B][Hq][d], K [B][n_max][Hkv][d] in dt; lse_sparse [L][B][Hq] fp32 (natural
 * log); seq_lens [B] device int32.  mass [L][B][Hq] fp32 out (0 where either lse is
 * -inf); lse_all [L][B][Hq] fp32 out, may be NULL.  Query head h reads KV head
 * h / (Hq / Hkv); scale <= 0 selects 1/sqrt(d).  V is not read (the lse does not use
 * it).  bf16 with d = 128 streams K once on the tensor cores (per-split row max and
 * sum, then one merge in split order: deterministic), 2 launches; other shapes take
 * the row lse from the split-k attention kernel.  Caller-owned workspace of
 * clsa_attention_mass_workspace_size bytes; errors as above. */
CLSA_API size_t clsa_attention_mass_workspace_size(int B, int n_max, int L, int Hq, int Hkv, int d);
CLSA_API clsa_status clsa_attention_mass(const void* Q, const void* K, const float* lse_sparse,
                                         const int32_t* seq_lens, int B, int n_max, int L, int Hq, int Hkv,
                                         int d, float scale, clsa_dtype dt, float* mass, float* lse_all,
                                         void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------ */
/* Distillation target of the shared indexer (forward only)                   */
/* ------------------------------------------------------------------------ */
/* picx.dev CLSA summary, Methodology > Architecture Overview, multi-layer
 * distillation: for each decode query b,
 *   Abar_b = 1/(L Hq) sum_{l,h} softmax(Q^(l)[b,h] K[b]^T * scale)  over its len_b rows
 *   kl[b]  = KL(Abar_b || softmax(I_b)),   I = the indexer scores (no scale)
 * Query head h reads KV head h / (Hq / Hkv); scale <= 0 selects 1/sqrt(d).
 * Q [L][B][Hq][d] and K [B][n_max][Hkv][d] in dt; scores [B][n_max] fp32 (e.g. from
 * clsa_index_scores); seq_lens [B] device int32.  abar [B][n_max] fp32 out (0 past
 * len_b), may be NULL; kl [B] fp32 out (0 for an empty sequence).  1 <= n_max <= 2^24.
 * fp32 arithmetic; the result is deterministic (fixed reduction orders).  bf16 with
 * d = 128 runs on the tensor cores (bf16 products, fp32 sums): two streaming passes over
 * K (row lse, then Abar), 4 launches; other shapes run on CUDA cores.
 * Caller-owned workspace of clsa_distill_workspace_size bytes; errors as above. */
CLSA_API size_t clsa_distill_workspace_size(int B, int n_max, int L, int Hq, int Hkv, int d);
CLSA_API clsa_status clsa_distill_target(const void* Q, const void* K, const float* scores,
                             const int32_t* seq_lens, int B, int n_max, int L, int Hq, int Hkv,
                             int d, float scale, clsa_dtype dt, float* abar, float* kl, void* ws,
                             size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------ */
/* One decode step: score once, select once, gather once, attend in L layers */
/* ------------------------------------------------------------------------ */
typedef struct clsa_decode_args {
  clsa_dtype dtype;
  int B, n_max, d_idx, k, L, Hq, Hkv, d;
  float scale;               /* <= 0: 1/sqrt(d)                                   */
  const void* q_idx;         /* [B][d_idx]                                        */
  const void* k_idx;         /* [B][n_max][d_idx]                                 */
  const void* K;             /* [B][n_max][Hkv][d]  shared by every layer         */
  const void* V;             /* [B][n_max][Hkv][d]                                */
  const void* Q;             /* [L][B][Hq][d]       one query per layer           */
  const int32_t* seq_lens;   /* [B]                                               */
  void* O;                   /* out [L][B][Hq][d]                                 */
  int32_t* idx;              /* out [B][k]  the shared S, ascending, -1 padded    */
  int32_t* count;            /* out [B]                                           */
  float* scores;             /* out [B][n_max] or NULL (kept in the workspace)    */
  float* lse;                /* out [L][B][Hq] or NULL                            */
  void* K_S;                 /* out [B][k][Hkv][d] compact gathered rows, or NULL */
  void* V_S;                 /* out, NULL exactly when K_S is NULL                */
} clsa_decode_args;
/* With K_S/V_S NULL the attention kernel reads each selected cache row once
 * straight from K/V for all L layers (the gather is fused); with them set,
 * the rows are first compacted there and attention reads the compact copy. */
CLSA_API size_t clsa_decode_workspace_size(const clsa_decode_args* a);
CLSA_API clsa_status clsa_decode_step(const clsa_decode_args* a, void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------ */
/* Prefill chunk: T new rows at cache positions n-T .. n-1, causal            */
/* ------------------------------------------------------------------------ */
typedef struct clsa_prefill_args {
  clsa_dtype dtype;          /* CLSA_BF16 (the scores GEMM runs on tcgen05)       */
  int n, T, d_idx, k, L, Hq, Hkv, d;
  float scale;
  const void* q_idx;         /* [T][d_idx]  index queries of the new rows         */
  const void* k_idx;         /* [n][d_idx]  index keys of the whole cache         */
  const void* K;             /* [n][Hkv][d]                                       */
  const void* V;             /* [n][Hkv][d]                                       */
  const void* Q;             /* [L][T][Hq][d]                                     */
  void* O;                   /* out [L][T][Hq][d]                                 */
  int32_t* idx;              /* out [T][k]: row i selects among tokens j <= n-T+i */
  int32_t* count;            /* out [T]: min(k, n-T+i+1)                          */
  float* lse;                /* out [L][T][Hq] or NULL                            */
} clsa_prefill_args;
CLSA_API size_t clsa_prefill_workspace_size(const clsa_prefill_args* a);
CLSA_API clsa_status clsa_prefill_chunk(const clsa_prefill_args* a, void* ws, size_t ws_bytes, void* stream);

/* The attention stage of a prefill chunk alone: the per-layer equation for every new row
 * over the selection already in a->idx / a->count (as clsa_prefill_chunk writes them:
 * ascending token order per row), writing a->O and a->lse.  q_idx and k_idx are not read.
 * mode 0: each row on its own (what clsa_prefill_chunk runs).
 * mode 1: key-centric.  Rows go in pairs (t, t + 1); a pair fetches each K/V row of the
 *   union of its two selections once and scores it against both rows' queries, each row
 *   keeping only the tokens it selected (an implementation choice, not on the pages; the
 *   results equal mode 0's up to the fp32 summation order).  bf16, d = 128, k <= 4096;
 *   other shapes return CLSA_ERR_UNSUPPORTED.
 * Workspace: clsa_prefill_workspace_size(a) bytes, zeroed as usual; errors as above. */
CLSA_API clsa_status clsa_prefill_attention(const clsa_prefill_args* a, int mode, void* ws, size_t ws_bytes,
                                            void* stream);

/* ------------------------------------------------------------------------ */
/* Helpers                                                                    */
/* ------------------------------------------------------------------------ */
/* Workspace bytes of an operation, given its argument struct: op CLSA_OP_DECODE_STEP
 * (args: const clsa_decode_args*) or CLSA_OP_PREFILL_CHUNK (args: const clsa_prefill_args*).
 * The same value as clsa_decode_workspace_size / clsa_prefill_workspace_size; 0 for an
 * unknown op, a NULL args, or arguments that call would reject.  The stage calls have their
 * own size functions above. */
typedef enum { CLSA_OP_DECODE_STEP = 0, CLSA_OP_PREFILL_CHUNK = 1 } clsa_op;
CLSA_API size_t clsa_workspace_size(int op, const void* args);
/* Zero `bytes` of workspace on `stream` (asynchronous). */
CLSA_API clsa_status clsa_workspace_init(void* ws, size_t bytes, void* stream);
/* Synchronise `stream`, return the first device-detected error recorded in
 * `ws` (CLSA_OK if none) and clear it.  `detail`, if not NULL, receives a
 * kernel-specific code (the offending index, or the wait site). */
CLSA_API clsa_status clsa_read_device_status(void* ws, void* stream, int64_t* detail);
CLSA_API const char* clsa_status_string(clsa_status s);
/* Failure-detection self-test.  Launches one CTA on `stream` whose wait nothing will
 * satisfy -- which = 0: the inter-CTA count barrier, for two CTAs with one launched;
 * which = 1: an mbarrier phase that expects one arrival and gets none.  The wait runs
 * out after the library's limit (200 ms of GPU time), records CLSA_ERR_TIMEOUT with
 * detail 900 + which in `ws`, and the kernel returns: clsa_read_device_status then
 * reports it, and the stream and context stay usable.  Returns CLSA_OK once launched;
 * CLSA_ERR_INVALID_ARG for another `which`; CLSA_ERR_WORKSPACE if `ws` is NULL, not
 * 16-byte aligned or under 512 bytes.  Uses the first 4 bytes after the 256-byte
 * header as its barrier word (zeroed on `stream` first). */
CLSA_API clsa_status clsa_selftest_timeout(int which, void* ws, size_t ws_bytes, void* stream);
/* Library version as major*10000 + minor*100 + patch. */
CLSA_API int clsa_version(void);
/* Number of kernel launches the last call made on this host thread. */
CLSA_API int clsa_last_launch_count(void);
/* Launch timing (instrumentation; no counterpart on the pages).  Arms the next
 * library call made on this host thread: on that call's stream it records
 * events[0] before its first kernel launch and events[i] right after its i-th
 * launch (a group of launches made together counts once), up to max_events
 * events in all.  events are cudaEvent_t handles the caller created (timing
 * enabled) and keeps alive until they complete; cudaEventElapsedTime of
 * consecutive events then gives each launch's device time.  max_events = 0
 * disarms.  Only the next call is armed.  clsa_timed_event_count() returns how
 * many events the last armed call recorded. */
CLSA_API clsa_status clsa_time_next_call(void* const* events, int max_events);
CLSA_API int clsa_timed_event_count(void);

#ifdef __cplusplus
}
#endif
#endif /* CLSA_H_ */
