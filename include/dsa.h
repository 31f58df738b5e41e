/*
 * dsa.h -- C ABI of libdsa.so: the hot path of DeepSeek Sparse Attention (DSA) for a GQA decoder
 * on NVIDIA B200 (sm_100a).
 *
 * The path has three steps (page "快手开源大模型Keye-VL-2.0：一个能“看懂“两小时视频AI",
 * gsyq.cn, section 一; page "从“看”到“想”多模态大模型推理能力的瓶颈与突破", wmrh.cn, section 2):
 *   1. an MQA-shared lightning indexer scores every causal key for each query token,
 *        score(t, s) = sum_h w[t,h] * max(0, qI[t,h,:] . kI[s,:])      (s <= t)
 *      (the pages give no formula; this is the one the library adopts: no scale, no bias);
 *   2. the top-k keys of each row are selected (k = 2048 on the pages), ties to the lower index;
 *   3. scaled-dot-product attention runs over the selected keys only, one index set per token
 *      shared by every GQA KV group (query head h reads KV head h / (Hq/Hkv)).
 *
 * Conventions for every entry point
 *   - Pointers are DEVICE pointers the caller owns (allocated by any means); the library never
 *     allocates device memory and never frees caller memory.  Tensors are contiguous,
 *     row-major, with the shapes given, and must be 16-byte aligned.
 *   - bf16 means IEEE bfloat16 stored as uint16; scores are fp32; indices are int32.
 *   - Every call runs on the calling thread's current CUDA device (cudaSetDevice); its pointers
 *     and `stream` must belong to that device.  A process may drive several devices in turn.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL is the legacy default stream).
 *     The return value reports host-side validation and launch errors only.  When it is not
 *     DSA_OK nothing was launched (or, for DSA_ERR_CUDA, a launch failed).
 *   - Problems found on the device (a bounded wait that expired, a context length beyond the
 *     cache) set a device error word; dsa_sync_status() synchronises the stream, reads and
 *     clears it.  Nothing in the library traps or aborts the process.
 *   - Supported shapes: head dim D = 128, indexer dim dI = 64, indexer heads HI in
 *     {1,2,4,8,16,32,64} (decode: {16,32,64}), Hkv in {1,2,4}, Hq = G * Hkv with G <= 16,
 *     1 <= topk <= 65536.  Anything else returns DSA_ERR_UNSUPPORTED.
 */
#ifndef DSA_H
#define DSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *dsa_stream_t; /* same type as cudaStream_t */

typedef enum {
    DSA_OK = 0,
    DSA_ERR_INVALID_ARG = 1,  /* null or misaligned pointer, non-positive size, bad stride */
    DSA_ERR_UNSUPPORTED = 2,  /* valid arguments outside the supported shapes above */
    DSA_ERR_WORKSPACE = 3,    /* workspace pointer null or smaller than required */
    DSA_ERR_CUDA = 4,         /* a CUDA runtime/driver call or a launch failed */
    DSA_ERR_TIMEOUT = 5,      /* a kernel's bounded wait expired (from dsa_sync_status) */
    DSA_ERR_DEVICE_INPUT = 6  /* a device-side input check failed, e.g. ctx_len >= Lmax
                                 (from dsa_sync_status) */
} dsa_status;

/* Workspace kinds for dsa_workspace_size(). */
enum { DSA_OP_INDEX = 0, DSA_OP_TOPK = 1, DSA_OP_SPARSE_ATTN = 2, DSA_OP_PREFILL = 3, DSA_OP_DECODE = 4,
       DSA_OP_INDEXER_KL = 5 };

/* Human-readable name of a status code (static string, never NULL). */
const char *dsa_status_string(int status);

/* Library version as major*10000 + minor*100 + patch. */
int dsa_version(void);

/*
 * Step 1 -- lightning-indexer scores for Lq query rows of one causal sequence.
 *   qI      bf16 [Lq, HI, dI]   indexer queries of rows q_pos0 .. q_pos0+Lq-1
 *   kI      bf16 [Lk, dI]       the MQA-shared indexer key of every position (Lk >= q_pos0+Lq)
 *   w       bf16 [Lq, HI]       per-token head weights (any sign)
 *   scores  fp32, row i at scores + i*ld_scores; for every i < Lq and s <= q_pos0+i,
 *           scores[i, s] = sum_h w[i,h] * max(0, qI[i,h,:] . kI[s,:]) with fp32 accumulation.
 *           Entries with s > q_pos0+i are not written.  ld_scores >= q_pos0+Lq, multiple of 4.
 * Runs on the tensor cores (tcgen05, TMA).  Cites: page gsyq.cn section 一 (MQA-shared scout).
 */
dsa_status dsa_index(const void *qI, const void *kI, const void *w, int Lq, int64_t Lk, int HI, int dI,
                     int64_t q_pos0, float *scores, int64_t ld_scores, dsa_stream_t stream);

/*
 * Step 2 -- per-row top-k.  Row i holds n_i = q_pos0+i+1 valid scores (row i at
 * scores + i*ld_scores, ld_scores a multiple of 4 and >= q_pos0+Lq).
 *   idx     int32 [Lq, k]: the min(k, n_i) keys with the largest scores (equal scores: lower key
 *           index first), then -1 padding.  Exact and deterministic: a row's output depends
 *           only on that row's scores (not on Lq, chunking or the kernel variant).  Order within
 *           a row: when the row has no more than k competing keys, all of them in ascending
 *           order; otherwise the selected keys grouped by region ((index / 32) mod 4, regions 0..3
 *           in turn), ascending within a region.  Callers may treat a row as a set.
 *   ws, ws_bytes  unused (may be NULL/0); kept so callers can pass a workspace uniformly.
 * Cites: page gsyq.cn section 一 (top 2048 per token), section 八 (deterministic top-k).
 */
dsa_status dsa_topk(const float *scores, int64_t ld_scores, int Lq, int64_t q_pos0, int k, int32_t *idx,
                    void *ws, size_t ws_bytes, dsa_stream_t stream);

/*
 * Step 2 with a sliding window (SW-DSA: page "DSA注意力机制：多模态学习中的强化推理新范式",
 * showapi.com, section 1.4, restricts the selection to a local window).  As dsa_topk, except
 * that row i (query position t = q_pos0+i) selects among keys max(0, t-window+1) .. t only:
 * the min(k, min(window, t+1)) best of them, -1 padded.  window = 0 means no window (identical to
 * dsa_topk); window < 0 is invalid.
 */
dsa_status dsa_topk_window(const float *scores, int64_t ld_scores, int Lq, int64_t q_pos0, int k, int64_t window,
                           int32_t *idx, dsa_stream_t stream);

/*
 * Step 3 -- sparse attention over selected keys (prefill layout).
 *   q       bf16 [Lq, Hq, D]    queries of rows q_pos0 .. q_pos0+Lq-1
 *   k, v    bf16 [Lk, Hkv, D]   keys/values of the whole sequence
 *   idx     int32 [Lq, topk]    selected keys; row i uses its first min(topk, q_pos0+i+1)
 *                               entries; entries < 0 or >= Lk are skipped
 *   out     bf16 [Lq, Hq, D];   lse fp32 [Lq, Hq] natural-log sum-exp of the scaled logits
 *                               (may be NULL)
 *   scale   softmax scale applied to q.k (1/sqrt(D) for standard attention)
 * Cites: page wmrh.cn section 2 step 3; page gsyq.cn section 一 (GQA adaptation).
 */
dsa_status dsa_sparse_attn(const void *q, const void *k, const void *v, const int32_t *idx, int Lq, int64_t Lk,
                           int64_t q_pos0, int Hq, int Hkv, int D, int topk, float scale, void *out, float *lse,
                           dsa_stream_t stream);

/*
 * Step 3 with adjacent-query deduplication (page gsyq.cn section 八): the same result as
 * dsa_sparse_attn, computed per block of 128/G adjacent rows (G = Hq/Hkv query heads per KV group)
 * over the union of the block's index sets: each union key's K/V rows are gathered once per KV
 * group, S = Q.K^T and O += P.V run as 128-row tensor-core tiles of the block's (row, head) pairs,
 * and each row's softmax masks the union keys it did not select.  Arguments and their layouts as
 * dsa_sparse_attn.  An index repeated within a row counts once (dsa_topk never repeats one).
 * Outputs differ from dsa_sparse_attn only by fp32 summation order and the bf16 rounding of the
 * probabilities.  Rows may list their keys in any order.
 * Errors: as dsa_sparse_attn; DSA_ERR_UNSUPPORTED unless G is 8 or 16, or if Lk > 2^21.
 */
dsa_status dsa_sparse_attn_dedup(const void *q, const void *k, const void *v, const int32_t *idx, int Lq, int64_t Lk,
                                 int64_t q_pos0, int Hq, int Hkv, int D, int topk, float scale, void *out,
                                 float *lse, dsa_stream_t stream);

/*
 * Steps 1-3 fused over a whole causal sequence of length L (prefill).  Processes query rows in
 * chunks whose score rows fit the workspace (more workspace = fewer, larger chunks; results do
 * not depend on the chunk size).
 *   q bf16 [L, Hq, D]; k, v bf16 [L, Hkv, D]; qI bf16 [L, HI, dI]; kI bf16 [L, dI]; w bf16 [L, HI]
 *   out bf16 [L, Hq, D]; idx_out int32 [L, topk] or NULL (then the workspace also holds indices)
 *   ws      device workspace of ws_bytes; at least dsa_workspace_size(DSA_OP_PREFILL, ...) for a
 *           minimal chunk: the score rows of one query block.  Recommended size: the value of
 *           dsa_workspace_size(DSA_OP_PREFILL, L, 1, Hq, HI, topk).
 * Cites: as the three steps.
 */
dsa_status dsa_prefill(const void *q, const void *k, const void *v, const void *qI, const void *kI, const void *w,
                       int64_t L, int Hq, int Hkv, int D, int HI, int dI, int topk, float scale, void *out,
                       int32_t *idx_out, void *ws, size_t ws_bytes, dsa_stream_t stream);

/*
 * Steps 1-3 for the query rows row0 .. row0+rows-1 of one causal sequence (chunked prefill, or
 * one rank's share of a sequence whose rows are spread over GPUs).  Row-local arrays:
 *   q bf16 [rows, Hq, D]; qI bf16 [rows, HI, dI]; w bf16 [rows, HI]; out bf16 [rows, Hq, D];
 *   idx_out int32 [rows, topk] or NULL.  Whole-sequence arrays, at least row0+rows positions:
 *   k, v bf16 [.., Hkv, D]; kI bf16 [.., dI].  window as in dsa_prefill_window (0 = none).
 *   ws      workspace for score rows of length row0+rows (see dsa_workspace_size with
 *           L = row0+rows).
 * Processing consecutive row ranges gives exactly dsa_prefill's results for those rows.
 */
dsa_status dsa_prefill_rows(const void *q, const void *k, const void *v, const void *qI, const void *kI,
                            const void *w, int64_t row0, int64_t rows, int Hq, int Hkv, int D, int HI, int dI,
                            int topk, int64_t window, float scale, void *out, int32_t *idx_out, void *ws,
                            size_t ws_bytes, dsa_stream_t stream);

/*
 * Indexer warm-up target, forward only (the pages' training stage 1 fits the scout to the full
 * attention distribution by minimising a KL divergence: page gsyq.cn, section 一; the pages
 * give no formula, this is the library's reading).  For every query position t < L:
 *   P_t(s) = (1/Hq) sum_h softmax_s(scale * q[t,h] . k[s, h / (Hq/Hkv)])   s = 0..t  (dense)
 *   Q_t(s) = softmax_s(score(t, s))          with score as in dsa_index
 *   kl[t]  = sum_s P_t(s) * (log P_t(s) - log Q_t(s))                      (natural log)
 *   q bf16 [L, Hq, D]; k bf16 [L, Hkv, D]; qI bf16 [L, HI, dI]; kI bf16 [L, dI]; w bf16 [L, HI]
 *   kl      float [L] (device, 4-byte aligned), written
 *   ws      a chunk of queries' score rows and per-head log-sum-exps (Hq floats a row): at least
 *           dsa_workspace_size(DSA_OP_INDEXER_KL, L, 1, Hq, HI, 1) bytes recommended; any size
 *           holding min(L, max(128, 256/HI)) rows works (smaller sizes mean more, shorter chunks;
 *           the results do not depend on the chunk size).
 * Supported: D = 128, dI = 64, Hq in {8, 16, 32, 64}, Hkv in {1, 2, 4} with Hq/Hkv >= 2, HI a
 * power of two <= 64.  Dense cost: 4 x Hq x D flop per causal (t, s) pair plus the indexer.
 * Status codes as dsa_prefill.
 */
dsa_status dsa_indexer_kl(const void *q, const void *k, const void *qI, const void *kI, const void *w, int64_t L,
                          int Hq, int Hkv, int D, int HI, int dI, float scale, float *kl, void *ws, size_t ws_bytes,
                          dsa_stream_t stream);

/*
 * dsa_prefill with a sliding window of `window` keys per query (SW-DSA, see dsa_topk_window): the
 * indexer skips key tiles that lie wholly before every window of a query block, top-k selects
 * within the window, attention runs over the selected keys.  window = 0: identical to dsa_prefill.
 */
dsa_status dsa_prefill_window(const void *q, const void *k, const void *v, const void *qI, const void *kI,
                              const void *w, int64_t L, int Hq, int Hkv, int D, int HI, int dI, int topk,
                              int64_t window, float scale, void *out, int32_t *idx_out, void *ws, size_t ws_bytes,
                              dsa_stream_t stream);

/*
 * One decode step for B sequences, each with one new token (the pages' decode path: page
 * gsyq.cn section 一 and section 八).
 *   ctx_len int32 [B] (device): tokens already cached per sequence.  The step writes the new
 *           token's k_new/v_new/kI_new rows at position ctx_len[b] of the caches, then attends
 *           over keys 0..ctx_len[b] (the new token included).  If update_ctx != 0, ctx_len[b] is
 *           incremented at the end of the step (so a loop of steps can run without the host).
 *           ctx_len[b] must be < Lmax; otherwise that sequence is skipped and dsa_sync_status()
 *           reports DSA_ERR_DEVICE_INPUT.
 *   q bf16 [B, Hq, D]; qI bf16 [B, HI, dI]; w bf16 [B, HI]
 *   k_new, v_new bf16 [B, Hkv, D]; kI_new bf16 [B, dI]
 *   k_cache, v_cache bf16 [B, Lmax, Hkv, D]; kI_cache bf16 [B, Lmax, dI]
 *   out bf16 [B, Hq, D]; idx_out int32 [B, topk] or NULL
 *   ws      at least dsa_workspace_size(DSA_OP_DECODE, Lmax, B, Hq, HI, topk) bytes.
 */
dsa_status dsa_decode(const void *q, const void *qI, const void *w, const void *k_new, const void *v_new,
                      const void *kI_new, void *k_cache, void *v_cache, void *kI_cache, int32_t *ctx_len, int B,
                      int64_t Lmax, int Hq, int Hkv, int D, int HI, int dI, int topk, float scale, int update_ctx,
                      void *out, int32_t *idx_out, void *ws, size_t ws_bytes, dsa_stream_t stream);

/*
 * dsa_decode without a caller workspace: the same decode step, with every piece of scratch it
 * needs (one fp32 score row per sequence, the index rows when idx_out is NULL, and the per-split
 * attention partials) taken from a fixed array inside the library's own device memory.  The
 * pages describe nothing like it: it exists for callers that cannot allocate device memory -- for
 * example a plugin inside a serving process whose memory pool owns the whole GPU and offers no
 * way to request workspace, or a caller that must not pay cudaMalloc's implicit device-wide
 * synchronisation on a latency-critical path.
 *   - The array holds dsa_decode_noalloc_scratch_bytes() = 16 MiB on every GPU where the library
 *     is loaded, from load until the process exits.
 *   - Sizes: the call returns DSA_ERR_WORKSPACE, launching nothing, when the step needs more than
 *     that, i.e. when dsa_workspace_size(DSA_OP_DECODE, Lmax, B, Hq, HI, topk) (with idx_out NULL;
 *     less when idx_out is given) exceeds 16 MiB.  B = 16 sequences of 131328 positions fit.
 *   - The first call on a device looks up the array's device address (cudaGetSymbolAddress) with
 *     that device current; make that first call before any stream capture.
 *   - All calls share the one array and it keeps the previous call's contents: no part of it has
 *     to start at zero (every kernel writes the scratch it later reads), but two calls that
 *     overlap on the GPU (different streams, or different threads) race on it.  Serialise them.
 *   - Arguments, results and errors are otherwise those of dsa_decode.
 */
dsa_status dsa_decode_noalloc(const void *q, const void *qI, const void *w, const void *k_new, const void *v_new,
                              const void *kI_new, void *k_cache, void *v_cache, void *kI_cache, int32_t *ctx_len,
                              int B, int64_t Lmax, int Hq, int Hkv, int D, int HI, int dI, int topk, float scale,
                              int update_ctx, void *out, int32_t *idx_out, dsa_stream_t stream);

/* Size in bytes of the fixed scratch array used by dsa_decode_noalloc. */
size_t dsa_decode_noalloc_scratch_bytes(void);

/*
 * Bytes of workspace an entry point needs.  op: DSA_OP_*.  L: sequence length (prefill) or cache
 * capacity Lmax (decode); B: sequences (decode); Hq: query heads; HI: indexer heads; topk.
 * DSA_OP_PREFILL returns the recommended size (score rows of up to 16 GiB per chunk plus index
 * rows; a smaller workspace works too, in more and shorter chunks, somewhat slower);
 * DSA_OP_INDEXER_KL the score rows alone, up to 4 GiB per chunk (topk ignored);
 * DSA_OP_INDEX/TOPK/SPARSE_ATTN return 0.  Returns 0 for invalid arguments.
 */
size_t dsa_workspace_size(int op, int64_t L, int B, int Hq, int HI, int topk);

/*
 * Synchronise `stream`, then read and clear the device error word.  Returns DSA_OK,
 * DSA_ERR_TIMEOUT, DSA_ERR_DEVICE_INPUT or DSA_ERR_CUDA (a sticky CUDA error).
 */
dsa_status dsa_sync_status(dsa_stream_t stream);

/*
 * Diagnostics: the code of the last device-side check or bounded wait that recorded an error
 * (low 12 bits: the site; higher bits: the loop index there, where the site has one); 0 if none
 * since the library was loaded.  Not cleared by dsa_sync_status.
 */
unsigned int dsa_error_site(void);

/*
 * Per-kernel timing.  dsa_profile_begin() starts recording a CUDA event pair around every
 * kernel the library launches (on the launching stream); dsa_profile_end() synchronises those
 * events, stops recording and returns, per kernel kind, the number of launches and the total
 * milliseconds.  Kinds: 0 indexer, 1 top-k, 2 sparse attention, 3 split combine, 4 decode
 * append and 5 context advance (both now done inside other kernels: always 0), 6 self-test,
 * 7 indexer warm-up KL.  Arrays have DSA_PROFILE_KINDS entries.
 */
#define DSA_PROFILE_KINDS 8
void dsa_profile_begin(void);
dsa_status dsa_profile_end(int64_t *launches, double *total_ms);

/*
 * Diagnostic path counters, accumulated on the device since load or the last reset:
 *   [0] top-k rows handled by the one-CTA-per-row kernel; [1] of those, rows whose first sampled
 *   threshold missed (a second estimate and pass followed); [4] rows whose second estimate also
 *   missed (exact radix select over the row); [2] rows handled by a CTA cluster (few long rows,
 *   decode), [3] of those, rows whose first threshold missed, [5] rows that took the exact radix
 *   select on the cluster's first CTA (a second miss, or more than 256 equal keys at the cutoff).  Copies up to n counters (n <= DSA_NUM_COUNTERS) into out after synchronising the
 *   device; if reset != 0 the counters are zeroed afterwards.  Returns DSA_ERR_CUDA on failure.
 */
#define DSA_NUM_COUNTERS 8
dsa_status dsa_read_counters(int64_t *out, int n, int reset);

/* Number of kernels the library has launched since it was loaded. */
int64_t dsa_launch_count(void);

/*
 * Failure-path self test: launches one tiny kernel whose mbarrier wait can never complete and is
 * bounded by wait_ns nanoseconds; the kernel records DSA_ERR_TIMEOUT in the device error word
 * and returns.  Used to check, on a GPU, that a bounded wait ends with an error status and
 * leaves the context usable (call dsa_sync_status() afterwards).  0 < wait_ns <= 2e9.
 */
dsa_status dsa_selftest_timeout(int64_t wait_ns, dsa_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* DSA_H */
