/*
 * minf.h -- C ABI of the B200 (sm_100a) dynamic sparse prefill attention library.
 *
 * The library implements the online half of MInference-style dynamic sparse
 * attention for the long-context pre-filling stage: per-head sparse-index
 * estimation (Vertical-Slash, Block-Sparse) and the causal sparse attention
 * that consumes the indices (Vertical-Slash, Block-Sparse, A-shape), plus a
 * dense causal attention kernel used as the comparison baseline.
 *
 * Sources (page title, section):
 *   [NEWS] "单卡A100实现百万token推理，速度快10倍，这是微软官方的大模型推理加速"
 *          (yntaolf.cn), section 方法介绍 -- the three patterns; Vertical-Slash
 *          indices estimated from the attention of the last queries against all
 *          keys; Block-Sparse indices from mean-pooled Q and K multiplied
 *          (pooling commutes with the product); block-sparse FlashAttention.
 *          Section 延迟和内核中的稀疏模式, Figure 4 -- inside the kernel the
 *          verticals are 1x64 pieces and the slashes 64x64 blocks.
 *   [TALK] "以 KV 缓存为中心的高效长文本方法" (AICon 2025 talk transcript,
 *          dify360.com), second observation -- A-shape (initial tokens plus a
 *          local window), vertical lines, slash lines, block clusters; the
 *          offline/online split with per-head patterns.
 *
 * Conventions shared by every call:
 *   - Tensors are CALLER-OWNED DEVICE buffers on one CUDA device; the library
 *     allocates no device memory.  Scratch space is the caller's `ws` buffer of
 *     at least minf_workspace_bytes(...) bytes (256-byte aligned).
 *   - q is bf16 [hq][n][128], k and v are bf16 [hkv][n][128], row-major and
 *     contiguous; d must be 128.  GQA: q-head h reads kv-head h / (hq / hkv).
 *   - n must be a positive multiple of 64 (MINF_ERR_UNSUPPORTED otherwise).
 *   - head_ids is an optional HOST array of n_heads q-head ids (distinct, each
 *     in [0, hq)); NULL means every head, n_heads = hq.  Outputs are indexed by
 *     position in that list: out [n_heads][n][128] bf16, lse [n_heads][n] fp32
 *     (natural log of the softmax denominator; -inf for a row with no key).
 *     At most MINF_MAX_HEADS heads per call.
 *   - scale multiplies q.k before the softmax and must be > 0 (1/sqrt(128) is
 *     the usual value).
 *   - Every call is asynchronous on `stream` (a cudaStream_t); the return value
 *     reports argument checks and launch errors only.  A device-side failure
 *     (a bounded wait that ran out) is recorded in the workspace status word and
 *     read back by minf_status().
 *   - Causal masking throughout: query i sees keys k <= i only.
 *
 * Return codes: MINF_OK, or a negative MINF_ERR_* value; arguments are checked
 * on the host before anything is launched, so an error return launches nothing.
 */
#ifndef MINF_H
#define MINF_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t minf_bf16;                /* raw bf16 bits */
typedef struct CUstream_st *minf_stream_t; /* the same type as cudaStream_t */

#define MINF_OK 0
#define MINF_ERR_INVALID (-1)     /* null pointer, hq % hkv != 0, budget < 1, bad head id, scale <= 0 */
#define MINF_ERR_UNSUPPORTED (-2) /* d != 128, n % 64 != 0, block != 64, last_q > 64, no sm_100 device */
#define MINF_ERR_CUDA (-3)        /* a CUDA runtime/driver call or launch failed */
#define MINF_ERR_TIMEOUT (-4)     /* a device-side bounded wait gave up (see minf_status) */
#define MINF_ERR_WORKSPACE (-5)   /* ws_bytes smaller than minf_workspace_bytes(...) */

#define MINF_MAX_HEADS 256

/* Operation codes for minf_workspace_bytes. */
#define MINF_OP_VS_ESTIMATE 1
#define MINF_OP_VS_ATTENTION 2
#define MINF_OP_BLOCK_ESTIMATE 3
#define MINF_OP_BLOCK_ATTENTION 4
#define MINF_OP_ASHAPE_ATTENTION 5
#define MINF_OP_DENSE_ATTENTION 6
#define MINF_OP_MIXED_LAYER 7
#define MINF_OP_TRISHAPE_ATTENTION 8

/* Per-head pattern codes for minf_mixed_layer. */
#define MINF_PATTERN_DENSE 0
#define MINF_PATTERN_VS 1
#define MINF_PATTERN_BLOCK 2
#define MINF_PATTERN_ASHAPE 3
#define MINF_PATTERN_TRISHAPE 4

/*
 * Bytes of workspace an operation needs.  p1/p2/p3 by op:
 *   VS_ESTIMATE, VS_ATTENTION: p1 = n_vertical, p2 = n_slash
 *   BLOCK_ESTIMATE, BLOCK_ATTENTION: p1 = topk
 *   MIXED_LAYER: p1 = n_vertical, p2 = n_slash, p3 = topk (n_heads ignored: all hq heads)
 *   others: unused.
 * Returns 0 for arguments the op would reject.  Growth: VS_ATTENTION keeps, per
 * listed head and 128-query tile, the list of vertical keys that no slash range
 * of the tile covers, so it needs about n_heads * (n / 128) * min(n_vertical, n)
 * * 4 bytes (1 GiB for 32 heads at 1M tokens with 1000 verticals); the others
 * grow as n_heads * n.  VS_ESTIMATE also serves minf_vs_estimate_topp.
 */
size_t minf_workspace_bytes(int op, int hq, int hkv, int n, int n_heads, int p1, int p2, int p3);

/*
 * Vertical-Slash index estimation ([NEWS] 方法介绍).  For each listed q-head,
 * the softmax rows of the last `last_q` queries (causal, keys k <= i) are
 * summed along columns (vertical score of key k) and along diagonals (slash
 * score of offset o = i - k).  Offset 0 is forced into the slash set and takes
 * one slot.  The best min(n_vertical, n) keys and min(n_slash, n) offsets are
 * kept, ties to the lower index, and written ASCENDING:
 *   v_idx int32 [n_heads][n_vertical], s_idx int32 [n_heads][n_slash],
 *   each row padded with -1 past its min(budget, n) valid entries.
 * 1 <= last_q <= 64.
 */
int minf_vs_estimate(const minf_bf16 *q, const minf_bf16 *k, int hq, int hkv, int n, int d,
                     int last_q, int n_vertical, int n_slash, float scale,
                     const int32_t *head_ids, int n_heads, int32_t *v_idx, int32_t *s_idx,
                     void *ws, size_t ws_bytes, minf_stream_t stream);

/*
 * Vertical-Slash index estimation with top-p budgets ([TALK], the part on the
 * work that followed MInference: a top-p of the attention weights instead of a
 * fixed top-k).  The scores are those of minf_vs_estimate.  Verticals: the
 * fewest keys, best first (ties to the lower index), whose column sums reach
 * p_vertical of the total column mass.  Slashes: offset 0 (forced, its own
 * diagonal mass counted), then the fewest further offsets, best first, until
 * the diagonal mass reaches p_slash of the total.  n_vertical and n_slash are
 * caps: they size the rows (ASCENDING, -1 padded, as minf_vs_estimate) and
 * bound the counts.  v_cnt, s_cnt (device int32 [n_heads], nullable) receive
 * the counts.  0 < p <= 1; n <= 2^20 (masses are summed exactly in 2^-32
 * fixed point).  Workspace: MINF_OP_VS_ESTIMATE.
 */
int minf_vs_estimate_topp(const minf_bf16 *q, const minf_bf16 *k, int hq, int hkv, int n, int d,
                          int last_q, int n_vertical, int n_slash, float p_vertical, float p_slash,
                          float scale, const int32_t *head_ids, int n_heads, int32_t *v_idx,
                          int32_t *s_idx, int32_t *v_cnt, int32_t *s_cnt, void *ws,
                          size_t ws_bytes, minf_stream_t stream);

/*
 * Vertical-Slash sparse attention.  Query i of head position p attends to
 * key k iff k <= i and (k is in v_idx[p] or i - k is in s_idx[p]); each such
 * key once.  Entries < 0 in the index rows are ignored; rows need not be
 * sorted.  Slash lines are computed as contiguous key ranges per 128-query
 * tile ([NEWS] Figure 4: slashes as dense blocks), verticals outside those
 * ranges are gathered by index ([NEWS] Figure 4: verticals as 1x64 pieces).
 */
int minf_vs_attention(const minf_bf16 *q, const minf_bf16 *k, const minf_bf16 *v, int hq, int hkv,
                      int n, int d, float scale, const int32_t *head_ids, int n_heads,
                      const int32_t *v_idx, int n_vertical, const int32_t *s_idx, int n_slash,
                      minf_bf16 *out, float *lse, void *ws, size_t ws_bytes,
                      minf_stream_t stream);

/*
 * Vertical-Slash sparse attention with whole slash tiles ([NEWS] Figure 4:
 * slashes are computed as dense blocks).  Query i, in the 128-query tile that
 * starts at r0 = i - i % 128, attends to key k iff k <= i and (k is in
 * v_idx[p], or r0 - o <= k <= r0 + 127 - o for some offset o in s_idx[p]):
 * every key a selected offset reaches from some row of the tile is attended by
 * all its rows.  A superset of minf_vs_attention's key set, with no element
 * mask inside the slash ranges.  Arguments, layouts, workspace
 * (MINF_OP_VS_ATTENTION) and errors as minf_vs_attention.
 */
int minf_vs_attention_tiles(const minf_bf16 *q, const minf_bf16 *k, const minf_bf16 *v, int hq,
                            int hkv, int n, int d, float scale, const int32_t *head_ids,
                            int n_heads, const int32_t *v_idx, int n_vertical,
                            const int32_t *s_idx, int n_slash, minf_bf16 *out, float *lse,
                            void *ws, size_t ws_bytes, minf_stream_t stream);

/*
 * Block-Sparse index estimation ([NEWS] 方法介绍).  Q and K are mean-pooled
 * over blocks of `block` (= 64) tokens in fp32; for query block i the pooled
 * score of key block j <= i is Qp_i . Kp_j.  The diagonal block i is always
 * kept; the best topk-1 blocks j < i join it (ties to the lower j).  Output,
 * ASCENDING, -1 padded:
 *   blk_idx int32 [n_heads][n/64][topk], blk_cnt int32 [n_heads][n/64].
 * The scores are computed on the tensor cores from three bf16 parts of each
 * pooled fp32 value (the part products down to 2^-16 relative size, fp32
 * accumulation): their error stays below that of an fp32 dot product.  A
 * bounded wait that gives up records MINF_ERR_TIMEOUT in the workspace's
 * status block (minf_status).
 */
int minf_block_estimate(const minf_bf16 *q, const minf_bf16 *k, int hq, int hkv, int n, int d,
                        int block, int topk, const int32_t *head_ids, int n_heads,
                        int32_t *blk_idx, int32_t *blk_cnt, void *ws, size_t ws_bytes,
                        minf_stream_t stream);

/*
 * The pooled block scores behind minf_block_estimate, for inspection and for
 * callers with their own selection ([NEWS] 方法介绍: the pooled product
 * estimates the block means of the attention logits).  Writes, for each
 * listed head p, query block i and key block j <= i,
 *   scores[p][i][j] = Qp_i . Kp_j          (fp32, device, [n_heads][n/64][n/64])
 * with the same arithmetic as minf_block_estimate; entries j > i are
 * unspecified (some are written).  The caller owns `scores`; workspace as
 * MINF_OP_BLOCK_ESTIMATE (its score rows stay unused).  Errors as
 * minf_block_estimate; a null `scores` is MINF_ERR_INVALID.
 */
int minf_block_scores(const minf_bf16 *q, const minf_bf16 *k, int hq, int hkv, int n, int d,
                      int block, const int32_t *head_ids, int n_heads, float *scores, void *ws,
                      size_t ws_bytes, minf_stream_t stream);

/*
 * Block-Sparse attention: query i of head position p attends to key k iff
 * k <= i and k / 64 is among blk_idx[p][i / 64][0 .. blk_cnt[p][i / 64]).
 * Each row of blk_idx must be ascending with distinct entries (as
 * minf_block_estimate writes it); negative entries are ignored.
 */
int minf_block_attention(const minf_bf16 *q, const minf_bf16 *k, const minf_bf16 *v, int hq,
                         int hkv, int n, int d, float scale, const int32_t *head_ids,
                         int n_heads, const int32_t *blk_idx, const int32_t *blk_cnt, int topk,
                         minf_bf16 *out, float *lse, void *ws, size_t ws_bytes,
                         minf_stream_t stream);

/*
 * A-shape attention ([TALK] second observation): query i attends to key k iff
 * k <= i and (k < n_sink or i - k < window).  The window counts the query
 * itself.  n_sink >= 0, window >= 1.
 */
int minf_ashape_attention(const minf_bf16 *q, const minf_bf16 *k, const minf_bf16 *v, int hq,
                          int hkv, int n, int d, float scale, const int32_t *head_ids,
                          int n_heads, int n_sink, int window, minf_bf16 *out, float *lse,
                          void *ws, size_t ws_bytes, minf_stream_t stream);

/*
 * Tri-shape attention ([TALK], SCBench part: named as an A-shape variant that
 * improves first-turn instruction following; the pages give no definition).
 * This library's reading: the A-shape mask plus dense rows for the last n_last
 * queries -- query i attends to key k iff k <= i and (k < n_sink or
 * i - k < window or i >= n - n_last).  n_last = 0 is A-shape, n_last >= n is
 * dense causal attention.
 */
int minf_trishape_attention(const minf_bf16 *q, const minf_bf16 *k, const minf_bf16 *v, int hq,
                            int hkv, int n, int d, float scale, const int32_t *head_ids,
                            int n_heads, int n_sink, int window, int n_last, minf_bf16 *out,
                            float *lse, void *ws, size_t ws_bytes, minf_stream_t stream);

/* Dense causal attention (the comparison baseline): query i attends to k <= i. */
int minf_dense_attention(const minf_bf16 *q, const minf_bf16 *k, const minf_bf16 *v, int hq,
                         int hkv, int n, int d, float scale, const int32_t *head_ids,
                         int n_heads, minf_bf16 *out, float *lse, void *ws, size_t ws_bytes,
                         minf_stream_t stream);

/*
 * One attention layer with a per-head pattern ([TALK] offline/online split:
 * each head has its own pattern; the online part estimates and attends).
 * head_pattern is a HOST array of hq MINF_PATTERN_* codes.  VS heads run
 * minf_vs_estimate + minf_vs_attention (last_q, n_vertical, n_slash), BLOCK
 * heads minf_block_estimate + minf_block_attention (64, topk), ASHAPE heads
 * minf_ashape_attention (n_sink, window), TRISHAPE heads
 * minf_trishape_attention (n_sink, window, n_last = last_q), DENSE heads
 * minf_dense_attention.
 * out [hq][n][128] bf16, lse [hq][n] fp32 (nullable).  The indices are kept in
 * the workspace.  VS, ASHAPE and TRISHAPE heads run on `stream`; BLOCK and
 * DENSE heads run on a library side stream that starts after the work already
 * queued on `stream`, so each group's estimate overlaps the other group's
 * attention; `stream` waits for the side stream before anything queued after
 * this call, so to the caller the whole layer is ordered on `stream`.
 */
int minf_mixed_layer(const minf_bf16 *q, const minf_bf16 *k, const minf_bf16 *v, int hq, int hkv,
                     int n, int d, float scale, const int8_t *head_pattern, int last_q,
                     int n_vertical, int n_slash, int topk, int n_sink, int window,
                     minf_bf16 *out, float *lse, void *ws, size_t ws_bytes,
                     minf_stream_t stream);

/*
 * Synchronises `stream`, then returns the device-side status word of the
 * workspace: MINF_OK, or MINF_ERR_TIMEOUT if a bounded wait in a kernel gave up
 * (that kernel then left its outputs incomplete).  Reading it resets it to
 * MINF_OK.  Returns MINF_ERR_CUDA if the synchronisation itself failed.
 */
int minf_status(void *ws, minf_stream_t stream);

/*
 * Synchronises `stream` and returns the work counters the last attention call
 * on `ws` accumulated: tiles = 128x128 query-key tiles computed on the tensor
 * cores, pairs = (query, key) pairs inside the mask (the useful work).
 */
int minf_stats(void *ws, minf_stream_t stream, uint64_t *tiles, uint64_t *pairs);

/*
 * The same counters split by kernel (no counterpart in the method's sources):
 * writes min(n_out, 7) values to the host array out -- tiles, pairs, then the
 * tiles of the dense, Vertical-Slash, Block-Sparse and A-shape (Tri-shape
 * included) attention kernels, then the pairs computed by the CUDA-core
 * sparse-slash pass (part of pairs) -- and returns how many it wrote.
 */
int minf_stats_detail(void *ws, minf_stream_t stream, uint64_t *out, int n_out);

/*
 * Sets the limit, in nanoseconds, after which a device-side wait gives up and
 * records MINF_ERR_TIMEOUT (default 2e9 ns; 0 restores the default).  Applies
 * to launches made after the call, process-wide.
 */
void minf_set_wait_limit_ns(uint64_t ns);

/*
 * Routing of Vertical-Slash slash groups (a tuning knob; the method's sources
 * compute every slash as dense blocks, [NEWS] Figure 4).  Offsets at most 128
 * apart form a group whose key range a 128-row query tile computes as H
 * half-tiles of 64 keys on the tensor cores, masked per element.  A group of m
 * offsets goes instead to a CUDA-core pass that computes only the m in-mask
 * pairs of each query row (one dot product, one exponential and one V update
 * per offset) when m < ratio * H.  The result is the same token-exact masked
 * softmax either way (the two partial states are merged per row); only the
 * time differs.  ratio <= 0 sends every group to the tensor cores.  Default
 * 1.0 (on B200 a lone offset costs the CUDA-core pass about as much as two
 * thirds of a 128x128 tensor-core tile, a triple about as much as its four
 * half-tiles); applies to minf_vs_attention and the mixed layer (not to
 * minf_vs_attention_tiles), process-wide, for calls made after it.
 */
void minf_set_vs_diag_ratio(float ratio);

/*
 * Failure-detection self-test: launches one kernel whose wait nothing will
 * ever satisfy, so it must give up after `limit_ns` and record
 * MINF_ERR_TIMEOUT in the workspace status word (read with minf_status).
 * Needs MINF_STATUS_BYTES of workspace.
 */
int minf_check_wait_timeout(void *ws, size_t ws_bytes, uint64_t limit_ns, minf_stream_t stream);

#define MINF_STATUS_BYTES 256

/*
 * Self-test of the exponentials inside the attention kernels (no counterpart
 * in the method's sources): for n fp32 inputs x (device), writes 2^x from the
 * FMA-pipe polynomial the softmax uses for a share of its columns (Cody-Waite
 * reduction to [-1/2, 1/2] plus a degree-3 minimax polynomial; 0 for
 * x <= -127) to y_poly, and from the hardware ex2.approx to y_hw.
 */
int minf_selftest_exp2(const float *x, float *y_poly, float *y_hw, int n, minf_stream_t stream);

/*
 * minf_vs_estimate without a workspace argument (no counterpart in the
 * method's sources: it exists for callers that cannot allocate device memory,
 * such as code inside a runtime that owns all device memory, or code that
 * must not call cudaMalloc at that point).  Same arguments and results as
 * minf_vs_estimate minus ws/ws_bytes; the scratch is a 32 MiB array inside
 * the library that every GPU loading the library keeps until the process
 * exits.  Calls needing more scratch than that (as sized by
 * minf_workspace_bytes(MINF_OP_VS_ESTIMATE, ...)) return MINF_ERR_WORKSPACE.
 * The first call on a device, in a given CUDA context, looks up the array's
 * address there (a later context, or a reset one, looks it up again): make
 * that first call before any stream capture.  All calls share the array, so
 * calls that may overlap on the GPU race; order them on one stream.  Each call
 * clears the status block at the start of the array; a device-side timeout of
 * the call is read back with minf_vs_estimate_noalloc_status.
 */
int minf_vs_estimate_noalloc(const minf_bf16 *q, const minf_bf16 *k, int hq, int hkv, int n, int d,
                             int last_q, int n_vertical, int n_slash, float scale,
                             const int32_t *head_ids, int n_heads, int32_t *v_idx, int32_t *s_idx,
                             minf_stream_t stream);

/*
 * Status of the last minf_vs_estimate_noalloc on `device` (no counterpart in
 * the method's sources): makes `device` current, waits for `stream`, returns
 * MINF_OK or the device-side error the call recorded in the built-in array's
 * status block (MINF_ERR_TIMEOUT: a bounded wait ran out and the returned
 * indices are not valid; minf_last_error() names where), and clears it.  Like
 * minf_status for the workspace calls.  MINF_ERR_INVALID for a device ordinal
 * out of range.
 */
int minf_vs_estimate_noalloc_status(int device, minf_stream_t stream);

/*
 * Self-test of that read-back (no counterpart in the method's sources): on
 * `device`, launches one bounded wait that nothing satisfies, which gives up
 * after limit_ns and records MINF_ERR_TIMEOUT in the built-in array's status
 * block, as a timed-out estimate would.  Asynchronous on `stream`.
 */
int minf_vs_estimate_noalloc_check_timeout(int device, uint64_t limit_ns, minf_stream_t stream);

/*
 * Launch timing (no counterpart in the method's sources; for measuring this
 * library): while enabled (on != 0), every attention, estimate and plan launch
 * sequence of the library is bracketed by two CUDA events on the stream it
 * runs on.  minf_profile_read waits for the recorded events, writes one line
 * per kernel name -- "name<TAB>launches<TAB>total milliseconds" -- into the
 * host buffer buf (at most len bytes, NUL-terminated), clears the records and
 * returns the length of the full text (larger than len - 1 if it was cut).
 * With buf NULL it only returns that length and keeps the records.
 * Do not read while calls of the library are being made on other threads.
 */
void minf_profile_enable(int on);
int minf_profile_read(char *buf, size_t len);

/* Library version string and the message of the last host-side error. */
const char *minf_version(void);
const char *minf_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* MINF_H */
