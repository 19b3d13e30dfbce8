/*
 * hga.h - C ABI of the HGA routed-attention library (libhga.so, sm_100a).
 *
 * Hierarchical Global Attention (HGA), exact-token two-level routed causal
 * attention for one layer's projected, RoPE-applied Q/K/V, as described on the
 * page "Long-Context Fine-Tuning with Limited VRAM", section 2.1 ("Exact-token
 * hierarchical routing"):
 *   1. a summary for every closed 64-token chunk and every 8-token group of
 *      the keys                                      -> hga_build_summaries
 *   2. each 64-query block scores the chunk summaries and keeps the best
 *      chunks, besides fixed sink and local windows  -> hga_route_chunks
 *   3. the kept chunks are opened and the best 8-token groups inside them are
 *      kept                                          -> hga_route_groups
 *   4. softmax attention over the exact token K/V of the kept groups, the
 *      sink, the local window and the causal diagonal -> hga_attend
 * Section 6.1 of the same page notes that one routing decision serves every
 * query of a block: routing is per (query block, KV head).
 *
 * Readings this library fixes where the pages are silent:
 *   - summary = mean of the post-RoPE keys, accumulated exactly (float64) and
 *     rounded once, to nearest even, to the storage dtype;
 *   - block score of a summary s = max over the block's queries and the query
 *     heads sharing the KV head of q.s/sqrt(d) (ranking uses q.s);
 *   - candidate chunks of the block at b0: sink/chunk <= c < (b0-local)/chunk;
 *   - local window = tokens [b0-local, b0) plus the block's causal diagonal;
 *     sink = tokens [0, sink);
 *   - top-k keeps the first min(k, n) candidates by (score desc, index asc);
 *     k <= 0 keeps all; the group budget is global over the kept chunks.
 *
 * Layouts (all row-major, element type = params.dtype):
 *   q, o        [n_q][n_q_heads][head_dim]          query i is position q_start+i
 *   k, v        [n_kv_heads][t_cap][head_dim]       token t of head h at (h*t_cap+t)*d
 *               (v in fp16 when params.v_f16 = 1)
 *   chunk_sum   [n_kv_heads][t_cap/chunk][head_dim]
 *   group_sum   [n_kv_heads][t_cap/group][head_dim]
 *   chunk_idx   [n_kv_heads][n_blocks][cap_c]  int32, cap_c = hga_index_capacity(p,t_cap,0)
 *   chunk_cnt   [n_kv_heads][n_blocks]         int32
 *   group_idx   [n_kv_heads][n_blocks][cap_g]  int32, cap_g = hga_index_capacity(p,t_cap,1)
 *   group_cnt   [n_kv_heads][n_blocks]         int32
 *   lse         [n_q][n_q_heads] float32 (natural log), optional
 * with n_blocks = ceil(n_q / qblock).  The context of a call is T = q_start + n_q
 * tokens; queries attend only to tokens < T (causal).
 *
 * Ownership: the caller owns every buffer (device memory unless stated); the
 * library never allocates or frees and keeps no per-call state.  Inputs are
 * read-only.  Index outputs are fully overwritten: unused slots become -1 and
 * lists are in ascending order.  Summary outputs are written only for the
 * chunks/groups the call covers.
 *
 * Errors: every call is asynchronous on `stream`.  Argument errors are
 * detected on the host and returned before anything is launched.  Launch
 * failures return HGA_ERR_CUDA.  Errors found by a kernel (an index list entry
 * outside the legal range, for example) are recorded in a device status word
 * and returned by hga_check(); kernels never trap.
 *
 * Supported: dtype bf16 (tensor-core path) or fp32 (exact FFMA path);
 * head_dim 64 or 128; chunk 64, group 8, qblock 64; sink and local multiples
 * of chunk; n_q_heads a multiple of n_kv_heads.
 */
#ifndef HGA_H
#define HGA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* hga_stream_t;   /* same object as cudaStream_t */

typedef enum {
  HGA_OK = 0,
  HGA_ERR_INVALID_ARG = 1,   /* bad pointer, size, alignment or parameter      */
  HGA_ERR_UNSUPPORTED = 2,   /* legal but not built: dtype, head_dim, sizes     */
  HGA_ERR_CUDA = 3,          /* a CUDA runtime call or launch failed            */
  HGA_ERR_DEVICE_CHECK = 4,  /* a kernel found an out-of-range index (hga_check)*/
  HGA_ERR_TIMEOUT = 5,       /* a bounded device wait gave up (hga_check)       */
  HGA_ERR_IO = 6,            /* a file open, read or write failed (K/V store)   */
  HGA_ERR_CAPACITY = 7       /* the store's page cache cannot hold one step     */
} hga_status;

typedef enum { HGA_BF16 = 0, HGA_FP32 = 1 } hga_dtype;

typedef struct hga_params {
  int32_t n_q_heads;    /* query heads; a multiple of n_kv_heads              */
  int32_t n_kv_heads;   /* key/value heads (GQA)                              */
  int32_t head_dim;     /* 64 or 128                                          */
  int32_t chunk;        /* chunk size in tokens (64)                          */
  int32_t group;        /* group size in tokens (8)                           */
  int32_t qblock;       /* query block size (64)                              */
  int32_t sink;         /* sink window, tokens [0, sink); multiple of chunk   */
  int32_t local;        /* local window before each block; multiple of chunk  */
  int32_t top_chunks;   /* chunk budget per (block, KV head); <= 0 = all       */
  int32_t top_groups;   /* group budget per (block, KV head); <= 0 = all       */
  int32_t dtype;        /* hga_dtype of q, k, v, o and the summaries          */
  int32_t v_f16;        /* 0: v in dtype.  1: v holds IEEE fp16 values, the  */
                        /* type of the attention kernels' P.V operand (fp16  */
                        /* P, 11 significant bits), so they read V as is     */
                        /* instead of converting each tile; dtype must be    */
                        /* HGA_BF16.  hga_convert_v fills such a buffer.     */
  int32_t q_ready;      /* 0 or 1.  Every kernel of this library is launched */
                        /* with programmatic dependent launch: it may start  */
                        /* while the kernel before it in the stream is still */
                        /* running, and waits for that kernel before reading */
                        /* its inputs.  1 promises that q is complete before */
                        /* that kernel can let its dependents start (kernels */
                        /* that never do so early, such as PyTorch's, and    */
                        /* this library's own kernels qualify); the          */
                        /* tensor-core routing and attention kernels then    */
                        /* request q before the wait, overlapping its load   */
                        /* with the previous kernel's tail.  0: q is read    */
                        /* after the wait.  hga_forward, hga_forward_causal  */
                        /* and hga_decode_step use 1 for their own calls     */
                        /* that follow one of their kernels.                 */
} hga_params;

/* Step 1 (section 2.1, "HGA builds two levels of key summaries from the
 * model's existing projected keys").  For every KV head h writes
 *   chunk_sum[h][c] = mean(k[h][c*chunk .. c*chunk+chunk-1])
 * for each chunk c with t_begin <= c*chunk and (c+1)*chunk <= t_end, and
 *   group_sum[h][j] = mean(k[h][j*group .. j*group+group-1])
 * for each group j with t_begin <= j*group and (j+1)*group <= t_end.
 * The mean is exact before a single round-to-nearest-even to the dtype.
 * Requires t_begin % chunk == 0 and 0 <= t_begin <= t_end <= t_cap. */
hga_status hga_build_summaries(const hga_params* p, const void* k,
                               int64_t t_cap, int64_t t_begin, int64_t t_end,
                               void* chunk_sum, void* group_sum,
                               hga_stream_t stream);

/* Commit of the tokens [t_begin, t_end) in one launch: the summaries of
 * hga_build_summaries (same arguments, same results) and, when v_f16 is not
 * NULL, the fp16 copy of V that hga_convert_v writes (v: [Hkv][t_cap][D]
 * bf16, v_f16: same layout, fp16; every token in [t_begin, t_end), including
 * a trailing partial chunk).  With v_f16 == NULL it is hga_build_summaries.
 * The pages have no counterpart; they keep summaries of the projected keys
 * (section 2.1), and storing V in the attention's operand type when a token
 * enters the cache is this library's choice.  Requires dtype HGA_BF16 when
 * v_f16 is given, 16-byte aligned v and v_f16, and v_f16 either equal to v
 * (in place) or not overlapping it.  A |v| above 65504 becomes inf and sets
 * HGA_ERR_DEVICE_CHECK (hga_check). */
hga_status hga_commit(const hga_params* p, const void* k, const void* v,
                      int64_t t_cap, int64_t t_begin, int64_t t_end,
                      void* chunk_sum, void* group_sum, void* v_f16,
                      hga_stream_t stream);

/* Step 2 (section 2.1, "Chunk selection").  For each query block b (queries
 * q_start + b*qblock ...) and KV head h: scores every candidate chunk
 * (sink/chunk <= c < (b0-local)/chunk) by the max over the block's rows of
 * q.chunk_sum[h][c], keeps min(top_chunks, n) by (score desc, index asc) and
 * writes them ascending to chunk_idx[h][b][:], the count to chunk_cnt[h][b].
 * chunk_sum must hold every candidate (built with t_end >= q_start).
 * Requires q_start % qblock == 0 and q_start + n_q <= t_cap. */
hga_status hga_route_chunks(const hga_params* p, const void* q,
                            int64_t q_start, int64_t n_q,
                            const void* chunk_sum, int64_t t_cap,
                            int32_t* chunk_idx, int32_t* chunk_cnt,
                            hga_stream_t stream);

/* Step 3 (section 2.1, "Group selection").  Candidates of (b, h) are the
 * chunk/group groups of every chunk in chunk_idx[h][b][0 .. chunk_cnt-1];
 * scored as in step 2 against group_sum; keeps min(top_groups, n) and writes
 * them ascending to group_idx[h][b][:], the count to group_cnt[h][b].
 * chunk_idx/chunk_cnt are the outputs of hga_route_chunks for the same
 * q_start/n_q/t_cap.  An out-of-range chunk index sets HGA_ERR_DEVICE_CHECK
 * (read by hga_check) and is skipped. */
hga_status hga_route_groups(const hga_params* p, const void* q,
                            int64_t q_start, int64_t n_q,
                            const void* group_sum, int64_t t_cap,
                            const int32_t* chunk_idx, const int32_t* chunk_cnt,
                            int32_t* group_idx, int32_t* group_cnt,
                            hga_stream_t stream);

/* Steps 2 and 3 in one call: the same chunk_idx/chunk_cnt and group_idx/
 * group_cnt as hga_route_chunks followed by hga_route_groups (bit for bit).
 * On the tensor-core path one CTA per (query block, KV head) runs both: the
 * block's rows are staged once and the kept chunks go straight from the
 * chunk selection into the group scoring.  Otherwise the two calls above are
 * made in order.  One launch instead of two; on the 64K-context workload the
 * fused kernel is faster alone but, inside a full step, the two launches
 * finish sooner (hga_forward uses them).  Arguments, capacities and errors
 * as for those two calls;
 * chunk_sum must hold every candidate chunk and group_sum every group of the
 * candidate chunks. */
hga_status hga_route(const hga_params* p, const void* q, int64_t q_start, int64_t n_q,
                     const void* chunk_sum, const void* group_sum, int64_t t_cap,
                     int32_t* chunk_idx, int32_t* chunk_cnt, int32_t* group_idx,
                     int32_t* group_cnt, hga_stream_t stream);

/* Step 4 (section 2.1, "Exact-token attention": only exact token K/V, never
 * summaries).  Query at position pos (block start b0, query head hq, KV head
 * h = hq / (n_q_heads/n_kv_heads)) attends the set
 *   [0, min(sink, pos+1))  U  tokens of group_idx[h][b][0..group_cnt-1]
 *   U  [max(0, b0-local), b0)  U  [b0, pos]
 * with softmax(q.k/sqrt(d)) and writes o (dtype) and, when lse != NULL, the
 * natural-log sum of exponentials of the scaled scores.  Group indices outside
 * the legal range set HGA_ERR_DEVICE_CHECK and are skipped. */
hga_status hga_attend(const hga_params* p, const void* q, int64_t q_start,
                      int64_t n_q, const void* k, const void* v, int64_t t_cap,
                      const int32_t* group_idx, const int32_t* group_cnt,
                      void* o, float* lse, hga_stream_t stream);

/* Backward of step 4: gradients of the gathered attention with the routing
 * held fixed.  The kept groups (group_idx/group_cnt, as used by the forward
 * pass) are inputs: the selection is piecewise constant, so gradients reach
 * q, k and v only through the exact-token attention of section 2.1.  For a
 * query row with attended set R (the same set as hga_attend):
 *   s_j = q.k_j/sqrt(d), p_j = exp(s_j - lse), dp_j = dO.v_j, D = dO.o,
 *   ds_j = p_j (dp_j - D); dq = sum_j ds_j k_j/sqrt(d),
 *   dk_j += ds_j q/sqrt(d), dv_j += p_j dO.
 * o and lse are the forward's outputs (lse natural log, as hga_attend writes
 * it); d_o has o's layout and dtype.  Outputs are fp32: d_q [n_q][Hq][d] is
 * fully written; d_k and d_v [Hkv][t_cap][d] are zeroed on every head's tokens
 * [0, T) and then accumulated (tokens past T are not touched).  The pages do
 * not describe a backward; training through the routed attention is how the
 * paper uses it (section 2.2).  Requires params.v_f16 = 0 (v in dtype),
 * 16-byte aligned d_q, d_k, d_v; same segment rules as hga_attend.  First
 * version: fp32 arithmetic on the CUDA cores, atomic adds for d_k and d_v (so
 * their low bits depend on the order of the adds). */
hga_status hga_attend_backward(const hga_params* p, const void* q, int64_t q_start,
                               int64_t n_q, const void* k, const void* v, int64_t t_cap,
                               const int32_t* group_idx, const int32_t* group_cnt,
                               const void* o, const float* lse, const void* d_o,
                               float* d_q, float* d_k, float* d_v, hga_stream_t stream);

/* Writes v_f16[h][t] = fp16(v[h][t]) for every KV head h and token
 * t_begin <= t < t_end (all head_dim values; same [n_kv_heads][t_cap]
 * [head_dim] layout), for use with params.v_f16 = 1.  Not a step of the
 * method: it fixes the storage type of V once per token, when the token is
 * committed, so that the attention kernels need no per-tile conversion.
 * bf16 -> fp16 rounds to nearest even; it is exact for 2^-14 <= |v| < 65504
 * and off by at most 2^-25 below.  A |v| above 65504 (inf included)
 * becomes inf and sets HGA_ERR_DEVICE_CHECK (read by hga_check).  dtype must
 * be HGA_BF16 (v_f16 in the params is ignored here); v_f16 may equal v (in
 * place) but must not otherwise overlap it; 0 <= t_begin <= t_end <= t_cap. */
hga_status hga_convert_v(const hga_params* p, const void* v, int64_t t_cap,
                         int64_t t_begin, int64_t t_end, void* v_f16,
                         hga_stream_t stream);

/* Steps 1-4 in one call for a query segment whose own K/V already sit in
 * k/v at [q_start, q_start+n_q): builds the summaries of the segment's
 * closed chunks/groups, then routes and attends.  Index buffers as above. */
hga_status hga_forward(const hga_params* p, const void* q, int64_t q_start,
                       int64_t n_q, const void* k, const void* v,
                       int64_t t_cap, void* chunk_sum, void* group_sum,
                       int32_t* chunk_idx, int32_t* chunk_cnt,
                       int32_t* group_idx, int32_t* group_cnt, void* o,
                       float* lse, hga_stream_t stream);

/* One generation step of one request (the decode form of the same
 * method).  The token at position pos has its K/V in the cache and
 * its query in row pos - b0 of q_block, which holds the queries of its query
 * block so far (positions b0 .. pos, b0 = pos - pos % qblock; layout of q).
 * The step commits the token (hga_commit of [b0, pos + 1): summaries of its
 * group and chunk once closed, and its V in fp16 into v_f16 when v_f16 is not
 * NULL), routes the block on the queries present and attends: one routing
 * decision per block, as in prefill (section 6.1 of the page), so the result
 * equals hga_forward of the segment [b0, pos + 1).  The token's output is row
 * pos - b0 of o ([n][Hq][d], n = pos - b0 + 1), and its LSE row pos - b0 of
 * lse; the attention computes only the token's rows (bit for bit the rows
 * hga_forward would give them), so the block's earlier rows of o and lse are
 * left as they are.  chunk_idx .. group_cnt are sized for one
 * block; chunk_sum/group_sum hold the committed history.  params.v_f16 must be
 * 0 (v in dtype); v_f16 must not alias v.  Composed of the calls above; the
 * pages describe generation only in prose (section 2.2). */
hga_status hga_decode_step(const hga_params* p, const void* q_block, int64_t pos,
                           const void* k, const void* v, int64_t t_cap,
                           void* chunk_sum, void* group_sum, int32_t* chunk_idx,
                           int32_t* chunk_cnt, int32_t* group_idx, int32_t* group_cnt,
                           void* v_f16, void* o, float* lse, hga_stream_t stream);

/* Strictly causal routing variant ("Long-Context Fine-Tuning with Limited
 * VRAM", section 6.1: sharing one routing decision across a block lets an
 * earlier token learn about later ones; a strictly causal variant is named
 * and its design left to future work).  This library's reading: block b is
 * routed on the queries of the block before it, as many rows as b has
 * (positions b0 - qblock .. b0 - qblock + n_b - 1), which all precede the
 * block's first token, so no output depends on a later input.  Same cost as
 * hga_forward.
 *   q_ext: [qblock + n_q][n_q_heads][head_dim]; rows 0..qblock-1 are the
 *          queries at positions q_start - qblock .. q_start - 1 (any finite
 *          values when q_start == 0: the first block of a sequence has no
 *          candidates), rows qblock.. the segment's queries.
 * Other arguments, layouts and errors as hga_forward.  The result equals
 * hga_route_chunks + hga_route_groups called with q = q_ext (routing) and
 * hga_attend with q = q_ext + qblock rows, after the segment's summaries. */
hga_status hga_forward_causal(const hga_params* p, const void* q_ext, int64_t q_start,
                              int64_t n_q, const void* k, const void* v, int64_t t_cap,
                              void* chunk_sum, void* group_sum, int32_t* chunk_idx,
                              int32_t* chunk_cnt, int32_t* group_idx, int32_t* group_cnt, void* o,
                              float* lse, hga_stream_t stream);

/* ---------------------------------------------------------------------------
 * Host-memory tier ("Long-Context Fine-Tuning with Limited VRAM", section 2.2
 * tiered KV storage; section 2.1 group summaries in a VRAM cache with misses
 * fetched from RAM; section 4.5 cache hit rate).  History = tokens < t_hist
 * (a multiple of group, <= q_start).  Its K/V and all group summaries live in
 * pinned host memory (readable by the device: page-locked, unified
 * addressing), [n_kv_heads][t_cap][head_dim] and [n_kv_heads][t_cap/group]
 * [head_dim].  Device "mirrors" with the all-HBM layouts receive what a step
 * needs, so hga_route_groups and hga_attend run on them unchanged:
 *   route chunks -> hga_fetch_group_summaries -> hga_route_groups
 *   -> hga_gather_history (may run on a side stream; hga_attend waits)
 *   -> hga_attend -> hga_install_group_cache.
 * Results equal the all-HBM path's exactly. */
typedef struct hga_group_cache {
  void* data;                  /* device [n_kv_heads][cap][head_dim], dtype       */
  int32_t* tags;               /* device [n_kv_heads][cap]: group held, -1 empty  */
  int32_t* claims;             /* device [n_kv_heads][cap]: largest group that    */
                               /*   missed on the slot this step, -1 none         */
  int64_t cap;                 /* slots per KV head; group j maps to j % cap      */
  unsigned long long* stats;   /* device [2] hits, misses (accumulated), nullable */
} hga_group_cache;

/* Group summaries of every kept history chunk of every (block, KV head) are
 * copied into group_sum_dev: from the cache on a hit, from group_sum_host on
 * a miss (the slot is then claimed).  tags/claims start at -1 (caller). */
hga_status hga_fetch_group_summaries(const hga_params* p, int64_t q_start, int64_t n_q,
                                     int64_t t_cap, int64_t t_hist, const int32_t* chunk_idx,
                                     const int32_t* chunk_cnt, const void* group_sum_host,
                                     const hga_group_cache* cache, void* group_sum_dev,
                                     hga_stream_t stream);

/* Copies the history K/V groups the step attends (sink, routed, local window,
 * below t_hist) from k_host/v_host into k_dev/v_dev, each (KV head, group) at
 * most once per step: gen ([n_kv_heads][t_cap/group] uint32, zero at first
 * use) is stamped with `step` (nonzero, distinct per call).  Adds the bytes
 * copied to *bytes when bytes != NULL. */
hga_status hga_gather_history(const hga_params* p, int64_t q_start, int64_t n_q, int64_t t_cap,
                              int64_t t_hist, const int32_t* group_idx, const int32_t* group_cnt,
                              const void* k_host, const void* v_host, void* k_dev, void* v_dev,
                              uint32_t* gen, uint32_t step, unsigned long long* bytes,
                              hga_stream_t stream);

/* Every claimed cache slot takes its claim (summary copied from
 * group_sum_host, tag set, claim cleared).  Run after the step's lookups. */
hga_status hga_install_group_cache(const hga_params* p, int64_t t_cap,
                                   const void* group_sum_host, const hga_group_cache* cache,
                                   hga_stream_t stream);

/* hga_gather_history without the caller's generation array.  The pages have
 * no counterpart: this call exists for callers that cannot allocate device
 * memory for the stamps, e.g. a runtime that sizes all device memory once at
 * start-up, or a host with no CUDA allocator of its own.
 * - Result: the same copies, in the same places, as one hga_gather_history
 *   call with a zeroed gen array; *bytes (when not NULL) grows by the same
 *   amount.
 * - Storage: the stamps live in a fixed 1 MiB array in the library's device
 *   memory. n_kv_heads * (t_cap / group) must be at most 262144, otherwise
 *   HGA_ERR_UNSUPPORTED is returned before any launch. Every call first zeroes
 *   the part it uses, so no state carries over between calls.
 * - Allocation: none. No cudaMalloc or cudaFree, and no allocating library
 *   call.
 * - First call on a device: it looks up the array's device address once, with
 *   that device current. That call must not be made while `stream` is being
 *   captured; if it is, the call returns HGA_ERR_UNSUPPORTED and launches
 *   nothing. Make the first call outside any capture.
 * - Concurrency: one array per device. Calls whose executions overlap on one
 *   device (other streams, other host threads) race on it and may skip or
 *   repeat copies. Order them on one stream, or with events.
 * - Other arguments and errors: as hga_gather_history. */
hga_status hga_gather_history_noalloc(const hga_params* p, int64_t q_start, int64_t n_q,
                                      int64_t t_cap, int64_t t_hist, const int32_t* group_idx,
                                      const int32_t* group_cnt, const void* k_host,
                                      const void* v_host, void* k_dev, void* v_dev,
                                      unsigned long long* bytes, hga_stream_t stream);

/* ---------------------------------------------------------------------------
 * File-backed K/V store ("Long-Context Fine-Tuning with Limited VRAM",
 * section 2.2: besides RAM-backed history the method has a filesystem store
 * in which RAM is a bounded page cache over disk, suited to NVMe; section 6.2
 * notes it was not benchmarked there).  The history's exact K/V lives in one
 * file; a step's routed, sink and local-window history groups are read into a
 * bounded page cache in pinned host memory, from which a kernel gathers them
 * into the device mirrors (as hga_gather_history does from whole-history
 * RAM).  Group summaries keep using the RAM tier above.
 *
 * File layout: pages of page_tokens tokens of one KV head; page (h, n) holds
 * K then V, each [page_tokens][head_dim] in the store's dtype, at byte offset
 * (h * n_pages + n) * page_bytes, page_bytes = 2 * page_tokens * head_dim *
 * elem_size, n_pages = ceil(t_cap / page_tokens).  Tokens never appended read
 * as zeros.  Cache slot i occupies cache[i * page_bytes ..) with the page's
 * file image.  page_table[h * n_pages + n] = the slot holding page (h, n), or
 * -1; it is written only by the store.
 *
 * Step:  route chunks -> hga_fetch_group_summaries -> hga_route_groups ->
 *        copy group_idx/group_cnt to the host, synchronise ->
 *        hga_store_prepare (misses read from the file, least recently used
 *        pages evicted) -> hga_gather_store -> hga_attend.
 * Results equal the all-HBM path's exactly.
 *
 * Threading: a store is not thread-safe; calls on one store are serial.
 * hga_store_prepare and hga_store_append rewrite cache slots and page_table:
 * the caller makes sure no hga_gather_store of this store is still running
 * (e.g. the synchronisation before hga_store_prepare covers the previous
 * step's gather when both run on one stream). */
typedef struct hga_kv_store hga_kv_store;

typedef struct hga_store_stats {
  int64_t pages_needed;   /* distinct (KV head, page) the step reads           */
  int64_t hits;           /* of those, already in the cache                     */
  int64_t misses;         /* read from the file                                 */
  int64_t evictions;      /* cached pages dropped to make room                  */
  int64_t bytes_read;     /* file bytes read                                    */
} hga_store_stats;

#define HGA_STORE_CREATE 1   /* create or truncate the file to its full size   */
#define HGA_STORE_DIRECT 2   /* read with O_DIRECT (bypasses the OS page cache; */
                             /* page_bytes and the cache must be 4096-aligned)  */

/* Opens the store file `path` for the layout of p (n_kv_heads, head_dim,
 * dtype) and context capacity t_cap.  page_tokens: a positive multiple of
 * p->group.  Without HGA_STORE_CREATE the file must exist and have the full
 * size; its length (tokens appended) starts at 0 and is set by
 * hga_store_append or hga_store_set_length.  *out receives the handle
 * (NULL on error).  Errors: HGA_ERR_INVALID_ARG, HGA_ERR_IO (open/truncate
 * failed, or O_DIRECT refused by the filesystem). */
hga_status hga_store_open(const char* path, const hga_params* p, int64_t t_cap,
                          int64_t page_tokens, int32_t flags, hga_kv_store** out);

/* Closes the file and frees the handle (the file stays).  NULL is a no-op. */
hga_status hga_store_close(hga_kv_store* s);

/* Gives the store its page cache: cache_pages slots of page_bytes at `cache`
 * and page_table [n_kv_heads][n_pages] int32, both caller-owned host memory
 * (pinned when a kernel reads them) that must outlive the store or the next
 * attach.  Every slot starts empty; page_table is filled with -1. */
hga_status hga_store_attach_cache(hga_kv_store* s, void* cache, int64_t cache_pages,
                                  int32_t* page_table);

/* Appends n tokens of K and V at the current length: k, v are host arrays
 * [n_kv_heads][n][head_dim] in the store's dtype.  Cached pages that the
 * tokens touch are updated too.  HGA_ERR_INVALID_ARG when length + n > t_cap. */
hga_status hga_store_append(hga_kv_store* s, const void* k, const void* v, int64_t n);

/* Declares the first `length` tokens of an existing file valid (reopening a
 * store written earlier).  0 <= length <= t_cap. */
hga_status hga_store_set_length(hga_kv_store* s, int64_t length);

/* Tokens appended (or declared), -1 for NULL. */
int64_t hga_store_length(const hga_kv_store* s);

/* Bytes of one page (K and V), -1 for NULL. */
int64_t hga_store_page_bytes(const hga_kv_store* s);

/* Pages per KV head, -1 for NULL. */
int64_t hga_store_pages_per_head(const hga_kv_store* s);

/* Reads tokens [t_begin, t_end) of K and V straight from the file into host
 * arrays [n_kv_heads][t_end - t_begin][head_dim] (the cache is not used). */
hga_status hga_store_read(hga_kv_store* s, int64_t t_begin, int64_t t_end, void* k, void* v);

/* Makes every page the step's history groups fall in resident: for each
 * (block, KV head) the sink groups, the routed groups group_idx/group_cnt
 * (HOST copies, layouts as hga_route_groups writes them for s's t_cap) and
 * the local-window groups that lie below t_hist.  Resident pages are marked
 * used; missing ones take free slots, else the least recently used slots
 * that this step does not need, and are read from the file by io_threads
 * threads (>= 1).  t_hist: a multiple of p->group, <= q_start and <= the
 * store's length.  *stats (when not NULL) receives this call's counts.
 * Errors: HGA_ERR_INVALID_ARG; HGA_ERR_CAPACITY when the step needs more
 * pages than the cache has (pages loaded so far stay valid); HGA_ERR_IO when
 * a read fails (that page stays absent). */
hga_status hga_store_prepare(hga_kv_store* s, const hga_params* p, int64_t q_start,
                             int64_t n_q, int64_t t_hist, const int32_t* group_idx,
                             const int32_t* group_cnt, int32_t io_threads,
                             hga_store_stats* stats);

/* hga_gather_history with the store's page cache as the source: copies the
 * same history groups from their cache slots into k_dev/v_dev (device
 * [n_kv_heads][t_cap][head_dim], t_cap = the store's, as given to
 * hga_store_open), each (KV head, group) once per step (gen, step as in
 * hga_gather_history).  group_idx/group_cnt are the DEVICE arrays, laid out
 * for the store's t_cap.  A group whose page is not resident sets HGA_ERR_DEVICE_CHECK
 * (hga_check) and is skipped: call hga_store_prepare first. */
hga_status hga_gather_store(const hga_params* p, const hga_kv_store* s, int64_t q_start,
                            int64_t n_q, int64_t t_hist, const int32_t* group_idx,
                            const int32_t* group_cnt, void* k_dev, void* v_dev, uint32_t* gen,
                            uint32_t step, unsigned long long* bytes, hga_stream_t stream);

/* Slots per (KV head, block) of chunk_idx (which = 0) or group_idx
 * (which = 1) for a context capacity t_cap; -1 on invalid parameters. */
int64_t hga_index_capacity(const hga_params* p, int64_t t_cap, int32_t which);

/* Validates a parameter block without launching anything. */
hga_status hga_validate_params(const hga_params* p);

/* Synchronises `stream`, then returns and clears the device status word
 * (HGA_OK, HGA_ERR_DEVICE_CHECK or HGA_ERR_TIMEOUT), or HGA_ERR_CUDA when the
 * synchronisation itself fails. */
hga_status hga_check(hga_stream_t stream);

/* Static string naming a status code. */
const char* hga_status_string(hga_status s);

/* Number of kernel launches issued by this library since load (for
 * accounting in benchmarks); never reset. */
int64_t hga_launch_count(void);

/* Text of the last CUDA error seen by this thread inside the library (the
 * cause behind an HGA_ERR_CUDA); static storage, never NULL. */
const char* hga_last_cuda_error(void);

/* Self-test of the software 2^x the attention kernel evaluates on the FMA
 * pipe for part of each softmax row (Cody-Waite reduction + degree-3
 * polynomial, relative error below 8e-5 for -125 <= x <= 127; smaller x
 * gives 2^-125).  Device arrays x, y of n floats; y[i] = 2^x[i].  Not part of
 * the method: it lets a test compare the kernel's exponential with exp2f. */
hga_status hga_selftest_exp2(const float* x, float* y, int64_t n, hga_stream_t stream);

/* Diagnostic switch (process-wide) of the bf16 kernels behind hga_attend,
 * hga_route_chunks, hga_route_groups and hga_forward: 0 = automatic (the
 * tcgen05 tensor-core kernels whenever the shapes allow them: 16-byte aligned
 * operands; attention: 128 divisible by the query heads per KV head and at
 * most 4608 attended groups per block; routing: at most 8 query heads per KV
 * head and 4096 candidates per block), 1 = the portable mma.sync kernels,
 * 2 = same as 0.  All variants compute the same function; tests use the
 * switch to check one against another.  Returns HGA_ERR_INVALID_ARG for any
 * other value. */
hga_status hga_set_kernel_variant(int32_t variant);

/* ---------------------------------------------------------------------------
 * Bounded waits.  Every wait of the tensor-core kernels (an mbarrier that a
 * TMA copy, an MMA commit or another warp completes) gives up after a limit,
 * raises HGA_ERR_TIMEOUT in the device status word (read by hga_check) and
 * lets the kernel drain what it issued and return, so a lost completion never
 * hangs the device.  No counterpart on the pages: this is the library's
 * failure detection. */

/* Sets the wait limit of the current device in nanoseconds (default 2e9,
 * i.e. 2 s).  1e6 <= ns <= 6e10, else HGA_ERR_INVALID_ARG.  Synchronous; the
 * limit applies to kernels launched afterwards on this device. */
hga_status hga_set_wait_limit_ns(uint64_t ns);

/* Self test of the bounded wait: one thread waits on an mbarrier that
 * nothing arrives on.  It gives up after the current limit, sets
 * HGA_ERR_TIMEOUT (returned by the next hga_check) and writes how long it
 * waited, in ns, to *elapsed_ns (8 bytes of device memory owned by the
 * caller).  Asynchronous on `stream`. */
hga_status hga_selftest_wait(unsigned long long* elapsed_ns, hga_stream_t stream);

/* Test hook (process-wide, one shot): the next launch of the tensor-core
 * attention kernel stops its K/V loads at ring load `load_index` (0-based,
 * counted over the CTA's K and V tiles in order), as if that copy never
 * completed.  The kernel's waits on it run into the limit, the kernel
 * returns and hga_check reports HGA_ERR_TIMEOUT; its output is then
 * incomplete.  -1 clears the hook; other negative values give
 * HGA_ERR_INVALID_ARG. */
hga_status hga_debug_stall_next_attend(int64_t load_index);

#ifdef __cplusplus
}
#endif
#endif /* HGA_H */
