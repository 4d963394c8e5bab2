/*
 * lsa.h -- C ABI of the Lookahead Sparse Attention (LSA) decode step on B200 (sm_100a).
 *
 * The method (arXiv 2606.09079, "FlashMemory-DeepSeek-V4: Lightning Index
 * Ultra-Long Context via Lookahead Sparse Attention"):
 *   every 64 decode steps a Neural Memory Indexer scores one compressed key
 *   per 64-token KV chunk and keeps every chunk whose sigmoid score is at
 *   least 0.5; inside the kept chunks the Lightning Indexer picks a finer
 *   top-k of tokens at every step; core attention runs over those tokens plus
 *   the always-resident most recent 8000 tokens.  Chunks outside the window
 *   may live in pinned host memory and are copied in when kept.
 *   (gist.science explainer, "Technisches Resuemee" section 2.1;
 *    cjcn.com.cn article, section 2.)
 *
 * Conventions shared by every entry point
 *   - bf16 data is passed as its 16-bit pattern (lsa_bf16).
 *   - Every pointer named *_dev or taking device data is a CUDA device
 *     pointer; *_host pointers are host memory.  The caller owns all memory:
 *     the library never allocates, frees or retains a pointer after return.
 *   - Work is enqueued asynchronously on the given stream.  Argument errors are
 *     detected on the host and returned before anything is launched; the
 *     message is available from lsa_last_error() (thread-local).
 *   - Conditions that only the device can see (a kept list longer than its
 *     capacity, a chunk-table entry that is -1 or out of range, a bounded wait
 *     that ran out) are OR-ed into *dev_status as LSA_DEV_* bits when
 *     dev_status is not NULL; the affected output is truncated or the bad row
 *     is skipped.  No call traps or aborts.
 *   - Scratch memory is passed in as (ws, ws_bytes); lsa_*_workspace_size()
 *     report the size.  Workspace contents need no initialisation.
 *   - Every entry point that enqueues work opens an NVTX range named after
 *     itself for the duration of the call (host side; free without a tool).
 *   - Chunk pools: token position p of sequence b lives in row p % 64 of pool
 *     slot chunk_table[b * table_stride + p / 64]; -1 marks a chunk that is not
 *     on the device.  Pools are [n_slots, 64, row_width] row-major.
 */
#ifndef LSA_H
#define LSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t lsa_bf16;
typedef struct CUstream_st *lsa_stream_t;   /* same type as cudaStream_t */
typedef struct CUevent_st *lsa_event_t;     /* same type as cudaEvent_t */

#define LSA_CHUNK 64            /* tokens per KV chunk */

enum {
    LSA_OK = 0,
    LSA_ERR_INVALID_ARG = 1,    /* null pointer, negative size, unsupported value */
    LSA_ERR_SHAPE = 2,          /* head count / width combination not supported */
    LSA_ERR_CUDA = 3,           /* a CUDA runtime call failed (message has the name) */
    LSA_ERR_CAPACITY = 4,       /* an output array is too small for the request */
    LSA_ERR_TIMEOUT = 5,
    LSA_ERR_TABLE = 6,          /* a host-side chunk table entry is invalid */
    LSA_ERR_WORKSPACE = 7       /* ws_bytes smaller than the workspace query */
};

/* bits OR-ed into *dev_status by kernels */
#define LSA_DEV_CAPACITY 1      /* a list was longer than its capacity and was cut */
#define LSA_DEV_TABLE 2         /* a needed chunk had no valid slot; its rows were skipped */
#define LSA_DEV_TIMEOUT 4       /* a bounded device wait ran out */
#define LSA_DEV_INDEX 8         /* an index input was out of range and was skipped */

/* Message of the last error returned on this thread ("" if none). */
const char *lsa_last_error(void);

/* Library version string. */
const char *lsa_version(void);

/*
 * Failure-path test switch (no counterpart in the paper).  The next launch of
 * the named tcgen05 kernel -- LSA_TEST_STALL_ATTENTION: the 128-head latent
 * attention of lsa_sparse_decode; LSA_TEST_STALL_INDEXER: the indexer scoring
 * of lsa_topk -- makes its first bounded wait wait on a barrier that nothing
 * arrives on, for 2 ms.  That wait runs out: the kernel sets LSA_DEV_TIMEOUT in
 * dev_status, its other waits return, the copies and tensor-core work it
 * already issued complete, and it returns; the stream and context stay
 * usable.  Only for tests of that path; the switch clears itself at that launch.
 */
#define LSA_TEST_STALL_ATTENTION 1
#define LSA_TEST_STALL_INDEXER 2
int lsa_test_stall_next_wait(int which);

/*
 * Failure-path test switch (no counterpart in the paper): after `after` more
 * host-issued copies of lsa_gather_chunks succeed, the next one reports failure
 * without being enqueued, as a failed cudaMemcpyAsync would; the switch then
 * turns itself off.  after = -1 turns it off.  Only for tests of that path.
 */
int lsa_test_fail_copy(int after);

/*
 * a1 -- Neural Memory Indexer chunk gate.
 * Passage: gist.science explainer 2.1 ("Scoring-Mechanismus", "Dynamisches
 * Fetching"); cjcn.com.cn article section 2 (ReLU replaced by Sigmoid, fixed
 * threshold 0.5, every chunk above it is fetched).
 *
 * For each sequence b and each of its chunks s:
 *   logit = sum_h w[b,h] * (q[b,h,:] . khat[off[b]+s, :]),  I = sigmoid(logit)
 *   keep s  iff  I >= 0.5  (evaluated as logit >= 0, which is the same test).
 * Kept chunk indices (relative to the sequence) are written ascending.
 *
 *   q          [B, Hn, dn] bf16 (device)
 *   w          [B, Hn]     bf16 (device), head weights
 *   khat       [total_chunks, dn] bf16 (device), one compressed key per chunk
 *   seq_chunk_offset [B+1] int64 (device), sequence b owns rows off[b]..off[b+1]-1
 *   max_chunks_per_seq     host upper bound of off[b+1]-off[b]
 *   kept_idx   [B, kept_cap] int32 (device, out): ascending; unused entries -1
 *   kept_count [B] int32 (device, out): number written (<= kept_cap); a longer
 *              list sets LSA_DEV_CAPACITY
 *   logits     [total_chunks] fp32 (device, out, optional)
 * Supported: dn in {64, 128}, Hn a multiple of 8 up to 128.
 */
int lsa_nmi_select(const lsa_bf16 *q, const lsa_bf16 *w, const lsa_bf16 *khat,
                   const int64_t *seq_chunk_offset, int B, int Hn, int dn,
                   int64_t total_chunks, int max_chunks_per_seq,
                   int32_t *kept_idx, int32_t *kept_count, int kept_cap,
                   float *logits, int32_t *dev_status,
                   void *ws, size_t ws_bytes, lsa_stream_t stream);
size_t lsa_nmi_select_workspace_size(int B, int max_chunks_per_seq);

/*
 * a1, OR mode -- several independent memory indexers gated together.
 * Passage: cjcn.com.cn article section 4 (one independent indexer at each of
 * layers 10, 12 and 20; a chunk is recalled when any of the three scores it at
 * 0.5 or more, "OR-mode routing"); gist.science explainer 2.4 (a union of the
 * three layers' predictions).
 *
 * Indexer i (0 <= i < n_idx) has its own queries q[i] [B, Hn, dn], head
 * weights w[i] [B, Hn] and compressed keys khat[i] [total_chunks, dn] (all
 * bf16, device); the ARRAYS q, w, khat of n_idx device pointers are host
 * memory.  Every indexer scores every chunk as lsa_nmi_select does; chunk s of
 * sequence b is kept iff at least one indexer's logit is >= 0.  The kept list
 * is the ascending union; kept_idx, kept_count, kept_cap, dev_status and the
 * capacity rule are those of lsa_nmi_select.
 *   logits  [n_idx, total_chunks] fp32 (device, out, optional): each indexer's logits
 * Supported: 1 <= n_idx <= 4, shapes as lsa_nmi_select (common to all indexers).
 * n_idx = 1 is exactly lsa_nmi_select.
 */
int lsa_nmi_select_union(int n_idx, const lsa_bf16 *const *q, const lsa_bf16 *const *w,
                         const lsa_bf16 *const *khat, const int64_t *seq_chunk_offset, int B, int Hn, int dn,
                         int64_t total_chunks, int max_chunks_per_seq,
                         int32_t *kept_idx, int32_t *kept_count, int kept_cap,
                         float *logits, int32_t *dev_status,
                         void *ws, size_t ws_bytes, lsa_stream_t stream);
size_t lsa_nmi_select_union_workspace_size(int n_idx, int B, int max_chunks_per_seq);

/*
 * Memory-indexer query encoder: the hidden state h_t of each token mapped to
 * the gate's low-rank queries and head weights (the inputs of lsa_nmi_select).
 * Passage: gist.science explainer 2.1 ("Memory Indexer": a dual encoder maps
 * h_t to low-rank indexer queries) and 2.3 (only the query encoder's low-rank
 * projections are trained); cjcn.com.cn article section 4 (randomly
 * initialised weights; query projection rank 2048 instead of 1536).
 *
 * Reading taken (the pages give no formula): for every token b
 *   c = W_down h[b]          rank entries
 *   q[b] = W_up c            Hn * dn entries, head-major (entry h * dn + d)
 *   w[b] = W_head h[b]       Hn entries
 * with no normalisation or nonlinearity.  Products accumulate in fp32; c
 * enters the second product as two bf16 parts (hi = bf16(c), lo = bf16(c - hi)).
 *
 *   h       [B, d_model] bf16 (device)
 *   w_down  [rank, d_model], w_up [Hn * dn, rank], w_head [Hn, d_model] bf16 (device, row-major)
 *   q_out   [B, Hn, dn] bf16 and w_out [B, Hn] bf16 (device, out): round to nearest even
 *   q_f32   [B, Hn, dn], w_f32 [B, Hn] fp32 (device, out, optional): before rounding
 * Supported: 1 <= B <= 32; d_model and rank multiples of 64.
 */
int lsa_query_encoder(const lsa_bf16 *h, int B, int d_model, const lsa_bf16 *w_down, int rank,
                      const lsa_bf16 *w_up, const lsa_bf16 *w_head, int Hn, int dn,
                      lsa_bf16 *q_out, lsa_bf16 *w_out, float *q_f32, float *w_f32, int32_t *dev_status,
                      void *ws, size_t ws_bytes, lsa_stream_t stream);
size_t lsa_query_encoder_workspace_size(int B, int d_model, int rank, int Hn, int dn);

/*
 * Baseline selectors: the two schemes the pages compare LSA with, producing a
 * kept list in the same form as lsa_nmi_select so that the same top-k,
 * attention and fetch calls run after them.
 * Passage: cjcn.com.cn article section 5 (a pure sliding window keeping the
 * recent 8K tokens, and random retention of 10 % of the history chunks; every
 * scheme keeps the recent window); gist.science explainer section 4 ("Recency
 * Only" and "Random 10%").
 *
 * n_old = window_start[b] / 64 chunks lie before sequence b's window.
 *   LSA_SELECT_RECENT: no older chunk is kept (kept_count 0, kept_idx all -1);
 *     window_start may be NULL.
 *   LSA_SELECT_RANDOM: m = floor((n_old * keep_num + keep_den / 2) / keep_den)
 *     older chunks are kept, uniformly at random: chunk s draws
 *     u = (output number b * 2^32 + s of a SplitMix64 stream started at seed) >> 40
 *     and the m chunks with the smallest u are kept, ties to the lower index.
 *     (SplitMix64: Steele, Lea and Flood, OOPSLA 2014; output c is
 *     mix(seed + (c + 1) * 0x9E3779B97F4A7C15).)
 *   window_start [B] int32 (device); max_old_chunks: host bound of n_old (larger
 *     n_old is cut to it and sets LSA_DEV_INDEX)
 *   kept_idx [B, kept_cap], kept_count [B] int32 (device, out): ascending, -1 after
 * Returns LSA_ERR_CAPACITY if round(max_old_chunks * keep_num / keep_den) > kept_cap.
 */
#define LSA_SELECT_RECENT 0
#define LSA_SELECT_RANDOM 1
int lsa_select_baseline(int mode, const int32_t *window_start, int B, int max_old_chunks, uint64_t seed,
                        int keep_num, int keep_den, int32_t *kept_idx, int32_t *kept_count, int kept_cap,
                        int32_t *dev_status, void *ws, size_t ws_bytes, lsa_stream_t stream);
size_t lsa_select_baseline_workspace_size(int B, int max_old_chunks);

/*
 * a2 + a3 -- Lightning-Indexer scoring and fine top-k inside the kept chunks.
 * Passage: gist.science explainer 2.1 ("Gestufte Selektion"); cjcn.com.cn
 * article section 2 (the native indexer takes a top-k inside the reduced set).
 *
 * Candidates of sequence b: every token of every kept chunk c with
 * c < window_start[b] / 64 (chunks in the recent window are attended anyway),
 * in ascending position.  Score of token t:
 *   I_t = sum_h w_li[b,h] * max(0, q_li[b,h,:] . key_t)
 * The k largest scores are kept, ties to the lower position; the kept
 * positions are written ascending, followed by -1 up to k.
 *
 *   q_li      [B, Hl, dl] bf16, w_li [B, Hl] bf16 (device)
 *   li_pool   [n_slots, 64, dl] bf16 (device): indexer key of every resident token
 *   chunk_table [B, table_stride] int32 (device)
 *   kept_idx  [B, kept_cap], kept_count [B] int32 (device): lsa_nmi_select output
 *             (strictly ascending chunk indices; the first kept_count[b] entries are read)
 *   window_start [B] int32 (device): first position of the recent window, multiple of 64
 *   topk_idx  [B, k] int32 (device, out); topk_count [B] int32 (device, out)
 *   scores    [B, kept_cap * 64] fp32 (device, out, optional): candidate scores
 * Supported: dl in {64, 128}, Hl a multiple of 8 up to 128, 1 <= k <= 65536.
 */
int lsa_topk(const lsa_bf16 *q_li, const lsa_bf16 *w_li, const lsa_bf16 *li_pool, int64_t n_slots,
             const int32_t *chunk_table, int table_stride,
             const int32_t *kept_idx, const int32_t *kept_count, int kept_cap,
             const int32_t *window_start, int B, int Hl, int dl, int k,
             int32_t *topk_idx, int32_t *topk_count, float *scores, int32_t *dev_status,
             void *ws, size_t ws_bytes, lsa_stream_t stream);
size_t lsa_topk_workspace_size(int B, int kept_cap);
/* Kernels one lsa_topk call launches for these sizes: 2 where the tcgen05
 * indexer kernel serves the shape (Hl in {32, 64, 128}, dl in {64, 128},
 * B <= 64) and counts the kept cold chunks in its own prologue, else 3 (a
 * counting kernel first); 0 for sizes that lsa_topk rejects.  Host only. */
int lsa_topk_kernel_count(int B, int Hl, int dl);

/*
 * a5 + a2 + a3 in one call: the append of the decoded token (lsa_append_token,
 * latent layout: one KV row of kv_width in kv_pool and one indexer key in
 * li_pool per sequence), then the indexer scoring and top-k (lsa_topk).
 * Passage: as lsa_append_token and lsa_topk.
 * Where the tcgen05 indexer serves the shape (lsa_topk_kernel_count == 2) the
 * append is done by the indexer launch itself -- that kernel reads neither the
 * window's rows nor window_len -- so the step has one launch less; other shapes
 * launch the append first.  Arguments, alignment rules and results are those
 * of the two calls (kv_row_stride and kv_width as k_row_stride and k_width).
 */
int lsa_append_topk(const lsa_bf16 *new_kv, const lsa_bf16 *new_li, lsa_bf16 *kv_pool, int64_t kv_row_stride,
                    int kv_width, int32_t *window_len, const lsa_bf16 *q_li, const lsa_bf16 *w_li,
                    lsa_bf16 *li_pool, int64_t n_slots, const int32_t *chunk_table, int table_stride,
                    const int32_t *kept_idx, const int32_t *kept_count, int kept_cap,
                    const int32_t *window_start, int B, int Hl, int dl, int k,
                    int32_t *topk_idx, int32_t *topk_count, float *scores, int32_t *dev_status,
                    void *ws, size_t ws_bytes, lsa_stream_t stream);

/*
 * a3 alone, on given fp32 scores (exact unit entry point).
 * Sequence b owns scores[cand_offset[b] .. cand_offset[b+1]); writes the
 * indices (relative to cand_offset[b]) of its min(k, n_b) largest scores,
 * ties to the lower index, ascending, then -1 up to k.
 *   cand_offset [B+1] int64 (device); max_cand host upper bound of n_b.
 */
int lsa_topk_from_scores(const float *scores, const int64_t *cand_offset, int B, int max_cand, int k,
                         int32_t *topk_idx, int32_t *topk_count,
                         void *ws, size_t ws_bytes, lsa_stream_t stream);

/*
 * a4 -- sparse decode attention over top-k rows plus the recent window.
 * Passage: cjcn.com.cn article section 2 (core attention over the selected
 * entries; the most recent 8000 tokens always kept on the GPU); gist.science
 * explainer 2.1 ("Gestufte Selektion": final core-attention computation).
 *
 * Row set of sequence b: S = {topk_idx[b, 0..topk_count[b])} followed by the
 * positions window_start[b] .. window_start[b] + window_len[b] - 1.  For each
 * query head h:
 *   o[b,h,:] = sum_{j in S} softmax_j(scale * q[b,h,:] . K_j) V_j
 *   lse[b,h] = log sum_{j in S} exp(scale * q[b,h,:] . K_j)
 * One KV head is shared by all query heads.  Latent layout (v_pool == NULL):
 * K_j is the dqk-wide row of k_pool and V_j its first dv columns.  Otherwise
 * V_j is the row of v_pool.
 *
 *   q       [B, Hq, dqk] bf16 (device)
 *   k_pool  [n_slots, 64, k_row_stride] bf16; v_pool [n_slots, 64, v_row_stride] or NULL
 *   topk_idx [B, k], topk_count [B], window_start [B], window_len [B] int32 (device)
 *   max_window_len   host upper bound of window_len[b] (sizes the split-K grid)
 *   out     [B, Hq, dv] fp32 (device, out); lse [B, Hq] fp32 (device, out, optional)
 * Supported: (Hq, dqk, dv) = (16, 128, 128) with separate K/V pools, and
 * (128 or 64, 576, 512) latent.  Strides in elements, multiples of 8.
 */
int lsa_sparse_decode(const lsa_bf16 *q, const lsa_bf16 *k_pool, int64_t k_row_stride,
                      const lsa_bf16 *v_pool, int64_t v_row_stride, int64_t n_slots,
                      const int32_t *chunk_table, int table_stride,
                      const int32_t *topk_idx, const int32_t *topk_count, int k,
                      const int32_t *window_start, const int32_t *window_len, int max_window_len,
                      int B, int Hq, int dqk, int dv, float scale,
                      float *out, float *lse, int32_t *dev_status,
                      void *ws, size_t ws_bytes, lsa_stream_t stream);
size_t lsa_sparse_decode_workspace_size(int B, int Hq, int dqk, int dv, int k, int max_window_len);

/*
 * a4 -- merge of attention results over disjoint row sets of the same queries.
 * Passage: as lsa_sparse_decode (softmax attention over the union of the row
 * sets); the split itself is this library's: the window rows and the top-k
 * rows of a step can be attended in two calls (the window part while cold
 * chunks are still being fetched), and a long sequence can be attended in
 * pieces, one per device.
 *
 *   o_parts [R, B, Hq, dv], lse_parts [R, B, Hq] fp32 (device): part r as written
 *   by lsa_sparse_decode over its rows (lse_r = -inf for a part without rows)
 *   out [B, Hq, dv], lse [B, Hq] (optional) fp32 (device, out):
 *     lse = log sum_r exp(lse_r),  out = sum_r exp(lse_r - lse) o_r
 *   (no rows in any part: out = 0, lse = -inf).  dv a multiple of 4.
 */
int lsa_merge_attention(const float *o_parts, const float *lse_parts, int R, int B, int Hq, int dv,
                        float *out, float *lse, lsa_stream_t stream);

/*
 * a5 -- lookahead reuse: append the decoded token to the recent window.
 * Passage: gist.science explainer 2.1 ("Periodische Triggerung", tau = 64);
 * cjcn.com.cn article section 2 (the selection serves the next 64 steps).
 *
 * For each sequence b the token at position p = window_start[b] + window_len[b]
 * gets new_k[b] (and new_v[b], new_li[b]) written into its pool row, then
 * window_len[b] is incremented.  The chunk of p must already have a slot; a
 * chunk without one sets LSA_DEV_TABLE in dev_status and leaves that sequence
 * unchanged.
 *   new_k [B, k_width], new_v [B, v_width] or NULL, new_li [B, dl] or NULL (device)
 * Widths and row strides are multiples of 8 elements and every base pointer is
 * 16-byte aligned (rows move as 16-byte vectors), else LSA_ERR_INVALID_ARG.
 */
int lsa_append_token(const lsa_bf16 *new_k, const lsa_bf16 *new_v, const lsa_bf16 *new_li,
                     lsa_bf16 *k_pool, int64_t k_row_stride, int k_width,
                     lsa_bf16 *v_pool, int64_t v_row_stride, int v_width,
                     lsa_bf16 *li_pool, int dl, int64_t n_slots,
                     const int32_t *chunk_table, int table_stride,
                     const int32_t *window_start, int32_t *window_len, int B,
                     int32_t *dev_status, lsa_stream_t stream);

/*
 * a6 -- cold-chunk fetch from the pinned host pool (one sequence).
 * Passage: cjcn.com.cn article section 2 (unselected chunks stay in CPU
 * memory; selected ones are moved to GPU memory); gist.science explainer 2.1
 * ("Dynamisches Fetching" from the CPU cold pool).
 *
 * Every kept chunk c (from the HOST copy of the kept list) with
 * c < first_window_chunk is given device slot first_free_slot + j (j = its
 * rank among those chunks) in each of the n_pools pools; runs of consecutive
 * chunks are copied with one cudaMemcpyAsync per pool on `stream`.  The slots
 * are written into chunk_table_host (pinned, table_len entries, caller-owned),
 * which is then copied to chunk_table_dev on the same stream, and `done` (if
 * not NULL) is recorded after the last copy.  The caller orders later work
 * after `done`, and leaves chunk_table_host unchanged until then (the table
 * copy reads it asynchronously).
 * A copy that cannot be enqueued returns LSA_ERR_CUDA with chunk_table_host as
 * it was and chunk_table_dev not rewritten; chunk copies enqueued before it
 * still run, into slots that neither table references.
 *   host_pools[i]  pinned host base of pool i, [n_host_chunks, chunk_bytes[i]]
 *   dev_pools[i]   device base of pool i, [n_slots, chunk_bytes[i]]
 *   n_fetched      (host, out) number of chunks copied
 */
int lsa_gather_chunks(int n_pools, const void *const *host_pools, const size_t *chunk_bytes,
                      void *const *dev_pools, int64_t n_host_chunks, int64_t n_slots,
                      const int32_t *kept_idx_host, int kept_count_host, int first_window_chunk,
                      int first_free_slot, int32_t *chunk_table_host, int32_t *chunk_table_dev,
                      int table_len, lsa_stream_t stream, lsa_event_t done, int *n_fetched);

/*
 * a6, device-driven -- residency plan of the next lookahead window (one sequence).
 * Passage: cjcn.com.cn article section 2 (every 64 steps the indexer predicts
 * the chunks the next 64 steps will need and only those are moved from the
 * CPU cold pool to GPU memory); gist.science explainer 2.1 ("Dynamisches
 * Fetching" from the CPU cold pool).
 *
 * The next window needs its window chunks [first_window_chunk,
 * window_end_chunk) -- the last of them receives the window's appended tokens --
 * and every chunk of the kept list (kept_idx[0 .. kept_count[0]), device, as
 * written by lsa_nmi_select with B = 1).  table_next (device, out, table_len
 * entries) keeps the slot of every needed chunk that table_cur already maps,
 * gives every other needed chunk a slot that table_cur leaves free (ascending
 * chunk and slot order), and holds -1 elsewhere.  Needed chunks before the
 * window that received a new slot are the copy list: copy_chunk / copy_slot
 * (device, out, ascending chunk order) and copy_count[0] (device, out).  So only
 * the delta against what is resident moves, and slots of chunks that are no
 * longer needed are free again once table_next replaces table_cur.
 * Not enough free slots, or more than copy_cap copies, sets LSA_DEV_CAPACITY
 * (the chunks without a slot get -1).  Slots are < n_slots.
 * Nothing here waits for the host: the call can run on a side stream while the
 * current window's steps run, since it only reads table_cur.
 */
int lsa_plan_residency(const int32_t *table_cur, int32_t *table_next, int table_len,
                       const int32_t *kept_idx, const int32_t *kept_count, int kept_cap,
                       int first_window_chunk, int window_end_chunk, int64_t n_slots,
                       int32_t *copy_chunk, int32_t *copy_slot, int32_t *copy_count, int copy_cap,
                       int32_t *dev_status, void *ws, size_t ws_bytes, lsa_stream_t stream);
size_t lsa_plan_residency_workspace_size(int table_len, int64_t n_slots);

/*
 * a6, device-driven -- copy listed chunks from the pinned host pools.
 * Passage: as lsa_plan_residency.
 *
 * For j < copy_count[0] (device): chunk copy_chunk[j] of every pool i is copied
 * from host_pools[i] + copy_chunk[j] * chunk_bytes[i] to dev_pools[i] +
 * copy_slot[j] * chunk_bytes[i].  A kernel reads the host pools through their
 * device mapping over the host link (one launch for the whole list, no
 * per-chunk copy calls and no host round trip for the list).  host_pools[i]
 * must be page-locked host memory (cudaHostAlloc / cudaHostRegister; checked,
 * LSA_ERR_INVALID_ARG otherwise); chunk_bytes[i] a multiple of 16.  A chunk or
 * slot out of range is skipped and sets LSA_DEV_TABLE.
 */
int lsa_fetch_chunks(int n_pools, const void *const *host_pools, const size_t *chunk_bytes,
                     void *const *dev_pools, int64_t n_host_chunks, int64_t n_slots,
                     const int32_t *copy_chunk, const int32_t *copy_slot, const int32_t *copy_count,
                     int copy_cap, int32_t *dev_status, lsa_stream_t stream);

/*
 * a5 -- start of the next lookahead window: window_start[b] += by (a multiple of
 * 64: the window slides by the tokens decoded in the last window) and
 * window_len[b] = new_len, for every b < B (device arrays).
 */
int lsa_advance_window(int32_t *window_start, int32_t *window_len, int B, int by, int new_len,
                       lsa_stream_t stream);

/*
 * a7 (offline) -- cross-layer majority-vote labels for one decode window.
 * Passage: gist.science explainer 2.2 (softmax, top-p 0.6, at least theta = 3
 * layers); cjcn.com.cn article section 3 (a chunk selected by at least 3 layers
 * at the same time is golden; golden chunks of all steps are merged).
 *
 * For each layer l and step t: p = softmax(scores[l,t,:]); order chunks by
 * score descending (ties to the lower index); keep the smallest prefix whose
 * cumulative p reaches top_p (crossing chunk included).  count[t][c] = number
 * of layers keeping c at step t.
 *   mode 0: max_votes[c] = max_t count[t][c]
 *   mode 1: max_votes[c] = number of distinct layers keeping c at any step
 *   labels[c] = (max_votes[c] >= min_layers)
 *   scores [n_layers, n_steps, n_chunks] fp32 (device); labels [n_chunks] uint8
 *   (device, out); max_votes [n_chunks] int32 (device, out, optional)
 * Supported: 1 <= n_layers <= 64, 1 <= n_chunks <= 16384.
 */
int lsa_label_vote(const float *scores, int n_layers, int n_steps, int n_chunks,
                   float top_p, int min_layers, int mode,
                   uint8_t *labels, int32_t *max_votes,
                   void *ws, size_t ws_bytes, lsa_stream_t stream);
size_t lsa_label_vote_workspace_size(int n_layers, int n_steps, int n_chunks);

/*
 * a7 without a workspace, for callers that cannot allocate device memory.
 * No passage of the paper corresponds to this entry point: it is the same
 * label vote as lsa_label_vote, offered to code that is not allowed to call
 * cudaMalloc at the point where it labels -- for example a plugin that may
 * only touch memory its host handed over, or code running while the
 * process's device allocator must not be entered.  Such callers pass only
 * their inputs and outputs; the vote masks live in a fixed 4 MiB array built
 * into the library (every GPU that loads the library keeps it until exit).
 *
 * Same arguments, results and limits as lsa_label_vote, plus:
 *   - n_steps * n_chunks * ceil(n_layers / 32) must not exceed 1,048,576
 *     (LSA_LABEL_VOTE_NOALLOC_MAX_WORDS); larger problems return
 *     LSA_ERR_CAPACITY before anything is launched.
 *   - The call allocates nothing (no cudaMalloc, cudaFree or allocating
 *     library routine).  It clears the part of the array it uses on `stream`
 *     before voting.
 *   - The first call on a device looks up the array's device address with
 *     that device current; make that first call before any stream capture.
 *     The address is kept for the life of the process: after a
 *     cudaDeviceReset of that device it is stale, so do not call this entry
 *     point on that device again in the same process.
 *   - Every call shares the one array: calls whose GPU work overlaps (on
 *     different streams, or from different threads) race and must be ordered
 *     by the caller.
 */
#define LSA_LABEL_VOTE_NOALLOC_MAX_WORDS (1u << 20)
int lsa_label_vote_noalloc(const float *scores, int n_layers, int n_steps, int n_chunks,
                           float top_p, int min_layers, int mode,
                           uint8_t *labels, int32_t *max_votes, lsa_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* LSA_H */
