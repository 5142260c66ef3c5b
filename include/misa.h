/*
 * misa.h -- C ABI of the MISA routed sparse-attention indexer for NVIDIA B200 (sm_100a).
 *
 * Method: "MISA: Mixture of Indexer Sparse Attention for Long-Context LLM
 * Inference" (Zhou et al., 2026).  The DSA indexer scores every prefix token
 * of a query with all H indexer heads,
 *     I[t,s] = sum_h w[t,h] * ReLU(q[t,h] . k[s]),   keys s = 0..t,
 * and keeps the top-k tokens for the main attention.  MISA treats the H heads
 * as a mixture-of-experts pool: a router on mean-pooled key blocks keeps m
 * heads per query, and only those m heads run the token-level scoring.
 * MISA-dagger keeps k_cand routed candidates and re-ranks them with all H heads.
 *
 * Conventions for every entry point
 *   - All array arguments are DEVICE pointers owned by the caller; the library
 *     allocates no device memory.  Scratch space is the caller's workspace
 *     (size from misa_workspace_size).
 *   - bf16 tensors are passed as uint16_t bit patterns.  Rows are row-major
 *     and 16-byte aligned; head_dim must be 128.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream).  The return code reports argument and launch errors
 *     only.  Device-side conditions (a bounded wait that timed out, an index
 *     out of range, a position or candidate out of its sequence) set bits in
 *     a per-device status word read by misa_stream_status.
 *   - No call throws; on error the message is kept in a thread-local buffer
 *     (misa_last_error_string).
 *   - Ties: heads are ranked by (router score desc, head index asc); tokens by
 *     (score desc, token index asc); -0 counts as +0.  A query whose prefix is
 *     shorter than k selects every prefix token and pads its row with index
 *     -1 and value -inf.  Row order of idx/val is unspecified.
 *   - NaN (from a NaN in q, w or K): a head whose router score is NaN is
 *     ranked last and MISA_STATUS_BAD_INPUT is set; a NaN token score ranks
 *     below every number, so it is selected only when its row has fewer
 *     other scores than min(k, prefix length), and then (with value NaN)
 *     the same bit is set.
 */
#ifndef MISA_H_
#define MISA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef void* misa_stream_t; /* cudaStream_t */

/* Return codes. */
enum {
  MISA_OK = 0,
  MISA_ERR_INVALID_ARG = 1,        /* null pointer, bad size, misaligned pointer */
  MISA_ERR_UNSUPPORTED = 2,        /* valid but not built: head_dim != 128, m not a power of two ... */
  MISA_ERR_WORKSPACE_TOO_SMALL = 3,
  MISA_ERR_CUDA = 4,               /* a CUDA runtime call failed (message has the CUDA error) */
  MISA_ERR_DEVICE_TIMEOUT = 5,     /* misa_stream_status only */
  MISA_ERR_DEVICE_BOUNDS = 6,      /* misa_stream_status only */
  MISA_ERR_DEVICE_BAD_INPUT = 7    /* misa_stream_status only */
};

/* Bits of the device status word. */
#define MISA_STATUS_TIMEOUT   0x1u /* a bounded wait in a kernel gave up; that CTA returned early */
#define MISA_STATUS_BOUNDS    0x2u /* an index fell outside its buffer; the access was skipped */
#define MISA_STATUS_BAD_INPUT 0x4u /* a query position or candidate outside its sequence, a NaN
                                      router score, or a NaN token score in a selection */

/*
 * Problem description (the shapes of one indexer call).
 *
 * Keys of all sequences are packed: K is [total_keys, head_dim] bf16 and
 * sequence s owns rows key_offsets[s] .. key_offsets[s+1]-1.  Its pooled keys
 * (one per block of `block` consecutive keys, the last block possibly
 * partial) are rows block_offsets[s] .. block_offsets[s+1]-1 of Kbar, with
 * block_offsets[s+1]-block_offsets[s] = ceil(L_s / block)  (gist.science
 * summary, "Methodologie: MISA": M = ceil(L/B) blocks).  Queries of sequence
 * s are rows query_offsets[s] .. query_offsets[s+1]-1 of q / w; query t sits
 * at position q_pos[t] in its sequence and sees keys 0..q_pos[t] (causal,
 * self included).
 */
typedef struct {
  int32_t num_seqs;              /* S >= 1 */
  int32_t num_queries;           /* T >= 0 */
  int32_t num_heads;             /* H, 1..64 */
  int32_t head_dim;              /* d, must be 128 */
  int32_t block;                 /* B, pooling block, 1..4096 */
  int32_t max_seq_len;           /* host-side upper bound on every L_s (sizes grids) */
  int64_t total_keys;            /* rows of K = key_offsets[S] */
  int64_t total_blocks;          /* rows of Kbar = block_offsets[S] */
  const int64_t* key_offsets;    /* device [S+1], non-decreasing, key_offsets[0] = 0 */
  const int64_t* block_offsets;  /* device [S+1], see misa_block_offsets */
  const int32_t* query_offsets;  /* device [S+1], non-decreasing, query_offsets[0] = 0 */
  const int32_t* q_pos;          /* device [T], 0 <= q_pos[t] < L_seq(t) */
} misa_problem_t;

/* Bytes of workspace that any entry point below needs for this problem with
 * m routed heads, final top-k `k` and MISA-dagger candidate count `k_cand`
 * (0 if unused), on its fastest path.  Returns 0 on invalid arguments.
 * For a prefill that streams (misa_score_topk, dsa_index_dense) this
 * includes candidate lists per query row for the exact selection after the
 * scoring pass, about T * (2 * 1.4 * k / 128 + 16) KB with that row count
 * between 32 and 256 (8.1 GB for 131072 queries at k = 2048, 25 GB at the
 * MISA-dagger keep k = 8192); a smaller workspace takes slower paths (selection
 * inside the scoring kernel, then score rows with a separate top-k) and
 * MISA_ERR_WORKSPACE_TOO_SMALL only below what the slowest path needs. */
size_t misa_workspace_size(const misa_problem_t* p, int32_t m, int32_t k, int32_t k_cand);

/* block_offsets[s] = sum_{s'<s} ceil(L_s' / block) from key_offsets
 * (device arrays, S+1 entries each). */
int misa_block_offsets(const int64_t* key_offsets, int32_t num_seqs, int32_t block,
                       int64_t* block_offsets, misa_stream_t stream);

/* Step 1 -- mean-pooled keys (gist.science summary, "Methodologie: MISA",
 * Lightweight Block-Pooled Router: mean-pooled indexer keys per block).
 * Kbar[b,:] = (1/|b|) sum_{s in b} K[s,:], the last block of a sequence
 * averaged over the keys present.  Summed in fp64, divided in fp64, rounded
 * once to fp32.
 *   K    [total_keys, 128] bf16;  Kbar [total_blocks, 128] fp32 (written). */
int misa_pool_keys(const misa_problem_t* p, const uint16_t* K, float* Kbar, misa_stream_t stream);

/* Step 1, incremental (decode): re-pools only the blocks of each sequence s
 * that hold keys at positions >= from_pos[s] (e.g. the keys appended since
 * Kbar was last computed); every other row of Kbar is left unchanged, so
 * Kbar must already hold the pooled means of the earlier blocks.  Same
 * arithmetic as misa_pool_keys, so the updated rows are bit-identical to a
 * full re-pooling.
 *   from_pos [S] int32 device array; a value <= 0 re-pools the whole
 *   sequence, a value >= its length leaves it unchanged.  One CTA per
 *   sequence. */
int misa_pool_keys_from(const misa_problem_t* p, const uint16_t* K, float* Kbar,
                        const int32_t* from_pos, misa_stream_t stream);

/* Step 2 -- block-pooled router (same passage: per-head affinities on the
 * pooled keys, aggregated into one importance score per head, top-h heads).
 *     r[t,h] = w[t,h] * sum_{b < M_t} ReLU(q[t,h] . Kbar_t[b]),  M_t = ceil((t+1)/B)
 * over the floor((t+1)/B) full blocks of Kbar plus, when (t+1) mod B != 0,
 * the causal partial block (mean of keys floor((t+1)/B)*B .. t).  Keeps the
 * m best heads per query.
 *   q [T, H, 128] bf16;  w [T, H] fp32;  K, Kbar as above;  1 <= m <= H, m a power of two.
 *   heads [T, m] int32  (written; rank order);
 *   q_r   [T, m, 128] bf16 (written; q_r[t,j] = q[t, heads[t,j]]);
 *   w_r   [T, m] fp32  (written; w_r[t,j] = w[t, heads[t,j]]);
 *   router_scores [T, H] fp32 or NULL (written if not NULL). */
int misa_route(const misa_problem_t* p, const uint16_t* q, const float* w, const uint16_t* K,
               const float* Kbar, int32_t m, int32_t* heads, uint16_t* q_r, float* w_r,
               float* router_scores, void* ws, size_t ws_bytes, misa_stream_t stream);

/* misa_route without a caller workspace: its scratch is a fixed 4 MiB device
 * array inside the library (one per device), for callers that cannot
 * allocate on the decode path (a host runtime with no device allocator of
 * its own, or code that must not call cudaMalloc there).  No counterpart in
 * the paper.  Arguments and results as misa_route, which it runs with that
 * array as its workspace; it allocates no memory.
 *   - The first call on each device (with that device current) looks up the
 *     array's address; make it before capturing a stream that uses the call.
 *   - Nothing in the array needs to start at zero.
 *   - Calls on one device must not overlap in execution: they share the
 *     array and race on it.  Issue them on one stream, or order them.
 *   - MISA_ERR_UNSUPPORTED when the problem needs more than 4 MiB of router
 *     scratch (the message gives both sizes): decode batches fit; prefill
 *     fits up to about 7K keys, since the tensor-core router keeps a 512-byte
 *     running block mean per key.  MISA_ERR_INVALID_ARG while tracing is on
 *     for the calling thread. */
int misa_route_static(const misa_problem_t* p, const uint16_t* q, const float* w,
                      const uint16_t* K, const float* Kbar, int32_t m, int32_t* heads,
                      uint16_t* q_r, float* w_r, float* router_scores, misa_stream_t stream);

/* Steps 3+4 -- routed token scoring and per-query top-k (same section,
 * Sparse Token Scoring: only the routed heads score the full prefix; the
 * top-k tokens come from these reduced scores).
 *     I[t,s] = sum_{j<m} w_r[t,j] * ReLU(q_r[t,j] . K[s]),  s = 0..q_pos[t]
 *   q_r [T, m, 128] bf16;  w_r [T, m] fp32;  1 <= k <= 65536.
 *   idx [T, k] int32 token indices within the sequence;  val [T, k] fp32 scores.
 *   scores_dbg: NULL, or [T, scores_ld] fp32 receiving I[t, 0..q_pos[t]]
 *   (entries past the prefix are unspecified); scores_ld >= max_seq_len. */
int misa_score_topk(const misa_problem_t* p, const uint16_t* q_r, const float* w_r, int32_t m,
                    const uint16_t* K, int32_t k, int32_t* idx, float* val, float* scores_dbg,
                    int64_t scores_ld, void* ws, size_t ws_bytes, misa_stream_t stream);

/* Step 5 -- MISA-dagger fine stage (gist.science summary, "Hierarchische
 * Variant (MISA†)"): the all-head DSA indexer re-scores only the candidate
 * tokens and keeps the final top-k.
 *   cand [T, k_cand] int32 token indices (e.g. the idx of misa_score_topk
 *   run with k = k_cand); entries < 0 are padding and skipped; an entry past
 *   the query's position sets MISA_STATUS_BAD_INPUT and is skipped.
 *   idx [T, k], val [T, k] as in misa_score_topk;  k <= k_cand <= 65536. */
int misa_hier_rerank(const misa_problem_t* p, const uint16_t* q, const float* w,
                     const uint16_t* K, const int32_t* cand, int32_t k_cand, int32_t k,
                     int32_t* idx, float* val, void* ws, size_t ws_bytes, misa_stream_t stream);

/* Head axis x token axis -- routed heads with block pruning.  The heads the
 * router kept (q_r, w_r of misa_route) first score the pooled key blocks,
 *     S[t,b] = sum_{j<m} w_r[t,j] * ReLU(q_r[t,j] . Kbar[b]),
 * over the full blocks b < floor((q_pos[t]+1)/B) of the query's sequence;
 * the n_blocks best blocks by (S desc, block asc) are kept (HISA abstract on
 * the thelatestinai.com papers page: a block-level coarse filter on pooled
 * block representations, then token-level refinement inside the kept
 * blocks; gist.science summary of the MISA paper, "Betekenis en Claims":
 * head-axis routing combines with token-level schemes).  The candidates are
 * the keys of the kept blocks plus the keys floor((q_pos[t]+1)/B)*B ..
 * q_pos[t] of the query's own incomplete block; the routed heads score them
 * (as misa_score_topk does the whole prefix) and the top-k is kept.  A query
 * with fewer than n_blocks full blocks keeps them all, so with n_blocks >=
 * ceil(max_seq_len / B) the result is misa_score_topk's.
 *   q_r [T, m, 128] bf16, w_r [T, m] fp32 (from misa_route); K; Kbar
 *   (misa_pool_keys); m a power of two <= min(64, H);
 *   n_blocks >= 1 with (n_blocks + 1) * B <= 65536;
 *   1 <= k <= (n_blocks + 1) * B;
 *   idx [T, k] int32, val [T, k] fp32 as in misa_score_topk;
 *   blocks: NULL, or [T, n_blocks] int32 receiving the kept block indices
 *   within the sequence (row order unspecified, -1 padding);
 *   ws: misa_block_workspace_size(p, n_blocks) bytes, 256-byte aligned.
 * Five launches on `stream` (block scores, block top-k, candidate
 * expansion, candidate scoring, top-k); no host synchronisation. */
size_t misa_block_workspace_size(const misa_problem_t* p, int32_t n_blocks);
int misa_block_score_topk(const misa_problem_t* p, const uint16_t* q_r, const float* w_r,
                          int32_t m, const uint16_t* K, const float* Kbar, int32_t n_blocks,
                          int32_t k, int32_t* idx, float* val, int32_t* blocks, void* ws,
                          size_t ws_bytes, misa_stream_t stream);

/* The dense DSA indexer, the in-run comparison (MISA abstract; gist.science
 * summary, "Probleemstelling"): every head scores every prefix token.
 *     I[t,s] = sum_{h<H} w[t,h] * ReLU(q[t,h] . K[s])
 * Same outputs as misa_score_topk; H must be a power of two. */
int dsa_index_dense(const misa_problem_t* p, const uint16_t* q, const float* w,
                    const uint16_t* K, int32_t k, int32_t* idx, float* val, float* scores_dbg,
                    int64_t scores_ld, void* ws, size_t ws_bytes, misa_stream_t stream);

/* Synchronises `stream`, returns the status word of the current device in
 * *device_status (may be NULL) and clears it.  Returns MISA_OK when the word
 * was zero, else the MISA_ERR_DEVICE_* code of its lowest set bit;
 * MISA_ERR_CUDA if the synchronisation itself failed. */
int misa_stream_status(misa_stream_t stream, int32_t* device_status);

/* Diagnostic: launches one CTA whose bounded wait on a barrier that nothing
 * arrives on runs out after `wait_ms` milliseconds (1..5000); the kernel then
 * sets MISA_STATUS_TIMEOUT and returns.  Used to test that a timed-out wait
 * leaves the context usable.  No counterpart in the paper. */
int misa_selftest_timeout(int32_t wait_ms, misa_stream_t stream);

/* Tracing.  While enabled (on != 0), every kernel the library launches from
 * the calling host thread is bracketed by CUDA events recorded on its launch
 * stream.  misa_profile_collect synchronises those events and returns, per
 * traced name (names: max_kernels x 32 chars), the summed device time in
 * milliseconds and the number of kernels launched under it (one per name,
 * except "plan_groups" for plans of more than 256 query groups: a scan and a
 * fill), then clears the record.  Returns the
 * number of kernel names (at most max_kernels) or a negative MISA_ERR code.
 * Names starting with '#' are counters, not kernels (time 0, the count in
 * `launches`): "#rescan_queries" sums, over the streaming top-k calls traced,
 * the queries whose sampled threshold did not hold and were rescanned.
 * While tracing, each such call also queues a 4-byte device-to-host copy
 * into pinned host memory the library keeps for this purpose.
 * No counterpart in the paper. */
int misa_profile_enable(int32_t on);
int misa_profile_collect(int32_t max_kernels, char* names, double* total_ms, int64_t* launches);

/* Message of the last failed call on this host thread ("" if none). */
const char* misa_last_error_string(void);

#ifdef __cplusplus
}
#endif

#endif /* MISA_H_ */
