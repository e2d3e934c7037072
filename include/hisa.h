/*
 * hisa.h — C ABI of the B200 (sm_100a) HISA token-selection indexer.
 *
 * Hierarchical indexed sparse attention (HISA) replaces the flat DeepSeek-style
 * (DSA) indexer of a sparse-attention layer.  The method, as summarised on
 * aitrends.kr, "HISA: 세밀한 희소 어텐션을 위한 효율적인 계층적 인덱싱":
 *   - block partition and mean pooling: the index keys of a sequence form
 *     contiguous blocks of B tokens; each block is represented by the mean of
 *     its keys (paragraph on block partition and pooling);
 *   - stage 1: each query scores every block representative with a dot
 *     product, blocks wholly after the query are masked, the first block and
 *     the last two blocks are always kept, and the top-m blocks survive
 *     (paragraph on stage 1);
 *   - stage 2: only the tokens of the surviving blocks are scored with the
 *     original DSA dot product and the top-k token indices are emitted in the
 *     layout the sparse attention operator consumes (paragraph on stage 2, and
 *     the paragraph on keeping the DSA output structure);
 *   - the representatives can be maintained as keys are appended to the KV
 *     cache (paragraph on KV-cache maintenance).
 * The flat DSA scan (idea.jsleekr.com, "긴 컨텍스트 LLM이 느려지는 이유와 희소
 * 어텐션(sparse attention)으로 해결하는 방법", section "DSA: 딥시크의 희소 어텐션")
 * scores every earlier key and keeps the top-k; it is provided for comparison
 * and as the m = M identity (HISA with every block selected is the flat scan).
 *
 * Readings of points the pages leave open (fixed by this library):
 *   - "last two blocks" are the query's own block and the block before it; the
 *     forced blocks count inside m; when at most m blocks are eligible all of
 *     them are selected; with m < 3 forced blocks are kept in the order own,
 *     previous, first;
 *   - the token score is the single-head dot product q.k over d = 64 index
 *     dimensions, accumulated in fp32;
 *   - every output row is ordered by score descending; equal scores go to the
 *     lower index (stage 1: lower block, stage 2: lower token); rows with fewer
 *     than k candidates are padded with -1; -0.0 and +0.0 compare equal;
 *   - indices are positions local to their sequence.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *   - Every array argument is a caller-owned DEVICE pointer; the library never
 *     allocates, frees or keeps a pointer after the call returns.  Scratch comes
 *     from a caller workspace sized by the matching *_workspace_size function.
 *   - Calls are asynchronous on the caller's stream (a cudaStream_t passed as
 *     void*; NULL = the legacy default stream) and never synchronise the host.
 *   - Entry points may be called from several host threads at once: a call keeps
 *     its state in its arguments and the library's per-device lookups are atomic.
 *     The exceptions are noted where they apply (hisa_select_noalloc shares one
 *     scratch array; event timing is not thread-safe, launch counting is).
 *   - The first call of any entry point on a device looks up the addresses of the
 *     library's device-resident words on that device (the status word and the
 *     scratch array of hisa_select_noalloc), with that device current.  Make that
 *     first call before any stream capture on the device; later calls may be
 *     captured in CUDA graphs.
 *   - Every call returns a hisa_status; nothing throws across the ABI.
 *     Argument errors visible on the host are returned directly and nothing is
 *     launched.  Errors that only the device can see (a region start that is
 *     not a multiple of B, lengths that do not fit their region, an append past
 *     the region's capacity, a wait that timed out) are OR-ed into a sticky
 *     per-device status word, read with hisa_device_status(); the rows or
 *     sequences concerned are skipped (their output rows are filled with -1).
 *   - bf16 values are passed as their 16-bit patterns (hisa_bf16).
 *   - Row-major layouts; q/k rows are d = 64 bf16 (128 bytes); every pointer
 *     must be 16-byte aligned (HISA_ERR_UNALIGNED otherwise).
 *   - The GPU path is built for d = HISA_INDEX_DIM (64) and B = HISA_BLOCK (128);
 *     any other B is rejected with HISA_ERR_INVALID_ARG.
 *
 * Sequence layout (prefill, decode and packed varlen alike)
 * ----------------------------------------------------------
 *   cu_seqlens_k  int32 [num_seqs+1]: sequence s owns key rows
 *                 [cu_seqlens_k[s], cu_seqlens_k[s+1]) of k_idx (its "region");
 *                 region starts must be multiples of B, so blocks never cross
 *                 sequences and the representative of the block holding key row
 *                 r is row r / B of reps.
 *   seqlens_k     int32 [num_seqs] or NULL: live key count of each sequence;
 *                 NULL means the whole region is live.
 *   cu_seqlens_q  int32 [num_seqs+1]: sequence s owns query rows
 *                 [cu_seqlens_q[s], cu_seqlens_q[s+1]) of q_idx; they are the
 *                 LAST q_len_s positions of the sequence (query r sits at
 *                 position len_s - q_len_s + r).  Prefill: q_len = len; decode:
 *                 q_len = 1.
 *   total_q       = cu_seqlens_q[num_seqs] (host copy, sizes the grids).
 *   max_seqlen_k  >= every live length (host copy, sizes the grids).
 */
#ifndef HISA_H_
#define HISA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define HISA_INDEX_DIM 64
#define HISA_BLOCK 128
#define HISA_MAX_M 512      /* largest block budget m (m * B <= 65536 candidates per query) */
#define HISA_MAX_TOPK 2048  /* largest k accepted by hisa_select / dsa_flat_select */

typedef uint16_t hisa_bf16;  /* bf16 bit pattern */
typedef void *hisa_stream_t; /* cudaStream_t */

typedef enum {
  HISA_OK = 0,
  HISA_ERR_INVALID_ARG = 1,    /* bad size, count, B, m or k; inconsistent lengths */
  HISA_ERR_UNALIGNED = 2,      /* pointer not 16-byte aligned, region start not a multiple of B */
  HISA_ERR_WORKSPACE = 3,      /* workspace missing or smaller than *_workspace_size() */
  HISA_ERR_CUDA = 4,           /* a CUDA runtime call failed (launch, attribute, copy) */
  HISA_ERR_TIMEOUT = 5,        /* a bounded device-side wait gave up */
  HISA_ERR_NOT_IMPLEMENTED = 6,
  HISA_ERR_CAPACITY = 7        /* hisa_append_keys would write past a region's end */
} hisa_status;

/* Text for a status code (static storage; never NULL). */
const char *hisa_status_string(hisa_status s);

/* Library version (major*10000 + minor*100 + patch). */
int hisa_version(void);

/*
 * hisa_pool_blocks — mean-pool the index keys of every sequence into one
 * representative per block of B tokens (HISA summary page, paragraph on block
 * partition and mean pooling).
 *
 *   k_idx         bf16 [rows_k, 64]; rows_k = cu_seqlens_k[num_seqs].
 *   reps (out)    fp32 [ceil(rows_k / B), 64]; row r/B receives the mean of the
 *                 live keys of the block containing key row r.  A partial last
 *                 block (len not a multiple of B) is divided by the number of
 *                 keys present.  Rows of blocks with no live key are untouched.
 * The sum runs over the block's keys in increasing row order in fp32 and is then
 * divided (round to nearest) by the count; hisa_append_keys uses the same order,
 * so representatives maintained incrementally are bit-identical to a re-pool.
 */
hisa_status hisa_pool_blocks(const hisa_bf16 *k_idx, const int32_t *cu_seqlens_k,
                             const int32_t *seqlens_k, int num_seqs, int max_seqlen_k, int B,
                             float *reps, hisa_stream_t stream);

/*
 * hisa_append_keys — decode-time KV-cache update (HISA summary page, paragraph
 * on maintaining representatives at KV-cache update time).
 *
 *   k_cache (in/out)   bf16 [rows_k, 64]; new rows are written at region row
 *                      seqlens_k[s] .. seqlens_k[s] + n_new - 1 of sequence s.
 *   reps (in/out)      fp32 [rows_k / B, 64]; every block touched by the new keys
 *                      is re-pooled (same order and rounding as hisa_pool_blocks).
 *   cu_seqlens_k       int32 [num_seqs+1] region starts; a region's size is its
 *                      capacity.
 *   seqlens_k (in/out) int32 [num_seqs] live lengths, incremented by n_new on the
 *                      device.
 *   new_keys           bf16 [num_seqs, n_new, 64].
 * A sequence whose region cannot take n_new more keys is left unchanged and
 * HISA_ERR_CAPACITY is raised in the device status word.
 */
hisa_status hisa_append_keys(hisa_bf16 *k_cache, float *reps, const int32_t *cu_seqlens_k,
                             int32_t *seqlens_k, const hisa_bf16 *new_keys, int n_new,
                             int num_seqs, int B, hisa_stream_t stream);

/*
 * hisa_select — the HISA indexer: stage 1 (block scores and top-m) followed by
 * stage 2 (scores of the tokens of the selected blocks and top-k).
 *
 *   q_idx          bf16 [total_q, 64] index queries.
 *   k_idx          bf16 [rows_k, 64] index keys (the same buffer that was pooled).
 *   reps           fp32 [rows_k / B, 64] block representatives (hisa_pool_blocks /
 *                  hisa_append_keys).
 *   m              blocks kept per query, 1 <= m <= HISA_MAX_M.  Blocks 0, the own
 *                  block and the previous block are forced and count inside m;
 *                  if the query sees at most m blocks, all are kept.
 *   k              tokens kept per query, 1 <= k <= HISA_MAX_TOPK.  m*B < k is
 *                  accepted (rows are then padded with -1).
 *   out_idx (out)  int32 [total_q, k]: sequence-local token positions j <= i of
 *                  the selected tokens, by score descending (ties: lower j), -1
 *                  padded.
 *   out_scores     fp32 [total_q, k] or NULL: the scores of out_idx (0 where -1).
 *   out_blocks     int32 [total_q, m] or NULL: the selected blocks (sequence-local
 *                  block numbers), ascending, -1 padded.
 *   ws, ws_bytes   device workspace of at least hisa_select_workspace_size(...)
 *                  bytes, 256-byte aligned; it must not be used by another call
 *                  that runs at the same time.
 */
hisa_status hisa_select(const hisa_bf16 *q_idx, const hisa_bf16 *k_idx, const float *reps,
                        const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k,
                        const int32_t *seqlens_k, int num_seqs, int total_q, int max_seqlen_k,
                        int B, int m, int k, int32_t *out_idx, float *out_scores,
                        int32_t *out_blocks, void *ws, size_t ws_bytes, hisa_stream_t stream);

size_t hisa_select_workspace_size(int total_q, int num_seqs, int max_seqlen_k, int B, int m,
                                  int k);

/*
 * hisa_decode_step — one decode step of a batch in one launch: the KV-cache update of
 * hisa_append_keys with one new key per sequence (the representative of the block
 * that receives it is refreshed, HISA summary page, paragraph on KV-cache maintenance)
 * and hisa_select for one query per sequence, placed at the new key's position.  The
 * outputs, the cache, the representatives and the lengths equal those of
 * hisa_append_keys(n_new = 1) followed by hisa_select with cu_seqlens_q = 0, 1, ...,
 * num_seqs, bit for bit.
 *
 *   k_cache, reps, cu_seqlens_k, seqlens_k (in/out)   as in hisa_append_keys.
 *   new_keys       bf16 [num_seqs, 64]: the key appended to each sequence.
 *   q_idx          bf16 [num_seqs, 64]: the query of each sequence.
 *   max_seqlen_k   >= every length after the append; at most 8192 blocks (the
 *                  few-query path), else HISA_ERR_NOT_IMPLEMENTED.
 *   m, k, out_idx, out_scores, out_blocks   as in hisa_select (m <= 128 here).
 * A sequence whose region cannot take one more key is left unchanged, its row is
 * written as -1 and HISA_ERR_CAPACITY is raised in the device status word.  No
 * workspace.
 */
hisa_status hisa_decode_step(hisa_bf16 *k_cache, float *reps, const int32_t *cu_seqlens_k,
                             int32_t *seqlens_k, const hisa_bf16 *new_keys,
                             const hisa_bf16 *q_idx, int num_seqs, int max_seqlen_k, int B, int m,
                             int k, int32_t *out_idx, float *out_scores, int32_t *out_blocks,
                             hisa_stream_t stream);

/*
 * hisa_select_varm — hisa_select with a block budget per sequence.  The pages mention
 * a fractional setting ("HISA 50%") and adaptive sparsity (idea.jsleekr.com summary
 * and its transcript) without defining them; this library reads them as a block
 * budget m_s per sequence, typically m_s = ceil(f * M_s) for a sequence of M_s blocks
 * (hisa_fraction_blocks computes that on the device).
 *
 *   m_seq          int32 [num_seqs] (device): the budget of every sequence,
 *                  1 <= m_seq[s] <= m_max.  A value outside that range is clamped
 *                  and raises HISA_ERR_INVALID_ARG in the device status word.
 *   m_max          largest budget, 1 <= m_max <= HISA_MAX_M; the row stride of
 *                  out_blocks (entries past a row's budget are -1) and the m of the
 *                  workspace size: hisa_select_workspace_size(..., m_max, k).
 * Every other argument, the output and the errors are those of hisa_select; a
 * sequence's rows equal those hisa_select gives that sequence alone with m = m_s.
 * Budgets above 128 take a slower select that reads each score row from memory
 * three times; the few-query cluster path takes budgets up to 128.
 */
hisa_status hisa_select_varm(const hisa_bf16 *q_idx, const hisa_bf16 *k_idx, const float *reps,
                             const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k,
                             const int32_t *seqlens_k, const int32_t *m_seq, int num_seqs,
                             int total_q, int max_seqlen_k, int B, int m_max, int k,
                             int32_t *out_idx, float *out_scores, int32_t *out_blocks, void *ws,
                             size_t ws_bytes, hisa_stream_t stream);

/*
 * hisa_fraction_blocks — m_seq[s] = min(m_max, max(1, ceil(f * ceil(len_s / B)))) for
 * every sequence, on the device (len_s = seqlens_k[s], or the region size when
 * seqlens_k is NULL), for hisa_select_varm.  0 < f <= 1, 1 <= m_max <= HISA_MAX_M.
 * A live length that does not fit its region raises HISA_ERR_INVALID_ARG in the
 * device status word (its budget is set to 1).
 */
hisa_status hisa_fraction_blocks(const int32_t *cu_seqlens_k, const int32_t *seqlens_k,
                                 int num_seqs, int B, double f, int m_max, int32_t *m_seq,
                                 hisa_stream_t stream);

/*
 * hisa_block_sparse_select — stage 1 on its own: the block-sparse selection HISA is
 * compared with in the Needle-in-a-Haystack paragraph of the HISA summary page.  The
 * m blocks of every query are chosen exactly as in hisa_select (block scores, causal
 * mask, forced blocks, top-m), and every token j <= i of them is emitted; no token is
 * scored.  With m * B = k this is the block-sparse baseline at the same token budget.
 *
 *   q_idx, reps, cu_seqlens_*, seqlens_k, num_seqs, total_q, max_seqlen_k, B, m:
 *                  as in hisa_select (no key rows are read).
 *   out_idx (out)  int32 [total_q, m * B]: the tokens of the selected blocks in
 *                  ascending order, -1 padded (the tail of the query's own block and
 *                  the slots of missing blocks).
 *   out_blocks     int32 [total_q, m] or NULL: the selected blocks, ascending.
 *   ws, ws_bytes   device workspace of at least hisa_block_sparse_workspace_size(...)
 *                  bytes, 256-byte aligned.
 */
hisa_status hisa_block_sparse_select(const hisa_bf16 *q_idx, const float *reps,
                                     const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k,
                                     const int32_t *seqlens_k, int num_seqs, int total_q,
                                     int max_seqlen_k, int B, int m, int32_t *out_idx,
                                     int32_t *out_blocks, void *ws, size_t ws_bytes,
                                     hisa_stream_t stream);

size_t hisa_block_sparse_workspace_size(int total_q, int num_seqs, int max_seqlen_k, int B,
                                        int m);

/*
 * dsa_flat_select — the flat DSA indexer: every causal key j <= i of the query's
 * sequence is scored with q.k and the top-k are emitted with the same ordering,
 * padding and layout as hisa_select (idea.jsleekr.com, section "DSA: 딥시크의
 * 희소 어텐션").  Token scores are computed with the same fp32 arithmetic as
 * hisa_select's stage 2, so hisa_select with m >= the number of blocks returns
 * exactly the rows of this function.
 *
 *   ws, ws_bytes   device workspace of at least dsa_flat_workspace_size(...) bytes.
 */
hisa_status dsa_flat_select(const hisa_bf16 *q_idx, const hisa_bf16 *k_idx,
                            const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k,
                            const int32_t *seqlens_k, int num_seqs, int total_q,
                            int max_seqlen_k, int k, int32_t *out_idx, float *out_scores,
                            void *ws, size_t ws_bytes, hisa_stream_t stream);

size_t dsa_flat_workspace_size(int total_q, int num_seqs, int max_seqlen_k, int k);

/*
 * hisa_sparse_attention — the sparse attention step that consumes the selected
 * indices (HISA summary page, paragraph on keeping the DSA output structure: the
 * top-k token indices go unchanged to the sparse attention operator, which attends
 * only to the selected tokens).  The pages name the operator without writing out its
 * arithmetic; this library computes the textbook scaled dot-product attention
 * restricted to the selection, with the heads of a query sharing its selection and
 * one key row and one value row per token shared by every head (one latent KV head,
 * as in multi-head latent attention):
 *   s_j       = scale * q_att[i][h] . k_att[j]        for the entries j >= 0 of topk_idx[i]
 *   out[i][h] = sum_j softmax(s)_j * v_att[j]          (fp32 accumulation)
 *   lse[i][h] = log sum_j exp(s_j)                     (-inf for a row with no index)
 *
 *   q_att        bf16 [total_q, num_heads, HISA_ATT_DIM]
 *   k_att, v_att bf16 [rows_k, HISA_ATT_DIM]: sequence s owns rows
 *                [cu_seqlens_k[s], cu_seqlens_k[s+1]) (the indexer's key regions).
 *   topk_idx     int32 [total_q, k]: sequence-local token positions, -1 = none (the
 *                out_idx of hisa_select or dsa_flat_select).  A position outside the
 *                sequence's region is ignored and HISA_ERR_INVALID_ARG is raised in
 *                the device status word.
 *   out (out)    fp32 [total_q, num_heads, HISA_ATT_DIM]; rows with no index are 0.
 *   lse (out)    fp32 [total_q, num_heads] or NULL.
 * 1 <= num_heads <= HISA_ATT_MAX_HEADS.  No workspace; q_att, k_att and v_att must be
 * 16-byte aligned.
 * Precision: the dot products are exact bf16 products summed in fp32 (tensor cores);
 * the softmax weights use the fast exponential and enter the value product as bf16
 * hi + lo (about 16 significant bits); sums and the output accumulate in fp32.
 * Errors: a null pointer, num_heads outside [1, HISA_ATT_MAX_HEADS] or k < 1 returns
 * HISA_ERR_INVALID_ARG and a misaligned pointer HISA_ERR_UNALIGNED, before any
 * launch; a launch failure returns HISA_ERR_CUDA; a device-side wait that times out (it should not) raises
 * HISA_ERR_TIMEOUT in the device status word and the call still completes.
 */
#define HISA_ATT_DIM 128
#define HISA_ATT_MAX_HEADS 32
hisa_status hisa_sparse_attention(const hisa_bf16 *q_att, const hisa_bf16 *k_att,
                                  const hisa_bf16 *v_att, const int32_t *topk_idx,
                                  const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k,
                                  int num_seqs, int total_q, int num_heads, int k, float scale,
                                  float *out, float *lse, hisa_stream_t stream);

/*
 * hisa_device_status — wait for `stream`, then copy the sticky device status word
 * of the current device into *status (0 = no device-side error; otherwise the
 * OR of (1 << hisa_status) bits).  clear != 0 resets the word afterwards.
 * Meant for tests and debugging: it synchronises the stream.
 */
hisa_status hisa_device_status(int32_t *status, int clear, hisa_stream_t stream);

/*
 * hisa_select_noalloc — hisa_select without a workspace (the pages have no
 * counterpart; it exists for callers of this library that cannot allocate).
 *
 * Some callers cannot allocate device memory at the moment they need a
 * selection: a plug-in running inside an inference engine whose memory plan is
 * fixed before it starts, or a latency-critical decode path where a cudaMalloc
 * would synchronise the device.  This entry point takes the same arguments and
 * produces the same outputs as hisa_select, minus ws/ws_bytes: its scratch is a
 * fixed array of HISA_NOALLOC_SCRATCH_BYTES bytes inside the library.  It calls
 * no cudaMalloc, cudaFree or other allocating routine.
 *
 *   - The array exists once per device and every device that loads the library
 *     holds it until the process exits.
 *   - Batches of fewer than twice as many queries as the GPU has SMs (decode) whose
 *     sequences hold at most 8192 blocks (1M tokens) and whose m is at most 128 run
 *     on a path that needs no scratch at all.  Other batches need the scratch
 *     hisa_select_workspace_size() reports for the same arguments (about
 *     m * 516 bytes per query plus the block-score matrix), and problems whose
 *     scratch exceeds HISA_NOALLOC_SCRATCH_BYTES are rejected with
 *     HISA_ERR_WORKSPACE before anything is launched.
 *   - Every call shares the array and it keeps the last call's contents; nothing
 *     in it needs to start at zero.  Calls whose kernels overlap on the GPU (on
 *     different streams, or from different host threads) race on the array and
 *     give wrong results: order them on one stream or serialise them.
 *   - The array's device address is looked up by the first call of any entry point
 *     on a device (see the shared conventions above).
 *   - Inputs, outputs, ordering, errors and the device status word are those of
 *     hisa_select.
 */
#define HISA_NOALLOC_SCRATCH_BYTES (16u << 20)
hisa_status hisa_select_noalloc(const hisa_bf16 *q_idx, const hisa_bf16 *k_idx, const float *reps,
                                const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k,
                                const int32_t *seqlens_k, int num_seqs, int total_q,
                                int max_seqlen_k, int B, int m, int k, int32_t *out_idx,
                                float *out_scores, int32_t *out_blocks, hisa_stream_t stream);

/*
 * hisa_test_fault — for tests of the timeout path only (no counterpart on the pages).
 * mode 1: the tensor-core token-scoring launches made from now on issue no loads, so
 * that their bounded waits (about one second) run out with no copy and no MMA in
 * flight; the launch then raises HISA_ERR_TIMEOUT in the device status word and
 * every row of that hisa_select call is written as -1 (scores 0).  mode 0: normal
 * operation (the default).  Process-wide, not thread-safe; returns
 * HISA_ERR_INVALID_ARG for any other mode.
 */
hisa_status hisa_test_fault(int mode);

/*
 * Launch accounting, for benchmarks and tests (no counterpart on the pages).
 * Every kernel launch made by this library is counted per kernel kind (atomic
 * counters).  With timing enabled, each launch is also bracketed by a pair of CUDA
 * events recorded on its launch stream: host-side state shared by all callers of
 * the process, not thread-safe; leave timing off while capturing a CUDA graph.
 *
 * hisa_timing_enable  — turn event timing on (1) or off (0).
 * hisa_kernel_kinds   — number of kernel kinds; hisa_kernel_name(i) names kind i.
 * hisa_timing_collect — wait for every recorded event, then write per kind the
 *                       total event time in ms (ms[i]), the launches counted
 *                       (launches[i]) and the launches timed (timed[i]) since the
 *                       last reset, for i < n; any of the arrays may be NULL.
 *                       reset != 0 zeroes the counters afterwards.
 */
hisa_status hisa_timing_enable(int on);
int hisa_kernel_kinds(void);
const char *hisa_kernel_name(int kind);
hisa_status hisa_timing_collect(double *ms, long long *launches, long long *timed, int n,
                                int reset);

#ifdef __cplusplus
}
#endif

#endif /* HISA_H_ */
