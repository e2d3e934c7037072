// Stage 2 of HISA: gather-score the tokens of the selected blocks and keep the top-k.
//
// HISA summary page (aitrends.kr), paragraph on stage 2: only the tokens inside
// the m selected blocks are scored with the original DSA dot product, and the k
// best token indices go to the sparse attention operator (the output keeps the
// DSA layout, paragraph on KV-cache maintenance and compatibility).
//
// Candidate c of a query is token j = blk[c / 128] * 128 + c % 128 of the query's
// sequence; blocks are listed in ascending order, so candidate order is token
// order.  The token causal mask admits j <= i.
//
// Two schedules produce each query's score row (order-preserving keys, candidate
// order) in workspace memory; one CTA per query then selects from it:
//   * many queries (prefill): the block-major tensor-core path of token_tc.cu;
//   * few queries (decode): the selected blocks of each query are split over several
//     CTAs that stage them through shared memory (cp.async, XOR-swizzled 16-byte
//     chunks, so each thread reads its own key row without bank conflicts) and score
//     them on the CUDA cores -- a memory-bound stream with no reuse to exploit.
#include "prof.cuh"
#include "select.cuh"

namespace hisa {

constexpr int TS_THREADS = 256;
constexpr int STAGE_ROWS = 256;  // two blocks per staging round

__device__ __forceinline__ void cp_async16(void *smem, const void *gmem) {
  unsigned s = (unsigned)__cvta_generic_to_shared(smem);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit_wait() {
  asm volatile("cp.async.commit_group;\n" ::: "memory");
  asm volatile("cp.async.wait_all;\n" ::: "memory");
}

// Scores selected-block slots [s0, s1) of one query; dst(candidate, raw score), -inf
// for a key after the query.
template <class Dst>
__device__ __forceinline__ void score_slots(const QRegs &q, const uint16_t *kseq, int pos,
                                            const int32_t *blkrow, int s0, int s1,
                                            uint8_t *stage, Dst dst) {
  const int tid = threadIdx.x;
  for (int p = s0; p < s1; p += 2) {
    const int nb2 = min(2, s1 - p);
    for (int i = tid; i < nb2 * BLK * 8; i += TS_THREADS) {
      const int r = i >> 3, c = i & 7;
      const int j = blkrow[p + (r >> 7)] * BLK + (r & 127);
      if (j <= pos)
        cp_async16(stage + r * ROW_BYTES + ((c ^ (r & 7)) << 4), kseq + (size_t)j * D + c * 8);
    }
    cp_async_commit_wait();
    __syncthreads();
    if (tid < nb2 * BLK) {
      const int r = tid;
      const int j = blkrow[p + (r >> 7)] * BLK + (r & 127);
      float sc = -__int_as_float(0x7f800000);
      if (j <= pos) {
        uint4 w[8];
#pragma unroll
        for (int c = 0; c < 8; c++)
          w[c] = *reinterpret_cast<const uint4 *>(stage + r * ROW_BYTES + ((c ^ (r & 7)) << 4));
        sc = token_score(q, w);
      }
      dst((p << 7) + r, sc);
    }
    __syncthreads();
  }
}

// Output index of candidate c: token blkrow[c / 128] * 128 + c % 128 of the sequence.
struct BlockTok {
  const int32_t *blkrow;
  __device__ int operator()(int c) const { return blkrow[c >> 7] * BLK + (c & 127); }
};

// shared memory of the selecting kernel: select working bytes | SlShared | the block
// list | the score segments of the blocks
__host__ __device__ inline size_t token_smem_bytes(int m, int topk) {
  return sl_work_bytes(topk) + sizeof(SlShared) + (size_t)m * 8;
}
__host__ __device__ inline size_t token_reg_smem_bytes(int m, int topk) {
  return (size_t)16 * topk + sizeof(LinShared) + (size_t)m * 8;
}

__global__ void __launch_bounds__(TS_THREADS)
token_score_split_kernel(const uint16_t *__restrict__ q, const uint16_t *__restrict__ k,
                         const int32_t *__restrict__ cu_q, const int32_t *__restrict__ cu_k,
                         const int32_t *__restrict__ seqlens, const int32_t *__restrict__ m_seq,
                         int S, int m, const int32_t *__restrict__ blk, int slots_per_cta,
                         float *__restrict__ scratch) {
  __shared__ __align__(16) uint8_t stage[STAGE_ROWS * ROW_BYTES];
  const int row = blockIdx.x;
  const QueryInfo qi = locate(cu_q, cu_k, seqlens, S, row, nullptr);
  if (!qi.ok) return;
  const int32_t *blkrow = blk + (size_t)row * m;
  // the block stage keeps exactly this many
  const int nsel = min(seq_budget(m_seq, qi.seq, m, nullptr), qi.pos / BLK + 1);
  const int s0 = blockIdx.y * slots_per_cta, s1 = min(nsel, s0 + slots_per_cta);
  if (s0 >= s1) return;
  QRegs qr;
  load_q(qr, q + (size_t)row * D);
  float *dst = scratch + (size_t)row * m * BLK;
  score_slots(qr, k + (size_t)qi.kbase * D, qi.pos, blkrow, s0, s1, stage,
              [&](int c, float sc) { dst[c] = sc; });
}

// Rows of the selecting kernels: locate the query, pad an invalid row, stage its
// selected blocks (and their score segments) in shared memory.  Returns the number of
// candidates (0 when the row is done).
template <int NT>
__device__ __forceinline__ int select_row_setup(const int32_t *cu_q, const int32_t *cu_k,
                                                const int32_t *seqlens, const int32_t *m_seq,
                                                int S, int m, int topk, const int32_t *blk,
                                                const int32_t *pmap, int list_base,
                                                const int *launch_abort, int row, int32_t *oi,
                                                float *os, int32_t *sblk, int32_t *sseg,
                                                int *pos_out = nullptr) {
  const QueryInfo qi = locate(cu_q, cu_k, seqlens, S, row, nullptr);
  // a scoring launch that gave up a wait left its score rows incomplete: pad every row
  if (!qi.ok || (launch_abort && *launch_abort)) {
    for (int r = threadIdx.x; r < topk; r += NT) {
      oi[r] = -1;
      if (os) os[r] = 0.f;
    }
    return 0;
  }
  // the block stage keeps exactly min(budget, own block + 1) blocks of a valid query
  const int nsel = min(seq_budget(m_seq, qi.seq, m, nullptr), qi.pos / BLK + 1);
  for (int i = threadIdx.x; i < nsel; i += NT) {
    sblk[i] = blk[(size_t)row * m + i];
    if (pmap) sseg[i] = pmap[(size_t)row * m + i] - list_base;  // segment in the chunk buffer
  }
  if (pos_out) *pos_out = qi.pos;
  __syncthreads();
  return nsel * BLK;
}

struct TokenOut {
  int32_t *idx;
  float *scores;
  const int32_t *blkrow;
  __device__ void operator()(int r, int c, uint32_t u) const {
    idx[r] = blkrow[c >> 7] * BLK + (c & 127);
    if (scores) scores[r] = key_score(u);
  }
};

struct RowPad {
  int32_t *idx;
  float *scores;
  __device__ void operator()(int r) const {
    idx[r] = -1;
    if (scores) scores[r] = 0.f;
  }
};

// One CTA per query: exact top-k of the query's score row, KPT candidates per thread
// held in registers (NT * KPT >= m * 128), by select_topk_reg.  pmap non-null: the
// segment of slot i is pmap[row * m + i] - list_base of the score buffer; else the
// row's segments are contiguous.
template <int NT, int KPT>
__global__ void __launch_bounds__(NT, 1024 / NT)
token_select_scratch_kernel(const int32_t *__restrict__ cu_q, const int32_t *__restrict__ cu_k,
                            const int32_t *__restrict__ seqlens, const int32_t *__restrict__ m_seq,
                            int S, int m, int topk, const int32_t *__restrict__ blk,
                            const float *__restrict__ scratch, const int32_t *__restrict__ pmap,
                            int list_base, const int *__restrict__ launch_abort, int row0,
                            int32_t *__restrict__ out_idx, float *__restrict__ out_scores) {
  extern __shared__ __align__(16) uint8_t smem[];
  uint32_t *work = reinterpret_cast<uint32_t *>(smem);
  LinShared &sh = *reinterpret_cast<LinShared *>(smem + (size_t)16 * topk);
  int32_t *sblk = reinterpret_cast<int32_t *>(smem + (size_t)16 * topk + sizeof(LinShared));
  int32_t *sseg = sblk + m;
  const int row = row0 + blockIdx.x;
  int32_t *oi = out_idx + (size_t)row * topk;
  float *os = out_scores ? out_scores + (size_t)row * topk : nullptr;
  const int n = select_row_setup<NT>(cu_q, cu_k, seqlens, m_seq, S, m, topk, blk, pmap,
                                     list_base, launch_abort, row, oi, os, sblk, sseg);
  if (n == 0) return;
  const TokenOut out{oi, os, sblk};
  const RowPad pad{oi, os};
  if (pmap)  // scores of slot i in segment sseg[i] of the buffer
    select_topk_reg<NT, KPT>(SegScores{scratch, sseg}, n, topk, sh, work, out, pad);
  else       // one contiguous score row per query
    select_topk_reg<NT, KPT>(RowScores{scratch + (size_t)row * m * BLK}, n, topk, sh, work, out,
                             pad);
}

// The same for rows longer than the registers hold (m > 128): every pass of the
// select reads the score row again from memory.
template <int NT>
__global__ void __launch_bounds__(NT)
token_select_mem_kernel(const int32_t *__restrict__ cu_q, const int32_t *__restrict__ cu_k,
                        const int32_t *__restrict__ seqlens, const int32_t *__restrict__ m_seq,
                        int S, int m, int topk, const int32_t *__restrict__ blk,
                        const float *__restrict__ scratch, const int32_t *__restrict__ pmap,
                        int list_base, const int *__restrict__ launch_abort, int row0,
                        int32_t *__restrict__ out_idx, float *__restrict__ out_scores) {
  extern __shared__ __align__(16) uint8_t smem[];
  uint8_t *work = smem;
  const size_t wb = sl_work_bytes(topk);
  SlShared &sh = *reinterpret_cast<SlShared *>(smem + wb);
  int32_t *sblk = reinterpret_cast<int32_t *>(smem + wb + sizeof(SlShared));
  int32_t *sseg = sblk + m;
  const int row = row0 + blockIdx.x;
  int32_t *oi = out_idx + (size_t)row * topk;
  float *os = out_scores ? out_scores + (size_t)row * topk : nullptr;
  const int n = select_row_setup<NT>(cu_q, cu_k, seqlens, m_seq, S, m, topk, blk, pmap,
                                     list_base, launch_abort, row, oi, os, sblk, sseg);
  if (n == 0) return;
  float mx, mn;
  if (pmap) {
    const MemCands<NT, SegScores> cs{SegScores{scratch, sseg}, n};
    cs.load(mx, mn);
    select_topk_lin<NT>(cs, mx, mn, cs.sc, n, topk, sh, work, BlockTok{sblk}, oi, os);
  } else {
    const MemCands<NT, RowScores> cs{RowScores{scratch + (size_t)row * m * BLK}, n};
    cs.load(mx, mn);
    select_topk_lin<NT>(cs, mx, mn, cs.sc, n, topk, sh, work, BlockTok{sblk}, oi, os);
  }
}

// Tensor-core schedule when there are enough queries to fill the GPU with tiles;
// otherwise (decode) the split CUDA-core schedule.
bool use_tc_path(int total_q, int num_sms) { return total_q >= 2 * num_sms; }
static bool token_use_split(int total_q, int num_sms) { return !use_tc_path(total_q, num_sms); }

size_t tc_workspace_bytes(int total_q, int num_seqs, int max_seqlen_k, int m);
size_t block_tc_workspace_bytes(int total_q, int num_seqs, int max_seqlen_k);

size_t token_scratch_bytes(int total_q, int num_seqs, int max_seqlen_k, int m, int num_sms) {
  if (token_use_split(total_q, num_sms)) return (size_t)total_q * m * BLK * 4;
  // the block-score matrix is dead before the token stage writes its lists and rows
  const size_t a = tc_workspace_bytes(total_q, num_seqs, max_seqlen_k, m);
  const size_t b = block_tc_workspace_bytes(total_q, num_seqs, max_seqlen_k);
  return a > b ? a : b;
}

template <class Kern>
static cudaError_t launch_select(Kern kern, int nt, size_t smem, std::atomic<int> *attr,
                                 int nrows, cudaStream_t st, const int32_t *cu_q,
                                 const int32_t *cu_k, const int32_t *seqlens,
                                 const int32_t *m_seq, int S, int m, int topk,
                                 const int32_t *blk, const float *scores, const int32_t *pmap,
                                 int list_base, const int *launch_abort, int row0,
                                 int32_t *out_idx, float *out_scores) {
  cudaError_t e = set_smem_once((const void *)kern, smem, attr);
  if (e != cudaSuccess) return e;
  ProfScope ps(K_TOKEN_SELECT_SCRATCH, st);
  kern<<<nrows, nt, smem, st>>>(cu_q, cu_k, seqlens, m_seq, S, m, topk, blk, scores, pmap,
                                list_base, launch_abort, row0, out_idx, out_scores);
  return cudaGetLastError();
}

// The exact select of query rows [row0, row0 + nrows): m is the row stride of blk (the
// largest block budget), m_seq (nullable) the budget of each sequence.  pmap non-null:
// the segment of slot i of a row is pmap[row * m + i] - list_base of `scores`; else
// every row's segments are contiguous (row stride m * 128).  split: few queries
// (wider CTAs).
cudaError_t launch_select_rows(const int32_t *cu_q, const int32_t *cu_k, const int32_t *seqlens,
                               const int32_t *m_seq, int S, int m, int topk, const int32_t *blk,
                               const float *scores, const int32_t *pmap, int list_base,
                               const int *launch_abort, int row0, int nrows, bool split,
                               int32_t *out_idx, float *out_scores, cudaStream_t st) {
  if (nrows <= 0) return cudaSuccess;
#define HISA_SELECT_ARGS nrows, st, cu_q, cu_k, seqlens, m_seq, S, m, topk, blk, scores, pmap, \
                         list_base, launch_abort, row0, out_idx, out_scores
  const int n = m * BLK;
  const size_t smem_reg = token_reg_smem_bytes(m, topk);
  if (split && n <= 1024 * 8) {  // few queries: a wider CTA per query shortens each selection
    static std::atomic<int> attr[64];
    return launch_select(token_select_scratch_kernel<1024, 8>, 1024, smem_reg, attr, HISA_SELECT_ARGS);
  }
  if (split && n <= 1024 * 16) {
    static std::atomic<int> attr[64];
    return launch_select(token_select_scratch_kernel<1024, 16>, 1024, smem_reg, attr, HISA_SELECT_ARGS);
  }
  if (n <= 256 * 32) {
    static std::atomic<int> attr[64];
    return launch_select(token_select_scratch_kernel<256, 32>, 256, smem_reg, attr, HISA_SELECT_ARGS);
  }
  if (n <= 512 * 32) {
    static std::atomic<int> attr[64];
    return launch_select(token_select_scratch_kernel<512, 32>, 512, smem_reg, attr, HISA_SELECT_ARGS);
  }
  {  // m > 128: the score row is read from memory on every pass
    static std::atomic<int> attr[64];
    return launch_select(token_select_mem_kernel<1024>, 1024, token_smem_bytes(m, topk), attr,
                         HISA_SELECT_ARGS);
  }
#undef HISA_SELECT_ARGS
}

cudaError_t launch_token_stage_tc(const uint16_t *q, const uint16_t *k, const int32_t *cu_q,
                                  const int32_t *cu_k, const int32_t *seqlens,
                                  const int32_t *m_seq, int S, int total_q, int max_seqlen_k,
                                  int m, int topk, const int32_t *blk, uint8_t *ws, int num_sms,
                                  int32_t *out_idx, float *out_scores, int *status,
                                  cudaStream_t st);

cudaError_t launch_token_select(const uint16_t *q, const uint16_t *k, const int32_t *cu_q,
                                const int32_t *cu_k, const int32_t *seqlens,
                                const int32_t *m_seq, int S, int total_q, int max_seqlen_k,
                                int m, int topk, const int32_t *blk, uint8_t *ws, int num_sms,
                                int32_t *out_idx, float *out_scores, int *status,
                                cudaStream_t st) {
  if (total_q == 0) return cudaSuccess;
  if (!token_use_split(total_q, num_sms))
    return launch_token_stage_tc(q, k, cu_q, cu_k, seqlens, m_seq, S, total_q, max_seqlen_k, m,
                                 topk, blk, ws, num_sms, out_idx, out_scores, status, st);
  // few queries: spread each query's blocks over enough CTAs to cover the SMs about twice
  float *scores = reinterpret_cast<float *>(ws);
  int splits = (2 * num_sms + total_q - 1) / total_q;
  splits = splits < 1 ? 1 : (splits > m ? m : splits);
  int slots = (m + splits - 1) / splits;
  slots = (slots + 1) & ~1;  // whole staging rounds
  splits = (m + slots - 1) / slots;
  {
    ProfScope ps(K_TOKEN_SCORE_SPLIT, st);
    token_score_split_kernel<<<dim3(total_q, splits), TS_THREADS, 0, st>>>(
        q, k, cu_q, cu_k, seqlens, m_seq, S, m, blk, slots, scores);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_select_rows(cu_q, cu_k, seqlens, m_seq, S, m, topk, blk, scores, nullptr, 0,
                            nullptr, 0, total_q, true, out_idx, out_scores, st);
}

}  // namespace hisa
