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

// shared memory of the selecting kernel: work (4k words) | LinShared | the block list |
// the score segments of the blocks
__host__ __device__ inline size_t token_smem_bytes(int m, int topk) {
  return (size_t)16 * topk + sizeof(LinShared) + (size_t)m * 8;
}

__global__ void __launch_bounds__(TS_THREADS)
token_score_split_kernel(const uint16_t *__restrict__ q, const uint16_t *__restrict__ k,
                         const int32_t *__restrict__ cu_q, const int32_t *__restrict__ cu_k,
                         const int32_t *__restrict__ seqlens, int S, int m,
                         const int32_t *__restrict__ blk, int slots_per_cta,
                         float *__restrict__ scratch) {
  __shared__ __align__(16) uint8_t stage[STAGE_ROWS * ROW_BYTES];
  const int row = blockIdx.x;
  const QueryInfo qi = locate(cu_q, cu_k, seqlens, S, row, nullptr);
  if (!qi.ok) return;
  const int32_t *blkrow = blk + (size_t)row * m;
  const int nsel = min(m, qi.pos / BLK + 1);  // the block stage keeps exactly this many
  const int s0 = blockIdx.y * slots_per_cta, s1 = min(nsel, s0 + slots_per_cta);
  if (s0 >= s1) return;
  QRegs qr;
  load_q(qr, q + (size_t)row * D);
  float *dst = scratch + (size_t)row * m * BLK;
  score_slots(qr, k + (size_t)qi.kbase * D, qi.pos, blkrow, s0, s1, stage,
              [&](int c, float sc) { dst[c] = sc; });
}

// One CTA per query: exact top-k of the query's score row.  NT threads hold KPT
// candidates each (NT * KPT >= m * 128).
template <int NT, int KPT>
__global__ void __launch_bounds__(NT, 1024 / NT)
token_select_scratch_kernel(const int32_t *__restrict__ cu_q, const int32_t *__restrict__ cu_k,
                            const int32_t *__restrict__ seqlens, int S, int m, int topk,
                            const int32_t *__restrict__ blk, const float *__restrict__ scratch,
                            const int32_t *__restrict__ pmap, int32_t *__restrict__ out_idx,
                            float *__restrict__ out_scores) {
  extern __shared__ __align__(16) uint8_t smem[];
  uint32_t *work = reinterpret_cast<uint32_t *>(smem);
  LinShared &sh = *reinterpret_cast<LinShared *>(smem + (size_t)16 * topk);
  int32_t *sblk = reinterpret_cast<int32_t *>(smem + (size_t)16 * topk + sizeof(LinShared));
  int32_t *sseg = sblk + m;
  const int row = blockIdx.x;
  RowPad pad{out_idx + (size_t)row * topk, out_scores ? out_scores + (size_t)row * topk : nullptr};
  const QueryInfo qi = locate(cu_q, cu_k, seqlens, S, row, nullptr);
  if (!qi.ok) {
    for (int r = threadIdx.x; r < topk; r += NT) pad(r);
    return;
  }
  // the block stage keeps exactly min(m, own block + 1) blocks of a valid query
  const int nsel = min(m, qi.pos / BLK + 1);
  for (int i = threadIdx.x; i < nsel; i += NT) {
    sblk[i] = blk[(size_t)row * m + i];
    if (pmap) sseg[i] = pmap[(size_t)row * m + i];
  }
  __syncthreads();
  TokenOut out{pad.idx, pad.scores, sblk};
  if (pmap)  // scores of slot i in segment sseg[i] of the buffer
    select_topk_reg<NT, KPT>(SegScores{scratch, sseg}, nsel * BLK, topk, sh, work, out, pad);
  else       // one contiguous score row per query
    select_topk_reg<NT, KPT>(RowScores{scratch + (size_t)row * m * BLK}, nsel * BLK, topk, sh,
                             work, out, pad);
}

// Tensor-core schedule when there are enough queries to fill the GPU with tiles;
// otherwise (decode) the split CUDA-core schedule.
bool use_tc_path(int total_q, int num_sms) { return total_q >= 2 * num_sms; }
static bool token_use_split(int total_q, int num_sms) { return !use_tc_path(total_q, num_sms); }

size_t tc_workspace_bytes(int total_q, int num_seqs, int max_seqlen_k, int m);
size_t block_tc_workspace_bytes(int total_q, int num_seqs, int max_seqlen_k);
cudaError_t launch_token_score_tc(const uint16_t *q, const uint16_t *k, const int32_t *cu_q,
                                  const int32_t *cu_k, const int32_t *seqlens, int S,
                                  int total_q, int max_seqlen_k, int m, const int32_t *blk,
                                  uint8_t *ws, float **scores_out, const int32_t **pmap_out,
                                  int num_sms, int *status, cudaStream_t st);

size_t token_scratch_bytes(int total_q, int num_seqs, int max_seqlen_k, int m, int num_sms) {
  if (token_use_split(total_q, num_sms)) return (size_t)total_q * m * BLK * 4;
  // the block-score matrix is dead before the token stage writes its lists and rows
  const size_t a = tc_workspace_bytes(total_q, num_seqs, max_seqlen_k, m);
  const size_t b = block_tc_workspace_bytes(total_q, num_seqs, max_seqlen_k);
  return a > b ? a : b;
}

cudaError_t launch_token_select(const uint16_t *q, const uint16_t *k, const int32_t *cu_q,
                                const int32_t *cu_k, const int32_t *seqlens, int S, int total_q,
                                int max_seqlen_k, int m, int topk, const int32_t *blk,
                                uint8_t *ws, int num_sms, int32_t *out_idx, float *out_scores,
                                int *status, cudaStream_t st) {
  if (total_q == 0) return cudaSuccess;
  cudaError_t e;
  float *scores = reinterpret_cast<float *>(ws);
  const int32_t *pmap = nullptr;  // contiguous score rows unless the tensor-core path maps them
  if (token_use_split(total_q, num_sms)) {
    // spread each query's blocks over enough CTAs to cover the SMs about twice
    int splits = (2 * num_sms + total_q - 1) / total_q;
    splits = splits < 1 ? 1 : (splits > m ? m : splits);
    int slots = (m + splits - 1) / splits;
    slots = (slots + 1) & ~1;  // whole staging rounds
    splits = (m + slots - 1) / slots;
    {
      ProfScope ps(K_TOKEN_SCORE_SPLIT, st);
      token_score_split_kernel<<<dim3(total_q, splits), TS_THREADS, 0, st>>>(
          q, k, cu_q, cu_k, seqlens, S, m, blk, slots, scores);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  } else {
    e = launch_token_score_tc(q, k, cu_q, cu_k, seqlens, S, total_q, max_seqlen_k, m, blk, ws,
                              &scores, &pmap, num_sms, status, st);
    if (e != cudaSuccess) return e;
  }
  const size_t smem = token_smem_bytes(m, topk);
  if (token_use_split(total_q, num_sms)) {
    // few queries: a wider CTA per query shortens each selection
    static std::atomic<int> attr_c[64], attr_d[64];
    if (m * BLK <= 1024 * 8) {
      auto kern = token_select_scratch_kernel<1024, 8>;
      if ((e = set_smem_once((const void *)kern, smem, attr_c)) != cudaSuccess) return e;
      ProfScope ps(K_TOKEN_SELECT_SCRATCH, st);
      kern<<<total_q, 1024, smem, st>>>(cu_q, cu_k, seqlens, S, m, topk, blk, scores, pmap,
                                        out_idx, out_scores);
    } else {
      auto kern = token_select_scratch_kernel<1024, 16>;
      if ((e = set_smem_once((const void *)kern, smem, attr_d)) != cudaSuccess) return e;
      ProfScope ps(K_TOKEN_SELECT_SCRATCH, st);
      kern<<<total_q, 1024, smem, st>>>(cu_q, cu_k, seqlens, S, m, topk, blk, scores, pmap,
                                        out_idx, out_scores);
    }
  } else if (m * BLK <= 256 * 32) {
    static std::atomic<int> attr_a[64];
    auto kern = token_select_scratch_kernel<256, 32>;
    if ((e = set_smem_once((const void *)kern, smem, attr_a)) != cudaSuccess) return e;
    ProfScope ps(K_TOKEN_SELECT_SCRATCH, st);
    kern<<<total_q, 256, smem, st>>>(cu_q, cu_k, seqlens, S, m, topk, blk, scores, pmap,
                                     out_idx, out_scores);
  } else {
    static std::atomic<int> attr_b[64];
    auto kern = token_select_scratch_kernel<512, 32>;
    if ((e = set_smem_once((const void *)kern, smem, attr_b)) != cudaSuccess) return e;
    ProfScope ps(K_TOKEN_SELECT_SCRATCH, st);
    kern<<<total_q, 512, smem, st>>>(cu_q, cu_k, seqlens, S, m, topk, blk, scores, pmap,
                                     out_idx, out_scores);
  }
  return cudaGetLastError();
}

}  // namespace hisa
