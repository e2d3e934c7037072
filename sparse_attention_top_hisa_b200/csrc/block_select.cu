// Stage 1 of HISA: block scores and top-m block selection (CUDA-core path).
//
// HISA summary page (aitrends.kr), paragraph on stage 1: the query is scored
// against every block representative with a dot product, blocks lying wholly
// after the query are masked, the first block and the last two blocks (read as
// the query's own block and the one before it) are always kept, and the top-m
// blocks survive.  The forced blocks count inside m; a query that sees at most
// m blocks keeps all of them; ties between block scores go to the lower block.
//
// The scores of the eligible, non-forced blocks become order-preserving keys in
// shared memory (computed on the tensor cores for many queries, on the CUDA cores
// by one CTA per query for few); one warp per query then finds the key of the
// (m - |forced|)-th best block with a 32-step bitwise search, and ballots over
// ascending block numbers resolve ties and emit the selected blocks in order.
#include "block_pick.cuh"
#include "prof.cuh"

namespace hisa {

constexpr int BS_WARPS = 4;

__device__ __forceinline__ float rep_score(const QRegs &q, const float *rep) {
  const float4 *p = reinterpret_cast<const float4 *>(rep);
  float a = 0.f, b = 0.f;
#pragma unroll
  for (int c = 0; c < 8; c++) {
    float4 x = __ldg(p + c);
    float4 y = __ldg(p + c + 8);
    a = fmaf(q.v[4 * c + 0], x.x, a);
    a = fmaf(q.v[4 * c + 1], x.y, a);
    a = fmaf(q.v[4 * c + 2], x.z, a);
    a = fmaf(q.v[4 * c + 3], x.w, a);
    b = fmaf(q.v[32 + 4 * c + 0], y.x, b);
    b = fmaf(q.v[32 + 4 * c + 1], y.y, b);
    b = fmaf(q.v[32 + 4 * c + 2], y.z, b);
    b = fmaf(q.v[32 + 4 * c + 3], y.w, b);
  }
  return a + b;
}

// Common front part of both kernels: locate the query, handle invalid rows and the
// take-all case.  m is the row's block budget, m_max the row stride of dst (entries
// m..m_max-1 are -1).  Returns false when the row is finished.
__device__ __forceinline__ bool block_row_setup(const int32_t *cu_q, const int32_t *cu_k,
                                                const int32_t *seqlens, const int32_t *m_seq,
                                                int S, int row, int m_max, int emax, int32_t *dst,
                                                int32_t *dst2, int *status, QueryInfo &qi,
                                                int &own, int &E, int &m, int lane_id,
                                                int nthreads) {
  qi = locate(cu_q, cu_k, seqlens, S, row, lane_id == 0 ? status : nullptr);
  m = m_max;
  if (!qi.ok) {
    for (int i = lane_id; i < m_max; i += nthreads) {
      dst[i] = -1;
      if (dst2) dst2[i] = -1;
    }
    return false;
  }
  m = seq_budget(m_seq, qi.seq, m_max, lane_id == 0 ? status : nullptr);
  own = qi.pos / BLK;
  E = own + 1;
  if (E > emax) {  // max_seqlen_k understated by the caller
    if (lane_id == 0) raise_status(status, HISA_ERR_INVALID_ARG);
    for (int i = lane_id; i < m_max; i += nthreads) {
      dst[i] = -1;
      if (dst2) dst2[i] = -1;
    }
    return false;
  }
  if (E <= m) {  // every eligible block is kept
    for (int i = lane_id; i < m_max; i += nthreads) {
      const int v = i < E ? i : -1;
      dst[i] = v;
      if (dst2) dst2[i] = v;
    }
    return false;
  }
  for (int i = m + lane_id; i < m_max; i += nthreads) {  // past this row's budget
    dst[i] = -1;
    if (dst2) dst2[i] = -1;
  }
  return true;
}

// Many queries: one warp per query reads the keys computed on the tensor cores.
__global__ void __launch_bounds__(BS_WARPS * 32)
block_select_kernel(const int32_t *__restrict__ cu_q, const int32_t *__restrict__ cu_k,
                    const int32_t *__restrict__ seqlens, const int32_t *__restrict__ m_seq,
                    int S, int total_q, int m_max, int emax,
                    const uint32_t *__restrict__ tc_keys, int tc_stride,
                    int32_t *__restrict__ blk, int32_t *__restrict__ out_blocks,
                    int *status) {
  extern __shared__ uint32_t bs_smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * BS_WARPS + warp;
  if (row >= total_q) return;
  uint32_t *hist = bs_smem + (size_t)warp * 256;
  uint32_t *keys = bs_smem + BS_WARPS * 256 + (size_t)warp * emax;
  int32_t *dst = blk + (size_t)row * m_max;
  int32_t *dst2 = out_blocks ? out_blocks + (size_t)row * m_max : nullptr;
  QueryInfo qi;
  int own, E, m;
  if (!block_row_setup(cu_q, cu_k, seqlens, m_seq, S, row, m_max, emax, dst, dst2, status, qi, own,
                       E, m, lane, 32))
    return;
  const uint32_t *src = tc_keys + (size_t)row * tc_stride;
#pragma unroll
  for (int i = 0; i < 8; i++) hist[lane * 8 + i] = 0u;
  __syncwarp();
  // eight keys per lane are loaded before any is used (the key matrix streams from
  // HBM at long contexts, so one load in flight per lane would leave the warp waiting)
  for (int b0 = lane; b0 < E; b0 += 32 * 8) {
    uint32_t u[8];
#pragma unroll
    for (int j = 0; j < 8; j++) u[j] = b0 + 32 * j < E ? __ldg(src + b0 + 32 * j) : 0u;
#pragma unroll
    for (int j = 0; j < 8; j++) {
      if (b0 + 32 * j < E) {
        keys[b0 + 32 * j] = u[j];
        if (u[j] != 0u) atomicAdd(&hist[u[j] >> 24], 1u);
      }
    }
  }
  __syncwarp();
  warp_select_blocks(keys, E, own, m, dst, dst2, hist, true);
}

// Few queries (decode): one CTA per query scores every eligible block on the CUDA
// cores (one thread per block, all representative rows in flight at once), then warp
// 0 selects.
constexpr int BS_CTA_THREADS = 256;

__global__ void __launch_bounds__(BS_CTA_THREADS)
block_select_cta_kernel(const uint16_t *__restrict__ q, const float *__restrict__ reps,
                        const int32_t *__restrict__ cu_q, const int32_t *__restrict__ cu_k,
                        const int32_t *__restrict__ seqlens, const int32_t *__restrict__ m_seq,
                        int S, int m_max, int emax, int32_t *__restrict__ blk,
                        int32_t *__restrict__ out_blocks, int *status) {
  extern __shared__ uint32_t bsc_smem[];
  const int row = blockIdx.x, tid = threadIdx.x;
  int32_t *dst = blk + (size_t)row * m_max;
  int32_t *dst2 = out_blocks ? out_blocks + (size_t)row * m_max : nullptr;
  QueryInfo qi;
  int own, E, m;
  if (!block_row_setup(cu_q, cu_k, seqlens, m_seq, S, row, m_max, emax, dst, dst2, status, qi,
                       own, E, m, tid, BS_CTA_THREADS))
    return;
  const int nf = min(m, 3);
  QRegs qr;
  load_q(qr, q + (size_t)row * D);
  const float *rbase = reps + (size_t)(qi.kbase / BLK) * D;
  for (int b = tid; b < E; b += BS_CTA_THREADS) {
    const bool forced = b == own || (nf >= 2 && b == own - 1) || (nf >= 3 && b == 0);
    bsc_smem[256 + b] = forced ? 0u : score_key(rep_score(qr, rbase + (size_t)b * D));
  }
  __syncthreads();
  if (tid < 32) warp_select_blocks(bsc_smem + 256, E, own, m, dst, dst2, bsc_smem, false);
}

bool use_tc_path(int total_q, int num_sms);
cudaError_t launch_block_score_tc(const uint16_t *q, const float *reps, const int32_t *cu_q,
                                  const int32_t *cu_k, const int32_t *seqlens,
                                  const int32_t *m_seq, int S, int total_q, int max_seqlen_k,
                                  int m, uint8_t *ws, uint32_t **scores_out, int *status,
                                  cudaStream_t st);
int block_score_stride(int max_seqlen_k);

// Many queries: scores on the tensor cores (block_tc.cu), then one warp per query
// selects.  Few queries (decode): one warp per query scores on the CUDA cores too.
cudaError_t launch_block_select(const uint16_t *q, const float *reps, const int32_t *cu_q,
                                const int32_t *cu_k, const int32_t *seqlens,
                                const int32_t *m_seq, int S, int total_q, int max_seqlen_k,
                                int m, int32_t *blk,
                                int32_t *out_blocks, uint8_t *ws, int num_sms, int *status,
                                cudaStream_t st) {
  if (total_q == 0) return cudaSuccess;
  const uint32_t *tc_keys = nullptr;
  int tc_stride = 0;
  if (use_tc_path(total_q, num_sms)) {
    uint32_t *sc = nullptr;
    cudaError_t e = launch_block_score_tc(q, reps, cu_q, cu_k, seqlens, m_seq, S, total_q,
                                          max_seqlen_k, m, ws, &sc, status, st);
    if (e != cudaSuccess) return e;
    tc_keys = sc;
    tc_stride = block_score_stride(max_seqlen_k);
  }
  const int emax = (max_seqlen_k + BLK - 1) / BLK;
  if (tc_keys) {
    const size_t smem = (size_t)BS_WARPS * (256 + (emax > 0 ? emax : 1)) * sizeof(uint32_t);
    static std::atomic<int> attr[64];
    if (smem > 48 * 1024) {
      cudaError_t e = set_smem_once((const void *)block_select_kernel, smem, attr);
      if (e != cudaSuccess) return e;
    }
    dim3 grid((total_q + BS_WARPS - 1) / BS_WARPS);
    ProfScope ps(K_BLOCK_SELECT, st);
    block_select_kernel<<<grid, BS_WARPS * 32, smem, st>>>(cu_q, cu_k, seqlens, m_seq, S, total_q, m,
                                                         emax > 0 ? emax : 1, tc_keys, tc_stride,
                                                         blk, out_blocks, status);
  } else {
    const size_t smem = (size_t)(256 + (emax > 0 ? emax : 1)) * sizeof(uint32_t);
    static std::atomic<int> attr_cta[64];
    if (smem > 48 * 1024) {
      cudaError_t e = set_smem_once((const void *)block_select_cta_kernel, smem, attr_cta);
      if (e != cudaSuccess) return e;
    }
    ProfScope ps(K_BLOCK_SELECT, st);
    block_select_cta_kernel<<<total_q, BS_CTA_THREADS, smem, st>>>(
        q, reps, cu_q, cu_k, seqlens, m_seq, S, m, emax > 0 ? emax : 1, blk, out_blocks, status);
  }
  return cudaGetLastError();
}

}  // namespace hisa
