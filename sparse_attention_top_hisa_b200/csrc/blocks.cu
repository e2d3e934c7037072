// Stage 1 on its own (the block-sparse baseline) and per-sequence block budgets.
//
// HISA summary page (aitrends.kr), Needle-in-a-Haystack paragraph: HISA is compared
// with a block-sparse selection that keeps whole blocks, chosen by their pooled
// representatives, without the token-level refinement of stage 2.  Here the blocks
// are chosen exactly as stage 1 of HISA chooses them (block scores, causal mask,
// forced blocks, top-m), and every token j <= i of them is emitted in ascending order.
//
// The idea.jsleekr.com summary mentions a fractional setting ("HISA 50%", adaptive
// sparsity) without defining it; this library reads it as a block budget per
// sequence, m_s = ceil(f * M_s) for M_s = ceil(len_s / B) blocks, and computes it on
// the device from the live lengths so that decode steps need no host round trip.
#include "common.cuh"
#include "prof.cuh"

namespace hisa {

constexpr int EXPAND_THREADS = 256;

// One CTA per query row: out[row][s * B + t] = blk[row][s] * B + t when that token lies
// at or before the query, else -1.  The selected blocks are ascending and the query's
// own block (the only one holding tokens after it) is the last one, so every -1
// lies in the row's tail.
__global__ void __launch_bounds__(EXPAND_THREADS)
expand_blocks_kernel(const int32_t *__restrict__ blk, const int32_t *__restrict__ cu_q,
                     const int32_t *__restrict__ cu_k, const int32_t *__restrict__ seqlens, int S,
                     int m, int32_t *__restrict__ out) {
  __shared__ int32_t sblk[HISA_MAX_M];
  __shared__ int pos_sh;
  const int row = blockIdx.x;
  if (threadIdx.x == 0) {
    const QueryInfo qi = locate(cu_q, cu_k, seqlens, S, row, nullptr);  // the block stage reports
    pos_sh = qi.ok ? qi.pos : -1;
  }
  for (int i = threadIdx.x; i < m; i += EXPAND_THREADS) sblk[i] = blk[(size_t)row * m + i];
  __syncthreads();
  const int pos = pos_sh;
  const int width = m * BLK;
  int32_t *dst = out + (size_t)row * width;
  for (int x = threadIdx.x; x < width; x += EXPAND_THREADS) {
    const int b = sblk[x >> 7];
    const int j = b * BLK + (x & 127);
    dst[x] = (pos >= 0 && b >= 0 && j <= pos) ? j : -1;
  }
}

cudaError_t launch_expand_blocks(const int32_t *blk, const int32_t *cu_q, const int32_t *cu_k,
                                 const int32_t *seqlens, int S, int total_q, int m,
                                 int32_t *out, cudaStream_t st) {
  if (total_q == 0) return cudaSuccess;
  ProfScope ps(K_EXPAND_BLOCKS, st);
  expand_blocks_kernel<<<total_q, EXPAND_THREADS, 0, st>>>(blk, cu_q, cu_k, seqlens, S, m, out);
  return cudaGetLastError();
}

// m_seq[s] = min(m_max, max(1, ceil(f * ceil(len_s / B)))).
__global__ void fraction_budget_kernel(const int32_t *__restrict__ cu_k,
                                       const int32_t *__restrict__ seqlens, int S, double f,
                                       int m_max, int32_t *__restrict__ m_seq, int *status) {
  const int s = blockIdx.x * blockDim.x + threadIdx.x;
  if (s >= S) return;
  const int cap = cu_k[s + 1] - cu_k[s];
  const int len = seqlens ? seqlens[s] : cap;
  if (len < 0 || len > cap) {
    raise_status(status, HISA_ERR_INVALID_ARG);
    m_seq[s] = 1;
    return;
  }
  const int M = (len + BLK - 1) / BLK;
  const double want = ceil(f * (double)M);
  m_seq[s] = want < 1.0 ? 1 : (want > (double)m_max ? m_max : (int)want);
}

cudaError_t launch_fraction_budget(const int32_t *cu_k, const int32_t *seqlens, int S, double f,
                                   int m_max, int32_t *m_seq, int *status, cudaStream_t st) {
  if (S == 0) return cudaSuccess;
  ProfScope ps(K_FRACTION_BUDGET, st);
  fraction_budget_kernel<<<(S + 127) / 128, 128, 0, st>>>(cu_k, seqlens, S, f, m_max, m_seq,
                                                         status);
  return cudaGetLastError();
}

}  // namespace hisa
