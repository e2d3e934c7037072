// Flat DSA indexer (dsa_flat_select): exact top-k over every causal key.
//
// idea.jsleekr.com, section "DSA: 딥시크의 희소 어텐션": each query scores every
// earlier key with a light dot product and keeps the best few.  Ordering, tie
// rule and output layout are the ones of hisa_select, and token scores use the
// same fp32 evaluation, so HISA with every block selected reproduces these rows.
//
// Schedule (the score matrix is never materialised):
//   1. key_norm_kernel: per sequence the largest key norm |k|max, so that every
//      score of query q lies in [-R, R] with R = |q| |k|max (Cauchy-Schwarz).
//   2. dsa_filter_tc_kernel (dsa_tc.cu): two threads per query, 128 queries per
//      CTA, scores on the tensor cores.  Pass 1 histograms the scores (of every key
//      block, or of every eighth for long tiles) into linear buckets over [-R, R]
//      (bucket 0 = highest) and picks the bucket b* that holds the k-th best score
//      (or an estimate of a threshold a little under it).  Pass 2 recomputes the
//      scores and appends every candidate in buckets <= b* to the query's candidate
//      list.  Bucketing is monotone in the score, so with at least k entries the
//      list is a superset of the top-k whatever the rounding.
//   3. dsa_select_kernel: exact top-k of each candidate list (shared routine).
//   4. dsa_fallback_kernel: a row whose list overflowed its capacity or came out
//      short (a sampled threshold set too high), or whose boundary holds heavy ties,
//      is redone exactly from a full score row in scratch memory.
#include "prof.cuh"
#include "select.cuh"

namespace hisa {

constexpr int DSA_Q = 128;   // queries per filter CTA
constexpr int DSA_SEL_THREADS = 256;
constexpr int DSA_SEL_KPT = 16;  // candidate lists hold at most 256 * 16 keys
constexpr int DSA_FB_CTAS = 64;

__global__ void __launch_bounds__(256)
key_norm_kernel(const uint16_t *__restrict__ k, const int32_t *__restrict__ cu_k,
                const int32_t *__restrict__ seqlens, float *__restrict__ kmax) {
  const int s = blockIdx.y;
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  const int start = cu_k[s], cap = cu_k[s + 1] - start;
  const int len = seqlens ? seqlens[s] : cap;
  if (start % BLK != 0 || len < 0 || len > cap) return;  // reported by the filter
  float nrm = 0.f;
  if (j < len) {
    const uint4 *p = reinterpret_cast<const uint4 *>(k + (size_t)(start + j) * D);
    float acc = 0.f;
#pragma unroll
    for (int c = 0; c < 8; c++) {
      uint4 w = __ldg(p + c);
      uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int u = 0; u < 4; u++) {
        float a = bf_lo(ws[u]), b = bf_hi(ws[u]);
        acc = fmaf(a, a, acc);
        acc = fmaf(b, b, acc);
      }
    }
    nrm = sqrtf(acc);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) nrm = fmaxf(nrm, __shfl_xor_sync(0xffffffffu, nrm, o));
  if ((threadIdx.x & 31) == 0 && nrm > 0.f) atomicMax(reinterpret_cast<int *>(kmax + s), __float_as_int(nrm));
}

// Output index of list entry c: the key position stored beside its score.
struct ListTok {
  const int32_t *bj;
  __device__ int operator()(int c) const { return bj[c]; }
};

struct DirectOut {
  int32_t *idx;
  float *scores;
  __device__ void operator()(int r, int c, uint32_t u) const {
    idx[r] = c;
    if (scores) scores[r] = key_score(u);
  }
};

struct DsaPad {
  int32_t *idx;
  float *scores;
  __device__ void operator()(int r) const {
    idx[r] = -1;
    if (scores) scores[r] = 0.f;
  }
};

__host__ __device__ inline size_t dsa_select_smem(int topk) {
  return sl_work_bytes(topk) + sizeof(SlShared);
}

__global__ void __launch_bounds__(DSA_SEL_THREADS)
dsa_select_kernel(int row0, int topk, int cap, const float *__restrict__ buf_key,
                  const int32_t *__restrict__ buf_j, int32_t *__restrict__ cnt,
                  int32_t *__restrict__ out_idx, float *__restrict__ out_scores) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int local = blockIdx.x, row = row0 + local;
  const int n = cnt[local];
  if (n > cap) return;  // the fallback kernel owns this row
  SlShared &sh = *reinterpret_cast<SlShared *>(smem + sl_work_bytes(topk));
  int32_t *oi = out_idx + (size_t)row * topk;
  float *os = out_scores ? out_scores + (size_t)row * topk : nullptr;
  const RowScores src{buf_key + (size_t)local * cap};
  RegCands<DSA_SEL_THREADS, DSA_SEL_KPT> cs;
  float mx, mn;
  cs.load(src, n, mx, mn);
  // the lists are not in token order, so heavy ties at the boundary (the radix route,
  // which breaks ties by list position) are left to the fallback kernel, launched next
  if (!select_topk_lin<DSA_SEL_THREADS, false>(cs, mx, mn, src, n, topk, sh, smem,
                                               ListTok{buf_j + (size_t)local * cap}, oi, os) &&
      threadIdx.x == 0)
    cnt[local] = cap + 1;
}

__global__ void __launch_bounds__(DSA_SEL_THREADS)
dsa_fallback_kernel(const uint16_t *__restrict__ q, const uint16_t *__restrict__ k,
                    const int32_t *__restrict__ cu_q, const int32_t *__restrict__ cu_k,
                    const int32_t *__restrict__ seqlens, int S, int row0, int nrows, int topk,
                    int cap, const int32_t *__restrict__ cnt, uint32_t *scratch,
                    size_t scratch_stride, int32_t *__restrict__ out_idx,
                    float *__restrict__ out_scores, int *status) {
  extern __shared__ __align__(16) uint8_t smem[];
  uint32_t *sel_key = reinterpret_cast<uint32_t *>(smem);
  int *sel_c = reinterpret_cast<int *>(smem + (size_t)4 * topk);
  uint32_t *tmp_key = reinterpret_cast<uint32_t *>(smem + (size_t)8 * topk);
  int *tmp_c = reinterpret_cast<int *>(smem + (size_t)12 * topk);
  SelectShared &sh = *reinterpret_cast<SelectShared *>(smem + (size_t)16 * topk);
  uint32_t *keys = scratch + (size_t)blockIdx.x * scratch_stride;
  __shared__ int ovf[DSA_SEL_THREADS];
  __shared__ int novf;
  // rows are checked DSA_SEL_THREADS at a time (one per thread) and the overflowing
  // ones, usually none, are then taken one after another by the whole CTA
  for (int base = blockIdx.x * DSA_SEL_THREADS; base < nrows;
       base += gridDim.x * DSA_SEL_THREADS) {
    if (threadIdx.x == 0) novf = 0;
    __syncthreads();
    {
      const int local = base + threadIdx.x;
      if (local < nrows && cnt[local] > cap) ovf[atomicAdd(&novf, 1)] = local;
    }
    __syncthreads();
    const int nov = novf;
    for (int e = 0; e < nov; e++) {
      const int local = ovf[e];
      const int row = row0 + local;
      const QueryInfo qi = locate(cu_q, cu_k, seqlens, S, row, nullptr);
      if (!qi.ok) continue;  // uniform: every thread sees the same row
      if ((size_t)qi.pos + 1 > scratch_stride) {  // max_seqlen_k understated by the caller
        if (threadIdx.x == 0) raise_status(status, HISA_ERR_INVALID_ARG);
        continue;
      }
      QRegs qr;
      load_q(qr, q + (size_t)row * D);
      const uint4 *kseq = reinterpret_cast<const uint4 *>(k + (size_t)qi.kbase * D);
      for (int j = threadIdx.x; j <= qi.pos; j += DSA_SEL_THREADS) {
        uint4 w[8];
#pragma unroll
        for (int c = 0; c < 8; c++) w[c] = __ldg(kseq + (size_t)j * 8 + c);
        keys[j] = score_key(token_score(qr, w));
      }
      __syncthreads();
      int32_t *oi = out_idx + (size_t)row * topk;
      float *os = out_scores ? out_scores + (size_t)row * topk : nullptr;
      select_topk<DSA_SEL_THREADS>([&](int c) { return keys[c]; }, qi.pos + 1, topk, sh, sel_key,
                                   sel_c, tmp_key, tmp_c, DirectOut{oi, os}, DsaPad{oi, os});
    }
    __syncthreads();
  }
}

// ---------------------------------------------------------------------------
// host side

struct DsaPlan {
  int cap;        // candidate-list capacity per row
  int chunk;      // rows per filter/select round
  size_t off_kmax, off_cnt, off_key, off_j, off_fb, total;
};

static size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

DsaPlan dsa_plan(int total_q, int num_seqs, int max_seqlen_k, int topk) {
  DsaPlan p;
  p.cap = (topk + 2048 + 3) & ~3;  // rows stay 16-byte aligned; at most 4096 entries
  // keep the candidate lists to about 8 GiB (one round covers 262144 queries at k = 2048)
  long long chunk = (8ll << 30) / ((long long)p.cap * 8);
  chunk = chunk < DSA_Q ? DSA_Q : chunk;
  chunk = chunk > total_q ? total_q : chunk;
  p.chunk = (int)(chunk < 1 ? 1 : chunk);
  size_t off = 0;
  p.off_kmax = off;
  off = align256(off + (size_t)(num_seqs > 0 ? num_seqs : 1) * 4);
  p.off_cnt = off;
  off = align256(off + (size_t)p.chunk * 4);
  p.off_key = off;
  off = align256(off + (size_t)p.chunk * p.cap * 4);
  p.off_j = off;
  off = align256(off + (size_t)p.chunk * p.cap * 4);
  p.off_fb = off;
  off = align256(off + (size_t)DSA_FB_CTAS * (size_t)(max_seqlen_k > 0 ? max_seqlen_k : 1) * 4);
  p.total = off;
  return p;
}

cudaError_t launch_dsa_filter_tc(const uint16_t *q, const uint16_t *k, const int32_t *cu_q,
                                 const int32_t *cu_k, const int32_t *seqlens, int S, int total_q,
                                 int row0, int nrows, int topk, int cap, const float *kmax,
                                 float *buf_key, int32_t *buf_j, int32_t *cnt, int *status,
                                 cudaStream_t st);

cudaError_t launch_dsa(const uint16_t *q, const uint16_t *k, const int32_t *cu_q,
                       const int32_t *cu_k, const int32_t *seqlens, int S, int total_q,
                       int max_seqlen_k, int topk, int32_t *out_idx, float *out_scores,
                       uint8_t *ws, int *status, cudaStream_t st) {
  if (total_q == 0) return cudaSuccess;
  const DsaPlan p = dsa_plan(total_q, S, max_seqlen_k, topk);
  float *kmax = reinterpret_cast<float *>(ws + p.off_kmax);
  int32_t *cnt = reinterpret_cast<int32_t *>(ws + p.off_cnt);
  float *bkey = reinterpret_cast<float *>(ws + p.off_key);
  int32_t *bj = reinterpret_cast<int32_t *>(ws + p.off_j);
  uint32_t *fb = reinterpret_cast<uint32_t *>(ws + p.off_fb);
  cudaError_t e = cudaMemsetAsync(kmax, 0, (size_t)S * 4, st);
  if (e != cudaSuccess) return e;
  if (max_seqlen_k > 0) {
    ProfScope ps(K_KEY_NORM, st);
    key_norm_kernel<<<dim3((max_seqlen_k + 255) / 256, S), 256, 0, st>>>(k, cu_k, seqlens, kmax);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  const size_t ssm = dsa_select_smem(topk);
  const size_t bsm = (size_t)16 * topk + sizeof(SelectShared);
  static std::atomic<int> attr_s[64], attr_b[64];
  if ((e = set_smem_once((const void *)dsa_select_kernel, ssm, attr_s)) != cudaSuccess) return e;
  if ((e = set_smem_once((const void *)dsa_fallback_kernel, bsm, attr_b)) != cudaSuccess) return e;
  for (int row0 = 0; row0 < total_q; row0 += p.chunk) {
    const int nrows = min(p.chunk, total_q - row0);
    e = launch_dsa_filter_tc(q, k, cu_q, cu_k, seqlens, S, total_q, row0, nrows, topk, p.cap, kmax,
                             bkey, bj, cnt, status, st);
    if (e != cudaSuccess) return e;
    {
      ProfScope ps(K_DSA_SELECT, st);
      dsa_select_kernel<<<nrows, DSA_SEL_THREADS, ssm, st>>>(row0, topk, p.cap, bkey, bj, cnt,
                                                              out_idx, out_scores);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    {
      ProfScope ps(K_DSA_FALLBACK, st);
      dsa_fallback_kernel<<<DSA_FB_CTAS, DSA_SEL_THREADS, bsm, st>>>(
          q, k, cu_q, cu_k, seqlens, S, row0, nrows, topk, p.cap, cnt, fb,
          (size_t)(max_seqlen_k > 0 ? max_seqlen_k : 1), out_idx, out_scores, status);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

size_t dsa_workspace_bytes(int total_q, int num_seqs, int max_seqlen_k, int topk) {
  return dsa_plan(total_q, num_seqs, max_seqlen_k, topk).total;
}

}  // namespace hisa
