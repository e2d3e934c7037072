// The sparse attention step that consumes the selected indices (hisa_sparse_attention).
//
// HISA summary page (aitrends.kr), paragraph on keeping the DSA output structure:
// the top-k token indices go unchanged to the sparse attention operator, which
// attends only to the selected tokens.  Arithmetic (the textbook scaled dot-product
// attention restricted to the selection): for query row i and head h,
//   s_j = scale * q[i][h] . k_att[j],  o[i][h] = sum_j softmax(s)_j v_att[j],
//   lse[i][h] = log sum_j exp(s_j),
// over the entries j >= 0 of the index row; the heads of a query share its selection
// and one key row and one value row per token (the single latent KV head of MLA).
//
// The index row is split over the C CTAs of a cluster (C = 8 when there are too few
// queries to fill the GPU, else 1).  Each CTA walks its share in tiles of 32 tokens:
// the tiles' key and value rows are gathered into shared memory by a double-buffered
// cp.async ring (rows padded to 272 bytes so that lanes reading different rows hit
// different banks), warp w scores heads w, w + 8, ... for the 32 tokens (lane = token),
// keeps a running maximum and sum per head (online softmax), and the 256 threads
// accumulate the output rows (head, 8 dims each).  The C partial results are merged
// through distributed shared memory: CTA c finishes the heads h with h % C == c.
#include <cooperative_groups.h>

#include "common.cuh"
#include "prof.cuh"

namespace cg = cooperative_groups;

namespace hisa {

constexpr int SA_DV = HISA_ATT_DIM;   // 128
constexpr int SA_THREADS = 256;
constexpr int SA_WARPS = SA_THREADS / 32;
constexpr int SA_TILE = 32;            // tokens per tile
constexpr int SA_MAXH = HISA_ATT_MAX_HEADS;
constexpr int SA_ROWB = SA_DV * 2 + 16;  // padded shared-memory row (272 bytes)
constexpr int SA_MAX_CLUSTER = 8;

struct SaSmem {
  float q[SA_MAXH][SA_DV];                 // the query's heads, fp32
  uint8_t kt[2][SA_TILE * SA_ROWB];        // key rows of the tile (ring of two)
  uint8_t vt[2][SA_TILE * SA_ROWB];        // value rows of the tile
  float p[SA_MAXH][SA_TILE];               // scores, then probabilities
  int tok[2][SA_TILE];                     // token positions of the tile (-1 = none)
  float m[SA_MAXH], l[SA_MAXH], alpha[SA_MAXH];
  float opart[SA_MAXH][SA_DV];             // this CTA's unnormalised output (cluster merge)
  int bad;
};

__device__ __forceinline__ void sa_cp16(void *smem, const void *gmem) {
  const unsigned s = (unsigned)__cvta_generic_to_shared(smem);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gmem) : "memory");
}

__global__ void __launch_bounds__(SA_THREADS, 1)
sparse_attn_kernel(const uint16_t *__restrict__ q, const uint16_t *__restrict__ kv_k,
                   const uint16_t *__restrict__ kv_v, const int32_t *__restrict__ idx,
                   const int32_t *__restrict__ cu_q, const int32_t *__restrict__ cu_k, int S,
                   int H, int topk, int per_cta, float scale, float *__restrict__ out,
                   float *__restrict__ lse, int *status) {
  extern __shared__ __align__(16) uint8_t sa_raw[];
  SaSmem &sm = *reinterpret_cast<SaSmem *>(sa_raw);
  cg::cluster_group cl = cg::this_cluster();
  const int C = (int)cl.num_blocks();
  const int me = (int)cl.block_rank();
  const int row = blockIdx.x / C;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const float NEG = -__int_as_float(0x7f800000);

  // the query's sequence (every CTA of the cluster finds the same one)
  const int s = find_seq(cu_q, S, row);
  const int kbase = __ldg(cu_k + s), kcap = __ldg(cu_k + s + 1) - kbase;
  // the query's heads, fp32
  for (int i = tid; i < H * SA_DV; i += SA_THREADS)
    sm.q[i / SA_DV][i % SA_DV] = __uint_as_float((uint32_t)__ldg(q + (size_t)row * H * SA_DV + i) << 16);
  if (tid < H) {
    sm.m[tid] = NEG;
    sm.l[tid] = 0.f;
  }
  if (tid == 0) sm.bad = 0;

  const int e0 = me * per_cta, e1 = min(topk, e0 + per_cta);
  const int ntiles = e1 > e0 ? (e1 - e0 + SA_TILE - 1) / SA_TILE : 0;
  const int32_t *irow = idx + (size_t)row * topk;
  auto gather = [&](int t, int buf) {  // tile t into ring slot buf
    const int base = e0 + t * SA_TILE;
    if (tid < SA_TILE) {
      int j = base + tid < e1 ? __ldg(irow + base + tid) : -1;
      if (j >= kcap) {  // outside the sequence's key region: not attended, reported
        sm.bad = 1;
        j = -1;
      }
      sm.tok[buf][tid] = j;
    }
    __syncthreads();
    // 32 rows x 16 pieces of 16 bytes, for keys and for values
    for (int x = tid; x < SA_TILE * 16; x += SA_THREADS) {
      const int r = x >> 4, c = x & 15;
      const int j = sm.tok[buf][r];
      if (j >= 0) {
        sa_cp16(sm.kt[buf] + r * SA_ROWB + c * 16, kv_k + (size_t)(kbase + j) * SA_DV + c * 8);
        sa_cp16(sm.vt[buf] + r * SA_ROWB + c * 16, kv_v + (size_t)(kbase + j) * SA_DV + c * 8);
      }
    }
    asm volatile("cp.async.commit_group;\n" ::: "memory");
  };

  // output accumulators: thread handles (head, 8 dims) pairs hg = tid, tid + 256
  float oacc[2][8];
#pragma unroll
  for (int a = 0; a < 2; a++)
#pragma unroll
    for (int d = 0; d < 8; d++) oacc[a][d] = 0.f;

  __syncthreads();
  if (ntiles > 0) gather(0, 0);
  for (int t = 0; t < ntiles; t++) {
    const int buf = t & 1;
    if (t + 1 < ntiles) {
      gather(t + 1, buf ^ 1);
      asm volatile("cp.async.wait_group 1;\n" ::: "memory");
    } else {
      asm volatile("cp.async.wait_group 0;\n" ::: "memory");
    }
    __syncthreads();
    // scores: warp w, heads w, w + 8, ...; lane = token of the tile
    {
      const int j = sm.tok[buf][lane];
      const uint8_t *kr = sm.kt[buf] + lane * SA_ROWB;
      for (int h = warp; h < H; h += SA_WARPS) {
        float acc = 0.f;
        if (j >= 0) {
#pragma unroll 4
          for (int c = 0; c < 16; c++) {
            const uint4 w = *reinterpret_cast<const uint4 *>(kr + c * 16);
            const float4 qa = *reinterpret_cast<const float4 *>(&sm.q[h][c * 8]);
            const float4 qb = *reinterpret_cast<const float4 *>(&sm.q[h][c * 8 + 4]);
            acc = fmaf(qa.x, bf_lo(w.x), acc);
            acc = fmaf(qa.y, bf_hi(w.x), acc);
            acc = fmaf(qa.z, bf_lo(w.y), acc);
            acc = fmaf(qa.w, bf_hi(w.y), acc);
            acc = fmaf(qb.x, bf_lo(w.z), acc);
            acc = fmaf(qb.y, bf_hi(w.z), acc);
            acc = fmaf(qb.z, bf_lo(w.w), acc);
            acc = fmaf(qb.w, bf_hi(w.w), acc);
          }
        }
        const float sc = j >= 0 ? acc * scale : NEG;
        // online softmax for head h over this tile
        float tmax = sc;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, o));
        const float m_old = sm.m[h];
        const float m_new = fmaxf(m_old, tmax);
        const float pj = (j >= 0) ? expf(sc - m_new) : 0.f;
        float psum = pj;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) psum += __shfl_xor_sync(0xffffffffu, psum, o);
        sm.p[h][lane] = pj;
        __syncwarp();
        if (lane == 0) {
          const float a = (m_new == NEG) ? 1.f : expf(m_old - m_new);  // m_old = -inf gives 0
          sm.alpha[h] = a;
          sm.l[h] = sm.l[h] * a + psum;
          sm.m[h] = m_new;
        }
      }
    }
    __syncthreads();
    // output rows: rescale, then add the tile's weighted values
#pragma unroll
    for (int a = 0; a < 2; a++) {
      const int hg = tid + a * SA_THREADS;
      if (hg < H * 16) {
        const int h = hg >> 4, dg = hg & 15;
        const float al = sm.alpha[h];
#pragma unroll
        for (int d = 0; d < 8; d++) oacc[a][d] *= al;
        for (int r = 0; r < SA_TILE; r++) {
          const float pr = sm.p[h][r];
          if (pr != 0.f) {
            const uint4 w = *reinterpret_cast<const uint4 *>(sm.vt[buf] + r * SA_ROWB + dg * 16);
            oacc[a][0] = fmaf(pr, bf_lo(w.x), oacc[a][0]);
            oacc[a][1] = fmaf(pr, bf_hi(w.x), oacc[a][1]);
            oacc[a][2] = fmaf(pr, bf_lo(w.y), oacc[a][2]);
            oacc[a][3] = fmaf(pr, bf_hi(w.y), oacc[a][3]);
            oacc[a][4] = fmaf(pr, bf_lo(w.z), oacc[a][4]);
            oacc[a][5] = fmaf(pr, bf_hi(w.z), oacc[a][5]);
            oacc[a][6] = fmaf(pr, bf_lo(w.w), oacc[a][6]);
            oacc[a][7] = fmaf(pr, bf_hi(w.w), oacc[a][7]);
          }
        }
      }
    }
    __syncthreads();  // the ring slot is refilled by the next iteration's gather
  }
  if (tid == 0 && sm.bad) raise_status(status, HISA_ERR_INVALID_ARG);

  // merge: this CTA's partial output into shared memory, then CTA c finishes heads
  // h % C == c from every CTA's (max, sum, partial output)
#pragma unroll
  for (int a = 0; a < 2; a++) {
    const int hg = tid + a * SA_THREADS;
    if (hg < H * 16) {
      const int h = hg >> 4, dg = hg & 15;
#pragma unroll
      for (int d = 0; d < 8; d++) sm.opart[h][dg * 8 + d] = oacc[a][d];
    }
  }
  cl.sync();
  for (int h = me; h < H; h += C) {
    float M = NEG;
    for (int c = 0; c < C; c++) M = fmaxf(M, cl.map_shared_rank(&sm.m[0], c)[h]);
    float L = 0.f;
    for (int c = 0; c < C; c++) {
      const float mc = cl.map_shared_rank(&sm.m[0], c)[h];
      if (mc != NEG) L += expf(mc - M) * cl.map_shared_rank(&sm.l[0], c)[h];
    }
    float *orow = out + ((size_t)row * H + h) * SA_DV;
    for (int d = tid; d < SA_DV; d += SA_THREADS) {
      float acc = 0.f;
      for (int c = 0; c < C; c++) {
        const float mc = cl.map_shared_rank(&sm.m[0], c)[h];
        if (mc != NEG) acc += expf(mc - M) * cl.map_shared_rank(&sm.opart[0][0], c)[h * SA_DV + d];
      }
      orow[d] = L > 0.f ? acc / L : 0.f;
    }
    if (lse && tid == 0) lse[(size_t)row * H + h] = L > 0.f ? M + logf(L) : NEG;
  }
  cl.sync();  // every CTA's shared memory stays readable until the merge is done
}

cudaError_t launch_sparse_attention(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                                    const int32_t *idx, const int32_t *cu_q, const int32_t *cu_k,
                                    int S, int total_q, int H, int topk, float scale, float *out,
                                    float *lse, int num_sms, int *status, cudaStream_t st) {
  if (total_q == 0) return cudaSuccess;
  static int attr[64];
  cudaError_t e = set_smem_once((const void *)sparse_attn_kernel, sizeof(SaSmem), attr);
  if (e != cudaSuccess) return e;
  int C = 1;
  while (C < SA_MAX_CLUSTER && total_q * C < 2 * num_sms) C *= 2;
  int per = (topk + C - 1) / C;
  per = (per + SA_TILE - 1) / SA_TILE * SA_TILE;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(total_q * C);
  cfg.blockDim = dim3(SA_THREADS);
  cfg.dynamicSmemBytes = sizeof(SaSmem);
  cfg.stream = st;
  cudaLaunchAttribute attrs[1];
  attrs[0].id = cudaLaunchAttributeClusterDimension;
  attrs[0].val.clusterDim.x = C;
  attrs[0].val.clusterDim.y = 1;
  attrs[0].val.clusterDim.z = 1;
  cfg.attrs = attrs;
  cfg.numAttrs = 1;
  ProfScope ps(K_SPARSE_ATTENTION, st);
  return cudaLaunchKernelEx(&cfg, sparse_attn_kernel, q, k, v, idx, cu_q, cu_k, S, H, topk, per,
                            scale, out, lse, status);
}

}  // namespace hisa
