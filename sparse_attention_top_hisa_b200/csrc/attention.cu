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
// The index row is split over the C CTAs of a cluster (up to 8 when there are too
// few queries to fill the GPU, else 1); each CTA runs both products of its tiles of
// 128 selected tokens on the tensor cores (below), keeps an online softmax per head,
// and the C partial results are merged through distributed shared memory: CTA c
// finishes the heads h with h % C == c.
#include <cooperative_groups.h>

#include "prof.cuh"
#include "tc.cuh"

namespace cg = cooperative_groups;

namespace hisa {

constexpr int SA_DV = HISA_ATT_DIM;   // 128
constexpr int SA_MAX_CLUSTER = 8;

// ---------------------------------------------------------------------------
// Tensor-core version.  Per tile of 128 selected tokens:
//   S^T [128 tokens x Hp] = K_tile [128 x 128] . Q^T [128 x Hp]     (tcgen05, TMEM cols 0..)
//   O^T [128 dims x Hp]  += V^T [128 x 128 tokens] . P^T [128 x Hp]  (TMEM cols 32..)
// with Hp = the head count rounded up to 16.  Every operand is K-major with the
// 128-byte swizzle (tiles of 64 K-elements, 8-row groups 1024 bytes apart): the key
// tile is gathered with cp.async, the value tile is transposed while it is gathered
// (two tokens' 16-byte pieces become four-byte pairs of eight V^T rows), and the
// probabilities are split into bf16 hi + lo (two MMAs) so that they keep about 16
// bits.  Thread t of the four warps is token t for the scores (online softmax per
// head across the CTA, running maximum and sum in shared memory) and dimension t for
// the output tile, which it folds into fp32 registers rescaled by the tile's factor.

constexpr int AT_THREADS = 128;
constexpr int AT_TILE = 128;                 // tokens per tile
constexpr int AT_NH = 32;                    // head rows of the Q and P operands
constexpr uint32_t AT_TMEM_COLS = 64;        // S^T in cols [0, 32), the O tile in [32, 64)

struct AtSmem {
  uint8_t kt[2 * AT_TILE * 128];   // key tile, two 64-dim atoms of 128 token rows
  uint8_t vt[2 * SA_DV * 128];     // V^T tile, two 64-token atoms of 128 dim rows
  uint8_t qb[2 * AT_NH * 128];     // Q, two 64-dim atoms of 32 head rows
  uint8_t ph[2 * AT_NH * 128];     // P hi, two 64-token atoms of 32 head rows
  uint8_t pl[2 * AT_NH * 128];     // P lo
  int tok[AT_TILE];
  float tmax[4][AT_NH], tsum[4][AT_NH];
  float m[AT_NH], l[AT_NH], alpha[AT_NH], mnew[AT_NH];
  float opart[AT_NH][SA_DV];
  uint64_t bar_mma;
  uint32_t tmem_base;
  int bad;
};
constexpr size_t AT_SMEM = sizeof(AtSmem) + 1024;

// byte offset of element (row, kidx) of a K-major SW128 operand whose 64-element atoms
// hold `rows` rows each
__device__ __forceinline__ uint32_t kmaj_off(int row, int kidx, int rows) {
  return (uint32_t)((kidx >> 6) * rows * 128) + sw128_offset(row, (kidx & 63) >> 3) +
         (uint32_t)((kidx & 7) * 2);
}

__device__ __forceinline__ uint16_t bf16_rn_bits(float x) {
  const uint32_t u = __float_as_uint(x);
  return (uint16_t)((u + 0x7fffu + ((u >> 16) & 1u)) >> 16);  // finite x
}

__global__ void __launch_bounds__(AT_THREADS, 1)
sparse_attn_tc_kernel(const uint16_t *__restrict__ q, const uint16_t *__restrict__ kv_k,
                      const uint16_t *__restrict__ kv_v, const int32_t *__restrict__ idx,
                      const int32_t *__restrict__ cu_q, const int32_t *__restrict__ cu_k, int S,
                      int H, int topk, int per_cta, float scale, float *__restrict__ out,
                      float *__restrict__ lse, int *status) {
  extern __shared__ uint8_t at_raw[];
  AtSmem &sm = *reinterpret_cast<AtSmem *>((reinterpret_cast<uintptr_t>(at_raw) + 1023) &
                                           ~(uintptr_t)1023);
  cg::cluster_group cl = cg::this_cluster();
  const int C = (int)cl.num_blocks();
  const int me = (int)cl.block_rank();
  const int row = blockIdx.x / C;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const float NEG = -__int_as_float(0x7f800000);
  const int Hp = (H + 15) & ~15;

  const int s = find_seq(cu_q, S, row);
  const int kbase = __ldg(cu_k + s), kcap = __ldg(cu_k + s + 1) - kbase;
  if (tid == 0) {
    mbar_init(&sm.bar_mma, 1);
    fence_barrier_init();
    sm.bad = 0;
  }
  if (warp == 0) {
    tmem_alloc(&sm.tmem_base, AT_TMEM_COLS);
    tmem_relinquish();
  }
  // Q (zero rows for padded heads) and zeroed P rows for padded heads
  for (int x = tid; x < AT_NH * 16; x += AT_THREADS) {
    const int h = x >> 4, c = x & 15;
    uint4 w = make_uint4(0u, 0u, 0u, 0u);
    if (h < H) w = __ldg(reinterpret_cast<const uint4 *>(q + ((size_t)row * H + h) * SA_DV) + c);
    *reinterpret_cast<uint4 *>(sm.qb + (c >> 3) * AT_NH * 128 + sw128_offset(h, c & 7)) = w;
    const uint4 z = make_uint4(0u, 0u, 0u, 0u);
    *reinterpret_cast<uint4 *>(sm.ph + (c >> 3) * AT_NH * 128 + sw128_offset(h, c & 7)) = z;
    *reinterpret_cast<uint4 *>(sm.pl + (c >> 3) * AT_NH * 128 + sw128_offset(h, c & 7)) = z;
  }
  if (tid < AT_NH) {
    sm.m[tid] = NEG;
    sm.l[tid] = 0.f;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
  const uint32_t skt = smem_u32(sm.kt), svt = smem_u32(sm.vt), sqb = smem_u32(sm.qb);
  const uint32_t sph = smem_u32(sm.ph), spl = smem_u32(sm.pl);
  const uint32_t id = idesc_bf16_f32(AT_TILE, Hp);

  float oacc[AT_NH];
#pragma unroll
  for (int h = 0; h < AT_NH; h++) oacc[h] = 0.f;

  const int e0 = me * per_cta, e1 = min(topk, e0 + per_cta);
  const int ntiles = e1 > e0 ? (e1 - e0 + AT_TILE - 1) / AT_TILE : 0;
  const int32_t *irow = idx + (size_t)row * topk;
  uint32_t phase = 0;
  for (int t = 0; t < ntiles; t++) {
    const int base = e0 + t * AT_TILE;
    {  // the tile's tokens (-1 = none; outside the region = none, reported)
      int j = base + tid < e1 ? __ldg(irow + base + tid) : -1;
      if (j >= kcap) {
        sm.bad = 1;
        j = -1;
      }
      sm.tok[tid] = j < 0 ? -1 : j;
    }
    __syncthreads();
    // key tile: row r = token, 16 pieces of 8 dims
    for (int x = tid; x < AT_TILE * 16; x += AT_THREADS) {
      const int r = x >> 4, c = x & 15;
      const int j = sm.tok[r];
      if (j >= 0)
        cp_async_16(skt + (c >> 3) * AT_TILE * 128 + sw128_offset(r, c & 7),
                    kv_k + (size_t)(kbase + j) * SA_DV + c * 8);
    }
    cp_async_commit();
    // V^T tile: token pair (2p, 2p + 1) x 8 dims -> eight 4-byte pairs, zeros for none.
    // Lanes take consecutive pairs of one 8-dim piece: a warp's stores to a V^T row
    // then cover 32 distinct banks (8 swizzled 16-byte chunks x 4 pairs).
#pragma unroll 2
    for (int x = tid; x < (AT_TILE / 2) * 16; x += AT_THREADS) {
      const int pr = x & 63, c = x >> 6;
      const int t0 = 2 * pr;
      const int j0 = sm.tok[t0], j1 = sm.tok[t0 + 1];
      uint4 a = make_uint4(0u, 0u, 0u, 0u), b = a;
      if (j0 >= 0) a = __ldg(reinterpret_cast<const uint4 *>(kv_v + (size_t)(kbase + j0) * SA_DV) + c);
      if (j1 >= 0) b = __ldg(reinterpret_cast<const uint4 *>(kv_v + (size_t)(kbase + j1) * SA_DV) + c);
      const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int i = 0; i < 8; i++) {
        const uint32_t lo16 = (i & 1) ? (aw[i >> 1] >> 16) : (aw[i >> 1] & 0xffffu);
        const uint32_t hi16 = (i & 1) ? (bw[i >> 1] >> 16) : (bw[i >> 1] & 0xffffu);
        *reinterpret_cast<uint32_t *>(sm.vt + kmaj_off(c * 8 + i, t0, SA_DV)) = lo16 | (hi16 << 16);
      }
    }
    cp_async_wait_all();
    fence_proxy_async_smem();
    __syncthreads();
    // S^T = K_tile . Q^T
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < 8; kk++)
        umma_bf16(tmem, sdesc_k_sw128(skt + (kk >> 2) * AT_TILE * 128 + (kk & 3) * 32),
                  sdesc_k_sw128(sqb + (kk >> 2) * AT_NH * 128 + (kk & 3) * 32), id, kk > 0);
      umma_commit(&sm.bar_mma);
    }
    __syncwarp();
    mbar_wait(&sm.bar_mma, phase, status);
    phase ^= 1u;
    tc_fence_after();
    // scores of token tid, online softmax per head across the tile
    float sc[AT_NH];
    {
      uint32_t v[16];
      tmem_ld16(tmem + lane_base, v);
      tmem_wait_ld();
#pragma unroll
      for (int u = 0; u < 16; u++) sc[u] = __uint_as_float(v[u]);
      if (Hp > 16) {
        tmem_ld16(tmem + lane_base + 16, v);
        tmem_wait_ld();
#pragma unroll
        for (int u = 0; u < 16; u++) sc[16 + u] = __uint_as_float(v[u]);
      }
    }
    const bool live = sm.tok[tid] >= 0;
#pragma unroll
    for (int h = 0; h < AT_NH; h++) {
      if (h < H) {
        sc[h] = live ? sc[h] * scale : NEG;
        float mx = sc[h];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        if (lane == 0) sm.tmax[warp][h] = mx;
      }
    }
    __syncthreads();
    if (tid < H) {
      const float tm = fmaxf(fmaxf(sm.tmax[0][tid], sm.tmax[1][tid]),
                             fmaxf(sm.tmax[2][tid], sm.tmax[3][tid]));
      const float mo = sm.m[tid], mn = fmaxf(mo, tm);
      sm.mnew[tid] = mn;
      sm.alpha[tid] = (mn == NEG) ? 1.f : expf(mo - mn);  // mo = -inf gives 0
    }
    __syncthreads();
#pragma unroll
    for (int h = 0; h < AT_NH; h++) {
      if (h < H) {
        const float p = live ? expf(sc[h] - sm.mnew[h]) : 0.f;
        const uint16_t hb = bf16_rn_bits(p);
        const uint16_t lb = bf16_rn_bits(p - __uint_as_float((uint32_t)hb << 16));
        *reinterpret_cast<uint16_t *>(sm.ph + kmaj_off(h, tid, AT_NH)) = hb;
        *reinterpret_cast<uint16_t *>(sm.pl + kmaj_off(h, tid, AT_NH)) = lb;
        float ps = p;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
        if (lane == 0) sm.tsum[warp][h] = ps;
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid < H) {
      sm.l[tid] = sm.l[tid] * sm.alpha[tid] + (sm.tsum[0][tid] + sm.tsum[1][tid]) +
                  (sm.tsum[2][tid] + sm.tsum[3][tid]);
      sm.m[tid] = sm.mnew[tid];
    }
    // O^T tile = V^T . (P_hi + P_lo)^T
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < 8; kk++)
        umma_bf16(tmem + 32, sdesc_k_sw128(svt + (kk >> 2) * SA_DV * 128 + (kk & 3) * 32),
                  sdesc_k_sw128(sph + (kk >> 2) * AT_NH * 128 + (kk & 3) * 32), id, kk > 0);
#pragma unroll
      for (int kk = 0; kk < 8; kk++)
        umma_bf16(tmem + 32, sdesc_k_sw128(svt + (kk >> 2) * SA_DV * 128 + (kk & 3) * 32),
                  sdesc_k_sw128(spl + (kk >> 2) * AT_NH * 128 + (kk & 3) * 32), id, 1u);
      umma_commit(&sm.bar_mma);
    }
    __syncwarp();
    mbar_wait(&sm.bar_mma, phase, status);
    phase ^= 1u;
    tc_fence_after();
    // fold the tile into dimension tid's accumulators
    {
      uint32_t v[16];
      tmem_ld16(tmem + lane_base + 32, v);
      tmem_wait_ld();
#pragma unroll
      for (int u = 0; u < 16; u++)
        if (u < H) oacc[u] = fmaf(oacc[u], sm.alpha[u], __uint_as_float(v[u]));
      if (Hp > 16) {
        tmem_ld16(tmem + lane_base + 48, v);
        tmem_wait_ld();
#pragma unroll
        for (int u = 0; u < 16; u++)
          if (16 + u < H) oacc[16 + u] = fmaf(oacc[16 + u], sm.alpha[16 + u], __uint_as_float(v[u]));
      }
    }
    tc_fence_before();
    __syncthreads();  // the next tile overwrites the operands and the accumulators
  }
  if (tid == 0 && sm.bad) raise_status(status, HISA_ERR_INVALID_ARG);

  // merge across the cluster: CTA c finishes heads h % C == c
#pragma unroll
  for (int h = 0; h < AT_NH; h++)
    if (h < H) sm.opart[h][tid] = oacc[h];
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
    for (int d = tid; d < SA_DV; d += AT_THREADS) {
      float acc = 0.f;
      for (int c = 0; c < C; c++) {
        const float mc = cl.map_shared_rank(&sm.m[0], c)[h];
        if (mc != NEG) acc += expf(mc - M) * cl.map_shared_rank(&sm.opart[0][0], c)[h * SA_DV + d];
      }
      orow[d] = L > 0.f ? acc / L : 0.f;
    }
    if (lse && tid == 0) lse[(size_t)row * H + h] = L > 0.f ? M + logf(L) : NEG;
  }
  cl.sync();
  if (warp == 0) tmem_dealloc(tmem, AT_TMEM_COLS);
}

cudaError_t launch_sparse_attention(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                                    const int32_t *idx, const int32_t *cu_q, const int32_t *cu_k,
                                    int S, int total_q, int H, int topk, float scale, float *out,
                                    float *lse, int num_sms, int *status, cudaStream_t st) {
  if (total_q == 0) return cudaSuccess;
  static int attr[64];
  cudaError_t e = set_smem_once((const void *)sparse_attn_tc_kernel, AT_SMEM, attr);
  if (e != cudaSuccess) return e;
  int C = 1;
  while (C < SA_MAX_CLUSTER && total_q * C < 2 * num_sms) C *= 2;
  int per = (topk + C - 1) / C;
  per = (per + AT_TILE - 1) / AT_TILE * AT_TILE;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(total_q * C);
  cfg.blockDim = dim3(AT_THREADS);
  cfg.dynamicSmemBytes = AT_SMEM;
  cfg.stream = st;
  cudaLaunchAttribute attrs[1];
  attrs[0].id = cudaLaunchAttributeClusterDimension;
  attrs[0].val.clusterDim.x = C;
  attrs[0].val.clusterDim.y = 1;
  attrs[0].val.clusterDim.z = 1;
  cfg.attrs = attrs;
  cfg.numAttrs = 1;
  ProfScope ps(K_SPARSE_ATTENTION, st);
  return cudaLaunchKernelEx(&cfg, sparse_attn_tc_kernel, q, k, v, idx, cu_q, cu_k, S, H, topk,
                            per, scale, out, lse, status);
}

}  // namespace hisa
