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
#include <cuda_bf16.h>

#include "prof.cuh"
#include "tc.cuh"

namespace cg = cooperative_groups;

namespace hisa {

constexpr int SA_DV = HISA_ATT_DIM;   // 128
constexpr int SA_MAX_CLUSTER = 8;
static_assert(SA_DV == 128, "the merge and the tile layouts take 128-dim rows");

// ---------------------------------------------------------------------------
// Tensor-core version.  Per tile of 128 selected tokens:
//   S^T [128 tokens x Hp]  = K_tile [128 x 128] . Q^T [128 x Hp]        (TMEM cols 0 / 32)
//   O^T [128 dims x 64]    = V^T [128 x 128 tokens] . [P_hi | P_lo]^T  (TMEM cols 64..127)
// with Hp = the head count rounded up to 16.  The key and value tiles are gathered
// with cp.async in the cache's own row layout (token rows, 128-byte swizzle): K is
// the K-major A operand of the first product and V the MN-major A operand of the
// second.  Q is a K-major B operand; the probabilities are split into bf16 hi + lo
// (about 16 bits) and stored MN-major, one 128-byte row per token holding the hi
// values at elements 0.. and the lo values at 32.., so one product of N = 64 gives
// O_hi and O_lo side by side.  Four loader warps fill a three-stage ring; thread t
// of the four compute warps is token t for the scores and dimension t for the output
// tile, which it folds into fp32 registers.  Each tcgen05 MMA of these shapes retires
// about 85 cycles after the previous one whatever its N, so the kernel keeps the MMA
// count low (eight per product) and overlaps the chains with the softmax rather
// than splitting them.

constexpr int AT_COMPUTE = 128;              // warps 0-3: MMAs, softmax, output fold
constexpr int AT_LOADERS = 128;              // warps 4-7: token ids, key and value tiles
constexpr int AT_THREADS = AT_COMPUTE + AT_LOADERS;
constexpr int AT_TILE = 128;                 // tokens per tile
constexpr int AT_STAGES = 3;                 // tiles in the loaders' ring
constexpr int AT_NH = 32;                    // head rows of the Q operand
constexpr uint32_t AT_TMEM_COLS = 128;       // S^T of even / odd tiles at cols 0 / 32, O at 64
constexpr int AT_PLO = 32;                   // P row: hi of head h at element h, lo at 32 + h
constexpr float AT_TAU = 8.f;                // tolerated growth of a head's maximum (nats)

struct AtSmem {
  uint8_t kt[AT_STAGES][2 * AT_TILE * 128];  // key tiles: two 64-dim atoms of 128 token rows
  uint8_t vt[AT_STAGES][2 * AT_TILE * 128];  // value tiles, same layout
  uint8_t qb[2 * AT_NH * 128];               // Q, two 64-dim atoms of 32 head rows
  uint8_t pb[AT_TILE * 128];                 // P, MN-major: one 128-byte row per token
  int tok[AT_STAGES][AT_TILE];
  float tmax[2][4][AT_NH], tsum[2][4][AT_NH];  // per warp and head, by tile parity
  float m[AT_NH], l[AT_NH];                    // the CTA's reference maximum and sum
  float wm[AT_NH][SA_MAX_CLUSTER], wl[AT_NH][SA_MAX_CLUSTER];  // merge weights
  uint64_t bar_s[2], bar_o, full[AT_STAGES], empty[AT_STAGES];  // bar_s per S buffer
  uint32_t tmem_base;
  int bad;
  int abort;  // set by the first wait that times out; the CTA's later waits give up
};
constexpr size_t AT_SMEM = sizeof(AtSmem) + 1024;
static_assert(AT_SMEM <= 232448, "one CTA per SM");
static_assert(AT_NH * SA_DV * 4 <= 2 * AT_TILE * 128, "the merge's partial outputs fit a key stage");

// barrier among the four compute warps only (the loaders never take id 1)
__device__ __forceinline__ void compute_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(AT_COMPUTE) : "memory");
}
// the same barrier, returning whether any compute thread passed v = true
__device__ __forceinline__ bool compute_vote(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.or.pred p, 1, %2, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "n"(AT_COMPUTE)
      : "memory");
  return r != 0;
}
// barrier among the four loader warps only
__device__ __forceinline__ void loader_sync() {
  asm volatile("bar.sync 2, %0;" ::"n"(AT_LOADERS) : "memory");
}

// Transposed warp reduction of NH values per lane (NH = 16 or 32): each step trades
// half of the live values with the partner lane and combines the other half, so the
// whole reduction takes NH - 1 independent shuffles.  Afterwards lane l holds the
// result for head l (NH = 32) or head l >> 1 (NH = 16, lanes 2h and 2h + 1).
template <int NH, bool MAX>
__device__ __forceinline__ float xreduce(float (&v)[NH], int lane) {
  constexpr int STEPS = NH == 32 ? 5 : 4;
#pragma unroll
  for (int st = 0; st < STEPS; st++) {
    const int o = 16 >> st, half = (NH >> st) >> 1;
    const bool up = (lane & o) != 0;
#pragma unroll
    for (int i = 0; i < half; i++) {
      const float send = up ? v[i] : v[i + half];
      const float keep = up ? v[i + half] : v[i];
      const float r = __shfl_xor_sync(0xffffffffu, send, o);
      v[i] = MAX ? fmaxf(keep, r) : keep + r;
    }
  }
  if (NH == 16) {
    const float r = __shfl_xor_sync(0xffffffffu, v[0], 1);
    v[0] = MAX ? fmaxf(v[0], r) : v[0] + r;
  }
  return v[0];
}

// The compute warps' side of one CTA over tiles 0 .. ntiles - 1 (stage t % AT_STAGES);
// NH = the padded head count (16 or 32), heads h >= H are masked.  The scores of tile
// t land in TMEM columns from 32 * (t & 1), so thread 0 issues the next tile's score product
// as soon as its stage is filled, and it runs under the current tile's softmax.  P is
// the MN-major B operand of the second product: thread t writes token t's 128-byte
// row (hi of head h at element h, lo at 32 + h, zeros elsewhere), and the product's
// N = 64 output columns are O hi | O lo.  The probabilities
// of a tile are taken against a reference maximum per head that every compute thread
// holds in registers; it is raised (and the output and sum rescaled) only on a tile
// where some score exceeds it by more than AT_TAU, which one barrier vote detects, so
// most tiles need neither the maximum reduction nor a rescale.  Leaves the CTA's
// unnormalised output for dimension tid in oacc and the reference maximum and the
// sum per head in sm.m and sm.l.
template <int NH>
__device__ __forceinline__ void attn_compute(AtSmem &sm, uint32_t tmem, uint32_t sqb, int ntiles,
                                             int H, float scale, int *status,
                                             float (&oacc)[AT_NH]) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const float NEG = -__int_as_float(0x7f800000);
  const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
  const uint32_t spb = smem_u32(sm.pb);
  const uint32_t id = idesc_bf16_f32(AT_TILE, NH);
  const uint32_t idv = idesc_bf16_f32_amn(SA_DV, 2 * AT_PLO) | (1u << 16);  // A and B MN-major
  const int hl = NH == 32 ? lane : lane >> 1;  // head whose warp reduction this lane holds
  const bool hl_writer = NH == 32 || (lane & 1) == 0;

  // S^T = K_tile . Q^T for tile t (thread 0), once its stage is filled; with
  // `block` false it only tries.  Returns whether it issued.
  auto issue_scores = [&](int t, bool block) -> bool {
    const int st = t % AT_STAGES;
    const uint32_t par = (uint32_t)(t / AT_STAGES) & 1u;
    if (block) {
      mbar_wait(&sm.full[st], par, status, &sm.abort);
    } else if (!mbar_try_wait(&sm.full[st], par)) {
      return false;
    }
    fence_proxy_async_smem();
    tc_fence_after();
    const uint32_t skt = smem_u32(sm.kt[st]);
#pragma unroll
    for (int kk = 0; kk < 8; kk++)
      umma_bf16(tmem + 32u * (uint32_t)(t & 1),
                sdesc_k_sw128(skt + (kk >> 2) * AT_TILE * 128 + (kk & 3) * 32),
                sdesc_k_sw128(sqb + (kk >> 2) * AT_NH * 128 + (kk & 3) * 32), id, kk > 0);
    umma_commit(&sm.bar_s[t & 1]);
    return true;
  };
  int issued = 0;  // thread 0: score products issued so far
  if (tid == 0 && ntiles > 0) {
    issue_scores(0, true);
    issued = 1;
  }
  __syncwarp();

  float mref[NH];
#pragma unroll
  for (int h = 0; h < NH; h++) mref[h] = NEG;
  float lsum = 0.f;  // thread h < H: the running sum of head h
  for (int t = 0; t < ntiles; t++) {
    const int st = t % AT_STAGES, par = t & 1;
    if (tid == 0 && issued == t + 1 && t + 1 < ntiles && issue_scores(t + 1, false)) issued++;
    __syncwarp();
    mbar_wait(&sm.full[st], (uint32_t)(t / AT_STAGES) & 1u, status, &sm.abort);
    const bool live = sm.tok[st][tid] >= 0;
    mbar_wait(&sm.bar_s[par], (uint32_t)(t >> 1) & 1u, status, &sm.abort);
    tc_fence_after();
    const uint32_t scol = tmem + lane_base + 32u * (uint32_t)par;
    float sc[NH];
    {
      uint32_t v[16];
      tmem_ld16(scol, v);
      tmem_wait_ld();
#pragma unroll
      for (int u = 0; u < 16; u++) sc[u] = __uint_as_float(v[u]);
      if (NH == 32) {
        tmem_ld16(scol + 16, v);
        tmem_wait_ld();
#pragma unroll
        for (int u = 0; u < 16; u++) sc[(16 + u) % NH] = __uint_as_float(v[u]);
      }
    }
    bool over = false;
#pragma unroll
    for (int h = 0; h < NH; h++) {
      sc[h] = (live && h < H) ? sc[h] * scale : NEG;
      over |= sc[h] > mref[h] + AT_TAU;  // a live score over a reference of -inf counts
    }
    tc_fence_before();
    const bool rescale = compute_vote(over);  // (1) the tile's scores are read
    if (tid == 0 && issued == t + 1 && t + 1 < ntiles && issue_scores(t + 1, true)) issued++;
    __syncwarp();
    float alpha_own = 1.f;  // thread h < H: the factor of head h's sum
    if (rescale) {
      {
        float w[NH];
#pragma unroll
        for (int h = 0; h < NH; h++) w[h] = sc[h];
        const float mx = xreduce<NH, true>(w, lane);
        if (hl_writer) sm.tmax[par][warp][hl] = mx;
      }
      compute_sync();
#pragma unroll
      for (int h = 0; h < NH; h++) {
        const float tm = fmaxf(fmaxf(sm.tmax[par][0][h], sm.tmax[par][1][h]),
                               fmaxf(sm.tmax[par][2][h], sm.tmax[par][3][h]));
        const float mn = fmaxf(mref[h], tm);
        const float a = (mn == NEG) ? 1.f : __expf(mref[h] - mn);  // reference -inf gives 0
        oacc[h] *= a;
        if (h == tid) alpha_own = a;
        mref[h] = mn;
      }
    }
    {
      float w[NH];
      uint32_t hi2[NH / 2], lo2[NH / 2];
#pragma unroll
      for (int h = 0; h < NH; h += 2) {
        const float p0 = (live && h < H) ? __expf(sc[h] - mref[h]) : 0.f;
        const float p1 = (live && h + 1 < H) ? __expf(sc[h + 1] - mref[h + 1]) : 0.f;
        const __nv_bfloat162 hb = __floats2bfloat162_rn(p0, p1);
        const __nv_bfloat162 lb = __floats2bfloat162_rn(p0 - __low2float(hb), p1 - __high2float(hb));
        hi2[h >> 1] = *reinterpret_cast<const uint32_t *>(&hb);
        lo2[h >> 1] = *reinterpret_cast<const uint32_t *>(&lb);
        w[h] = p0;
        w[h + 1] = p1;
      }
      // token tid's row: 16-byte chunk c (8 heads) at its swizzled place
      uint8_t *prow = sm.pb + (tid >> 3) * 1024 + (tid & 7) * 128;
#pragma unroll
      for (int c = 0; c < NH / 8; c++) {
        *reinterpret_cast<uint4 *>(prow + ((c ^ (tid & 7)) << 4)) =
            make_uint4(hi2[4 * c], hi2[4 * c + 1], hi2[4 * c + 2], hi2[4 * c + 3]);
        *reinterpret_cast<uint4 *>(prow + (((AT_PLO / 8 + c) ^ (tid & 7)) << 4)) =
            make_uint4(lo2[4 * c], lo2[4 * c + 1], lo2[4 * c + 2], lo2[4 * c + 3]);
      }
      const float ps = xreduce<NH, false>(w, lane);
      if (hl_writer) sm.tsum[par][warp][hl] = ps;
    }
    fence_proxy_async_smem();
    tc_fence_before();
    compute_sync();  // (2) P and the tile's sums are in; the previous fold is done
    // [O_hi | O_lo]^T = V^T . [P_hi | P_lo]^T, both operands read MN-major from token
    // rows: V's dims 0-63 and 64-127 are 16 KB apart, 8-token groups 1 KB apart in both,
    // 16 tokens per MMA.  The stage is free once these have run.
    if (tid == 0) {
      tc_fence_after();
      const uint32_t svt = smem_u32(sm.vt[st]);
#pragma unroll
      for (int kk = 0; kk < 8; kk++)
        umma_bf16(tmem + 64, sdesc_mn_sw128(svt + kk * 2048, AT_TILE * 128, 1024),
                  sdesc_mn_sw128(spb + kk * 2048, 1024, 1024), idv, kk > 0);
      umma_commit(&sm.bar_o);
      if (t + AT_STAGES < ntiles) umma_commit(&sm.empty[st]);
    }
    __syncwarp();
    if (tid < H)
      lsum = lsum * alpha_own + (sm.tsum[par][0][tid] + sm.tsum[par][1][tid]) +
             (sm.tsum[par][2][tid] + sm.tsum[par][3][tid]);
    mbar_wait(&sm.bar_o, (uint32_t)par, status, &sm.abort);
    tc_fence_after();
    // fold the tile into dimension tid's accumulators
#pragma unroll
    for (int g = 0; g < NH / 16; g++) {
      uint32_t hi[16], lo[16];
      tmem_ld16(tmem + lane_base + 64 + 16 * g, hi);
      tmem_ld16(tmem + lane_base + 64 + AT_PLO + 16 * g, lo);
      tmem_wait_ld();
#pragma unroll
      for (int u = 0; u < 16; u++)
        oacc[16 * g + u] += __uint_as_float(hi[u]) + __uint_as_float(lo[u]);
    }
    tc_fence_before();
  }
  if (tid < H) {
    float mo = NEG;
#pragma unroll
    for (int h = 0; h < NH; h++)
      if (h == tid) mo = mref[h];
    sm.m[tid] = mo;
    sm.l[tid] = lsum;
  }
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
  const int tid = threadIdx.x, warp = tid >> 5;
  const float NEG = -__int_as_float(0x7f800000);
  const int Hp = (H + 15) & ~15;

  const int s = find_seq(cu_q, S, row);
  const int kbase = __ldg(cu_k + s), kcap = __ldg(cu_k + s + 1) - kbase;
  if (tid == 0) {
    mbar_init(&sm.bar_s[0], 1);
    mbar_init(&sm.bar_s[1], 1);
    mbar_init(&sm.bar_o, 1);
    for (int i = 0; i < AT_STAGES; i++) {
      mbar_init(&sm.full[i], AT_LOADERS);
      mbar_init(&sm.empty[i], 1);
    }
    fence_barrier_init();
    sm.bad = 0;
    sm.abort = 0;
  }
  if (warp == 0) {
    tmem_alloc(&sm.tmem_base, AT_TMEM_COLS);
    tmem_relinquish();
  }
  // Q, zero rows for padded heads
  for (int x = tid; x < AT_NH * 16; x += AT_THREADS) {
    const int h = x >> 4, c = x & 15;
    uint4 w = make_uint4(0u, 0u, 0u, 0u);
    if (h < H) w = __ldg(reinterpret_cast<const uint4 *>(q + ((size_t)row * H + h) * SA_DV) + c);
    *reinterpret_cast<uint4 *>(sm.qb + (c >> 3) * AT_NH * 128 + sw128_offset(h, c & 7)) = w;
  }
  for (int x = tid; x < AT_TILE * 8; x += AT_THREADS)
    reinterpret_cast<uint4 *>(sm.pb)[x] = make_uint4(0u, 0u, 0u, 0u);
  if (tid < AT_NH) {
    sm.m[tid] = NEG;
    sm.l[tid] = 0.f;
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base, sqb = smem_u32(sm.qb);
  const int e0 = me * per_cta, e1 = min(topk, e0 + per_cta);
  const int ntiles = e1 > e0 ? (e1 - e0 + AT_TILE - 1) / AT_TILE : 0;
  const int32_t *irow = idx + (size_t)row * topk;
  float oacc[AT_NH];
#pragma unroll
  for (int h = 0; h < AT_NH; h++) oacc[h] = 0.f;

  if (tid >= AT_COMPUTE) {
    // ---- loaders: fill stage t % AT_STAGES with the tile's token ids and its key and
    // value rows; both tiles keep the row layout of the cache (token rows, dims
    // contiguous), swizzled in 128-byte rows; rows of no token are zeros.  A thread
    // keeps two tiles' copies in flight and signals a tile once its copies are done.
    const int lt = tid - AT_COMPUTE;
    for (int t = 0; t < ntiles; t++) {
      const int st = t % AT_STAGES, base = e0 + t * AT_TILE;
      if (t >= AT_STAGES)
        mbar_wait(&sm.empty[st], (uint32_t)(t / AT_STAGES - 1) & 1u, status, &sm.abort);
      {  // token of tile position lt (-1 = none; outside the region = none, reported)
        const int j = base + lt < e1 ? __ldg(irow + base + lt) : -1;
        if (j >= kcap) sm.bad = 1;
        sm.tok[st][lt] = j < kcap ? j : -1;
      }
      loader_sync();
      const uint32_t skt = smem_u32(sm.kt[st]), svt = smem_u32(sm.vt[st]);
#pragma unroll 4
      for (int x = lt; x < AT_TILE * 16; x += AT_LOADERS) {
        const int r = x >> 4, c = x & 15;
        const int j = sm.tok[st][r];
        const uint32_t off = (c >> 3) * AT_TILE * 128 + sw128_offset(r, c & 7);
        if (j >= 0) {
          const size_t src = (size_t)(kbase + j) * SA_DV + c * 8;
          cp_async_16(skt + off, kv_k + src);
          cp_async_16(svt + off, kv_v + src);
        } else {
          const uint4 z = make_uint4(0u, 0u, 0u, 0u);
          *reinterpret_cast<uint4 *>(sm.kt[st] + off) = z;
          *reinterpret_cast<uint4 *>(sm.vt[st] + off) = z;
        }
      }
      cp_async_commit();
      if (t > 0) {
        cp_async_wait_group1();
        fence_proxy_async_smem();
        mbar_arrive(&sm.full[(t - 1) % AT_STAGES]);
      }
    }
    if (ntiles > 0) {
      cp_async_wait_all();
      fence_proxy_async_smem();
      mbar_arrive(&sm.full[(ntiles - 1) % AT_STAGES]);
    }
  } else if (Hp == 16) {
    attn_compute<16>(sm, tmem, sqb, ntiles, H, scale, status, oacc);
  } else {
    attn_compute<32>(sm, tmem, sqb, ntiles, H, scale, status, oacc);
  }
  __syncthreads();
  if (tid == 0 && sm.bad) raise_status(status, HISA_ERR_INVALID_ARG);

  // merge across the cluster: CTA me finishes heads me, me + C, ... Every remote read
  // of a step is issued at once: (head, rank) pairs, then (head, dim) outputs.  The
  // partial outputs go to the first key stage, free now.
  float *opart = reinterpret_cast<float *>(sm.kt[0]);
  if (tid < AT_COMPUTE) {
#pragma unroll
    for (int h = 0; h < AT_NH; h++)
      if (h < H) opart[h * SA_DV + tid] = oacc[h];
  }
  cl.sync();
  const int nloc = me < H ? (H - me + C - 1) / C : 0;
  if (tid < nloc * C) {
    const int i = tid / C, c = tid - i * C, h = me + C * i;
    sm.wm[i][c] = cl.map_shared_rank(&sm.m[0], c)[h];
    sm.wl[i][c] = cl.map_shared_rank(&sm.l[0], c)[h];
  }
  __syncthreads();
  if (tid < nloc) {
    float M = NEG;
    for (int c = 0; c < C; c++) M = fmaxf(M, sm.wm[tid][c]);
    float L = 0.f;
    for (int c = 0; c < C; c++) {
      const float mc = sm.wm[tid][c];
      sm.wm[tid][c] = mc != NEG ? expf(mc - M) : 0.f;
      L += sm.wm[tid][c] * sm.wl[tid][c];
    }
    const float inv = L > 0.f ? 1.f / L : 0.f;
    for (int c = 0; c < C; c++) sm.wm[tid][c] *= inv;
    if (lse) lse[(size_t)row * H + me + C * tid] = L > 0.f ? M + logf(L) : NEG;
  }
  __syncthreads();
  for (int x = tid; x < nloc * SA_DV; x += AT_THREADS) {
    const int i = x >> 7, d = x & (SA_DV - 1), h = me + C * i;
    float part[SA_MAX_CLUSTER];
#pragma unroll
    for (int c = 0; c < SA_MAX_CLUSTER; c++)
      part[c] = c < C ? cl.map_shared_rank(opart, c)[h * SA_DV + d] : 0.f;
    float acc = 0.f;
#pragma unroll
    for (int c = 0; c < SA_MAX_CLUSTER; c++)
      if (c < C) acc = fmaf(sm.wm[i][c], part[c], acc);
    out[((size_t)row * H + h) * SA_DV + d] = acc;
  }
  cl.sync();
  if (warp == 0) tmem_dealloc(tmem, AT_TMEM_COLS);
}

cudaError_t launch_sparse_attention(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                                    const int32_t *idx, const int32_t *cu_q, const int32_t *cu_k,
                                    int S, int total_q, int H, int topk, float scale, float *out,
                                    float *lse, int num_sms, int *status, cudaStream_t st) {
  if (total_q == 0) return cudaSuccess;
  static std::atomic<int> attr[64];
  cudaError_t e = set_smem_once((const void *)sparse_attn_tc_kernel, AT_SMEM, attr);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(AT_THREADS);
  cfg.dynamicSmemBytes = AT_SMEM;
  cfg.stream = st;
  cudaLaunchAttribute attrs[1];
  attrs[0].id = cudaLaunchAttributeClusterDimension;
  attrs[0].val.clusterDim.y = 1;
  attrs[0].val.clusterDim.z = 1;
  cfg.attrs = attrs;
  cfg.numAttrs = 1;
  // Split the rows over clusters of C CTAs while the grid is small: among the C whose
  // clusters are all resident at once (a second wave of clusters costs more than the
  // split saves), take the one with the fewest tiles per CTA, the smaller on a tie.
  static std::atomic<int> fits[64][SA_MAX_CLUSTER + 1];  // clusters resident at once, per device
  int dev = 0;
  cudaGetDevice(&dev);
  const int tiles = (topk + AT_TILE - 1) / AT_TILE;
  int C = 1, best = tiles;
  for (int c = 2; c <= SA_MAX_CLUSTER; c++) {
    if (total_q * c > 2 * num_sms) break;  // enough CTAs without splitting this far
    const int cost = (tiles + c - 1) / c;
    if (cost >= best) continue;
    int n = fits[dev & 63][c].load(std::memory_order_relaxed);
    if (n == 0) {
      cfg.gridDim = dim3(c);
      attrs[0].val.clusterDim.x = c;
      if (cudaOccupancyMaxActiveClusters(&n, sparse_attn_tc_kernel, &cfg) != cudaSuccess) {
        (void)cudaGetLastError();  // the query's own error; the launch below decides
        n = -1;
      } else if (n <= 0) {
        n = -1;
      }
      fits[dev & 63][c].store(n, std::memory_order_relaxed);
    }
    if (n < total_q) continue;
    C = c;
    best = cost;
  }
  const int per = best * AT_TILE;
  cfg.gridDim = dim3(total_q * C);
  attrs[0].val.clusterDim.x = C;
  ProfScope ps(K_SPARSE_ATTENTION, st);
  return cudaLaunchKernelEx(&cfg, sparse_attn_tc_kernel, q, k, v, idx, cu_q, cu_k, S, H, topk,
                            per, scale, out, lse, status);
}

}  // namespace hisa
