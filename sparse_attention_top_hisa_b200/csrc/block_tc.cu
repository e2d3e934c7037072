// Stage 1 of HISA on the tensor cores: query x block-representative scores.
//
// HISA summary page (aitrends.kr), paragraph on stage 1: each query is scored
// against the representative of every block that is not wholly after it.  For a
// tile of 128 consecutive queries of one sequence this is the dense product
// Q [128 x 64] . R^T [64 x E] over the E blocks the tile can see.
//
// The representatives are fp32 means; bf16 alone would round them (a mean of 128
// bf16 keys has up to 16 significant bits), so each is split as rep = hi + lo with
// hi = bf16(rep) and lo = bf16(rep - hi), and the score is q.hi + q.lo accumulated
// in fp32 (8 MMA K-steps).  For integer-valued keys (means are multiples of 1/128
// with at most 10 significant bits) the split is exact; otherwise it keeps about 16
// bits of every representative.
//
//   reps_split_kernel   fp32 representatives -> bf16 hi/lo rows, indexed by compact
//                       block id (sequence * emax + block);
//   block_score_tc_kernel  one CTA per 128-query tile: TMA loads of the query tile and
//                       of 256-block hi/lo tiles, tcgen05.mma into a 128 x 256 fp32 TMEM
//                       accumulator, and an epilogue that writes order-preserving keys
//                       (0 for the forced blocks and for blocks after the query) to a
//                       dense [total_q x emax] score matrix read by the top-m kernel.
#include "prof.cuh"
#include "tc.cuh"

namespace hisa {

constexpr int BS_TC_THREADS = 128;
constexpr int BS_TC_N = 256;  // blocks per MMA tile
constexpr uint32_t BS_TC_TMEM_COLS = 256;

__device__ __forceinline__ uint32_t bf16_bits_rn(float x) {
  const uint32_t u = __float_as_uint(x);
  return (u + 0x7fffu + ((u >> 16) & 1u)) >> 16;  // round to nearest, ties to even (finite x)
}

__global__ void __launch_bounds__(128)
reps_split_kernel(const float *__restrict__ reps, const int32_t *__restrict__ cu_k,
                  const int32_t *__restrict__ seqlens, int S, int emax,
                  uint32_t *__restrict__ hi, uint32_t *__restrict__ lo) {
  const int cb = blockIdx.x * 4 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (cb >= S * emax) return;
  const int s = cb / emax, b = cb - s * emax;
  const int start = __ldg(cu_k + s), cap = __ldg(cu_k + s + 1) - start;
  const int len = seqlens ? __ldg(seqlens + s) : cap;
  uint32_t h = 0u, l = 0u;
  if (start % BLK == 0 && len >= 0 && len <= cap && b * BLK < len) {
    const float2 r = reinterpret_cast<const float2 *>(reps + (size_t)(start / BLK + b) * D)[lane];
    const uint32_t h0 = bf16_bits_rn(r.x), h1 = bf16_bits_rn(r.y);
    const uint32_t l0 = bf16_bits_rn(r.x - __uint_as_float(h0 << 16));
    const uint32_t l1 = bf16_bits_rn(r.y - __uint_as_float(h1 << 16));
    h = h0 | (h1 << 16);
    l = l0 | (l1 << 16);
  }
  hi[(size_t)cb * 32 + lane] = h;
  lo[(size_t)cb * 32 + lane] = l;
}

struct BsSmem {
  uint8_t a[BLK * ROW_BYTES];         // query tile
  uint8_t bh[BS_TC_N * ROW_BYTES];    // representative hi tile
  uint8_t bl[BS_TC_N * ROW_BYTES];    // representative lo tile
  uint64_t bar_a, bar_b, bar_mma;
  uint32_t tmem_base;
  int info[2];
};
constexpr size_t BS_TC_SMEM = sizeof(BsSmem) + 1024;

__global__ void __launch_bounds__(BS_TC_THREADS, 1)
block_score_tc_kernel(const __grid_constant__ CUtensorMap qmap,
                      const __grid_constant__ CUtensorMap himap,
                      const __grid_constant__ CUtensorMap lomap, const int32_t *__restrict__ cu_q,
                      const int32_t *__restrict__ cu_k, const int32_t *__restrict__ seqlens,
                      const int32_t *__restrict__ m_seq, int S, int emax, int estride, int m,
                      uint32_t *__restrict__ scores, int *status) {
  extern __shared__ uint8_t bs_smem_raw[];
  BsSmem &sm = *reinterpret_cast<BsSmem *>((reinterpret_cast<uintptr_t>(bs_smem_raw) + 1023) &
                                           ~(uintptr_t)1023);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // which (sequence, first query row) this CTA owns
  if (tid == 0) {
    int t = blockIdx.x, acc = 0, found = -1, r0 = 0;
    for (int s = 0; s < S; s++) {
      const int nt = (__ldg(cu_q + s + 1) - __ldg(cu_q + s) + BLK - 1) / BLK;
      if (t < acc + nt) {
        found = s;
        r0 = (t - acc) * BLK;
        break;
      }
      acc += nt;
    }
    sm.info[0] = found;
    sm.info[1] = r0;
  }
  __syncthreads();
  const int s = sm.info[0], r0 = sm.info[1];
  if (s < 0) return;  // block-uniform: beyond the last tile
  const int q0 = __ldg(cu_q + s), qlen = __ldg(cu_q + s + 1) - q0;
  const int kbase = __ldg(cu_k + s), cap = __ldg(cu_k + s + 1) - kbase;
  const int len = seqlens ? __ldg(seqlens + s) : cap;
  if (kbase % BLK != 0 || len < 0 || len > cap || qlen > len) return;  // reported by the top-m stage
  const int nr = min(BLK, qlen - r0);
  const int pos_first = len - qlen + r0;
  const int e_tile = (pos_first + nr - 1) / BLK + 1;
  if (e_tile > emax) return;  // max_seqlen_k understated: reported by the top-m stage

  if (tid == 0) {
    mbar_init(&sm.bar_a, 1);
    mbar_init(&sm.bar_b, 1);
    mbar_init(&sm.bar_mma, 1);
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(&sm.tmem_base, BS_TC_TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  const uint32_t sa = smem_u32(sm.a), sbh = smem_u32(sm.bh), sbl = smem_u32(sm.bl);
  if (tid == 0) {
    mbar_arrive_expect_tx(&sm.bar_a, BLK * ROW_BYTES);
    tma_load_2d(sm.a, &qmap, &sm.bar_a, 0, q0 + r0);
  }
  const int row_local = warp * 32 + lane;
  const bool row_ok = row_local < nr;
  const int pos = pos_first + row_local;
  const int own = pos / BLK;
  const int nf = min(seq_budget(m_seq, s, m, nullptr), 3);  // the top-m stage reports bad budgets
  uint32_t *out_row = scores + (size_t)(q0 + r0 + row_local) * estride;
  uint32_t phase = 0;
  for (int c0 = 0; c0 < e_tile; c0 += BS_TC_N, phase ^= 1u) {
    const int nb = min(BS_TC_N, e_tile - c0);
    const int npad = (nb + 15) & ~15;
    if (tid == 0) {
      mbar_arrive_expect_tx(&sm.bar_b, 2 * BS_TC_N * ROW_BYTES);
      tma_load_2d(sm.bh, &himap, &sm.bar_b, 0, s * emax + c0);
      tma_load_2d(sm.bl, &lomap, &sm.bar_b, 0, s * emax + c0);
      if (c0 == 0) mbar_wait(&sm.bar_a, 0, status);
      mbar_wait(&sm.bar_b, phase, status);
      tc_fence_after();
      const uint32_t id = idesc_bf16_f32(BLK, npad);
#pragma unroll
      for (int kk = 0; kk < 4; kk++)
        umma_bf16(tmem, sdesc_k_sw128(sa + kk * 32), sdesc_k_sw128(sbh + kk * 32), id, kk > 0);
#pragma unroll
      for (int kk = 0; kk < 4; kk++)
        umma_bf16(tmem, sdesc_k_sw128(sa + kk * 32), sdesc_k_sw128(sbl + kk * 32), id, 1u);
      umma_commit(&sm.bar_mma);
    }
    __syncwarp();
    mbar_wait(&sm.bar_mma, phase, status);
    tc_fence_after();
    // 64 columns per wait: four TMEM loads in flight (npad is warp-uniform)
    for (int c64 = 0; c64 < npad; c64 += 64) {
      uint32_t v[4][16];
#pragma unroll
      for (int j = 0; j < 4; j++)
        if (c64 + 16 * j < npad)
          tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)(c64 + 16 * j), v[j]);
      tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < 4; j++) {
        const int cc = c64 + 16 * j;
        if (cc < npad && row_ok && c0 + cc < e_tile) {
          uint32_t key[16];
#pragma unroll
          for (int u = 0; u < 16; u++) {
            const int b = c0 + cc + u;
            const bool forced = b == own || (nf >= 2 && b == own - 1) || (nf >= 3 && b == 0);
            key[u] = (b <= own && !forced) ? score_key(__uint_as_float(v[j][u])) : 0u;
          }
          // rows are estride (a multiple of 16) keys long; columns past e_tile get 0
          uint4 *dst = reinterpret_cast<uint4 *>(out_row + c0 + cc);
#pragma unroll
          for (int u = 0; u < 4; u++)
            dst[u] = make_uint4(key[4 * u], key[4 * u + 1], key[4 * u + 2], key[4 * u + 3]);
        }
      }
    }
    tc_fence_before();
    __syncthreads();
  }
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, BS_TC_TMEM_COLS);
}

// ---------------------------------------------------------------------------
// host side

bool make_rows_tensor_map(CUtensorMap *map, const void *base, uint64_t rows, uint32_t box_rows);

struct BsPlan {
  size_t off_hi, off_lo, off_scores, total;
};

static size_t b256(size_t x) { return (x + 255) & ~(size_t)255; }

int block_score_stride(int max_seqlen_k) {
  const int emax = (max_seqlen_k + BLK - 1) / BLK;
  return (emax + 15) & ~15;  // rows are written 16 keys at a time
}

static BsPlan bs_plan(int total_q, int num_seqs, int max_seqlen_k) {
  BsPlan p;
  const int emax = (max_seqlen_k + BLK - 1) / BLK;
  const size_t nb = (size_t)(num_seqs > 0 ? num_seqs : 1) * (emax > 0 ? emax : 1);
  size_t off = 0;
  p.off_hi = off;
  off = b256(off + nb * ROW_BYTES);
  p.off_lo = off;
  off = b256(off + nb * ROW_BYTES);
  p.off_scores = off;
  off = b256(off + (size_t)(total_q > 0 ? total_q : 1) * block_score_stride(max_seqlen_k) * 4 + 64);
  p.total = off;
  return p;
}

size_t block_tc_workspace_bytes(int total_q, int num_seqs, int max_seqlen_k) {
  return bs_plan(total_q, num_seqs, max_seqlen_k).total;
}

// Writes the dense score matrix [total_q x emax] (order-preserving keys) into ws.
cudaError_t launch_block_score_tc(const uint16_t *q, const float *reps, const int32_t *cu_q,
                                  const int32_t *cu_k, const int32_t *seqlens,
                                  const int32_t *m_seq, int S, int total_q, int max_seqlen_k,
                                  int m, uint8_t *ws, uint32_t **scores_out, int *status,
                                  cudaStream_t st) {
  const BsPlan p = bs_plan(total_q, S, max_seqlen_k);
  const int emax = (max_seqlen_k + BLK - 1) / BLK;
  uint32_t *hi = reinterpret_cast<uint32_t *>(ws + p.off_hi);
  uint32_t *lo = reinterpret_cast<uint32_t *>(ws + p.off_lo);
  uint32_t *scores = reinterpret_cast<uint32_t *>(ws + p.off_scores);
  *scores_out = scores;
  if (emax == 0) return cudaSuccess;
  CUtensorMap qmap, himap, lomap;
  if (!make_rows_tensor_map(&qmap, q, (uint64_t)total_q, BLK) ||
      !make_rows_tensor_map(&himap, hi, (uint64_t)S * emax, BS_TC_N) ||
      !make_rows_tensor_map(&lomap, lo, (uint64_t)S * emax, BS_TC_N))
    return cudaErrorInvalidValue;
  cudaError_t e;
  {
    ProfScope ps(K_REPS_SPLIT, st);
    reps_split_kernel<<<(S * emax + 3) / 4, 128, 0, st>>>(reps, cu_k, seqlens, S, emax, hi, lo);
  }
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  static std::atomic<int> attr[64];
  if ((e = set_smem_once((const void *)block_score_tc_kernel, BS_TC_SMEM, attr)) != cudaSuccess)
    return e;
  const int tiles = (total_q + BLK - 1) / BLK + S;  // per-sequence tiles, upper bound
  {
    ProfScope ps(K_BLOCK_SCORE_TC, st);
    block_score_tc_kernel<<<tiles, BS_TC_THREADS, BS_TC_SMEM, st>>>(
        qmap, himap, lomap, cu_q, cu_k, seqlens, m_seq, S, emax, block_score_stride(max_seqlen_k),
        m, scores, status);
  }
  return cudaGetLastError();
}

}  // namespace hisa
