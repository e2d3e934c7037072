// Flat DSA filter on the tensor cores.
//
// idea.jsleekr.com, section "DSA: 딥시크의 희소 어텐션": every query scores every
// earlier key.  For a tile of 128 queries of one sequence and a key block of 128 keys
// this is S = Q [128 x 64] . K_b^T [64 x 128], one tcgen05.mma chain (K = 4 x 16) into
// a 128 x 128 fp32 TMEM accumulator whose lane i is query i.  Two epilogue threads own
// query i: thread i reads columns 0..63 of its TMEM lane, thread i + 128 columns
// 64..127 (warps w and w + 4 reach the same 32 lanes), and they share the query's
// state in shared memory:
//   pass 1: the scores of the query are counted in DSA_TC_NB buckets linear over
//           [-R, R] (R = |q| |k|max, so every score falls inside), or over [0, R] for a
//           query with more than 4k candidates.  A tile whose queries see at most
//           DSA_SAMPLE_FROM key blocks counts every score and b* is the bucket holding
//           the k-th best; a longer tile counts only every DSA_SS-th key block and b* is
//           the bucket holding the best DSA_MARGIN * k * (sampled / all) + DSA_SLACK
//           sampled scores, an estimate of a threshold a little under the k-th best;
//   pass 2: the scores are recomputed and every score above a threshold just under the
//           lower edge of b* is appended, in token order, to the query's candidate list.
//           When the list holds at least k (or every causal) candidate it is a superset
//           of the top-k; a sampled estimate that came out too high leaves fewer, and
//           the row is then marked for the exact fallback (count = cap + 1), as is a
//           list that overflowed its capacity.  The two threads of a query append
//           through one shared counter, so a list is not in token order (the select
//           breaks ties by token index, and sends rows with heavy ties to the fallback).
// Warp-specialised: a producer warp streams the key blocks through a two-stage
// TMA ring (a sequence's partial last block comes by guarded cp.async) and issues
// the MMAs into two TMEM accumulators; four epilogue warps drain them.  Full/empty
// mbarrier pairs hand the stages and accumulators back and forth, so loads, MMAs and
// the epilogue of consecutive blocks overlap (eight epilogue warps; two CTAs per SM).  The two passes are one pipeline of
// 2 * nblocks steps.  The same bf16 x bf16 -> fp32 MMA as
// hisa_select's token stage, so equal inputs give equal scores.
#include "prof.cuh"
#include "tc.cuh"

namespace hisa {

constexpr int DSA_TC_Q = 128;                  // queries per tile (TMEM lanes)
constexpr int DSA_TC_EPI = 2 * DSA_TC_Q;       // epilogue threads: two per query
constexpr int DSA_TC_THREADS = DSA_TC_EPI + 32;  // + one producer warp (TMA and MMA issue)
constexpr int DSA_TC_NB = 96;                // score buckets per query
constexpr uint32_t DSA_TC_TMEM_COLS = 256;   // two 128-column accumulators
// sampled pass 1: tiles whose last query sees more than DSA_SAMPLE_FROM key blocks
// histogram every DSA_SS-th block only
constexpr int DSA_SAMPLE_FROM = 64;
constexpr int DSA_SS = 8;
constexpr float DSA_MARGIN = 1.2f;
constexpr int DSA_SLACK = 16;

struct DsaTcSmem {
  uint8_t q[BLK * ROW_BYTES];      // query tile
  uint8_t k[2][BLK * ROW_BYTES];   // key block ring
  uint32_t hist[DSA_TC_Q * (DSA_TC_NB + 1)];  // per query, shared by its two threads
  int qcount[DSA_TC_Q];                      // candidates appended per query
  int qseen[DSA_TC_Q];                       // scores counted by pass 1 per query
  float qthr[DSA_TC_Q];                      // pass-2 threshold per query
  uint64_t bar_q, k_full[2], k_empty[2], acc_full[2], acc_empty[2];
  uint32_t tmem_base;
  int info[2];
};
constexpr size_t DSA_TC_SMEM = sizeof(DsaTcSmem) + 1024;

__device__ __forceinline__ int dsa_bucket(float s, float R, float inv) {
  const int b = __float2int_rz((R - s) * inv);
  return min(max(b, 0), DSA_TC_NB - 1);
}

__global__ void __launch_bounds__(DSA_TC_THREADS, 2)
dsa_filter_tc_kernel(const __grid_constant__ CUtensorMap qmap,
                     const __grid_constant__ CUtensorMap kmap, const uint16_t *__restrict__ k,
                     const int32_t *__restrict__ cu_q, const int32_t *__restrict__ cu_k,
                     const int32_t *__restrict__ seqlens, int S, int row0, int nrows, int topk,
                     int cap, const float *__restrict__ kmax, float *__restrict__ buf_key,
                     int32_t *__restrict__ buf_j, int32_t *__restrict__ cnt_out, int *status) {
  extern __shared__ uint8_t dsa_tc_raw[];
  DsaTcSmem &sm = *reinterpret_cast<DsaTcSmem *>((reinterpret_cast<uintptr_t>(dsa_tc_raw) + 1023) &
                                                 ~(uintptr_t)1023);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // tiles are enumerated per sequence over the chunk rows [row0, row0 + nrows);
  // the longest tiles (latest queries) go first
  if (tid == 0) {
    int t = (int)(gridDim.x - 1 - blockIdx.x), acc = 0, found = -1, first = 0;
    for (int s = 0; s < S; s++) {
      const int a = max(__ldg(cu_q + s), row0), b = min(__ldg(cu_q + s + 1), row0 + nrows);
      const int nt = b > a ? (b - a + BLK - 1) / BLK : 0;
      if (t < acc + nt) {
        found = s;
        first = a + (t - acc) * BLK;
        break;
      }
      acc += nt;
    }
    sm.info[0] = found;
    sm.info[1] = first;
  }
  __syncthreads();
  const int s = sm.info[0], first = sm.info[1];
  if (s < 0) return;
  const int q0 = __ldg(cu_q + s), qend = min(__ldg(cu_q + s + 1), row0 + nrows);
  const int kbase = __ldg(cu_k + s), kcap = __ldg(cu_k + s + 1) - kbase;
  const int len = seqlens ? __ldg(seqlens + s) : kcap;
  const int qlen = __ldg(cu_q + s + 1) - q0;
  const int nr = min(BLK, qend - first);
  const int qi = tid & (DSA_TC_Q - 1), half = tid / DSA_TC_Q;  // query of the tile, column half
  const int row = first + qi;
  const bool active = tid < DSA_TC_EPI && qi < nr;  // false for the producer warp
  if (kbase % BLK != 0 || len < 0 || len > kcap || qlen > len) {
    if (tid == 0) raise_status(status, kbase % BLK ? HISA_ERR_UNALIGNED : HISA_ERR_INVALID_ARG);
    if (active && half == 0) cnt_out[row - row0] = 0;
    return;
  }
  const int pos_last = len - qlen + (first + nr - 1 - q0);
  const int nblk = pos_last / BLK + 1;
  // pass 1 walks blocks 0, ss, 2 ss, ... (ns of them), pass 2 every block 0 .. nblk-1
  const int ss = nblk > DSA_SAMPLE_FROM ? DSA_SS : 1;
  const int ns = (nblk + ss - 1) / ss;
  const int steps = ns + nblk;

  if (tid == 0) {
    mbar_init(&sm.bar_q, 1);
    for (int i = 0; i < 2; i++) {
      mbar_init(&sm.k_full[i], 1);
      mbar_init(&sm.k_empty[i], 1);
      mbar_init(&sm.acc_full[i], 1);
      mbar_init(&sm.acc_empty[i], DSA_TC_EPI);
    }
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(&sm.tmem_base, DSA_TC_TMEM_COLS);
    tmem_relinquish();
  }
  for (int i = tid; i < DSA_TC_Q * (DSA_TC_NB + 1); i += DSA_TC_THREADS) sm.hist[i] = 0u;
  for (int i = tid; i < DSA_TC_Q; i += DSA_TC_THREADS) {
    sm.qcount[i] = 0;
    sm.qseen[i] = 0;
    sm.qthr[i] = -__int_as_float(0x7f800000);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp == DSA_TC_EPI / 32) {
    // ---------------- producer warp: TMA loads and MMA issue ----------------
    const uint32_t sq = smem_u32(sm.q);
    const uint32_t sk[2] = {smem_u32(sm.k[0]), smem_u32(sm.k[1])};
    auto load = [&](int it) {  // whole warp
      const int b = it < ns ? it * ss : it - ns, st = it & 1;
      if (it >= 2 && lane == 0) mbar_wait(&sm.k_empty[st], (uint32_t)(((it - 2) >> 1) & 1), status);
      __syncwarp();
      const int live = len - b * BLK;
      if (live >= BLK) {
        if (lane == 0) {
          mbar_arrive_expect_tx(&sm.k_full[st], BLK * ROW_BYTES);
          tma_load_2d(sm.k[st], &kmap, &sm.k_full[st], 0, kbase + b * BLK);
        }
      } else {  // a sequence's partial last block: only the rows that exist
        for (int i = lane; i < BLK * 8; i += 32) {
          const int r = i >> 3, c = i & 7;
          if (r < live)
            cp_async_16(sk[st] + sw128_offset(r, c), k + (size_t)(kbase + b * BLK + r) * D + c * 8);
          else
            *reinterpret_cast<uint4 *>(sm.k[st] + sw128_offset(r, c)) = make_uint4(0u, 0u, 0u, 0u);
        }
        cp_async_wait_all();
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.k_full[st]);
      }
    };
    if (lane == 0) {
      mbar_arrive_expect_tx(&sm.bar_q, BLK * ROW_BYTES);
      tma_load_2d(sm.q, &qmap, &sm.bar_q, 0, first);
    }
    load(0);
    if (steps > 1) load(1);
    const uint32_t id = idesc_bf16_f32(BLK, BLK);
    for (int it = 0; it < steps; it++) {
      const int st = it & 1;
      if (lane == 0) {
        if (it == 0) mbar_wait(&sm.bar_q, 0, status);
        mbar_wait(&sm.k_full[st], (uint32_t)((it >> 1) & 1), status);
        if (it >= 2) mbar_wait(&sm.acc_empty[st], (uint32_t)(((it - 2) >> 1) & 1), status);
        tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(st * BLK);
#pragma unroll
        for (int kk = 0; kk < 4; kk++)
          umma_bf16(d, sdesc_k_sw128(sq + kk * 32), sdesc_k_sw128(sk[st] + kk * 32), id, kk > 0);
        umma_commit(&sm.acc_full[st]);
        umma_commit(&sm.k_empty[st]);
      }
      __syncwarp();
      if (it + 2 < steps) load(it + 2);
    }
  } else {
    // ------- epilogue warps: threads qi and qi + 128 own query row first + qi -------
    uint32_t *hist = sm.hist + qi * (DSA_TC_NB + 1);
    // named barrier 1: the eight epilogue warps (between the passes and at the end)
    auto epi_sync = [] { asm volatile("bar.sync 1, %0;" ::"n"(DSA_TC_EPI) : "memory"); };
    mbar_wait(&sm.bar_q, 0, status);
    float R = 0.f, inv = 0.f;
    if (active) {  // |q| from the staged tile (row qi, 128-byte swizzle)
      float qq = 0.f;
#pragma unroll
      for (int c = 0; c < 8; c++) {
        const uint4 w = *reinterpret_cast<const uint4 *>(sm.q + sw128_offset(qi, c));
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int u = 0; u < 4; u++) {
          qq = fmaf(bf_lo(ws[u]), bf_lo(ws[u]), qq);
          qq = fmaf(bf_hi(ws[u]), bf_hi(ws[u]), qq);
        }
      }
      R = sqrtf(qq) * __ldg(kmax + s) * (1.0f + 1.0f / 1024.0f);
    }
    const int pos = len - qlen + (row - q0);
    if (active) {
      // A query with more than 4k candidates keeps under a quarter of them, so for a
      // score distribution symmetric about 0 its k-th best score is well above 0: the
      // buckets then cover [0, R] (twice as fine) and lower scores share the last one.
      // A k-th score below 0 only makes that last bucket the boundary one: every
      // candidate is kept, the list overflows and the exact fallback takes the row.
      const float lo = pos + 1 > 4 * topk ? 0.f : -R;
      inv = R > 0.f ? (float)DSA_TC_NB / (R - lo) : 0.f;
    }
    int counted = 0;                          // scores this thread counted in pass 1
    float thr = -__int_as_float(0x7f800000);  // pass 2 keeps the scores >= thr
    float *bk = buf_key + (size_t)(row - row0) * cap;
    int32_t *bj = buf_j + (size_t)(row - row0) * cap;
    const int cbeg = half * (BLK / 2), cend = cbeg + BLK / 2;  // this thread's columns
    for (int it = 0; it < steps; it++) {
      const int st = it & 1;
      if (it == ns) {
        // between the passes (both threads of every query are done with pass 1):
        // bucket of the k-th best score, or of the best scaled share of the sampled
        // scores with a margin
        if (active) atomicAdd(&sm.qseen[qi], counted);
        epi_sync();
        if (active && half == 0) {
          const int seen = sm.qseen[qi];
          const int target =
              ss == 1 ? topk
                      : min(seen, (int)ceilf(DSA_MARGIN * (float)topk * (float)seen /
                                             (float)(pos + 1)) + DSA_SLACK);
          int bstar = DSA_TC_NB - 1, cum = 0;
          for (int q = 0; q < DSA_TC_NB; q++) {
            cum += (int)hist[q];
            if (cum >= target) {
              bstar = q;
              break;
            }
          }
          // every score of buckets 0..b* is above R - (b* + 1) / inv; the threshold sits
          // a little lower, so that rounding can only add candidates (the select is
          // exact over any superset of the top-k)
          if (bstar < DSA_TC_NB - 1 && inv > 0.f)
            sm.qthr[qi] = R - (float)(bstar + 1) / inv - R * (1.0f / 65536.0f);
        }
        epi_sync();
        thr = sm.qthr[qi];
      }
      mbar_wait(&sm.acc_full[st], (uint32_t)((it >> 1) & 1), status);
      tc_fence_after();
      const int b = it < ns ? it * ss : it - ns;
      const bool pass2 = it >= ns;
      const int jmax = active ? pos - b * BLK : -1;  // keys 0..jmax of this block are causal
      for (int c32 = cbeg; c32 < cend; c32 += 32) {
        // 32 columns per wait: two TMEM loads in flight
        uint32_t vv[2][16];
        tmem_ld16(tmem + ((uint32_t)((warp & 3) * 32) << 16) + (uint32_t)(st * BLK + c32), vv[0]);
        tmem_ld16(tmem + ((uint32_t)((warp & 3) * 32) << 16) + (uint32_t)(st * BLK + c32 + 16),
                  vv[1]);
        tmem_wait_ld();
#pragma unroll
        for (int h = 0; h < 2; h++) {
          const int c0 = c32 + 16 * h;
          const uint32_t *v = vv[h];
          if (c0 + 15 <= jmax) {  // the whole chunk is causal
            if (!pass2) {
#pragma unroll
              for (int u = 0; u < 16; u++) atomicAdd(&hist[dsa_bucket(__uint_as_float(v[u]), R, inv)], 1u);
              counted += 16;
            } else {
#pragma unroll
              for (int u = 0; u < 16; u++) {
                const float sc = __uint_as_float(v[u]);
                if (sc >= thr) {
                  const int p = atomicAdd(&sm.qcount[qi], 1);
                  if (p < cap) {
                    bk[p] = sc;
                    bj[p] = b * BLK + c0 + u;
                  }
                }
              }
            }
          } else if (c0 <= jmax) {  // the diagonal chunk
#pragma unroll
            for (int u = 0; u < 16; u++) {
              if (c0 + u <= jmax) {
                const float sc = __uint_as_float(v[u]);
                if (!pass2) {
                  atomicAdd(&hist[dsa_bucket(sc, R, inv)], 1u);
                  counted++;
                } else if (sc >= thr) {
                  const int p = atomicAdd(&sm.qcount[qi], 1);
                  if (p < cap) {
                    bk[p] = sc;
                    bj[p] = b * BLK + c0 + u;
                  }
                }
              }
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&sm.acc_empty[st]);
    }
    epi_sync();  // both threads of every query have appended
    // fewer candidates than the top-k needs (a sampled threshold set too high): the
    // list is not a superset, so the row goes to the exact fallback like an overflow
    if (active && half == 0) {
      const int count = sm.qcount[qi];
      cnt_out[row - row0] = count < min(topk, pos + 1) ? cap + 1 : count;
    }
  }
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, DSA_TC_TMEM_COLS);
}

// ---------------------------------------------------------------------------
// host side

bool make_rows_tensor_map(CUtensorMap *map, const void *base, uint64_t rows, uint32_t box_rows);
bool make_key_tensor_map(CUtensorMap *map, const uint16_t *k);

cudaError_t launch_dsa_filter_tc(const uint16_t *q, const uint16_t *k, const int32_t *cu_q,
                                 const int32_t *cu_k, const int32_t *seqlens, int S, int total_q,
                                 int row0, int nrows, int topk, int cap, const float *kmax,
                                 float *buf_key, int32_t *buf_j, int32_t *cnt, int *status,
                                 cudaStream_t st) {
  CUtensorMap qmap, kmap;
  if (!make_rows_tensor_map(&qmap, q, (uint64_t)total_q, BLK) || !make_key_tensor_map(&kmap, k))
    return cudaErrorInvalidValue;
  static std::atomic<int> attr[64];
  cudaError_t e = set_smem_once((const void *)dsa_filter_tc_kernel, DSA_TC_SMEM, attr);
  if (e != cudaSuccess) return e;
  const int tiles = (nrows + BLK - 1) / BLK + S;  // per-sequence tiles, upper bound
  ProfScope ps(K_DSA_FILTER, st);
  dsa_filter_tc_kernel<<<tiles, DSA_TC_THREADS, DSA_TC_SMEM, st>>>(
      qmap, kmap, k, cu_q, cu_k, seqlens, S, row0, nrows, topk, cap, kmax, buf_key, buf_j, cnt,
      status);
  return cudaGetLastError();
}

}  // namespace hisa
