// Stage 2 of HISA on the tensor cores: block-major gather-scoring.
//
// HISA summary page (aitrends.kr), paragraph on stage 2: every query scores the
// tokens of its m selected blocks with the original DSA dot product.  Grouped by
// key block instead of by query, this is a dense contraction: for key block b and
// the queries that selected it, S = K_b [128 x 64] . Q_sel^T [64 x N].  Each key
// block then crosses the memory hierarchy once per 256 selecting queries instead of
// once per query.
//
//   1. inv_lists_kernel (count, then fill): the (query, slot) pairs are bucketed by
//      key block, with warp-aggregated atomics (block 0 is selected by every query);
//   2. inv_scan_kernel: list offsets per key block and tile descriptors (one tile =
//      one key block and up to 256 of its selecting queries);
//   3. token_score_tc_kernel: persistent, warp-specialised CTAs (one per SM).  Per
//      tile the key block arrives by TMA (or by cp.async when it is the partial last
//      block of a sequence) and the selecting queries are gathered with cp.async into
//      the 128-byte-swizzled K-major layout, through a three-stage shared-memory ring
//      filled by three loader warps (each with two tiles' copies in flight).  One thread issues the tcgen05.mma chain
//      S = K_b [128 x 64] . Q_sel^T [64 x N] (K = 4 x 16, N <= 256) into one of two
//      TMEM accumulators, so that the loads, the MMAs and the epilogue of
//      consecutive tiles overlap.  The accumulator lane is the key row: each of the
//      eight epilogue warps owns 32 key rows (TMEM lane quarter w % 4) of half of the
//      queries (w / 4).  The scores of list entry p (a (query, slot) pair) go to
//      segment p of the score buffer (128 fp32), so a tile writes one contiguous run of
//      segments and every store instruction one 128-byte line of it;
//   4. the exact select of token_select.cu reads the score rows.
// Key j of block b is admitted for a query at position i only when j <= i.
#include <cudaTypedefs.h>

#include "prof.cuh"
#include "tc.cuh"

namespace hisa {

constexpr int TC_N = 256;  // selecting queries per tile (two MMA chains of M = 128, at most)

struct TileDesc {
  int list_off;  // first list entry of the tile
  int cb;        // compact key block: sequence * emax + block
  int n;         // entries in the tile (1..TC_N)
  int pad;
};

constexpr int TC_STAGES = 3;       // shared-memory ring depth
constexpr int TC_EPI_WARPS = 8;    // epilogue: warp w owns TMEM lanes 32 (w % 4).., queries half w / 4
constexpr int TC_MMA_WARP = TC_EPI_WARPS;
constexpr int TC_LOAD_WARP0 = TC_EPI_WARPS + 1;
constexpr int TC_LOAD_WARPS = 3;
constexpr int TC_LOADERS = TC_LOAD_WARPS * 32;
constexpr int TC_THREADS = (TC_EPI_WARPS + 1 + TC_LOAD_WARPS) * 32;
constexpr uint32_t TC_TMEM_COLS = 512;  // two accumulators of 256 columns

struct TcSmem {
  uint8_t q[TC_STAGES][TC_N * ROW_BYTES];  // gathered queries (MMA B), 1024-byte aligned
  uint8_t k[TC_STAGES][BLK * ROW_BYTES];   // key block (MMA A)
  uint64_t full[TC_STAGES], empty[TC_STAGES], acc_full[2], acc_empty[2];
  uint32_t tmem_base;
  int abort;
};
constexpr size_t TC_SMEM_BYTES = sizeof(TcSmem) + 1024;

// ---------------------------------------------------------------------------
// inverted lists

// The (query, slot) pairs of a range of INV_ROWS consecutive query rows are first
// aggregated per compact key block in shared memory, so that global atomics are
// issued once per (CTA, key block) instead of once per pair.  A CTA whose rows span
// more compact blocks than fit in shared memory uses global atomics directly.
//   mode 0: add the pair counts of every key block to cnt;
//   mode 1: reserve each key block's share of its list (cursor holds the list
//           starts), write the entries row << sb | slot, and record each pair's list
//           position in pmap[row * m + slot] (where its scores will be).
// Slots past a row's block budget hold -1 and are skipped.
constexpr int INV_THREADS = 256;
constexpr int INV_ROWS = 256;
constexpr int INV_LOCAL_BINS = 8192;
constexpr int INV_RB = 8;  // rows whose block ids a warp loads at once

__global__ void __launch_bounds__(INV_THREADS)
inv_lists_kernel(const int32_t *__restrict__ blk, int total_q, int m, int sb,
                 const int32_t *__restrict__ cu_q, int S, int emax, int mode,
                 int *__restrict__ cnt, int *__restrict__ cursor, uint32_t *__restrict__ list,
                 int32_t *__restrict__ pmap) {
  __shared__ int loc[INV_LOCAL_BINS];
  __shared__ int seq_range[2];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int NW = INV_THREADS / 32;
  const int r0 = blockIdx.x * INV_ROWS, r1 = min(total_q, r0 + INV_ROWS);
  if (tid == 0) {
    seq_range[0] = find_seq(cu_q, S, r0);
    seq_range[1] = find_seq(cu_q, S, r1 - 1);
  }
  __syncthreads();
  const int s0 = seq_range[0], s1 = seq_range[1];
  const int base = s0 * emax;
  const int nbl = (s1 - s0 + 1) * emax;
  const bool local = nbl <= INV_LOCAL_BINS;
  // walk the pairs: warp w takes rows r0 + w, r0 + w + NW, ...; lane = slot within a
  // chunk of 32 slots.  The block ids of INV_RB rows are loaded before any is used, so
  // that a warp keeps that many loads in flight instead of one.
  auto walk = [&](auto &&fn) {
    int s = s0;
    for (int rb = r0 + warp; rb < r1; rb += NW * INV_RB) {
      int sq[INV_RB];
#pragma unroll
      for (int u = 0; u < INV_RB; u++) {
        const int row = rb + u * NW;
        if (row < r1)
          while (s < s1 && __ldg(cu_q + s + 1) <= row) s++;
        sq[u] = s;
      }
      for (int c0 = 0; c0 < m; c0 += 32) {
        const int slot = c0 + lane;
        int b[INV_RB];
#pragma unroll
        for (int u = 0; u < INV_RB; u++) {
          const int row = rb + u * NW;
          b[u] = (row < r1 && slot < m) ? __ldg(blk + (size_t)row * m + slot) : -1;
        }
#pragma unroll
        for (int u = 0; u < INV_RB; u++)
          if (b[u] >= 0) fn(rb + u * NW, slot, sq[u] * emax + b[u]);
      }
    }
  };
  if (!local) {  // wide row range: global atomics per pair
    if (mode == 0)
      walk([&](int, int, int cb) { atomicAdd(cnt + cb, 1); });
    else
      walk([&](int row, int slot, int cb) {
        const int p = atomicAdd(cursor + cb, 1);
        list[p] = ((uint32_t)row << sb) | (uint32_t)slot;
        pmap[(size_t)row * m + slot] = p;
      });
    return;
  }
  for (int i = tid; i < nbl; i += INV_THREADS) loc[i] = 0;
  __syncthreads();
  walk([&](int, int, int cb) { atomicAdd(&loc[cb - base], 1); });
  __syncthreads();
  if (mode == 0) {
    for (int i = tid; i < nbl; i += INV_THREADS)
      if (loc[i]) atomicAdd(cnt + base + i, loc[i]);
    return;
  }
  for (int i = tid; i < nbl; i += INV_THREADS)
    if (loc[i]) loc[i] = atomicAdd(cursor + base + i, loc[i]);
  __syncthreads();
  walk([&](int row, int slot, int cb) {
    const int p = atomicAdd(&loc[cb - base], 1);
    list[p] = ((uint32_t)row << sb) | (uint32_t)slot;
    pmap[(size_t)row * m + slot] = p;
  });
}

constexpr int SCAN_THREADS = 1024;

__global__ void __launch_bounds__(SCAN_THREADS)
inv_scan_kernel(const int *__restrict__ cnt, int nb, int *__restrict__ cursor,
                TileDesc *__restrict__ tiles, int *__restrict__ ntiles) {
  __shared__ int warp_tot[SCAN_THREADS / 32 + 1];
  const int per = (nb + SCAN_THREADS - 1) / SCAN_THREADS;
  const int b0 = threadIdx.x * per, b1 = min(nb, b0 + per);
  int sc = 0, st = 0;
  for (int i = b0; i < b1; i++) {
    const int c = cnt[i];
    sc += c;
    st += (c + TC_N - 1) / TC_N;
  }
  int total_c, total_t;
  int oc = block_exclusive_scan<SCAN_THREADS>(sc, warp_tot, &total_c);
  int ot = block_exclusive_scan<SCAN_THREADS>(st, warp_tot, &total_t);
  // Tile descriptors: the warp writes its lanes' blocks one after another, 32
  // descriptors per store instruction (one block can own hundreds of tiles: block 0
  // is selected by every query).
  const int lane = threadIdx.x & 31;
  for (int j = 0; j < per; j++) {
    const int i = b0 + j;
    const int c = i < b1 ? cnt[i] : 0;
    if (i < b1) cursor[i] = oc;
    const int nt = (c + TC_N - 1) / TC_N;
    for (int src = 0; src < 32; src++) {
      const int si = __shfl_sync(0xffffffffu, i, src);
      const int sc_ = __shfl_sync(0xffffffffu, c, src);
      const int soc = __shfl_sync(0xffffffffu, oc, src);
      const int sot = __shfl_sync(0xffffffffu, ot, src);
      const int snt = __shfl_sync(0xffffffffu, nt, src);
      for (int t = lane; t < snt; t += 32) {
        TileDesc d;
        d.list_off = soc + t * TC_N;
        d.cb = si;
        d.n = min(TC_N, sc_ - t * TC_N);
        d.pad = 0;
        tiles[sot + t] = d;
      }
    }
    oc += c;
    ot += nt;
  }
  if (threadIdx.x == 0) *ntiles = total_t;
}

// ---------------------------------------------------------------------------
// tensor-core scoring

struct TileSeq {
  int b, kbase, len, pos_off;  // key block, region start, live keys, position = row + pos_off
};

__device__ __forceinline__ TileSeq tile_seq(const TileDesc &td, int emax, const int32_t *cu_q,
                                            const int32_t *cu_k, const int32_t *seqlens) {
  TileSeq r;
  const int s = td.cb / emax;
  r.b = td.cb - s * emax;
  r.kbase = __ldg(cu_k + s);
  r.len = seqlens ? __ldg(seqlens + s) : __ldg(cu_k + s + 1) - r.kbase;
  const int q0 = __ldg(cu_q + s);
  r.pos_off = r.len - (__ldg(cu_q + s + 1) - q0) - q0;
  return r;
}

__global__ void __launch_bounds__(TC_THREADS, 1)
token_score_tc_kernel(const uint16_t *__restrict__ q,
                      const uint16_t *__restrict__ k, const int32_t *__restrict__ cu_q,
                      const int32_t *__restrict__ cu_k, const int32_t *__restrict__ seqlens,
                      int emax, int sb, const TileDesc *__restrict__ tiles,
                      const int *__restrict__ ntiles_ptr, const uint32_t *__restrict__ list,
                      float *__restrict__ scratch, int *status, int *launch_abort,
                      int test_no_loads) {
  extern __shared__ uint8_t tc_smem_raw[];
  TcSmem &sm = *reinterpret_cast<TcSmem *>((reinterpret_cast<uintptr_t>(tc_smem_raw) + 1023) &
                                           ~(uintptr_t)1023);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int i = 0; i < TC_STAGES; i++) {
      mbar_init(&sm.full[i], TC_LOADERS);  // every loader thread, once its copies landed
      mbar_init(&sm.empty[i], 1);
    }
    for (int i = 0; i < 2; i++) {
      mbar_init(&sm.acc_full[i], 1);
      mbar_init(&sm.acc_empty[i], TC_EPI_WARPS * 32);
    }
    sm.abort = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(&sm.tmem_base, TC_TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  const int ntiles = *ntiles_ptr;
  volatile int *abort_flag = &sm.abort;

  if (warp >= TC_LOAD_WARP0) {
    // ---------------- loaders: key block (TMA or cp.async) and query gather ----------------
    const int lt = tid - TC_LOAD_WARP0 * 32;
    int i = 0;
    // test_no_loads (tests of the timeout path only): the loaders issue nothing, so the
    // MMA thread's first wait runs out with no copy and no MMA in flight
    for (int t = test_no_loads ? ntiles : blockIdx.x; t < ntiles; t += gridDim.x, i++) {
      const int s = i % TC_STAGES;
      const TileDesc td = tiles[t];  // fetched while the stage drains
      const TileSeq ts = tile_seq(td, emax, cu_q, cu_k, seqlens);
      if (i >= TC_STAGES &&
          !mbar_wait(&sm.empty[s], (uint32_t)(((i / TC_STAGES) & 1) ^ 1), status, abort_flag)) {
        *abort_flag = 1;
        atomicExch(launch_abort, 1);
        break;
      }
      if (*abort_flag) break;
      const int live = min(BLK, ts.len - ts.b * BLK);
      const uint32_t sq = smem_u32(sm.q[s]), sk = smem_u32(sm.k[s]);
      // the key block, by cp.async like the queries, so that one wait_all covers every
      // copy a loader has in flight; a partial last block loads only the rows that
      // exist (the others are masked)
      for (int x = lt; x < live * 8; x += TC_LOADERS) {
        const int r = x >> 3, c = x & 7;
        cp_async_16(sk + sw128_offset(r, c), k + (size_t)(ts.kbase + ts.b * BLK + r) * D + c * 8);
      }
      // the selecting queries, in chunks of 32 rows (chunk c is loaded by loader warp
      // c % TC_LOAD_WARPS): one coalesced read of the chunk's list entries, then lane l
      // copies 16-byte piece l % 8 of row 4 i + l / 8 for i = 0..7.  Rows past n stay
      // stale (their accumulator columns are ignored).
      {
        const int lw = lt >> 5;
        constexpr int MAXC = (TC_N / 32 + TC_LOAD_WARPS - 1) / TC_LOAD_WARPS;
        uint32_t ent[MAXC];
#pragma unroll
        for (int j = 0; j < MAXC; j++) {
          const int row = (lw + j * TC_LOAD_WARPS) * 32 + lane;
          ent[j] = row < td.n ? __ldg(list + td.list_off + row) : 0u;
        }
#pragma unroll
        for (int j = 0; j < MAXC; j++) {
          const int c = lw + j * TC_LOAD_WARPS;
          if (c * 32 < td.n) {  // warp-uniform
#pragma unroll
            for (int i2 = 0; i2 < 8; i2++) {
              const int rl = i2 * 4 + (lane >> 3), row = c * 32 + rl, piece = lane & 7;
              const uint32_t e = __shfl_sync(0xffffffffu, ent[j], rl);
              if (row < td.n)
                cp_async_16(sq + sw128_offset(row, piece), q + (size_t)(e >> sb) * D + piece * 8);
            }
          }
        }
      }
      // two tiles in flight: tile i's copies were just issued; tile i - 1's are
      // waited for here and its stage released to the MMA thread
      cp_async_commit();
      if (i > 0) {
        cp_async_wait_group1();
        fence_proxy_async_smem();
        mbar_arrive(&sm.full[(i - 1) % TC_STAGES]);
      }
    }
    if (i > 0) {  // the last tile issued; after an abort, every copy still lands first
      cp_async_wait_all();
      fence_proxy_async_smem();
      if (!*abort_flag) mbar_arrive(&sm.full[(i - 1) % TC_STAGES]);
    }
  } else if (warp == TC_MMA_WARP) {
    // ---------------- MMA issue (one thread) ----------------
    if (lane == 0) {
      int i = 0;
      for (int t = blockIdx.x; t < ntiles; t += gridDim.x, i++) {
        const int s = i % TC_STAGES, a = i & 1;
        const int n = tiles[t].n;
        if (!mbar_wait(&sm.full[s], (uint32_t)((i / TC_STAGES) & 1), status) ||
            (i >= 2 && !mbar_wait(&sm.acc_empty[a], (uint32_t)(((i >> 1) & 1) ^ 1), status))) {
          *abort_flag = 1;
          atomicExch(launch_abort, 1);  // the select pads every row of this launch
          break;
        }
        if (*abort_flag) break;
        tc_fence_after();
        const uint32_t sq = smem_u32(sm.q[s]), sk = smem_u32(sm.k[s]);
        const uint32_t id = idesc_bf16_f32(BLK, (n + 15) & ~15);
#pragma unroll
        for (int kk = 0; kk < 4; kk++)
          umma_bf16(tmem + (uint32_t)(a * 256), sdesc_k_sw128(sk + kk * 32),
                    sdesc_k_sw128(sq + kk * 32), id, kk > 0);
        umma_commit(&sm.empty[s]);
        umma_commit(&sm.acc_full[a]);
      }
      // before the CTA frees TMEM, the last issued product (and so every earlier one)
      // has completed, also when the loop above gave up
      if (i > 0) mbar_wait(&sm.acc_full[(i - 1) & 1], (uint32_t)(((i - 1) >> 1) & 1), status);
    }
    __syncwarp();
  } else {
    // ---------------- epilogue: thread = key row of the block ----------------
    const int h = warp >> 2, quarter = warp & 3;
    const int r = quarter * 32 + lane;  // key row of the block
    const float NEG = -__int_as_float(0x7f800000);
    int i = 0;
    for (int t = blockIdx.x; t < ntiles; t += gridDim.x, i++) {
      const int a = i & 1;
      const TileDesc td = tiles[t];
      const int c_beg = h * 128, c_end = min(td.n, c_beg + 128);
      // the list entries of this warp's queries, fetched while the MMA runs:
      // entry c_beg + 32 j + lane in ej[j]
      uint32_t ej[4];
#pragma unroll
      for (int j = 0; j < 4; j++) {
        const int c = c_beg + 32 * j + lane;
        ej[j] = c < c_end ? __ldg(list + td.list_off + c) : 0u;
      }
      if (!mbar_wait(&sm.acc_full[a], (uint32_t)((i >> 1) & 1), status, abort_flag)) {
        *abort_flag = 1;
        atomicExch(launch_abort, 1);
        break;
      }
      tc_fence_after();
      if (c_beg < c_end) {  // warp-uniform
        const TileSeq ts = tile_seq(td, emax, cu_q, cu_k, seqlens);
        const int rlim = ts.b * BLK + r - ts.pos_off;  // key row r is causal for rows >= rlim
        const uint32_t taddr = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(a * 256);
#pragma unroll
        for (int j = 0; j < 4; j++) {
          const int c0 = c_beg + 32 * j;
          if (c0 < c_end) {  // warp-uniform
            uint32_t v[32];
            tmem_ld16(taddr + (uint32_t)c0, *reinterpret_cast<uint32_t(*)[16]>(&v[0]));
            tmem_ld16(taddr + (uint32_t)(c0 + 16), *reinterpret_cast<uint32_t(*)[16]>(&v[16]));
            tmem_wait_ld();
#pragma unroll
            for (int u = 0; u < 32; u++) {
              const uint32_t e = __shfl_sync(0xffffffffu, ej[j], u);
              if (c0 + u < c_end) {
                const int row = (int)(e >> sb);
                scratch[(size_t)(td.list_off + c0 + u) * BLK + r] =
                    row >= rlim ? __uint_as_float(v[u]) : NEG;
              }
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&sm.acc_empty[a]);
    }
  }
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, TC_TMEM_COLS);
}

// ---------------------------------------------------------------------------
// host side

static PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &qr) ==
            cudaSuccess &&
        qr == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 2-D map over rows of 64 bf16 (128 bytes each), boxes of box_rows rows, 128-byte
// swizzle (the K-major SW128 operand layout); rows past `rows` read as zero.
bool make_rows_tensor_map(CUtensorMap *map, const void *base, uint64_t rows, uint32_t box_rows) {
  auto enc = tensor_map_encoder();
  if (!enc || rows == 0) return false;
  cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)ROW_BYTES};
  cuuint32_t box[2] = {(cuuint32_t)D, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Map over the key rows.  Their count is not passed to hisa_select, so the extent is
// left open (2^31 rows): the kernel only asks for whole blocks that lie inside a
// sequence's live keys.
bool make_key_tensor_map(CUtensorMap *map, const uint16_t *k) {
  return make_rows_tensor_map(map, k, (uint64_t)1 << 31, BLK);
}

struct TcPlan {
  size_t off_cnt, off_cursor, off_ntiles, off_tiles, off_list, off_pmap, off_scores, total;
  int nb, max_tiles;
};

static size_t a256(size_t x) { return (x + 255) & ~(size_t)255; }

TcPlan tc_plan(int total_q, int num_seqs, int max_seqlen_k, int m) {
  TcPlan p;
  const int emax = (max_seqlen_k + BLK - 1) / BLK;
  p.nb = (num_seqs > 0 ? num_seqs : 1) * (emax > 0 ? emax : 1);
  const long long pairs = (long long)total_q * m;
  p.max_tiles = (int)(pairs / TC_N + p.nb + 1);
  size_t off = 0;
  p.off_cnt = off;  // nb counters, then the launch's abort word
  off = a256(off + (size_t)(p.nb + 1) * 4);
  p.off_cursor = off;
  off = a256(off + (size_t)p.nb * 4);
  p.off_ntiles = off;
  off = a256(off + 4);
  p.off_tiles = off;
  off = a256(off + (size_t)p.max_tiles * sizeof(TileDesc));
  p.off_list = off;
  off = a256(off + (size_t)pairs * 4);
  p.off_pmap = off;
  off = a256(off + (size_t)pairs * 4);
  p.off_scores = off;
  off = a256(off + (size_t)pairs * BLK * 4);
  p.total = off;
  return p;
}

size_t tc_workspace_bytes(int total_q, int num_seqs, int max_seqlen_k, int m) {
  return tc_plan(total_q, num_seqs, max_seqlen_k, m).total;
}

// Scores every selected (query, block) pair into ws's score buffer (one 128-score
// segment per list entry; *pmap_out[row * m + slot] names the segment of each pair),
// ready for the select kernel.
// Tests of the timeout path only (hisa_test_fault): launches made while it is set
// issue no loads.
std::atomic<int> g_test_no_loads{0};

cudaError_t launch_token_score_tc(const uint16_t *q, const uint16_t *k, const int32_t *cu_q,
                                  const int32_t *cu_k, const int32_t *seqlens, int S,
                                  int total_q, int max_seqlen_k, int m, const int32_t *blk,
                                  uint8_t *ws, float **scores_out, const int32_t **pmap_out,
                                  int **abort_out, int num_sms, int *status, cudaStream_t st) {
  const TcPlan p = tc_plan(total_q, S, max_seqlen_k, m);
  const int emax = (max_seqlen_k + BLK - 1) / BLK;
  int *cnt = reinterpret_cast<int *>(ws + p.off_cnt);
  int *cursor = reinterpret_cast<int *>(ws + p.off_cursor);
  int *ntiles = reinterpret_cast<int *>(ws + p.off_ntiles);
  TileDesc *tiles = reinterpret_cast<TileDesc *>(ws + p.off_tiles);
  uint32_t *list = reinterpret_cast<uint32_t *>(ws + p.off_list);
  float *scores = reinterpret_cast<float *>(ws + p.off_scores);
  int32_t *pmap = reinterpret_cast<int32_t *>(ws + p.off_pmap);
  *scores_out = scores;
  *pmap_out = pmap;
  int *launch_abort = cnt + p.nb;
  *abort_out = launch_abort;
  cudaError_t e = cudaMemsetAsync(cnt, 0, (size_t)(p.nb + 1) * 4, st);
  if (e != cudaSuccess) return e;
  const int grid = (total_q + INV_ROWS - 1) / INV_ROWS;
  const int sb = m > 128 ? 9 : 7;  // slot bits of a list entry (row << sb | slot)
  {
    ProfScope ps(K_INV_LISTS, st);
    inv_lists_kernel<<<grid, INV_THREADS, 0, st>>>(blk, total_q, m, sb, cu_q, S, emax, 0, cnt, cursor, list,
                                                   pmap);
  }
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  {
    ProfScope ps(K_INV_SCAN, st);
    inv_scan_kernel<<<1, SCAN_THREADS, 0, st>>>(cnt, p.nb, cursor, tiles, ntiles);
  }
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  {
    ProfScope ps(K_INV_LISTS, st);
    inv_lists_kernel<<<grid, INV_THREADS, 0, st>>>(blk, total_q, m, sb, cu_q, S, emax, 1, cnt, cursor, list,
                                                   pmap);
  }
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  static std::atomic<int> attr[64];
  if ((e = set_smem_once((const void *)token_score_tc_kernel, TC_SMEM_BYTES, attr)) != cudaSuccess)
    return e;
  {
    ProfScope ps(K_TOKEN_SCORE_TC, st);
    token_score_tc_kernel<<<num_sms, TC_THREADS, TC_SMEM_BYTES, st>>>(
        q, k, cu_q, cu_k, seqlens, emax, sb, tiles, ntiles, list, scores, status,
        launch_abort, g_test_no_loads.load(std::memory_order_relaxed));
  }
  return cudaGetLastError();
}

}  // namespace hisa
