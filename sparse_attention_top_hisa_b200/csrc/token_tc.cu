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

// Query rows are processed in chunks (see tc_chunking); the lists are kept per (chunk,
// compact key block).  The (query, slot) pairs of a range of INV_ROWS consecutive query
// rows are first aggregated per compact key block in shared memory, so that global atomics are
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
inv_lists_kernel(const int32_t *__restrict__ blk, int total_q, int m, int sb, int chunk_rows,
                 int nb, const int32_t *__restrict__ cu_q, int S, int emax, int mode,
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
  // the counters of a chunk of query rows follow those of the previous chunk; a CTA's
  // rows lie in one chunk (chunk_rows is a multiple of INV_ROWS)
  const int cbase = (r0 / chunk_rows) * nb;
  const int base = cbase + s0 * emax;
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
          if (b[u] >= 0) fn(rb + u * NW, slot, cbase + sq[u] * emax + b[u]);
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

// One CTA per chunk of query rows: list offsets of the chunk's key blocks (the chunk's
// list region starts at list_stride * chunk) and its tile descriptors (tile region at
// tile_stride * chunk), and the chunk's tile count.
__global__ void __launch_bounds__(SCAN_THREADS)
inv_scan_kernel(const int *__restrict__ cnt, int nb, long long list_stride, int tile_stride,
                int *__restrict__ cursor, TileDesc *__restrict__ tiles,
                int *__restrict__ ntiles) {
  __shared__ int warp_tot[SCAN_THREADS / 32 + 1];
  const int chunk = blockIdx.x;
  cnt += (size_t)chunk * nb;
  cursor += (size_t)chunk * nb;
  tiles += (size_t)chunk * tile_stride;
  const int per = (nb + SCAN_THREADS - 1) / SCAN_THREADS;
  const int b0 = threadIdx.x * per, b1 = min(nb, b0 + per);
  int sc = 0, st = 0;
  for (int i = b0; i < b1; i++) {
    const int c = cnt[i];
    sc += c;
    st += (c + TC_N - 1) / TC_N;
  }
  int total_c, total_t;
  int oc = (int)(list_stride * chunk) + block_exclusive_scan<SCAN_THREADS>(sc, warp_tot, &total_c);
  int ot = block_exclusive_scan<SCAN_THREADS>(st, warp_tot, &total_t);
  // Tile descriptors: the warp writes its lanes' blocks one after another, 32
  // descriptors per store instruction (one block can own several tiles: block 0 is
  // selected by every query).
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
  if (threadIdx.x == 0) ntiles[chunk] = total_t;
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
                      int list_base, float *__restrict__ scratch, int *status,
                      int *launch_abort, int test_no_loads) {
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
                scratch[(size_t)(td.list_off - list_base + c0 + u) * BLK + r] =
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

// Stage 2 can run over chunks of consecutive query rows, scoring then selecting one chunk
// at a time, with a score buffer of one chunk; each chunk's list region, tile
// descriptors and counters sit at fixed offsets, so no scan across chunks is needed.
// Chunks sized for L2 (tens of MB of scores) were measured slower than one chunk: each
// scoring and selecting launch pays its ramp and tail, which outweighed the HBM traffic
// saved (10.2 ms against 5.7 ms per 131072-query step with 1024-row chunks).  So the
// whole batch is one chunk unless its score buffer would exceed kChunkScoreBytes.
constexpr size_t kChunkScoreBytes = (size_t)64 << 30;

struct TcChunks {
  int rows;     // query rows per chunk (a multiple of INV_ROWS)
  int nchunks;
};

TcChunks tc_chunking(int total_q, int m) {
  TcChunks c;
  long long rows = (long long)(kChunkScoreBytes / ((size_t)m * BLK * 4));
  rows = rows / INV_ROWS * INV_ROWS;
  if (rows < INV_ROWS) rows = INV_ROWS;
  const long long whole = ((long long)total_q + INV_ROWS - 1) / INV_ROWS * INV_ROWS;
  if (rows > whole) rows = whole > 0 ? whole : INV_ROWS;
  c.rows = (int)rows;
  c.nchunks = (int)((total_q + rows - 1) / rows);
  if (c.nchunks < 1) c.nchunks = 1;
  return c;
}

struct TcPlan {
  size_t off_cnt, off_cursor, off_ntiles, off_tiles, off_list, off_pmap, off_scores, total;
  int nb;            // counters per chunk (sequences x blocks)
  int tile_stride;   // tile descriptors reserved per chunk
  long long list_stride;  // list entries reserved per chunk (rows x m)
  TcChunks ch;
};

static size_t a256(size_t x) { return (x + 255) & ~(size_t)255; }

TcPlan tc_plan(int total_q, int num_seqs, int max_seqlen_k, int m) {
  TcPlan p;
  const int emax = (max_seqlen_k + BLK - 1) / BLK;
  p.ch = tc_chunking(total_q, m);
  p.nb = (num_seqs > 0 ? num_seqs : 1) * (emax > 0 ? emax : 1);
  p.list_stride = (long long)p.ch.rows * m;
  p.tile_stride = (int)(p.list_stride / TC_N + p.nb + 1);
  const long long pairs = (long long)total_q * m;
  const size_t nbt = (size_t)p.nb * p.ch.nchunks;
  size_t off = 0;
  p.off_cnt = off;  // every chunk's counters, then the launch's abort word
  off = a256(off + (nbt + 1) * 4);
  p.off_cursor = off;
  off = a256(off + nbt * 4);
  p.off_ntiles = off;
  off = a256(off + (size_t)p.ch.nchunks * 4);
  p.off_tiles = off;
  off = a256(off + (size_t)p.tile_stride * p.ch.nchunks * sizeof(TileDesc));
  p.off_list = off;
  off = a256(off + (size_t)p.list_stride * p.ch.nchunks * 4);
  p.off_pmap = off;
  off = a256(off + (size_t)pairs * 4);
  p.off_scores = off;  // one chunk's score segments
  off = a256(off + (size_t)p.list_stride * BLK * 4);
  p.total = off;
  return p;
}

size_t tc_workspace_bytes(int total_q, int num_seqs, int max_seqlen_k, int m) {
  return tc_plan(total_q, num_seqs, max_seqlen_k, m).total;
}

// Tests of the timeout path only (hisa_test_fault): launches made while it is set
// issue no loads.
std::atomic<int> g_test_no_loads{0};

// The chunked stage 2 of the tensor-core path, as carved from ws.
struct TcStage {
  TcPlan p;
  int emax, sb;
  int *cnt, *cursor, *ntiles, *launch_abort;
  TileDesc *tiles;
  uint32_t *list;
  int32_t *pmap;
  float *scores;
};

TcStage tc_stage(int total_q, int S, int max_seqlen_k, int m, uint8_t *ws) {
  TcStage t;
  t.p = tc_plan(total_q, S, max_seqlen_k, m);
  t.emax = (max_seqlen_k + BLK - 1) / BLK;
  t.sb = m > 128 ? 9 : 7;  // slot bits of a list entry (row << sb | slot)
  t.cnt = reinterpret_cast<int *>(ws + t.p.off_cnt);
  t.cursor = reinterpret_cast<int *>(ws + t.p.off_cursor);
  t.ntiles = reinterpret_cast<int *>(ws + t.p.off_ntiles);
  t.tiles = reinterpret_cast<TileDesc *>(ws + t.p.off_tiles);
  t.list = reinterpret_cast<uint32_t *>(ws + t.p.off_list);
  t.pmap = reinterpret_cast<int32_t *>(ws + t.p.off_pmap);
  t.scores = reinterpret_cast<float *>(ws + t.p.off_scores);
  t.launch_abort = t.cnt + (size_t)t.p.nb * t.p.ch.nchunks;
  return t;
}

// Every chunk's (query, slot) lists and tile descriptors.
cudaError_t launch_token_lists(const TcStage &t, const int32_t *cu_q, int S, int total_q, int m,
                               const int32_t *blk, cudaStream_t st) {
  const size_t nbt = (size_t)t.p.nb * t.p.ch.nchunks;
  cudaError_t e = cudaMemsetAsync(t.cnt, 0, (nbt + 1) * 4, st);
  if (e != cudaSuccess) return e;
  const int grid = (total_q + INV_ROWS - 1) / INV_ROWS;
  {
    ProfScope ps(K_INV_LISTS, st);
    inv_lists_kernel<<<grid, INV_THREADS, 0, st>>>(blk, total_q, m, t.sb, t.p.ch.rows, t.p.nb,
                                                   cu_q, S, t.emax, 0, t.cnt, t.cursor, t.list,
                                                   t.pmap);
  }
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  {
    ProfScope ps(K_INV_SCAN, st);
    inv_scan_kernel<<<t.p.ch.nchunks, SCAN_THREADS, 0, st>>>(t.cnt, t.p.nb, t.p.list_stride,
                                                              t.p.tile_stride, t.cursor, t.tiles,
                                                              t.ntiles);
  }
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  {
    ProfScope ps(K_INV_LISTS, st);
    inv_lists_kernel<<<grid, INV_THREADS, 0, st>>>(blk, total_q, m, t.sb, t.p.ch.rows, t.p.nb,
                                                   cu_q, S, t.emax, 1, t.cnt, t.cursor, t.list,
                                                   t.pmap);
  }
  return cudaGetLastError();
}

// Scores the selected (query, block) pairs of one chunk into the chunk score buffer:
// the segment of list entry p is segment p - chunk * list_stride.
cudaError_t launch_token_score_chunk(const TcStage &t, int chunk, const uint16_t *q,
                                     const uint16_t *k, const int32_t *cu_q, const int32_t *cu_k,
                                     const int32_t *seqlens, int num_sms, int *status,
                                     cudaStream_t st) {
  static std::atomic<int> attr[64];
  cudaError_t e = set_smem_once((const void *)token_score_tc_kernel, TC_SMEM_BYTES, attr);
  if (e != cudaSuccess) return e;
  ProfScope ps(K_TOKEN_SCORE_TC, st);
  token_score_tc_kernel<<<num_sms, TC_THREADS, TC_SMEM_BYTES, st>>>(
      q, k, cu_q, cu_k, seqlens, t.emax, t.sb, t.tiles + (size_t)chunk * t.p.tile_stride,
      t.ntiles + chunk, t.list, (int)(t.p.list_stride * chunk), t.scores, status, t.launch_abort,
      g_test_no_loads.load(std::memory_order_relaxed));
  return cudaGetLastError();
}

cudaError_t launch_select_rows(const int32_t *cu_q, const int32_t *cu_k, const int32_t *seqlens,
                               const int32_t *m_seq, int S, int m, int topk, const int32_t *blk,
                               const float *scores, const int32_t *pmap, int list_base,
                               const int *launch_abort, int row0, int nrows, bool split,
                               int32_t *out_idx, float *out_scores, cudaStream_t st);

// Stage 2 on the tensor-core path: every chunk's lists, then per chunk its scores and
// the exact select of its rows (stream order keeps one chunk's segments in the buffer).
cudaError_t launch_token_stage_tc(const uint16_t *q, const uint16_t *k, const int32_t *cu_q,
                                  const int32_t *cu_k, const int32_t *seqlens,
                                  const int32_t *m_seq, int S, int total_q, int max_seqlen_k,
                                  int m, int topk, const int32_t *blk, uint8_t *ws, int num_sms,
                                  int32_t *out_idx, float *out_scores, int *status,
                                  cudaStream_t st) {
  const TcStage t = tc_stage(total_q, S, max_seqlen_k, m, ws);
  cudaError_t e = launch_token_lists(t, cu_q, S, total_q, m, blk, st);
  if (e != cudaSuccess) return e;
  for (int c = 0; c < t.p.ch.nchunks; c++) {
    e = launch_token_score_chunk(t, c, q, k, cu_q, cu_k, seqlens, num_sms, status, st);
    if (e != cudaSuccess) return e;
    const int row0 = c * t.p.ch.rows;
    e = launch_select_rows(cu_q, cu_k, seqlens, m_seq, S, m, topk, blk, t.scores, t.pmap,
                           (int)(t.p.list_stride * c), t.launch_abort, row0,
                           min(t.p.ch.rows, total_q - row0), false, out_idx, out_scores, st);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace hisa
