// HISA selection for few queries (decode): one 8-CTA thread-block cluster per query.
//
// HISA summary page (aitrends.kr): stage 1 (paragraph on block filtering) scores
// the query against every eligible block representative and keeps the forced
// blocks plus the best others, m in all; stage 2 (paragraph on token refinement)
// scores the m * 128 tokens of those blocks and keeps the k best.  In decode there
// are too few queries to fill the GPU with one CTA each, so the work of one query
// is spread over the 8 CTAs of a cluster (on 8 SMs), which exchange data through
// distributed shared memory:
//   A. block scores: CTA c scores a contiguous share of the eligible blocks (eight
//      lanes per representative row, fp32) into order-preserving keys;
//   B. every CTA gathers all keys from the cluster and runs the same CTA-wide top-m
//      (linear score buckets, exact ranking of the boundary bucket; radix select on
//      heavy ties) on identical inputs, so no broadcast step is needed;
//   C. CTA c gathers and scores its share of the selected blocks' tokens straight
//      from HBM (four lanes per key row, 16 dims each, eight rows in flight per lane);
//   D. exact top-k across the cluster: global max / min / count, per-CTA bucket
//      histograms (1024 buckets linear in the score) summed across the cluster
//      with 16-byte remote loads, one scan for the bucket offsets and the boundary
//      bucket; every survivor is then stored (one remote store) at its bucket's
//      offset in the staging array of the CTA that owns the bucket (the CTAs split
//      the output positions evenly; the prefix of the lower-ranked CTAs' counts
//      keeps the slots disjoint), and each owner ranks its buckets from local memory;
//      the boundary bucket's members go to CTA 0, which ranks them.
// Every branch that skips a cluster barrier depends only on values all CTAs of the
// cluster hold identically (the query's position, the cluster-wide sums), so the
// barriers always match.  Heavy ties at the boundary bucket (more than k members)
// send the query through the radix routine of select.cuh, run by CTA 0 over the
// candidates of all CTAs.
#include <cooperative_groups.h>

#include "block_pick.cuh"
#include "prof.cuh"
#include "select.cuh"

namespace cg = cooperative_groups;

namespace hisa {

constexpr int DC_CTAS = 8;
constexpr int DC_THREADS = 256;
constexpr int DC_WARPS = DC_THREADS / 32;
constexpr int DC_MAX_E = 8192;  // eligible blocks of one query (a 1M-token sequence)
constexpr int DC_MAX_M = 128;                            // block budgets this path takes
constexpr int DC_MAX_CAND = DC_MAX_M * BLK / DC_CTAS;    // candidates of one CTA
constexpr int DC_KPT = DC_MAX_CAND / DC_THREADS;
constexpr int DC_BINS = 1024;
constexpr int DC_BIN_WORDS = DC_BINS + DC_BINS / 32;  // bucket b at word b + b / 32
constexpr int DC_MAXK = HISA_MAX_TOPK;
constexpr int DC_LOC_MAX = 1024;  // sequences looked up cooperatively (else by binary search)
constexpr int DC_WARP_TOPM_E = 1024;  // eligible blocks up to which one warp runs the top-m
constexpr size_t LIN_BLK_SCRATCH_MAX = (size_t)LIN_BLK_CAP * 8 + DC_MAX_E;
static_assert(DC_KPT * DC_THREADS == DC_MAX_CAND, "candidates split evenly");

struct DcRed {
  float mx, mn;
  int nv, pad;
};

struct __align__(16) DcSmem {
  union {
    uint32_t allkeys[DC_MAX_E];  // B: every eligible block's key
    SelectShared radix;          // heavy-tie route (CTA 0)
  } u1;
  union {
    struct {
      uint64_t stage[DC_MAXK];  // D: survivors at their bucket offsets
      uint64_t bnd[DC_MAXK];    // D: boundary bucket members
    } s;
    uint32_t radix_work[4 * DC_MAXK];  // heavy-tie route (CTA 0)
  } u2;
  __align__(16) uint32_t keys_local[DC_MAX_E / DC_CTAS];  // A: this CTA's block keys
  float cand[DC_MAX_CAND];                  // C: this CTA's candidate scores
  __align__(16) uint32_t binc[DC_BINS];     // D: this CTA's bucket counts (read remotely)
  uint32_t boff[DC_BIN_WORDS];              // D: global bucket offsets
  uint32_t bcnt[DC_BIN_WORDS];              // D: global bucket counts
  uint32_t curs[DC_BIN_WORDS];              // D: this CTA's scatter cursors
  uint32_t whist[256 + 2 * DC_WARPS];       // B: top-m histogram and warp partials
  int32_t blocks[DC_MAX_M];                 // B: selected blocks, ascending
  int pos_lo[DC_CTAS];                      // D: first output position ranked by each CTA
  int bsc[4 + DC_WARPS];                    // B: top-m scratch
  int32_t cuq[DC_LOC_MAX + 1];              // cu_seqlens_q, for the sequence lookup
  uint4 qrow[D / 8];                        // the query row
  int seqinfo[4];                           // sequence, region start, region end, live keys
  DcRed red;
  int warp_tot[33];
  int wn[DC_WARPS];
  float wmx[DC_WARPS], wmn[DC_WARPS];
  int misc[8];
};

__device__ __forceinline__ int dc_slot(int b) { return b + (b >> 5); }

__device__ __forceinline__ int dc_bucket(float s, float smax, float inv) {
  const int b = __float2int_rz((smax - s) * inv);
  return min(max(b, 0), DC_BINS - 1);
}

struct DcOut {
  int32_t *idx;
  float *scores;
  const int32_t *blocks;
  __device__ void operator()(int r, int c, uint32_t u) const {
    idx[r] = blocks[c >> 7] * BLK + (c & 127);
    if (scores) scores[r] = key_score(u);
  }
};

struct DcPad {
  int32_t *idx;
  float *scores;
  __device__ void operator()(int r) const {
    idx[r] = -1;
    if (scores) scores[r] = 0.f;
  }
};

// The append of a fused decode step (hisa_decode_step); all null otherwise.  The new
// key of sequence s is new_keys[s]; the step appends it at position seqlens[s] and the
// query of row s sits there.
struct DcAppend {
  uint16_t *kc;              // the key cache (written: the new row)
  float *reps;               // the representatives (written: the new key's block)
  int32_t *seqlens;          // live lengths (written: + 1)
  const uint16_t *new_keys;  // [num_seqs, 64]
};

// The append of a fused step for sequence s (k0: its region start, len0: its live
// length before the step), by threads t of nt: the rows of the block that receives
// the new key are staged, the new key row is written, the block is summed again in
// increasing row order exactly like the pooling kernels (bit-identical to a fresh
// pool), and the length grows by one.  sync(): a barrier over the nt threads.
template <class Sync>
__device__ void decode_append_block(uint4 *stage, const DcAppend &ap, int k0, int len0, int s,
                                    int t, int nt, Sync sync) {
  const int b = len0 / BLK, count = len0 - b * BLK + 1;
  const uint4 *src = reinterpret_cast<const uint4 *>(ap.new_keys + (size_t)s * D);
  uint4 *rows = reinterpret_cast<uint4 *>(ap.kc + (size_t)k0 * D);
  for (int i = t; i < count * 8; i += nt) {
    const int r = b * BLK + (i >> 3);
    stage[i] = r < len0 ? rows[(size_t)r * 8 + (i & 7)] : src[i & 7];
  }
  if (t < 8) rows[(size_t)len0 * 8 + t] = src[t];
  sync();
  if (t < 32) {
    const uint32_t *w = reinterpret_cast<const uint32_t *>(stage);
    float a = 0.f, c = 0.f;
    for (int r = 0; r < count; r++) {
      const uint32_t x = w[r * 32 + t];
      a += bf_lo(x);
      c += bf_hi(x);
    }
    const float cnt = (float)count;
    reinterpret_cast<float2 *>(ap.reps + (size_t)(k0 / BLK + b) * D)[t] =
        make_float2(__fdiv_rn(a, cnt), __fdiv_rn(c, cnt));
  }
  if (t == 0) ap.seqlens[s] = len0 + 1;
}

// Rarely taken routes, kept out of line so that the hot path's code stays compact (every
// decode launch starts with a cold instruction cache).
// Heavy ties: CTA 0 runs the radix select over the candidates of every CTA of the
// cluster (read through distributed shared memory).
__device__ __noinline__ void decode_radix_select(DcSmem &sm, int cper, int n, int topk,
                                                 DcOut out, DcPad pad) {
  cg::cluster_group cl = cg::this_cluster();
  const float NEG = -__int_as_float(0x7f800000);
  auto key = [&](int c) -> uint32_t {
    const int owner = c / cper;
    const float *rc = cl.map_shared_rank(sm.cand, owner);
    const float x = rc[c - owner * cper];
    return x != NEG ? score_key(x) : 0u;
  };
  uint32_t *w = sm.u2.radix_work;
  select_topk<DC_THREADS>(key, n, topk, sm.u1.radix, w, reinterpret_cast<int *>(w + topk),
                          w + 2 * topk, reinterpret_cast<int *>(w + 3 * topk), out, pad);
}

// More eligible blocks than one warp selects quickly: the CTA-wide top-m.
__device__ __noinline__ void decode_cta_select_blocks(DcSmem &sm, int E, int own, int m,
                                                      int32_t *ob) {
  if (!cta_select_blocks_lin<DC_THREADS>(sm.u1.allkeys, E, own, m, sm.blocks, ob, sm.whist,
                                         sm.warp_tot, sm.bsc, reinterpret_cast<uint8_t *>(&sm.u2)))
    cta_select_blocks<DC_THREADS>(sm.u1.allkeys, E, own, m, sm.blocks, ob, sm.whist, sm.warp_tot,
                                  sm.bsc);
}

// appended: set when a fused step's append was done here (by warps 1..7 of CTA 0 while
// warp 0 selects the blocks); otherwise the kernel appends after the selection.
__device__ void decode_select_body(DcSmem &sm, const DcAppend &ap, bool &appended,
                                   const uint16_t *__restrict__ q,
                                   const uint16_t *__restrict__ k, const float *__restrict__ reps,
                                   const int32_t *__restrict__ cu_q,
                                   const int32_t *__restrict__ cu_k,
                                   const int32_t *__restrict__ seqlens,
                                   const int32_t *__restrict__ m_seq, int S, int m_max, int topk,
                                   int emax, int32_t *__restrict__ out_idx,
                                   float *__restrict__ out_scores,
                                   int32_t *__restrict__ out_blocks, int *status) {
  cg::cluster_group cl = cg::this_cluster();
  const int me = (int)cl.block_rank();
  const int row = blockIdx.x / DC_CTAS;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const float NEG = -__int_as_float(0x7f800000);
  int32_t *oi = out_idx + (size_t)row * topk;
  float *os = out_scores ? out_scores + (size_t)row * topk : nullptr;
  int32_t *ob = out_blocks ? out_blocks + (size_t)row * m_max : nullptr;
  DcPad pad{oi, os};

  // every CTA of the cluster locates the same query (the sequence lookup and the query
  // row in one memory round trip, the sequence's region in a second); nothing below
  // this early exit has touched another CTA's shared memory
  QueryInfo qi;
  if (ap.new_keys) {
    // fused step: row s is sequence s, whose query sits at the position of its new key
    if (tid < D / 8) sm.qrow[tid] = __ldg(reinterpret_cast<const uint4 *>(q + (size_t)row * D) + tid);
    if (tid == 0) {
      sm.seqinfo[1] = cu_k[row];
      sm.seqinfo[2] = cu_k[row + 1];
      sm.seqinfo[3] = ap.seqlens[row];
    }
    __syncthreads();
    const int k0 = sm.seqinfo[1], k1 = sm.seqinfo[2], len0 = sm.seqinfo[3];
    qi.seq = row;
    qi.kbase = k0;
    qi.len = len0 + 1;
    qi.pos = len0;
    qi.ok = true;
    if (k0 % BLK != 0) {
      if (me == 0 && tid == 0) raise_status(status, HISA_ERR_UNALIGNED);
      qi.ok = false;
    } else if (len0 < 0 || len0 > k1 - k0) {
      if (me == 0 && tid == 0) raise_status(status, HISA_ERR_INVALID_ARG);
      qi.ok = false;
    } else if (len0 + 1 > k1 - k0) {
      if (me == 0 && tid == 0) raise_status(status, HISA_ERR_CAPACITY);
      qi.ok = false;
    }
  } else if (S <= DC_LOC_MAX) {
    for (int i = tid; i <= S; i += DC_THREADS) sm.cuq[i] = __ldg(cu_q + i);
    if (tid < D / 8) sm.qrow[tid] = __ldg(reinterpret_cast<const uint4 *>(q + (size_t)row * D) + tid);
    if (tid == 0) sm.seqinfo[0] = -1;
    __syncthreads();
    for (int i = tid; i < S; i += DC_THREADS)
      if (sm.cuq[i] <= row && row < sm.cuq[i + 1]) sm.seqinfo[0] = i;  // one sequence matches
    __syncthreads();
    if (tid == 0 && sm.seqinfo[0] >= 0) {
      const int sq = sm.seqinfo[0];
      sm.seqinfo[1] = __ldg(cu_k + sq);
      sm.seqinfo[2] = __ldg(cu_k + sq + 1);
      sm.seqinfo[3] = seqlens ? __ldg(seqlens + sq) : sm.seqinfo[2] - sm.seqinfo[1];
    }
    __syncthreads();
    const int sq = sm.seqinfo[0];
    const int k0 = sq >= 0 ? sm.seqinfo[1] : 0, k1 = sq >= 0 ? sm.seqinfo[2] : 0;
    const int q0 = sq >= 0 ? sm.cuq[sq] : 0, q1 = sq >= 0 ? sm.cuq[sq + 1] : 0;
    qi.seq = sq;
    qi.kbase = k0;
    qi.len = sq >= 0 ? sm.seqinfo[3] : 0;
    qi.pos = qi.len - (q1 - q0) + (row - q0);
    qi.ok = true;
    if (sq < 0) {  // cu_seqlens_q does not cover this row
      if (me == 0 && tid == 0) raise_status(status, HISA_ERR_INVALID_ARG);
      qi.ok = false;
    } else if (k0 % BLK != 0) {
      if (me == 0 && tid == 0) raise_status(status, HISA_ERR_UNALIGNED);
      qi.ok = false;
    } else if (qi.len < 0 || qi.len > k1 - k0 || qi.pos < 0 || qi.pos >= qi.len) {
      if (me == 0 && tid == 0) raise_status(status, HISA_ERR_INVALID_ARG);
      qi.ok = false;
    }
  } else {
    qi = locate(cu_q, cu_k, seqlens, S, row, (me == 0 && tid == 0) ? status : nullptr);
    if (tid < D / 8) sm.qrow[tid] = __ldg(reinterpret_cast<const uint4 *>(q + (size_t)row * D) + tid);
    __syncthreads();
  }
  const int own = qi.ok ? qi.pos / BLK : 0, E = own + 1;
  if (!qi.ok || E > emax) {
    if (qi.ok && me == 0 && tid == 0) raise_status(status, HISA_ERR_INVALID_ARG);
    for (int r = me * DC_THREADS + tid; r < topk; r += DC_CTAS * DC_THREADS) pad(r);
    if (ob && me == 0)
      for (int i = tid; i < m_max; i += DC_THREADS) ob[i] = -1;
    return;
  }
  // this row's block budget; out_blocks entries past it are -1
  const int m = seq_budget(m_seq, qi.seq, m_max, (me == 0 && tid == 0) ? status : nullptr);
  if (ob && me == 0)
    for (int i = m + tid; i < m_max; i += DC_THREADS) ob[i] = -1;

  // ---------------- stage 1: blocks ----------------
  if (E > m) {
    // A. this CTA's share of the block scores: eight lanes per representative row
    //    (lane holds 8 of its dims), every row of a pass loaded before any is reduced
    const int per = ((E + DC_CTAS - 1) / DC_CTAS + 3) & ~3;  // whole 16-byte groups
    const int b0 = me * per, b1 = min(E, b0 + per);
    const int nf = min(m, 3);
    const int part = lane & 7;
    for (int i = max(b1 - b0, 0) + tid; i < per; i += DC_THREADS) sm.keys_local[i] = 0u;
    float qf[8];
    {
      const uint4 w = sm.qrow[part];
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int u = 0; u < 4; u++) {
        qf[2 * u] = bf_lo(ws[u]);
        qf[2 * u + 1] = bf_hi(ws[u]);
      }
    }
    const float4 *rbase = reinterpret_cast<const float4 *>(reps + (size_t)(qi.kbase / BLK) * D);
    constexpr int ROWS_PER_PASS = DC_WARPS * 4;  // four rows per warp
    constexpr int PASSES = 4;                    // rows in flight per lane
    for (int bb = b0; bb < b1; bb += ROWS_PER_PASS * PASSES) {
      float4 x[PASSES][2];
      int bl[PASSES];
#pragma unroll
      for (int p = 0; p < PASSES; p++) {
        bl[p] = bb + p * ROWS_PER_PASS + warp * 4 + (lane >> 3);
        const bool forced =
            bl[p] == own || (nf >= 2 && bl[p] == own - 1) || (nf >= 3 && bl[p] == 0);
        x[p][0] = x[p][1] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (bl[p] < b1 && !forced) {
          x[p][0] = __ldg(rbase + (size_t)bl[p] * (D / 4) + part * 2);
          x[p][1] = __ldg(rbase + (size_t)bl[p] * (D / 4) + part * 2 + 1);
        }
      }
#pragma unroll
      for (int p = 0; p < PASSES; p++) {
        float sc = qf[0] * x[p][0].x;
        sc = fmaf(qf[1], x[p][0].y, sc);
        sc = fmaf(qf[2], x[p][0].z, sc);
        sc = fmaf(qf[3], x[p][0].w, sc);
        sc = fmaf(qf[4], x[p][1].x, sc);
        sc = fmaf(qf[5], x[p][1].y, sc);
        sc = fmaf(qf[6], x[p][1].z, sc);
        sc = fmaf(qf[7], x[p][1].w, sc);
        sc += __shfl_xor_sync(0xffffffffu, sc, 1);
        sc += __shfl_xor_sync(0xffffffffu, sc, 2);
        sc += __shfl_xor_sync(0xffffffffu, sc, 4);
        const int b = bl[p];
        const bool forced = b == own || (nf >= 2 && b == own - 1) || (nf >= 3 && b == 0);
        if (part == 0 && b < b1) sm.keys_local[b - b0] = forced ? 0u : score_key(sc);
      }
    }
    cl.sync();
    // B. all keys of the cluster (16-byte remote loads), then the same top-m in
    //    every CTA
    for (int g = tid; g * 4 < DC_CTAS * per && g * 4 < E + 3; g += DC_THREADS) {
      const int b = g * 4, owner = b / per;
      const uint4 *rk = reinterpret_cast<const uint4 *>(cl.map_shared_rank(sm.keys_local, owner));
      *reinterpret_cast<uint4 *>(&sm.u1.allkeys[b]) = rk[(b - owner * per) >> 2];
    }
    __syncthreads();
    static_assert(sizeof(sm.u2) >= LIN_BLK_SCRATCH_MAX, "top-m scratch fits the staging area");
    if (E <= DC_WARP_TOPM_E) {
      // few blocks: one warp selects (radix digits over a per-warp histogram, no CTA
      // barrier between the rounds) while the others wait once
      const bool append_here = ap.new_keys && me == 0;
      if (warp == 0) {
        warp_select_blocks(sm.u1.allkeys, E, own, m, sm.blocks, me == 0 ? ob : nullptr, sm.whist,
                           false);
      } else if (append_here) {
        // meanwhile the fused step's append (every CTA of the cluster read the old length
        // before the cluster barrier above; the selection reads neither the new key's
        // cache row nor its block's representative, the block being forced)
        decode_append_block(reinterpret_cast<uint4 *>(&sm.u2), ap, qi.kbase, qi.pos, row,
                            tid - 32, DC_THREADS - 32,
                            [] { asm volatile("bar.sync 1, %0;" ::"n"(DC_THREADS - 32) : "memory"); });
      }
      appended = append_here;  // every thread of the CTA, warp 0 included
      __syncthreads();
    } else {
      decode_cta_select_blocks(sm, E, own, m, me == 0 ? ob : nullptr);
    }
  } else {
    for (int i = tid; i < m; i += DC_THREADS) {
      const int v = i < E ? i : -1;
      sm.blocks[i] = v;
      if (ob && me == 0) ob[i] = v;
    }
    __syncthreads();
  }
  const int nsel = min(m, E);
  DcOut out{oi, os, sm.blocks};

  // ---------------- stage 2: gather-score ----------------
  // CTA me owns selected slots [me * bp, me * bp + its count); local candidate lc is
  // global candidate me * bp * 128 + lc, i.e. token blocks[c >> 7] * 128 + (c & 127)
  const int bp = (nsel + DC_CTAS - 1) / DC_CTAS;
  const int my_slots = max(0, min(nsel - me * bp, bp));
  const int nloc = my_slots * BLK;
  const int cbase = me * bp * BLK;
  {
    const int quarter = lane & 3, sub = lane >> 2;  // four lanes per key row
    float qf[16];
    {
      const uint4 a = sm.qrow[quarter * 2], b = sm.qrow[quarter * 2 + 1];
      const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
      for (int u = 0; u < 8; u++) {
        qf[2 * u] = bf_lo(w[u]);
        qf[2 * u + 1] = bf_hi(w[u]);
      }
    }
    const uint16_t *kseq = k + (size_t)qi.kbase * D;
    constexpr int KEYS_PER_PASS = DC_WARPS * 8;
    constexpr int BATCH = 8;  // passes whose key loads are in flight together
    for (int lk0 = 0; lk0 < nloc; lk0 += KEYS_PER_PASS * BATCH) {
      uint4 a[BATCH], b[BATCH];
      bool live[BATCH];
#pragma unroll
      for (int p = 0; p < BATCH; p++) {
        const int lk = lk0 + p * KEYS_PER_PASS + warp * 8 + sub;
        live[p] = false;
        a[p] = b[p] = make_uint4(0u, 0u, 0u, 0u);
        if (lk < nloc) {
          const int j = sm.blocks[me * bp + (lk >> 7)] * BLK + (lk & 127);
          live[p] = j <= qi.pos;
          if (live[p]) {
            // a fused step's new key is read from the step's input (the cache row is
            // written at the end of the step)
            const uint16_t *krow = (ap.new_keys && j == qi.pos) ? ap.new_keys + (size_t)row * D
                                                                : kseq + (size_t)j * D;
            const uint4 *kr = reinterpret_cast<const uint4 *>(krow) + quarter * 2;
            a[p] = __ldg(kr);
            b[p] = __ldg(kr + 1);
          }
        }
      }
#pragma unroll
      for (int p = 0; p < BATCH; p++) {
        const uint32_t w[8] = {a[p].x, a[p].y, a[p].z, a[p].w, b[p].x, b[p].y, b[p].z, b[p].w};
        float acc = 0.f;
#pragma unroll
        for (int u = 0; u < 8; u++) {
          acc = fmaf(qf[2 * u], bf_lo(w[u]), acc);
          acc = fmaf(qf[2 * u + 1], bf_hi(w[u]), acc);
        }
        acc += __shfl_xor_sync(0xffffffffu, acc, 1);
        acc += __shfl_xor_sync(0xffffffffu, acc, 2);
        const int lk = lk0 + p * KEYS_PER_PASS + warp * 8 + sub;
        if (quarter == 0 && lk < nloc) sm.cand[lk] = live[p] ? acc : NEG;
      }
    }
  }
  __syncthreads();

  // ---------------- stage 2: exact top-k across the cluster ----------------
  float f[DC_KPT];
  float mx = NEG, mn = -NEG;
  int nv = 0;
#pragma unroll
  for (int i = 0; i < DC_KPT; i++) {
    const int lc = i * DC_THREADS + tid;
    f[i] = lc < nloc ? sm.cand[lc] : NEG;
    if (f[i] != NEG) {
      mx = fmaxf(mx, f[i]);
      mn = fminf(mn, f[i]);
      nv++;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    nv += __shfl_xor_sync(0xffffffffu, nv, o);
  }
  if (lane == 0) {
    sm.wmx[warp] = mx;
    sm.wmn[warp] = mn;
    sm.wn[warp] = nv;
  }
  for (int i = tid; i < DC_BINS; i += DC_THREADS) sm.binc[i] = 0u;
  if (tid < DC_CTAS) sm.pos_lo[tid] = 0x7fffffff;
  __syncthreads();
  if (tid == 0) {
    float a = NEG, b = -NEG;
    int c = 0;
    for (int w = 0; w < DC_WARPS; w++) {
      a = fmaxf(a, sm.wmx[w]);
      b = fminf(b, sm.wmn[w]);
      c += sm.wn[w];
    }
    sm.red.mx = a;
    sm.red.mn = b;
    sm.red.nv = c;
    sm.misc[5] = 0;  // boundary fill counter
  }
  cl.sync();
  // cluster-wide max / min / count, summed in rank order (identical in every CTA)
  float smax = NEG, smin = -NEG;
  int nvalid = 0;
  if (lane < DC_CTAS) {  // lane c reads CTA c; the warp reduction order is fixed
    const DcRed *r = cl.map_shared_rank(&sm.red, lane);
    smax = r->mx;
    smin = r->mn;
    nvalid = r->nv;
  }
#pragma unroll
  for (int o = 4; o > 0; o >>= 1) {
    smax = fmaxf(smax, __shfl_xor_sync(0xffffffffu, smax, o));
    smin = fminf(smin, __shfl_xor_sync(0xffffffffu, smin, o));
    nvalid += __shfl_xor_sync(0xffffffffu, nvalid, o);
  }
  smax = __shfl_sync(0xffffffffu, smax, 0);
  smin = __shfl_sync(0xffffffffu, smin, 0);
  nvalid = __shfl_sync(0xffffffffu, nvalid, 0);
  const int kp = min(topk, nvalid);
  const float range = smax - smin;
  const float inv = range > 0.f ? (float)DC_BINS / range : 0.f;

  // the radix route over all candidates of the cluster (run by CTA 0)
  auto radix_route = [&]() {
    cl.sync();  // every CTA is done with the exchanged counts
    if (me == 0) decode_radix_select(sm, bp * BLK, nsel * BLK, topk, out, pad);
    cl.sync();  // the other CTAs' candidates stay readable until CTA 0 is done
  };
  if (nvalid == 0) {
    for (int r = me * DC_THREADS + tid; r < topk; r += DC_CTAS * DC_THREADS) pad(r);
    cl.sync();
    return;
  }
  if (!(range > 0.f) || !isfinite(inv)) {
    radix_route();
    return;
  }
#pragma unroll
  for (int i = 0; i < DC_KPT; i++)
    if (f[i] != NEG) atomicAdd(&sm.binc[dc_bucket(f[i], smax, inv)], 1u);
  cl.sync();
  {
    // global counts, and the counts of the lower-ranked CTAs, of four buckets per
    // thread (one 16-byte remote load per CTA)
    constexpr int per = DC_BINS / DC_THREADS;
    static_assert(per == 4, "four buckets per thread");
    int g[per], before[per];
#pragma unroll
    for (int i = 0; i < per; i++) {
      g[i] = 0;
      before[i] = 0;
    }
#pragma unroll
    for (int c = 0; c < DC_CTAS; c++) {
      const uint4 v = reinterpret_cast<const uint4 *>(cl.map_shared_rank(sm.binc, c))[tid];
      const int vv[4] = {(int)v.x, (int)v.y, (int)v.z, (int)v.w};
#pragma unroll
      for (int i = 0; i < per; i++) {
        g[i] += vv[i];
        if (c < me) before[i] += vv[i];
      }
    }
    int local = 0;
#pragma unroll
    for (int i = 0; i < per; i++) local += g[i];
    int total;
    int run = block_exclusive_scan<DC_THREADS>(local, sm.warp_tot, &total);
    if (tid == 0) {
      sm.misc[0] = DC_BINS;  // boundary bucket (none when every candidate survives)
      sm.misc[1] = kp;       // survivors before it
      sm.misc[2] = 0;        // its members in lower-ranked CTAs
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < per; i++) {
      const int b = tid * per + i;
      if (nvalid > topk && run < topk && run + g[i] >= topk) {
        sm.misc[0] = b;
        sm.misc[1] = run;
        sm.misc[2] = before[i];
      }
      sm.boff[dc_slot(b)] = (uint32_t)run;
      sm.bcnt[dc_slot(b)] = (uint32_t)g[i];
      sm.curs[dc_slot(b)] = (uint32_t)(run + before[i]);
      run += g[i];
    }
  }
  __syncthreads();
  const int bstar = sm.misc[0], above = sm.misc[1], bnd_before = sm.misc[2];
  const int need = kp - above;
  const int nbnd = bstar < DC_BINS ? (int)sm.bcnt[dc_slot(bstar)] : 0;
  if (nbnd > DC_MAXK) {  // heavy ties at the boundary
    radix_route();
    return;
  }
  // Every survivor bucket is ranked by one CTA, its owner: the CTA whose share of the
  // output positions [c * ppo, (c + 1) * ppo) holds the bucket's first position.  A
  // CTA ranks the positions from its first bucket's start to the next owner's.
  const int ppo = (above + DC_CTAS - 1) / DC_CTAS;
  auto owner = [&](int b) { return min(DC_CTAS - 1, (int)sm.boff[dc_slot(b)] / max(ppo, 1)); };
  for (int b = tid; b < bstar; b += DC_THREADS)
    if (sm.bcnt[dc_slot(b)] > 0u) atomicMin(&sm.pos_lo[owner(b)], (int)sm.boff[dc_slot(b)]);
  // scatter: each survivor to its bucket owner's staging array, each boundary member
  // to CTA 0's list (one remote store each)
#pragma unroll
  for (int i = 0; i < DC_KPT; i++) {
    if (f[i] != NEG) {
      const int b = dc_bucket(f[i], smax, inv);
      if (b <= bstar) {
        const uint64_t key = rank_key(f[i], cbase + i * DC_THREADS + tid);
        if (b < bstar) {
          const int p = (int)atomicAdd(&sm.curs[dc_slot(b)], 1u);
          cl.map_shared_rank(sm.u2.s.stage, owner(b))[p] = key;
        } else {
          const int p = bnd_before + atomicAdd(&sm.misc[5], 1);
          cl.map_shared_rank(sm.u2.s.bnd, 0)[p] = key;
        }
      }
    }
  }
  cl.sync();  // no access to another CTA's shared memory follows

  // rank the survivors of the buckets this CTA owns
  int p_lo = sm.pos_lo[me], p_hi = above;
#pragma unroll
  for (int c = 0; c < DC_CTAS; c++)
    if (c > me) p_hi = min(p_hi, sm.pos_lo[c]);
  const uint64_t *stage = sm.u2.s.stage;
  for (int p = p_lo + tid; p < p_hi; p += DC_THREADS) {
    const uint64_t mk = stage[p];
    const int b = dc_bucket(key_score((uint32_t)(mk >> 32)), smax, inv);
    const int st = (int)sm.boff[dc_slot(b)], en = st + (int)sm.bcnt[dc_slot(b)];
    int rank = 0;
    for (int t = st; t < en; t++) rank += stage[t] > mk;
    out(st + rank, (int)~(uint32_t)mk, (uint32_t)(mk >> 32));
  }
  if (need > 0 && me == 0) {
    const uint64_t *bnd = sm.u2.s.bnd;
    for (int e = tid; e < nbnd; e += DC_THREADS) {
      const uint64_t mk = bnd[e];
      int rank = 0;
      for (int t = 0; t < nbnd; t++) rank += bnd[t] > mk;
      if (rank < need) out(above + rank, (int)~(uint32_t)mk, (uint32_t)(mk >> 32));
    }
  }
  for (int r = kp + me * DC_THREADS + tid; r < topk; r += DC_CTAS * DC_THREADS) pad(r);
}

// The append of a fused step, by CTA 0 of the row's cluster once its selection is done
// (every CTA of the cluster read the old length long before), when the selection did
// not already do it beside its block top-m.
__device__ __noinline__ void decode_append_tail(DcSmem &sm, const DcAppend &ap,
                                               const int32_t *cu_k, int s) {
  __syncthreads();
  const int k0 = cu_k[s], k1 = cu_k[s + 1];
  const int len0 = ap.seqlens[s];
  if (k0 % BLK != 0 || len0 < 0 || len0 + 1 > k1 - k0) return;  // reported by the body
  decode_append_block(reinterpret_cast<uint4 *>(&sm.u2), ap, k0, len0, s, threadIdx.x, DC_THREADS,
                      [] { __syncthreads(); });
}

__global__ void __cluster_dims__(DC_CTAS, 1, 1) __launch_bounds__(DC_THREADS, 1)
decode_select_kernel(const uint16_t *__restrict__ q, const uint16_t *__restrict__ k,
                     const float *__restrict__ reps, const int32_t *__restrict__ cu_q,
                     const int32_t *__restrict__ cu_k, const int32_t *__restrict__ seqlens,
                     const int32_t *__restrict__ m_seq, int S, int m_max, int topk, int emax,
                     int32_t *__restrict__ out_idx, float *__restrict__ out_scores,
                     int32_t *__restrict__ out_blocks, DcAppend ap, int *status) {
  extern __shared__ __align__(16) uint8_t dc_raw[];
  DcSmem &sm = *reinterpret_cast<DcSmem *>(dc_raw);
  // Launched as a programmatic dependent of the previous kernel on the stream (when
  // the stream allows it): nothing is read before that kernel has completed, and the
  // next kernel may begin launching at once (it waits the same way).
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  bool appended = false;
  decode_select_body(sm, ap, appended, q, k, reps, cu_q, cu_k, seqlens, m_seq, S, m_max, topk,
                     emax, out_idx, out_scores, out_blocks, status);
  if (ap.new_keys && !appended && cg::this_cluster().block_rank() == 0)
    decode_append_tail(sm, ap, cu_k, blockIdx.x / DC_CTAS);
}

// The cluster path covers every query whose eligible blocks fit DC_MAX_E and whose
// block budget fits DC_MAX_M.
bool decode_path_fits(int max_seqlen_k, int m) {
  return (max_seqlen_k + BLK - 1) / BLK <= DC_MAX_E && m <= DC_MAX_M;
}

cudaError_t launch_decode_select(const uint16_t *q, const uint16_t *k, const float *reps,
                                 const int32_t *cu_q, const int32_t *cu_k,
                                 const int32_t *seqlens, const int32_t *m_seq, int S,
                                 int total_q, int max_seqlen_k, int m, int topk,
                                 int32_t *out_idx, float *out_scores, int32_t *out_blocks,
                                 int *status, cudaStream_t st, uint16_t *append_kc,
                                 float *append_reps, int32_t *append_seqlens,
                                 const uint16_t *new_keys) {
  if (total_q == 0) return cudaSuccess;
  static std::atomic<int> attr[64];
  cudaError_t e = set_smem_once((const void *)decode_select_kernel, sizeof(DcSmem), attr);
  if (e != cudaSuccess) return e;
  const int emax = (max_seqlen_k + BLK - 1) / BLK;
  const DcAppend ap{append_kc, append_reps, append_seqlens, new_keys};
  {
    ProfScope ps(K_DECODE_SELECT, st);
    e = launch_pdl((const void *)decode_select_kernel, dim3(total_q * DC_CTAS), dim3(DC_THREADS),
                   sizeof(DcSmem), st, q, k, reps, cu_q, cu_k, seqlens, m_seq, S, m, topk,
                   emax > 0 ? emax : 1, out_idx, out_scores, out_blocks, ap, status);
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace hisa
