// CTA-cooperative exact top-k over order-preserving uint32 score keys.
//
// Given n candidate keys (0 = not a candidate) listed in increasing token order,
// select_topk emits the k best by (score descending, token ascending) and pads
// the tail.  Three phases:
//   1. radix select: 3 MSD rounds (11, 11 and 10 bits) of a shared-memory
//      histogram find the k-th largest key T and how many keys equal to T are
//      still needed (the lowest-index ones win, as the tie rule demands);
//   2. stable compaction: every warp walks a contiguous slice of the candidates
//      in rounds of 32; ballots give each survivor its slot, so survivors keep
//      token order;
//   3. bucketed sort: survivors are binned by (max - key) >> shift into 2048
//      buckets (higher score -> lower bucket), scattered, and each one counts the
//      members of its own bucket that beat it to find its final rank.  Buckets
//      are tiny for continuous scores; equal scores cost O(bucket^2) but stay exact.
#pragma once

#include "common.cuh"

namespace hisa {

constexpr int SEL_BINS = 2048;

struct SelectShared {
  uint32_t hist[SEL_BINS];
  uint32_t cursor[SEL_BINS];
  int warp_tot[33];
  int wgt[32], weq[32], web[32], wsb[32];
  uint32_t misc[8];
};

// Max and min over one value per thread (NT threads).
template <int NT>
__device__ __forceinline__ void block_minmax(uint32_t &mx, uint32_t &mn, SelectShared &sh) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    mn = min(mn, __shfl_xor_sync(0xffffffffu, mn, o));
  }
  if (lane == 0) {
    sh.wgt[warp] = (int)mx;
    sh.weq[warp] = (int)mn;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t a = 0, b = 0xffffffffu;
    for (int w = 0; w < NT / 32; w++) {
      a = max(a, (uint32_t)sh.wgt[w]);
      b = min(b, (uint32_t)sh.weq[w]);
    }
    sh.misc[6] = a;
    sh.misc[7] = b;
  }
  __syncthreads();
  mx = sh.misc[6];
  mn = sh.misc[7];
  __syncthreads();
}

// key(c): the order-preserving key of candidate c (0 = not a candidate), token order.
// sel_key/sel_c/tmp_key/tmp_c: shared arrays of at least k entries.
// out(rank, c, key) writes one output slot; pad(rank) fills a slot past the survivors.
template <int NT, class Key, class Out, class Pad>
__device__ void select_topk(Key key, int n, int k, SelectShared &sh, uint32_t *sel_key,
                            int *sel_c, uint32_t *tmp_key, int *tmp_c, Out out, Pad pad) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int NW = NT / 32;

  // ---- phase 1: radix select -------------------------------------------------
  uint32_t prefix = 0, pmask = 0, T = 0;
  int remaining = k, need_eq = 0;
  bool take_all = false, done = false;
#pragma unroll 1
  for (int r = 0; r < 3; r++) {
    const int shift = r == 0 ? 21 : (r == 1 ? 10 : 0);
    const int nb = r == 2 ? 1024 : 2048;
    for (int i = tid; i < nb; i += NT) sh.hist[i] = 0;
    __syncthreads();
    for (int c = tid; c < n; c += NT) {
      uint32_t u = key(c);
      if (u != 0u && (u & pmask) == prefix) atomicAdd(&sh.hist[(u >> shift) & (nb - 1)], 1u);
    }
    __syncthreads();
    const int per = nb / NT;  // bins per thread, walked from the top bin down
    int local = 0;
    for (int i = 0; i < per; i++) local += (int)sh.hist[nb - 1 - (tid * per + i)];
    int total;
    int run = block_exclusive_scan<NT>(local, sh.warp_tot, &total);
    if (r == 0 && total <= k) {
      take_all = true;
      break;
    }
    for (int i = 0; i < per; i++) {
      int d = nb - 1 - (tid * per + i);
      int h = (int)sh.hist[d];
      if (run < remaining && run + h >= remaining) {
        sh.misc[0] = (uint32_t)d;
        sh.misc[1] = (uint32_t)run;
        sh.misc[2] = (uint32_t)h;
      }
      run += h;
    }
    __syncthreads();
    const uint32_t dig = sh.misc[0];
    const int above = (int)sh.misc[1], in_bin = (int)sh.misc[2];
    __syncthreads();
    remaining -= above;
    prefix |= dig << shift;
    pmask |= (uint32_t)(nb - 1) << shift;
    if (in_bin == remaining) {  // the whole bin survives
      T = prefix ? prefix - 1u : 0u;
      need_eq = 0;
      done = true;
      break;
    }
  }
  if (take_all) {
    T = 0u;
    need_eq = 0;
  } else if (!done) {
    T = prefix;
    need_eq = remaining;
  }
  const bool eq_live = (T != 0u) && (need_eq > 0);

  // ---- phase 2: stable compaction ---------------------------------------------
  const int seg = ((n + NW - 1) / NW + 31) & ~31;
  const int c0 = warp * seg, c1 = min(n, c0 + seg);
  int ngt = 0, neq = 0;
  for (int base = c0; base < c1; base += 32) {
    int c = base + lane;
    uint32_t u = c < c1 ? key(c) : 0u;
    ngt += __popc(__ballot_sync(0xffffffffu, u > T));
    neq += __popc(__ballot_sync(0xffffffffu, eq_live && u == T));
  }
  if (lane == 0) {
    sh.wgt[warp] = ngt;
    sh.weq[warp] = neq;
  }
  __syncthreads();
  if (tid == 0) {
    int eb = 0, sb = 0;
    for (int w = 0; w < NW; w++) {
      sh.web[w] = eb;
      sh.wsb[w] = sb;
      int take = min(max(need_eq - eb, 0), sh.weq[w]);
      sb += sh.wgt[w] + (eq_live ? take : 0);
      eb += sh.weq[w];
    }
    sh.misc[3] = (uint32_t)sb;
  }
  __syncthreads();
  const int kp = (int)sh.misc[3];
  {
    int eqr = sh.web[warp], selr = sh.wsb[warp];
    const unsigned lt = (1u << lane) - 1u;
    for (int base = c0; base < c1; base += 32) {
      int c = base + lane;
      uint32_t u = c < c1 ? key(c) : 0u;
      bool is_eq = eq_live && u == T;
      unsigned beq = __ballot_sync(0xffffffffu, is_eq);
      bool sel = (u > T) || (is_eq && eqr + __popc(beq & lt) < need_eq);
      unsigned bsel = __ballot_sync(0xffffffffu, sel);
      if (sel) {
        int p = selr + __popc(bsel & lt);
        sel_key[p] = u;
        sel_c[p] = c;
      }
      eqr += __popc(beq);
      selr += __popc(bsel);
    }
  }
  __syncthreads();

  // ---- phase 3: bucketed sort -----------------------------------------------------
  uint32_t mx = 0u, mn = 0xffffffffu;
  for (int i = tid; i < kp; i += NT) {
    mx = max(mx, sel_key[i]);
    mn = min(mn, sel_key[i]);
  }
  block_minmax<NT>(mx, mn, sh);
  const uint32_t range = kp > 0 ? mx - mn : 0u;
  const int shift = range < (uint32_t)SEL_BINS ? 0 : (32 - __clz((int)range)) - 11;
  for (int i = tid; i < SEL_BINS; i += NT) sh.hist[i] = 0;
  __syncthreads();
  for (int i = tid; i < kp; i += NT) atomicAdd(&sh.hist[(mx - sel_key[i]) >> shift], 1u);
  __syncthreads();
  {
    constexpr int per = SEL_BINS / NT;
    int local = 0;
    for (int i = 0; i < per; i++) local += (int)sh.hist[tid * per + i];
    int total;
    int run = block_exclusive_scan<NT>(local, sh.warp_tot, &total);
    for (int i = 0; i < per; i++) {
      int b = tid * per + i;
      int h = (int)sh.hist[b];
      sh.hist[b] = (uint32_t)run;
      sh.cursor[b] = (uint32_t)run;
      run += h;
    }
  }
  __syncthreads();
  for (int i = tid; i < kp; i += NT) {
    uint32_t u = sel_key[i];
    uint32_t slot = atomicAdd(&sh.cursor[(mx - u) >> shift], 1u);
    tmp_key[slot] = u;
    tmp_c[slot] = sel_c[i];
  }
  __syncthreads();
  for (int s = tid; s < kp; s += NT) {
    uint32_t u = tmp_key[s];
    int c = tmp_c[s];
    uint32_t b = (mx - u) >> shift;
    int st = (int)sh.hist[b], en = (int)sh.cursor[b];
    int rank = 0;
    for (int t = st; t < en; t++) {
      uint32_t u2 = tmp_key[t];
      rank += (u2 > u) || (u2 == u && tmp_c[t] < c);
    }
    out(st + rank, c, u);
  }
  for (int r = kp + tid; r < k; r += NT) pad(r);
  __syncthreads();
}

}  // namespace hisa
namespace hisa {

// ---------------------------------------------------------------------------
// Exact top-k through 4096 linear score buckets.
//
// Input: n raw fp32 scores in candidate order, -inf marking a position that is not
// a candidate (finite scores are the contract).  The candidates are visited through
// a "cands" object: RegCands loads them into registers once (thread t keeps
// candidates ((i / 4) * NT + t) * 4 + i % 4, read with 16-byte loads); MemCands
// reads the row again from memory on every pass (rows longer than the registers
// hold).  Then:
//  1. max and min of the candidate scores (fused with the load);
//  2. a shared-memory histogram over SL_BINS buckets linear in the score, bucket 0
//     at the maximum; the bucket map is monotone, so bucket order is score order;
//  3. one scan gives every bucket its first output slot and finds b*, the bucket of
//     the kp-th best score (kp = min(k, number of candidates));
//  4. the candidates of buckets 0..b* are scattered, (score, candidate number), to
//     their bucket's slots; each bucket's cursor then marks its end, which is the
//     next bucket's start;
//  5. every survivor counts the members of its own bucket that beat it (score desc,
//     candidate asc); its bucket start plus that count is its output slot, and the
//     slots below kp are kept (b* keeps its best kp - start(b*));
//  6. the staged row (token index, score) is written with coalesced stores.
// Every step is predicated rather than branched, so that a warp's candidates share
// one instruction stream.  A b* with more members than fit past the k-th slot
// (heavy ties) sends the row through the radix routine above instead.

constexpr int SL_BINS = 4096;
// Bucket b lives at word b + b / 32: a thread scanning its run of consecutive buckets
// touches a different bank from every other thread of its warp.
constexpr int SL_WORDS = SL_BINS + SL_BINS / 32;
constexpr int SL_SLACK = 512;  // members of b* that may lie past the k-th slot
__device__ __forceinline__ int sl_slot(int b) { return b + (b >> 5); }

// Survivor capacity of the staging area for k outputs.
__host__ __device__ inline int sl_cap(int k) { return (k + SL_SLACK + 7) & ~7; }

// Bytes of shared working memory select_topk_lin needs for k outputs (16-byte
// multiple).  Layout: staged token indices int32[k] | staged scores f32[k] |
// survivor scores f32[cap] | survivor candidates u16[cap]; the radix route reuses the
// same bytes as its four k-entry lists (the staged rows over its first two).
__host__ __device__ inline size_t sl_work_bytes(int k) {
  const size_t a = (size_t)8 * k + (size_t)6 * sl_cap(k);
  const size_t b = (size_t)16 * k;
  return ((a > b ? a : b) + 15) & ~(size_t)15;
}

struct SlShared {
  union {
    SelectShared radix;
    struct {
      uint32_t off[SL_WORDS];  // counts, then first slots, then (after the scatter) ends
      int warp_tot[33];
      float wmx[32], wmn[32];
      int misc[4];
    } lin;
  };
};

// bucket(x) = min(round((smax - x) * inv), SL_BINS - 1).  The fused multiply-add adds
// 2^23, so its result lies where consecutive floats are 1 apart and the low bits of
// the sum are the rounded product; both roundings are monotone, and so is the map.
// -inf maps to the last bucket (the sum is +inf).
struct LinMap {
  float smax, inv;
  __device__ __forceinline__ int operator()(float x) const {
    const float t = fmaf(smax - x, inv, 8388608.0f);
    return min(__float_as_int(t) - 0x4B000000, SL_BINS - 1);
  }
};

// Sources of a row of raw scores in candidate order.
// A contiguous row (global or shared memory, 16-byte aligned):
struct RowScores {
  const float *p;
  __device__ float4 ld4(int c) const { return *reinterpret_cast<const float4 *>(p + c); }
  __device__ float ld1(int c) const { return p[c]; }
};
// A row assembled from segments of 128 scores: candidate c is score c % 128 of
// segment seg[c / 128], which starts at base + seg[c / 128] * 128.
struct SegScores {
  const float *base;
  const int32_t *seg;
  __device__ const float *at(int c) const { return base + (size_t)seg[c >> 7] * 128 + (c & 127); }
  __device__ float4 ld4(int c) const { return *reinterpret_cast<const float4 *>(at(c)); }
  __device__ float ld1(int c) const { return *at(c); }
};

__device__ __forceinline__ float neg_inf() { return -__int_as_float(0x7f800000); }

// 64-bit (score, candidate) composite whose unsigned order is the output order:
// score descending, then candidate ascending.
__device__ __forceinline__ uint64_t rank_key(float s, int c) {
  return ((uint64_t)score_key(s) << 32) | (uint32_t)(~(uint32_t)c);
}

// One 16-byte group of candidates c0..c0+3 (c0 % 4 == 0), -inf past n.
template <class Src>
__device__ __forceinline__ float4 load_group(const Src &sc, int c0, int n) {
  const float NEG = neg_inf();
  float4 v = make_float4(NEG, NEG, NEG, NEG);
  if (c0 + 3 < n) {
    v = sc.ld4(c0);
  } else if (c0 < n) {
    v.x = sc.ld1(c0);
    if (c0 + 1 < n) v.y = sc.ld1(c0 + 1);
    if (c0 + 2 < n) v.z = sc.ld1(c0 + 2);
  }
  return v;
}

// Candidates held in registers (n <= NT * KPT).
template <int NT, int KPT>
struct RegCands {
  static_assert(KPT % 4 == 0, "scores are loaded four at a time");
  float f[KPT];
  template <class Src>
  __device__ __forceinline__ void load(const Src &sc, int n, float &mx, float &mn) {
    const float NEG = neg_inf();
#pragma unroll
    for (int j = 0; j < KPT / 4; j++) {
      const float4 v = load_group(sc, (j * NT + (int)threadIdx.x) * 4, n);
      f[4 * j] = v.x;
      f[4 * j + 1] = v.y;
      f[4 * j + 2] = v.z;
      f[4 * j + 3] = v.w;
    }
    mx = NEG;
    mn = -NEG;
#pragma unroll
    for (int i = 0; i < KPT; i++) {
      mx = fmaxf(mx, f[i]);
      if (f[i] != NEG) mn = fminf(mn, f[i]);
    }
  }
  template <class F>
  __device__ __forceinline__ void each(F fn) const {
#pragma unroll
    for (int i = 0; i < KPT; i++) fn(f[i], ((i >> 2) * NT + (int)threadIdx.x) * 4 + (i & 3));
  }
};

// Candidates read from memory on every pass (any n <= 65536).
template <int NT, class Src>
struct MemCands {
  Src sc;
  int n;
  __device__ __forceinline__ void load(float &mx, float &mn) const {
    const float NEG = neg_inf();
    mx = NEG;
    mn = -NEG;
    each([&](float x, int) {
      mx = fmaxf(mx, x);
      if (x != NEG) mn = fminf(mn, x);
    });
  }
  template <class F>
  __device__ __forceinline__ void each(F fn) const {
    for (int c0 = (int)threadIdx.x * 4; c0 < n; c0 += NT * 4) {
      const float4 v = load_group(sc, c0, n);
      fn(v.x, c0);
      fn(v.y, c0 + 1);
      fn(v.z, c0 + 2);
      fn(v.w, c0 + 3);
    }
  }
};

// Output slot writers of the radix route (staging in shared memory).
template <class Tok>
struct StageOut {
  int32_t *sj;
  float *ss;
  Tok tok;
  __device__ void operator()(int r, int c, uint32_t u) const {
    sj[r] = tok(c);
    ss[r] = key_score(u);
  }
};
struct StagePad {
  int32_t *sj;
  float *ss;
  __device__ void operator()(int r) const {
    sj[r] = -1;
    ss[r] = 0.f;
  }
};

// cs: the candidates (loaded; mx/mn: this thread's max and min of them, as load()
// returns).  sc: the same scores, read again by the radix route.  n <= 65536.
// work: sl_work_bytes(k) bytes of shared memory, 16-byte aligned.  tok(c): the
// output index of candidate c.  out_idx / out_scores (nullable): the global row.
// Called by all NT threads; contains __syncthreads().
template <int NT, class Cands, class Src, class Tok>
__device__ void select_topk_lin(const Cands &cs, float mx, float mn, const Src &sc, int n, int k,
                                SlShared &sh, uint8_t *work, Tok tok, int32_t *out_idx,
                                float *out_scores) {
  static_assert(SL_BINS % NT == 0 && NT % 32 == 0, "whole buckets per thread");
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int NW = NT / 32;
  const float NEG = neg_inf();
  int32_t *st_j = reinterpret_cast<int32_t *>(work);
  float *st_s = reinterpret_cast<float *>(work + (size_t)4 * k);
  const int cap = sl_cap(k);
  float *sv_s = reinterpret_cast<float *>(work + (size_t)8 * k);
  uint16_t *sv_c = reinterpret_cast<uint16_t *>(work + (size_t)8 * k + (size_t)4 * cap);
  uint32_t *off = sh.lin.off;

  // 1. max and min over the CTA
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
  }
  if (lane == 0) {
    sh.lin.wmx[warp] = mx;
    sh.lin.wmn[warp] = mn;
  }
  for (int i = tid; i < SL_WORDS; i += NT) off[i] = 0u;
  if (tid == 0) {
    sh.lin.misc[0] = -1;  // b*: none until the scan finds it
    sh.lin.misc[1] = 0;
    sh.lin.misc[2] = 0;
  }
  __syncthreads();
  mx = NEG;
  mn = -NEG;
#pragma unroll
  for (int w = 0; w < NW; w++) {
    mx = fmaxf(mx, sh.lin.wmx[w]);
    mn = fminf(mn, sh.lin.wmn[w]);
  }
  const LinMap map{mx, (mn < mx) ? (float)SL_BINS / (mx - mn) : 0.f};

  // 2. histogram
  cs.each([&](float x, int) {
    if (x != NEG) atomicAdd(&off[sl_slot(map(x))], 1u);
  });
  __syncthreads();

  // 3. first slot of every bucket, and b*
  int kp;
  {
    constexpr int PER = SL_BINS / NT;
    uint32_t h[PER];
    int local = 0;
#pragma unroll
    for (int i = 0; i < PER; i++) {
      h[i] = off[sl_slot(tid * PER + i)];
      local += (int)h[i];
    }
    int total;
    int run = block_exclusive_scan<NT>(local, sh.lin.warp_tot, &total);
    kp = min(k, total);
#pragma unroll
    for (int i = 0; i < PER; i++) {
      const int b = tid * PER + i;
      if (run < kp && run + (int)h[i] >= kp) {
        sh.lin.misc[0] = b;
        sh.lin.misc[1] = run;
        sh.lin.misc[2] = (int)h[i];
      }
      off[sl_slot(b)] = (uint32_t)run;
      run += (int)h[i];
    }
  }
  __syncthreads();
  const int bstar = sh.lin.misc[0];
  const int nsurv = bstar >= 0 ? sh.lin.misc[1] + sh.lin.misc[2] : 0;

  if (nsurv > cap) {
    // heavy ties at the boundary: the radix route (its lists reuse the working bytes)
    __syncthreads();
    auto key = [&](int c) -> uint32_t {
      const float x = sc.ld1(c);
      return x != NEG ? score_key(x) : 0u;
    };
    select_topk<NT>(key, n, k, sh.radix, reinterpret_cast<uint32_t *>(work),
                    reinterpret_cast<int *>(work + (size_t)4 * k),
                    reinterpret_cast<uint32_t *>(work + (size_t)8 * k),
                    reinterpret_cast<int *>(work + (size_t)12 * k), StageOut<Tok>{st_j, st_s, tok},
                    StagePad{st_j, st_s});
  } else {
    // 4. scatter the survivors to their buckets
    cs.each([&](float x, int c) {
      const int b = map(x);
      if (x != NEG && b <= bstar) {
        const uint32_t p = atomicAdd(&off[sl_slot(b)], 1u);
        sv_s[p] = x;
        sv_c[p] = (uint16_t)c;
      }
    });
    __syncthreads();
    // 5. rank within the bucket; bucket b now spans [end(b - 1), end(b))
    for (int p = tid; p < nsurv; p += NT) {
      const float x = sv_s[p];
      const int c = sv_c[p];
      const int b = map(x);
      const int st = b ? (int)off[sl_slot(b - 1)] : 0, en = (int)off[sl_slot(b)];
      int r = st;
      for (int t = st; t < en; t++) {
        const float y = sv_s[t];
        r += (y > x) || (y == x && (int)sv_c[t] < c);
      }
      if (r < kp) {
        st_j[r] = tok(c);
        st_s[r] = x;
      }
    }
    for (int r = kp + tid; r < k; r += NT) {
      st_j[r] = -1;
      st_s[r] = 0.f;
    }
    __syncthreads();
  }

  // 6. the row, with coalesced stores
  const bool vec = (k & 3) == 0 && (reinterpret_cast<uintptr_t>(out_idx) & 15) == 0 &&
                   (reinterpret_cast<uintptr_t>(out_scores) & 15) == 0;
  if (vec) {
    const int k4 = k >> 2;
    for (int r = tid; r < k4; r += NT) {
      reinterpret_cast<int4 *>(out_idx)[r] = reinterpret_cast<const int4 *>(st_j)[r];
      if (out_scores)
        reinterpret_cast<float4 *>(out_scores)[r] = reinterpret_cast<const float4 *>(st_s)[r];
    }
  } else {
    for (int r = tid; r < k; r += NT) {
      out_idx[r] = st_j[r];
      if (out_scores) out_scores[r] = st_s[r];
    }
  }
  __syncthreads();
}

}  // namespace hisa

namespace hisa {

// ---------------------------------------------------------------------------
// Exact top-k of a row made of whole 128-score segments (the token stage: one segment
// per selected block), candidates in registers.
//
// The steps of select_topk_lin, shaped for this row layout:
//  * register group j of warp w is segment j * NT/32 + w (four scores per lane), so
//    the segment lookups and the "is this the query's own block" test are uniform
//    across the warp;
//  * the number of candidates is known from the block list (the caller passes it),
//    so the buckets need not count every candidate: the buckets cover
//    [hi - span, hi] with span = (hi - lo) * min(1, 2.4 k / n) -- with k a quarter of
//    n the k-th best score lies well inside it for bell-shaped rows, so the buckets
//    are about twice as fine where the output is -- and only scores inside the span
//    are counted; the last bucket takes the rest (its count is the remainder) and
//    -inf is never counted.  Exactness never depends on the span: a k-th score below
//    it only makes the last bucket the boundary one, whose members then all survive
//    (or, past the survivor space, take the radix route);
//  * survivors are scattered as (score, token) pairs, so that ranking needs no
//    lookup, and each counts the higher scores of its bucket four at a time (the
//    survivor array is followed by -inf pads, and later buckets only hold lower
//    scores, so reading past the bucket's end never changes a count); equal scores
//    compare tokens (blocks are ascending, so token order is candidate order).
constexpr int SG_BINS = 4096;
constexpr int SG_LAST = SG_BINS - 1;   // scores below the span (and the remainder count)
constexpr int SG_WORDS = SG_BINS + 4;  // + the -inf bin, rounded to 16 bytes

struct SgShared {
  union {
    SelectShared radix;
    struct {
      uint32_t off[SG_WORDS];  // counts, then first slots, then (after the scatter) ends
      int warp_tot[33];
      float wmx[32], wmn[32];
      int misc[4];
    } lin;
  };
};

// Working bytes: staged indices int32[k] | staged scores f32[k] | survivors
// (f32 score, i32 token)[cap + 4]; the radix route reuses them as its four lists.
__host__ __device__ inline int sg_cap(int k) { return (k + SL_SLACK + 7) & ~7; }
__host__ __device__ inline size_t sg_work_bytes(int k) {
  const size_t a = (size_t)8 * k + (size_t)8 * (sg_cap(k) + 4);
  const size_t b = (size_t)16 * k;
  return ((a > b ? a : b) + 15) & ~(size_t)15;
}

// bucket(x) = min(round((hi - x) * inv), SG_LAST) for a finite x <= hi, and SG_BINS
// for -inf: the sum of the multiply-add is then +inf (or NaN when inv = 0), whose bit
// pattern lies at least 2^29 above that of 2^23 while every finite sum lies far below,
// so bit 29 of the difference separates the two.
struct SgMap {
  float hi, inv;
  __device__ __forceinline__ int operator()(float x) const {
    const float t = fmaf(hi - x, inv, 8388608.0f);
    const uint32_t u = (uint32_t)__float_as_int(t) - 0x4B000000u;
    return (int)min(u, (uint32_t)SG_LAST) + (int)(u >> 29);
  }
};

// f: KPT scores per thread (group j of warp w = segment j * NW + w; lane l holds its
// scores 4l..4l+3), -inf past the row.  nseg: segments in the row (only the last may
// hold -inf); nvalid: its finite scores.  seg_base(s): the first score of segment s
// in memory (the radix route reads the row again); seg_tok[s]: the token of its first
// score (shared memory).  k >= 1; nseg * 128 <= 65536.
template <int NT, int KPT, class SegBase>
__device__ void select_topk_seg(const float (&f)[KPT], int nseg, int nvalid, int k, SgShared &sh,
                                uint8_t *work, SegBase seg_base, const int32_t *seg_tok,
                                int32_t *out_idx, float *out_scores) {
  static_assert(SG_BINS % NT == 0 && NT % 32 == 0 && KPT % 4 == 0, "layout");
  constexpr int NW = NT / 32;
  constexpr int PER = SG_BINS / NT;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const float NEG = neg_inf();
  const int n = nseg * 128;
  int32_t *st_j = reinterpret_cast<int32_t *>(work);
  float *st_s = reinterpret_cast<float *>(work + (size_t)4 * k);
  const int cap = sg_cap(k);
  float2 *sv = reinterpret_cast<float2 *>(work + (size_t)8 * k);  // (score, token bits)
  uint32_t *off = sh.lin.off;

  // 1. max and min (only the own block, the last segment, can hold -inf)
  float mx = NEG, mn = -NEG;
#pragma unroll
  for (int j = 0; j < KPT / 4; j++) {
    const int s = j * NW + warp;
#pragma unroll
    for (int e = 0; e < 4; e++) mx = fmaxf(mx, f[4 * j + e]);
    if (s < nseg - 1) {
#pragma unroll
      for (int e = 0; e < 4; e++) mn = fminf(mn, f[4 * j + e]);
    } else if (s == nseg - 1) {
#pragma unroll
      for (int e = 0; e < 4; e++)
        if (f[4 * j + e] != NEG) mn = fminf(mn, f[4 * j + e]);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
  }
  if (lane == 0) {
    sh.lin.wmx[warp] = mx;
    sh.lin.wmn[warp] = mn;
  }
  for (int i = tid; i < SG_WORDS / 4; i += NT)
    reinterpret_cast<uint4 *>(off)[i] = make_uint4(0u, 0u, 0u, 0u);
  if (tid == 0) {
    sh.lin.misc[0] = -1;
    sh.lin.misc[1] = 0;
    sh.lin.misc[2] = 0;
  }
  __syncthreads();
  mx = NEG;
  mn = -NEG;
#pragma unroll
  for (int w = 0; w < NW; w++) {
    mx = fmaxf(mx, sh.lin.wmx[w]);
    mn = fminf(mn, sh.lin.wmn[w]);
  }
  const float frac = fminf(1.f, 2.4f * (float)k / (float)n);
  const float span = (mx - mn) * frac;
  const SgMap map{mx, (mn < mx && span > 0.f) ? (float)SG_LAST / span : 0.f};

  // 2. histogram of the scores inside the span
#pragma unroll
  for (int i = 0; i < KPT; i++) {
    const int b = map(f[i]);
    if (b < SG_LAST) atomicAdd(&off[b], 1u);
  }
  __syncthreads();

  // 3. first slots and b* (thread t owns buckets PER t .. PER t + PER - 1, read four at
  // a time; the last bucket's count is what the others leave of nvalid)
  const int kp = min(k, nvalid);
  {
    uint4 *off4 = reinterpret_cast<uint4 *>(off) + tid * (PER / 4);
    int local = 0;
#pragma unroll
    for (int i = 0; i < PER / 4; i++) {
      const uint4 v = off4[i];
      local += (int)(v.x + v.y + v.z + v.w);
    }
    int total;
    int run = block_exclusive_scan<NT>(local, sh.lin.warp_tot, &total);
#pragma unroll
    for (int i = 0; i < PER / 4; i++) {
      const uint4 v = off4[i];
      uint32_t h[4] = {v.x, v.y, v.z, v.w};
      if (tid == NT - 1 && i == PER / 4 - 1) h[3] = (uint32_t)(nvalid - total);
      uint32_t o[4];
#pragma unroll
      for (int e = 0; e < 4; e++) {
        if (run < kp && run + (int)h[e] >= kp) {
          sh.lin.misc[0] = tid * PER + 4 * i + e;
          sh.lin.misc[1] = run;
          sh.lin.misc[2] = (int)h[e];
        }
        o[e] = (uint32_t)run;
        run += (int)h[e];
      }
      off4[i] = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
  __syncthreads();
  const int bstar = sh.lin.misc[0];
  const int nsurv = bstar >= 0 ? sh.lin.misc[1] + sh.lin.misc[2] : 0;

  if (nsurv > cap) {
    // heavy ties at the boundary: the radix route (its lists reuse the working bytes)
    __syncthreads();
    auto key = [&](int c) -> uint32_t {
      const float x = seg_base(c >> 7)[c & 127];
      return x != NEG ? score_key(x) : 0u;
    };
    auto tok = [&](int c) { return seg_tok[c >> 7] + (c & 127); };
    select_topk<NT>(key, n, k, sh.radix, reinterpret_cast<uint32_t *>(work),
                    reinterpret_cast<int *>(work + (size_t)4 * k),
                    reinterpret_cast<uint32_t *>(work + (size_t)8 * k),
                    reinterpret_cast<int *>(work + (size_t)12 * k),
                    StageOut<decltype(tok)>{st_j, st_s, tok}, StagePad{st_j, st_s});
  } else {
    // 4. scatter the survivors (buckets 0..b*) as (score, token) to their buckets
#pragma unroll
    for (int j = 0; j < KPT / 4; j++) {
      const int s = j * NW + warp;
      const int t0 = (s < nseg ? seg_tok[s] : 0) + lane * 4;
#pragma unroll
      for (int e = 0; e < 4; e++) {
        const float x = f[4 * j + e];
        const int b = map(x);
        if (b <= bstar) {
          const uint32_t p = atomicAdd(&off[b], 1u);
          if (p < (uint32_t)cap) sv[p] = make_float2(x, __int_as_float(t0 + e));
        }
      }
    }
    if (tid < 4) sv[nsurv + tid] = make_float2(NEG, 0.f);  // pads read by the last bucket
    __syncthreads();
    // 5. rank within the bucket; bucket b spans [end(b - 1), end(b))
    for (int p = tid; p < nsurv; p += NT) {
      const float2 me = sv[p];
      const float x = me.x;
      const int tk = __float_as_int(me.y);
      const int b = map(x);
      const int st = b ? (int)off[b - 1] : 0, en = (int)off[b];
      int r = st;
      for (int t = st; t < en; t += 4) {
        const float2 y0 = sv[t], y1 = sv[t + 1], y2 = sv[t + 2], y3 = sv[t + 3];
        r += (y0.x > x) + (y1.x > x) + (y2.x > x) + (y3.x > x);
        // equal scores: the lower token first (past the bucket's end no score is equal)
        r += (y0.x == x && __float_as_int(y0.y) < tk) + (y1.x == x && __float_as_int(y1.y) < tk) +
             (y2.x == x && __float_as_int(y2.y) < tk) + (y3.x == x && __float_as_int(y3.y) < tk);
      }
      if (r < kp) {
        st_j[r] = tk;
        st_s[r] = x;
      }
    }
    for (int r = kp + tid; r < k; r += NT) {
      st_j[r] = -1;
      st_s[r] = 0.f;
    }
    __syncthreads();
  }

  // 6. the row, with coalesced stores
  const bool vec = (k & 3) == 0 && (reinterpret_cast<uintptr_t>(out_idx) & 15) == 0 &&
                   (reinterpret_cast<uintptr_t>(out_scores) & 15) == 0;
  if (vec) {
    const int k4 = k >> 2;
    for (int r = tid; r < k4; r += NT) {
      reinterpret_cast<int4 *>(out_idx)[r] = reinterpret_cast<const int4 *>(st_j)[r];
      if (out_scores)
        reinterpret_cast<float4 *>(out_scores)[r] = reinterpret_cast<const float4 *>(st_s)[r];
    }
  } else {
    for (int r = tid; r < k; r += NT) {
      out_idx[r] = st_j[r];
      if (out_scores) out_scores[r] = st_s[r];
    }
  }
  __syncthreads();
}

}  // namespace hisa
