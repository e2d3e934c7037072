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
//     then output index asc, so candidates need not come in index order); its bucket
//     start plus that count is its output slot, and the slots below kp are kept (b*
//     keeps its best kp - start(b*));
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
// Called by all NT threads; contains __syncthreads().  The radix route breaks ties by
// candidate number, which is the output order only when the candidates come in
// increasing tok order; without RADIX the routine instead writes nothing and returns
// false when it would need that route (heavy ties at the boundary), else true.
template <int NT, bool RADIX = true, class Cands, class Src, class Tok>
__device__ bool select_topk_lin(const Cands &cs, float mx, float mn, const Src &sc, int n, int k,
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

  if (!RADIX && nsurv > cap) return false;  // uniform: every thread read the same b*
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
      int tk = -1;  // this candidate's output index, looked up only for an equal score
      for (int t = st; t < en; t++) {
        const float y = sv_s[t];
        if (y == x && t != p) {
          if (tk < 0) tk = tok(c);
          r += tok((int)sv_c[t]) < tk;
        }
        r += y > x;
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
  return true;
}

}  // namespace hisa

namespace hisa {

// ---------------------------------------------------------------------------
// Exact top-k through linear score buckets, candidates held in registers (the
// token stage).
//
// Input: n raw fp32 scores in candidate (= token) order, -inf marking a position
// that is not a candidate (finite scores are the contract).  Each of the NT threads
// loads KPT of them once (coalesced 16-byte loads; candidate c = ((i/4)*NT +
// thread)*4 + i%4) and keeps them in registers.  Then:
// 1. max/min and count of the candidate scores (fused with the load);
// 2. histogram over LIN_BINS buckets linear in the score between max and min
//    (bucket 0 holds the highest scores).  The bucket map is monotone in the score,
//    so bucket order is score order;
// 3. one scan gives every bucket its output offset and finds the bucket b* that
//    holds the k-th best score;
// 4. candidates in buckets before b* are scattered to their bucket's output range,
//    those in b* are gathered apart, each as a 64-bit (key, ~index) composite whose
//    unsigned order is the output order (score desc, index asc);
// 5. the b* candidates are ranked exactly and the best k - |buckets before b*| of
//    them fill the end of the output;
// 6. every other survivor is ranked within its own bucket (a handful of elements for
//    continuous scores) and written to its final slot.
// A boundary bucket with more than k members (heavy ties) sends the query through
// the radix routine above instead, reading the scores again.

constexpr int LIN_BINS = 2048;
// Bucket b lives at word b + b / 32 of the count arrays: a thread scanning eight
// consecutive buckets then touches 32 distinct banks across its warp.
constexpr int LIN_WORDS = LIN_BINS + LIN_BINS / 32;
__device__ __forceinline__ int lin_slot(int b) { return b + (b >> 5); }

struct LinShared {
  union {
    SelectShared radix;
    struct {
      uint32_t cnt[LIN_WORDS];
      uint32_t off[LIN_WORDS];
      int warp_tot[33];
      int wn[32];
      float wmx[32], wmn[32];
      uint32_t misc[8];
    } lin;
  };
};

// rint((smax - s) * inv) clamped to the last bucket, through the 2^23 magic number
// instead of a float-to-int conversion: smax - s >= 0, so the sum stays in [2^23, 2^24)
// where a float's bits count in units of one; monotone (non-increasing) in s.
__device__ __forceinline__ int lin_bucket(float s, float smax, float inv) {
  return min(__float_as_int(fmaf(smax - s, inv, 8388608.0f)) - 0x4B000000, LIN_BINS - 1);
}

// sc: the n raw scores (RowScores or SegScores; four consecutive candidates never
// straddle a segment).  work: 4*k words (2*k uint64) of shared scratch.
template <int NT, int KPT, class Src, class Out, class Pad>
__device__ void select_topk_reg(Src sc, int n, int k, LinShared &sh, uint32_t *work, Out out,
                                Pad pad) {
  static_assert(KPT % 4 == 0, "scores are loaded four at a time");
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int NW = NT / 32;
  uint64_t *surv = reinterpret_cast<uint64_t *>(work);      // k survivors
  uint64_t *bnd = reinterpret_cast<uint64_t *>(work) + k;   // up to k boundary members
  const float NEG = -__int_as_float(0x7f800000);             // -inf

  float f[KPT];
  float mx = NEG, mn = -NEG;
  int nv = 0;
#pragma unroll
  for (int j = 0; j < KPT / 4; j++) {
    const int c0 = (j * NT + tid) * 4;
    float4 v = make_float4(NEG, NEG, NEG, NEG);
    if (c0 + 3 < n) {
      v = sc.ld4(c0);
    } else if (c0 < n) {
      v.x = sc.ld1(c0);
      if (c0 + 1 < n) v.y = sc.ld1(c0 + 1);
      if (c0 + 2 < n) v.z = sc.ld1(c0 + 2);
    }
    f[4 * j] = v.x;
    f[4 * j + 1] = v.y;
    f[4 * j + 2] = v.z;
    f[4 * j + 3] = v.w;
#pragma unroll
    for (int e = 0; e < 4; e++) {
      const float x = f[4 * j + e];
      if (x != NEG) {
        mx = fmaxf(mx, x);
        mn = fminf(mn, x);
        nv++;
      }
    }
  }
  auto cand = [&](int i) { return ((i >> 2) * NT + tid) * 4 + (i & 3); };
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    nv += __shfl_xor_sync(0xffffffffu, nv, o);
  }
  if (lane == 0) {
    sh.lin.wmx[warp] = mx;
    sh.lin.wmn[warp] = mn;
    sh.lin.wn[warp] = nv;
  }
  for (int i = tid; i < LIN_WORDS; i += NT) sh.lin.cnt[i] = 0u;
  __syncthreads();
  mx = NEG;
  mn = -NEG;
  nv = 0;
#pragma unroll
  for (int w = 0; w < NW; w++) {
    mx = fmaxf(mx, sh.lin.wmx[w]);
    mn = fminf(mn, sh.lin.wmn[w]);
    nv += sh.lin.wn[w];
  }
  const int nvalid = nv;
  const float smax = mx;
  const float range = mx - mn;
  float inv = (nvalid > 0 && range > 0.f) ? (float)LIN_BINS / range : 0.f;
  if (!isfinite(inv)) inv = 0.f;  // a range too narrow to divide: one bucket, radix route

  // 2. histogram
#pragma unroll
  for (int i = 0; i < KPT; i++)
    if (f[i] != NEG) atomicAdd(&sh.lin.cnt[lin_slot(lin_bucket(f[i], smax, inv))], 1u);
  __syncthreads();

  // 3. offsets and the boundary bucket
  const int kp = min(k, nvalid);
  {
    constexpr int per = LIN_BINS / NT;
    uint32_t h[per];
    int local = 0;
#pragma unroll
    for (int i = 0; i < per; i++) {
      h[i] = sh.lin.cnt[lin_slot(tid * per + i)];
      local += (int)h[i];
    }
    int total;
    int run = block_exclusive_scan<NT>(local, sh.lin.warp_tot, &total);
    if (tid == 0) {
      sh.lin.misc[3] = LIN_BINS;  // no boundary bucket when every candidate survives
      sh.lin.misc[4] = (uint32_t)kp;
      sh.lin.misc[5] = 0u;        // boundary fill counter
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < per; i++) {
      const int b = tid * per + i;
      if (nvalid > k && run < k && run + (int)h[i] >= k) {
        sh.lin.misc[3] = (uint32_t)b;
        sh.lin.misc[4] = (uint32_t)run;
      }
      sh.lin.off[lin_slot(b)] = (uint32_t)run;
      sh.lin.cnt[lin_slot(b)] = (uint32_t)run;  // becomes the scatter cursor
      run += (int)h[i];
    }
  }
  __syncthreads();
  const int bstar = (int)sh.lin.misc[3];
  const int above = (int)sh.lin.misc[4];  // survivors in buckets before b*
  const int need = kp - above;             // survivors taken from b*

  // 4. scatter
#pragma unroll
  for (int i = 0; i < KPT; i++) {
    if (f[i] != NEG) {
      const int b = lin_bucket(f[i], smax, inv);
      if (b < bstar) {
        const uint32_t slot = atomicAdd(&sh.lin.cnt[lin_slot(b)], 1u);
        surv[slot] = rank_key(f[i], cand(i));
      } else if (b == bstar) {
        const uint32_t e = atomicAdd(&sh.lin.misc[5], 1u);
        if (e < (uint32_t)k) bnd[e] = rank_key(f[i], cand(i));
      }
    }
  }
  __syncthreads();
  const int nbnd = (int)sh.lin.misc[5];
  if (nbnd > k) {  // heavy ties at the boundary: exact radix route
    __syncthreads();
    auto key = [&](int c) -> uint32_t {
      const float x = sc.ld1(c);
      return x != NEG ? score_key(x) : 0u;
    };
    select_topk<NT>(key, n, k, sh.radix, work, reinterpret_cast<int *>(work + k), work + 2 * k,
                    reinterpret_cast<int *>(work + 3 * k), out, pad);
    return;
  }

  // 5. the boundary bucket, ranked exactly
  if (need > 0) {
    for (int e = tid; e < nbnd; e += NT) {
      const uint64_t me = bnd[e];
      int rank = 0;
      for (int t = 0; t < nbnd; t++) rank += bnd[t] > me;
      if (rank < need) out(above + rank, (int)~(uint32_t)me, (uint32_t)(me >> 32));
    }
  }
  // 6. everything above the boundary, ranked within its own bucket
  for (int s = tid; s < above; s += NT) {
    const uint64_t me = surv[s];
    const int b = lin_bucket(key_score((uint32_t)(me >> 32)), smax, inv);
    const int st = (int)sh.lin.off[lin_slot(b)], en = (int)sh.lin.cnt[lin_slot(b)];
    int rank = 0;
    for (int t = st; t < en; t++) rank += surv[t] > me;
    out(st + rank, (int)~(uint32_t)me, (uint32_t)(me >> 32));
  }
  for (int r = kp + tid; r < k; r += NT) pad(r);
  __syncthreads();
}

}  // namespace hisa
