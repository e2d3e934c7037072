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

// key: n candidate keys (shared or global memory), token order.
// sel_key/sel_c/tmp_key/tmp_c: shared arrays of at least k entries.
// out(rank, c, key) writes one output slot; pad(rank) fills a slot past the survivors.
template <int NT, class Out, class Pad>
__device__ void select_topk(const uint32_t *key, int n, int k, SelectShared &sh,
                            uint32_t *sel_key, int *sel_c, uint32_t *tmp_key, int *tmp_c,
                            Out out, Pad pad) {
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
      uint32_t u = key[c];
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
    uint32_t u = c < c1 ? key[c] : 0u;
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
      uint32_t u = c < c1 ? key[c] : 0u;
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
