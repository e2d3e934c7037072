// Top-m block choice of HISA stage 1 for one query, executed by one warp.
//
// HISA summary page (aitrends.kr), paragraph on stage 1: the first block and the
// last two blocks (read as the query's own block and the one before it) are always
// kept and count inside m; the rest of the m slots go to the best-scoring eligible
// blocks, ties to the lower block.  The scores arrive as order-preserving keys
// (0 = forced or not eligible).
#pragma once

#include "common.cuh"

namespace hisa {

// Key T of the mfree-th best free block and how many blocks with key == T are
// still needed, by a radix select over 8-bit digits (most significant first) with a
// per-warp histogram of 256 bins in shared memory.  keys[b] == 0 marks a block that
// is not free (forced, or after the query).  Executed by one full warp; `hist0`, if
// not null, already holds the histogram of the top digit of keys[0..E).
__device__ __forceinline__ void warp_radix_threshold(const uint32_t *keys, int E, int mfree, uint32_t *hist,
                                     bool hist0_ready, uint32_t &T_out, int &need_eq_out) {
  const int lane = threadIdx.x & 31;
  uint32_t prefix = 0u, pmask = 0u;
  int remaining = mfree;
#pragma unroll 1
  for (int shift = 24; shift >= 0; shift -= 8) {
    if (!(shift == 24 && hist0_ready)) {
#pragma unroll
      for (int i = 0; i < 8; i++) hist[lane * 8 + i] = 0u;
      __syncwarp();
      for (int b = lane; b < E; b += 32) {
        const uint32_t u = keys[b];
        if (u != 0u && (u & pmask) == prefix) atomicAdd(&hist[(u >> shift) & 255u], 1u);
      }
      __syncwarp();
    }
    // lane l owns bins 255 - 8l .. 248 - 8l (highest digits first)
    int h[8], local = 0;
#pragma unroll
    for (int i = 0; i < 8; i++) {
      h[i] = (int)hist[255 - lane * 8 - i];
      local += h[i];
    }
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    const int excl = incl - local;
    // the lane whose range holds the remaining-th key
    const unsigned who = __ballot_sync(0xffffffffu, excl < remaining && incl >= remaining);
    const int src = __ffs(who) - 1;
    int digit = 0, above = 0, inbin = 0;
    if (lane == src) {
      int run = excl;
#pragma unroll
      for (int i = 0; i < 8; i++) {
        if (run < remaining && run + h[i] >= remaining) {
          digit = 255 - lane * 8 - i;
          above = run;
          inbin = h[i];
        }
        run += h[i];
      }
    }
    digit = __shfl_sync(0xffffffffu, digit, src);
    above = __shfl_sync(0xffffffffu, above, src);
    inbin = __shfl_sync(0xffffffffu, inbin, src);
    __syncwarp();
    remaining -= above;
    prefix |= (uint32_t)digit << shift;
    pmask |= 255u << shift;
    if (inbin == remaining) {  // the whole bin is selected
      T_out = prefix ? prefix - 1u : 0u;
      need_eq_out = 0;
      return;
    }
  }
  T_out = prefix;
  need_eq_out = remaining;
}

// Top-(m - |forced|) of the keys[0..E) of one query (forced blocks and blocks after
// the query hold key 0), written in ascending block order with the forced blocks.
// Executed by one full warp.
__device__ __forceinline__ void warp_select_blocks(const uint32_t *keys, int E, int own, int m,
                                   int32_t *dst, int32_t *dst2, uint32_t *hist,
                                   bool hist0_ready) {
  const int lane = threadIdx.x & 31;
  const int nf = min(m, 3);  // forced: own, previous, first (E > m >= 3 makes them distinct)
  const int mfree = m - nf;
  auto forced = [&](int b) {
    return b == own || (nf >= 2 && b == own - 1) || (nf >= 3 && b == 0);
  };
  uint32_t T = 0xffffffffu;  // nothing free is taken when mfree == 0
  int need_eq = 0;
  if (mfree > 0) warp_radix_threshold(keys, E, mfree, hist, hist0_ready, T, need_eq);
  const unsigned lt = (1u << lane) - 1u;
  int eqr = 0, outp = 0;
  for (int b0 = 0; b0 < E; b0 += 32) {
    const int b = b0 + lane;
    const uint32_t u = b < E ? keys[b] : 0u;
    const bool is_eq = need_eq > 0 && u != 0u && u == T;
    const unsigned beq = __ballot_sync(0xffffffffu, is_eq);
    const bool sel = (b < E && forced(b)) || (mfree > 0 && u != 0u && u > T) ||
                     (is_eq && eqr + __popc(beq & lt) < need_eq);
    const unsigned bsel = __ballot_sync(0xffffffffu, sel);
    if (sel) {
      const int p = outp + __popc(bsel & lt);
      dst[p] = b;
      if (dst2) dst2[p] = b;
    }
    eqr += __popc(beq);
    outp += __popc(bsel);
  }
  for (int i = outp + lane; i < m; i += 32) {  // only reachable if fewer than m exist
    dst[i] = -1;
    if (dst2) dst2[i] = -1;
  }
}

}  // namespace hisa

namespace hisa {

// CTA-wide version of the above for NT >= 256 threads: the radix select over 8-bit
// digits uses one histogram bin per thread, and the selected blocks are emitted in
// ascending order through block scans (thread t owns a contiguous range of blocks).
// `hist` holds 256 words, `warp_tot` NT/32 + 1 ints, `bc` 4 ints of shared memory.
template <int NT>
__device__ void cta_select_blocks(const uint32_t *keys, int E, int own, int m, int32_t *dst,
                                  int32_t *dst2, uint32_t *hist, int *warp_tot, int *bc) {
  static_assert(NT >= 256, "one histogram bin per thread");
  const int tid = threadIdx.x;
  const int nf = min(m, 3);
  const int mfree = m - nf;
  uint32_t T = 0xffffffffu;  // nothing free is taken when mfree == 0
  int need_eq = 0;
  if (mfree > 0) {
    uint32_t prefix = 0u, pmask = 0u;
    int remaining = mfree;
    bool done = false;
#pragma unroll 1
    for (int shift = 24; shift >= 0 && !done; shift -= 8) {
      if (tid < 256) hist[tid] = 0u;
      __syncthreads();
      for (int b = tid; b < E; b += NT) {
        const uint32_t u = keys[b];
        if (u != 0u && (u & pmask) == prefix) atomicAdd(&hist[(u >> shift) & 255u], 1u);
      }
      __syncthreads();
      const int h = tid < 256 ? (int)hist[255 - tid] : 0;  // highest digit first
      int total;
      const int run = block_exclusive_scan<NT>(h, warp_tot, &total);
      if (tid < 256 && run < remaining && run + h >= remaining) {
        bc[0] = 255 - tid;
        bc[1] = run;
        bc[2] = h;
      }
      __syncthreads();
      const int digit = bc[0], above = bc[1], inbin = bc[2];
      remaining -= above;
      prefix |= (uint32_t)digit << shift;
      pmask |= 255u << shift;
      if (inbin == remaining) {  // the whole bin is selected
        T = prefix ? prefix - 1u : 0u;
        need_eq = 0;
        done = true;
      } else if (shift == 0) {
        T = prefix;
        need_eq = remaining;
      }
    }
  }
  auto forced = [&](int b) {
    return b == own || (nf >= 2 && b == own - 1) || (nf >= 3 && b == 0);
  };
  // emission in ascending block order
  const int per = (E + NT - 1) / NT;
  const int b0 = min(E, tid * per), b1 = min(E, b0 + per);
  int neq = 0;
  for (int b = b0; b < b1; b++) {
    const uint32_t u = keys[b];
    neq += (need_eq > 0 && u != 0u && u == T);
  }
  int tot;
  int eqr = block_exclusive_scan<NT>(neq, warp_tot, &tot);
  int nsel = 0;
  {
    int e = eqr;
    for (int b = b0; b < b1; b++) {
      const uint32_t u = keys[b];
      const bool is_eq = need_eq > 0 && u != 0u && u == T;
      nsel += forced(b) || (mfree > 0 && u != 0u && u > T) || (is_eq && e < need_eq);
      e += is_eq;
    }
  }
  int outp = block_exclusive_scan<NT>(nsel, warp_tot, &tot);
  for (int b = b0; b < b1; b++) {
    const uint32_t u = keys[b];
    const bool is_eq = need_eq > 0 && u != 0u && u == T;
    if (forced(b) || (mfree > 0 && u != 0u && u > T) || (is_eq && eqr < need_eq)) {
      dst[outp] = b;
      if (dst2) dst2[outp] = b;
      outp++;
    }
    eqr += is_eq;
  }
  for (int i = tot + tid; i < m; i += NT) {  // only reachable if fewer than m exist
    dst[i] = -1;
    if (dst2) dst2[i] = -1;
  }
  __syncthreads();
}

}  // namespace hisa

namespace hisa {

// Top-m by linear score buckets, for NT >= 256 threads: 256 buckets linear in the
// score between the lowest and the highest free key, one scan for the bucket that
// holds the mfree-th best block, exact ranking (score desc, block asc) of that
// bucket's members, and emission in ascending block order by warp ballots over
// contiguous ranges.  Returns false, with nothing written, when the boundary bucket
// has more than LIN_BLK_CAP members (heavy ties); the caller then uses
// cta_select_blocks.  `scratch` must hold lin_blk_scratch_bytes(E) bytes.
constexpr int LIN_BLK_CAP = 512;

__host__ __device__ inline size_t lin_blk_scratch_bytes(int E) {
  return (size_t)LIN_BLK_CAP * 8 + (size_t)((E + 15) & ~15);
}

template <int NT>
__device__ bool cta_select_blocks_lin(const uint32_t *keys, int E, int own, int m,
                                      int32_t *dst, int32_t *dst2, uint32_t *hist,
                                      int *warp_tot, int *bc, uint8_t *scratch) {
  static_assert(NT >= 256, "one bucket per thread");
  constexpr int NW = NT / 32;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nf = min(m, 3);
  const int mfree = m - nf;
  uint32_t *mem_key = reinterpret_cast<uint32_t *>(scratch);
  int32_t *mem_blk = reinterpret_cast<int32_t *>(scratch) + LIN_BLK_CAP;
  uint8_t *selb = scratch + (size_t)LIN_BLK_CAP * 8;
  auto forced = [&](int b) {
    return b == own || (nf >= 2 && b == own - 1) || (nf >= 3 && b == 0);
  };
  // 1. range of the free scores
  const float NEG = -__int_as_float(0x7f800000);
  float mx = NEG, mn = -NEG;
  for (int b = tid; b < E; b += NT) {
    const uint32_t u = keys[b];
    if (u != 0u) {
      const float s = key_score(u);
      mx = fmaxf(mx, s);
      mn = fminf(mn, s);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
  }
  float *wr = reinterpret_cast<float *>(hist);  // 2 * NW floats, before the histogram
  if (tid < 256) hist[tid] = 0u;
  __syncthreads();
  if (lane == 0) {
    wr[256 + warp] = mx;  // hist has 256 + 2 * NW words
    wr[256 + NW + warp] = mn;
  }
  __syncthreads();
  mx = NEG;
  mn = -NEG;
#pragma unroll
  for (int w = 0; w < NW; w++) {
    mx = fmaxf(mx, wr[256 + w]);
    mn = fminf(mn, wr[256 + NW + w]);
  }
  const float range = mx - mn;
  const float inv = range > 0.f ? 256.f / range : 0.f;
  if (mfree > 0 && !(inv > 0.f && isfinite(inv))) return false;  // one distinct score
  auto bucket = [&](uint32_t u) { return min(__float2int_rz((mx - key_score(u)) * inv), 255); };
  // 2. histogram, 3. boundary bucket
  int bstar = 256, above = 0, nb = 0;
  if (mfree > 0) {
    for (int b = tid; b < E; b += NT) {
      const uint32_t u = keys[b];
      if (u != 0u) atomicAdd(&hist[bucket(u)], 1u);
    }
    __syncthreads();
    const int h = tid < 256 ? (int)hist[tid] : 0;
    int total;
    const int run = block_exclusive_scan<NT>(h, warp_tot, &total);
    if (tid == 0) bc[3] = 0;
    if (tid < 256 && run < mfree && run + h >= mfree) {
      bc[0] = tid;
      bc[1] = run;
      bc[2] = h;
    }
    __syncthreads();
    bstar = bc[0];
    above = bc[1];
    nb = bc[2];
    if (nb > LIN_BLK_CAP) return false;
  }
  const int need = mfree - above;
  // 4. sure picks and forced blocks flagged, boundary members gathered
  for (int b = tid; b < E; b += NT) {
    const uint32_t u = keys[b];
    bool s = forced(b);
    if (u != 0u && mfree > 0) {
      const int bk = bucket(u);
      s = s || bk < bstar;
      if (bk == bstar) {
        const int e = atomicAdd(&bc[3], 1);
        mem_key[e] = u;
        mem_blk[e] = b;
      }
    }
    selb[b] = s ? 1 : 0;
  }
  __syncthreads();
  // 5. the best `need` boundary members
  for (int e = tid; e < nb; e += NT) {
    const uint32_t mk = mem_key[e];
    const int mb = mem_blk[e];
    int rank = 0;
    for (int t = 0; t < nb; t++) {
      const uint32_t tk = mem_key[t];
      rank += (tk > mk) || (tk == mk && mem_blk[t] < mb);
    }
    if (rank < need) selb[mb] = 1;
  }
  __syncthreads();
  // 6. emission: warp w walks blocks [w * per, (w + 1) * per) twice (count, write)
  const int per = ((E + NW - 1) / NW + 31) & ~31;
  const int w0 = min(E, warp * per), w1 = min(E, w0 + per);
  int cnt = 0;
  for (int b0 = w0; b0 < w1; b0 += 32) {
    const int b = b0 + lane;
    cnt += __popc(__ballot_sync(0xffffffffu, b < w1 && selb[b]));
  }
  if (lane == 0) bc[4 + warp] = cnt;  // bc holds 4 + NW ints
  __syncthreads();
  int outp = 0, tot = 0;
  for (int w = 0; w < NW; w++) {
    if (w < warp) outp += bc[4 + w];
    tot += bc[4 + w];
  }
  const unsigned lt = (1u << lane) - 1u;
  for (int b0 = w0; b0 < w1; b0 += 32) {
    const int b = b0 + lane;
    const bool s = b < w1 && selb[b];
    const unsigned mask = __ballot_sync(0xffffffffu, s);
    if (s) {
      dst[outp + __popc(mask & lt)] = b;
      if (dst2) dst2[outp + __popc(mask & lt)] = b;
    }
    outp += __popc(mask);
  }
  for (int i = tot + tid; i < m; i += NT) {  // only reachable if fewer than m exist
    dst[i] = -1;
    if (dst2) dst2[i] = -1;
  }
  __syncthreads();
  return true;
}

}  // namespace hisa
