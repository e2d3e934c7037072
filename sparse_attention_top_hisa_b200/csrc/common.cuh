// Shared device helpers for the HISA indexer kernels (sm_100a).
#pragma once

#include <atomic>

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/hisa.h"

namespace hisa {

constexpr int D = HISA_INDEX_DIM;  // index-head width (64 bf16 = 128 bytes per row)
constexpr int BLK = HISA_BLOCK;    // tokens per block
constexpr int ROW_BYTES = D * 2;

// ---------------------------------------------------------------------------
// device status word: kernels OR (1 << hisa_status) into it

__device__ __forceinline__ void raise_status(int *status, hisa_status s) {
  if (status) atomicOr(status, 1 << (int)s);
}

// ---------------------------------------------------------------------------
// bf16 helpers (bit patterns packed two per 32-bit word, element 0 in the low half)

__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Order-preserving map of a finite fp32 score to uint32 (larger score -> larger key).
// -0.0 is folded onto +0.0 first so that they compare equal. Every finite score maps
// to a key >= 0x00800000, so 0 is free to mean "not a candidate".
__device__ __forceinline__ uint32_t score_key(float s) {
  uint32_t b = __float_as_uint(s);
  if (b == 0x80000000u) b = 0u;
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

__device__ __forceinline__ float key_score(uint32_t u) {
  uint32_t b = (u & 0x80000000u) ? (u & 0x7fffffffu) : ~u;
  return __uint_as_float(b);
}

// ---------------------------------------------------------------------------
// token score: q . k over 64 dims, fp32.  Both the HISA token stage and the flat
// scan use exactly this evaluation (two sequential FMA chains over dims 0..31 and
// 32..63, then one add), so equal inputs give bit-identical scores in both paths.

struct QRegs {
  float v[D];
};

__device__ __forceinline__ void load_q(QRegs &q, const uint16_t *qrow) {
  const uint4 *p = reinterpret_cast<const uint4 *>(qrow);
#pragma unroll
  for (int c = 0; c < 8; c++) {
    uint4 w = __ldg(p + c);
    q.v[c * 8 + 0] = bf_lo(w.x);
    q.v[c * 8 + 1] = bf_hi(w.x);
    q.v[c * 8 + 2] = bf_lo(w.y);
    q.v[c * 8 + 3] = bf_hi(w.y);
    q.v[c * 8 + 4] = bf_lo(w.z);
    q.v[c * 8 + 5] = bf_hi(w.z);
    q.v[c * 8 + 6] = bf_lo(w.w);
    q.v[c * 8 + 7] = bf_hi(w.w);
  }
}

// one 16-byte chunk (8 dims starting at 8*c) into the chain
__device__ __forceinline__ float fma_chunk(const QRegs &q, int c, uint4 w, float acc) {
  acc = fmaf(q.v[c * 8 + 0], bf_lo(w.x), acc);
  acc = fmaf(q.v[c * 8 + 1], bf_hi(w.x), acc);
  acc = fmaf(q.v[c * 8 + 2], bf_lo(w.y), acc);
  acc = fmaf(q.v[c * 8 + 3], bf_hi(w.y), acc);
  acc = fmaf(q.v[c * 8 + 4], bf_lo(w.z), acc);
  acc = fmaf(q.v[c * 8 + 5], bf_hi(w.z), acc);
  acc = fmaf(q.v[c * 8 + 6], bf_lo(w.w), acc);
  acc = fmaf(q.v[c * 8 + 7], bf_hi(w.w), acc);
  return acc;
}

// Score of one key given its 8 chunks (chunk c holds dims 8c..8c+7).
__device__ __forceinline__ float token_score(const QRegs &q, const uint4 (&w)[8]) {
  float a = 0.f, b = 0.f;
#pragma unroll
  for (int c = 0; c < 4; c++) {
    a = fma_chunk(q, c, w[c], a);
    b = fma_chunk(q, c + 4, w[c + 4], b);
  }
  return a + b;
}

// ---------------------------------------------------------------------------
// sequence bookkeeping

// Sequence owning query row `row` (last s with cu_q[s] <= row < cu_q[s+1]).
__device__ __forceinline__ int find_seq(const int32_t *cu_q, int S, int row) {
  int lo = 0, hi = S - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (__ldg(cu_q + mid) <= row) lo = mid; else hi = mid - 1;
  }
  while (lo < S - 1 && __ldg(cu_q + lo + 1) <= row) lo++;
  return lo;
}

struct QueryInfo {
  int seq;    // sequence index
  int pos;    // sequence-local position of the query
  int kbase;  // first key row of the sequence's region
  int len;    // live key count
  bool ok;
};

// Locate a query row and validate its sequence (region alignment and lengths).
__device__ __forceinline__ QueryInfo locate(const int32_t *cu_q, const int32_t *cu_k,
                                            const int32_t *seqlens, int S, int row,
                                            int *status) {
  QueryInfo r;
  r.seq = find_seq(cu_q, S, row);
  int q0 = __ldg(cu_q + r.seq), q1 = __ldg(cu_q + r.seq + 1);
  int k0 = __ldg(cu_k + r.seq), k1 = __ldg(cu_k + r.seq + 1);
  r.kbase = k0;
  r.len = seqlens ? __ldg(seqlens + r.seq) : (k1 - k0);
  r.pos = r.len - (q1 - q0) + (row - q0);
  r.ok = true;
  if (k0 % BLK != 0) {
    raise_status(status, HISA_ERR_UNALIGNED);
    r.ok = false;
  } else if (r.len < 0 || r.len > k1 - k0 || row < q0 || row >= q1 || r.pos < 0 ||
             r.pos >= r.len) {
    raise_status(status, HISA_ERR_INVALID_ARG);
    r.ok = false;
  }
  return r;
}

// Block budget of sequence s: m_seq[s] when a per-sequence array is given, else m_max.
// A value outside [1, m_max] is clamped into it and raises HISA_ERR_INVALID_ARG (when
// `status` is not null).
__device__ __forceinline__ int seq_budget(const int32_t *m_seq, int s, int m_max, int *status) {
  if (!m_seq) return m_max;
  const int v = __ldg(m_seq + s);
  if (v < 1 || v > m_max) {
    raise_status(status, HISA_ERR_INVALID_ARG);
    return v < 1 ? 1 : m_max;
  }
  return v;
}

// ---------------------------------------------------------------------------
// block-wide exclusive scan of one value per thread (NT threads, NT % 32 == 0).
// `warp_tot` must hold NT/32 + 1 ints of shared memory. Returns the exclusive
// prefix; *total receives the sum over the block. Contains __syncthreads().

template <int NT>
__device__ __forceinline__ int block_exclusive_scan(int v, int *warp_tot, int *total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_tot[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int t = lane < NT / 32 ? warp_tot[lane] : 0;
    int s = t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    if (lane < NT / 32) warp_tot[lane] = s - t;
    if (lane == 31) warp_tot[NT / 32] = s;
  }
  __syncthreads();
  int excl = warp_tot[warp] + x - v;
  *total = warp_tot[NT / 32];
  __syncthreads();
  return excl;
}

// Launch `func` as a programmatic dependent of the previous kernel on `st` (its
// launch may overlap that kernel's tail; the kernel itself must execute
// griddepcontrol.wait before touching memory).  On the legacy default stream the
// launch is an ordinary one.
template <typename... Args>
inline cudaError_t launch_pdl(const void *func, dim3 grid, dim3 block, size_t smem,
                              cudaStream_t st, Args... args) {
  void *argv[] = {(void *)&args...};
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  const bool legacy = st == nullptr || st == cudaStreamLegacy || st == cudaStreamPerThread;
  cfg.attrs = legacy ? nullptr : attr;
  cfg.numAttrs = legacy ? 0 : 1;
  return cudaLaunchKernelExC(&cfg, func, argv);
}

// Raise a kernel's dynamic shared-memory limit once per device; later calls (for
// example while a CUDA graph is being captured) find it already set.
// cache: one word per device (64), static storage; atomic so that host threads calling
// the library at the same time do not race on it (both may set the attribute, harmlessly).
inline cudaError_t set_smem_once(const void *func, size_t bytes, std::atomic<int> *cache) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
  if (cache[dev].load(std::memory_order_relaxed) >= (int)bytes) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e == cudaSuccess) cache[dev].store((int)bytes, std::memory_order_relaxed);
  return e;
}

}  // namespace hisa
