// Block pooling (hisa_pool_blocks) and decode-time append (hisa_append_keys).
//
// HISA summary page (aitrends.kr), paragraph on block partition and mean pooling:
// each block of B = 128 consecutive keys is represented by the mean of its keys.
// Paragraph on KV-cache maintenance: the representatives are refreshed when keys
// are appended.  Both kernels pool with the same warp routine (keys summed in
// increasing row order in fp32, then one correctly rounded division by the count),
// so incrementally maintained representatives equal a fresh pool bit for bit.
#include "common.cuh"
#include "prof.cuh"

namespace hisa {

// One warp pools one block: lane l owns dims 2l and 2l+1 (one 32-bit word per row).
// Plain (coherent) loads: the append kernel reads rows written earlier in the same CTA.
__device__ __forceinline__ void pool_block_warp(const uint32_t *rows, int count, float *rep) {
  const int lane = threadIdx.x & 31;
  float a = 0.f, b = 0.f;
  int t = 0;
  for (; t + 8 <= count; t += 8) {
    uint32_t w[8];
#pragma unroll
    for (int u = 0; u < 8; u++) w[u] = rows[(t + u) * 32 + lane];
#pragma unroll
    for (int u = 0; u < 8; u++) {
      a += bf_lo(w[u]);
      b += bf_hi(w[u]);
    }
  }
  for (; t < count; t++) {
    uint32_t w = rows[t * 32 + lane];
    a += bf_lo(w);
    b += bf_hi(w);
  }
  const float cnt = (float)count;
  float2 r = make_float2(__fdiv_rn(a, cnt), __fdiv_rn(b, cnt));
  reinterpret_cast<float2 *>(rep)[lane] = r;
}

constexpr int POOL_WARPS = 4;

__global__ void __launch_bounds__(POOL_WARPS * 32)
pool_blocks_kernel(const uint16_t *__restrict__ k, const int32_t *__restrict__ cu_k,
                   const int32_t *__restrict__ seqlens, float *__restrict__ reps, int *status) {
  const int s = blockIdx.y;
  const int b = blockIdx.x * POOL_WARPS + (threadIdx.x >> 5);
  const int start = cu_k[s], cap = cu_k[s + 1] - start;
  const int len = seqlens ? seqlens[s] : cap;
  if (start % BLK != 0) {
    if (blockIdx.x == 0 && threadIdx.x == 0) raise_status(status, HISA_ERR_UNALIGNED);
    return;
  }
  if (len < 0 || len > cap) {
    if (blockIdx.x == 0 && threadIdx.x == 0) raise_status(status, HISA_ERR_INVALID_ARG);
    return;
  }
  if (b * BLK >= len) return;
  const int count = min(BLK, len - b * BLK);
  const int row0 = start + b * BLK;
  pool_block_warp(reinterpret_cast<const uint32_t *>(k + (size_t)row0 * D), count,
                  reps + (size_t)(row0 / BLK) * D);
}

// Append: one CTA per sequence.  The block that receives the new rows is staged in
// shared memory by all threads at once (one memory round trip), then summed row by
// row in increasing order exactly like pool_block_warp, so the result is
// bit-identical to pooling the grown block from scratch.
constexpr int APPEND_THREADS = 256;

__global__ void __launch_bounds__(APPEND_THREADS)
append_keys_kernel(uint16_t *__restrict__ kc, float *__restrict__ reps,
                   const int32_t *__restrict__ cu_k, int32_t *__restrict__ seqlens,
                   const uint16_t *__restrict__ new_keys, int n_new, int *status) {
  __shared__ __align__(16) uint4 blockrows[BLK * 8];
  // programmatic dependent launch (see launch_append): wait for the previous kernel
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int s = blockIdx.x, tid = threadIdx.x;
  const int start = cu_k[s], cap = cu_k[s + 1] - start;
  const int len = seqlens[s];
  if (start % BLK != 0) {
    if (tid == 0) raise_status(status, HISA_ERR_UNALIGNED);
    return;
  }
  if (len < 0 || len > cap) {
    if (tid == 0) raise_status(status, HISA_ERR_INVALID_ARG);
    return;
  }
  if (len + n_new > cap) {
    if (tid == 0) raise_status(status, HISA_ERR_CAPACITY);
    return;
  }
  const uint4 *src = reinterpret_cast<const uint4 *>(new_keys + (size_t)s * n_new * D);
  uint4 *rows = reinterpret_cast<uint4 *>(kc + (size_t)start * D);
  const int nlen = len + n_new;
  // copy the new rows to the cache
  for (int i = tid; i < n_new * 8; i += APPEND_THREADS) rows[(size_t)len * 8 + i] = src[i];
  // re-pool every touched block from shared memory
  const int first = len / BLK, last = (nlen - 1) / BLK;
  for (int b = first; b <= last; b++) {
    const int count = min(BLK, nlen - b * BLK);
    for (int i = tid; i < count * 8; i += APPEND_THREADS) {
      const int r = b * BLK + (i >> 3);  // row within the sequence
      blockrows[i] = r < len ? rows[(size_t)r * 8 + (i & 7)]
                             : src[(size_t)(r - len) * 8 + (i & 7)];
    }
    __syncthreads();
    if (tid < 32) {
      const uint32_t *w = reinterpret_cast<const uint32_t *>(blockrows);
      float a = 0.f, c = 0.f;
      for (int t = 0; t < count; t++) {
        const uint32_t x = w[t * 32 + tid];
        a += bf_lo(x);
        c += bf_hi(x);
      }
      const float cnt = (float)count;
      reinterpret_cast<float2 *>(reps + (size_t)(start / BLK + b) * D)[tid] =
          make_float2(__fdiv_rn(a, cnt), __fdiv_rn(c, cnt));
    }
    __syncthreads();
  }
  if (tid == 0) seqlens[s] = nlen;
}

cudaError_t launch_pool(const uint16_t *k, const int32_t *cu_k, const int32_t *seqlens,
                        int num_seqs, int max_seqlen_k, float *reps, int *status,
                        cudaStream_t st) {
  const int nblk = (max_seqlen_k + BLK - 1) / BLK;
  if (nblk == 0 || num_seqs == 0) return cudaSuccess;
  dim3 grid((nblk + POOL_WARPS - 1) / POOL_WARPS, num_seqs);
  {
    ProfScope ps(K_POOL, st);
    pool_blocks_kernel<<<grid, POOL_WARPS * 32, 0, st>>>(k, cu_k, seqlens, reps, status);
  }
  return cudaGetLastError();
}

cudaError_t launch_append(uint16_t *kc, float *reps, const int32_t *cu_k, int32_t *seqlens,
                          const uint16_t *new_keys, int n_new, int num_seqs, int *status,
                          cudaStream_t st) {
  if (num_seqs == 0 || n_new == 0) return cudaSuccess;
  cudaError_t e;
  {
    ProfScope ps(K_APPEND, st);
    e = launch_pdl((const void *)append_keys_kernel, dim3(num_seqs), dim3(APPEND_THREADS), 0, st,
                   kc, reps, cu_k, seqlens, new_keys, n_new, status);
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace hisa
