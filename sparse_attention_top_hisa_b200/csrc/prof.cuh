// Launch accounting for the library's kernels: a launch counter per kernel kind
// and, when enabled, a CUDA event pair recorded on the launch stream around each
// launch (read back by hisa_timing_collect).
#pragma once

#include <cuda_runtime.h>

namespace hisa {

enum KernelKind {
  K_POOL = 0,
  K_APPEND,
  K_BLOCK_SELECT,
  K_TOKEN_FUSED,
  K_TOKEN_SCORE_SPLIT,
  K_TOKEN_SELECT_SCRATCH,
  K_KEY_NORM,
  K_DSA_FILTER,
  K_DSA_SELECT,
  K_DSA_FALLBACK,
  K_INV_LISTS,
  K_INV_SCAN,
  K_TOKEN_SCORE_TC,
  K_REPS_SPLIT,
  K_BLOCK_SCORE_TC,
  K_DECODE_SELECT,
  K_SPARSE_ATTENTION,
  K_EXPAND_BLOCKS,
  K_FRACTION_BUDGET,
  K_NUM_KINDS
};

void prof_before(int kind, cudaStream_t st);
void prof_after(int kind, cudaStream_t st);

struct ProfScope {
  int kind;
  cudaStream_t st;
  ProfScope(int k, cudaStream_t s) : kind(k), st(s) { prof_before(kind, st); }
  ~ProfScope() { prof_after(kind, st); }
};

}  // namespace hisa
