// C ABI of the HISA indexer library: argument validation, workspace carving and
// kernel launches.  Declarations and the contract of every entry point are in
// include/hisa.h.
#include <cuda_runtime.h>
#include <stdint.h>

#include <vector>

#include "common.cuh"
#include "prof.cuh"

namespace hisa {
cudaError_t launch_pool(const uint16_t *k, const int32_t *cu_k, const int32_t *seqlens,
                        int num_seqs, int max_seqlen_k, float *reps, int *status,
                        cudaStream_t st);
cudaError_t launch_append(uint16_t *kc, float *reps, const int32_t *cu_k, int32_t *seqlens,
                          const uint16_t *new_keys, int n_new, int num_seqs, int *status,
                          cudaStream_t st);
cudaError_t launch_block_select(const uint16_t *q, const float *reps, const int32_t *cu_q,
                                const int32_t *cu_k, const int32_t *seqlens,
                                const int32_t *m_seq, int S, int total_q, int max_seqlen_k,
                                int m, int32_t *blk, int32_t *out_blocks, uint8_t *ws,
                                int num_sms, int *status, cudaStream_t st);
cudaError_t launch_token_select(const uint16_t *q, const uint16_t *k, const int32_t *cu_q,
                                const int32_t *cu_k, const int32_t *seqlens,
                                const int32_t *m_seq, int S, int total_q, int max_seqlen_k,
                                int m, int topk, const int32_t *blk, uint8_t *ws, int num_sms,
                                int32_t *out_idx, float *out_scores, int *status,
                                cudaStream_t st);
size_t block_tc_workspace_bytes(int total_q, int num_seqs, int max_seqlen_k);
cudaError_t launch_expand_blocks(const int32_t *blk, const int32_t *cu_q, const int32_t *cu_k,
                                 const int32_t *seqlens, int S, int total_q, int m,
                                 int32_t *out, cudaStream_t st);
cudaError_t launch_fraction_budget(const int32_t *cu_k, const int32_t *seqlens, int S, double f,
                                   int m_max, int32_t *m_seq, int *status, cudaStream_t st);
extern std::atomic<int> g_test_no_loads;
size_t token_scratch_bytes(int total_q, int num_seqs, int max_seqlen_k, int m, int num_sms);
cudaError_t launch_dsa(const uint16_t *q, const uint16_t *k, const int32_t *cu_q,
                       const int32_t *cu_k, const int32_t *seqlens, int S, int total_q,
                       int max_seqlen_k, int topk, int32_t *out_idx, float *out_scores,
                       uint8_t *ws, int *status, cudaStream_t st);
size_t dsa_workspace_bytes(int total_q, int num_seqs, int max_seqlen_k, int topk);
bool use_tc_path(int total_q, int num_sms);
bool decode_path_fits(int max_seqlen_k, int m);
cudaError_t launch_sparse_attention(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                                    const int32_t *idx, const int32_t *cu_q, const int32_t *cu_k,
                                    int S, int total_q, int H, int topk, float scale, float *out,
                                    float *lse, int num_sms, int *status, cudaStream_t st);
cudaError_t launch_decode_select(const uint16_t *q, const uint16_t *k, const float *reps,
                                 const int32_t *cu_q, const int32_t *cu_k,
                                 const int32_t *seqlens, const int32_t *m_seq, int S,
                                 int total_q, int max_seqlen_k, int m, int topk,
                                 int32_t *out_idx, float *out_scores, int32_t *out_blocks,
                                 int *status, cudaStream_t st, uint16_t *append_kc = nullptr,
                                 float *append_reps = nullptr, int32_t *append_seqlens = nullptr,
                                 const uint16_t *new_keys = nullptr);
}  // namespace hisa

using namespace hisa;

// ---------------------------------------------------------------------------
// launch accounting (see prof.cuh): the launch counters are atomic; the event timing
// state is host-side and not thread-safe

namespace {
const char *kKindNames[K_NUM_KINDS] = {
    "pool_blocks",        "append_keys",         "block_select",   "token_fused",
    "token_score_split",  "token_select_scratch", "key_norm",      "dsa_filter",
    "dsa_select",         "dsa_fallback",         "inv_lists",      "inv_scan",
    "token_score_tc",     "reps_split",          "block_score_tc",  "decode_select",  "sparse_attention",
    "expand_blocks",      "fraction_budget"};
std::atomic<long long> g_launches[K_NUM_KINDS];
double g_ms[K_NUM_KINDS];
long long g_timed[K_NUM_KINDS];
bool g_timing = false;
struct Pending {
  int kind;
  cudaEvent_t a, b;
};
std::vector<Pending> g_pending;
std::vector<cudaEvent_t> g_free_events;
Pending g_open{-1, nullptr, nullptr};

cudaEvent_t take_event() {
  if (!g_free_events.empty()) {
    cudaEvent_t e = g_free_events.back();
    g_free_events.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}
}  // namespace

namespace hisa {
void prof_before(int kind, cudaStream_t st) {
  if (kind >= 0 && kind < K_NUM_KINDS) g_launches[kind].fetch_add(1, std::memory_order_relaxed);
  if (!g_timing) return;
  g_open.kind = kind;
  g_open.a = take_event();
  g_open.b = take_event();
  if (g_open.a) cudaEventRecord(g_open.a, st);
}
void prof_after(int kind, cudaStream_t st) {
  if (!g_timing || g_open.kind != kind || !g_open.a || !g_open.b) return;
  cudaEventRecord(g_open.b, st);
  g_pending.push_back(g_open);
  g_open.kind = -1;
}
}  // namespace hisa

// Sticky device status word (one per device that loads the library).
static __device__ int g_hisa_status;

// Scratch of hisa_select_noalloc (see there).  Every device that loads the library
// holds this array until the process exits.
static __device__ __align__(256) unsigned char g_noalloc_scratch[HISA_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
// Per-device values looked up once; atomic so that host threads calling the library at
// the same time do not race (both may look the value up, harmlessly).
std::atomic<int *> g_status_ptr[kMaxDevices];
std::atomic<uint8_t *> g_noalloc_ptr[kMaxDevices];
std::atomic<int> g_num_sms[kMaxDevices];

int current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return -1;
  return dev;
}

// Device addresses of the library's two device arrays on the current device, looked
// up together by the first call of any entry point on that device (host code only has
// host-side stand-ins for the symbols).  The scratch address is stored before the
// status address, so a status address seen by another thread implies both.
bool resolve_device_symbols(int dev) {
  if (g_status_ptr[dev].load(std::memory_order_acquire)) return true;
  void *ps = nullptr, *pn = nullptr;
  if (cudaGetSymbolAddress(&ps, g_hisa_status) != cudaSuccess || !ps) return false;
  if (cudaGetSymbolAddress(&pn, g_noalloc_scratch) != cudaSuccess || !pn) return false;
  g_noalloc_ptr[dev].store(static_cast<uint8_t *>(pn), std::memory_order_relaxed);
  g_status_ptr[dev].store(static_cast<int *>(ps), std::memory_order_release);
  return true;
}

// Device address of the status word on the current device.
int *status_word() {
  const int dev = current_device();
  if (dev < 0 || !resolve_device_symbols(dev)) return nullptr;
  return g_status_ptr[dev].load(std::memory_order_acquire);
}

// Device address of hisa_select_noalloc's scratch array on the current device.
uint8_t *noalloc_scratch() {
  const int dev = current_device();
  if (dev < 0 || !resolve_device_symbols(dev)) return nullptr;
  return g_noalloc_ptr[dev].load(std::memory_order_relaxed);
}

int num_sms() {
  const int dev = current_device();
  if (dev < 0) return 148;
  int n = g_num_sms[dev].load(std::memory_order_relaxed);
  if (!n) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    g_num_sms[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

hisa_status from_cuda(cudaError_t e) { return e == cudaSuccess ? HISA_OK : HISA_ERR_CUDA; }

struct SelectPlan {
  size_t off_blk, off_scratch, total;
};

SelectPlan select_plan(int total_q, int num_seqs, int max_seqlen_k, int m) {
  SelectPlan p;
  size_t off = 0;
  p.off_blk = off;
  off = align256(off + (size_t)(total_q > 0 ? total_q : 1) * m * 4);
  p.off_scratch = off;
  off = align256(off + token_scratch_bytes(total_q, num_seqs, max_seqlen_k, m, num_sms()));
  p.total = off;
  return p;
}

}  // namespace

extern "C" {

const char *hisa_status_string(hisa_status s) {
  switch (s) {
    case HISA_OK: return "ok";
    case HISA_ERR_INVALID_ARG: return "invalid argument";
    case HISA_ERR_UNALIGNED: return "unaligned pointer or region start";
    case HISA_ERR_WORKSPACE: return "workspace missing or too small";
    case HISA_ERR_CUDA: return "CUDA runtime error";
    case HISA_ERR_TIMEOUT: return "device-side wait timed out";
    case HISA_ERR_NOT_IMPLEMENTED: return "not implemented";
    case HISA_ERR_CAPACITY: return "key region capacity exceeded";
  }
  return "unknown status";
}

int hisa_version(void) { return 100; }

hisa_status hisa_pool_blocks(const hisa_bf16 *k_idx, const int32_t *cu_seqlens_k,
                             const int32_t *seqlens_k, int num_seqs, int max_seqlen_k, int B,
                             float *reps, hisa_stream_t stream) {
  if (B != HISA_BLOCK || num_seqs < 0 || max_seqlen_k < 0) return HISA_ERR_INVALID_ARG;
  if (num_seqs == 0 || max_seqlen_k == 0) return HISA_OK;
  if (!k_idx || !cu_seqlens_k || !reps) return HISA_ERR_INVALID_ARG;
  if (!aligned(k_idx, 16) || !aligned(reps, 16) || !aligned(cu_seqlens_k, 4) ||
      !aligned(seqlens_k, 4))
    return HISA_ERR_UNALIGNED;
  int *st = status_word();
  if (!st) return HISA_ERR_CUDA;
  return from_cuda(launch_pool(k_idx, cu_seqlens_k, seqlens_k, num_seqs, max_seqlen_k, reps, st,
                               static_cast<cudaStream_t>(stream)));
}

hisa_status hisa_append_keys(hisa_bf16 *k_cache, float *reps, const int32_t *cu_seqlens_k,
                             int32_t *seqlens_k, const hisa_bf16 *new_keys, int n_new,
                             int num_seqs, int B, hisa_stream_t stream) {
  if (B != HISA_BLOCK || num_seqs < 0 || n_new < 0) return HISA_ERR_INVALID_ARG;
  if (num_seqs == 0 || n_new == 0) return HISA_OK;
  if (!k_cache || !reps || !cu_seqlens_k || !seqlens_k || !new_keys) return HISA_ERR_INVALID_ARG;
  if (!aligned(k_cache, 16) || !aligned(reps, 16) || !aligned(new_keys, 16) ||
      !aligned(cu_seqlens_k, 4) || !aligned(seqlens_k, 4))
    return HISA_ERR_UNALIGNED;
  int *st = status_word();
  if (!st) return HISA_ERR_CUDA;
  return from_cuda(launch_append(k_cache, reps, cu_seqlens_k, seqlens_k, new_keys, n_new,
                                 num_seqs, st, static_cast<cudaStream_t>(stream)));
}

size_t hisa_select_workspace_size(int total_q, int num_seqs, int max_seqlen_k, int B, int m,
                                  int k) {
  (void)B;
  (void)k;
  if (total_q < 0 || m < 1 || num_seqs < 0 || max_seqlen_k < 0) return 0;
  return select_plan(total_q, num_seqs, max_seqlen_k, m).total;
}

}  // extern "C"

namespace {

// Host-side checks shared by the selection entry points (nothing is launched when
// they fail).
hisa_status select_args(const hisa_bf16 *q_idx, const hisa_bf16 *k_idx, const float *reps,
                        const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k,
                        const int32_t *seqlens_k, const int32_t *m_seq, int num_seqs,
                        int total_q, int max_seqlen_k, int B, int m, int k, int32_t *out_idx,
                        float *out_scores, int32_t *out_blocks) {
  if (B != HISA_BLOCK || m < 1 || m > HISA_MAX_M || k < 1 || k > HISA_MAX_TOPK)
    return HISA_ERR_INVALID_ARG;
  if (num_seqs < 0 || total_q < 0 || max_seqlen_k < 0) return HISA_ERR_INVALID_ARG;
  if (total_q == 0) return HISA_OK;
  if (num_seqs == 0) return HISA_ERR_INVALID_ARG;
  if (!q_idx || !k_idx || !reps || !cu_seqlens_q || !cu_seqlens_k || !out_idx)
    return HISA_ERR_INVALID_ARG;
  if (!aligned(q_idx, 16) || !aligned(k_idx, 16) || !aligned(reps, 16) ||
      !aligned(cu_seqlens_q, 4) || !aligned(cu_seqlens_k, 4) || !aligned(seqlens_k, 4) ||
      !aligned(m_seq, 4) || !aligned(out_idx, 4) || !aligned(out_scores, 4) ||
      !aligned(out_blocks, 4))
    return HISA_ERR_UNALIGNED;
  // list entries hold row << 7 | slot (m <= 128) or row << 9 | slot, and list positions
  // (rows rounded up to a whole chunk, times m) are int32
  if (total_q >= (m > 128 ? (1 << 23) : (1 << 25))) return HISA_ERR_INVALID_ARG;
  if ((long long)(total_q + 65536) * m >= (1ll << 31)) return HISA_ERR_INVALID_ARG;
  return HISA_OK;
}

// Launches a selection whose arguments passed select_args.  w: the workspace (or the
// no-allocation scratch), p its plan; nullptr when the few-query cluster path, which
// needs none, is taken.
hisa_status select_launch(const hisa_bf16 *q_idx, const hisa_bf16 *k_idx, const float *reps,
                          const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k,
                          const int32_t *seqlens_k, const int32_t *m_seq, int num_seqs,
                          int total_q, int max_seqlen_k, int m, int k, int32_t *out_idx,
                          float *out_scores, int32_t *out_blocks, uint8_t *w,
                          const SelectPlan &p, int *st, cudaStream_t s) {
  if (!use_tc_path(total_q, num_sms()) && decode_path_fits(max_seqlen_k, m))
    return from_cuda(launch_decode_select(q_idx, k_idx, reps, cu_seqlens_q, cu_seqlens_k,
                                          seqlens_k, m_seq, num_seqs, total_q, max_seqlen_k, m,
                                          k, out_idx, out_scores, out_blocks, st, s));
  if (!w) return HISA_ERR_WORKSPACE;
  int32_t *blk = reinterpret_cast<int32_t *>(w + p.off_blk);
  cudaError_t e = launch_block_select(q_idx, reps, cu_seqlens_q, cu_seqlens_k, seqlens_k, m_seq,
                                      num_seqs, total_q, max_seqlen_k, m, blk, out_blocks,
                                      w + p.off_scratch, num_sms(), st, s);
  if (e != cudaSuccess) return HISA_ERR_CUDA;
  e = launch_token_select(q_idx, k_idx, cu_seqlens_q, cu_seqlens_k, seqlens_k, m_seq, num_seqs,
                          total_q, max_seqlen_k, m, k, blk, w + p.off_scratch, num_sms(),
                          out_idx, out_scores, st, s);
  return from_cuda(e);
}

hisa_status select_with_workspace(const hisa_bf16 *q_idx, const hisa_bf16 *k_idx,
                                  const float *reps, const int32_t *cu_seqlens_q,
                                  const int32_t *cu_seqlens_k, const int32_t *seqlens_k,
                                  const int32_t *m_seq, int num_seqs, int total_q,
                                  int max_seqlen_k, int B, int m, int k, int32_t *out_idx,
                                  float *out_scores, int32_t *out_blocks, void *ws,
                                  size_t ws_bytes, hisa_stream_t stream) {
  hisa_status rc = select_args(q_idx, k_idx, reps, cu_seqlens_q, cu_seqlens_k, seqlens_k, m_seq,
                               num_seqs, total_q, max_seqlen_k, B, m, k, out_idx, out_scores,
                               out_blocks);
  if (rc != HISA_OK || total_q == 0) return rc;
  const SelectPlan p = select_plan(total_q, num_seqs, max_seqlen_k, m);
  if (!ws || ws_bytes < p.total) return HISA_ERR_WORKSPACE;
  if (!aligned(ws, 256)) return HISA_ERR_UNALIGNED;
  int *st = status_word();
  if (!st) return HISA_ERR_CUDA;
  return select_launch(q_idx, k_idx, reps, cu_seqlens_q, cu_seqlens_k, seqlens_k, m_seq,
                       num_seqs, total_q, max_seqlen_k, m, k, out_idx, out_scores, out_blocks,
                       static_cast<uint8_t *>(ws), p, st, static_cast<cudaStream_t>(stream));
}

}  // namespace

extern "C" {

hisa_status hisa_select(const hisa_bf16 *q_idx, const hisa_bf16 *k_idx, const float *reps,
                        const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k,
                        const int32_t *seqlens_k, int num_seqs, int total_q, int max_seqlen_k,
                        int B, int m, int k, int32_t *out_idx, float *out_scores,
                        int32_t *out_blocks, void *ws, size_t ws_bytes, hisa_stream_t stream) {
  return select_with_workspace(q_idx, k_idx, reps, cu_seqlens_q, cu_seqlens_k, seqlens_k,
                               nullptr, num_seqs, total_q, max_seqlen_k, B, m, k, out_idx,
                               out_scores, out_blocks, ws, ws_bytes, stream);
}

hisa_status hisa_select_varm(const hisa_bf16 *q_idx, const hisa_bf16 *k_idx, const float *reps,
                             const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k,
                             const int32_t *seqlens_k, const int32_t *m_seq, int num_seqs,
                             int total_q, int max_seqlen_k, int B, int m_max, int k,
                             int32_t *out_idx, float *out_scores, int32_t *out_blocks, void *ws,
                             size_t ws_bytes, hisa_stream_t stream) {
  if (!m_seq && total_q > 0) return HISA_ERR_INVALID_ARG;
  return select_with_workspace(q_idx, k_idx, reps, cu_seqlens_q, cu_seqlens_k, seqlens_k, m_seq,
                               num_seqs, total_q, max_seqlen_k, B, m_max, k, out_idx,
                               out_scores, out_blocks, ws, ws_bytes, stream);
}

hisa_status hisa_decode_step(hisa_bf16 *k_cache, float *reps, const int32_t *cu_seqlens_k,
                             int32_t *seqlens_k, const hisa_bf16 *new_keys,
                             const hisa_bf16 *q_idx, int num_seqs, int max_seqlen_k, int B, int m,
                             int k, int32_t *out_idx, float *out_scores, int32_t *out_blocks,
                             hisa_stream_t stream) {
  if (B != HISA_BLOCK || m < 1 || m > HISA_MAX_M || k < 1 || k > HISA_MAX_TOPK ||
      num_seqs < 0 || max_seqlen_k < 0)
    return HISA_ERR_INVALID_ARG;
  if (num_seqs == 0) return HISA_OK;
  if (!k_cache || !reps || !cu_seqlens_k || !seqlens_k || !new_keys || !q_idx || !out_idx)
    return HISA_ERR_INVALID_ARG;
  if (!aligned(k_cache, 16) || !aligned(reps, 16) || !aligned(new_keys, 16) ||
      !aligned(q_idx, 16) || !aligned(cu_seqlens_k, 4) || !aligned(seqlens_k, 4) ||
      !aligned(out_idx, 4) || !aligned(out_scores, 4) || !aligned(out_blocks, 4))
    return HISA_ERR_UNALIGNED;
  if (!decode_path_fits(max_seqlen_k, m)) return HISA_ERR_NOT_IMPLEMENTED;
  int *st = status_word();
  if (!st) return HISA_ERR_CUDA;
  return from_cuda(launch_decode_select(q_idx, k_cache, reps, nullptr, cu_seqlens_k, seqlens_k,
                                        nullptr, num_seqs, num_seqs, max_seqlen_k, m, k, out_idx,
                                        out_scores, out_blocks, st,
                                        static_cast<cudaStream_t>(stream), k_cache, reps,
                                        seqlens_k, new_keys));
}

hisa_status hisa_fraction_blocks(const int32_t *cu_seqlens_k, const int32_t *seqlens_k,
                                 int num_seqs, int B, double f, int m_max, int32_t *m_seq,
                                 hisa_stream_t stream) {
  if (B != HISA_BLOCK || num_seqs < 0 || m_max < 1 || m_max > HISA_MAX_M || !(f > 0.0) ||
      !(f <= 1.0))
    return HISA_ERR_INVALID_ARG;
  if (num_seqs == 0) return HISA_OK;
  if (!cu_seqlens_k || !m_seq) return HISA_ERR_INVALID_ARG;
  if (!aligned(cu_seqlens_k, 4) || !aligned(seqlens_k, 4) || !aligned(m_seq, 4))
    return HISA_ERR_UNALIGNED;
  int *st = status_word();
  if (!st) return HISA_ERR_CUDA;
  return from_cuda(launch_fraction_budget(cu_seqlens_k, seqlens_k, num_seqs, f, m_max, m_seq, st,
                                          static_cast<cudaStream_t>(stream)));
}

size_t hisa_block_sparse_workspace_size(int total_q, int num_seqs, int max_seqlen_k, int B,
                                        int m) {
  (void)B;
  if (total_q < 0 || m < 1 || num_seqs < 0 || max_seqlen_k < 0) return 0;
  size_t off = align256((size_t)(total_q > 0 ? total_q : 1) * m * 4);
  if (use_tc_path(total_q, num_sms()))
    off = align256(off + block_tc_workspace_bytes(total_q, num_seqs, max_seqlen_k));
  return off;
}

hisa_status hisa_block_sparse_select(const hisa_bf16 *q_idx, const float *reps,
                                     const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k,
                                     const int32_t *seqlens_k, int num_seqs, int total_q,
                                     int max_seqlen_k, int B, int m, int32_t *out_idx,
                                     int32_t *out_blocks, void *ws, size_t ws_bytes,
                                     hisa_stream_t stream) {
  if (B != HISA_BLOCK || m < 1 || m > HISA_MAX_M || num_seqs < 0 || total_q < 0 ||
      max_seqlen_k < 0)
    return HISA_ERR_INVALID_ARG;
  if (total_q == 0) return HISA_OK;
  if (num_seqs == 0 || total_q >= (1 << 25)) return HISA_ERR_INVALID_ARG;
  if (!q_idx || !reps || !cu_seqlens_q || !cu_seqlens_k || !out_idx) return HISA_ERR_INVALID_ARG;
  if (!aligned(q_idx, 16) || !aligned(reps, 16) || !aligned(cu_seqlens_q, 4) ||
      !aligned(cu_seqlens_k, 4) || !aligned(seqlens_k, 4) || !aligned(out_idx, 4) ||
      !aligned(out_blocks, 4))
    return HISA_ERR_UNALIGNED;
  const size_t need = hisa_block_sparse_workspace_size(total_q, num_seqs, max_seqlen_k, B, m);
  if (!ws || ws_bytes < need) return HISA_ERR_WORKSPACE;
  if (!aligned(ws, 256)) return HISA_ERR_UNALIGNED;
  int *st = status_word();
  if (!st) return HISA_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t *w = static_cast<uint8_t *>(ws);
  int32_t *blk = reinterpret_cast<int32_t *>(w);
  cudaError_t e = launch_block_select(q_idx, reps, cu_seqlens_q, cu_seqlens_k, seqlens_k, nullptr,
                                      num_seqs, total_q, max_seqlen_k, m, blk, out_blocks,
                                      w + align256((size_t)total_q * m * 4), num_sms(), st, s);
  if (e != cudaSuccess) return HISA_ERR_CUDA;
  return from_cuda(launch_expand_blocks(blk, cu_seqlens_q, cu_seqlens_k, seqlens_k, num_seqs,
                                        total_q, m, out_idx, s));
}

size_t dsa_flat_workspace_size(int total_q, int num_seqs, int max_seqlen_k, int k) {
  if (total_q < 0 || num_seqs < 0 || max_seqlen_k < 0 || k < 1) return 0;
  return dsa_workspace_bytes(total_q, num_seqs, max_seqlen_k, k);
}

hisa_status dsa_flat_select(const hisa_bf16 *q_idx, const hisa_bf16 *k_idx,
                            const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k,
                            const int32_t *seqlens_k, int num_seqs, int total_q,
                            int max_seqlen_k, int k, int32_t *out_idx, float *out_scores,
                            void *ws, size_t ws_bytes, hisa_stream_t stream) {
  if (k < 1 || k > HISA_MAX_TOPK || num_seqs < 0 || total_q < 0 || max_seqlen_k < 0)
    return HISA_ERR_INVALID_ARG;
  if (total_q == 0) return HISA_OK;
  if (num_seqs == 0) return HISA_ERR_INVALID_ARG;
  if (!q_idx || !k_idx || !cu_seqlens_q || !cu_seqlens_k || !out_idx) return HISA_ERR_INVALID_ARG;
  if (!aligned(q_idx, 16) || !aligned(k_idx, 16) || !aligned(cu_seqlens_q, 4) ||
      !aligned(cu_seqlens_k, 4) || !aligned(seqlens_k, 4) || !aligned(out_idx, 4) ||
      !aligned(out_scores, 4))
    return HISA_ERR_UNALIGNED;
  const size_t need = dsa_workspace_bytes(total_q, num_seqs, max_seqlen_k, k);
  if (!ws || ws_bytes < need) return HISA_ERR_WORKSPACE;
  if (!aligned(ws, 256)) return HISA_ERR_UNALIGNED;
  int *st = status_word();
  if (!st) return HISA_ERR_CUDA;
  return from_cuda(launch_dsa(q_idx, k_idx, cu_seqlens_q, cu_seqlens_k, seqlens_k, num_seqs,
                              total_q, max_seqlen_k, k, out_idx, out_scores,
                              static_cast<uint8_t *>(ws), st, static_cast<cudaStream_t>(stream)));
}

hisa_status hisa_sparse_attention(const hisa_bf16 *q_att, const hisa_bf16 *k_att,
                                  const hisa_bf16 *v_att, const int32_t *topk_idx,
                                  const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k,
                                  int num_seqs, int total_q, int num_heads, int k, float scale,
                                  float *out, float *lse, hisa_stream_t stream) {
  if (num_heads < 1 || num_heads > HISA_ATT_MAX_HEADS || k < 1 || num_seqs < 0 || total_q < 0 ||
      !(scale == scale))
    return HISA_ERR_INVALID_ARG;
  if (total_q == 0) return HISA_OK;
  if (num_seqs == 0 || total_q >= (1 << 25)) return HISA_ERR_INVALID_ARG;
  if (!q_att || !k_att || !v_att || !topk_idx || !cu_seqlens_q || !cu_seqlens_k || !out)
    return HISA_ERR_INVALID_ARG;
  if (!aligned(q_att, 16) || !aligned(k_att, 16) || !aligned(v_att, 16) ||
      !aligned(topk_idx, 4) || !aligned(cu_seqlens_q, 4) || !aligned(cu_seqlens_k, 4) ||
      !aligned(out, 4) || !aligned(lse, 4))
    return HISA_ERR_UNALIGNED;
  int *st = status_word();
  if (!st) return HISA_ERR_CUDA;
  return from_cuda(launch_sparse_attention(q_att, k_att, v_att, topk_idx, cu_seqlens_q,
                                           cu_seqlens_k, num_seqs, total_q, num_heads, k, scale,
                                           out, lse, num_sms(), st,
                                           static_cast<cudaStream_t>(stream)));
}

hisa_status hisa_timing_enable(int on) {
  g_timing = on != 0;
  return HISA_OK;
}

int hisa_kernel_kinds(void) { return K_NUM_KINDS; }

const char *hisa_kernel_name(int kind) {
  return (kind >= 0 && kind < K_NUM_KINDS) ? kKindNames[kind] : "";
}

hisa_status hisa_timing_collect(double *ms, long long *launches, long long *timed, int n,
                                int reset) {
  hisa_status rc = HISA_OK;
  for (const Pending &p : g_pending) {
    float t = 0.f;
    if (cudaEventSynchronize(p.b) != cudaSuccess || cudaEventElapsedTime(&t, p.a, p.b) != cudaSuccess) {
      rc = HISA_ERR_CUDA;
    } else if (p.kind >= 0 && p.kind < K_NUM_KINDS) {
      g_ms[p.kind] += t;
      g_timed[p.kind]++;
    }
    g_free_events.push_back(p.a);
    g_free_events.push_back(p.b);
  }
  g_pending.clear();
  for (int i = 0; i < n && i < K_NUM_KINDS; i++) {
    if (ms) ms[i] = g_ms[i];
    if (launches) launches[i] = g_launches[i].load(std::memory_order_relaxed);
    if (timed) timed[i] = g_timed[i];
  }
  if (reset) {
    for (int i = 0; i < K_NUM_KINDS; i++) {
      g_ms[i] = 0.0;
      g_launches[i].store(0, std::memory_order_relaxed);
      g_timed[i] = 0;
    }
  }
  return rc;
}

hisa_status hisa_test_fault(int mode) {
  if (mode != 0 && mode != 1) return HISA_ERR_INVALID_ARG;
  g_test_no_loads.store(mode, std::memory_order_relaxed);
  return HISA_OK;
}

hisa_status hisa_device_status(int32_t *status, int clear, hisa_stream_t stream) {
  if (!status) return HISA_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return HISA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_hisa_status, sizeof(int)) != cudaSuccess) return HISA_ERR_CUDA;
  *status = v;
  if (clear) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_hisa_status, &zero, sizeof(int)) != cudaSuccess) return HISA_ERR_CUDA;
  }
  return HISA_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// hisa_select_noalloc: hisa_select for callers that cannot allocate device memory
// when they need a selection (for example a plug-in inside an inference engine
// whose memory plan is fixed before it runs, or a latency-critical path where a
// cudaMalloc would synchronise the device).  Its scratch is a fixed array inside
// this library instead of a caller workspace.

extern "C" hisa_status hisa_select_noalloc(const hisa_bf16 *q_idx, const hisa_bf16 *k_idx,
                                           const float *reps, const int32_t *cu_seqlens_q,
                                           const int32_t *cu_seqlens_k, const int32_t *seqlens_k,
                                           int num_seqs, int total_q, int max_seqlen_k, int B,
                                           int m, int k, int32_t *out_idx, float *out_scores,
                                           int32_t *out_blocks, hisa_stream_t stream) {
  hisa_status rc = select_args(q_idx, k_idx, reps, cu_seqlens_q, cu_seqlens_k, seqlens_k, nullptr,
                               num_seqs, total_q, max_seqlen_k, B, m, k, out_idx, out_scores,
                               out_blocks);
  if (rc != HISA_OK || total_q == 0) return rc;
  int *st = status_word();
  if (!st) return HISA_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // few queries (up to 8192 blocks per sequence): the cluster kernel, which needs no
  // scratch at all (as in hisa_select)
  const SelectPlan p = select_plan(total_q, num_seqs, max_seqlen_k, m);
  if (!use_tc_path(total_q, num_sms()) && decode_path_fits(max_seqlen_k, m))
    return select_launch(q_idx, k_idx, reps, cu_seqlens_q, cu_seqlens_k, seqlens_k, nullptr,
                         num_seqs, total_q, max_seqlen_k, m, k, out_idx, out_scores, out_blocks,
                         nullptr, p, st, s);
  // the same scratch layout hisa_select carves from its workspace must fit the array
  if (p.total > (size_t)HISA_NOALLOC_SCRATCH_BYTES) return HISA_ERR_WORKSPACE;
  uint8_t *w = noalloc_scratch();
  if (!w) return HISA_ERR_CUDA;
  // Nothing in the scratch has to start at zero: the block lists are written in full by
  // the block stage, the list counters are cleared by the token stage, and every score
  // row is written before it is read.
  return select_launch(q_idx, k_idx, reps, cu_seqlens_q, cu_seqlens_k, seqlens_k, nullptr,
                       num_seqs, total_q, max_seqlen_k, m, k, out_idx, out_scores, out_blocks, w,
                       p, st, s);
}
