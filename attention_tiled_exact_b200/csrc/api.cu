// C ABI of libattn_b200.so: host-side validation and dispatch. Every argument
// check happens here, before anything is enqueued; the kernels only see
// arguments that passed. See include/attn.h for the contract.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <string.h>

#include <atomic>
#include <chrono>
#include <mutex>

#include "attn.h"
#include "internal.h"
#include "bounds_check.cuh"

namespace attn {

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// About one second at the B200's 1.9 GHz boost clock.
constexpr long long kDefaultWaitLimit = 2000000000LL;
static std::atomic<long long> g_wait_limit{kDefaultWaitLimit};

long long pipeline_wait_limit() { return g_wait_limit.load(std::memory_order_relaxed); }

static std::atomic<int> g_planted_site{0};

int planted_bounds_site() { return g_planted_site.load(std::memory_order_relaxed); }

static bool mult8(int64_t s) { return (s % 8) == 0; }

cudaStream_t side_stream(int which) {
  static std::mutex mu;
  static cudaStream_t streams[2][kMaxDevices] = {};
  int dev = 0;
  if (which < 0 || which > 1) return nullptr;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(mu);
  cudaStream_t& s = streams[which][dev];
  if (!s && cudaStreamCreateWithFlags(&s, cudaStreamNonBlocking) != cudaSuccess) {
    cudaGetLastError();
    s = nullptr;
  }
  return s;
}

int device_sm_count() {
  static std::mutex mu;
  static int cache[kMaxDevices] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
  std::lock_guard<std::mutex> lock(mu);
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

attn_status_t check_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return ATTN_ERR_NO_DEVICE;
  }
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
    cudaGetLastError();
    return ATTN_ERR_NO_DEVICE;
  }
  return (major == 10 && minor == 0) ? ATTN_OK : ATTN_ERR_NO_DEVICE;
}

attn_status_t validate_prefill(const attn_prefill_params* p) {
  if (!p) return ATTN_ERR_INVALID_ARG;
  if (p->batch < 0 || p->num_q_heads < 0 || p->num_kv_heads < 0 || p->seqlen_q < 0 || p->seqlen_k < 0)
    return ATTN_ERR_INVALID_ARG;
  if (p->batch > 65535 * 32) return ATTN_ERR_INVALID_ARG;
  if (p->num_kv_heads == 0 || p->num_q_heads == 0) return ATTN_ERR_INVALID_ARG;
  if (p->num_q_heads % p->num_kv_heads != 0) return ATTN_ERR_UNSUPPORTED;
  if (p->head_dim != 64 && p->head_dim != 128) return ATTN_ERR_UNSUPPORTED;
  if (!(p->scale > 0.f) || !isfinite(p->scale)) return ATTN_ERR_INVALID_ARG;
  if (p->o_dtype != ATTN_DTYPE_BF16 && p->o_dtype != ATTN_DTYPE_F32) return ATTN_ERR_INVALID_ARG;
  if (p->cu_seqlens_q && (p->seqlens_q || p->total_q < 0)) return ATTN_ERR_INVALID_ARG;
  const bool paged = p->k_cache != nullptr || p->v_cache != nullptr;
  if (!p->q || !p->o) return ATTN_ERR_INVALID_ARG;
  if (paged) {
    if (!p->k_cache || !p->v_cache || p->k || p->v || !p->block_table || !p->seqlens_k) return ATTN_ERR_INVALID_ARG;
    if (p->block_size != 16) return ATTN_ERR_UNSUPPORTED;
    if (p->max_blocks_per_seq <= 0 || p->num_blocks <= 0) return ATTN_ERR_INVALID_ARG;
    if (!aligned16(p->k_cache) || !aligned16(p->v_cache)) return ATTN_ERR_UNSUPPORTED;
  } else {
    if ((!p->k || !p->v) && p->seqlen_k > 0) return ATTN_ERR_INVALID_ARG;
    if (!aligned16(p->k) || !aligned16(p->v)) return ATTN_ERR_UNSUPPORTED;
    if (!mult8(p->k_batch_stride) || !mult8(p->k_head_stride) || !mult8(p->k_row_stride) ||
        !mult8(p->v_batch_stride) || !mult8(p->v_head_stride) || !mult8(p->v_row_stride))
      return ATTN_ERR_UNSUPPORTED;
    if (p->k_row_stride < p->head_dim || p->v_row_stride < p->head_dim) return ATTN_ERR_INVALID_ARG;
  }
  if (!aligned16(p->q) || !aligned16(p->o)) return ATTN_ERR_UNSUPPORTED;
  if (!mult8(p->q_batch_stride) || !mult8(p->q_head_stride) || !mult8(p->q_row_stride) ||
      !mult8(p->o_batch_stride) || !mult8(p->o_head_stride) || !mult8(p->o_row_stride))
    return ATTN_ERR_UNSUPPORTED;
  if (p->q_row_stride < p->head_dim || p->o_row_stride < p->head_dim) return ATTN_ERR_INVALID_ARG;
  return ATTN_OK;
}

static attn_status_t validate_backward(const attn_backward_params* p) {
  if (!p) return ATTN_ERR_INVALID_ARG;
  if (p->batch < 0 || p->num_q_heads < 0 || p->num_kv_heads < 0 || p->seqlen_q < 0 || p->seqlen_k < 0)
    return ATTN_ERR_INVALID_ARG;
  if (p->num_kv_heads == 0 || p->num_q_heads == 0) return ATTN_ERR_INVALID_ARG;
  if (p->num_q_heads % p->num_kv_heads != 0) return ATTN_ERR_UNSUPPORTED;
  if (p->head_dim != 64 && p->head_dim != 128) return ATTN_ERR_UNSUPPORTED;
  if (!(p->scale > 0.f) || !isfinite(p->scale)) return ATTN_ERR_INVALID_ARG;
  if (p->o_dtype != ATTN_DTYPE_BF16 && p->o_dtype != ATTN_DTYPE_F32) return ATTN_ERR_INVALID_ARG;
  if (p->grad_dtype != ATTN_DTYPE_BF16 && p->grad_dtype != ATTN_DTYPE_F32) return ATTN_ERR_INVALID_ARG;
  if (!p->q || !p->k || !p->v || !p->o || !p->lse || !p->dout || !p->dq || !p->dk || !p->dv)
    return ATTN_ERR_INVALID_ARG;
  const void* ptrs[] = {p->q, p->k, p->v, p->o, p->lse, p->dout, p->dq, p->dk, p->dv};
  for (const void* q : ptrs)
    if (!aligned16(q)) return ATTN_ERR_UNSUPPORTED;
  const int64_t strides[] = {p->q_batch_stride,  p->q_head_stride,  p->q_row_stride,  p->k_batch_stride,
                             p->k_head_stride,   p->k_row_stride,   p->v_batch_stride,  p->v_head_stride,
                             p->v_row_stride,    p->o_batch_stride,  p->o_head_stride,  p->o_row_stride,
                             p->do_batch_stride, p->do_head_stride, p->do_row_stride, p->dq_batch_stride,
                             p->dq_head_stride,  p->dq_row_stride,  p->dk_batch_stride, p->dk_head_stride,
                             p->dk_row_stride,   p->dv_batch_stride, p->dv_head_stride, p->dv_row_stride};
  for (int64_t st : strides)
    if (!mult8(st)) return ATTN_ERR_UNSUPPORTED;
  const int64_t rows[] = {p->q_row_stride, p->k_row_stride, p->v_row_stride, p->o_row_stride,
                          p->do_row_stride, p->dq_row_stride, p->dk_row_stride, p->dv_row_stride};
  for (int64_t rs : rows)
    if (rs < p->head_dim) return ATTN_ERR_INVALID_ARG;
  return ATTN_OK;
}

attn_status_t validate_decode(const attn_decode_params* p) {
  if (!p) return ATTN_ERR_INVALID_ARG;
  if (p->batch < 0 || p->batch > 65535) return ATTN_ERR_INVALID_ARG;
  if (p->num_q_heads <= 0 || p->num_kv_heads <= 0 || p->num_kv_heads > 65535) return ATTN_ERR_INVALID_ARG;
  if (p->num_q_heads % p->num_kv_heads != 0) return ATTN_ERR_UNSUPPORTED;
  const int g = p->num_q_heads / p->num_kv_heads;
  if (g != 1 && g != 2 && g != 4 && g != 8) return ATTN_ERR_UNSUPPORTED;
  if (p->head_dim != 128) return ATTN_ERR_UNSUPPORTED;
  if (p->block_size != 16) return ATTN_ERR_UNSUPPORTED;
  if (p->max_blocks_per_seq <= 0 || p->num_blocks <= 0 || p->max_seq_len < 0 || p->num_splits < 0)
    return ATTN_ERR_INVALID_ARG;
  if ((int64_t)p->max_blocks_per_seq * 16 > INT32_MAX / 2) return ATTN_ERR_INVALID_ARG;
  if (!(p->scale > 0.f) || !isfinite(p->scale)) return ATTN_ERR_INVALID_ARG;
  if (p->o_dtype != ATTN_DTYPE_BF16 && p->o_dtype != ATTN_DTYPE_F32) return ATTN_ERR_INVALID_ARG;
  if (p->kv_dtype != ATTN_DTYPE_BF16 && p->kv_dtype != ATTN_DTYPE_FP8_E4M3) return ATTN_ERR_INVALID_ARG;
  if (p->kv_dtype == ATTN_DTYPE_FP8_E4M3 &&
      (!(p->k_scale > 0.f) || !isfinite(p->k_scale) || !(p->v_scale > 0.f) || !isfinite(p->v_scale)))
    return ATTN_ERR_INVALID_ARG;
  if (!p->q || !p->k_cache || !p->v_cache || !p->block_table || !p->seq_lens || !p->o) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(p->q) || !aligned16(p->k_cache) || !aligned16(p->v_cache) || !aligned16(p->o))
    return ATTN_ERR_UNSUPPORTED;
  return ATTN_OK;
}

}  // namespace attn

extern "C" {

attn_status_t attn_prefill(const attn_prefill_params* p, attn_stream_t stream) {
  attn_status_t st = attn::validate_prefill(p);
  if (st != ATTN_OK) return st;
  if (p->batch == 0 || p->seqlen_q == 0 || (p->cu_seqlens_q && p->total_q == 0)) return ATTN_OK;
  st = attn::check_device();
  if (st != ATTN_OK) return st;
  return attn::launch_prefill(*p, reinterpret_cast<cudaStream_t>(stream));
}

attn_status_t attn_decode_paged(const attn_decode_params* p, void* workspace, size_t workspace_bytes,
                                size_t* workspace_needed, attn_stream_t stream) {
  attn_status_t st = attn::validate_decode(p);
  if (st != ATTN_OK) return st;
  const bool have_dev = attn::check_device() == ATTN_OK;
  attn::DecodePlan plan = attn::plan_decode(*p);
  if (workspace_needed) *workspace_needed = plan.workspace_bytes;
  if (workspace == nullptr && workspace_needed != nullptr) return ATTN_OK;  // size query only
  if (workspace_bytes < plan.workspace_bytes) return ATTN_ERR_WORKSPACE;
  if (plan.workspace_bytes > 0 && (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return ATTN_ERR_UNSUPPORTED;
  if (p->batch == 0) return ATTN_OK;
  if (!have_dev) return ATTN_ERR_NO_DEVICE;
  return attn::launch_decode(*p, plan, workspace, reinterpret_cast<cudaStream_t>(stream));
}

attn_status_t attn_prefill_backward(const attn_backward_params* p, void* workspace, size_t workspace_bytes,
                                    size_t* workspace_needed, attn_stream_t stream) {
  attn_status_t st = attn::validate_backward(p);
  if (st != ATTN_OK) return st;
  const size_t need = attn::backward_workspace_bytes(*p);
  if (workspace_needed) *workspace_needed = need;
  if (workspace == nullptr && workspace_needed != nullptr) return ATTN_OK;  // size query only
  if (workspace_bytes < need) return ATTN_ERR_WORKSPACE;
  if (need > 0 && (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return ATTN_ERR_UNSUPPORTED;
  if (p->batch == 0) return ATTN_OK;
  st = attn::check_device();
  if (st != ATTN_OK) return st;
  return attn::launch_backward(*p, workspace, reinterpret_cast<cudaStream_t>(stream));
}

attn_status_t attn_decode_paged_shared_prefix(const attn_decode_params* p, int32_t prefix_len, void* workspace,
                                             size_t workspace_bytes, size_t* workspace_needed,
                                             attn_stream_t stream) {
  attn_status_t st = attn::validate_decode(p);
  if (st != ATTN_OK) return st;
  if (prefix_len < 0 || prefix_len % 16 != 0 || (int64_t)prefix_len > (int64_t)p->max_blocks_per_seq * 16)
    return ATTN_ERR_INVALID_ARG;
  if (prefix_len == 0) return attn_decode_paged(p, workspace, workspace_bytes, workspace_needed, stream);
  if (p->kv_dtype != ATTN_DTYPE_BF16) return ATTN_ERR_UNSUPPORTED;
  const bool have_dev = attn::check_device() == ATTN_OK;
  attn::CascadePlan plan = attn::plan_cascade(*p, prefix_len);
  if (workspace_needed) *workspace_needed = plan.workspace_bytes;
  if (workspace == nullptr && workspace_needed != nullptr) return ATTN_OK;  // size query only
  if (workspace_bytes < plan.workspace_bytes) return ATTN_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return ATTN_ERR_UNSUPPORTED;
  if (p->batch == 0) return ATTN_OK;
  if (!have_dev) return ATTN_ERR_NO_DEVICE;
  return attn::launch_cascade(*p, plan, workspace, reinterpret_cast<cudaStream_t>(stream));
}

attn_status_t splitkv_lse_combine(const float* part_o, const float* part_lse, int num_splits, int rows,
                                  int head_dim, const int32_t* splits_per_row, void* out_o, attn_dtype_t out_dtype,
                                  float* out_lse, attn_stream_t stream) {
  if (num_splits < 0 || rows < 0) return ATTN_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return ATTN_ERR_UNSUPPORTED;
  if (out_dtype != ATTN_DTYPE_BF16 && out_dtype != ATTN_DTYPE_F32) return ATTN_ERR_INVALID_ARG;
  if (rows == 0) return ATTN_OK;
  if (!out_o || (num_splits > 0 && (!part_o || !part_lse))) return ATTN_ERR_INVALID_ARG;
  if ((num_splits > 0 && !attn::aligned16(part_o)) || !attn::aligned16(out_o)) return ATTN_ERR_UNSUPPORTED;
  attn_status_t st = attn::check_device();
  if (st != ATTN_OK) return st;
  return attn::launch_combine(part_o, part_lse, num_splits, rows, head_dim, splits_per_row, nullptr, 1, 1, out_o,
                              out_dtype, out_lse, reinterpret_cast<cudaStream_t>(stream));
}

attn_status_t attn_decode_persistent_workspace(const attn_decode_params* p, size_t* bytes) {
  attn_status_t st = attn::validate_decode(p);
  if (st != ATTN_OK) return st;
  if (!bytes) return ATTN_ERR_INVALID_ARG;
  if (attn::check_device() != ATTN_OK) return ATTN_ERR_NO_DEVICE;  // the size depends on the SM count
  *bytes = attn::decode_persistent_workspace_bytes(*p);
  return ATTN_OK;
}

attn_status_t attn_decode_persistent_launch(const attn_decode_params* p, attn_persistent_cmd* cmd, void* workspace,
                                            size_t workspace_bytes, long long idle_cycles, attn_stream_t stream) {
  attn_status_t st = attn::validate_decode(p);
  if (st != ATTN_OK) return st;
  if (!cmd || !workspace || p->batch <= 0 || idle_cycles <= 0) return ATTN_ERR_INVALID_ARG;
  st = attn::check_device();
  if (st != ATTN_OK) return st;
  if (workspace_bytes < attn::decode_persistent_workspace_bytes(*p)) return ATTN_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return ATTN_ERR_UNSUPPORTED;
  // The command block is host memory the device must reach: pinned and mapped.
  void* dev = nullptr;
  if (cudaHostGetDevicePointer(&dev, cmd, 0) != cudaSuccess || dev == nullptr) {
    cudaGetLastError();
    return ATTN_ERR_INVALID_ARG;
  }
  memset(cmd, 0, sizeof(*cmd));
  std::atomic_thread_fence(std::memory_order_seq_cst);
  return attn::launch_decode_persistent(*p, reinterpret_cast<int32_t*>(dev), workspace, idle_cycles,
                                        reinterpret_cast<cudaStream_t>(stream));
}

attn_status_t attn_decode_persistent_submit(attn_persistent_cmd* cmd, int32_t batch, int32_t max_seq_len,
                                            int32_t* step) {
  if (!cmd || batch < 0 || max_seq_len < 0) return ATTN_ERR_INVALID_ARG;
  const int32_t seq = __atomic_load_n(&cmd->seq, __ATOMIC_ACQUIRE);
  if (__atomic_load_n(&cmd->done, __ATOMIC_ACQUIRE) != seq) return ATTN_ERR_INVALID_ARG;  // previous step pending
  __atomic_store_n(&cmd->batch, batch, __ATOMIC_RELAXED);
  __atomic_store_n(&cmd->max_seq_len, max_seq_len, __ATOMIC_RELAXED);
  __atomic_store_n(&cmd->seq, seq + 1, __ATOMIC_RELEASE);  // publishes batch and max_seq_len with it
  if (step) *step = seq + 1;
  return ATTN_OK;
}

attn_status_t attn_decode_persistent_wait(const attn_persistent_cmd* cmd, int32_t step, long long timeout_us) {
  if (!cmd) return ATTN_ERR_INVALID_ARG;
  const auto t0 = std::chrono::steady_clock::now();
  while (true) {
    if (__atomic_load_n(&cmd->done, __ATOMIC_ACQUIRE) >= step) return ATTN_OK;
    if (__atomic_load_n(&cmd->status, __ATOMIC_ACQUIRE) != 0) return ATTN_ERR_TIMEOUT;  // the kernel gave up
    const long long us =
        std::chrono::duration_cast<std::chrono::microseconds>(std::chrono::steady_clock::now() - t0).count();
    if (us > timeout_us) return ATTN_ERR_TIMEOUT;
  }
}

void attn_decode_persistent_stop(attn_persistent_cmd* cmd) {
  if (cmd) __atomic_store_n(&cmd->stop, 1, __ATOMIC_RELEASE);
}

void attn_set_wait_limit(long long cycles) {
  attn::g_wait_limit.store(cycles > 0 ? cycles : attn::kDefaultWaitLimit, std::memory_order_relaxed);
}

int attn_debug_bounds_enabled(void) { return ATTN_DEBUG_BOUNDS ? 1 : 0; }

attn_status_t attn_debug_plant_bounds(int site) {
  if (!ATTN_DEBUG_BOUNDS) return ATTN_ERR_UNSUPPORTED;
  if (site < 0 || site > 255) return ATTN_ERR_INVALID_ARG;
  attn::g_planted_site.store(site, std::memory_order_relaxed);
  return ATTN_OK;
}

attn_status_t attn_status_from_flags(int32_t flags) {
  if (flags & ATTN_FAULT_TIMEOUT) return ATTN_ERR_TIMEOUT;
  if (flags != 0) return ATTN_ERR_DEVICE_FAULT;
  return ATTN_OK;
}

attn_status_t attn_sync_error_flags(const int32_t* error_flags, attn_stream_t stream, int32_t* flags_out) {
  if (!error_flags) return ATTN_ERR_INVALID_ARG;
  int32_t word = 0;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(&word, error_flags, sizeof(word), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess) {
    cudaGetLastError();
    return ATTN_ERR_CUDA;
  }
  if (flags_out) *flags_out = word;
  return attn_status_from_flags(word);
}

const char* attn_status_string(attn_status_t status) {
  switch (status) {
    case ATTN_OK: return "ok";
    case ATTN_ERR_INVALID_ARG: return "invalid argument";
    case ATTN_ERR_UNSUPPORTED: return "unsupported shape, dtype or alignment";
    case ATTN_ERR_WORKSPACE: return "workspace too small";
    case ATTN_ERR_CUDA: return "CUDA runtime or launch error";
    case ATTN_ERR_DEVICE_FAULT: return "device-side fault flagged";
    case ATTN_ERR_TIMEOUT: return "device-side wait timed out";
    case ATTN_ERR_NO_DEVICE: return "no sm_100 device is current";
  }
  return "unknown status";
}

int attn_version(void) { return 100; }

}  // extern "C"
