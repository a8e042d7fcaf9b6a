// Internal declarations shared by the C-ABI layer and the kernel launchers.
#pragma once

#include <cuda_runtime.h>

#include <atomic>
#include <mutex>

#include "attn.h"

namespace attn {

constexpr int kMaxDevices = 64;

// One-time setup of a kernel (its attributes), done once per device and
// thread-safe. cudaFuncSetAttribute applies to the current device only, so a
// process that drives several GPUs needs it on each of them. `fn` runs with
// the device current, under a lock, until it returns something other than
// ATTN_ERR_CUDA; that status is then returned by every later call on that
// device without taking the lock.
class DeviceOnce {
 public:
  template <class F>
  attn_status_t run(F&& fn) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
      cudaGetLastError();
      return ATTN_ERR_NO_DEVICE;
    }
    if (dev < 0 || dev >= kMaxDevices) return ATTN_ERR_UNSUPPORTED;
    int st = state_[dev].load(std::memory_order_acquire);
    if (st != 0) return static_cast<attn_status_t>(st - 1);
    std::lock_guard<std::mutex> lock(mu_);
    st = state_[dev].load(std::memory_order_relaxed);
    if (st != 0) return static_cast<attn_status_t>(st - 1);
    const attn_status_t r = fn();
    if (r != ATTN_ERR_CUDA) state_[dev].store(static_cast<int>(r) + 1, std::memory_order_release);
    return r;
  }

 private:
  std::mutex mu_;
  std::atomic<int> state_[kMaxDevices] = {};  // 0: not done; else the status + 1
};

// Cycle bound of every pipeline wait of the prefill and backward kernels
// (attn_set_wait_limit; about one second by default).
long long pipeline_wait_limit();

// The bounds-check site that debug kernels launched now report as failed
// (attn_debug_plant_bounds; 0: none).
int planted_bounds_site();

// Number of SMs of the current device (cached per device).
int device_sm_count();

// Returns ATTN_OK if the current device is sm_100.
attn_status_t check_device();

// Host-side argument checks of attn_decode_paged (ATTN_OK when valid).
attn_status_t validate_decode(const attn_decode_params* p);

// Prefill launcher. Arguments were validated by the caller.
attn_status_t launch_prefill(const attn_prefill_params& p, cudaStream_t stream);

// Non-blocking streams of the current device (which = 0 or 1), created once
// and kept for the process: the extra streams of calls that overlap kernels
// or copies with their main stream.
cudaStream_t side_stream(int which = 0);

// Host-side argument checks of attn_prefill (ATTN_OK when valid).
attn_status_t validate_prefill(const attn_prefill_params* p);

// Decode plan: tokens per split (multiple of 16) and the maximum number of
// splits a sequence can have.
struct DecodePlan {
  int split_tokens;
  int max_splits;
  size_t workspace_bytes;
};
DecodePlan plan_decode(const attn_decode_params& p);

// combine = false: rows of more than one split keep their partials in the
// workspace (O at its start, LSE 256-byte aligned after it) for the caller to
// merge; rows of one split are written to p.o / p.lse as usual.
attn_status_t launch_decode(const attn_decode_params& p, const DecodePlan& plan, void* workspace,
                            cudaStream_t stream, bool combine = true);

// The decode kernels' one-time set-up for these parameters (kernel
// attributes), without launching anything: to be done before a stream capture.
attn_status_t prepare_decode(const attn_decode_params& p);

attn_status_t launch_combine(const float* part_o, const float* part_lse, int num_splits, int rows,
                             int head_dim, const int32_t* splits_per_row, const int32_t* seq_lens,
                             int split_tokens, int rows_per_seq, void* out_o, attn_dtype_t out_dtype,
                             float* out_lse, cudaStream_t stream, int32_t* error_flags = nullptr);

// Persistent decode: workspace size and launch (arguments validated by the
// caller; cmd_dev is the device address of the host command block).
size_t decode_persistent_workspace_bytes(const attn_decode_params& p);
attn_status_t launch_decode_persistent(const attn_decode_params& p, int32_t* cmd_dev, void* workspace,
                                       long long idle_cycles, cudaStream_t stream);

// Backward (dQ, dK, dV). Arguments were validated by the caller.
size_t backward_workspace_bytes(const attn_backward_params& p);
attn_status_t launch_backward(const attn_backward_params& p, void* workspace, cudaStream_t stream);

// Shared-prefix (cascade) decode: key ranges of the prefix prefill, the suffix
// decode (its parameters and split plan) and the workspace layout.
struct CascadePlan {
  int prefix_len;
  int ranges;        // prefix key ranges (batch entries of the prefix prefill)
  int range_blocks;  // cache blocks per range (the last range may hold fewer)
  int suffix_cap;    // most tokens a sequence can hold past the prefix
  attn_decode_params suffix;
  DecodePlan suffix_plan;
  size_t off_suffix_lens, off_range_lens, off_q_rep, off_pre_o, off_pre_lse, off_suf_o, off_suf_lse, off_decode;
  size_t workspace_bytes;
};
CascadePlan plan_cascade(const attn_decode_params& p, int prefix_len);
attn_status_t launch_cascade(const attn_decode_params& p, const CascadePlan& plan, void* workspace,
                             cudaStream_t stream);

}  // namespace attn
