// Internal declarations shared by the C-ABI layer and the kernel launchers.
#pragma once

#include <cuda_runtime.h>

#include "attn.h"

namespace attn {

// Number of SMs of the current device (cached per device).
int device_sm_count();

// Returns ATTN_OK if the current device is sm_100.
attn_status_t check_device();

// Host-side argument checks of attn_decode_paged (ATTN_OK when valid).
attn_status_t validate_decode(const attn_decode_params* p);

// Prefill launcher. Arguments were validated by the caller.
attn_status_t launch_prefill(const attn_prefill_params& p, cudaStream_t stream);

// Decode plan: tokens per split (multiple of 16) and the maximum number of
// splits a sequence can have.
struct DecodePlan {
  int split_tokens;
  int max_splits;
  size_t workspace_bytes;
};
DecodePlan plan_decode(const attn_decode_params& p);

attn_status_t launch_decode(const attn_decode_params& p, const DecodePlan& plan, void* workspace,
                            cudaStream_t stream);

attn_status_t launch_combine(const float* part_o, const float* part_lse, int num_splits, int rows,
                             int head_dim, const int32_t* splits_per_row, const int32_t* seq_lens,
                             int split_tokens, int rows_per_seq, void* out_o, attn_dtype_t out_dtype,
                             float* out_lse, cudaStream_t stream);

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
