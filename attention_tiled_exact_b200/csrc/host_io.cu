// attn_prefill_from_host: a dense prefill whose inputs come from, and whose
// outputs go back to, host memory, with the copies overlapped with compute.
//
// The batch is cut into chunks of one batch entry and a group of key/value
// heads (with their query heads): in the contiguous [batch, heads, seqlen,
// head_dim] layout every chunk's Q, K, V, O and LSE is one contiguous range
// of host and device memory, so each chunk is three host-to-device copies,
// one prefill launch over the chunk (batch 1, the group's heads) and two
// device-to-host copies. Copies in each direction go on their own side
// stream (the two PCIe directions run at the same time) and events order them
// against the prefill on the caller's stream: chunk c's prefill waits for its
// inputs, its outputs' copy waits for its prefill. One cudaMemcpyAsync per
// copy.
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <vector>

#include "internal.h"

namespace attn {

namespace {

struct Events {
  std::vector<cudaEvent_t> ev;
  ~Events() {
    for (cudaEvent_t e : ev) cudaEventDestroy(e);  // released once the recorded work completes
  }
  cudaEvent_t make() {
    cudaEvent_t e = nullptr;
    if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) {
      cudaGetLastError();
      return nullptr;
    }
    ev.push_back(e);
    return e;
  }
};

bool contiguous(int64_t bs, int64_t hs, int64_t rs, int heads, int rows, int D) {
  return rs == D && hs == (int64_t)rows * D && bs == (int64_t)heads * rows * D;
}

}  // namespace

attn_status_t launch_prefill_from_host(const attn_prefill_params& p, const attn_prefill_host_io& io,
                                       cudaStream_t stream) {
  const int D = p.head_dim, G = p.num_q_heads / p.num_kv_heads;
  const int hpc = io.kv_heads_per_chunk > 0 ? io.kv_heads_per_chunk : p.num_kv_heads;
  const size_t osz = p.o_dtype == ATTN_DTYPE_F32 ? 4 : 2;
  // Bytes of one query head / key head of one batch entry.
  const size_t qh = (size_t)p.seqlen_q * D * 2, kh = (size_t)p.seqlen_k * D * 2;
  const size_t oh = (size_t)p.seqlen_q * D * osz, lh = (size_t)p.seqlen_q * 4;
  cudaStream_t s_in = side_stream(0), s_out = side_stream(1);
  if (!s_in || !s_out) return ATTN_ERR_CUDA;
  Events evs;
  // Both side streams start after the work already on `stream` (an earlier
  // call's compute may still read the device buffers).
  cudaEvent_t start = evs.make();
  if (!start || cudaEventRecord(start, stream) != cudaSuccess || cudaStreamWaitEvent(s_in, start, 0) != cudaSuccess ||
      cudaStreamWaitEvent(s_out, start, 0) != cudaSuccess) {
    cudaGetLastError();
    return ATTN_ERR_CUDA;
  }
  const uint8_t* hq = static_cast<const uint8_t*>(io.q);
  const uint8_t* hk = static_cast<const uint8_t*>(io.k);
  const uint8_t* hv = static_cast<const uint8_t*>(io.v);
  uint8_t* ho = static_cast<uint8_t*>(io.o);
  uint8_t* hl = reinterpret_cast<uint8_t*>(io.lse);
  const uint8_t* dq = static_cast<const uint8_t*>(p.q);
  const uint8_t* dk = static_cast<const uint8_t*>(p.k);
  const uint8_t* dv = static_cast<const uint8_t*>(p.v);
  uint8_t* d_o = static_cast<uint8_t*>(p.o);
  uint8_t* dl = reinterpret_cast<uint8_t*>(p.lse);
  attn_status_t st = ATTN_OK;
  for (int b = 0; b < p.batch && st == ATTN_OK; ++b) {
    for (int h0 = 0; h0 < p.num_kv_heads && st == ATTN_OK; h0 += hpc) {
      // This chunk: kv heads [h0, h0 + hpc), query heads [h0 G, (h0 + hpc) G).
      const size_t qoff = ((size_t)b * p.num_q_heads + (size_t)h0 * G) * qh;
      const size_t koff = ((size_t)b * p.num_kv_heads + h0) * kh;
      const size_t ooff = ((size_t)b * p.num_q_heads + (size_t)h0 * G) * oh;
      const size_t loff = ((size_t)b * p.num_q_heads + (size_t)h0 * G) * lh;
      const size_t nq = (size_t)hpc * G;
      cudaEvent_t in_done = evs.make(), computed = evs.make();
      if (!in_done || !computed) return ATTN_ERR_CUDA;
      bool ok = cudaMemcpyAsync((void*)(dq + qoff), hq + qoff, nq * qh, cudaMemcpyHostToDevice, s_in) == cudaSuccess;
      if (p.seqlen_k > 0) {
        ok = ok && cudaMemcpyAsync((void*)(dk + koff), hk + koff, hpc * kh, cudaMemcpyHostToDevice, s_in) == cudaSuccess;
        ok = ok && cudaMemcpyAsync((void*)(dv + koff), hv + koff, hpc * kh, cudaMemcpyHostToDevice, s_in) == cudaSuccess;
      }
      ok = ok && cudaEventRecord(in_done, s_in) == cudaSuccess && cudaStreamWaitEvent(stream, in_done, 0) == cudaSuccess;
      if (!ok) {
        cudaGetLastError();
        st = ATTN_ERR_CUDA;
        break;
      }
      attn_prefill_params c = p;
      c.batch = 1;
      c.num_q_heads = (int)nq;
      c.num_kv_heads = hpc;
      c.q = dq + qoff;
      c.k = p.seqlen_k > 0 ? dk + koff : nullptr;
      c.v = p.seqlen_k > 0 ? dv + koff : nullptr;
      c.o = d_o + ooff;
      c.lse = dl ? reinterpret_cast<float*>(dl + loff) : nullptr;
      st = launch_prefill(c, stream);
      if (st != ATTN_OK) break;
      ok = cudaEventRecord(computed, stream) == cudaSuccess && cudaStreamWaitEvent(s_out, computed, 0) == cudaSuccess;
      ok = ok && cudaMemcpyAsync(ho + ooff, d_o + ooff, nq * oh, cudaMemcpyDeviceToHost, s_out) == cudaSuccess;
      if (dl) ok = ok && cudaMemcpyAsync(hl + loff, dl + loff, nq * lh, cudaMemcpyDeviceToHost, s_out) == cudaSuccess;
      if (!ok) {
        cudaGetLastError();
        st = ATTN_ERR_CUDA;
      }
    }
  }
  // Join: work enqueued on `stream` after the call starts after every copy
  // (also on the error path, so that no copy of this call is left unordered).
  cudaEvent_t in_end = evs.make(), out_end = evs.make();
  if (!in_end || !out_end || cudaEventRecord(in_end, s_in) != cudaSuccess ||
      cudaEventRecord(out_end, s_out) != cudaSuccess || cudaStreamWaitEvent(stream, in_end, 0) != cudaSuccess ||
      cudaStreamWaitEvent(stream, out_end, 0) != cudaSuccess) {
    cudaGetLastError();
    return ATTN_ERR_CUDA;
  }
  return st;
}

}  // namespace attn

attn_status_t attn_prefill_from_host(const attn_prefill_params* p, const attn_prefill_host_io* io,
                                     attn_stream_t stream) {
  attn_status_t st = attn::validate_prefill(p);
  if (st != ATTN_OK) return st;
  if (!io || !io->q || !io->o || (p->seqlen_k > 0 && (!io->k || !io->v)) || (p->lse && !io->lse))
    return ATTN_ERR_INVALID_ARG;
  if (p->k_cache || p->seqlens_q || p->seqlens_k || p->cu_seqlens_q) return ATTN_ERR_UNSUPPORTED;
  const int hpc = io->kv_heads_per_chunk;
  if (hpc < 0 || (hpc > 0 && p->num_kv_heads % hpc != 0)) return ATTN_ERR_INVALID_ARG;
  const int D = p->head_dim;
  if (!attn::contiguous(p->q_batch_stride, p->q_head_stride, p->q_row_stride, p->num_q_heads, p->seqlen_q, D) ||
      !attn::contiguous(p->o_batch_stride, p->o_head_stride, p->o_row_stride, p->num_q_heads, p->seqlen_q, D) ||
      (p->seqlen_k > 0 &&
       (!attn::contiguous(p->k_batch_stride, p->k_head_stride, p->k_row_stride, p->num_kv_heads, p->seqlen_k, D) ||
        !attn::contiguous(p->v_batch_stride, p->v_head_stride, p->v_row_stride, p->num_kv_heads, p->seqlen_k, D))))
    return ATTN_ERR_UNSUPPORTED;
  if (p->batch == 0 || p->seqlen_q == 0) return ATTN_OK;
  st = attn::check_device();
  if (st != ATTN_OK) return st;
  return attn::launch_prefill_from_host(*p, *io, reinterpret_cast<cudaStream_t>(stream));
}
