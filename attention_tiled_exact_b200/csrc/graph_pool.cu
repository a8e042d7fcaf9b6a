// A pool of CUDA graphs of the paged decode step, one per static shape.
//
// The decode step (split kernel + combine) of a given batch and length bound
// is captured once and replayed for every later step of that shape, which
// removes the per-kernel launch cost ("GPU Kernel 调度:大模型推理的拐点 2026",
// CUDA Graph section: capture a pool of static shapes up front and replay the
// nearest one). The captured kernels read the sequence lengths, the block
// tables and q from the caller's static buffers on every replay, so one graph
// serves every step whose batch and length bound fit its shape: the pool
// replays the smallest (batch bucket, length bucket) that covers the step.
#include <cuda_runtime.h>

#include <algorithm>
#include <mutex>
#include <new>
#include <vector>

#include "attn.h"
#include "internal.h"

struct attn_decode_graph_pool {
  attn_decode_params base;            // static buffers; batch and max_seq_len vary per graph
  void* workspace = nullptr;
  size_t workspace_bytes = 0;
  std::vector<int32_t> batches, lens;  // ascending buckets
  std::vector<cudaGraphExec_t> execs;  // [batch bucket][length bucket]
  std::mutex mu;                       // replays are serialised by the caller; this only guards the handles
};

namespace attn {
namespace {

bool ascending_positive(const int32_t* v, int n) {
  if (!v || n <= 0 || n > 1024) return false;
  for (int i = 0; i < n; ++i)
    if (v[i] <= 0 || (i > 0 && v[i] <= v[i - 1])) return false;
  return true;
}

attn_decode_params bucket_params(const attn_decode_params& p, int32_t batch, int32_t len) {
  attn_decode_params q = p;
  q.batch = batch;
  q.max_seq_len = len;
  return q;
}

void destroy_execs(attn_decode_graph_pool* pool) {
  for (cudaGraphExec_t e : pool->execs)
    if (e) cudaGraphExecDestroy(e);
  pool->execs.clear();
}

}  // namespace
}  // namespace attn

extern "C" {

attn_status_t attn_decode_graph_pool_workspace(const attn_decode_params* p, const int32_t* batch_buckets, int n_batch,
                                               const int32_t* len_buckets, int n_len, size_t* bytes) {
  attn_status_t st = attn::validate_decode(p);
  if (st != ATTN_OK) return st;
  if (!bytes || !attn::ascending_positive(batch_buckets, n_batch) || !attn::ascending_positive(len_buckets, n_len))
    return ATTN_ERR_INVALID_ARG;
  if (batch_buckets[n_batch - 1] > p->batch) return ATTN_ERR_INVALID_ARG;  // buckets must fit the static buffers
  if (attn::check_device() != ATTN_OK) return ATTN_ERR_NO_DEVICE;  // the plan depends on the SM count
  size_t need = 0;
  for (int i = 0; i < n_batch; ++i)
    for (int j = 0; j < n_len; ++j)
      need = std::max(need, attn::plan_decode(attn::bucket_params(*p, batch_buckets[i], len_buckets[j])).workspace_bytes);
  *bytes = need;
  return ATTN_OK;
}

attn_status_t attn_decode_graph_pool_create(const attn_decode_params* p, const int32_t* batch_buckets, int n_batch,
                                            const int32_t* len_buckets, int n_len, void* workspace,
                                            size_t workspace_bytes, attn_decode_graph_pool** out) {
  if (!out) return ATTN_ERR_INVALID_ARG;
  *out = nullptr;
  size_t need = 0;
  attn_status_t st = attn_decode_graph_pool_workspace(p, batch_buckets, n_batch, len_buckets, n_len, &need);
  if (st != ATTN_OK) return st;
  if (workspace_bytes < need || (need > 0 && !workspace)) return ATTN_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return ATTN_ERR_UNSUPPORTED;
  st = attn::prepare_decode(*p);  // kernel attributes before any capture
  if (st != ATTN_OK) return st;
  attn_decode_graph_pool* pool = new (std::nothrow) attn_decode_graph_pool();
  if (!pool) return ATTN_ERR_INVALID_ARG;
  pool->base = *p;
  pool->workspace = workspace;
  pool->workspace_bytes = workspace_bytes;
  pool->batches.assign(batch_buckets, batch_buckets + n_batch);
  pool->lens.assign(len_buckets, len_buckets + n_len);
  cudaStream_t s = nullptr;
  if (cudaStreamCreateWithFlags(&s, cudaStreamNonBlocking) != cudaSuccess) {
    cudaGetLastError();
    delete pool;
    return ATTN_ERR_CUDA;
  }
  st = ATTN_OK;
  for (int i = 0; i < n_batch && st == ATTN_OK; ++i) {
    for (int j = 0; j < n_len && st == ATTN_OK; ++j) {
      const attn_decode_params q = attn::bucket_params(*p, batch_buckets[i], len_buckets[j]);
      cudaGraph_t g = nullptr;
      cudaGraphExec_t e = nullptr;
      if (cudaStreamBeginCapture(s, cudaStreamCaptureModeThreadLocal) != cudaSuccess) {
        st = ATTN_ERR_CUDA;
        break;
      }
      const attn_status_t call = attn_decode_paged(&q, workspace, workspace_bytes, nullptr,
                                                   reinterpret_cast<attn_stream_t>(s));
      const cudaError_t end = cudaStreamEndCapture(s, &g);
      if (call != ATTN_OK) st = call;
      else if (end != cudaSuccess || cudaGraphInstantiate(&e, g, 0) != cudaSuccess) st = ATTN_ERR_CUDA;
      if (g) cudaGraphDestroy(g);
      pool->execs.push_back(e);
    }
  }
  cudaStreamDestroy(s);
  if (st != ATTN_OK) {
    cudaGetLastError();
    attn::destroy_execs(pool);
    delete pool;
    return st;
  }
  *out = pool;
  return ATTN_OK;
}

attn_status_t attn_decode_graph_pool_replay(attn_decode_graph_pool* pool, int32_t batch, int32_t max_seq_len,
                                            attn_stream_t stream, int32_t* bucket_batch, int32_t* bucket_len) {
  if (!pool || batch < 0 || max_seq_len < 0) return ATTN_ERR_INVALID_ARG;
  if (batch == 0) return ATTN_OK;
  const auto ib = std::lower_bound(pool->batches.begin(), pool->batches.end(), batch);
  const auto il = max_seq_len == 0 ? pool->lens.end() - 1
                                   : std::lower_bound(pool->lens.begin(), pool->lens.end(), max_seq_len);
  if (ib == pool->batches.end() || il == pool->lens.end()) return ATTN_ERR_INVALID_ARG;  // no bucket covers it
  const size_t k = (size_t)(ib - pool->batches.begin()) * pool->lens.size() + (size_t)(il - pool->lens.begin());
  if (bucket_batch) *bucket_batch = *ib;
  if (bucket_len) *bucket_len = *il;
  cudaGraphExec_t e;
  {
    std::lock_guard<std::mutex> lock(pool->mu);
    e = pool->execs[k];
  }
  if (cudaGraphLaunch(e, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) {
    cudaGetLastError();
    return ATTN_ERR_CUDA;
  }
  return ATTN_OK;
}

void attn_decode_graph_pool_destroy(attn_decode_graph_pool* pool) {
  if (!pool) return;
  attn::destroy_execs(pool);
  delete pool;
}

}  // extern "C"
