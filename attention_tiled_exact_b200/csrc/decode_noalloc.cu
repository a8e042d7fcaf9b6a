// Paged decode for callers that cannot allocate device memory.
//
// attn_decode_paged needs a caller-provided workspace for the split partials.
// Some callers have no way to provide one: a host program that only receives
// tensor pointers from another component (and has no allocator of its own to
// pass through a C ABI), or a latency-critical loop that must not call
// cudaMalloc, which can synchronise the device. This entry point keeps the
// partials in a fixed-size array of device memory that belongs to the library
// instead, so it allocates nothing per call.
//
// The array is a file-scope __device__ variable: every GPU on which the library
// is loaded holds kNoAllocScratchBytes of it until the process exits. In host
// code the variable's name is only a host-side stand-in, so its device address
// is looked up with cudaGetSymbolAddress, once per device, with that device
// current, on the first call made on that device. That first call should come
// before any stream capture. All calls share the one array and it keeps the
// last call's contents: the decode kernel writes every partial that the combine
// later reads, so nothing has to start at zero, but calls whose kernels overlap
// on the GPU (for example on two streams) race on the array.
#include <cuda_runtime.h>

#include <mutex>

#include "attn.h"
#include "internal.h"

namespace attn {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;  // 16 MiB
static __device__ __align__(256) unsigned char g_decode_scratch[kNoAllocScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices];
bool g_scratch_ready[kMaxDevices];

// Device address of g_decode_scratch on the current device (looked up once per device).
attn_status_t scratch_on_current_device(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return ATTN_ERR_NO_DEVICE;
  }
  if (dev < 0 || dev >= kMaxDevices) return ATTN_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ready[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_decode_scratch) != cudaSuccess || ptr == nullptr) {
      cudaGetLastError();
      return ATTN_ERR_CUDA;
    }
    g_scratch_ptr[dev] = ptr;
    g_scratch_ready[dev] = true;
  }
  *out = g_scratch_ptr[dev];
  return ATTN_OK;
}

}  // namespace
}  // namespace attn

extern "C" attn_status_t attn_decode_paged_noalloc(const attn_decode_params* p, attn_stream_t stream) {
  attn_status_t st = attn::validate_decode(p);
  if (st != ATTN_OK) return st;
  const attn::DecodePlan plan = attn::plan_decode(*p);
  if (plan.workspace_bytes > attn::kNoAllocScratchBytes) return ATTN_ERR_WORKSPACE;
  if (p->batch == 0) return ATTN_OK;
  st = attn::check_device();
  if (st != ATTN_OK) return st;
  void* scratch = nullptr;
  if (plan.workspace_bytes > 0) {
    st = attn::scratch_on_current_device(&scratch);
    if (st != ATTN_OK) return st;
  }
  return attn::launch_decode(*p, plan, scratch, reinterpret_cast<cudaStream_t>(stream));
}
