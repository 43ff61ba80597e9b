// topk_noalloc.cu -- ddt_topk for callers that cannot allocate device memory.
//
// Some callers of a top-k cannot obtain scratch memory at the point of the
// call: code that runs inside an allocator-free region (a custom memory
// manager that owns the whole heap, an embedded runtime with a fixed memory
// plan, a plug-in loaded into a host that forbids cudaMalloc from plug-ins).
// ddt_topk_noalloc serves them.  Its scratch is one fixed array in device
// global memory that belongs to this library: every GPU that loads libddt.so
// keeps DDT_TOPK_NOALLOC_SCRATCH_BYTES of it until the process exits.
//
// * The array's device address is looked up (cudaGetSymbolAddress) on
//   every call made outside stream capture, with the calling device
//   current, and remembered per device; a call made while its stream is
//   being captured uses the remembered address, so the first call on a
//   device must come before any capture.  A device reset (or a new primary
//   context) reloads the library's device code at another address: the next
//   call outside capture picks that up.
// * The array is shared by every call on that device and keeps whatever the
//   last call left in it.  Each call checks its arguments exactly as
//   ddt_topk does (same status codes) and only then clears the part it
//   needs (an asynchronous memset on the caller's stream), so calls that
//   follow each other on one stream are independent; calls that overlap on
//   the GPU (on different streams) race on the array and give wrong results.
// * The entry point never calls cudaMalloc, cudaFree or any allocating
//   library routine.
#include <mutex>

#include "ddt.h"
#include "launch.h"

namespace {

static __device__ __align__(256) unsigned char g_topk_scratch[DDT_TOPK_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device: looked up
// again outside capture, the remembered one inside.
ddt_status scratch_address(cudaStream_t stream, void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return DDT_ERR_CUDA;
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(stream, &cap) != cudaSuccess) return DDT_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (cap == cudaStreamCaptureStatusNone) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_topk_scratch) != cudaSuccess || p == nullptr)
      return DDT_ERR_CUDA;
    g_addr[dev] = p;
  } else if (g_addr[dev] == nullptr) {
    return DDT_ERR_CUDA;  // never called on this device outside capture
  }
  *out = g_addr[dev];
  return DDT_OK;
}

}  // namespace

extern "C" ddt_status ddt_topk_noalloc(const void* logits, ddt_dtype dtype, int batch, int L,
                                       int V, int64_t row_stride, int k, float inv_temperature,
                                       int32_t* ids, float* zk, float* logp, float* lse,
                                       cudaStream_t stream) {
  const ddt_status chk = ddt::topk_check(logits, dtype, batch, L, V, row_stride, k,
                                         inv_temperature, ids, zk, lse);
  if (chk != DDT_OK) return chk;
  const size_t need = ddt_topk_workspace_size(batch, L, V, k);
  if (need > (size_t)DDT_TOPK_NOALLOC_SCRATCH_BYTES) return DDT_ERR_WORKSPACE;
  void* scratch = nullptr;
  if (need > 0) {
    const ddt_status st = scratch_address(stream, &scratch);
    if (st != DDT_OK) return st;
    if (cudaMemsetAsync(scratch, 0, need, stream) != cudaSuccess) return DDT_ERR_CUDA;
  }
  return ddt_topk(logits, dtype, batch, L, V, row_stride, k, inv_temperature, ids, zk, logp, lse,
                  scratch, (size_t)DDT_TOPK_NOALLOC_SCRATCH_BYTES, stream);
}
