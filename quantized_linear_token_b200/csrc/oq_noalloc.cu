// oq_linear_fused_static: the fused layer call for callers that cannot
// allocate device memory.  Some callers have no allocator to call: inference
// runtimes that hand out no device memory to plug-ins, deployments whose
// device memory is fixed when the process starts, and real-time loops in
// which an allocation (and the synchronisation it can imply) is not allowed.
// For them the scratch that oq_linear_fused takes from the caller lives in a
// fixed array in device memory that belongs to this library.  That scratch is
// the fused call's least workspace: the A operand that the rotate-quantize
// kernel hands to the contraction (the fp16 levels of the activation codes
// for bf16 x with d_out % 256 == 0, the packed codes otherwise) and the token
// norms.
//
// The array is a file-scope static __device__ array of OQ_STATIC_SCRATCH_BYTES
// bytes: every GPU that loads the library holds it until the process exits.
// Host code cannot use the array's name as a device address, so the first
// call on each device looks the address up with cudaGetSymbolAddress (with
// that device current) and keeps it.  That first call should therefore come
// before any stream capture.  No call allocates or frees memory.
//
// All calls share the one array and it keeps the last call's contents.  Every
// byte a call reads is written earlier in the same call (the A operand and
// norms of its own tokens), so nothing needs clearing, but two calls that run
// at the same time on the GPU (different streams, or different host threads)
// race on the array and give wrong results.
#include <cuda_runtime.h>

#include <mutex>
#include <string>

#include "oq_internal.h"

namespace {

__device__ __align__(256) unsigned char oq_static_scratch[OQ_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch[kMaxDevices] = {nullptr};

// device address of the scratch array on the current device (looked up once)
oq_status scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    oq::set_error(std::string("oq_linear_fused_static: cudaGetDevice: ") + cudaGetErrorString(e));
    return OQ_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) {
    oq::set_error("oq_linear_fused_static: device index out of range");
    return OQ_ERR_UNSUPPORTED;
  }
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, oq_static_scratch);
    if (e != cudaSuccess || !p) {
      oq::set_error(std::string("oq_linear_fused_static: cudaGetSymbolAddress: ") + cudaGetErrorString(e));
      return OQ_ERR_CUDA;
    }
    g_scratch[dev] = p;
  }
  *out = g_scratch[dev];
  return OQ_OK;
}

}  // namespace

extern "C" oq_status oq_linear_fused_static(const oq_layer* layer, const void* x, int32_t x_dtype, int64_t T,
                                            const uint32_t* Wcodes, const float* r, float* y, void* stream) {
  if (!layer) {
    oq::set_error("oq_linear_fused_static: layer is null");
    return OQ_ERR_INVALID_ARG;
  }
  if (T < 0) {
    oq::set_error("oq_linear_fused_static: T < 0");
    return OQ_ERR_INVALID_ARG;
  }
  if (T == 0) return OQ_OK;
  // the static array serves as the fused call's least workspace, so the
  // weights are decoded inside the contraction at every batch size
  const size_t need = oq::fused_min_workspace(layer, T);
  if (need > (size_t)OQ_STATIC_SCRATCH_BYTES) {
    oq::set_error("oq_linear_fused_static: " + std::to_string(T) + " tokens need " + std::to_string(need) +
                  " bytes of scratch, more than the " + std::to_string((size_t)OQ_STATIC_SCRATCH_BYTES) +
                  "-byte static array; use oq_linear_fused with a caller workspace or split the batch");
    return OQ_ERR_INVALID_ARG;
  }
  void* scratch = nullptr;
  const oq_status st = scratch_address(&scratch);
  if (st != OQ_OK) return st;
  return oq_linear_fused(layer, x, x_dtype, T, Wcodes, r, y, OQ_DTYPE_F32, scratch, need, stream);
}
