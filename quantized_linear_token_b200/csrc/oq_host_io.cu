// oq_linear_fused_host: the fused layer call on HOST buffers, with the
// host-to-device copy of x, the computation and the device-to-host copy of y
// overlapped chunk by chunk.  (The pages have no counterpart; this is the
// interface for callers whose activations live in host memory.)
//
// The batch is cut into chunks of CHUNK tokens.  Chunk i's x is copied on the
// layer's input stream into one of two device slots, computed on the caller's
// stream, and its y copied back on the layer's output stream from one of two
// device slots, so that the input copy of chunk i + 1 and the output copy of
// chunk i - 1 run while chunk i computes.  When the fused call would decode
// the weights once (large batches), they are decoded once for all chunks, and
// every chunk then runs the same kernels on the same operands as the fused call
// on the whole batch: y is the same bit for bit.
#include <cuda_runtime.h>

#include <algorithm>
#include <mutex>
#include <string>

#include "oq_internal.h"

namespace oq {
namespace {

constexpr int64_t CHUNK = 1024;   // tokens per pipeline chunk
std::mutex g_io_mutex;

size_t r256(size_t b) { return (b + 255) & ~(size_t)255; }

size_t x_row_bytes(const oq_layer* L, int32_t x_dtype) { return (size_t)L->d_in * (x_dtype == OQ_DTYPE_BF16 ? 2 : 4); }

// workspace layout: [fused-call workspace for one chunk | decoded weights (if
// used) | x slot 0 | x slot 1 | y slot 0 | y slot 1]
struct IoLayout {
  int64_t chunk;
  bool w16;
  size_t fused_bytes, w16_off, x_off[2], y_off[2], total;
};

IoLayout io_layout(const oq_layer* L, int32_t x_dtype, int64_t T) {
  IoLayout o{};
  o.chunk = std::min<int64_t>(T, CHUNK);
  o.w16 = fused_decodes_weights(L, x_dtype, T);
  // one chunk's fused workspace; with pre-decoded weights the chunk needs its
  // operand, norms and the fused kernel's flags, and the weights sit after it
  o.fused_bytes = r256(fused_min_workspace(L, o.chunk));
  size_t at = o.fused_bytes;
  if (o.w16) {
    o.fused_bytes = r256(fused_decoded_min_workspace(L, o.chunk));
    at = o.fused_bytes;
    o.w16_off = at;
    at += r256(fused_w16_workspace(L, o.chunk) - fused_min_workspace(L, o.chunk));
  } else if (o.chunk == T) {
    // a single chunk: the fused call's own workspace (its fastest route)
    o.fused_bytes = r256(oq_linear_fused_workspace_size(L, T));
    at = o.fused_bytes;
  }
  for (int k = 0; k < 2; ++k) {
    o.x_off[k] = at;
    at += r256((size_t)o.chunk * x_row_bytes(L, x_dtype));
  }
  for (int k = 0; k < 2; ++k) {
    o.y_off[k] = at;
    at += r256((size_t)o.chunk * (size_t)L->d_out * 4);
  }
  o.total = at;
  return o;
}

oq_status io_init(oq_layer* L) {
  std::lock_guard<std::mutex> lock(g_io_mutex);
  if (L->io_ready) return OQ_OK;
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev != L->device) {
    set_error("oq_linear_fused_host: the layer's device is not current");
    return OQ_ERR_INVALID_ARG;
  }
  for (int k = 0; k < 2; ++k) {
    cudaStream_t s = nullptr;
    if (cudaStreamCreateWithFlags(&s, cudaStreamNonBlocking) != cudaSuccess) {
      set_error("oq_linear_fused_host: cudaStreamCreateWithFlags failed");
      return OQ_ERR_CUDA;
    }
    L->io_stream[k] = s;
  }
  for (int k = 0; k < 8; ++k) {
    cudaEvent_t e = nullptr;
    if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) {
      set_error("oq_linear_fused_host: cudaEventCreateWithFlags failed");
      return OQ_ERR_CUDA;
    }
    L->io_event[k] = e;
  }
  L->io_ready = true;
  return OQ_OK;
}

oq_status cu(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return OQ_OK;
  set_error(std::string("oq_linear_fused_host: ") + what + ": " + cudaGetErrorString(e));
  return OQ_ERR_CUDA;
}

}  // namespace

void io_release(oq_layer* L) {
  if (!L || !L->io_ready) return;
  for (int k = 0; k < 2; ++k)
    if (L->io_stream[k]) cudaStreamDestroy(static_cast<cudaStream_t>(L->io_stream[k]));
  for (int k = 0; k < 8; ++k)
    if (L->io_event[k]) cudaEventDestroy(static_cast<cudaEvent_t>(L->io_event[k]));
  L->io_ready = false;
}

}  // namespace oq

using namespace oq;

extern "C" {

size_t oq_linear_fused_host_workspace_size(const oq_layer* L, int32_t x_dtype, int64_t T) {
  if (!L || T <= 0 || L->int4_only || (x_dtype != OQ_DTYPE_BF16 && x_dtype != OQ_DTYPE_F32)) return 0;
  return io_layout(L, x_dtype, T).total;
}

oq_status oq_linear_fused_host(const oq_layer* layer, const void* x_host, int32_t x_dtype, int64_t T,
                               const uint32_t* Wcodes, const float* r, void* y_host, int32_t y_dtype, void* workspace,
                               size_t workspace_bytes, void* stream) {
  // the copy streams and events are a cache inside the layer
  oq_layer* L = const_cast<oq_layer*>(layer);
  oq_status st =
      fused_check_args(L, x_host, x_dtype, T, Wcodes, r, y_host, y_dtype, workspace, "oq_linear_fused_host");
  if (st != OQ_OK || T == 0) return st;
  if (L->int4_only) {
    set_error("oq_linear_fused_host: not available on an INT4 weight-only layer");
    return OQ_ERR_UNSUPPORTED;
  }
  const IoLayout lay = io_layout(L, x_dtype, T);
  if (workspace_bytes < lay.total) {
    set_error("oq_linear_fused_host: workspace too small (see oq_linear_fused_host_workspace_size)");
    return OQ_ERR_INVALID_ARG;
  }
  st = io_init(L);
  if (st != OQ_OK) return st;
  cudaStream_t comp = static_cast<cudaStream_t>(stream);
  cudaStream_t s_in = static_cast<cudaStream_t>(L->io_stream[0]);
  cudaStream_t s_out = static_cast<cudaStream_t>(L->io_stream[1]);
  cudaEvent_t* ev = reinterpret_cast<cudaEvent_t*>(L->io_event);
  // ev[0]: start (caller's stream); ev[1 + k]: x slot k filled; ev[3 + k]:
  // chunk in slot k computed; ev[5 + k]: y slot k copied out; ev[7]: done
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  const bool y_bf16 = y_dtype == OQ_DTYPE_BF16;
  const size_t xrow = x_row_bytes(L, x_dtype), yrow = (size_t)L->d_out * (y_bf16 ? 2 : 4);
  const unsigned char* xh = static_cast<const unsigned char*>(x_host);
  unsigned char* yh = reinterpret_cast<unsigned char*>(y_host);

  if ((st = cu(cudaEventRecord(ev[0], comp), "record start")) != OQ_OK) return st;
  if ((st = cu(cudaStreamWaitEvent(s_in, ev[0], 0), "wait start")) != OQ_OK) return st;
  if ((st = cu(cudaStreamWaitEvent(s_out, ev[0], 0), "wait start")) != OQ_OK) return st;
  const uint16_t* w16 = nullptr;
  if (lay.w16) {
    uint16_t* w = reinterpret_cast<uint16_t*>(ws + lay.w16_off);
    st = decode_weight_levels(L, Wcodes, w, comp);
    if (st != OQ_OK) return st;
    w16 = w;
  }
  const int64_t n = (T + lay.chunk - 1) / lay.chunk;
  for (int64_t i = 0; i < n; ++i) {
    const int k = (int)(i & 1);
    const int64_t t0 = i * lay.chunk, tc = std::min(lay.chunk, T - t0);
    void* xd = ws + lay.x_off[k];
    void* yd = ws + lay.y_off[k];
    // x slot k is free once chunk i - 2 has been computed
    if (i >= 2 && (st = cu(cudaStreamWaitEvent(s_in, ev[3 + k], 0), "wait slot")) != OQ_OK) return st;
    if ((st = cu(cudaMemcpyAsync(xd, xh + (size_t)t0 * xrow, (size_t)tc * xrow, cudaMemcpyHostToDevice, s_in),
                 "copy x in")) != OQ_OK)
      return st;
    if ((st = cu(cudaEventRecord(ev[1 + k], s_in), "record x")) != OQ_OK) return st;
    // compute once x has arrived and y slot k has been copied out (chunk i - 2)
    if ((st = cu(cudaStreamWaitEvent(comp, ev[1 + k], 0), "wait x")) != OQ_OK) return st;
    if (i >= 2 && (st = cu(cudaStreamWaitEvent(comp, ev[5 + k], 0), "wait y slot")) != OQ_OK) return st;
    st = fused_run(L, xd, x_dtype, tc, Wcodes, r, yd, y_bf16, ws, lay.fused_bytes, comp, w16);
    if (st != OQ_OK) return st;
    if ((st = cu(cudaEventRecord(ev[3 + k], comp), "record compute")) != OQ_OK) return st;
    if ((st = cu(cudaStreamWaitEvent(s_out, ev[3 + k], 0), "wait compute")) != OQ_OK) return st;
    if ((st = cu(cudaMemcpyAsync(yh + (size_t)t0 * yrow, yd, (size_t)tc * yrow, cudaMemcpyDeviceToHost, s_out),
                 "copy y out")) != OQ_OK)
      return st;
    if ((st = cu(cudaEventRecord(ev[5 + k], s_out), "record y")) != OQ_OK) return st;
  }
  // the caller's stream continues after the last copy out
  if ((st = cu(cudaEventRecord(ev[7], s_out), "record done")) != OQ_OK) return st;
  return cu(cudaStreamWaitEvent(comp, ev[7], 0), "wait done");
}

}  // extern "C"
