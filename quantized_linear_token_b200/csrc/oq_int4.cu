// INT4 weight-only round-to-nearest of weight rows: the AdaLN exception path
// (gecl notes Method 5: the dynamic AdaLN modulation projection cannot absorb
// a static rotation, so it is kept at INT4 weight-only RTN).  The pages leave
// the scale open; per output row r_o = max_i |w_oi| / 7 and
// q = round-half-even(w / r_o) in [-7, 7], each decision taken in fp32 with
// IEEE division.  Codes use the 4-bit format of the Lloyd-Max codes (q >= 0 ->
// q + 8, q < 0 -> q + 7; 7 never occurs), packed eight per word.
#include <cuda_bf16.h>

#include "oq_internal.h"

namespace oq {
namespace {

template <typename WT>
__device__ __forceinline__ float as_f32(WT v) {
  if constexpr (sizeof(WT) == 2) return __bfloat162float(v);
  else return v;
}

template <typename WT>
__global__ void __launch_bounds__(256) rtn4_kernel(const WT* __restrict__ W, int rows, int d,
                                                   uint32_t* __restrict__ codes, float* __restrict__ scale) {
  __shared__ float red[8];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int row = blockIdx.x; row < rows; row += gridDim.x) {
    const WT* w = W + (size_t)row * d;
    float m = 0.f;
    for (int i = threadIdx.x; i < d; i += blockDim.x) m = fmaxf(m, fabsf(as_f32(w[i])));
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    if (lane == 0) red[warp] = m;
    __syncthreads();
    float amax = red[0];
#pragma unroll
    for (int k = 1; k < 8; ++k) amax = fmaxf(amax, red[k]);
    const float sc = __fdiv_rn(amax, 7.0f);
    for (int gq = threadIdx.x; gq < d / 8; gq += blockDim.x) {
      uint32_t word = 0u;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        float q = (sc > 0.f) ? rintf(__fdiv_rn(as_f32(w[8 * gq + e]), sc)) : 0.f;
        q = fminf(fmaxf(q, -7.f), 7.f);
        const int qi = (int)q;
        word |= (uint32_t)(qi >= 0 ? qi + 8 : qi + 7) << (4 * e);
      }
      codes[(size_t)row * (d / 8) + gq] = word;
    }
    if (threadIdx.x == 0) scale[row] = sc;
    __syncthreads();   // red is reused by the next row
  }
}

}  // namespace

oq_status rtn4_prepare_launch(const void* W, int w_dtype, int rows, int d, uint32_t* codes, float* scale,
                              void* stream) {
  if (rows == 0) return OQ_OK;
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = rows < 8 * sms ? rows : 8 * sms;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (w_dtype == OQ_DTYPE_BF16)
    rtn4_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(W), rows, d, codes, scale);
  else
    rtn4_kernel<float><<<grid, 256, 0, st>>>(static_cast<const float*>(W), rows, d, codes, scale);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error(std::string("INT4 weight prepare launch: ") + cudaGetErrorString(e));
    return OQ_ERR_CUDA;
  }
  return OQ_OK;
}

}  // namespace oq
