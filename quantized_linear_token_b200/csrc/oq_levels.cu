// Decode-then-contract route for large batches, first kernel: packed code
// rows [R, K] -> their fp16 operand values alpha * C[code] (row-major [R, K];
// gecl notes Limitation 3, the centroid lookup of every code).  One pass over
// the codes; for the weights this is once per call instead of once per
// 256-token tile inside the contraction, and the 2 d_out d_in bytes it writes
// stay in L2 for the contraction that follows (oq_gemm_w16.cu).
#include <algorithm>

#include "oq_decode.cuh"
#include "oq_internal.h"

namespace oq {
namespace {

// K % 64 == 0: the rows of codes and of levels are both contiguous, so 8-value
// chunk i of the flat output is chunk i % CPP of flat code part i / CPP.  One
// chunk (16 output bytes) per thread and step: consecutive lanes write
// consecutive 16-byte pieces, and the CPP lanes of a part load the same bytes
// (one L1 line serves them).  Each thread takes UNROLL steps of the grid
// stride at a time and issues their loads before any decode, so that several
// loads per thread are in flight (one at a time left the kernel bound by
// load latency).
template <int BITS>
__global__ void __launch_bounds__(256) levels_flat_kernel(const uint32_t* __restrict__ codes, int64_t chunks,
                                                          uint4 tabv, DecK kc, const uint16_t* lut8_g,
                                                          uint4* __restrict__ out) {
  constexpr int UNROLL = 4;
  __shared__ uint16_t lut8[256];
  // a kernel launched as this one's programmatic dependent (the fused layer
  // kernel) may start now: it waits for this grid before it reads the levels
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if constexpr (BITS == 8) {
    for (int i = threadIdx.x; i < 256; i += blockDim.x) lut8[i] = lut8_g[i];
    __syncthreads();
  }
  const uint32_t t[4] = {tabv.x, tabv.y, tabv.z, tabv.w};
  constexpr int CPP = Fmt<BITS>::CPP;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i0 < chunks; i0 += UNROLL * stride) {
    uint4 v[UNROLL];
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      const int64_t i = i0 + u * stride;
      v[u] = make_uint4(0u, 0u, 0u, 0u);
      if (i < chunks) {
        const int64_t part = i / CPP;
        if constexpr (BITS == 3) {
          const uint32_t* pw = codes + part * 3;   // 32 codes in three words
          v[u] = make_uint4(__ldg(pw), __ldg(pw + 1), __ldg(pw + 2), 0u);
        } else {
          v[u] = __ldg(reinterpret_cast<const uint4*>(codes) + part);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      const int64_t i = i0 + u * stride;
      if (i < chunks) out[i] = decode_chunk_k<BITS>(v[u], (int)(i % CPP), t, lut8, kc);
    }
  }
}

// any K % 32 == 0 (a row may end in half a K block)
template <int BITS>
__global__ void __launch_bounds__(256) levels_kernel(const uint32_t* __restrict__ codes, int rows, int K, int wpr,
                                                     uint4 tabv, DecK kc, const uint16_t* lut8_g,
                                                     uint16_t* __restrict__ out) {
  __shared__ uint16_t lut8[256];
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if constexpr (BITS == 8) {
    for (int i = threadIdx.x; i < 256; i += blockDim.x) lut8[i] = lut8_g[i];
    __syncthreads();
  }
  const uint32_t t[4] = {tabv.x, tabv.y, tabv.z, tabv.w};
  constexpr int QP = Fmt<BITS>::QP, CPP = Fmt<BITS>::CPP;
  const int nkb = (K + DEC_BK - 1) / DEC_BK;
  const int cpr = nkb * QP * CPP;   // 8-value chunks per row, including any past K
  const int chunks = rows * cpr;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < chunks; i += gridDim.x * blockDim.x) {
    const int r = i / cpr, w = i - r * cpr;
    const int part = w / CPP, j = w - part * CPP;
    const int kb = part / QP, q = part - kb * QP;
    const int k = kb * DEC_BK + (q * CPP + j) * 8;
    if (k < K) {
      const uint4 v = load_part<BITS>(codes + (int64_t)r * wpr, kb, q, K);
      *reinterpret_cast<uint4*>(out + (int64_t)r * K + k) = decode_chunk_k<BITS>(v, j, t, lut8, kc);
    }
  }
}

template <int BITS>
oq_status levels_launch_t(const uint32_t* codes, int64_t rows, int K, const uint16_t* levels_host,
                          const uint16_t* levels_dev, uint16_t* out, void* stream) {
  uint32_t t[4] = {0u, 0u, 0u, 0u};
  make_decode_tables(BITS, levels_host, t);
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t chunks = rows * (int64_t)((K + DEC_BK - 1) / DEC_BK) * Fmt<BITS>::QP * Fmt<BITS>::CPP;
  const int64_t grid = std::max<int64_t>(1, std::min<int64_t>((chunks + 255) / 256, (int64_t)sms * 8));
  const uint4 tab = make_uint4(t[0], t[1], t[2], t[3]);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (K % DEC_BK == 0) {
    levels_flat_kernel<BITS><<<(unsigned)grid, 256, 0, st>>>(codes, chunks, tab, make_deck(), levels_dev,
                                                            reinterpret_cast<uint4*>(out));
  } else {
    if (chunks >= ((int64_t)1 << 31)) return OQ_ERR_UNSUPPORTED;   // 32-bit chunk indices
    levels_kernel<BITS><<<(unsigned)grid, 256, 0, st>>>(codes, (int)rows, K, K * BITS / 32, tab, make_deck(),
                                                       levels_dev, out);
  }
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error(std::string("levels launch: ") + cudaGetErrorString(e));
    return OQ_ERR_CUDA;
  }
  return OQ_OK;
}

}  // namespace

oq_status levels_launch(const uint32_t* codes, int64_t rows, int K, int bits, const uint16_t* levels_host,
                        const uint16_t* levels_dev, uint16_t* out, void* stream) {
  if (rows == 0) return OQ_OK;
  if (K % 32 != 0) return OQ_ERR_UNSUPPORTED;
  switch (bits) {
    case 2: return levels_launch_t<2>(codes, rows, K, levels_host, levels_dev, out, stream);
    case 3: return levels_launch_t<3>(codes, rows, K, levels_host, levels_dev, out, stream);
    case 4: return levels_launch_t<4>(codes, rows, K, levels_host, levels_dev, out, stream);
    case 8: return levels_launch_t<8>(codes, rows, K, levels_host, levels_dev, out, stream);
    default: return OQ_ERR_UNSUPPORTED;
  }
}

}  // namespace oq
