// The contraction epilogue's last step, shared by the CTA-pair kernels: one
// 32-row x 32-column chunk of the accumulator, already read from tensor
// memory (this lane's row in v), is scaled to y = acc * s_row * r[col] (the
// magnitudes restored, gecl notes Method 1) and staged in shared memory in
// the layout of a TMA store box:
//   fp32 y: rows of 128 bytes, 16-byte chunks in the 128-byte swizzle
//           (chunk c of row l at c ^ (l % 8));
//   bf16 y: rows of 64 bytes (round to nearest even), chunks in the 64-byte
//           swizzle (chunk c of row l at c ^ ((l / 2) % 4)).
// Both are conflict-free for the warp's vector stores.
#pragma once

#include <cuda_bf16.h>

#include <cstdint>

#include "oq_ptx.cuh"

namespace oq {

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&b);
}

__device__ __forceinline__ void stage_y_chunk(const uint32_t (&v)[32], float srow, const float* rcol, uint32_t buf,
                                              int lane, bool bf16) {
  if (!bf16) {
    const uint32_t rb = buf + (uint32_t)lane * 128u;
#pragma unroll
    for (int k4 = 0; k4 < 8; ++k4) {
      const float4 rr = __ldg(reinterpret_cast<const float4*>(rcol) + k4);
      uint4 o;
      o.x = __float_as_uint(__uint_as_float(v[4 * k4 + 0]) * srow * rr.x);
      o.y = __float_as_uint(__uint_as_float(v[4 * k4 + 1]) * srow * rr.y);
      o.z = __float_as_uint(__uint_as_float(v[4 * k4 + 2]) * srow * rr.z);
      o.w = __float_as_uint(__uint_as_float(v[4 * k4 + 3]) * srow * rr.w);
      st_shared_v4(rb + ((uint32_t)(k4 ^ (lane & 7)) << 4), o);
    }
  } else {
    const uint32_t rb = buf + (uint32_t)lane * 64u;
#pragma unroll
    for (int k8 = 0; k8 < 4; ++k8) {
      const float4 r0 = __ldg(reinterpret_cast<const float4*>(rcol) + 2 * k8);
      const float4 r1 = __ldg(reinterpret_cast<const float4*>(rcol) + 2 * k8 + 1);
      const uint32_t* w = v + 8 * k8;
      uint4 o;
      o.x = pack_bf16x2(__uint_as_float(w[0]) * srow * r0.x, __uint_as_float(w[1]) * srow * r0.y);
      o.y = pack_bf16x2(__uint_as_float(w[2]) * srow * r0.z, __uint_as_float(w[3]) * srow * r0.w);
      o.z = pack_bf16x2(__uint_as_float(w[4]) * srow * r1.x, __uint_as_float(w[5]) * srow * r1.y);
      o.w = pack_bf16x2(__uint_as_float(w[6]) * srow * r1.z, __uint_as_float(w[7]) * srow * r1.w);
      st_shared_v4(rb + ((uint32_t)(k8 ^ ((lane >> 1) & 3)) << 4), o);
    }
  }
}

}  // namespace oq
