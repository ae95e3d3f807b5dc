// Device code of rotate-quantize with the block Walsh-Hadamard transform on
// the CUDA cores, for blocks of h = 1024 (gecl notes Method 3 and 4; pith
// Supplementary A).  Sylvester's H_1024 is H_32 (x) H_32: with the block viewed
// as a 32 x 32 matrix Y[a][b] = y[32 a + b], its transform is Z = H_32 Y H_32.
// One warp owns one block:
//   - lane l gathers column b = l through pi (32 values Y[a][l]);
//   - H_32 over a in registers (five butterfly stages, fp32);
//   - the 32 x 32 tile goes through the warp's shared-memory tile (columns
//     written, rows read back; 16-byte chunks XOR-swizzled so that both
//     directions are free of bank conflicts);
//   - H_32 over b in registers: lane l then holds Z[l][0..31], the 32
//     consecutive positions 32 l .. 32 l + 31 of the block -- one code group.
// No tensor-core instruction is used, so the transform can run beside tcgen05
// contractions without waiting on them.  Each output lane then quantizes its
// group with the bin-table search and writes either the group's fp16 levels
// (64 contiguous bytes) or its packed codes (4 BITS contiguous bytes).
#pragma once

#include <cstdint>

#include "oq_ptx.cuh"

namespace oq {
namespace rqcc {

// (a0, a1), (b0, b1) -> (a0 + b0, a1 + b1), (a0 - b0, a1 - b1) on the paired
// fp32 pipe (add.f32x2 / sub.f32x2: each lane of the pair rounds as a scalar
// add or subtract would)
__device__ __forceinline__ void bfly2(float& a0, float& a1, float& b0, float& b1) {
  asm("{\n\t.reg .b64 A, B, S, D;\n\tmov.b64 A, {%0, %1};\n\tmov.b64 B, {%2, %3};\n\t"
      "add.rn.f32x2 S, A, B;\n\tsub.rn.f32x2 D, A, B;\n\tmov.b64 {%0, %1}, S;\n\tmov.b64 {%2, %3}, D;\n\t}"
      : "+f"(a0), "+f"(a1), "+f"(b0), "+f"(b1));
}

// in-register butterflies on v[0..32): stride S pairs (i, i + S) for i & S == 0;
// from stride 2 on, the pairs (i, i + S) and (i + 1, i + S + 1) go together
template <int S>
__device__ __forceinline__ void stage(float (&v)[32]) {
  if constexpr (S >= 2) {
#pragma unroll
    for (int i = 0; i < 32; i += 2)
      if ((i & S) == 0) bfly2(v[i], v[i + 1], v[i + S], v[i + S + 1]);
  } else {
#pragma unroll
    for (int i = 0; i < 32; ++i)
      if ((i & S) == 0) {
        const float a = v[i], b = v[i + S];
        v[i] = a + b;
        v[i + S] = a - b;
      }
  }
}

__device__ __forceinline__ void fwht32(float (&v)[32]) {
  stage<16>(v);
  stage<8>(v);
  stage<4>(v);
  stage<2>(v);
  stage<1>(v);
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// The transform of one block of the row staged at shared address `sa`.
// gtab: the gather table, entry qq * gstride + gidx holds the byte offsets of
// Y[8 qq .. 8 qq + 7][lane] as eight uint16; tile: this warp's 32 x 32 fp32
// shared-memory tile (4 KB, 16-byte aligned).  Returns this block's sum of y^2
// reduced over the warp; z receives Z[lane][0..31].
__device__ __forceinline__ float transform_block(const uint4* gtab, int gstride, int gidx, uint32_t sa, float* tile,
                                                 int lane, float (&z)[32]) {
  float v[32];
#pragma unroll
  for (int qq = 0; qq < 4; ++qq) {
    const uint4 gq = gtab[qq * gstride + gidx];
    const uint32_t gw[4] = {gq.x, gq.y, gq.z, gq.w};
#pragma unroll
    for (int hp = 0; hp < 4; ++hp) {
      uint16_t v0, v1;
      asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v0) : "r"(sa + (gw[hp] & 0xFFFFu)));
      asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v1) : "r"(sa + (gw[hp] >> 16)));
      v[8 * qq + 2 * hp] = __uint_as_float((uint32_t)v0 << 16);
      v[8 * qq + 2 * hp + 1] = __uint_as_float((uint32_t)v1 << 16);
    }
  }
  float ss0 = 0.f, ss1 = 0.f;
#pragma unroll
  for (int i = 0; i < 32; i += 2) {
    ss0 = fmaf(v[i], v[i], ss0);
    ss1 = fmaf(v[i + 1], v[i + 1], ss1);
  }
  float ss = ss0 + ss1;
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);

  // H_32 over a: v[a] = sum_a' H[a][a'] Y[a'][lane]
  fwht32(v);
  // column `lane` of the tile as row `lane` of its transpose Qt[b][a]: chunk c
  // (a = 4c .. 4c + 3) at chunk position c ^ (lane & 7)
  const uint32_t base = smem_u32(tile);
#pragma unroll
  for (int c = 0; c < 8; ++c)
    st_shared_v4(base + (uint32_t)(lane * 128 + ((c ^ (lane & 7)) << 4)),
                 make_uint4(__float_as_uint(v[4 * c]), __float_as_uint(v[4 * c + 1]), __float_as_uint(v[4 * c + 2]),
                            __float_as_uint(v[4 * c + 3])));
  __syncwarp();
  // row a = lane: Qt[b][lane] for b = 0..31
#pragma unroll
  for (int b = 0; b < 32; ++b) {
    float x;
    asm volatile("ld.shared.f32 %0, [%1];"
                 : "=f"(x)
                 : "r"(base + (uint32_t)(b * 128 + ((((lane >> 2) ^ (b & 7))) << 4) + ((lane & 3) << 2))));
    z[b] = x;
  }
  __syncwarp();   // the tile is free for this warp's next block
  fwht32(z);
  return ss;
}

// Quantizes this lane's 32 consecutive values and writes their fp16 levels:
// table entries {threshold bits, fp16 level of the lower | upper code << 16}.
template <bool CLAMP>
__device__ __forceinline__ void quantize_levels(const float (&z)[32], float ks, float magic, int bin_lo, int bin_hi,
                                                uint32_t tbl_shift, uint16_t* out) {
  uint32_t w[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float g0 = z[2 * i] * ks, g1 = z[2 * i + 1] * ks;
    int m0 = __float_as_int(g0 + magic), m1 = __float_as_int(g1 + magic);
    if (CLAMP) {
      m0 = min(max(m0, bin_lo), bin_hi);
      m1 = min(max(m1, bin_lo), bin_hi);
    }
    uint2 e0, e1;
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(e0.x), "=r"(e0.y) : "r"(tbl_shift + 8u * (uint32_t)m0));
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(e1.x), "=r"(e1.y) : "r"(tbl_shift + 8u * (uint32_t)m1));
    const uint32_t sel = 0x5410u | (g0 > __uint_as_float(e0.x) ? 0x22u : 0u) | (g1 > __uint_as_float(e1.x) ? 0x2200u : 0u);
    w[i] = __byte_perm(e0.y, e1.y, sel);
  }
  uint4* o = reinterpret_cast<uint4*>(out);
#pragma unroll
  for (int i = 0; i < 4; ++i) o[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
}

// The same search writing the group's packed codes (BITS words): table
// entries {threshold bits, base code}
template <bool CLAMP, int BITS>
__device__ __forceinline__ void quantize_codes(const float (&z)[32], float ks, float magic, int bin_lo, int bin_hi,
                                               uint32_t tbl_shift, uint32_t* out) {
  uint32_t w[BITS];
#pragma unroll
  for (int i = 0; i < BITS; ++i) w[i] = 0u;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const float gv = z[i] * ks;
    int m = __float_as_int(gv + magic);
    if (CLAMP) m = min(max(m, bin_lo), bin_hi);
    uint2 e;
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(e.x), "=r"(e.y) : "r"(tbl_shift + 8u * (uint32_t)m));
    const uint32_t c = e.y + (gv > __uint_as_float(e.x) ? 1u : 0u);
    const int bit = BITS * i;
    w[bit >> 5] |= c << (bit & 31);
    if ((bit & 31) + BITS > 32) w[(bit >> 5) + 1] |= c >> (32 - (bit & 31));
  }
  if constexpr (BITS == 4) {
    *reinterpret_cast<uint4*>(out) = make_uint4(w[0], w[1], w[2], w[3]);
  } else if constexpr (BITS == 8) {
    reinterpret_cast<uint4*>(out)[0] = make_uint4(w[0], w[1], w[2], w[3]);
    reinterpret_cast<uint4*>(out)[1] = make_uint4(w[4], w[5], w[6], w[7]);
  } else if constexpr (BITS == 2) {
    *reinterpret_cast<uint2*>(out) = make_uint2(w[0], w[1]);
  } else {
#pragma unroll
    for (int i = 0; i < BITS; ++i) out[i] = w[i];
  }
}

}  // namespace rqcc
}  // namespace oq
