// Device code of the tensor-core rotate-quantize step, shared by the
// stand-alone kernel (oq_rotate_quantize_tc.cu) and the fused layer kernel
// (oq_fused.cu): the block Walsh-Hadamard transform of one block of h = 32 A
// positions of a staged bf16 row as two passes of warp MMAs, and the
// bin-table quantizer writing fp16 levels.  The math is described in
// oq_rotate_quantize_tc.cu (gecl notes Method 3 and 4; pith Supplementary A).
#pragma once

#include <cstdint>

#include "oq_ptx.cuh"

namespace oq {
namespace rqtc {

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_tf32_1688(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                              uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// (a0, a1) * (k, k) + (c, c) on the paired fp32 pipe, in two rounded steps
// (a product, then a sum), as mul.f32x2 and add.f32x2
__device__ __forceinline__ void mul2(float& r0, float& r1, float a0, float a1, float k) {
  asm("{\n\t.reg .b64 A, K, R;\n\tmov.b64 A, {%2, %3};\n\tmov.b64 K, {%4, %4};\n\t"
      "mul.rn.f32x2 R, A, K;\n\tmov.b64 {%0, %1}, R;\n\t}"
      : "=f"(r0), "=f"(r1)
      : "f"(a0), "f"(a1), "f"(k));
}
__device__ __forceinline__ void add2(float& r0, float& r1, float a0, float a1, float c) {
  asm("{\n\t.reg .b64 A, C, R;\n\tmov.b64 A, {%2, %3};\n\tmov.b64 C, {%4, %4};\n\t"
      "add.rn.f32x2 R, A, C;\n\tmov.b64 {%0, %1}, R;\n\t}"
      : "=f"(r0), "=f"(r1)
      : "f"(a0), "f"(a1), "f"(c));
}
__device__ __forceinline__ void sub2(float& r0, float& r1, float a0, float a1, float b0, float b1) {
  asm("{\n\t.reg .b64 A, B, R;\n\tmov.b64 A, {%2, %3};\n\tmov.b64 B, {%4, %5};\n\t"
      "sub.rn.f32x2 R, A, B;\n\tmov.b64 {%0, %1}, R;\n\t}"
      : "=f"(r0), "=f"(r1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

// all ones when a > b, else zero
__device__ __forceinline__ uint32_t gt_mask(float a, float b) {
  uint32_t r;
  asm("set.gt.u32.f32 %0, %1, %2;" : "=r"(r) : "f"(a), "f"(b));
  return r;
}

__device__ __forceinline__ uint2 lds_v2(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
  return v;
}

// s += a0 * a0 + a1 * a1 on the paired fp32 pipe
__device__ __forceinline__ void sumsq2(float& s0, float& s1, float a0, float a1) {
  asm("{\n\t.reg .b64 A, S;\n\tmov.b64 A, {%2, %3};\n\tmov.b64 S, {%0, %1};\n\t"
      "fma.rn.f32x2 S, A, A, S;\n\tmov.b64 {%0, %1}, S;\n\t}"
      : "+f"(s0), "+f"(s1)
      : "f"(a0), "f"(a1));
}

__device__ __forceinline__ uint32_t hbit(int r, int c) { return (__popc(r & c) & 1) ? 0xBF80u : 0x3F80u; }
__device__ __forceinline__ uint32_t hbit32(int r, int c) { return (__popc(r & c) & 1) ? 0xBF800000u : 0x3F800000u; }

// Quantizes the warp's A x 32 block Z (pass-2 accumulators: rows a' =
// 16 mt + g + 8 half, columns b' = 8 nt + 2q + {0, 1}) with the bin table and
// stores the fp16 level pairs as words of the output row.
template <bool CLAMP, int MT2>
__device__ __forceinline__ void quantize_store(const float (&D2)[MT2][4][4], float ks, float magic, int bin_lo,
                                               int bin_hi, uint32_t tbl_shift, uint16_t* rowout, int g) {
#pragma unroll
  for (int mt = 0; mt < MT2; ++mt)
#pragma unroll
    for (int half = 0; half < 2; ++half)
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) {
        float g0, g1, t0, t1;
        mul2(g0, g1, D2[mt][nt][2 * half], D2[mt][nt][2 * half + 1], ks);
        add2(t0, t1, g0, g1, magic);
        int m0 = __float_as_int(t0), m1 = __float_as_int(t1);
        if (CLAMP) {
          m0 = min(max(m0, bin_lo), bin_hi);
          m1 = min(max(m1, bin_lo), bin_hi);
        }
        const uint2 e0 = lds_v2(tbl_shift + 8u * (uint32_t)m0);
        const uint2 e1 = lds_v2(tbl_shift + 8u * (uint32_t)m1);
        // byte selector: bytes 0-1 from e0's level pair (upper level if g0 is
        // above the bin's threshold), bytes 2-3 likewise from e1's
        const uint32_t sel = 0x5410u | (gt_mask(g0, __uint_as_float(e0.x)) & 0x22u) |
                             (gt_mask(g1, __uint_as_float(e1.x)) & 0x2200u);
        const int a = 16 * mt + g + 8 * half;
        *reinterpret_cast<uint32_t*>(rowout + 32 * a + 8 * nt) = __byte_perm(e0.y, e1.y, sel);
      }
}

// The same quantization writing packed codes (the format of oq_rotate_quantize:
// each group of 32 positions is a little-endian stream of 32 BITS bits in BITS
// words).  Row a' of the block is positions [32 a', 32 a' + 32): one group.
// A lane holds 8 of its codes (positions 8 nt + 2q + {0, 1}), placed at bits
// BITS (8 nt + 2q + j) of the group's stream; the four lanes of the quad OR
// their words together and lane q stores words q, q + 4 (BITS words in all,
// one 4 BITS-byte run per group).  `grp` points to group 0 of the block.
template <bool CLAMP, int MT2, int BITS>
__device__ __forceinline__ void quantize_store_codes(const float (&D2)[MT2][4][4], float ks, float magic, int bin_lo,
                                                     int bin_hi, uint32_t tbl_shift, uint32_t* grp, int g, int q) {
#pragma unroll
  for (int mt = 0; mt < MT2; ++mt)
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      uint32_t w[BITS];
#pragma unroll
      for (int i = 0; i < BITS; ++i) w[i] = 0u;
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) {
        float g0, g1, t0, t1;
        mul2(g0, g1, D2[mt][nt][2 * half], D2[mt][nt][2 * half + 1], ks);
        add2(t0, t1, g0, g1, magic);
        int m0 = __float_as_int(t0), m1 = __float_as_int(t1);
        if (CLAMP) {
          m0 = min(max(m0, bin_lo), bin_hi);
          m1 = min(max(m1, bin_lo), bin_hi);
        }
        const uint2 e0 = lds_v2(tbl_shift + 8u * (uint32_t)m0);
        const uint2 e1 = lds_v2(tbl_shift + 8u * (uint32_t)m1);
        // code = the bin's base code, plus one above the bin's threshold
        const uint32_t c0 = e0.y + (g0 > __uint_as_float(e0.x) ? 1u : 0u);
        const uint32_t c1 = e1.y + (g1 > __uint_as_float(e1.x) ? 1u : 0u);
        // both codes of the pair: 2 BITS bits starting at bit BITS (8 nt + 2q)
        const uint32_t pair = c0 | (c1 << BITS);
        const int bit = BITS * (8 * nt + 2 * q);
#pragma unroll
        for (int i = 0; i < BITS; ++i) {
          const int lo = bit - 32 * i;     // the pair's offset within word i
          if (lo >= 0 && lo < 32) w[i] |= pair << lo;
          if (lo < 0 && lo > -2 * BITS) w[i] |= pair >> (-lo);
        }
      }
#pragma unroll
      for (int i = 0; i < BITS; ++i) {
        w[i] |= __shfl_xor_sync(0xffffffffu, w[i], 1);
        w[i] |= __shfl_xor_sync(0xffffffffu, w[i], 2);
      }
      uint32_t* out = grp + (16 * mt + g + 8 * half) * BITS;
#pragma unroll
      for (int i = 0; i < BITS; ++i)
        if ((i & 3) == q) out[i] = w[i];
    }
}

// Per-lane constants of the two passes: the pass-1 A fragments of H_32 (hp,
// and hn = the negated tile) and the four values that make up every pass-2 A
// fragment of H_A.
struct Lane {
  uint32_t hp[4], hn[4];
  uint32_t u, v, un, vn;
};

__device__ __forceinline__ Lane make_lane(int lane) {
  const int q = lane & 3, g = lane >> 2;
  Lane c;
  // A fragments of H_32 = [[H16, H16], [H16, -H16]]: rows g, g + 8 and
  // columns 2q, 2q + 1, 2q + 8, 2q + 9 of H16; tile (1, 1) is negated
  c.hp[0] = hbit(g, 2 * q) | hbit(g, 2 * q + 1) << 16;
  c.hp[1] = hbit(g + 8, 2 * q) | hbit(g + 8, 2 * q + 1) << 16;
  c.hp[2] = hbit(g, 2 * q + 8) | hbit(g, 2 * q + 9) << 16;
  c.hp[3] = hbit(g + 8, 2 * q + 8) | hbit(g + 8, 2 * q + 9) << 16;
#pragma unroll
  for (int i = 0; i < 4; ++i) c.hn[i] = c.hp[i] ^ 0x80008000u;
  // pass 2 (tf32, K order of k-tile nt: k = q <-> a = 8 nt + 2q, k = q + 4
  // <-> a = 8 nt + 2q + 1): A[a'][k] = H_A[a'][a].  For rows a' = 16 mt + g
  // + 8 h the sign is sgn(g & a) times (-1)^(mt & nt >> 1) times (-1)^(h &
  // nt & 1), so four values cover every fragment.
  c.u = hbit32(g, 2 * q);
  c.v = hbit32(g, 2 * q + 1);
  c.un = c.u ^ 0x80000000u;
  c.vn = c.v ^ 0x80000000u;
  return c;
}

// The transform of one block (A x 32 positions) of the row staged at shared
// address `sa`: gather through pi (offsets from the transposed table `gtab`,
// entry qq * gstride + gidx), pass 1, pass 2.  D2 receives Z = H_A Y H_32
// (unnormalised); the return value is this lane's share of sum P^2 =
// 32 sum y^2 over the block, reduced over the warp (every lane gets it).
template <int A>
__device__ __forceinline__ float transform_block(const Lane& c, const uint4* gtab, int gstride, int gidx,
                                                 uint32_t sa, float (&D2)[A / 16][4][4]) {
  constexpr int NT1 = A / 8, MT2 = A / 16;
  // ---- gather through pi into pass-1 B fragments (bf16 pairs)
  uint32_t B1[2][NT1][2];
#pragma unroll
  for (int qq = 0; qq < A / 8; ++qq) {
    const uint4 gq = gtab[qq * gstride + gidx];
    const uint32_t gw[4] = {gq.x, gq.y, gq.z, gq.w};
#pragma unroll
    for (int hpair = 0; hpair < 4; ++hpair) {
      uint16_t v0, v1;
      asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v0) : "r"(sa + (gw[hpair] & 0xFFFFu)));
      asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v1) : "r"(sa + (gw[hpair] >> 16)));
      // slots e = 8 qq + 2 hpair, +1: (kt, nt) = divmod(2 qq + hpair / 2, NT1), register hpair % 2
      const int kn = 2 * qq + (hpair >> 1), kt = kn / NT1, nt = kn % NT1;
      B1[kt][nt][hpair & 1] = (uint32_t)v0 | ((uint32_t)v1 << 16);
    }
  }

  // ---- pass 1: P^T = H_32 Y^T (rows b', columns a)
  float D1[2][NT1][4];
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int nt = 0; nt < NT1; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) D1[mt][nt][i] = 0.f;
#pragma unroll
  for (int kt = 0; kt < 2; ++kt)
#pragma unroll
    for (int nt = 0; nt < NT1; ++nt)
#pragma unroll
      for (int mt = 0; mt < 2; ++mt) mma_bf16_16816(D1[mt][nt], (mt & kt) ? c.hn : c.hp, B1[kt][nt][0], B1[kt][nt][1]);

  // norm partial: sum P^2 = 32 sum y^2 over the block
  float ss0 = 0.f, ss1 = 0.f;
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int nt = 0; nt < NT1; ++nt) {
      sumsq2(ss0, ss1, D1[mt][nt][0], D1[mt][nt][1]);
      sumsq2(ss0, ss1, D1[mt][nt][2], D1[mt][nt][3]);
    }
  float ss = ss0 + ss1;
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);

  // ---- pass 2: Z = H_A P in tf32, P as hi + lo.  K tile nt of the
  // contraction over a takes a = 8 nt + 2q + {0, 1} from lane (g, q): the
  // pair D1[mt][nt][2h], D1[mt][nt][2h + 1] = P[8 nt + 2q + {0, 1}][16 mt + g
  // + 8 h] is the B fragment of (k tile nt, n tile 2 mt + h).
#pragma unroll
  for (int mt = 0; mt < MT2; ++mt)
#pragma unroll
    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) D2[mt][nt][i] = 0.f;
#pragma unroll
  for (int nt = 0; nt < NT1; ++nt)
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const float x0 = D1[mt][nt][2 * h], x1 = D1[mt][nt][2 * h + 1];
        const uint32_t hi0 = __float_as_uint(x0) & 0xFFFFE000u, hi1 = __float_as_uint(x1) & 0xFFFFE000u;
        float lo0, lo1;
        sub2(lo0, lo1, x0, x1, __uint_as_float(hi0), __uint_as_float(hi1));
        const int nt2 = 2 * mt + h;
#pragma unroll
        for (int mt2 = 0; mt2 < MT2; ++mt2) {
          const bool na = mt2 & (nt >> 1), nh = na ^ (nt & 1);
          const uint32_t a0 = na ? c.un : c.u, a1 = nh ? c.un : c.u, a2 = na ? c.vn : c.v, a3 = nh ? c.vn : c.v;
          mma_tf32_1688(D2[mt2][nt2], a0, a1, a2, a3, hi0, hi1);
          mma_tf32_1688(D2[mt2][nt2], a0, a1, a2, a3, __float_as_uint(lo0), __float_as_uint(lo1));
        }
      }
  return ss;
}

}  // namespace rqtc
}  // namespace oq
