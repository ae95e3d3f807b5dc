// Code decoding shared by the codebook-contraction kernels: loading the packed
// codes of one K block of a row and expanding 8 codes into 8 fp16 values (one
// 16-byte chunk of a 128B-swizzled K-major operand tile) with byte-permute
// lookups into codebook tables held in registers.
#pragma once

#include <cstdint>

namespace oq {

constexpr int DEC_BK = 64;   // K elements per operand block (128 bytes of fp16)

// per bit width: 16-byte code parts per row per K block and 8-code chunks per part
template <int BITS> struct Fmt;
template <> struct Fmt<2> { static constexpr int QP = 1, CPP = 8; };
template <> struct Fmt<3> { static constexpr int QP = 2, CPP = 4; };
template <> struct Fmt<4> { static constexpr int QP = 2, CPP = 4; };
template <> struct Fmt<8> { static constexpr int QP = 4, CPP = 2; };

// the codes of part q of K block kb of a row (zeros past K)
template <int BITS>
__device__ __forceinline__ uint4 load_part(const uint32_t* row, int kb, int q, int K) {
  const int k0 = kb * DEC_BK + q * (DEC_BK / Fmt<BITS>::QP);
  if (k0 >= K) return make_uint4(0u, 0u, 0u, 0u);
  if constexpr (BITS == 3) {
    const uint32_t* p = row + kb * 6 + q * 3;
    return make_uint4(__ldg(p), __ldg(p + 1), __ldg(p + 2), 0u);
  } else if constexpr (BITS == 2) {
    // rows are only 8-byte aligned when K % 64 == 32
    const uint2* p = reinterpret_cast<const uint2*>(row + kb * 4);
    const uint2 lo = __ldg(p);
    const uint2 hi = (k0 + 32 < K) ? __ldg(p + 1) : make_uint2(0u, 0u);
    return make_uint4(lo.x, lo.y, hi.x, hi.y);
  } else {
    return __ldg(reinterpret_cast<const uint4*>(row) + kb * (BITS / 2) + q);
  }
}

// ---- 8 codes -> 8 fp16 (one 16-byte chunk of the operand tile)
__device__ __forceinline__ uint4 dec4(uint32_t w, const uint32_t (&t)[4]) {
  // symmetric codebook: code c >= 8 -> +P[c-8], c < 8 -> -P[7-c]
  const uint32_t n = ((~w) & 0x88888888u) >> 3;            // 1 per negative code
  const uint32_t m = (w & 0x77777777u) ^ (n * 7u);         // magnitude index
  const uint32_t mh = m >> 16, nh = n >> 16;
  const uint32_t lo_a = __byte_perm(t[0], t[1], m), hi_a = __byte_perm(t[2], t[3], m) | __byte_perm(0x8000u, 0u, n);
  const uint32_t lo_b = __byte_perm(t[0], t[1], mh), hi_b = __byte_perm(t[2], t[3], mh) | __byte_perm(0x8000u, 0u, nh);
  return make_uint4(__byte_perm(lo_a, hi_a, 0x5140), __byte_perm(lo_a, hi_a, 0x7362),
                    __byte_perm(lo_b, hi_b, 0x5140), __byte_perm(lo_b, hi_b, 0x7362));
}

__device__ __forceinline__ uint4 dec2(uint32_t x, const uint32_t (&t)[4]) {
  // 2-bit fields -> one selector nibble per code; 4-entry table in one register
  uint32_t y = (x | (x << 8)) & 0x00FF00FFu;
  y = (y | (y << 4)) & 0x0F0F0F0Fu;
  y = (y | (y << 2)) & 0x33333333u;
  const uint32_t yh = y >> 16;
  const uint32_t lo_a = __byte_perm(t[0], t[0], y), hi_a = __byte_perm(t[1], t[1], y);
  const uint32_t lo_b = __byte_perm(t[0], t[0], yh), hi_b = __byte_perm(t[1], t[1], yh);
  return make_uint4(__byte_perm(lo_a, hi_a, 0x5140), __byte_perm(lo_a, hi_a, 0x7362),
                    __byte_perm(lo_b, hi_b, 0x5140), __byte_perm(lo_b, hi_b, 0x7362));
}

__device__ __forceinline__ uint4 dec3(uint32_t x, const uint32_t (&t)[4]) {
  // 3-bit fields -> one selector nibble per code; 8-entry table in two registers
  uint32_t y = (x & 0xFFFu) | ((x & 0xFFF000u) << 4);
  y = (y & 0x003F003Fu) | ((y & 0x0FC00FC0u) << 2);
  y = (y & 0x07070707u) | ((y & 0x38383838u) << 1);
  const uint32_t yh = y >> 16;
  const uint32_t lo_a = __byte_perm(t[0], t[1], y), hi_a = __byte_perm(t[2], t[3], y);
  const uint32_t lo_b = __byte_perm(t[0], t[1], yh), hi_b = __byte_perm(t[2], t[3], yh);
  return make_uint4(__byte_perm(lo_a, hi_a, 0x5140), __byte_perm(lo_a, hi_a, 0x7362),
                    __byte_perm(lo_b, hi_b, 0x5140), __byte_perm(lo_b, hi_b, 0x7362));
}

__device__ __forceinline__ uint4 dec8(uint32_t w0, uint32_t w1, const uint16_t* lut) {
  auto pr = [&](uint32_t w, int b) {
    return (uint32_t)lut[(w >> (8 * b)) & 0xFF] | ((uint32_t)lut[(w >> (8 * b + 8)) & 0xFF] << 16);
  };
  return make_uint4(pr(w0, 0), pr(w0, 2), pr(w1, 0), pr(w1, 2));
}

// ---- the same decoders with their shifts and multiplies done as integer
// multiply-adds: the multipliers come from kernel parameters, so they stay
// opaque to the compiler and the work lands on the FMA pipe instead of the
// integer ALU pipe (where the byte permutes already queue).  x >> s is the high
// word of x * 2^(32-s); x << s is x * 2^s.
struct DecK {
  uint32_t hi16;   // 2^16: x >> 16 as a high multiply
  uint32_t hi29;   // 2^29: x >> 3
  uint32_t seven;  // 7
  uint32_t m256;   // 2^8
  uint32_t m16;    // 2^4
  uint32_t m4;     // 2^2
  uint32_t m2;     // 2^1
};

__host__ __forceinline__ DecK make_deck() { return DecK{1u << 16, 1u << 29, 7u, 256u, 16u, 4u, 2u}; }

__device__ __forceinline__ uint4 dec4k(uint32_t w, const uint32_t (&t)[4], const DecK& k) {
  const uint32_t n = (__umulhi(w, k.hi29) & 0x11111111u) ^ 0x11111111u;  // 1 per negative code (bit 3 clear)
  const uint32_t m = (w & 0x77777777u) ^ (n * k.seven);                   // magnitude index
  const uint32_t mh = __umulhi(m, k.hi16), nh = __umulhi(n, k.hi16);
  const uint32_t lo_a = __byte_perm(t[0], t[1], m), hi_a = __byte_perm(t[2], t[3], m) | __byte_perm(0x8000u, 0u, n);
  const uint32_t lo_b = __byte_perm(t[0], t[1], mh), hi_b = __byte_perm(t[2], t[3], mh) | __byte_perm(0x8000u, 0u, nh);
  return make_uint4(__byte_perm(lo_a, hi_a, 0x5140), __byte_perm(lo_a, hi_a, 0x7362),
                    __byte_perm(lo_b, hi_b, 0x5140), __byte_perm(lo_b, hi_b, 0x7362));
}

// x: 16 bits (eight 2-bit codes) in the low half
__device__ __forceinline__ uint4 dec2k(uint32_t x, const uint32_t (&t)[4], const DecK& k) {
  uint32_t y = (x | (x * k.m256)) & 0x00FF00FFu;
  y = (y | (y * k.m16)) & 0x0F0F0F0Fu;
  y = (y | (y * k.m4)) & 0x33333333u;
  const uint32_t yh = __umulhi(y, k.hi16);
  const uint32_t lo_a = __byte_perm(t[0], t[0], y), hi_a = __byte_perm(t[1], t[1], y);
  const uint32_t lo_b = __byte_perm(t[0], t[0], yh), hi_b = __byte_perm(t[1], t[1], yh);
  return make_uint4(__byte_perm(lo_a, hi_a, 0x5140), __byte_perm(lo_a, hi_a, 0x7362),
                    __byte_perm(lo_b, hi_b, 0x5140), __byte_perm(lo_b, hi_b, 0x7362));
}

// x: 24 bits (eight 3-bit codes) in the low three bytes
__device__ __forceinline__ uint4 dec3k(uint32_t x, const uint32_t (&t)[4], const DecK& k) {
  uint32_t y = (x & 0xFFFu) + (x & 0xFFF000u) * k.m16;
  y = (y & 0x003F003Fu) + (y & 0x0FC00FC0u) * k.m4;
  y = (y & 0x07070707u) + (y & 0x38383838u) * k.m2;
  const uint32_t yh = __umulhi(y, k.hi16);
  const uint32_t lo_a = __byte_perm(t[0], t[1], y), hi_a = __byte_perm(t[2], t[3], y);
  const uint32_t lo_b = __byte_perm(t[0], t[1], yh), hi_b = __byte_perm(t[2], t[3], yh);
  return make_uint4(__byte_perm(lo_a, hi_a, 0x5140), __byte_perm(lo_a, hi_a, 0x7362),
                    __byte_perm(lo_b, hi_b, 0x5140), __byte_perm(lo_b, hi_b, 0x7362));
}

template <int BITS>
__device__ __forceinline__ uint4 decode_chunk_k(const uint4& v, int j, const uint32_t (&t)[4], const uint16_t* lut8,
                                                const DecK& k) {
  if constexpr (BITS == 4) {
    const uint32_t w = j == 0 ? v.x : (j == 1 ? v.y : (j == 2 ? v.z : v.w));
    return dec4k(w, t, k);
  } else if constexpr (BITS == 2) {
    const uint32_t w = (j < 2) ? v.x : (j < 4 ? v.y : (j < 6 ? v.z : v.w));
    return dec2k((j & 1) ? __umulhi(w, k.hi16) : (w & 0xFFFFu), t, k);
  } else if constexpr (BITS == 3) {
    uint32_t x;
    if (j == 0) x = v.x & 0xFFFFFFu;
    else if (j == 1) x = ((v.x >> 24) | (v.y << 8)) & 0xFFFFFFu;
    else if (j == 2) x = ((v.y >> 16) | (v.z << 16)) & 0xFFFFFFu;
    else x = v.z >> 8;
    return dec3k(x, t, k);
  } else {
    return j == 0 ? dec8(v.x, v.y, lut8) : dec8(v.z, v.w, lut8);
  }
}

// ---- FP8 (e4m3) decode of 4-bit codes, for the lower-precision contraction
// mode: one byte per value, so a byte permute yields four values at once.
// t[0], t[1]: e4m3 bytes of the eight positive levels (magnitude index 0-7).
constexpr int DEC_BK_F8 = 128;   // K elements per operand block (128 bytes of e4m3)

__device__ __forceinline__ uint2 dec4_e4m3k(uint32_t w, const uint32_t (&t)[4], const DecK& k) {
  const uint32_t n = (__umulhi(w, k.hi29) & 0x11111111u) ^ 0x11111111u;  // 1 per negative code (bit 3 clear)
  const uint32_t m = (w & 0x77777777u) ^ (n * k.seven);                   // magnitude index
  const uint32_t mh = __umulhi(m, k.hi16), nh = __umulhi(n, k.hi16);
  return make_uint2(__byte_perm(t[0], t[1], m) | __byte_perm(0x8000u, 0u, n),
                    __byte_perm(t[0], t[1], mh) | __byte_perm(0x8000u, 0u, nh));
}

// the codes of part q (32 codes, 16 bytes) of FP8 K block kb of a 4-bit row (zeros past K)
__device__ __forceinline__ uint4 load_part_f8(const uint32_t* row, int kb, int q, int K) {
  if (kb * DEC_BK_F8 + q * 32 >= K) return make_uint4(0u, 0u, 0u, 0u);
  return __ldg(reinterpret_cast<const uint4*>(row) + kb * 4 + q);
}

// chunk j (16 codes -> 16 e4m3 bytes) of an FP8 part
__device__ __forceinline__ uint4 decode_chunk_f8(const uint4& v, int j, const uint32_t (&t)[4], const DecK& k) {
  const uint2 a = dec4_e4m3k(j == 0 ? v.x : v.z, t, k), b = dec4_e4m3k(j == 0 ? v.y : v.w, t, k);
  return make_uint4(a.x, a.y, b.x, b.y);
}

// chunk j of a part -> 8 fp16
template <int BITS>
__device__ __forceinline__ uint4 decode_chunk(const uint4& v, int j, const uint32_t (&t)[4], const uint16_t* lut8) {
  if constexpr (BITS == 4) {
    const uint32_t w = j == 0 ? v.x : (j == 1 ? v.y : (j == 2 ? v.z : v.w));
    return dec4(w, t);
  } else if constexpr (BITS == 2) {
    const uint32_t w = (j < 2) ? v.x : (j < 4 ? v.y : (j < 6 ? v.z : v.w));
    return dec2((j & 1) ? (w >> 16) : (w & 0xFFFFu), t);
  } else if constexpr (BITS == 3) {
    uint32_t x;
    if (j == 0) x = v.x & 0xFFFFFFu;
    else if (j == 1) x = ((v.x >> 24) | (v.y << 8)) & 0xFFFFFFu;
    else if (j == 2) x = ((v.y >> 16) | (v.z << 16)) & 0xFFFFFFu;
    else x = v.z >> 8;
    return dec3(x, t);
  } else {
    return j == 0 ? dec8(v.x, v.y, lut8) : dec8(v.z, v.w, lut8);
  }
}

// byte offset of 16-byte chunk `ch` of row `r` in a 128B-swizzled K-major tile
__device__ __forceinline__ uint32_t sw128_offset(int r, int ch) {
  return (uint32_t)((r >> 3) * 1024 + (r & 7) * 128 + ((ch ^ (r & 7)) << 4));
}

}  // namespace oq
