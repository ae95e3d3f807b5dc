// Rotate + quantize with the block Walsh-Hadamard transform on the tensor
// cores, for blocks of h = 1024 or 512 and bf16 activations, writing the fp16
// levels of the codes (the A operand of the fused layer call).  Same arithmetic
// contract as rq_kernel (gecl notes Method 1, 3, 4; pith Supplementary A):
//   s = ||x||_2,  y = P_pi x,  z_j = H_h y_j (block j, unnormalised),
//   code_i = #{k : t_k < z_i / (s sqrt(h))},  output fp16(a_scale C[code_i]).
//
// Sylvester's H_h is H_A (x) H_32 (A = h / 32 = 32 or 16): with a block
// viewed as an A x 32 matrix Y[a][b] = y[32 a + b], its transform is
// Z = H_A Y H_32.  One warp owns one block and computes it with two passes of
// warp-level MMAs:
//   pass 1: P^T = H_32 Y^T (m16n8k16, bf16 operands, fp32 accumulate).
//            The B operand is Y^T, gathered through pi straight into the
//            fragment registers: bf16 inputs and +-1 entries, so the
//            products are exact.
//   pass 2: Z = H_A P.  The accumulator layout of pass 1 already holds,
//            in every lane, the pairs of P that its pass-2 B fragments need,
//            so P never leaves the registers.  P is fp32; it enters as two
//            tf32 terms, hi = P with its low 13 mantissa bits cleared and
//            lo = P - hi (which the tensor core reads to 11 bits), so the
//            operand is P to 2^-20 of its value; both products accumulate
//            into the same fp32 result (m16n8k8 tf32 MMAs, whose K order is
//            chosen to match the pairs a lane holds).
// The norm comes from pass 1: sum P^2 = 32 sum y^2 per block.  Then every
// coordinate is quantized with the same bin-table search as rq_kernel and its
// fp16 level stored.  One CTA = d / h warps = one row at a time; rows
// stream through shared memory with double-buffered bulk copies.
#include <cuda_bf16.h>

#include <algorithm>
#include <cstring>

#include "oq_internal.h"
#include "oq_ptx.cuh"

namespace oq {

// Gather table of the tensor-core kernel (block size h, A = h / 32 values per
// lane): entry (w * 32 + lane) * A + e is the byte offset (2 x the input
// channel) of in-block position 32 a + b of block w in the staged bf16 row,
// with e = (kt * A / 8 + nt) * 4 + i, a = 8 nt + lane / 4 and
// b = 16 kt + 2 (lane % 4) + {0, 1, 8, 9}[i]: the order in which a lane fills
// its pass-1 B fragments.
void rqtc_build_gather(int d, int h, const std::vector<uint32_t>& perm, std::vector<uint16_t>& gather) {
  static const int boff[4] = {0, 1, 8, 9};
  const int A = h / 32, NT = A / 8;
  gather.assign((size_t)d, 0);
  for (int w = 0; w < d / h; ++w)
    for (int lane = 0; lane < 32; ++lane)
      for (int kt = 0; kt < 2; ++kt)
        for (int nt = 0; nt < NT; ++nt)
          for (int i = 0; i < 4; ++i) {
            const int a = 8 * nt + lane / 4, b = 16 * kt + 2 * (lane % 4) + boff[i];
            const int e = (kt * NT + nt) * 4 + i;
            gather[((size_t)w * 32 + lane) * A + e] = (uint16_t)(2 * perm[(size_t)w * h + 32 * a + b]);
          }
}

namespace {

struct TCParams {
  const void* src;     // [rows, d] bf16
  int64_t rows;
  int d, nw;           // nw = d / h warps per CTA
  int stage_bytes;     // per row buffer
  const uint16_t* gather;
  uint16_t* out16;     // fp16 levels [rows, d]
  float* norms;
  int* err;
  const uint2* bins;   // {threshold bits, fp16 level pair}
  int nb, b0;
  int full;            // the table spans every g of a token with a normal fp32 norm
  float kscale;
};

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

// A = rows of the block matrix (h / 32): NT1 = A / 8 pass-1 column tiles,
// MT2 = A / 16 pass-2 row tiles
template <int A>
__global__ void __launch_bounds__(A == 32 ? 256 : 1024) rqtc_kernel(const __grid_constant__ TCParams p) {
  constexpr int NT1 = A / 8, MT2 = A / 16, H = 32 * A;
  extern __shared__ __align__(128) unsigned char smem[];
  const int nw = p.nw, nthreads = nw * 32;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, q = lane & 3, g = lane >> 2;

  // shared memory: mbarriers | norm partials [2][32] | threshold table |
  // gather offsets [A / 8][threads] (uint4) | two row buffers
  uint64_t* mbar = reinterpret_cast<uint64_t*>(smem);
  float* red = reinterpret_cast<float*>(smem + 16);
  uint2* tbl = reinterpret_cast<uint2*>(smem + 272);
  const int gtab_off = (272 + 8 * p.nb + 15) & ~15;
  uint4* gtab = reinterpret_cast<uint4*>(smem + gtab_off);
  unsigned char* stage = smem + ((gtab_off + 2 * A * nthreads + 127) & ~127);
  const uint32_t stage_addr0 = smem_u32(stage);

  for (int i = tid; i < (A / 8) * nthreads; i += nthreads) {
    const int t = i % nthreads, qq = i / nthreads;
    gtab[i] = __ldg(reinterpret_cast<const uint4*>(p.gather) + (size_t)t * (A / 8) + qq);
  }
  for (int i = tid; i < p.nb; i += nthreads) tbl[i] = __ldg(p.bins + i);
  if (tid == 0) {
    mbar_init(&mbar[0], 1);
    mbar_init(&mbar[1], 1);
    fence_mbar_init();
  }
  __syncthreads();

  // A fragments of H_32 = [[H16, H16], [H16, -H16]]: rows g, g + 8 and
  // columns 2q, 2q + 1, 2q + 8, 2q + 9 of H16; tile (1, 1) is negated
  uint32_t hp[4], hn[4];
  hp[0] = hbit(g, 2 * q) | hbit(g, 2 * q + 1) << 16;
  hp[1] = hbit(g + 8, 2 * q) | hbit(g + 8, 2 * q + 1) << 16;
  hp[2] = hbit(g, 2 * q + 8) | hbit(g, 2 * q + 9) << 16;
  hp[3] = hbit(g + 8, 2 * q + 8) | hbit(g + 8, 2 * q + 9) << 16;
#pragma unroll
  for (int i = 0; i < 4; ++i) hn[i] = hp[i] ^ 0x80008000u;
  // pass 2 (tf32, K order of k-tile nt: k = q <-> a = 8 nt + 2q, k = q + 4
  // <-> a = 8 nt + 2q + 1): A[a'][k] = H_A[a'][a].  For rows a' = 16 mt + g
  // + 8 h the sign is sgn(g & a) times (-1)^(mt & nt >> 1) times (-1)^(h &
  // nt & 1), so four values cover every fragment.
  const uint32_t u = hbit32(g, 2 * q), v = hbit32(g, 2 * q + 1);
  const uint32_t un = u ^ 0x80000000u, vn = v ^ 0x80000000u;

  const uint32_t row_bytes = (uint32_t)p.d * 2u;
  const unsigned char* src = static_cast<const unsigned char*>(p.src);
  // bin search: t = g + (1.5 2^23 + b0) rounds g to an integer and offsets it
  // by b0, so bits(t) = 0x4B400000 + bin; the table address is taken from the
  // clamped bits directly
  const float magic = 12582912.0f + (float)p.b0;
  const int bin_lo = 0x4B400000, bin_hi = 0x4B400000 + p.nb - 1;
  const uint32_t tbl_shift = smem_u32(tbl) - 0x4B400000u * 8u;
  if (tid == 0 && (int64_t)blockIdx.x < p.rows) {
    mbar_arrive_expect_tx(&mbar[0], row_bytes);
    bulk_g2s(stage, src + (size_t)blockIdx.x * row_bytes, row_bytes, &mbar[0]);
  }

  int it = 0;
  for (int64_t t = blockIdx.x; t < p.rows; t += gridDim.x, ++it) {
    const int buf = it & 1;
    bool issued = false;
    if (tid == 0) {
      const int64_t tn = t + gridDim.x;
      if (tn < p.rows) {
        issued = true;
        mbar_arrive_expect_tx(&mbar[buf ^ 1], row_bytes);
        bulk_g2s(stage + (buf ^ 1) * p.stage_bytes, src + (size_t)tn * row_bytes, row_bytes, &mbar[buf ^ 1]);
      }
    }
    const bool ok = mbar_wait(&mbar[buf], (uint32_t)(it >> 1) & 1u, p.err);
    const uint32_t sa = stage_addr0 + (uint32_t)(buf * p.stage_bytes);

    // ---- gather through pi into pass-1 B fragments (bf16 pairs)
    uint32_t B1[2][NT1][2];
#pragma unroll
    for (int qq = 0; qq < A / 8; ++qq) {
      const uint4 gq = gtab[qq * nthreads + tid];
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
        for (int mt = 0; mt < 2; ++mt) mma_bf16_16816(D1[mt][nt], (mt & kt) ? hn : hp, B1[kt][nt][0], B1[kt][nt][1]);

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
    if (lane == 0) red[buf * 32 + warp] = ss;

    // ---- pass 2: Z = H_A P in tf32, P as hi + lo.  K tile nt of the
    // contraction over a takes a = 8 nt + 2q + {0, 1} from lane (g, q): the
    // pair D1[mt][nt][2h], D1[mt][nt][2h + 1] = P[8 nt + 2q + {0, 1}][16 mt + g
    // + 8 h] is the B fragment of (k tile nt, n tile 2 mt + h).
    float D2[MT2][4][4];
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
            const uint32_t a0 = na ? un : u, a1 = nh ? un : u, a2 = na ? vn : v, a3 = nh ? vn : v;
            mma_tf32_1688(D2[mt2][nt2], a0, a1, a2, a3, hi0, hi1);
            mma_tf32_1688(D2[mt2][nt2], a0, a1, a2, a3, __float_as_uint(lo0), __float_as_uint(lo1));
          }
        }

    // ---- norm across the row's blocks; every gather of this buffer is done
    const int failed = __syncthreads_or(!ok);
    if (failed) {
      if (issued) mbar_wait(&mbar[buf ^ 1], (uint32_t)((it + 1) >> 1) & 1u, p.err);
      break;
    }
    float s2 = 0.f;
    for (int w = 0; w < nw; ++w) s2 += red[buf * 32 + w];
    const float s = sqrtf(s2 * (1.0f / 32.0f));

    // ---- quantize: Z[a'][b'] for a' = 16 mt + g + 8 half, b' = 8 nt + 2q + {0, 1}
    // (the bin-table search of rq_kernel), fp16 level pairs stored as words
    const float ks = (s > 0.f) ? p.kscale / s : 0.f;
    uint16_t* rowout = p.out16 + (size_t)t * p.d + (size_t)warp * H + 2 * q;
    // With a full-range table every finite g of a token whose squared norm is
    // a normal fp32 number lies inside it (|g| <= K sqrt(d) up to rounding),
    // so the bin index needs no clamp.  Other tokens (a norm that under- or
    // overflowed in fp32, non-finite values, zero) take the clamped search.
    if (p.full && s2 >= 1e-30f && s2 <= 1e30f)
      quantize_store<false, MT2>(D2, ks, magic, bin_lo, bin_hi, tbl_shift, rowout, g);
    else
      quantize_store<true, MT2>(D2, ks, magic, bin_lo, bin_hi, tbl_shift, rowout, g);
    if (tid == 0) p.norms[t] = s;
  }
}

}  // namespace

bool rqtc_supported(const RQArgs& a) {
  return a.out16 && (a.h == 1024 || a.h == 512) && a.src_dtype == OQ_DTYPE_BF16 && !a.signmask && a.gather_tc &&
         a.d % a.h == 0 && a.d / a.h >= 1 && a.d / a.h <= (a.h == 1024 ? 8 : 32) && a.nb >= 1 &&
         a.nb <= OQ_MAX_BINS;
}

template <int A>
static oq_status rqtc_launch_t(const TCParams& p, void* stream) {
  const int threads = p.nw * 32;
  const size_t gtab_off = (272 + 8 * (size_t)p.nb + 15) & ~(size_t)15;
  const size_t smem = ((gtab_off + 2 * A * (size_t)threads + 127) & ~(size_t)127) + 2 * (size_t)p.stage_bytes;
  if (smem > 227 * 1024) return OQ_ERR_UNSUPPORTED;
  auto kern = rqtc_kernel<A>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
  if (e != cudaSuccess) {
    set_error(std::string("cudaFuncSetAttribute: ") + cudaGetErrorString(e));
    return OQ_ERR_CUDA;
  }
  int dev = 0, sms = 0, per_sm = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, smem);
  if (per_sm < 1) per_sm = 1;
  const int64_t grid = std::min<int64_t>(p.rows, (int64_t)sms * per_sm);
  kern<<<(unsigned)grid, threads, smem, static_cast<cudaStream_t>(stream)>>>(p);
  e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error(std::string("rotate_quantize (tensor-core FWHT) launch: ") + cudaGetErrorString(e));
    return OQ_ERR_CUDA;
  }
  return OQ_OK;
}

oq_status rqtc_launch(const RQArgs& a, void* stream) {
  if (a.rows == 0) return OQ_OK;
  if (!rqtc_supported(a)) return OQ_ERR_UNSUPPORTED;
  TCParams p;
  std::memset(&p, 0, sizeof(p));
  p.src = a.src;
  p.rows = a.rows;
  p.d = a.d;
  p.nw = a.d / a.h;
  p.stage_bytes = (a.d * 2 + 127) & ~127;
  p.gather = a.gather_tc;
  p.out16 = a.out16;
  p.norms = a.norms;
  p.err = a.err;
  if (a.bins_full) {
    p.bins = reinterpret_cast<const uint2*>(a.bins_full);
    p.nb = a.nb_full;
    p.b0 = a.b0_full;
    p.full = 1;
  } else {
    p.bins = reinterpret_cast<const uint2*>(a.bins);
    p.nb = a.nb;
    p.b0 = a.b0;
  }
  p.kscale = a.kscale;
  return a.h == 1024 ? rqtc_launch_t<32>(p, stream) : rqtc_launch_t<16>(p, stream);
}

}  // namespace oq
