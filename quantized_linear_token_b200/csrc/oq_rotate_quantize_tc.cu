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
#include "oq_rqtc_dev.cuh"

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
  uint16_t* out16;     // fp16 levels [rows, d], or
  uint32_t* codes;     // packed codes [rows, d * bits / 32]
  int bits;
  float* norms;
  int* err;
  const uint2* bins;   // {threshold bits, fp16 level pair} (or {threshold bits, base code} for codes)
  int nb, b0;
  int full;            // the table spans every g of a token with a normal fp32 norm
  float kscale;
};

// packed-code output at the layer's activation width
template <int MT2>
__device__ __forceinline__ void store_codes(int bits, bool unclamped, const float (&D2)[MT2][4][4], float ks,
                                            float magic, int bin_lo, int bin_hi, uint32_t tbl_shift, uint32_t* grp,
                                            int g, int q) {
#define OQ_STORE_CODES(B)                                                                                  \
  if (unclamped)                                                                                           \
    rqtc::quantize_store_codes<false, MT2, B>(D2, ks, magic, bin_lo, bin_hi, tbl_shift, grp, g, q);         \
  else                                                                                                     \
    rqtc::quantize_store_codes<true, MT2, B>(D2, ks, magic, bin_lo, bin_hi, tbl_shift, grp, g, q);
  switch (bits) {
    case 2: OQ_STORE_CODES(2) break;
    case 3: OQ_STORE_CODES(3) break;
    case 4: OQ_STORE_CODES(4) break;
    default: OQ_STORE_CODES(8) break;
  }
#undef OQ_STORE_CODES
}

// A = rows of the block matrix (h / 32): MT2 = A / 16 pass-2 row tiles
template <int A>
__global__ void __launch_bounds__(A == 32 ? 256 : 1024) rqtc_kernel(const __grid_constant__ TCParams p) {
  constexpr int MT2 = A / 16, H = 32 * A;
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

  const rqtc::Lane lc = rqtc::make_lane(lane);

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

    // ---- gather, pass 1, norm partial, pass 2 (oq_rqtc_dev.cuh)
    float D2[MT2][4][4];
    const float ss = rqtc::transform_block<A>(lc, gtab, nthreads, tid, sa, D2);
    if (lane == 0) red[buf * 32 + warp] = ss;

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
    // With a full-range table every finite g of a token whose squared norm is
    // a normal fp32 number lies inside it (|g| <= K sqrt(d) up to rounding),
    // so the bin index needs no clamp.  Other tokens (a norm that under- or
    // overflowed in fp32, non-finite values, zero) take the clamped search.
    const bool unclamped = p.full && s2 >= 1e-30f && s2 <= 1e30f;
    if (p.codes) {
      uint32_t* grp = p.codes + (size_t)t * ((size_t)p.d * p.bits / 32) + (size_t)warp * A * p.bits;
      store_codes<MT2>(p.bits, unclamped, D2, ks, magic, bin_lo, bin_hi, tbl_shift, grp, g, q);
    } else {
      uint16_t* rowout = p.out16 + (size_t)t * p.d + (size_t)warp * H + 2 * q;
      if (unclamped)
        rqtc::quantize_store<false, MT2>(D2, ks, magic, bin_lo, bin_hi, tbl_shift, rowout, g);
      else
        rqtc::quantize_store<true, MT2>(D2, ks, magic, bin_lo, bin_hi, tbl_shift, rowout, g);
    }
    if (tid == 0) p.norms[t] = s;
  }
}

}  // namespace

bool rqtc_supported(const RQArgs& a) {
  return (a.out16 || (a.codes && (a.bits == 2 || a.bits == 3 || a.bits == 4 || a.bits == 8))) &&
         (a.h == 1024 || a.h == 512) && a.src_dtype == OQ_DTYPE_BF16 && !a.signmask && a.gather_tc &&
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
  p.codes = a.out16 ? nullptr : a.codes;
  p.bits = a.bits;
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
