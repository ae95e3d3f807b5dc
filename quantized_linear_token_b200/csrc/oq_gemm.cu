// Codebook contraction on the tcgen05 tensor cores (gecl notes Method 2 and
// Takeaway 3: a native non-uniform low-bit GEMM in the shared rotated basis):
//   y[m, n] = a_scale[m] b_scale[n] out_scale sum_k LA[A[m, k]] LB[B[n, k]]
// A and B are packed code matrices (K-major rows); LA, LB are the two
// codebooks as fp16 (pre-scaled, see oq_host.cpp).
//
// One CTA computes a BM x BN tile of y:
//   * warps 0-3 decode the codes of each K block (BK = 64) through small
//     shared-memory tables straight into fp16 operand tiles laid out in the
//     128-byte-swizzled K-major form that tcgen05 reads (8 codes -> one
//     16-byte chunk per store);
//   * warp 4 allocates the tensor-memory accumulator, and one of its threads
//     issues tcgen05.mma (M = 128, N = BN, K = 16 per instruction) for every
//     full stage, releasing the stage with tcgen05.commit;
//   * warps 0-3 then read the fp32 accumulator back (tcgen05.ld) and write
//     y with the per-row and per-column magnitudes applied.
// Every mbarrier wait is bounded (see oq_ptx.cuh).
#include <algorithm>
#include <cstring>

#include "oq_internal.h"
#include "oq_ptx.cuh"

namespace oq {
namespace {

constexpr int BM = 128, BK = 64, UMMA_K = 16;

struct GemmKParams {
  const uint32_t* a_codes;
  const uint32_t* b_codes;
  const float* a_scale;
  const float* b_scale;
  const uint16_t* a_levels;
  const uint16_t* b_levels;
  float out_scale;
  float* y;
  int64_t M;
  int N, K, a_wpr, b_wpr;
  int* err;
};

// decode tables: one entry per byte of codes (2/4/8 bits) or per 6 bits (3 bits)
template <int BITS> struct Lut;
template <> struct Lut<2> { static constexpr int ENTRIES = 256; using T = uint2; };
template <> struct Lut<3> { static constexpr int ENTRIES = 64; using T = uint32_t; };
template <> struct Lut<4> { static constexpr int ENTRIES = 256; using T = uint32_t; };
template <> struct Lut<8> { static constexpr int ENTRIES = 256; using T = uint32_t; };

template <int BITS>
__device__ void build_lut(typename Lut<BITS>::T* lut, const uint16_t* lv, int tid, int nthreads) {
  for (int e = tid; e < Lut<BITS>::ENTRIES; e += nthreads) {
    if constexpr (BITS == 4) {
      lut[e] = (uint32_t)lv[e & 15] | ((uint32_t)lv[e >> 4] << 16);
    } else if constexpr (BITS == 2) {
      lut[e] = make_uint2((uint32_t)lv[e & 3] | ((uint32_t)lv[(e >> 2) & 3] << 16),
                          (uint32_t)lv[(e >> 4) & 3] | ((uint32_t)lv[e >> 6] << 16));
    } else if constexpr (BITS == 3) {
      lut[e] = (uint32_t)lv[e & 7] | ((uint32_t)lv[e >> 3] << 16);
    } else {
      lut[e] = (uint32_t)lv[e];
    }
  }
}

// 8 codes of a row starting at element k (k % 8 == 0) -> 8 fp16 values
template <int BITS>
__device__ __forceinline__ uint4 decode8(const uint32_t* row, int k, const typename Lut<BITS>::T* lut) {
  if constexpr (BITS == 4) {
    const uint32_t w = __ldg(row + (k >> 3));
    return make_uint4(lut[w & 0xFF], lut[(w >> 8) & 0xFF], lut[(w >> 16) & 0xFF], lut[w >> 24]);
  } else if constexpr (BITS == 2) {
    const uint32_t w = __ldg(row + (k >> 4)) >> ((k & 15) * 2);
    const uint2 a = lut[w & 0xFF], b = lut[(w >> 8) & 0xFF];
    return make_uint4(a.x, a.y, b.x, b.y);
  } else if constexpr (BITS == 8) {
    const uint2 w = __ldg(reinterpret_cast<const uint2*>(row + (k >> 2)));
    return make_uint4(lut[w.x & 0xFF] | (lut[(w.x >> 8) & 0xFF] << 16),
                      lut[(w.x >> 16) & 0xFF] | (lut[w.x >> 24] << 16),
                      lut[w.y & 0xFF] | (lut[(w.y >> 8) & 0xFF] << 16),
                      lut[(w.y >> 16) & 0xFF] | (lut[w.y >> 24] << 16));
  } else {
    const int bit = k * 3, wi = bit >> 5, sh = bit & 31;
    uint32_t v = __ldg(row + wi) >> sh;
    if (sh > 8) v |= __ldg(row + wi + 1) << (32 - sh);
    return make_uint4(lut[v & 63], lut[(v >> 6) & 63], lut[(v >> 12) & 63], lut[(v >> 18) & 63]);
  }
}

// byte offset of 16-byte chunk `ch` of row `r` in a 128B-swizzled K-major tile
__device__ __forceinline__ uint32_t sw128_offset(int r, int ch) {
  return (uint32_t)((r >> 3) * 1024 + (r & 7) * 128 + ((ch ^ (r & 7)) << 4));
}

template <int A_BITS, int B_BITS, int BN, int STAGES>
__global__ void __launch_bounds__(160, 1) gemm_kernel(const __grid_constant__ GemmKParams p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  constexpr int A_TILE = BM * BK * 2;
  constexpr int B_TILE = BN * BK * 2;
  constexpr int STAGE_BYTES = A_TILE + B_TILE;
  using LA = typename Lut<A_BITS>::T;
  using LB = typename Lut<B_BITS>::T;
  LA* lutA = reinterpret_cast<LA*>(smem + STAGES * STAGE_BYTES);
  LB* lutB = reinterpret_cast<LB*>(smem + STAGES * STAGE_BYTES + 2048);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES + 4096);
  uint64_t* empty = full + STAGES;
  uint64_t* accf = empty + STAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accf + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * BN;
  const int64_t m0 = (int64_t)blockIdx.y * BM;
  const int num_kb = (p.K + BK - 1) / BK;

  build_lut<A_BITS>(lutA, p.a_levels, threadIdx.x, blockDim.x);
  build_lut<B_BITS>(lutB, p.b_levels, threadIdx.x, blockDim.x);
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 128);
      mbar_init(&empty[s], 1);
    }
    mbar_init(accf, 1);
    fence_mbar_init();
  }
  if (warp == 4) {
    tmem_alloc(tmem_slot, BN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp < 4) {
    // ------------------------------------------------ decode producers
    const int pt = threadIdx.x;
    for (int kb = 0; kb < num_kb; ++kb) {
      const int s = kb % STAGES;
      const uint32_t ph = (uint32_t)(kb / STAGES) & 1u;
      if (kb >= STAGES && !mbar_wait(&empty[s], ph ^ 1u, p.err)) break;
      unsigned char* At = smem + s * STAGE_BYTES;
      unsigned char* Bt = At + A_TILE;
      const int kbase = kb * BK;
#pragma unroll 4
      for (int i = 0; i < (BM * 8) / 128; ++i) {
        const int id = pt + 128 * i, r = id >> 3, ch = id & 7;
        const int64_t row = m0 + r;
        const int k = kbase + ch * 8;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (row < p.M && k < p.K) v = decode8<A_BITS>(p.a_codes + row * p.a_wpr, k, lutA);
        *reinterpret_cast<uint4*>(At + sw128_offset(r, ch)) = v;
      }
#pragma unroll 4
      for (int i = 0; i < (BN * 8) / 128; ++i) {
        const int id = pt + 128 * i, r = id >> 3, ch = id & 7;
        const int row = n0 + r;
        const int k = kbase + ch * 8;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (row < p.N && k < p.K) v = decode8<B_BITS>(p.b_codes + (int64_t)row * p.b_wpr, k, lutB);
        *reinterpret_cast<uint4*>(Bt + sw128_offset(r, ch)) = v;
      }
      fence_proxy_async_smem();
      mbar_arrive(&full[s]);
    }

    // ------------------------------------------------ epilogue
    mbar_wait(accf, 0u, p.err);
    tc_fence_after();
    const int rl = warp * 32 + lane;
    const int64_t row = m0 + rl;
    const float srow = (row < p.M) ? __ldg(p.a_scale + row) * p.out_scale : 0.f;
#pragma unroll 1
    for (int cc = 0; cc < BN / 32; ++cc) {
      uint32_t v[32];
      tmem_ld_32x32b_x32(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)(cc * 32), v);
      tmem_wait_ld();
      const int nb = n0 + cc * 32;
      if (row < p.M && nb < p.N) {
        float* dst = p.y + row * p.N + nb;
        if (nb + 32 <= p.N) {
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const float4 rr = __ldg(reinterpret_cast<const float4*>(p.b_scale + nb) + q);
            float4 o;
            o.x = __uint_as_float(v[4 * q + 0]) * srow * rr.x;
            o.y = __uint_as_float(v[4 * q + 1]) * srow * rr.y;
            o.z = __uint_as_float(v[4 * q + 2]) * srow * rr.z;
            o.w = __uint_as_float(v[4 * q + 3]) * srow * rr.w;
            reinterpret_cast<float4*>(dst)[q] = o;
          }
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (nb + i < p.N) dst[i] = __uint_as_float(v[i]) * srow * __ldg(p.b_scale + nb + i);
        }
      }
    }
  } else if (warp == 4) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f16_f32(BM, BN);
      const uint32_t tiles = smem_u32(smem);
      for (int kb = 0; kb < num_kb; ++kb) {
        const int s = kb % STAGES;
        const uint32_t ph = (uint32_t)(kb / STAGES) & 1u;
        if (!mbar_wait(&full[s], ph, p.err)) break;
        tc_fence_after();
        const uint32_t a_addr = tiles + s * STAGE_BYTES, b_addr = a_addr + A_TILE;
#pragma unroll
        for (int kk = 0; kk < BK / UMMA_K; ++kk)
          tc_mma_f16_ss(tmem, smem_desc_sw128(a_addr + kk * 32), smem_desc_sw128(b_addr + kk * 32), idesc,
                        (kb > 0 || kk > 0) ? 1u : 0u);
        tc_commit(&empty[s]);
      }
      tc_commit(accf);
    }
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tmem, BN);
  }
}

template <int A_BITS, int B_BITS, int BN>
oq_status launch(const GemmKParams& kp, void* stream) {
  constexpr int STAGES = (BN == 256) ? 4 : 6;
  auto kern = gemm_kernel<A_BITS, B_BITS, BN, STAGES>;
  const size_t smem = 1024 + (size_t)STAGES * (BM * BK * 2 + BN * BK * 2) + 4096 + 8 * (2 * STAGES + 1) + 16;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) {
    set_error(std::string("cudaFuncSetAttribute(gemm): ") + cudaGetErrorString(e));
    return OQ_ERR_CUDA;
  }
  const dim3 grid((unsigned)((kp.N + BN - 1) / BN), (unsigned)((kp.M + BM - 1) / BM));
  kern<<<grid, 160, smem, static_cast<cudaStream_t>(stream)>>>(kp);
  e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error(std::string("gemm launch: ") + cudaGetErrorString(e));
    return OQ_ERR_CUDA;
  }
  return OQ_OK;
}

template <int A_BITS, int B_BITS>
oq_status launch_bn(const GemmKParams& kp, void* stream) {
  if (kp.N >= 256 && kp.N % 256 == 0) return launch<A_BITS, B_BITS, 256>(kp, stream);
  return launch<A_BITS, B_BITS, 128>(kp, stream);
}

template <int A_BITS>
oq_status launch_b(const GemmKParams& kp, int b_bits, void* stream) {
  switch (b_bits) {
    case 2: return launch_bn<A_BITS, 2>(kp, stream);
    case 3: return launch_bn<A_BITS, 3>(kp, stream);
    case 4: return launch_bn<A_BITS, 4>(kp, stream);
    default: return OQ_ERR_UNSUPPORTED;
  }
}

}  // namespace

oq_status gemm_launch(const GemmArgs& g, void* stream) {
  if (g.M == 0) return OQ_OK;
  GemmKParams kp;
  std::memset(&kp, 0, sizeof(kp));
  kp.a_codes = g.a_codes;
  kp.b_codes = g.b_codes;
  kp.a_scale = g.a_scale;
  kp.b_scale = g.b_scale;
  kp.a_levels = g.a_levels;
  kp.b_levels = g.b_levels;
  kp.out_scale = g.out_scale;
  kp.y = g.y;
  kp.M = g.M;
  kp.N = g.N;
  kp.K = g.K;
  kp.a_wpr = g.K * g.a_bits / 32;
  kp.b_wpr = g.K * g.b_bits / 32;
  kp.err = g.err;
  if (g.M > (int64_t)65535 * BM) return OQ_ERR_UNSUPPORTED;
  switch (g.a_bits) {
    case 2: return launch_b<2>(kp, g.b_bits, stream);
    case 3: return launch_b<3>(kp, g.b_bits, stream);
    case 4: return launch_b<4>(kp, g.b_bits, stream);
    case 8: return launch_b<8>(kp, g.b_bits, stream);
    default: return OQ_ERR_UNSUPPORTED;
  }
}

}  // namespace oq
