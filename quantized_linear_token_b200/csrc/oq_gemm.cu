// Codebook contraction on the tcgen05 tensor cores (gecl notes Method 2 and
// Takeaway 3: a native non-uniform low-bit GEMM in the shared rotated basis):
//   y[m, n] = a_scale[m] b_scale[n] out_scale sum_k LA[A[m, k]] LB[B[n, k]]
// A and B are packed code matrices (K-major rows); LA, LB are the two
// codebooks as fp16 values (pre-scaled, see oq_host.cpp).
//
// Persistent kernel, one CTA per SM, tiles of BM x BN outputs, K blocks of 64:
//   * warps 0-7 ("decoders") stream the codes of each K block straight from
//     global memory (one 16-byte load per 32-64 codes, prefetched one K block
//     ahead) and expand them in registers into fp16 operand tiles in the
//     128-byte-swizzled K-major layout tcgen05 reads.  The expansion uses
//     byte-permute (prmt) lookups into codebook tables held in registers:
//     4-bit codes use the codebook's symmetry (magnitude table + sign byte),
//     2- and 3-bit codes a full table; 8-bit codes a shared-memory table;
//   * warp 12 allocates 2 x BN columns of tensor memory (two accumulators)
//     and one of its threads issues tcgen05.mma (M=128, N=BN, K=16) for each
//     decoded stage, releasing it with tcgen05.commit;
//   * warps 8-11 drain the other accumulator (tcgen05.ld), apply
//     s[m] r[n] / (alpha_a alpha_w) and store y, overlapping the next tile.
// All mbarrier waits are bounded (oq_ptx.cuh).
#include <algorithm>
#include <cstring>

#include "oq_decode.cuh"
#include "oq_internal.h"
#include "oq_epilogue.cuh"
#include "oq_ptx.cuh"

namespace oq {
namespace {

constexpr int BM = 128, BK = 64, UMMA_K = 16;
constexpr int NDEC = 256;          // decoder threads (warps 0-7)
constexpr int EPI_WARP0 = 8;       // epilogue warps 8-11
constexpr int MMA_WARP = 12;
constexpr int NTHREADS = 13 * 32;
constexpr int OS = 4;              // operand stages

struct GemmKParams {
  const uint32_t* a_codes;
  const uint32_t* b_codes;
  const float* a_scale;
  const float* b_scale;
  float out_scale;
  bool y_bf16;         // y is bf16 (else fp32)
  void* y;             // [M, N] fp32, or bf16 with y_bf16
  int64_t M;
  int N, K, a_wpr, b_wpr;
  int n_tiles, nkb;
  int64_t tiles;
  uint32_t a_tab[4], b_tab[4];
  const uint16_t* a_lut8;
  int* err;
};

template <int A_BITS, int B_BITS, int BN>
__global__ void __launch_bounds__(NTHREADS, 1) gemm_kernel(const __grid_constant__ GemmKParams p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  constexpr int A_TILE = BM * BK * 2;
  constexpr int B_TILE = BN * BK * 2;
  constexpr int STAGE_BYTES = A_TILE + B_TILE;
  constexpr int QA = Fmt<A_BITS>::QP, QB = Fmt<B_BITS>::QP;
  constexpr int ITEMS_A = BM * QA, ITEMS = BM * QA + BN * QB;
  constexpr int IPT = (ITEMS + NDEC - 1) / NDEC;
  constexpr uint32_t TMEM_COLS = 2 * BN;

  uint16_t* lut8 = reinterpret_cast<uint16_t*>(smem + OS * STAGE_BYTES);
  uint64_t* op_full = reinterpret_cast<uint64_t*>(smem + OS * STAGE_BYTES + 512);
  uint64_t* op_empty = op_full + OS;
  uint64_t* acc_full = op_empty + OS;
  uint64_t* acc_empty = acc_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nkb = p.nkb;
  const int64_t my_tiles = (p.tiles > (int64_t)blockIdx.x) ? (p.tiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;

  if (A_BITS == 8 && p.a_lut8)
    for (int i = threadIdx.x; i < 256; i += blockDim.x) lut8[i] = p.a_lut8[i];
  if (threadIdx.x == 0) {
    for (int s = 0; s < OS; ++s) {
      mbar_init(&op_full[s], NDEC);
      mbar_init(&op_empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 128);
    }
    fence_mbar_init();
  }
  if (warp == MMA_WARP) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp < NDEC / 32) {
    // ------------------------------------------------ decoders
    uint32_t ta[4], tb[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      ta[i] = p.a_tab[i];
      tb[i] = p.b_tab[i];
    }
    const int64_t total = my_tiles * nkb;
    uint4 cur[IPT], nxt[IPT];
    // rows past M or N only feed outputs the epilogue never stores, so their
    // loads are skipped and their (arbitrary) decoded values left in place;
    // K past the end must contribute zero and is cleared on the A side.
    auto fetch = [&](int64_t m0, int n0, int kb, uint4 (&dst)[IPT]) {
#pragma unroll
      for (int it = 0; it < IPT; ++it) {
        const int id = threadIdx.x + NDEC * it;
        dst[it] = make_uint4(0u, 0u, 0u, 0u);
        if (id < ITEMS_A) {
          const int64_t row = m0 + id / QA;
          if (row < p.M) dst[it] = load_part<A_BITS>(p.a_codes + row * p.a_wpr, kb, id % QA, p.K);
        } else if (id < ITEMS) {
          const int row = n0 + (id - ITEMS_A) / QB;
          if (row < p.N) dst[it] = load_part<B_BITS>(p.b_codes + (int64_t)row * p.b_wpr, kb, (id - ITEMS_A) % QB, p.K);
        }
      }
    };
    auto tile_origin = [&](int64_t tile_i, int64_t& m0, int& n0) {
      const int64_t tt = blockIdx.x + tile_i * gridDim.x;
      m0 = (tt / p.n_tiles) * BM;
      n0 = (int)(tt % p.n_tiles) * BN;
    };
    int64_t m0 = 0, m0n = 0;
    int n0 = 0, n0n = 0;
    int64_t tile_i = 0;
    int kb = 0;
    if (total > 0) {
      tile_origin(0, m0, n0);
      fetch(m0, n0, 0, cur);
    }
    for (int64_t g = 0; g < total; ++g) {
      // position of the next K block (no divisions on the per-block path)
      int kbn = kb + 1;
      int64_t tile_n = tile_i;
      m0n = m0;
      n0n = n0;
      if (kbn == nkb) {
        kbn = 0;
        ++tile_n;
        if (g + 1 < total) tile_origin(tile_n, m0n, n0n);
      }
      if (g + 1 < total) fetch(m0n, n0n, kbn, nxt);
      const int s = (int)(g & (OS - 1));
      const uint32_t n = (uint32_t)(g / OS);
      if (n > 0 && !mbar_wait(&op_empty[s], (n - 1) & 1u, p.err)) break;
      unsigned char* At = smem + s * STAGE_BYTES;
      unsigned char* Bt = At + A_TILE;
      const bool kfull = (kb + 1) * BK <= p.K;
#pragma unroll
      for (int it = 0; it < IPT; ++it) {
        const int id = threadIdx.x + NDEC * it;
        if (id < ITEMS_A) {
          const int r = id / QA, q = id % QA;
#pragma unroll
          for (int j = 0; j < Fmt<A_BITS>::CPP; ++j) {
            uint4 o = decode_chunk<A_BITS>(cur[it], j, ta, lut8);
            if (!kfull && kb * BK + (q * Fmt<A_BITS>::CPP + j) * 8 >= p.K) o = make_uint4(0u, 0u, 0u, 0u);
            *reinterpret_cast<uint4*>(At + sw128_offset(r, q * Fmt<A_BITS>::CPP + j)) = o;
          }
        } else if (id < ITEMS) {
          const int r = (id - ITEMS_A) / QB, q = (id - ITEMS_A) % QB;
#pragma unroll
          for (int j = 0; j < Fmt<B_BITS>::CPP; ++j)
            *reinterpret_cast<uint4*>(Bt + sw128_offset(r, q * Fmt<B_BITS>::CPP + j)) =
                decode_chunk<B_BITS>(cur[it], j, tb, lut8);
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(&op_full[s]);
#pragma unroll
      for (int it = 0; it < IPT; ++it) cur[it] = nxt[it];
      kb = kbn;
      tile_i = tile_n;
      m0 = m0n;
      n0 = n0n;
    }
  } else if (warp >= EPI_WARP0 && warp < EPI_WARP0 + 4) {
    // ------------------------------------------------ epilogue
    const int q = warp & 3;
    for (int64_t i = 0; i < my_tiles; ++i) {
      const int a = (int)(i & 1);
      const uint32_t u = (uint32_t)(i >> 1);
      if (!mbar_wait(&acc_full[a], u & 1u, p.err)) break;
      tc_fence_after();
      const int64_t tt = blockIdx.x + i * gridDim.x;
      const int64_t row = (tt / p.n_tiles) * BM + q * 32 + lane;
      const int n0 = (int)(tt % p.n_tiles) * BN;
      const float srow = (row < p.M) ? __ldg(p.a_scale + row) * p.out_scale : 0.f;
#pragma unroll 1
      for (int cc = 0; cc < BN / 32; ++cc) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(a * BN + cc * 32), v);
        tmem_wait_ld();
        const int nb = n0 + cc * 32;
        if (row < p.M && nb < p.N && !p.y_bf16) {
          float* dst = static_cast<float*>(p.y) + row * p.N + nb;
          if (nb + 32 <= p.N) {
#pragma unroll
            for (int k4 = 0; k4 < 8; ++k4) {
              const float4 rr = __ldg(reinterpret_cast<const float4*>(p.b_scale + nb) + k4);
              float4 o;
              o.x = __uint_as_float(v[4 * k4 + 0]) * srow * rr.x;
              o.y = __uint_as_float(v[4 * k4 + 1]) * srow * rr.y;
              o.z = __uint_as_float(v[4 * k4 + 2]) * srow * rr.z;
              o.w = __uint_as_float(v[4 * k4 + 3]) * srow * rr.w;
              reinterpret_cast<float4*>(dst)[k4] = o;
            }
          } else {
#pragma unroll
            for (int k1 = 0; k1 < 32; ++k1)
              if (nb + k1 < p.N) dst[k1] = __uint_as_float(v[k1]) * srow * __ldg(p.b_scale + nb + k1);
          }
        } else if (row < p.M && nb < p.N) {
          // bf16 y: pairs rounded to nearest even; 32 columns are 64
          // contiguous, 16-byte aligned bytes (N % 16 == 0)
          uint16_t* dst = static_cast<uint16_t*>(p.y) + row * p.N + nb;
          if (nb + 32 <= p.N) {
#pragma unroll
            for (int k8 = 0; k8 < 4; ++k8) {
              const float4 r0 = __ldg(reinterpret_cast<const float4*>(p.b_scale + nb) + 2 * k8);
              const float4 r1 = __ldg(reinterpret_cast<const float4*>(p.b_scale + nb) + 2 * k8 + 1);
              const uint32_t* w = v + 8 * k8;
              uint4 o;
              o.x = pack_bf16x2(__uint_as_float(w[0]) * srow * r0.x, __uint_as_float(w[1]) * srow * r0.y);
              o.y = pack_bf16x2(__uint_as_float(w[2]) * srow * r0.z, __uint_as_float(w[3]) * srow * r0.w);
              o.z = pack_bf16x2(__uint_as_float(w[4]) * srow * r1.x, __uint_as_float(w[5]) * srow * r1.y);
              o.w = pack_bf16x2(__uint_as_float(w[6]) * srow * r1.z, __uint_as_float(w[7]) * srow * r1.w);
              reinterpret_cast<uint4*>(dst)[k8] = o;
            }
          } else {
#pragma unroll
            for (int k1 = 0; k1 < 32; ++k1)
              if (nb + k1 < p.N) {
                const __nv_bfloat16 b = __float2bfloat16_rn(__uint_as_float(v[k1]) * srow * __ldg(p.b_scale + nb + k1));
                dst[k1] = *reinterpret_cast<const uint16_t*>(&b);
              }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[a]);
    }
  } else if (warp == MMA_WARP) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f16_f32(BM, BN);
      const uint32_t tiles_base = smem_u32(smem);
      int64_t g = 0;
      bool ok = true;
      for (int64_t i = 0; i < my_tiles && ok; ++i) {
        const int a = (int)(i & 1);
        const uint32_t u = (uint32_t)(i >> 1);
        if (u > 0 && !mbar_wait(&acc_empty[a], (u - 1) & 1u, p.err)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem + (uint32_t)(a * BN);
        for (int kb = 0; kb < nkb; ++kb, ++g) {
          const int s = (int)(g % OS);
          const uint32_t n = (uint32_t)(g / OS);
          if (!mbar_wait(&op_full[s], n & 1u, p.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = tiles_base + s * STAGE_BYTES, b_addr = a_addr + A_TILE;
#pragma unroll
          for (int kk = 0; kk < BK / UMMA_K; ++kk)
            tc_mma_f16_ss(d_tmem, smem_desc_sw128(a_addr + kk * 32), smem_desc_sw128(b_addr + kk * 32), idesc,
                          (kb > 0 || kk > 0) ? 1u : 0u);
          tc_commit(&op_empty[s]);
        }
        tc_commit(&acc_full[a]);
      }
    }
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

template <int A_BITS, int B_BITS, int BN>
oq_status launch(const GemmKParams& kp_in, void* stream) {
  GemmKParams kp = kp_in;
  auto kern = gemm_kernel<A_BITS, B_BITS, BN>;
  const size_t smem = 1024 + (size_t)OS * (BM * BK * 2 + BN * BK * 2) + 512 + 8 * (2 * OS + 4) + 16;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) {
    set_error(std::string("cudaFuncSetAttribute(gemm): ") + cudaGetErrorString(e));
    return OQ_ERR_CUDA;
  }
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  kp.n_tiles = (kp.N + BN - 1) / BN;
  kp.nkb = (kp.K + BK - 1) / BK;
  kp.tiles = ((kp.M + BM - 1) / BM) * (int64_t)kp.n_tiles;
  const int grid = (int)std::min<int64_t>(kp.tiles, sms);
  kern<<<grid, NTHREADS, smem, static_cast<cudaStream_t>(stream)>>>(kp);
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

// register tables for the prmt decoders
void make_decode_tables(int bits, const uint16_t* lv, uint32_t* t) {
  auto pack = [](const uint8_t* b) {
    return (uint32_t)b[0] | ((uint32_t)b[1] << 8) | ((uint32_t)b[2] << 16) | ((uint32_t)b[3] << 24);
  };
  uint8_t lo[8] = {0}, hi[8] = {0};
  t[0] = t[1] = t[2] = t[3] = 0;
  if (bits == 4) {
    for (int m = 0; m < 8; ++m) {  // positive magnitudes, ascending
      lo[m] = (uint8_t)(lv[8 + m] & 0xFF);
      hi[m] = (uint8_t)(lv[8 + m] >> 8);
    }
  } else if (bits == 3 || bits == 2) {
    for (int c = 0; c < (1 << bits); ++c) {
      lo[c] = (uint8_t)(lv[c] & 0xFF);
      hi[c] = (uint8_t)(lv[c] >> 8);
    }
  } else {
    return;
  }
  if (bits == 2) {
    t[0] = pack(lo);
    t[1] = pack(hi);
  } else {
    t[0] = pack(lo);
    t[1] = pack(lo + 4);
    t[2] = pack(hi);
    t[3] = pack(hi + 4);
  }
}

oq_status gemm_launch(const GemmArgs& g, void* stream) {
  if (g.M == 0) return OQ_OK;
  if (g.fp8) return gemm_pair_launch(g, stream);   // the FP8 mode exists only on CTA pairs
  // CTA-pair tiles (256 x 256) whenever the output width allows them
  if (g.N % 256 == 0) {
    const oq_status st = gemm_pair_launch(g, stream);
    if (st != OQ_ERR_UNSUPPORTED) return st;
  }
  GemmKParams kp;
  std::memset(&kp, 0, sizeof(kp));
  kp.a_codes = g.a_codes;
  kp.b_codes = g.b_codes;
  kp.a_scale = g.a_scale;
  kp.b_scale = g.b_scale;
  kp.out_scale = g.out_scale;
  kp.y_bf16 = g.y_bf16;
  kp.y = g.y;
  kp.M = g.M;
  kp.N = g.N;
  kp.K = g.K;
  kp.a_wpr = g.K * g.a_bits / 32;
  kp.b_wpr = g.K * g.b_bits / 32;
  make_decode_tables(g.a_bits, g.a_levels_host, kp.a_tab);
  make_decode_tables(g.b_bits, g.b_levels_host, kp.b_tab);
  kp.a_lut8 = g.a_levels;
  kp.err = g.err;
  switch (g.a_bits) {
    case 2: return launch_b<2>(kp, g.b_bits, stream);
    case 3: return launch_b<3>(kp, g.b_bits, stream);
    case 4: return launch_b<4>(kp, g.b_bits, stream);
    case 8: return launch_b<8>(kp, g.b_bits, stream);
    default: return OQ_ERR_UNSUPPORTED;
  }
}

}  // namespace oq
