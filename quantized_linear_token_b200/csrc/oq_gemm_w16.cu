// Decode-then-contract route for large batches, second kernel: the
// contraction of two fp16 level operands on CTA pairs (tcgen05 cta_group::2,
// M = 256, N = 256, K = 16 per MMA):
//   y[m, n] = a_scale[m] b_scale[n] out_scale sum_k A[m, k] B[n, k]
// (gecl notes Method 2 and Takeaway 3: the product of the two codebook
// operands in the shared rotated basis; the levels are exact in fp16 up to the
// codebook's fp16 scale, and the tensor cores add them in fp32).  The weight
// operand comes from oq_levels.cu, decoded once per call.
//
// Each CTA of a pair loads its 128 A rows and 128 B rows of every K block of
// 64 by TMA into its own shared memory and counts the bytes on the even CTA's
// `full` barrier (the .cta_group::2 form of the load, no multicast), so the
// MMA issuer needs no software hand-off between the CTAs.  The MMA completion
// is multicast by tcgen05.commit to both CTAs' `empty` / `acc_full` barriers;
// the epilogue warps of both CTAs arrive on the even CTA's `acc_empty`.  Two
// accumulators of 256 columns in tensor memory let the epilogue of one tile
// overlap the main loop of the next.  Every wait is bounded (oq_ptx.cuh).
//
// Warps: 0-3 epilogue (tensor-memory lane quarters 0-3), 4 TMA producer,
// 5 allocates tensor memory and (even CTA) issues the MMAs.
#include <cuda.h>

#include <algorithm>
#include <cstring>

#include "oq_internal.h"
#include "oq_epilogue.cuh"
#include "oq_ptx.cuh"
#include "oq_tmap.cuh"

namespace oq {
namespace {

// ------------------------------------------------------------------ (2) contraction

constexpr int RM = 128;            // A rows per CTA (pair M = 256)
constexpr int PN = 256;            // output columns per pair tile
constexpr int RN = 128;            // B rows per CTA
constexpr int BK = 64;             // K elements per stage (128 bytes of fp16: one swizzle row)
constexpr int OS = 6;              // operand stages
constexpr int A_TILE = RM * BK * 2;
constexpr int B_TILE = RN * BK * 2;
constexpr int STAGE_BYTES = A_TILE + B_TILE;
constexpr int TMA_WARP = 4, MMA_WARP = 5;
constexpr int NTHREADS = 6 * 32;
constexpr uint32_t TMEM_COLS = 2 * PN;
constexpr uint32_t ACC_EMPTY_COUNT = 2 * 4;        // one per epilogue warp, both CTAs
constexpr int EPI_BYTES = 4 * 2 * 32 * 32 * 4;     // per epilogue warp: two 32 x 32 fp32 staging boxes

struct W16Params {
  CUtensorMap a_map;   // fp16 A [M, K], 128B-swizzled boxes of 128 x 64
  CUtensorMap b_map;   // fp16 B [N, K], same boxes
  CUtensorMap y_map;   // fp32 y [M, N], 128B-swizzled boxes of 32 x 32
  const float* a_scale;
  const float* b_scale;
  float out_scale;
  bool y_bf16;         // y is bf16 (else fp32)
  int64_t M;
  int N, K, n_tiles, nkb;
  int64_t tiles;
  int* err;
};

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NTHREADS, 1)
    gemm_w16_kernel(const __grid_constant__ W16Params p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  unsigned char* epi = smem + OS * STAGE_BYTES;      // epilogue staging (1024-aligned)
  uint64_t* op_full = reinterpret_cast<uint64_t*>(epi + EPI_BYTES);
  uint64_t* op_empty = op_full + OS;
  uint64_t* acc_full = op_empty + OS;
  uint64_t* acc_empty = acc_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int64_t pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int nkb = p.nkb;
  const int my_tiles = (p.tiles > pair) ? (int)((p.tiles - 1 - pair) / npairs + 1) : 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < OS; ++s) {
      mbar_init(&op_full[s], 1);    // the even CTA's producer: arrive + expect both CTAs' bytes
      mbar_init(&op_empty[s], 1);   // the MMA commit
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], ACC_EMPTY_COUNT);
    }
    fence_mbar_init();
  }
  if (warp == MMA_WARP) {
    tmem_alloc_pair(tmem_slot, TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();   // barriers of both CTAs initialised before any remote arrival or load
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t smem_base = smem_u32(smem);
  const int total = my_tiles * nkb;   // K blocks this CTA pair runs through

  if (warp == TMA_WARP) {
    // ------------------------------------------------ TMA producer (both CTAs)
    if (lane == 0) {
      // the even CTA's `full` barriers, as shared::cluster addresses
      const uint32_t full0 = mapa_shared(smem_u32(&op_full[0]), 0);
      int s = 0, kb = 0, tile = 0;
      uint32_t n = 0;
      auto origin = [&](int tile_i, int32_t& m0, int32_t& n0) {
        const int64_t tt = pair + (int64_t)tile_i * npairs;
        m0 = (int32_t)((tt / p.n_tiles) * (2 * RM) + rank * RM);
        n0 = (int32_t)((tt % p.n_tiles) * PN + rank * RN);
      };
      int32_t m0 = 0, n0 = 0;
      origin(0, m0, n0);
      for (int g = 0; g < total; ++g) {
        if (n > 0 && !mbar_wait(&op_empty[s], (n - 1) & 1u, p.err)) break;
        // rows past M / N and columns past K arrive as zeros; the full box
        // counts either way
        if (rank == 0) mbar_arrive_expect_tx(&op_full[s], (uint32_t)(2 * STAGE_BYTES));
        unsigned char* st = smem + s * STAGE_BYTES;
        tma_load_2d_pair(st, &p.a_map, kb * BK, m0, full0 + 8u * (uint32_t)s);
        tma_load_2d_pair(st + A_TILE, &p.b_map, kb * BK, n0, full0 + 8u * (uint32_t)s);
        if (++s == OS) {
          s = 0;
          ++n;
        }
        if (++kb == nkb) {
          kb = 0;
          origin(++tile, m0, n0);
        }
      }
    }
    __syncwarp();
  } else if (warp < 4) {
    // ------------------------------------------------ epilogue (both CTAs)
    // Each warp drains its 32 tensor-memory lanes (rows) in chunks of 32
    // columns, scales them, stages the 32 x 32 box in shared memory (128B
    // swizzle, conflict-free) and writes it with one TMA store.  Rows past M
    // are clipped by TMA.
    const int q = warp;
    unsigned char* ebuf = epi + q * (2 * 32 * 32 * 4);
    for (int64_t i = 0; i < my_tiles; ++i) {
      const int a = (int)(i & 1);
      const uint32_t u = (uint32_t)(i >> 1);
      if (!mbar_wait(&acc_full[a], u & 1u, p.err)) break;
      tc_fence_after();
      const int64_t tt = pair + i * npairs;
      const int64_t row0 = (tt / p.n_tiles) * (2 * RM) + rank * RM + q * 32;
      const int64_t row = row0 + lane;
      const int n0 = (int)(tt % p.n_tiles) * PN;
      const float srow = (row < p.M) ? __ldg(p.a_scale + row) * p.out_scale : 0.f;
#pragma unroll 1
      for (int cc = 0; cc < PN / 32; ++cc) {
        const int nb = n0 + cc * 32;
        uint32_t v[32];
        tmem_ld_32x32b_x32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(a * PN + cc * 32), v);
        tmem_wait_ld();
        unsigned char* buf = ebuf + (cc & 1) * (32 * 32 * 4);
        // the store that last read this buffer (two chunks ago) must be done
        if (lane == 0) bulk_wait_read<1>();
        __syncwarp();
        stage_y_chunk(v, srow, p.b_scale + nb, smem_u32(buf), lane, p.y_bf16);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&p.y_map, nb, (int32_t)row0, buf);
          bulk_commit();
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&acc_empty[a]), 0));
    }
    // every store has finished reading shared memory and writing y
    if (lane == 0) bulk_wait<0>();
    __syncwarp();
  } else if (warp == MMA_WARP && rank == 0) {
    // ------------------------------------------------ paired MMA issuer (even CTA)
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f16_f32(2 * RM, PN);
      int s = 0;
      uint32_t n = 0;
      bool ok = true, rdy = false;
      // every stage's descriptors share their high word; a K step of 16 is +2
      // on the low word (32 bytes / 16)
      const uint64_t desc0 = smem_desc_sw128(smem_base);
      const uint32_t d_hi = (uint32_t)(desc0 >> 32), a_lo0 = (uint32_t)desc0;
      for (int64_t i = 0; i < my_tiles && ok; ++i) {
        const int a = (int)(i & 1);
        const uint32_t u = (uint32_t)(i >> 1);
        if (u > 0 && !mbar_wait_cluster(&acc_empty[a], (u - 1) & 1u, p.err)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem + (uint32_t)(a * PN);
        for (int kb = 0; kb < nkb; ++kb) {
          if (!rdy && !mbar_wait_cluster(&op_full[s], n & 1u, p.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          // probe the next stage while this one's MMAs issue
          int s1 = s + 1;
          uint32_t n1 = n;
          if (s1 == OS) {
            s1 = 0;
            ++n1;
          }
          const bool more = kb + 1 < nkb || i + 1 < my_tiles;
          const uint32_t a_lo = a_lo0 + (uint32_t)s * (uint32_t)(STAGE_BYTES >> 4);
          rdy = tc_kblock_4mma<2, false>(d_tmem, a_lo, a_lo + (A_TILE >> 4), d_hi, idesc, kb > 0 ? 1u : 0u,
                                         &op_empty[s], (uint16_t)0x3, &op_full[s1], n1 & 1u, more ? 1u : 0u);
          s = s1;
          n = n1;
        }
        if (ok) tc_commit_pair_mc(&acc_full[a], (uint16_t)0x3);
      }
    }
    __syncwarp();
  }

  // neither CTA may leave while its peer can still read its tiles or arrive
  // on its barriers
  tc_fence_before();
  cluster_sync_all();
  if (warp == MMA_WARP) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, TMEM_COLS);
  }
}

}  // namespace

oq_status gemm_w16_launch(const GemmArgs& g, void* stream) {
  if (g.M == 0) return OQ_OK;
  if (!g.a_f16 || !g.b_f16 || g.N % PN != 0 || g.K % 8 != 0) return OQ_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(g.a_f16) | reinterpret_cast<uintptr_t>(g.b_f16) |
       reinterpret_cast<uintptr_t>(g.y)) & 15)
    return OQ_ERR_UNSUPPORTED;
  W16Params kp;
  std::memset(&kp, 0, sizeof(kp));
  kp.a_scale = g.a_scale;
  kp.b_scale = g.b_scale;
  kp.out_scale = g.out_scale;
  kp.y_bf16 = g.y_bf16;
  kp.M = g.M;
  kp.N = g.N;
  kp.K = g.K;
  kp.err = g.err;
  oq_status st = encode_operand_map(&kp.a_map, g.a_f16, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, g.M, g.K, RM,
                                    "the fp16 A operand");
  if (st == OQ_OK)
    st = encode_operand_map(&kp.b_map, g.b_f16, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, g.N, g.K, RN,
                            "the fp16 B operand");
  if (st == OQ_OK) st = encode_y_map(&kp.y_map, g.y, g.M, g.N, g.y_bf16);
  if (st != OQ_OK) return st;

  const size_t smem = 1024 + (size_t)OS * STAGE_BYTES + EPI_BYTES + 8 * (2 * OS + 4) + 16;
  cudaError_t e = cudaFuncSetAttribute(gemm_w16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) {
    set_error(std::string("cudaFuncSetAttribute(gemm w16): ") + cudaGetErrorString(e));
    return OQ_ERR_CUDA;
  }
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  kp.n_tiles = kp.N / PN;
  kp.nkb = (kp.K + BK - 1) / BK;
  kp.tiles = ((kp.M + 2 * RM - 1) / (2 * RM)) * (int64_t)kp.n_tiles;
  const int64_t grid = std::min<int64_t>(2 * kp.tiles, (int64_t)(sms & ~1));
  // K-block counters are 32-bit
  if (((kp.tiles + grid / 2 - 1) / (grid / 2)) * (int64_t)kp.nkb >= (int64_t)1 << 31) return OQ_ERR_UNSUPPORTED;
  gemm_w16_kernel<<<(unsigned)grid, NTHREADS, smem, static_cast<cudaStream_t>(stream)>>>(kp);
  e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error(std::string("gemm w16 launch: ") + cudaGetErrorString(e));
    return OQ_ERR_CUDA;
  }
  return OQ_OK;
}

}  // namespace oq
