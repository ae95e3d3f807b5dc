// Codebook contraction for small batches (T <= 256 tokens): the roles of the
// operands are swapped so that the tensor cores' M dimension is 128 weight
// rows and N is the (padded) token count,
//   y[t, o] = a_scale[t] b_scale[o] out_scale sum_k A[t, k] LB[B[o, k]],
// with A the fp16 levels of the activation codes (written by the rotate-
// quantize kernel, fetched by TMA) and the weight codes decoded to fp16 in
// shared memory (gecl notes Method 2 and Takeaway 3; the batch-1 / GEMV end of
// the workload sweep).  Every weight row is decoded once per call.  With few
// weight-row tiles the K range is split so that every SM gets work; the splits
// of a tile add into y one after another (split s waits for split s - 1 on a
// per-tile counter), so the result does not depend on timing.  The waits need
// every CTA of the grid resident at once, which the cooperative launch
// guarantees.
//
// Warps: 0-15 decode weight codes (two groups on alternate K blocks), 16-19
// epilogue (TMEM lane quarters 0-3), 20 issues the MMAs (M 128, N = padded T,
// K 16), 21 issues the TMA loads of the token tiles and 22 those of the
// weight-code tiles (a ring of eight
// stages of two K blocks, deep enough to cover DRAM latency; the decoders read
// their codes from shared memory).  Two TMEM accumulators let one work item's epilogue
// overlap the next item's main loop.  Every wait is bounded.
#include <cuda.h>

#include <algorithm>
#include <cstring>

#include "oq_decode.cuh"
#include "oq_internal.h"
#include "oq_ptx.cuh"
#include "oq_tmap.cuh"

namespace oq {
namespace {

constexpr int WR = 128;            // weight rows per tile (MMA M)
constexpr int BK = DEC_BK, UMMA_K = 16;
constexpr int NGROUP = 256;        // decoder threads per group (two groups: warps 0-7 and 8-15)
constexpr int EPI_WARP0 = 16;      // epilogue warps 16-19
constexpr int MMA_WARP = 20, TMA_WARP = 21, CODE_WARP = 22;
constexpr int NTHREADS = 23 * 32;
constexpr int W_TILE = WR * BK * 2;
constexpr int MAX_STAGES = 8;
constexpr int NCS = 8;             // code-tile stages (two K blocks each)

struct SkinnyParams {
  CUtensorMap x_map;          // fp16 A [T, K], boxes of NT x 64, 128B swizzle (rows past T read as 0)
  CUtensorMap w_map;          // weight codes as bytes [N, K bits / 8], boxes of 128 rows x two K blocks
  const uint32_t* b_codes;
  const float* a_scale;       // [T]
  const float* b_scale;       // [N]
  float out_scale;
  float* y;                   // [T, N]
  int* counters;              // [n_tiles * 4], zero between calls
  int* err;
  int T, N, K, b_wpr, NT, n_tiles, nkb, ks, kps, items, stages, stage_bytes, ring_off;
  uint32_t b_tab[4];
  DecK kc;
};

__device__ __forceinline__ int ld_acquire_gpu(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void st_release_gpu(int* p, int v) {
  asm volatile("st.release.gpu.global.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// bounded wait for a split counter to reach `want`
__device__ __forceinline__ bool wait_counter(const int* c, int want, int* err) {
  if (ld_acquire_gpu(c) == want) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    for (int i = 0; i < 32; ++i)
      if (ld_acquire_gpu(c) == want) return true;
    __nanosleep(64);
    if (globaltimer_ns() - t0 > OQ_WAIT_NS) {
      if (err) atomicOr(err, OQ_DEVERR_TIMEOUT);
      return false;
    }
  }
}

// the K-block range of work item w (split-major order: every split-s item
// comes before any split-(s+1) item, so an item only ever waits on earlier ones)
struct Item {
  int tile, split, k0, k1;
};
__device__ __forceinline__ Item item_of(const SkinnyParams& p, int w) {
  Item it;
  it.tile = w % p.n_tiles;
  it.split = w / p.n_tiles;
  it.k0 = it.split * p.kps;
  it.k1 = min(p.nkb, it.k0 + p.kps);
  return it;
}

// TOK_BF16: the token operand is bf16 (the INT4 weight-only layer's x), and
// the weight levels are decoded as bf16 too (one operand type per MMA)
template <int B_BITS, bool TOK_BF16>
__global__ void __launch_bounds__(NTHREADS, 1) gemm_skinny_kernel(const __grid_constant__ SkinnyParams p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  constexpr int QB = Fmt<B_BITS>::QP, CPB = Fmt<B_BITS>::CPP;
  constexpr int ITEMS = WR * QB;                          // 16-byte code parts per K block
  constexpr int DEC_WARPS = ITEMS / 32;                    // per group
  static_assert(ITEMS <= NGROUP, "one part per decoder thread");
  const int S = p.stages;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + p.ring_off + NCS * WR * (2 * BK * B_BITS / 8));
  uint64_t* empty = full + MAX_STAGES;
  uint64_t* acc_full = empty + MAX_STAGES;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* code_full = acc_empty + 2;
  uint64_t* code_empty = code_full + NCS;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(code_empty + NCS);
  constexpr int CBB = 2 * BK * B_BITS / 8;                // code bytes per row per ring stage
  unsigned char* ring = smem + p.ring_off;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = gridDim.x;
  const int my_items = (p.items > (int)blockIdx.x) ? (p.items - 1 - (int)blockIdx.x) / G + 1 : 0;
  // TMEM columns: two accumulators of NT columns, rounded up to a power of two
  uint32_t ncols = 32;
  while (ncols < 2u * (uint32_t)p.NT) ncols <<= 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], DEC_WARPS + 1);   // one group's decoder warps + the TMA's expect_tx arrival
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 4);
    }
    for (int c = 0; c < NCS; ++c) {
      mbar_init(&code_full[c], 1);
      mbar_init(&code_empty[c], 2 * DEC_WARPS);
    }
    fence_mbar_init();
  }
  if (warp == MMA_WARP) {
    tmem_alloc(tmem_slot, ncols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t smem_base = smem_u32(smem);
  const uint32_t acc_cols = ncols / 2;

  // the flattened sequence of (item, K block) steps this CTA runs through
  int total = 0;
  for (int i = 0; i < my_items; ++i) {
    const Item it = item_of(p, (int)blockIdx.x + i * G);
    total += it.k1 - it.k0;
  }

  const int grp = warp / 8;
  if (warp % 8 < DEC_WARPS && grp < 2) {
    // ------------------------------------------------ weight decoders
    // group grp takes K block grp of every ring stage (a K-block pair); a
    // block is decoded from the ring into registers before the wait for its
    // operand stage, so only the stores follow the release
    uint32_t tb[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) tb[i] = p.b_tab[i];
    const DecK kc = p.kc;
    const int gt = (int)threadIdx.x % NGROUP;
    const int r = gt / QB, q = gt % QB;
    uint32_t sts[CPB];
#pragma unroll
    for (int j = 0; j < CPB; ++j)
      sts[j] = smem_base + (uint32_t)((r >> 3) * 1024 + (r & 7) * 128) +
               ((((uint32_t)(q * CPB + j)) << 4) ^ ((uint32_t)(r & 7) << 4));
    // this thread's 16-byte code part of K block grp of a ring stage
    const unsigned char* my_codes = ring + r * CBB + q * (BK * B_BITS / 8 / QB) + grp * (BK * B_BITS / 8);
    auto read_part = [&](int c) -> uint4 {
      const unsigned char* src_p = my_codes + c * (WR * CBB);
      if constexpr (B_BITS == 3) {
        const uint32_t* w = reinterpret_cast<const uint32_t*>(src_p);
        return make_uint4(w[0], w[1], w[2], 0u);
      } else if constexpr (B_BITS == 2) {
        const uint2 lo = *reinterpret_cast<const uint2*>(src_p), hi = *reinterpret_cast<const uint2*>(src_p + 8);
        return make_uint4(lo.x, lo.y, hi.x, hi.y);
      } else {
        return *reinterpret_cast<const uint4*>(src_p);
      }
    };
    int g = 0, cs = 0;   // K blocks and ring stages passed (both groups)
    bool dead = false;
    for (int i = 0; i < my_items; ++i) {
      const Item it = item_of(p, (int)blockIdx.x + i * G);
      for (int kb = it.k0; kb < it.k1; kb += 2, ++cs) {
        const int c = cs % NCS;
        const uint32_t cn = (uint32_t)(cs / NCS);
        const int mine = kb + grp;
        if (mine < it.k1) {
          if (!dead && !mbar_wait(&code_full[c], cn & 1u, p.err)) dead = true;
          const uint4 cur = read_part(c);
          uint4 dec[CPB];
#pragma unroll
          for (int jj = 0; jj < CPB; ++jj) dec[jj] = decode_chunk_k<B_BITS>(cur, jj, tb, nullptr, kc);
          __syncwarp();
          if (lane == 0) mbar_arrive(&code_empty[c]);
          const int gg = g + grp, s = gg % S;
          const uint32_t n = (uint32_t)(gg / S);
          // after a timed-out wait (error recorded) keep stepping without waiting
          if (n > 0 && !dead && !mbar_wait(&empty[s], (n - 1) & 1u, p.err)) dead = true;
          const uint32_t so = (uint32_t)(s * p.stage_bytes);
#pragma unroll
          for (int jj = 0; jj < CPB; ++jj) st_shared_v4(sts[jj] + so, dec[jj]);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&full[s]);
        } else {
          // the item's last ring stage holds a single K block: nothing to read
          __syncwarp();
          if (lane == 0) mbar_arrive(&code_empty[c]);
        }
        g += min(2, it.k1 - kb);
      }
    }
  } else if (warp == CODE_WARP) {
    // ------------------------------------------------ weight-code tiles by TMA
    if (lane == 0) {
      int c = 0;
      uint32_t cn = 0;
      const uint32_t tx = (uint32_t)(WR * CBB);
      for (int i = 0; i < my_items; ++i) {
        const Item it = item_of(p, (int)blockIdx.x + i * G);
        for (int kb = it.k0; kb < it.k1; kb += 2) {
          if (cn > 0 && !mbar_wait(&code_empty[c], (cn - 1) & 1u, p.err)) {
            i = my_items;
            break;
          }
          // columns past K (the last pair of an odd K-block count) arrive as 0
          mbar_arrive_expect_tx(&code_full[c], tx);
          tma_load_2d(ring + c * (WR * CBB), &p.w_map, kb * (BK * B_BITS / 8), it.tile * WR, &code_full[c]);
          if (++c == NCS) {
            c = 0;
            ++cn;
          }
        }
      }
    }
    __syncwarp();
  } else if (warp == TMA_WARP) {
    // ------------------------------------------------ token tiles by TMA
    if (lane == 0) {
      int s = 0;
      uint32_t n = 0;
      const uint32_t tx = (uint32_t)(p.NT * BK * 2);
      for (int i = 0; i < my_items; ++i) {
        const Item it = item_of(p, (int)blockIdx.x + i * G);
        for (int kb = it.k0; kb < it.k1; ++kb) {
          if (n > 0 && !mbar_wait(&empty[s], (n - 1) & 1u, p.err)) {
            i = my_items;
            break;
          }
          mbar_arrive_expect_tx(&full[s], tx);
          tma_load_2d(smem + s * p.stage_bytes + W_TILE, &p.x_map, kb * BK, 0, &full[s]);
          if (++s == S) {
            s = 0;
            ++n;
          }
        }
      }
    }
    __syncwarp();
  } else if (warp == MMA_WARP) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = TOK_BF16 ? idesc_bf16_f32(WR, p.NT) : idesc_f16_f32(WR, p.NT);
      const uint64_t desc0 = smem_desc_sw128(smem_base);
      const uint32_t d_hi = (uint32_t)(desc0 >> 32), w_lo0 = (uint32_t)desc0;
      int s = 0;
      uint32_t n = 0;
      bool ok = true, rdy = false;
      for (int i = 0; i < my_items && ok; ++i) {
        const Item it = item_of(p, (int)blockIdx.x + i * G);
        const int a = i & 1;
        const uint32_t u = (uint32_t)(i >> 1);
        if (u > 0 && !mbar_wait(&acc_empty[a], (u - 1) & 1u, p.err)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem + (uint32_t)a * acc_cols;
        for (int kb = it.k0; kb < it.k1; ++kb) {
          if (!rdy && !mbar_wait(&full[s], n & 1u, p.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          // probe the next stage while this one's MMAs issue (a barrier check
          // costs ~200 cycles even when the phase is long complete)
          int s1 = s + 1;
          uint32_t n1 = n;
          if (s1 == S) {
            s1 = 0;
            ++n1;
          }
          const bool more = kb + 1 < it.k1 || i + 1 < my_items;
          const uint32_t w_lo = w_lo0 + (uint32_t)(s * p.stage_bytes >> 4);
          const bool rdy1 = tc_kblock64_f16<1>(d_tmem, w_lo, w_lo + (W_TILE >> 4), d_hi, idesc, kb > it.k0 ? 1u : 0u,
                                               &empty[s], (uint16_t)0, &full[s1], n1 & 1u, more ? 1u : 0u);
          s = s1;
          n = n1;
          rdy = rdy1;
        }
        tc_commit(&acc_full[a]);
      }
    }
    __syncwarp();
  } else if (warp >= EPI_WARP0 && warp < EPI_WARP0 + 4) {
    // ------------------------------------------------ epilogue
    // lane = weight row o of this warp's quarter, TMEM column = token t; the
    // splits of a tile add into y in split order (counter per tile and quarter)
    const int qd = warp & 3;
    bool dead = false;
    for (int i = 0; i < my_items; ++i) {
      const Item it = item_of(p, (int)blockIdx.x + i * G);
      const int a = i & 1;
      const uint32_t u = (uint32_t)(i >> 1);
      if (!dead && !mbar_wait(&acc_full[a], u & 1u, p.err)) dead = true;
      tc_fence_after();
      const int o = it.tile * WR + qd * 32 + lane;
      const float ro = __ldg(p.b_scale + o) * p.out_scale;
      int* ctr = p.counters + it.tile * 4 + qd;
      // every lane acquires the counter itself before reading y
      if (it.split > 0 && !dead && !wait_counter(ctr, it.split, p.err)) dead = true;
      __syncwarp();
      for (int c0 = 0; c0 < p.NT; c0 += 32) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(tmem + ((uint32_t)(qd * 32) << 16) + (uint32_t)a * acc_cols + (uint32_t)c0, v);
        tmem_wait_ld();
        // the previous splits' sums, 16 tokens at a time: all loads first (no
        // load waits behind a store), then the stores
#pragma unroll
        for (int h = 0; h < 32; h += 16) {
          float old[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int t = c0 + h + j;
            old[j] = (it.split > 0 && t < p.T) ? __ldcg(p.y + (int64_t)t * p.N + o) : 0.f;
          }
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int t = c0 + h + j;
            if (t < p.T) {
              const float st = p.a_scale ? __ldg(p.a_scale + t) : 1.f;
              p.y[(int64_t)t * p.N + o] = __uint_as_float(v[h + j]) * ro * st + old[j];
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[a]);
      // publish this split's additions, then hand the tile to the next split
      // (the last split resets the counter for the next call)
      __threadfence();
      __syncwarp();
      if (lane == 0) st_release_gpu(ctr, (it.split + 1 == p.ks) ? 0 : it.split + 1);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, ncols);
  }
}

template <int B_BITS, bool TOK_BF16>
oq_status launch_skinny(const SkinnyParams& kp_in, void* stream) {
  SkinnyParams kp = kp_in;
  auto kern = gemm_skinny_kernel<B_BITS, TOK_BF16>;
  kp.stage_bytes = W_TILE + kp.NT * BK * 2;
  constexpr int ring_bytes = NCS * WR * (2 * BK * B_BITS / 8);
  kp.stages = std::min(MAX_STAGES, (208 * 1024 - ring_bytes) / kp.stage_bytes);
  kp.ring_off = kp.stages * kp.stage_bytes;   // 1024-aligned: stage_bytes is a multiple of 2048
  const size_t smem = 1024 + (size_t)kp.ring_off + ring_bytes + 8 * (2 * MAX_STAGES + 4 + 2 * NCS) + 16;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) {
    set_error(std::string("cudaFuncSetAttribute(gemm skinny): ") + cudaGetErrorString(e));
    return OQ_ERR_CUDA;
  }
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // split K so that the items cover the SMs, with at least two K blocks each
  int ks = std::max(1, std::min((sms + kp.n_tiles - 1) / kp.n_tiles, kp.nkb / 2));
  kp.kps = (kp.nkb + ks - 1) / ks;
  kp.kps += kp.kps & 1;   // items start on even K blocks (ring stages hold K-block pairs)
  kp.ks = (kp.nkb + kp.kps - 1) / kp.kps;
  kp.items = kp.n_tiles * kp.ks;
  const int grid = std::min(kp.items, sms);
  // the splits of a tile hand over through counters, so every CTA of the grid
  // must be resident at once: a cooperative launch guarantees that, or fails
  // (and the caller takes another kernel) when the GPU cannot hold the grid
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(NTHREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = static_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, kp);
  if (e == cudaErrorCooperativeLaunchTooLarge) {
    cudaGetLastError();
    set_error("gemm skinny: the GPU cannot hold the whole grid at once");
    return OQ_ERR_UNSUPPORTED;
  }
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error(std::string("gemm skinny launch: ") + cudaGetErrorString(e));
    return OQ_ERR_CUDA;
  }
  return OQ_OK;
}

}  // namespace

oq_status gemm_skinny_launch(const GemmArgs& g, int* counters, void* stream) {
  if (g.M == 0) return OQ_OK;
  if (!g.a_f16 || g.M > SKINNY_MAX_T || g.N % WR != 0 || g.K % 8 != 0) return OQ_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(g.a_f16) & 15) || (reinterpret_cast<uintptr_t>(g.y) & 3)) return OQ_ERR_UNSUPPORTED;
  SkinnyParams kp;
  std::memset(&kp, 0, sizeof(kp));
  kp.b_codes = g.b_codes;
  kp.a_scale = g.a_scale;
  kp.b_scale = g.b_scale;
  kp.out_scale = g.out_scale;
  if (g.y_bf16) return OQ_ERR_UNSUPPORTED;   // the splits add in fp32 in y itself
  kp.y = static_cast<float*>(g.y);
  kp.counters = counters;
  kp.err = g.err;
  kp.T = (int)g.M;
  kp.N = g.N;
  kp.K = g.K;
  kp.b_wpr = g.K * g.b_bits / 32;
  kp.NT = (int)((g.M + 15) / 16) * 16;
  kp.n_tiles = g.N / WR;
  kp.nkb = (g.K + BK - 1) / BK;
  make_decode_tables(g.b_bits, g.b_levels_host, kp.b_tab);
  kp.kc = make_deck();
  oq_status st = encode_operand_map(&kp.x_map, g.a_f16,
                                    g.a_bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, g.M,
                                    g.K, kp.NT, "the token operand");
  if (st != OQ_OK) return st;
  {
    // weight codes as a byte matrix [N, K bits / 8]; rows must be 16-byte multiples
    const int64_t row_bytes = (int64_t)g.K * g.b_bits / 8;
    if (row_bytes % 16 || (reinterpret_cast<uintptr_t>(g.b_codes) & 15)) return OQ_ERR_UNSUPPORTED;
    EncodeTiledFn fn = nullptr;
    st = tmap_encode_fn(&fn);
    if (st != OQ_OK) return st;
    const cuuint64_t dims[2] = {(cuuint64_t)row_bytes, (cuuint64_t)g.N};
    const cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
    const cuuint32_t box[2] = {(cuuint32_t)(2 * BK * g.b_bits / 8), (cuuint32_t)WR};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = fn(&kp.w_map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint32_t*>(g.b_codes), dims,
                          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
      set_error("cuTensorMapEncodeTiled failed for the weight codes (code " + std::to_string((int)r) + ")");
      return OQ_ERR_CUDA;
    }
  }
  if (g.a_bf16) return g.b_bits == 4 ? launch_skinny<4, true>(kp, stream) : OQ_ERR_UNSUPPORTED;
  switch (g.b_bits) {
    case 2: return launch_skinny<2, false>(kp, stream);
    case 3: return launch_skinny<3, false>(kp, stream);
    case 4: return launch_skinny<4, false>(kp, stream);
    default: return OQ_ERR_UNSUPPORTED;
  }
}

}  // namespace oq
