// Codebook contraction for the batch-1 / GEMV end of the workload sweep
// (T <= 8 tokens): y[t, o] = a_scale[t] b_scale[o] out_scale sum_k A[t, k]
// C_w[Wc[o, k]], with A the fp16 levels of the activation codes (gecl notes
// Method 2; the weights are streamed once and are the whole cost, so the
// kernel is built to read them at HBM speed).
//
// A CTA owns 16 weight rows; its 8 warps split K.  Each warp runs warp-level
// MMAs (m16n8k16: M = 16 weight rows, N = 8 tokens, K = 16, fp32 accumulate)
// with its own mapping of the MMA's K slots to positions, chosen so that a
// lane's operands are contiguous in memory: in a chunk of 128 positions,
// lane q of each quad owns positions [32 q, 32 q + 32), and MMA step s (of 8)
// maps the lane's K slots {2q, 2q + 1} to positions 32 q + 4 s + {0, 1} and
// {2q + 8, 2q + 9} to 32 q + 4 s + {2, 3}.  The same mapping on both operands
// leaves the sum unchanged.  So a lane reads one 32-code group of each of its
// two weight rows (one 16-byte load at 4 bits) and 64 contiguous bytes of its
// token's levels per chunk, and decodes the codes with byte-permute lookups in
// registers.  The 8 warps' partial sums meet in shared memory and are added in
// a fixed order, so results repeat bit for bit; no CTA waits on another.
#include <cuda_bf16.h>

#include <algorithm>
#include <cstring>

#include "oq_decode.cuh"
#include "oq_internal.h"
#include "oq_ptx.cuh"

namespace oq {
namespace {

constexpr int ROWS = 16;           // weight rows per CTA (the MMA's M)
constexpr int NWARP = 8;           // warps per CTA, splitting K
constexpr int CHUNK = 128;         // K positions per warp step (32 per quad lane)

struct GemvParams {
  const uint32_t* codes;           // weight codes [N, K * bits / 32]
  const uint16_t* a16;             // fp16 levels [T, K]
  const float* a_scale;            // [T]
  const float* b_scale;            // [N]
  void* y;                         // [T, N] fp32, or bf16 with y_bf16
  float out_scale;
  int T, N, K, wpr;                // wpr: code words per weight row
  int y_bf16;
  uint32_t tab[4];                 // byte-permute decode tables of the weight codebook
};

__device__ __forceinline__ void mma_f16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                              uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// the 32 codes of group `grp` of a weight row (BITS words; zeros past the row)
template <int BITS>
__device__ __forceinline__ uint4 load_group(const uint32_t* row, int grp, bool valid) {
  if (!valid) return make_uint4(0u, 0u, 0u, 0u);
  const uint32_t* p = row + (size_t)grp * BITS;
  if constexpr (BITS == 4) {
    return __ldg(reinterpret_cast<const uint4*>(p));
  } else if constexpr (BITS == 2) {
    const uint2 v = __ldg(reinterpret_cast<const uint2*>(p));
    return make_uint4(v.x, v.y, 0u, 0u);
  } else {
    return make_uint4(__ldg(p), __ldg(p + 1), __ldg(p + 2), 0u);
  }
}

// positions 8 j .. 8 j + 7 of a group -> four fp16 pairs (.x = 8j, 8j+1, ...)
template <int BITS>
__device__ __forceinline__ uint4 decode8(const uint4& v, int j, const uint32_t (&t)[4]) {
  return decode_chunk<BITS>(v, j, t, nullptr);
}

template <int BITS>
__global__ void __launch_bounds__(NWARP * 32, 4) gemv_kernel(const __grid_constant__ GemvParams p) {
  __shared__ __align__(16) float part[NWARP][32][4];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
  const int o0 = blockIdx.x * ROWS;
  const uint32_t* row_lo = p.codes + (size_t)(o0 + g) * p.wpr;       // weight row g of the tile
  const uint32_t* row_hi = p.codes + (size_t)(o0 + g + 8) * p.wpr;   // weight row g + 8
  const bool tok = g < p.T;                                          // this lane's token (B column g)
  const uint16_t* arow = p.a16 + (size_t)(tok ? g : 0) * p.K;
  uint32_t t[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) t[i] = p.tab[i];

  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  const int nchunks = (p.K + CHUNK - 1) / CHUNK;
#pragma unroll 1
  for (int c = warp; c < nchunks; c += NWARP) {
    const int pos0 = c * CHUNK + 32 * q;                              // this lane's 32 positions
    const bool valid = pos0 < p.K;                                    // K % 32 == 0: whole groups
    const uint4 wl = load_group<BITS>(row_lo, pos0 >> 5, valid);
    const uint4 wh = load_group<BITS>(row_hi, pos0 >> 5, valid);
    uint4 av[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
      av[i] = (valid && tok) ? __ldg(reinterpret_cast<const uint4*>(arow + pos0) + i) : make_uint4(0u, 0u, 0u, 0u);
    const uint32_t aw[16] = {av[0].x, av[0].y, av[0].z, av[0].w, av[1].x, av[1].y, av[1].z, av[1].w,
                             av[2].x, av[2].y, av[2].z, av[2].w, av[3].x, av[3].y, av[3].z, av[3].w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint4 dl = decode8<BITS>(wl, j, t), dh = decode8<BITS>(wh, j, t);
      // step 2j: positions 8j .. 8j + 3; step 2j + 1: 8j + 4 .. 8j + 7
      mma_f16_16816(acc, dl.x, dh.x, dl.y, dh.y, aw[4 * j], aw[4 * j + 1]);
      mma_f16_16816(acc, dl.z, dh.z, dl.w, dh.w, aw[4 * j + 2], aw[4 * j + 3]);
    }
  }
  // the warps' partial sums, added in warp order
  *reinterpret_cast<float4*>(part[warp][lane]) = make_float4(acc[0], acc[1], acc[2], acc[3]);
  __syncthreads();
  if (warp != 0) return;
  float s[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int w = 0; w < NWARP; ++w) {
    const float4 v = *reinterpret_cast<const float4*>(part[w][lane]);
    s[0] += v.x;
    s[1] += v.y;
    s[2] += v.z;
    s[3] += v.w;
  }
  // accumulator (row m, column n): d0 = (g, 2q), d1 = (g, 2q + 1),
  // d2 = (g + 8, 2q), d3 = (g + 8, 2q + 1); rows are weight rows, columns tokens
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int o = o0 + g + 8 * (i >> 1), tk = 2 * q + (i & 1);
    if (tk >= p.T) continue;
    const float v = s[i] * __ldg(p.a_scale + tk) * p.out_scale * __ldg(p.b_scale + o);
    const size_t at = (size_t)tk * p.N + o;
    if (p.y_bf16) {
      const __nv_bfloat16 b = __float2bfloat16_rn(v);
      static_cast<uint16_t*>(p.y)[at] = *reinterpret_cast<const uint16_t*>(&b);
    } else {
      static_cast<float*>(p.y)[at] = v;
    }
  }
}

}  // namespace

oq_status gemv_launch(const GemmArgs& g, void* stream) {
  if (g.M == 0) return OQ_OK;
  if (!g.a_f16 || g.a_bf16 || g.fp8 || g.M > GEMV_MAX_T || g.N % ROWS != 0 || g.K % 32 != 0 ||
      !(g.b_bits == 2 || g.b_bits == 3 || g.b_bits == 4))
    return OQ_ERR_UNSUPPORTED;
  if (reinterpret_cast<uintptr_t>(g.a_f16) & 15) return OQ_ERR_UNSUPPORTED;
  GemvParams kp;
  std::memset(&kp, 0, sizeof(kp));
  kp.codes = g.b_codes;
  kp.a16 = g.a_f16;
  kp.a_scale = g.a_scale;
  kp.b_scale = g.b_scale;
  kp.y = g.y;
  kp.out_scale = g.out_scale;
  kp.T = (int)g.M;
  kp.N = g.N;
  kp.K = g.K;
  kp.wpr = g.K * g.b_bits / 32;
  kp.y_bf16 = g.y_bf16 ? 1 : 0;
  make_decode_tables(g.b_bits, g.b_levels_host, kp.tab);
  const unsigned grid = (unsigned)(g.N / ROWS);
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  switch (g.b_bits) {
    case 2: gemv_kernel<2><<<grid, NWARP * 32, 0, s>>>(kp); break;
    case 3: gemv_kernel<3><<<grid, NWARP * 32, 0, s>>>(kp); break;
    default: gemv_kernel<4><<<grid, NWARP * 32, 0, s>>>(kp); break;
  }
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error(std::string("gemv launch: ") + cudaGetErrorString(e));
    return OQ_ERR_CUDA;
  }
  return OQ_OK;
}

}  // namespace oq
