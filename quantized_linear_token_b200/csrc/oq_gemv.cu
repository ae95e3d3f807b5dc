// Codebook contraction for the batch-1 / GEMV end of the workload sweep
// (T <= 24 tokens): y[t, o] = a_scale[t] b_scale[o] out_scale sum_k A[t, k]
// C_w[Wc[o, k]], with A the fp16 levels of the activation codes (gecl notes
// Method 2; the weights are streamed once and are the whole cost, so the
// kernel is built to read them at HBM speed).
//
// A CTA owns 16 weight rows; its 8 warps split K.  Each warp runs warp-level
// MMAs (m16n8k16: M = 16 weight rows, N = a tile of 8 tokens, K = 16, fp32
// accumulate; up to three token tiles share each decoded weight fragment)
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
//
// Each warp keeps the weight groups of its next chunks in registers (PREFETCH
// of them for one token tile, one fewer for more tiles, whose MMAs take longer
// per chunk): the loads of chunk i + PF are issued before chunk i is decoded
// and multiplied.  The kernel is bound by instruction issue (the decode) more
// than by the loads in flight: depths of 1 to 6 chunks measured alike.
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
constexpr int PREFETCH = 3;        // chunks of weight codes in flight per warp
constexpr int MIN_CTAS = 3;        // resident CTAs per SM the register budget allows

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

template <int BITS, int NT>
__global__ void __launch_bounds__(NWARP * 32, MIN_CTAS) gemv_kernel(const __grid_constant__ GemvParams p) {
  __shared__ __align__(16) float part[NWARP][NT][32][4];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
  const int o0 = blockIdx.x * ROWS;
  const uint32_t* row_lo = p.codes + (size_t)(o0 + g) * p.wpr;       // weight row g of the tile
  const uint32_t* row_hi = p.codes + (size_t)(o0 + g + 8) * p.wpr;   // weight row g + 8
  // this lane's token in token tile n (B column g of tile n) is 8 n + g; its
  // levels start at arow + 8 n K
  const uint16_t* arow = p.a16 + (size_t)g * p.K;
  uint32_t t[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) t[i] = p.tab[i];

  // this warp's chunks are warp, warp + NWARP, ...: chunk i of the warp starts
  // at position (warp + i NWARP) CHUNK, and the lane's 32 positions at 32 q
  // past that (K % 32 == 0, so a lane's group lies wholly inside or past K)
  const int nchunks = (p.K + CHUNK - 1) / CHUNK;
  const int nmine = warp < nchunks ? (nchunks - 1 - warp) / NWARP + 1 : 0;
  auto pos_of = [&](int i) { return (warp + i * NWARP) * CHUNK + 32 * q; };
  constexpr int PF = NT == 1 ? PREFETCH : PREFETCH - 1;
  uint4 wl[PF], wh[PF];
#pragma unroll
  for (int u = 0; u < PF; ++u) {
    const int pos = pos_of(u);
    const bool valid = u < nmine && pos < p.K;
    wl[u] = load_group<BITS>(row_lo, pos >> 5, valid);
    wh[u] = load_group<BITS>(row_hi, pos >> 5, valid);
  }

  float acc[NT][4];
#pragma unroll
  for (int n = 0; n < NT; ++n)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[n][i] = 0.f;
#pragma unroll 1
  for (int i0 = 0; i0 < nmine; i0 += PF) {
#pragma unroll
    for (int u = 0; u < PF; ++u) {
      const int i = i0 + u;
      if (i >= nmine) break;                                          // warp-uniform
      const int pos0 = pos_of(i);
      const bool valid = pos0 < p.K;
      const uint4 cl = wl[u], ch = wh[u];
      // refill the slot with chunk i + PF before working on chunk i
      const int posn = pos_of(i + PF);
      const bool vn = i + PF < nmine && posn < p.K;
      wl[u] = load_group<BITS>(row_lo, posn >> 5, vn);
      wh[u] = load_group<BITS>(row_hi, posn >> 5, vn);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        // positions 8j .. 8j + 7 of the lane's group: the weights decoded
        // once, then step 2j (8j .. 8j + 3) and 2j + 1 (8j + 4 .. 8j + 7) for
        // every token tile
        const uint4 dl = decode8<BITS>(cl, j, t), dh = decode8<BITS>(ch, j, t);
#pragma unroll
        for (int n = 0; n < NT; ++n) {
          const uint4 a = (valid && 8 * n + g < p.T)
                              ? __ldg(reinterpret_cast<const uint4*>(arow + (size_t)(8 * n) * p.K + pos0) + j)
                              : make_uint4(0u, 0u, 0u, 0u);
          mma_f16_16816(acc[n], dl.x, dh.x, dl.y, dh.y, a.x, a.y);
          mma_f16_16816(acc[n], dl.z, dh.z, dl.w, dh.w, a.z, a.w);
        }
      }
    }
  }
  // the warps' partial sums, added in warp order
#pragma unroll
  for (int n = 0; n < NT; ++n)
    *reinterpret_cast<float4*>(part[warp][n][lane]) = make_float4(acc[n][0], acc[n][1], acc[n][2], acc[n][3]);
  __syncthreads();
  if (warp >= NT) return;
  // warp n writes token tile n
  const int n = warp;
  float s[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int w = 0; w < NWARP; ++w) {
    const float4 v = *reinterpret_cast<const float4*>(part[w][n][lane]);
    s[0] += v.x;
    s[1] += v.y;
    s[2] += v.z;
    s[3] += v.w;
  }
  // accumulator (row m, column c): d0 = (g, 2q), d1 = (g, 2q + 1),
  // d2 = (g + 8, 2q), d3 = (g + 8, 2q + 1); rows are weight rows, column c is
  // token 8 n + c
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int o = o0 + g + 8 * (i >> 1), tk = 8 * n + 2 * q + (i & 1);
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

template <int BITS>
cudaError_t launch_bits(const GemvParams& kp, unsigned grid, cudaStream_t s) {
  switch ((kp.T + 7) / 8) {
    case 1: gemv_kernel<BITS, 1><<<grid, NWARP * 32, 0, s>>>(kp); break;
    case 2: gemv_kernel<BITS, 2><<<grid, NWARP * 32, 0, s>>>(kp); break;
    default: gemv_kernel<BITS, 3><<<grid, NWARP * 32, 0, s>>>(kp); break;
  }
  return cudaGetLastError();
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
  cudaError_t e;
  switch (g.b_bits) {
    case 2: e = launch_bits<2>(kp, grid, s); break;
    case 3: e = launch_bits<3>(kp, grid, s); break;
    default: e = launch_bits<4>(kp, grid, s); break;
  }
  if (e != cudaSuccess) {
    set_error(std::string("gemv launch: ") + cudaGetErrorString(e));
    return OQ_ERR_CUDA;
  }
  return OQ_OK;
}

}  // namespace oq
