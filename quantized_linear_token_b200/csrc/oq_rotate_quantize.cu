// Rotate + quantize: the online activation codec of OrbitQuant (also used
// offline for weight rows).  Per row x of length d (gecl notes Method 1, 2, 4;
// pith Supplementary A):
//   s = ||x||_2,  y = P_pi x,  z_j = H_h y_j (block j, unnormalised),
//   code_i = #{k : t_k < z_i / (s sqrt(h))}   (t = Lloyd-Max thresholds),
// codes packed b bits each, 32 per group of b words, little-endian.
//
// Layout of the work, for one row ("token slot", d/E threads):
//   * the row is copied into shared memory with one bulk async copy (double
//     buffered: the next row streams in while this one is processed);
//   * pass A: thread (j, c) of block j gathers the E rotated positions
//     c + r (h/E), r = 0..E-1, through pi (gather offsets held in registers)
//     and applies the butterflies of the high log2(E) bits in registers;
//   * the values go through shared memory in a layout where every thread of
//     pass B owns E consecutive positions (16-byte sub-chunks rotated by
//     chunk index, so both the scattered writes and the vector reads are free
//     of bank conflicts);
//   * pass B applies the remaining low bits, compares with the thresholds
//     scaled by s sqrt(h), packs and stores the codes with vector stores.
// When h <= 64 a thread holds a whole block and pass B is skipped.
#include <cuda_bf16.h>

#include <algorithm>
#include <cstring>

#include "oq_internal.h"
#include "oq_ptx.cuh"

namespace oq {

int rq_elems_per_thread(int h) { return h <= 64 ? h : (h <= 1024 ? 32 : 64); }

// Kernel order of the gather table: entry tid*E + r is the input channel of
// rotated position j*h + c + r*(h/E), with j = tid / (h/E), c = tid % (h/E).
void rq_build_gather(int d, int h, const std::vector<uint32_t>& perm, const std::vector<int8_t>* signs,
                     std::vector<uint16_t>& gather, std::vector<uint32_t>& signmask) {
  const int E = rq_elems_per_thread(h), HE = h / E, NT = d / E;
  gather.assign((size_t)NT * E, 0);
  signmask.assign((size_t)NT * (E / 32), 0);
  for (int tid = 0; tid < NT; ++tid) {
    const int j = tid / HE, c = tid % HE;
    for (int r = 0; r < E; ++r) {
      const int pos = j * h + c + r * HE;
      gather[(size_t)tid * E + r] = (uint16_t)perm[pos];
      if (signs && (*signs)[pos] < 0) signmask[(size_t)tid * (E / 32) + r / 32] |= 1u << (r % 32);
    }
  }
}

namespace {

struct RQKParams {
  const void* src;
  int64_t rows;
  int d, h, log_h, NT, S, e;
  int work_words;      // per slot
  int stage_bytes;     // per buffer per slot
  const uint16_t* gather;
  const uint32_t* signmask;
  uint32_t* codes;
  float* norms;
  int* err;
  float thr[128];      // sqrt(h) * positive thresholds tau_1.., +inf padded
};

template <typename XT>
__device__ __forceinline__ float load_x(const unsigned char* stage, uint32_t idx) {
  if constexpr (sizeof(XT) == 2) {
    const unsigned short v = *reinterpret_cast<const unsigned short*>(stage + 2u * idx);
    return __uint_as_float(((uint32_t)v) << 16);
  } else {
    return *reinterpret_cast<const float*>(stage + 4u * idx);
  }
}

// in-register Walsh-Hadamard butterflies over register-index bits [lo, hi)
template <int E, int LO, int HI>
__device__ __forceinline__ void fwht_regs(float (&v)[E]) {
#pragma unroll
  for (int s = (1 << LO); s < (1 << HI); s <<= 1) {
#pragma unroll
    for (int r = 0; r < E; ++r) {
      if ((r & s) == 0) {
        const float a = v[r], b = v[r + s];
        v[r] = a + b;
        v[r + s] = a - b;
      }
    }
  }
}

// number of thresholds strictly below `a` among th[0..n-1] (sorted, last = +inf)
template <int BITS>
__device__ __forceinline__ int count_below(const float* th, float a) {
  if constexpr (BITS == 2) {
    return th[0] < a ? 1 : 0;
  } else if constexpr (BITS == 3) {
    const bool c1 = th[1] < a;
    const float t2 = c1 ? th[2] : th[0];
    const bool c2 = t2 < a;
    return (c1 ? 2 : 0) + (c2 ? 1 : 0);
  } else {
    static_assert(BITS == 4, "register search for 2..4 bits");
    const bool c1 = th[3] < a;
    const float t2 = c1 ? th[5] : th[1];
    const bool c2 = t2 < a;
    const float t3 = c1 ? (c2 ? th[6] : th[4]) : (c2 ? th[2] : th[0]);
    const bool c3 = t3 < a;
    return (c1 ? 4 : 0) + (c2 ? 2 : 0) + (c3 ? 1 : 0);
  }
}

template <int BITS, int E, int PASSES, typename XT, bool SIGNS>
__global__ void __launch_bounds__(E == 64 ? 256 : 448) rq_kernel(const __grid_constant__ RQKParams p) {
  constexpr int N_HALF = 1 << (BITS - 1);   // levels on each side of 0
  constexpr int NTH = (BITS <= 4) ? N_HALF : 1;
  extern __shared__ __align__(1024) unsigned char smem[];

  const int S = p.S, NT = p.NT, d = p.d, h = p.h;
  const int HE = h / E;
  const int slot_raw = threadIdx.x / NT;
  const bool active = slot_raw < S;
  const int slot = active ? slot_raw : 0;
  const int tid = active ? (int)threadIdx.x - slot * NT : 0;
  const int j = tid / HE, c = tid - (tid / HE) * HE;

  // shared memory: mbarriers | reduction partials | 8-bit thresholds | slots
  uint64_t* mbar = reinterpret_cast<uint64_t*>(smem);                      // [S][2]
  float* red = reinterpret_cast<float*>(smem + 16 * S);                    // [blockDim]
  float* thr8 = red + blockDim.x;                                          // [S][128] (8-bit)
  unsigned char* slots = smem + (((16 * S + 4 * blockDim.x + (BITS == 8 ? 512 * S : 0)) + 1023) & ~1023);
  const int slot_bytes = 2 * p.stage_bytes + 4 * p.work_words;
  unsigned char* stage0 = slots + (size_t)slot * slot_bytes;
  float* work = reinterpret_cast<float*>(stage0 + 2 * p.stage_bytes);

  // gather offsets and sign bits of this thread, kept in registers
  uint32_t gidx[E / 2];
  uint32_t smask[E / 32];
  {
    const uint4* g4 = reinterpret_cast<const uint4*>(p.gather + (size_t)tid * E);
#pragma unroll
    for (int q = 0; q < E / 8; ++q) {
      const uint4 v = active ? __ldg(g4 + q) : make_uint4(0, 0, 0, 0);
      gidx[4 * q + 0] = v.x;
      gidx[4 * q + 1] = v.y;
      gidx[4 * q + 2] = v.z;
      gidx[4 * q + 3] = v.w;
    }
#pragma unroll
    for (int q = 0; q < E / 32; ++q) smask[q] = (SIGNS && active) ? __ldg(p.signmask + (size_t)tid * (E / 32) + q) : 0u;
  }
  float th[NTH];
#pragma unroll
  for (int k = 0; k < NTH; ++k) th[k] = p.thr[k];

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2 * S; ++i) mbar_init(&mbar[i], 1);
    fence_mbar_init();
  }
  __syncthreads();

  const int64_t groups = (p.rows + S - 1) / S;
  const int words_per_row = d * BITS / 32;
  const uint32_t row_bytes = (uint32_t)d * (uint32_t)sizeof(XT);
  const unsigned char* src = static_cast<const unsigned char*>(p.src);

  // prologue: first row of this slot
  if (active && tid == 0) {
    const int64_t t0 = (int64_t)blockIdx.x * S + slot;
    if ((int64_t)blockIdx.x < groups && t0 < p.rows) {
      mbar_arrive_expect_tx(&mbar[2 * slot], row_bytes);
      bulk_g2s(stage0, src + (size_t)t0 * row_bytes, row_bytes, &mbar[2 * slot]);
    }
  }

  int it = 0;
  for (int64_t G = blockIdx.x; G < groups; G += gridDim.x, ++it) {
    const int64_t t = G * S + slot;
    const bool valid = active && t < p.rows;
    const int buf = it & 1;
    // prefetch the next row of this slot into the other buffer
    bool issued = false;
    if (active && tid == 0) {
      const int64_t Gn = G + gridDim.x, tn = Gn * S + slot;
      if (Gn < groups && tn < p.rows) {
        issued = true;
        mbar_arrive_expect_tx(&mbar[2 * slot + (buf ^ 1)], row_bytes);
        bulk_g2s(stage0 + (buf ^ 1) * p.stage_bytes, src + (size_t)tn * row_bytes, row_bytes,
                 &mbar[2 * slot + (buf ^ 1)]);
      }
    }
    bool ok = true;
    if (valid) ok = mbar_wait(&mbar[2 * slot + buf], (uint32_t)(it >> 1) & 1u, p.err);

    // ---------------- pass A: gather through pi, high-bit butterflies
    const unsigned char* stage = stage0 + buf * p.stage_bytes;
    float v[E];
    float ss = 0.f;
#pragma unroll
    for (int r = 0; r < E; ++r) {
      const uint32_t gi = (r & 1) ? (gidx[r >> 1] >> 16) : (gidx[r >> 1] & 0xFFFFu);
      float x = valid ? load_x<XT>(stage, gi) : 0.f;
      if constexpr (SIGNS) {
        if ((smask[r >> 5] >> (r & 31)) & 1u) x = -x;
      }
      ss = fmaf(x, x, ss);
      v[r] = x;
    }
    constexpr int LOGE = (E == 32) ? 5 : (E == 64 ? 6 : (E == 16 ? 4 : 0));
    static_assert(LOGE > 0, "E must be 16, 32 or 64");
    fwht_regs<E, 0, LOGE>(v);

    if (PASSES == 2 && active) {
      // scatter into the pass-B layout of block j (see file comment)
      const int pad = HE < 32 ? HE : 0;
      float* wb = work + j * (h + pad);
#pragma unroll
      for (int r = 0; r < E; ++r) {
        const int pos = c + r * HE;
        const int q = pos / E, w = pos - q * E;
        wb[q * E + ((((w >> 2) + q) & (E / 4 - 1)) << 2) + (w & 3)] = v[r];
      }
    }

    // ---------------- norm: segmented warp reduction, then per slot
    const int W = NT & -NT;                      // lanes per aligned segment
    const int Wc = W < 32 ? W : 32;
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1)
      if (off < Wc) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    if ((threadIdx.x & (Wc - 1)) == 0) red[threadIdx.x / Wc] = ss;

    const int failed = __syncthreads_or(!ok);
    if (failed) {
      // let a copy still in flight land before the CTA leaves (bounded)
      if (issued) mbar_wait(&mbar[2 * slot + (buf ^ 1)], (uint32_t)((it + 1) >> 1) & 1u, p.err);
      break;
    }

    float s2 = 0.f;
    {
      const int base = (slot * NT) / Wc, cnt = NT / Wc;
      for (int q = 0; q < cnt; ++q) s2 += red[base + q];
    }
    const float s = sqrtf(s2);

    // ---------------- pass B: low-bit butterflies, quantize, pack
    float z[E];
    if constexpr (PASSES == 2) {
      const int pad = HE < 32 ? HE : 0;
      const float* wb = work + j * (h + pad) + c * E;
#pragma unroll
      for (int q = 0; q < E / 4; ++q) {
        const float4 f = *reinterpret_cast<const float4*>(wb + (((q + c) & (E / 4 - 1)) << 2));
        z[4 * q + 0] = f.x;
        z[4 * q + 1] = f.y;
        z[4 * q + 2] = f.z;
        z[4 * q + 3] = f.w;
      }
    } else {
#pragma unroll
      for (int r = 0; r < E; ++r) z[r] = v[r];
    }

    if constexpr (PASSES == 2) {
      // remaining bits [0, log_h - LOGE): at most LOGE of them
      const int nb = p.log_h - LOGE;
#pragma unroll
      for (int b = 0; b < LOGE; ++b) {
        if (b < nb) {
          const int st = 1 << b;
#pragma unroll
          for (int r = 0; r < E; ++r) {
            if ((r & st) == 0) {
              const float a0 = z[r], b0 = z[r + st];
              z[r] = a0 + b0;
              z[r + st] = a0 - b0;
            }
          }
        }
      }
    }

    if constexpr (BITS == 8) {
      // this token's scaled thresholds (127 and +inf) in shared memory
      if (valid)
        for (int k = tid; k < 128; k += NT) thr8[slot * 128 + k] = p.thr[k] * s;
      __syncthreads();
    }

    if (valid) {
      float ts[NTH];
#pragma unroll
      for (int k = 0; k < NTH; ++k) ts[k] = th[k] * s;
      const int pos0 = (PASSES == 2) ? (j * h + c * E) : (j * h);
      uint32_t* crow = p.codes + (size_t)t * words_per_row;
#pragma unroll
      for (int gi = 0; gi < E / 32; ++gi) {
        // quantize 32 consecutive positions straight into BITS packed words
        uint32_t w[BITS];
#pragma unroll
        for (int q = 0; q < BITS; ++q) w[q] = 0u;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float zz = z[gi * 32 + i];
          const float a = fabsf(zz);
          const bool pos = zz > 0.f;
          // ties: a value exactly on a threshold takes the lower code, i.e.
          // count t < a for positive values and t <= a for the others
          const float acmp = pos ? a : __uint_as_float(__float_as_uint(a) + 1u);
          int cnt;
          if constexpr (BITS <= 4) {
            cnt = count_below<BITS>(ts, acmp);
          } else {
            const float* t8 = thr8 + slot * 128;
            int lo = 0;
#pragma unroll
            for (int st = 64; st >= 1; st >>= 1)
              if (t8[lo + st - 1] < acmp) lo += st;
            cnt = lo;
          }
          int cd = pos ? (N_HALF + cnt) : (N_HALF - 1 - cnt);
          if (s == 0.f) cd = N_HALF - 1;
          const uint32_t cv = (uint32_t)cd;
          const int bit = i * BITS;
          w[bit >> 5] |= cv << (bit & 31);
          if ((bit & 31) + BITS > 32) w[(bit >> 5) + 1] |= cv >> (32 - (bit & 31));
        }
        uint32_t* dst = crow + (size_t)((pos0 >> 5) + gi) * BITS;
        if constexpr (BITS == 4) {
          *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
        } else if constexpr (BITS == 2) {
          *reinterpret_cast<uint2*>(dst) = make_uint2(w[0], w[1]);
        } else if constexpr (BITS == 8) {
          reinterpret_cast<uint4*>(dst)[0] = make_uint4(w[0], w[1], w[2], w[3]);
          reinterpret_cast<uint4*>(dst)[1] = make_uint4(w[4], w[5], w[6], w[7]);
        } else {
#pragma unroll
          for (int q = 0; q < BITS; ++q) dst[q] = w[q];
        }
      }
      if (tid == 0) p.norms[t] = s;
    }
    __syncthreads();
  }
}

template <int BITS, int E, int PASSES, typename XT, bool SIGNS>
oq_status launch_t(const RQArgs& a, const RQKParams& kp_in, void* stream) {
  RQKParams kp = kp_in;
  auto kern = rq_kernel<BITS, E, PASSES, XT, SIGNS>;
  const int NT = kp.NT;
  int S = 1;
  while (S * NT < 128 && S < 64) S *= 2;
  const int threads = ((S * NT + 31) / 32) * 32;
  if (threads > (E == 64 ? 256 : 448)) return OQ_ERR_UNSUPPORTED;
  kp.S = S;
  kp.stage_bytes = (int)(((size_t)a.d * sizeof(XT) + 15) & ~(size_t)15);
  const int slot_bytes = 2 * kp.stage_bytes + 4 * kp.work_words;
  const size_t head = ((16 * S + 4 * threads + (BITS == 8 ? 512 * S : 0)) + 1023) & ~(size_t)1023;
  const size_t smem = head + (size_t)S * slot_bytes;
  if (smem > 227 * 1024) return OQ_ERR_UNSUPPORTED;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) {
    set_error(std::string("cudaFuncSetAttribute: ") + cudaGetErrorString(e));
    return OQ_ERR_CUDA;
  }
  int dev = 0, sms = 0, per_sm = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, smem);
  if (per_sm < 1) per_sm = 1;
  const int64_t groups = (a.rows + S - 1) / S;
  const int64_t grid = std::min<int64_t>(groups, (int64_t)sms * per_sm);
  kern<<<(unsigned)grid, threads, smem, static_cast<cudaStream_t>(stream)>>>(kp);
  e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error(std::string("rotate_quantize launch: ") + cudaGetErrorString(e));
    return OQ_ERR_CUDA;
  }
  return OQ_OK;
}

}  // namespace

oq_status rq_launch(const RQArgs& a, void* stream) {
  if (a.rows == 0) return OQ_OK;
  RQKParams kp;
  std::memset(&kp, 0, sizeof(kp));
  kp.src = a.src;
  kp.rows = a.rows;
  kp.d = a.d;
  kp.h = a.h;
  kp.log_h = a.log_h;
  const int E = rq_elems_per_thread(a.h);
  kp.e = E;
  kp.NT = a.d / E;
  const int HE = a.h / E;
  kp.work_words = (a.h <= 64) ? 0 : (a.d / a.h) * (a.h + (HE < 32 ? HE : 0));
  kp.gather = a.gather;
  kp.signmask = a.signmask;
  kp.codes = a.codes;
  kp.norms = a.norms;
  kp.err = a.err;
  std::memcpy(kp.thr, a.thr, sizeof(kp.thr));
  const bool sg = a.signmask != nullptr;
  const bool bf = a.src_dtype == OQ_DTYPE_BF16;

#define OQ_RQ_CASE(BITS, EE, PP, XT, SG) \
  return launch_t<BITS, EE, PP, XT, SG>(a, kp, stream);
#define OQ_RQ_SHAPES(BITS, XT, SG)                                   \
  switch (a.h) {                                                     \
    case 32: OQ_RQ_CASE(BITS, 32, 1, XT, SG)                         \
    case 64: OQ_RQ_CASE(BITS, 64, 1, XT, SG)                         \
    case 128: case 256: case 512: case 1024: OQ_RQ_CASE(BITS, 32, 2, XT, SG) \
    case 2048: case 4096: OQ_RQ_CASE(BITS, 64, 2, XT, SG)            \
    default: return OQ_ERR_UNSUPPORTED;                              \
  }
#define OQ_RQ_DT(BITS)                                               \
  if (bf) {                                                          \
    if (sg) { OQ_RQ_SHAPES(BITS, __nv_bfloat16, true) }              \
    else { OQ_RQ_SHAPES(BITS, __nv_bfloat16, false) }                \
  } else {                                                           \
    if (sg) { OQ_RQ_SHAPES(BITS, float, true) }                      \
    else { OQ_RQ_SHAPES(BITS, float, false) }                        \
  }
  switch (a.bits) {
    case 2: OQ_RQ_DT(2)
    case 3: OQ_RQ_DT(3)
    case 4: OQ_RQ_DT(4)
    case 8: OQ_RQ_DT(8)
    default: return OQ_ERR_UNSUPPORTED;
  }
#undef OQ_RQ_DT
#undef OQ_RQ_SHAPES
#undef OQ_RQ_CASE
}

}  // namespace oq
