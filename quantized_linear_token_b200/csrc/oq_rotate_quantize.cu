// Rotate + quantize: the online activation codec of OrbitQuant (also used
// offline for weight rows).  Per row x of length d (gecl notes Method 1, 2, 4;
// pith Supplementary A):
//   s = ||x||_2,  y = P_pi x,  z_j = H_h y_j (block j, unnormalised),
//   code_i = #{k : t_k < z_i / (s sqrt(h))}   (t = Lloyd-Max thresholds),
// codes packed b bits each, 32 per group of b words, little-endian.
//
// Layout of the work, for one row ("token slot", d/E threads; the block size
// h is a compile-time constant so that every index below is fixed):
//   * the row is copied into shared memory with one bulk async copy (double
//     buffered: the next row streams in while this one is processed);
//   * pass A: thread (j, c) of block j gathers the E rotated positions
//     c + r (h/E), r = 0..E-1, through pi (gather offsets held in registers)
//     and applies the butterflies of the high log2(E) bits in registers;
//   * the values go through shared memory in a layout where every thread of
//     pass B owns E consecutive positions (the 16-byte sub-chunks of chunk q
//     are XOR-swizzled by q, so both the scattered writes -- one LOP3 of a
//     compile-time offset per value -- and the vector reads are free of bank
//     conflicts);
//   * pass B applies the remaining low bits, compares with the thresholds
//     scaled by s sqrt(h), packs and stores the codes with vector stores (or,
//     for the fused layer call, stores the codes' fp16 levels: the operand
//     the tensor-core contraction reads).
// Butterflies with stride >= 2 use the paired fp32 adds of sm_100 (f32x2).
// When h <= 64 a thread holds a whole block and pass B is skipped.
#include <cuda_bf16.h>

#include <algorithm>
#include <cstring>

#include "oq_decode.cuh"
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
  int d, NT, S;
  int work_words;      // per slot
  int stage_bytes;     // per buffer per slot
  int has_signs;
  const uint16_t* gather;
  const uint32_t* signmask;
  uint32_t* codes;     // packed codes, or
  uint16_t* out16;     // fp16 levels [rows, d] (fused layer call)
  float* norms;
  int* err;
  const uint2* bins;   // threshold search table {TK bits, base code | fp16 level pair}
  int nb, b0;
  float kscale;        // g = z * kscale / s in bin units
};

template <typename XT>
__device__ __forceinline__ float load_x(uint32_t stage_addr, uint32_t idx) {
  if constexpr (sizeof(XT) == 2) {
    uint16_t v;
    asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(stage_addr + 2u * idx));
    return __uint_as_float(((uint32_t)v) << 16);
  } else {
    float v;
    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(stage_addr + 4u * idx));
    return v;
  }
}

// (a0, a1) <- (a0 + b0, a1 + b1), (b0, b1) <- (a0 - b0, a1 - b1) with the
// paired fp32 adds of sm_100
__device__ __forceinline__ void bfly2(float& a0, float& a1, float& b0, float& b1) {
  asm("{\n\t.reg .b64 A, B, S, D;\n\t"
      "mov.b64 A, {%0, %1};\n\tmov.b64 B, {%2, %3};\n\t"
      "add.rn.f32x2 S, A, B;\n\tsub.rn.f32x2 D, A, B;\n\t"
      "mov.b64 {%0, %1}, S;\n\tmov.b64 {%2, %3}, D;\n\t}"
      : "+f"(a0), "+f"(a1), "+f"(b0), "+f"(b1));
}

// in-register Walsh-Hadamard butterflies over register-index bits [LO, HI)
template <int E, int LO, int HI>
__device__ __forceinline__ void fwht_regs(float (&v)[E]) {
#pragma unroll
  for (int s = (1 << LO); s < (1 << HI); s <<= 1) {
    if (s == 1) {
#pragma unroll
      for (int r = 0; r < E; r += 2) {
        const float a = v[r], b = v[r + 1];
        v[r] = a + b;
        v[r + 1] = a - b;
      }
    } else {
#pragma unroll
      for (int r = 0; r < E; r += 2)
        if ((r & s) == 0) bfly2(v[r], v[r + 1], v[r + s], v[r + s + 1]);
    }
  }
}

// Word offset (inside its block) of the value that thread c of a block holds
// in register r after pass A, minus the thread-dependent part: the value at
// in-block position pos = c + r*HE lives in chunk q = pos / E, sub-chunk
// v = (pos % E) / 4 stored at slot v ^ (q mod E/4).  With cb = c / 4 and
// pos % E = A_r + c (A_r a multiple of HE), the offset is
//   (scatter_imm(r) ^ 4 cb) | (c & 3).
template <int E, int HE>
__host__ __device__ constexpr uint32_t scatter_imm(int r) {
  return (uint32_t)(E * ((r * HE) / E) + 4 * ((((r * HE) % E) / 4) ^ (((r * HE) / E) & (E / 4 - 1))));
}

__host__ __device__ constexpr int elems_per_thread(int h) { return h <= 64 ? h : (h <= 1024 ? 32 : 64); }
__host__ __device__ constexpr int log2i(int x) { return x <= 1 ? 0 : 1 + log2i(x / 2); }

// register budget: 96 for 32 values per thread (seven CTAs of 96 threads per
// SM), 168 for 64 values per thread
template <int BITS, int LOG_H, typename XT, bool OUT16>
__global__ void __maxnreg__(elems_per_thread(1 << LOG_H) == 64 ? 168 : 96)
    rq_kernel(const __grid_constant__ RQKParams p) {
  constexpr int H = 1 << LOG_H;
  constexpr int E = elems_per_thread(H);
  constexpr int LOGE = log2i(E);
  constexpr int HE = H / E;
  constexpr int PASSES = (H <= 64) ? 1 : 2;
  constexpr int PAD = (PASSES == 2 && HE < 32) ? HE : 0;   // words between blocks
  extern __shared__ __align__(1024) unsigned char smem[];

  const int S = p.S, NT = p.NT, d = p.d;
  const int slot_raw = threadIdx.x / NT;
  const bool active = slot_raw < S;
  const int slot = active ? slot_raw : 0;
  const int tid = active ? (int)threadIdx.x - slot * NT : 0;
  const int j = tid / HE, c = tid % HE;

  // shared memory: mbarriers | reduction partials | threshold search table |
  // gather offsets | slots (two row buffers + exchange area each)
  uint64_t* mbar = reinterpret_cast<uint64_t*>(smem);
  float* red = reinterpret_cast<float*>(smem + 16 * S);
  const int tbl_off = (16 * S + 4 * blockDim.x + 15) & ~15;
  uint2* tbl = reinterpret_cast<uint2*>(smem + tbl_off);
  const int gtab_off = (tbl_off + 8 * p.nb + 15) & ~15;
  uint4* gtab = reinterpret_cast<uint4*>(smem + gtab_off);   // [E/8][NT]: conflict-free per q
  unsigned char* slots = smem + ((gtab_off + 2 * d + 1023) & ~1023);
  const int slot_bytes = 2 * p.stage_bytes + 4 * p.work_words;
  unsigned char* stage0 = slots + (size_t)slot * slot_bytes;
  float* work = reinterpret_cast<float*>(stage0 + 2 * p.stage_bytes);
  const uint32_t stage0_addr = smem_u32(stage0);

  // the gather offsets (16-bit channel indices, kernel order) go to shared
  // memory transposed so that a warp reads its threads' next eight offsets
  // with one conflict-free 16-byte load each; this thread's sign bits stay in
  // registers
  for (int i = threadIdx.x; i < d / 8; i += blockDim.x) {
    const int t = i % NT, q = i / NT;
    gtab[i] = __ldg(reinterpret_cast<const uint4*>(p.gather) + (size_t)t * (E / 8) + q);
  }
  uint32_t smask[E / 32 > 0 ? E / 32 : 1];
  {
#pragma unroll
    for (int q = 0; q < (E / 32 > 0 ? E / 32 : 1); ++q)
      smask[q] = (p.has_signs && active) ? __ldg(p.signmask + (size_t)tid * (E / 32) + q) : 0u;
  }
  for (int i = threadIdx.x; i < p.nb; i += blockDim.x) tbl[i] = __ldg(p.bins + i);
  const int nb1 = p.nb - 1, boff = p.b0 - 0x4B400000;
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2 * S; ++i) mbar_init(&mbar[i], 1);
    fence_mbar_init();
  }
  __syncthreads();

  const int64_t groups = (p.rows + S - 1) / S;
  const int words_per_row = d * BITS / 32;
  const uint32_t row_bytes = (uint32_t)d * (uint32_t)sizeof(XT);
  const unsigned char* src = static_cast<const unsigned char*>(p.src);
  // segmented warp reduction width: lanes of one slot share aligned segments
  const int W = NT & -NT;
  const int Wc = W < 32 ? W : 32;

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
    const uint32_t stage_addr = stage0_addr + (uint32_t)(buf * p.stage_bytes);
    float v[E];
    float ss = 0.f;
#pragma unroll
    for (int q = 0; q < E / 8; ++q) {
      const uint4 gq = gtab[q * NT + tid];
      const uint32_t gw[4] = {gq.x, gq.y, gq.z, gq.w};
#pragma unroll
      for (int e8 = 0; e8 < 8; ++e8) {
        const uint32_t gi = (e8 & 1) ? (gw[e8 >> 1] >> 16) : (gw[e8 >> 1] & 0xFFFFu);
        v[8 * q + e8] = valid ? load_x<XT>(stage_addr, gi) : 0.f;
      }
    }
    if (p.has_signs) {
#pragma unroll
      for (int r = 0; r < E; ++r)
        if ((smask[r >> 5] >> (r & 31)) & 1u) v[r] = -v[r];
    }
#pragma unroll
    for (int r = 0; r < E; ++r) ss = fmaf(v[r], v[r], ss);
    fwht_regs<E, 0, LOGE>(v);

    if constexpr (PASSES == 2) {
      if (active) {
        float* wb = work + j * (H + PAD);
        const uint32_t cb4 = (uint32_t)(c >> 2) << 2, c3 = (uint32_t)(c & 3);
#pragma unroll
        for (int r = 0; r < E; ++r) wb[(scatter_imm<E, HE>(r) ^ cb4) | c3] = v[r];
      }
    }

    // ---------------- norm: segmented warp reduction, then per slot
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1)
      if (off < Wc) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    if ((threadIdx.x & (Wc - 1)) == 0) red[threadIdx.x / Wc] = ss;

    const int failed = __syncthreads_or(!ok);
    if (failed) {
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
      const float* wb = work + j * (H + PAD) + c * E;
#pragma unroll
      for (int q = 0; q < E / 4; ++q) {
        const float4 f = *reinterpret_cast<const float4*>(wb + ((q ^ (c & (E / 4 - 1))) << 2));
        z[4 * q + 0] = f.x;
        z[4 * q + 1] = f.y;
        z[4 * q + 2] = f.z;
        z[4 * q + 3] = f.w;
      }
      fwht_regs<E, 0, LOG_H - LOGE>(z);
    } else {
#pragma unroll
      for (int r = 0; r < E; ++r) z[r] = v[r];
    }

    if (valid) {
      // g = sqrt(d) K u with u = z / (s sqrt(h)): bin rint(g) (by the fp32
      // magic-number round), clamped to the table, then one compare against
      // the bin's threshold: code = #{thresholds below g} exactly (a value on
      // a threshold takes the lower code).  A zero token (s = 0) gets g = 0 and
      // code L/2 - 1; non-finite values land in a clamped bin.
      const float ks = (s > 0.f) ? p.kscale / s : 0.f;
      const int pos0 = (PASSES == 2) ? (j * H + c * E) : (j * H);
      const int boffv = boff;
#pragma unroll
      for (int gi = 0; gi < E / 32; ++gi) {
        if constexpr (OUT16) {
          // the codes' fp16 levels (the contraction's A operand), two per
          // word, eight per 16-byte chunk
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint32_t o[4];
#pragma unroll
            for (int i = 0; i < 8; i += 2) {
              uint32_t sel = 0u, pay[2];
#pragma unroll
              for (int e2 = 0; e2 < 2; ++e2) {
                const float g = z[gi * 32 + q * 8 + i + e2] * ks;
                int m = __float_as_int(g + 12582912.0f) + boffv;
                m = min(max(m, 0), nb1);
                const uint2 en = tbl[m];
                pay[e2] = en.y;
                const bool up = g > __uint_as_float(en.x);
                sel |= (up ? 0x32u : 0x10u) << (8 * e2);
              }
              o[i >> 1] = __byte_perm(pay[0], pay[1], sel | 0x4400u);
            }
            const uint4 ch = make_uint4(o[0], o[1], o[2], o[3]);
            if constexpr (PASSES == 2) {
              // into this thread's own exchange region (its z values are
              // already in registers), slot swizzled by c so that both this
              // store and the group reads below are free of bank conflicts
              reinterpret_cast<uint4*>(work + j * (H + PAD) + c * E)[(gi * 4 + q) ^ (c & 7)] = ch;
            } else {
              reinterpret_cast<uint4*>(p.out16 + (size_t)t * d + pos0 + gi * 32)[q] = ch;
            }
          }
        } else {
          // 32 consecutive positions straight into BITS packed words
          uint32_t w[BITS];
#pragma unroll
          for (int q = 0; q < BITS; ++q) w[q] = 0u;
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float g = z[gi * 32 + i] * ks;
            int m = __float_as_int(g + 12582912.0f) + boffv;
            m = min(max(m, 0), nb1);
            const uint2 en = tbl[m];
            const uint32_t cv = en.y + (g > __uint_as_float(en.x) ? 1u : 0u);
            const int bit = i * BITS;
            w[bit >> 5] |= cv << (bit & 31);
            if ((bit & 31) + BITS > 32) w[(bit >> 5) + 1] |= cv >> (32 - (bit & 31));
          }
          uint32_t* dst = p.codes + (size_t)t * words_per_row + (size_t)((pos0 >> 5) + gi) * BITS;
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
      }
      if (tid == 0) p.norms[t] = s;
    }
    if constexpr (OUT16 && PASSES == 2) {
      // Each thread's 32 fp16 levels are 64 contiguous output bytes; stored
      // directly, a warp's 16-byte stores would land 64 bytes apart and write
      // every 32-byte sector in halves.  Instead the four threads of a group
      // (consecutive c, one row, one warp) swap chunks through their exchange
      // regions: in store qq lane i writes chunk i of thread c0 + qq, so each
      // store of the group covers 64 contiguous bytes (two whole sectors).
      __syncwarp();
      if (valid) {
        const int i4 = c & 3, c0 = c & ~3;
        const float* base = work + j * (H + PAD) + c0 * E;
        uint16_t* rowout = p.out16 + (size_t)t * d + j * H;
#pragma unroll
        for (int gi = 0; gi < E / 32; ++gi) {
#pragma unroll
          for (int qq = 0; qq < 4; ++qq) {
            const int cs = c0 + qq;
            const uint4 ch = reinterpret_cast<const uint4*>(base + qq * E)[(gi * 4 + i4) ^ (cs & 7)];
            reinterpret_cast<uint4*>(rowout + cs * E + gi * 32)[i4] = ch;
          }
        }
      }
    }
    __syncthreads();
  }
}

template <int BITS, int LOG_H, typename XT, bool OUT16>
oq_status launch_t(const RQKParams& kp_in, void* stream) {
  constexpr int H = 1 << LOG_H;
  constexpr int E = elems_per_thread(H);
  constexpr int MAXT = (E == 64) ? 256 : 448;
  RQKParams kp = kp_in;
  auto kern = rq_kernel<BITS, LOG_H, XT, OUT16>;
  const int NT = kp.NT;
  // one row per CTA once a row has 64 threads: small CTAs pack into the SM
  // sub-partitions' register files better than 6-warp ones
  int S = 1;
  while (S * NT < 64 && S < 64) S *= 2;
  const int threads = ((S * NT + 31) / 32) * 32;
  if (threads > MAXT) return OQ_ERR_UNSUPPORTED;
  kp.S = S;
  kp.stage_bytes = (int)(((size_t)kp.d * sizeof(XT) + 15) & ~(size_t)15);
  const int slot_bytes = 2 * kp.stage_bytes + 4 * kp.work_words;
  const size_t head = ((((((16 * S + 4 * threads + 15) & ~(size_t)15) + 8 * (size_t)kp.nb + 15) & ~(size_t)15) +
                        2 * (size_t)kp.d) + 1023) & ~(size_t)1023;
  const size_t smem = head + (size_t)S * slot_bytes;
  if (smem > 227 * 1024) return OQ_ERR_UNSUPPORTED;
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
  const int64_t groups = (kp.rows + S - 1) / S;
  const int64_t grid = std::min<int64_t>(groups, (int64_t)sms * per_sm);
  kern<<<(unsigned)grid, threads, smem, static_cast<cudaStream_t>(stream)>>>(kp);
  e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error(std::string("rotate_quantize launch: ") + cudaGetErrorString(e));
    return OQ_ERR_CUDA;
  }
  return OQ_OK;
}

template <int BITS, typename XT, bool OUT16>
oq_status launch_h(const RQKParams& kp, int log_h, void* stream) {
  switch (log_h) {
    case 5: return launch_t<BITS, 5, XT, OUT16>(kp, stream);
    case 6: return launch_t<BITS, 6, XT, OUT16>(kp, stream);
    case 7: return launch_t<BITS, 7, XT, OUT16>(kp, stream);
    case 8: return launch_t<BITS, 8, XT, OUT16>(kp, stream);
    case 9: return launch_t<BITS, 9, XT, OUT16>(kp, stream);
    case 10: return launch_t<BITS, 10, XT, OUT16>(kp, stream);
    case 11: return launch_t<BITS, 11, XT, OUT16>(kp, stream);
    case 12: return launch_t<BITS, 12, XT, OUT16>(kp, stream);
    default: return OQ_ERR_UNSUPPORTED;
  }
}

template <int BITS>
oq_status launch_bits(const RQKParams& kp, const RQArgs& a, void* stream) {
  const bool bf = a.src_dtype == OQ_DTYPE_BF16;
  if (a.out16) {
    // fp16 operand output only for bf16 activations (the fused layer call)
    if (!bf) return OQ_ERR_UNSUPPORTED;
    return launch_h<BITS, __nv_bfloat16, true>(kp, a.log_h, stream);
  }
  if (bf) return launch_h<BITS, __nv_bfloat16, false>(kp, a.log_h, stream);
  return launch_h<BITS, float, false>(kp, a.log_h, stream);
}

}  // namespace

oq_status rq_launch(const RQArgs& a, void* stream) {
  if (a.rows == 0) return OQ_OK;
  RQKParams kp;
  std::memset(&kp, 0, sizeof(kp));
  kp.src = a.src;
  kp.rows = a.rows;
  kp.d = a.d;
  const int E = rq_elems_per_thread(a.h);
  kp.NT = a.d / E;
  const int HE = a.h / E;
  kp.work_words = (a.h <= 64) ? 0 : (a.d / a.h) * (a.h + (HE < 32 ? HE : 0));
  kp.has_signs = a.signmask != nullptr;
  kp.gather = a.gather;
  kp.signmask = a.signmask;
  kp.codes = a.codes;
  kp.out16 = a.out16;
  kp.norms = a.norms;
  kp.err = a.err;
  kp.bins = reinterpret_cast<const uint2*>(a.bins);
  kp.nb = a.nb;
  kp.b0 = a.b0;
  kp.kscale = a.kscale;
  if (a.nb < 1 || a.nb > OQ_MAX_BINS) return OQ_ERR_UNSUPPORTED;
  switch (a.bits) {
    case 2: return launch_bits<2>(kp, a, stream);
    case 3: return launch_bits<3>(kp, a, stream);
    case 4: return launch_bits<4>(kp, a, stream);
    case 8: return launch_bits<8>(kp, a, stream);
    default: return OQ_ERR_UNSUPPORTED;
  }
}

}  // namespace oq
