// The fused layer kernel: rotate + quantize as the producer of the
// contraction's A operand, inside the contraction kernel (gecl notes Method 2:
// the codes of R x meet the pre-rotated weight codes with no inverse rotation;
// llmdb Mathematical Formulation, y = Q_w(W R^-1) Q_a(R x)).
//
// One persistent CTA pair per two SMs runs two groups of warps side by side:
//   - producer teams (d / h warps each, several teams per CTA) claim groups
//     of RG token rows from a queue shared by the whole grid (one atomic
//     counter), stage each row with a bulk copy, compute its norm, block
//     Walsh-Hadamard transform and codes (oq_rqtc_dev.cuh: the arithmetic of
//     the stand-alone tensor-core rotate-quantize kernel), write the codes'
//     fp16 levels and the norms to the workspace, and publish the group with
//     a release flag;
//   - the contraction of oq_gemm_w16.cu: its TMA warp waits for the flags of
//     a tile's 128 A rows before loading them, so the tile's MMAs start as
//     soon as its rows exist, while the producers work ahead on later rows.
// The rotation runs on the CUDA cores and the legacy warp MMAs while the
// tcgen05 tensor cores contract earlier tiles; the fp16 A operand is written
// and read back through L2 shortly after.
//
// Forward progress needs no co-residency: a group is claimed only by a
// running team, whose producer loop waits on nothing but its own row copies
// and its own team's barriers, so every claimed group gets published; a
// consumer waiting for an unclaimed group belongs to a running CTA whose own
// teams keep claiming until the queue is empty.  Every wait is bounded.
//
// Warps: 0-3 epilogue, 4 TMA, 5 MMA issuer (even CTA) and tensor memory,
// 6.. producer teams.
#include <cuda.h>

#include <algorithm>
#include <cstring>

#include "oq_internal.h"
#include "oq_epilogue.cuh"
#include "oq_ptx.cuh"
#include "oq_rqcc_dev.cuh"
#include "oq_rqtc_dev.cuh"
#include "oq_tmap.cuh"

namespace oq {
namespace {

constexpr int RM = 128;            // A rows per CTA (pair M = 256)
constexpr int PN = 256;            // output columns per pair tile
constexpr int RN = 128;            // B rows per CTA
constexpr int BK = 64;             // K elements per stage
constexpr int MAX_OS = 6;          // operand stages (the launch picks 3 to 6)
constexpr int A_TILE = RM * BK * 2;
constexpr int B_TILE = RN * BK * 2;
constexpr int STAGE_BYTES = A_TILE + B_TILE;
constexpr int TMA_WARP = 4, MMA_WARP = 5, GEMM_WARPS = 6;
constexpr int MAX_WARPS = 18;      // register budget: 65536 / (18 * 32) = 113 per thread
constexpr uint32_t TMEM_COLS = 2 * PN;
constexpr uint32_t ACC_EMPTY_COUNT = 2 * 4;
constexpr int EPI_BYTES = 4 * 2 * 32 * 32 * 4;
constexpr int BAR_BYTES = 256;
constexpr int TEAM_HDR = 384;      // per team: 2 mbarriers, norm partials [2][32], two claim slots

struct FusedParams {
  CUtensorMap a_map;   // fp16 A [M, K] in the workspace, 128B-swizzled boxes of 128 x 64
  CUtensorMap b_map;   // fp16 B [N, K] (decoded weights), same boxes
  CUtensorMap y_map;   // fp32 y [M, N], boxes of 32 x 32
  const float* b_scale;
  float out_scale;
  bool y_bf16;         // y is bf16 (else fp32)
  int64_t M;
  int N, K, n_tiles, nkb;
  int64_t tiles;
  int* err;
  // producer
  const unsigned char* x;    // bf16 [M, K]
  uint16_t* a16;             // fp16 levels [M, K]
  float* norms;              // [M]
  int* flags;                // [n_items]: 1 once the group's rows are written
  int* counter;              // the queue's next group
  int n_items;               // ceil(M / RG)
  const uint16_t* gather;    // tensor-core gather table (kernel order)
  const uint2* bins;         // {threshold bits, fp16 level pair}
  int nb, b0, full;
  float kscale;
  int nw, teams;             // warps per team (d / h), teams per CTA
  int stage_bytes;           // one staged row, 128-byte multiple
  int row_bufs;              // staged rows per team: 2 (the next row loads during this one) or 1
  int os;                    // operand stages of the contraction
  int prod_off;              // byte offset of the producer region in shared memory
};

constexpr int RG = 4;              // token rows per queue group: 32 groups per 128-row tile
// the contraction's operand stages and the producer teams' staged rows: the
// shared memory left by the stages holds the teams, so these trade the
// contraction's latency cover against the number of producer warps
constexpr int kStages = 4;
constexpr int kRowBuffers = 2;

// Waits (bounded) until the `cnt` (<= 32) flags at f are all set, polling
// with every lane of the warp.  Each lane turns the relaxed read that saw its
// flag set into an acquire with a fence, and the warp then synchronises, so
// everything the producers wrote before their releases is visible to the
// lane that goes on to issue the TMA loads.
__device__ __forceinline__ bool wait_flags(const int* f, int cnt, int lane, int* err) {
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    const int v = lane < cnt ? ld_relaxed_gpu(f + lane) : 1;
    if (__all_sync(0xffffffffu, v != 0)) {
      fence_acq_rel_gpu();
      __syncwarp();
      return true;
    }
    // the lanes decide together, so the warp leaves the loop as one
    if (__any_sync(0xffffffffu, globaltimer_ns() - t0 > OQ_WAIT_NS)) {
      if (lane == 0) atomicOr(err, OQ_DEVERR_TIMEOUT);
      return false;
    }
    __nanosleep(128);
  }
}

// CC: the producers' block transform runs on the CUDA cores (h = 1024,
// oq_rqcc_dev.cuh: no warp MMAs, so they never wait behind the contraction's
// tcgen05 MMAs), with a 4 KB transpose tile per producer warp; otherwise on
// the warp MMAs (oq_rqtc_dev.cuh)
template <int A, bool CC>
__global__ void __cluster_dims__(2, 1, 1) __maxnreg__(112)
    fused_kernel(const __grid_constant__ FusedParams p) {
  constexpr int MT2 = A / 16, H = 32 * A;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const int OS = p.os;
  unsigned char* epi = smem + OS * STAGE_BYTES;
  uint64_t* op_full = reinterpret_cast<uint64_t*>(epi + EPI_BYTES);
  uint64_t* op_empty = op_full + MAX_OS;
  uint64_t* acc_full = op_empty + MAX_OS;
  uint64_t* acc_empty = acc_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
  // producer region: threshold table | gather offsets (transposed, uint4) | teams
  unsigned char* prod = smem + p.prod_off;
  uint2* tbl = reinterpret_cast<uint2*>(prod);
  const int team_threads = p.nw * 32;
  const int gtab_off = (8 * p.nb + 15) & ~15;
  uint4* gtab = reinterpret_cast<uint4*>(prod + gtab_off);
  const int teams_off = (gtab_off + 2 * A * team_threads + 127) & ~127;
  const int team_bytes = TEAM_HDR + (CC ? p.nw * 4096 : 0) + p.row_bufs * p.stage_bytes;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int64_t pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int nkb = p.nkb;
  const int my_tiles = (p.tiles > pair) ? (int)((p.tiles - 1 - pair) / npairs + 1) : 0;

  // ------------------------------------------------ set-up
  for (int i = threadIdx.x; i < p.nb; i += blockDim.x) tbl[i] = __ldg(p.bins + i);
  for (int i = threadIdx.x; i < (A / 8) * team_threads; i += blockDim.x) {
    const int t = i % team_threads, qq = i / team_threads;
    gtab[i] = __ldg(reinterpret_cast<const uint4*>(p.gather) + (size_t)t * (A / 8) + qq);
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < OS; ++s) {
      mbar_init(&op_full[s], 1);
      mbar_init(&op_empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], ACC_EMPTY_COUNT);
    }
    for (int tm = 0; tm < p.teams; ++tm) {
      uint64_t* tb = reinterpret_cast<uint64_t*>(prod + teams_off + tm * team_bytes);
      mbar_init(&tb[0], 1);
      mbar_init(&tb[1], 1);
    }
    fence_mbar_init();
  }
  if (warp == MMA_WARP) {
    tmem_alloc_pair(tmem_slot, TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t smem_base = smem_u32(smem);

  if (warp >= GEMM_WARPS) {
    // ------------------------------------------------ producer teams
    const int pw = warp - GEMM_WARPS, tm = pw / p.nw, w = pw % p.nw;
    const int ttid = w * 32 + lane;
    const bool leader = ttid == 0;
    const int bar_id = 1 + tm;
    unsigned char* tbase = prod + teams_off + tm * team_bytes;
    uint64_t* mbar = reinterpret_cast<uint64_t*>(tbase);
    float* red = reinterpret_cast<float*>(tbase + 16);
    volatile int* slot = reinterpret_cast<volatile int*>(tbase + 16 + 256);
    float* tile = reinterpret_cast<float*>(tbase + TEAM_HDR + w * 4096);   // CC only
    unsigned char* stage = tbase + TEAM_HDR + (CC ? p.nw * 4096 : 0);
    const uint32_t stage_addr0 = smem_u32(stage);
    const rqtc::Lane lc = rqtc::make_lane(lane);   // tensor-core transform only
    const uint32_t row_bytes = (uint32_t)p.K * 2u;
    const float magic = 12582912.0f + (float)p.b0;
    const int bin_lo = 0x4B400000, bin_hi = 0x4B400000 + p.nb - 1;
    const uint32_t tbl_shift = smem_u32(tbl) - 0x4B400000u * 8u;
    const int g = lane >> 2, q = lane & 3;

    if (leader) {
      const int item = atomicAdd(p.counter, 1);
      slot[0] = item;
      if (item < p.n_items) {
        mbar_arrive_expect_tx(&mbar[0], row_bytes);
        bulk_g2s(stage, p.x + (size_t)item * RG * row_bytes, row_bytes, &mbar[0]);
      }
    }
    named_bar_sync(bar_id, team_threads);
    int item = slot[0];
    int it = 0, done = 0;
    bool failed = false;
    // two row buffers: the next row's copy starts with this row; one: it
    // starts once every warp of the team has gathered this row
    const bool dbl = p.row_bufs == 2;
    // the row after t: the next in its group, or the first of a newly
    // claimed group (whose index the team reads from slot after the group)
    auto next_row = [&](int64_t t, int64_t r1) -> int64_t {
      if (t + 1 < r1) return t + 1;
      const int nitem = atomicAdd(p.counter, 1);
      slot[(done + 1) & 1] = nitem;
      return nitem < p.n_items ? (int64_t)nitem * RG : -1;
    };
    while (item < p.n_items && !failed) {
      const int64_t r0 = (int64_t)item * RG, r1 = (r0 + RG < p.M) ? r0 + RG : p.M;
      for (int64_t t = r0; t < r1; ++t, ++it) {
        const int buf = dbl ? (it & 1) : 0;
        const uint32_t parity = dbl ? (uint32_t)(it >> 1) & 1u : (uint32_t)it & 1u;
        bool issued = false;
        if (leader && dbl) {
          const int64_t next = next_row(t, r1);
          if (next >= 0) {
            issued = true;
            mbar_arrive_expect_tx(&mbar[buf ^ 1], row_bytes);
            bulk_g2s(stage + (buf ^ 1) * p.stage_bytes, p.x + (size_t)next * row_bytes, row_bytes, &mbar[buf ^ 1]);
          }
        }
        const bool ok = mbar_wait(&mbar[buf], parity, p.err);
        const uint32_t sa = stage_addr0 + (uint32_t)(buf * p.stage_bytes);
        float D2[MT2][4][4];
        float zc[32];
        float ss;
        if constexpr (CC)
          ss = rqcc::transform_block(gtab, team_threads, ttid, sa, tile, lane, zc);
        else
          ss = rqtc::transform_block<A>(lc, gtab, team_threads, ttid, sa, D2);
        if (lane == 0) red[buf * 32 + w] = ss;
        if (named_bar_or(bar_id, team_threads, !ok)) {
          if (issued) mbar_wait(&mbar[buf ^ 1], (uint32_t)((it + 1) >> 1) & 1u, p.err);
          failed = true;
          break;
        }
        if (leader && !dbl) {
          // every warp of the team is past its gather: the buffer is free
          const int64_t next = next_row(t, r1);
          if (next >= 0) {
            mbar_arrive_expect_tx(&mbar[0], row_bytes);
            bulk_g2s(stage, p.x + (size_t)next * row_bytes, row_bytes, &mbar[0]);
          }
        }
        float s2 = 0.f;
        for (int v = 0; v < p.nw; ++v) s2 += red[buf * 32 + v];
        // the tensor-core transform's partials are 32 sum y^2 (from P)
        const float s = CC ? sqrtf(s2) : sqrtf(s2 * (1.0f / 32.0f));
        const float ks = (s > 0.f) ? p.kscale / s : 0.f;
        const bool unclamped = p.full && s2 >= 1e-30f && s2 <= 1e30f;
        if constexpr (CC) {
          uint16_t* out = p.a16 + (size_t)t * p.K + (size_t)w * H + 32 * lane;
          if (unclamped)
            rqcc::quantize_levels<false>(zc, ks, magic, bin_lo, bin_hi, tbl_shift, out);
          else
            rqcc::quantize_levels<true>(zc, ks, magic, bin_lo, bin_hi, tbl_shift, out);
        } else {
          uint16_t* rowout = p.a16 + (size_t)t * p.K + (size_t)w * H + 2 * q;
          if (unclamped)
            rqtc::quantize_store<false, MT2>(D2, ks, magic, bin_lo, bin_hi, tbl_shift, rowout, g);
          else
            rqtc::quantize_store<true, MT2>(D2, ks, magic, bin_lo, bin_hi, tbl_shift, rowout, g);
        }
        if (leader) p.norms[t] = s;
      }
      if (failed) break;
      // publish the group: every thread's stores before the leader's release
      fence_proxy_async_global();
      __threadfence();
      named_bar_sync(bar_id, team_threads);
      if (leader) st_release_gpu(p.flags + item, 1);
      ++done;
      item = slot[done & 1];
    }
  } else if (warp == TMA_WARP) {
    // ------------------------------------------------ TMA producer (both CTAs)
    // the decoded weights may come from the kernel just before this one (a
    // programmatic dependent launch): wait for that grid and its writes before
    // the first B load (returns at once after an ordinary launch)
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const uint32_t full0 = mapa_shared(smem_u32(&op_full[0]), 0);
    int s = 0;
    uint32_t n = 0;
    bool ok = true;
    for (int i = 0; i < my_tiles && ok; ++i) {
      const int64_t tt = pair + (int64_t)i * npairs;
      const int64_t m0 = (tt / p.n_tiles) * (2 * RM) + rank * RM;
      const int32_t n0 = (int32_t)((tt % p.n_tiles) * PN + rank * RN);
      // this CTA's 128 A rows must be written before they are loaded
      const int first = (int)(m0 / RG);
      const int left = p.n_items - first, cnt = left < 0 ? 0 : (left < RM / RG ? left : RM / RG);
      ok = wait_flags(p.flags + first, cnt, lane, p.err);
      if (!ok) break;
      if (lane == 0) {
        fence_proxy_async_global();
        for (int kb = 0; kb < nkb; ++kb) {
          if (n > 0 && !mbar_wait(&op_empty[s], (n - 1) & 1u, p.err)) {
            ok = false;
            break;
          }
          if (rank == 0) mbar_arrive_expect_tx(&op_full[s], (uint32_t)(2 * STAGE_BYTES));
          unsigned char* st = smem + s * STAGE_BYTES;
          tma_load_2d_pair(st, &p.a_map, kb * BK, (int32_t)m0, full0 + 8u * (uint32_t)s);
          tma_load_2d_pair(st + A_TILE, &p.b_map, kb * BK, n0, full0 + 8u * (uint32_t)s);
          if (++s == OS) {
            s = 0;
            ++n;
          }
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
    }
    __syncwarp();
  } else if (warp < 4) {
    // ------------------------------------------------ epilogue (both CTAs)
    const int qw = warp;
    unsigned char* ebuf = epi + qw * (2 * 32 * 32 * 4);
    for (int64_t i = 0; i < my_tiles; ++i) {
      const int a = (int)(i & 1);
      const uint32_t u = (uint32_t)(i >> 1);
      if (!mbar_wait(&acc_full[a], u & 1u, p.err)) break;
      tc_fence_after();
      const int64_t tt = pair + i * npairs;
      const int64_t row0 = (tt / p.n_tiles) * (2 * RM) + rank * RM + qw * 32;
      const int64_t row = row0 + lane;
      const int n0 = (int)(tt % p.n_tiles) * PN;
      // the norm was written by a producer team: acquire its group's flag
      float srow = 0.f;
      if (row < p.M && ld_acquire_gpu(p.flags + row / RG) != 0) srow = __ldcg(p.norms + row) * p.out_scale;
#pragma unroll 1
      for (int cc = 0; cc < PN / 32; ++cc) {
        const int nb = n0 + cc * 32;
        uint32_t v[32];
        tmem_ld_32x32b_x32(tmem + ((uint32_t)(qw * 32) << 16) + (uint32_t)(a * PN + cc * 32), v);
        tmem_wait_ld();
        unsigned char* buf = ebuf + (cc & 1) * (32 * 32 * 4);
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
    if (lane == 0) bulk_wait<0>();
    __syncwarp();
  } else if (warp == MMA_WARP && rank == 0) {
    // ------------------------------------------------ paired MMA issuer (even CTA)
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f16_f32(2 * RM, PN);
      int s = 0;
      uint32_t n = 0;
      bool ok = true, rdy = false;
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

  tc_fence_before();
  cluster_sync_all();
  if (warp == MMA_WARP) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, TMEM_COLS);
  }
}

size_t smem_bytes(int A, bool cc, int nb, int nw, int teams, int stage_bytes, int os, int row_bufs, int* prod_off) {
  const int off = os * STAGE_BYTES + EPI_BYTES + BAR_BYTES;
  const int team_threads = nw * 32;
  const int gtab_off = (8 * nb + 15) & ~15;
  const int teams_off = (gtab_off + 2 * A * team_threads + 127) & ~127;
  if (prod_off) *prod_off = off;
  return 1024 + (size_t)off + teams_off + (size_t)teams * (TEAM_HDR + (cc ? (size_t)nw * 4096 : 0) +
                                                           (size_t)row_bufs * (size_t)stage_bytes);
}

}  // namespace

// Gather table of the producers' CUDA-core block transform (h = 1024): entry
// (w * 32 + lane) * 32 + a is the byte offset (2 x the input channel) of
// in-block position 32 a + lane of block w, the order in which a lane gathers
// its column.
void rqcc_build_gather(int d, const std::vector<uint32_t>& perm, std::vector<uint16_t>& gather) {
  gather.assign((size_t)d, 0);
  for (int w = 0; w < d / 1024; ++w)
    for (int lane = 0; lane < 32; ++lane)
      for (int a = 0; a < 32; ++a)
        gather[((size_t)w * 32 + lane) * 32 + a] = (uint16_t)(2 * perm[(size_t)w * 1024 + 32 * a + lane]);
}

size_t fused_flag_bytes(int64_t T) { return (size_t)((T + RG - 1) / RG + 64) * sizeof(int); }

bool fused_kernel_supported(const RQArgs& a, int N) {
  if (!rqtc_supported(a) || N % PN != 0 || a.d % 64 != 0) return false;
  const int A = a.h / 32, nw = a.d / a.h;
  if (GEMM_WARPS + nw > MAX_WARPS) return false;
  const int stage_bytes = (a.d * 2 + 127) & ~127;
  const int nb = a.bins_full ? a.nb_full : a.nb;
  return smem_bytes(A, A == 32 && a.gather_cc, nb, nw, 1, stage_bytes, 3, 1, nullptr) <= 227 * 1024;
}

oq_status fused_clear_flags(int* flags, int64_t T, void* stream) {
  const cudaError_t e = cudaMemsetAsync(flags, 0, fused_flag_bytes(T), static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) {
    set_error(std::string("clear fused flags: ") + cudaGetErrorString(e));
    return OQ_ERR_CUDA;
  }
  return OQ_OK;
}

oq_status fused_launch(const RQArgs& a, const GemmArgs& g, int* flags, void* stream, bool after_levels) {
  if (g.M == 0) return OQ_OK;
  if (!fused_kernel_supported(a, g.N) || !g.b_f16) return OQ_ERR_UNSUPPORTED;
  FusedParams kp;
  std::memset(&kp, 0, sizeof(kp));
  kp.b_scale = g.b_scale;
  kp.out_scale = g.out_scale;
  kp.y_bf16 = g.y_bf16;
  kp.M = g.M;
  kp.N = g.N;
  kp.K = g.K;
  kp.err = g.err;
  kp.x = static_cast<const unsigned char*>(a.src);
  kp.a16 = a.out16;
  kp.norms = a.norms;
  kp.n_items = (int)((g.M + RG - 1) / RG);
  kp.flags = flags;
  kp.counter = flags + kp.n_items + 32;   // its own line, away from the flags
  const bool cc = a.h == 1024 && a.gather_cc;
  kp.gather = cc ? a.gather_cc : a.gather_tc;
  if (a.bins_full) {
    kp.bins = reinterpret_cast<const uint2*>(a.bins_full);
    kp.nb = a.nb_full;
    kp.b0 = a.b0_full;
    kp.full = 1;
  } else {
    kp.bins = reinterpret_cast<const uint2*>(a.bins);
    kp.nb = a.nb;
    kp.b0 = a.b0;
  }
  kp.kscale = a.kscale;
  const int A = a.h / 32;
  kp.nw = a.d / a.h;
  kp.stage_bytes = (a.d * 2 + 127) & ~127;
  auto kern = cc ? fused_kernel<32, true> : (A == 32 ? fused_kernel<32, false> : fused_kernel<16, false>);
  // as many teams as the warp budget, shared memory and the SM's registers
  // allow (the occupancy query says whether one CTA of that shape fits)
  kp.os = kStages;
  kp.row_bufs = kRowBuffers;
  int teams = (MAX_WARPS - GEMM_WARPS) / kp.nw;
  size_t smem = 0;
  for (; teams >= 1; --teams) {
    smem = smem_bytes(A, cc, kp.nb, kp.nw, teams, kp.stage_bytes, kp.os, kp.row_bufs, &kp.prod_off);
    if (smem > 227 * 1024) continue;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess) continue;
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, (GEMM_WARPS + teams * kp.nw) * 32, smem) ==
            cudaSuccess &&
        per_sm >= 1)
      break;
  }
  cudaGetLastError();   // a refused configuration above is not an error of this call
  if (teams < 1) return OQ_ERR_UNSUPPORTED;
  kp.teams = teams;

  oq_status st = encode_operand_map(&kp.a_map, a.out16, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, g.M, g.K, RM,
                                    "the fp16 A operand");
  if (st == OQ_OK)
    st = encode_operand_map(&kp.b_map, g.b_f16, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, g.N, g.K, RN, "the fp16 B operand");
  if (st == OQ_OK) st = encode_y_map(&kp.y_map, g.y, g.M, g.N, g.y_bf16);
  if (st != OQ_OK) return st;

  cudaError_t e = cudaSuccess;
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  kp.n_tiles = kp.N / PN;
  kp.nkb = (kp.K + BK - 1) / BK;
  kp.tiles = ((kp.M + 2 * RM - 1) / (2 * RM)) * (int64_t)kp.n_tiles;
  const int grid = sms & ~1;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  // the flags and the queue counter start at zero on every call
  if (!after_levels) {
    const oq_status cs = fused_clear_flags(flags, g.M, stream);
    if (cs != OQ_OK) return cs;
  }
  const unsigned threads = (unsigned)((GEMM_WARPS + teams * kp.nw) * 32);
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = after_levels ? 1 : 0;
  e = cudaLaunchKernelEx(&cfg, kern, kp);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) {
    cudaFuncAttributes fa;
    std::memset(&fa, 0, sizeof(fa));
    cudaFuncGetAttributes(&fa, kern);
    set_error(std::string("fused kernel launch: ") + cudaGetErrorString(e) + " (threads " + std::to_string(threads) +
              ", dynamic shared memory " + std::to_string(smem) + ", registers " + std::to_string(fa.numRegs) +
              ", max threads " + std::to_string(fa.maxThreadsPerBlock) + ", static shared " +
              std::to_string(fa.sharedSizeBytes) + ")");
    return OQ_ERR_CUDA;
  }
  return OQ_OK;
}

}  // namespace oq
