// Codebook contraction on CTA pairs (tcgen05 cta_group::2), the main path for
// d_out % 256 == 0:
//   y[m, n] = a_scale[m] b_scale[n] out_scale sum_k LA[A[m, k]] LB[B[n, k]]
// (gecl notes Method 2 and Takeaway 3: a native non-uniform low-bit GEMM in
// the shared rotated basis).
//
// A cluster of two CTAs computes a 256 x 256 tile of y.  Each CTA decodes 128
// rows of activation codes and 128 rows of weight codes per K block of 64
// into fp16 operand tiles (128B-swizzled, K-major) in its own shared memory;
// one thread of the even CTA issues the paired MMA (M = 256, N = 256, K = 16),
// which reads A rows and B rows from both CTAs and leaves each CTA's 128 output
// rows in its own tensor memory.  Compared with one-SM 128 x 256 tiles this
// halves the weight decode per SM, and each SM still holds two accumulators,
// so the epilogue of one tile overlaps the next tile's main loop.
//
// Warps: 0-15 decode (codes prefetched two K blocks ahead into registers),
// 16-19 epilogue, 20 allocates tensor memory and (even CTA) issues the MMAs,
// 20 and 21 of the odd CTA forward the decoders' arrivals to the even CTA
// (alternate K blocks), and in the fused call 22 fetches the fp16 A tiles by
// TMA.
// Synchronisation: decoders of both CTAs arrive (one thread per warp, release
// at cluster scope) on the even CTA's `full` barrier; the MMA completion is
// multicast by tcgen05.commit to both CTAs' `empty` / `acc_full` barriers;
// epilogue warps of both CTAs arrive on the even CTA's `acc_empty`.  Every
// wait is bounded (oq_ptx.cuh).
#include <cuda.h>

#include <algorithm>
#include <cstring>

#include "oq_decode.cuh"
#include "oq_internal.h"
#include "oq_epilogue.cuh"
#include "oq_ptx.cuh"
#include "oq_tmap.cuh"

namespace oq {
namespace {

constexpr int RM = 128;            // activation rows per CTA (pair M = 256)
constexpr int PN = 256;            // output columns per pair tile
constexpr int RN = 128;            // weight rows per CTA
constexpr int BK = DEC_BK, UMMA_K = 16;
constexpr int NDEC = 512;          // decoder threads (warps 0-15)
constexpr int EPI_WARP0 = 16;      // epilogue warps 16-19 (TMEM lane quarters 0-3)
constexpr int MMA_WARP = 20;       // and the first forwarder (odd CTA)
constexpr int FWD2_WARP = 21;      // second forwarder (odd CTA)
constexpr int NTHREADS = 22 * 32;
constexpr int TMA_WARP = 22;       // fused call only: A-tile TMA producer
constexpr int OS = 6;              // operand stages
constexpr int A_TILE = RM * BK * 2;
constexpr int B_TILE = RN * BK * 2;
constexpr int STAGE_BYTES = A_TILE + B_TILE;
constexpr uint32_t TMEM_COLS = 2 * PN;
constexpr uint32_t ACC_EMPTY_COUNT = 2 * 4;           // one per epilogue warp, both CTAs

constexpr int EPI_BYTES = 4 * 2 * 32 * 32 * 4;   // per epilogue warp: two 32 x 32 fp32 staging boxes

struct PairParams {
  CUtensorMap a_map;          // fp16 A operand [M, K] (A_TMA kernels), 128B-swizzled boxes of 128 x 64
  CUtensorMap y_map;          // fp32 y [M, N], 128B-swizzled boxes of 32 x 32 (epilogue stores)
  const uint32_t* a_codes;
  const uint32_t* b_codes;
  const float* a_scale;
  const float* b_scale;
  float out_scale;
  bool y_bf16;         // y is bf16 (else fp32)
  void* y;                    // unused: the epilogue stores through y_map
  int64_t M;
  int N, K, a_wpr, b_wpr;
  int n_tiles, nkb;
  int64_t tiles;
  uint32_t a_tab[4], b_tab[4];
  DecK kc;                    // decode multipliers (opaque to the compiler)
  const uint16_t* a_lut8;
  int* err;
};

// A_TMA: the A operand is already fp16 levels in global memory (written by
// the rotate-quantize kernel in the fused layer call); a producer warp of its
// own fetches each 128 x 64 A tile with a TMA load in the swizzled layout as
// soon as the MMA has released the stage, and the decoders expand only the
// weight codes.
// F8: the lower-precision contraction mode (4-bit codes of both operands
// decoded to e4m3, K blocks of 128, kind::f8f6f4 MMAs with K 32).
template <int A_BITS, int B_BITS, bool A_TMA, bool F8>
// registers: six warps of one SM sub-partition share its 16K registers
__global__ void __cluster_dims__(2, 1, 1) __maxnreg__(80)
    gemm_pair_kernel(const __grid_constant__ PairParams p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  static_assert(OS == 6, "the decoder loop is unrolled over six stages");
  static_assert(!F8 || (A_BITS == 4 && B_BITS == 4 && !A_TMA), "the FP8 mode takes 4-bit codes of both operands");
  constexpr int BKE = F8 ? DEC_BK_F8 : BK;                 // K elements per stage
  constexpr int CHUNK_E = F8 ? 16 : 8;                     // K elements per 16-byte operand chunk
  constexpr int QA = A_TMA ? 0 : (F8 ? 4 : Fmt<A_BITS>::QP), QB = F8 ? 4 : Fmt<B_BITS>::QP;
  constexpr int ITEMS_A = RM * QA, ITEMS = RM * QA + RN * QB;
  // when the items fill at most half of the decoder threads (weights only, in
  // the fused call) the decoders split into two groups that take alternate K
  // blocks, so each warp has two MMA periods per stage it fills
  constexpr int NG = (2 * ITEMS <= NDEC) ? 2 : 1;
  constexpr int GT = NDEC / NG;                      // threads per group
  constexpr int IPT = (ITEMS + GT - 1) / GT;
  constexpr int DEC_WARPS = NDEC / 32;
  constexpr uint32_t FULL_CTA = GT / 32 + (A_TMA ? 1 : 0);   // + the TMA's expect_tx arrival

  unsigned char* epi = smem + OS * STAGE_BYTES;      // epilogue staging (1024-aligned)
  uint16_t* lut8 = reinterpret_cast<uint16_t*>(smem + OS * STAGE_BYTES + EPI_BYTES);
  uint64_t* op_full = reinterpret_cast<uint64_t*>(smem + OS * STAGE_BYTES + EPI_BYTES + 512);
  uint64_t* op_empty = op_full + OS;
  uint64_t* acc_full = op_empty + OS;
  uint64_t* acc_empty = acc_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int64_t pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int nkb = p.nkb;
  const int my_tiles = (p.tiles > pair) ? (int)((p.tiles - 1 - pair) / npairs + 1) : 0;

  if (A_BITS == 8 && p.a_lut8)
    for (int i = threadIdx.x; i < 256; i += blockDim.x) lut8[i] = p.a_lut8[i];
  if (threadIdx.x == 0) {
    for (int s = 0; s < OS; ++s) {
      // the even CTA also counts the odd CTA's forwarded arrival
      mbar_init(&op_full[s], rank == 0 ? FULL_CTA + 1 : FULL_CTA);
      mbar_init(&op_empty[s], 1);
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
  cluster_sync_all();   // barriers of both CTAs initialised before any remote arrival
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t smem_base = smem_u32(smem);
  const int total = my_tiles * nkb;   // K blocks this CTA pair runs through

  if (warp < DEC_WARPS) {
    // ------------------------------------------------ decoders
    uint32_t ta[4], tb[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      ta[i] = p.a_tab[i];
      tb[i] = p.b_tab[i];
    }
    const DecK kc = p.kc;
    // fixed per-thread items: operand row r, 16-byte code part q; the shared
    // address of each of its 16-byte chunks in stage 0 does not change
    constexpr int CPA = F8 ? 2 : Fmt<A_BITS>::CPP, CPB = F8 ? 2 : Fmt<B_BITS>::CPP;
    constexpr int CPM = CPA > CPB ? CPA : CPB;
    uint32_t sts[IPT][CPM];
    int item_r[IPT], item_q[IPT];
    bool item_a[IPT], item_on[IPT];
    const int group = (int)threadIdx.x / GT, gtid = (int)threadIdx.x % GT;
#pragma unroll
    for (int it = 0; it < IPT; ++it) {
      const int id = gtid + GT * it;
      const bool is_a = id < ITEMS_A;
      const int r = is_a ? id / (QA ? QA : 1) : (id - ITEMS_A) / QB;
      item_a[it] = is_a;
      item_on[it] = id < ITEMS;
      item_r[it] = r;
      item_q[it] = is_a ? id % (QA ? QA : 1) : (id - ITEMS_A) % QB;
      const uint32_t row_base = smem_base + (is_a ? 0u : (uint32_t)A_TILE) + (uint32_t)((r >> 3) * 1024 + (r & 7) * 128);
      const int cpp = is_a ? CPA : CPB;
#pragma unroll
      for (int j = 0; j < CPM; ++j)
        sts[it][j] = row_base + ((((uint32_t)(item_q[it] * cpp + j)) << 4) ^ ((uint32_t)(r & 7) << 4));
    }
    // code-row pointers of the tile the fetch cursor is in; activation rows
    // past M read row M - 1 instead (they only reach outputs the store clips)
    const uint32_t* frow[IPT];
    auto origin = [&](int tile_i) {
      const int64_t tt = pair + (int64_t)tile_i * npairs;
      const int64_t m0 = (tt / p.n_tiles) * (2 * RM) + rank * RM;
      const int n0 = (int)(tt % p.n_tiles) * PN + (int)rank * RN;
#pragma unroll
      for (int it = 0; it < IPT; ++it) {
        if (item_a[it]) {
          const int64_t row = m0 + item_r[it];
          frow[it] = p.a_codes + (row < p.M ? row : p.M - 1) * p.a_wpr;
        } else {
          frow[it] = p.b_codes + (int64_t)(n0 + item_r[it]) * p.b_wpr;
        }
      }
    };
    auto fetch = [&](int kb, uint4 (&dst)[IPT]) {
#pragma unroll
      for (int it = 0; it < IPT; ++it) {
        dst[it] = make_uint4(0u, 0u, 0u, 0u);
        if (item_on[it]) {
          if constexpr (F8) dst[it] = load_part_f8(frow[it], kb, item_q[it], p.K);
          else if (item_a[it]) dst[it] = load_part<A_BITS>(frow[it], kb, item_q[it], p.K);
          else dst[it] = load_part<B_BITS>(frow[it], kb, item_q[it], p.K);
        }
      }
    };
    auto dec_a = [&](const uint4& v, int j) -> uint4 {
      if constexpr (F8) return decode_chunk_f8(v, j, ta, kc);
      else return decode_chunk_k<A_BITS>(v, j, ta, lut8, kc);
    };
    auto dec_b = [&](const uint4& v, int j) -> uint4 {
      if constexpr (F8) return decode_chunk_f8(v, j, tb, kc);
      else return decode_chunk_k<B_BITS>(v, j, tb, lut8, kc);
    };
    // decode one K block (TAIL: the block runs past K and the A chunks beyond
    // it must be zero) into registers, and store decoded chunks into stage S
    // (called with literal S and TAIL: after inlining the stage offset folds
    // into the store's address)
    auto decode_regs = [&](bool TAIL, const uint4 (&cur)[IPT], int kb, uint4 (&dec)[IPT][CPM]) {
#pragma unroll
      for (int it = 0; it < IPT; ++it) {
        if (item_a[it]) {
#pragma unroll
          for (int j = 0; j < CPA; ++j) {
            uint4 o = dec_a(cur[it], j);
            if (TAIL && kb * BKE + (item_q[it] * CPA + j) * CHUNK_E >= p.K) o = make_uint4(0u, 0u, 0u, 0u);
            dec[it][j] = o;
          }
        } else if (item_on[it]) {
#pragma unroll
          for (int j = 0; j < CPB; ++j) dec[it][j] = dec_b(cur[it], j);
        }
      }
    };
    auto store = [&](int S, const uint4 (&dec)[IPT][CPM]) {
      const uint32_t so = (uint32_t)(S * STAGE_BYTES);
#pragma unroll
      for (int it = 0; it < IPT; ++it) {
        if (item_a[it]) {
#pragma unroll
          for (int j = 0; j < CPA; ++j) st_shared_v4(sts[it][j] + so, dec[it][j]);
        } else if (item_on[it]) {
#pragma unroll
          for (int j = 0; j < CPB; ++j) st_shared_v4(sts[it][j] + so, dec[it][j]);
        }
      }
    };
    // decode and store chunk by chunk (few registers live)
    auto decode_store = [&](int S, bool TAIL, const uint4 (&cur)[IPT], int kb) {
      const uint32_t so = (uint32_t)(S * STAGE_BYTES);
#pragma unroll
      for (int it = 0; it < IPT; ++it) {
        if (item_a[it]) {
#pragma unroll
          for (int j = 0; j < CPA; ++j) {
            uint4 o = dec_a(cur[it], j);
            if (TAIL && kb * BKE + (item_q[it] * CPA + j) * CHUNK_E >= p.K) o = make_uint4(0u, 0u, 0u, 0u);
            st_shared_v4(sts[it][j] + so, o);
          }
        } else if (item_on[it]) {
#pragma unroll
          for (int j = 0; j < CPB; ++j)
            st_shared_v4(sts[it][j] + so, dec_b(cur[it], j));
        }
      }
    };
    // with at most four decoded chunks per thread the decode runs before the
    // wait for the stage to be free (off the MMA's critical path); larger
    // per-thread loads decode after it (registers)
    constexpr bool AHEAD = IPT * CPM <= 4;
    // the fetch cursor runs two steps (2 NG K blocks) ahead of the decode
    // cursor; the three register buffers and the stages rotate by unrolling
    // (no copies of registers whose loads are still in flight, and every stage
    // offset is an immediate)
    int f_tile = group / nkb, f_kb = group % nkb;   // this group's first K block
    origin(f_tile);
    auto advance = [&]() {
      f_kb += NG;
      while (f_kb >= nkb) {   // (nkb may be 1 with two groups)
        f_kb -= nkb;
        ++f_tile;
        origin(f_tile);
      }
    };
    uint4 c0[IPT], c1[IPT], c2[IPT];
    if (group < total) {
      fetch(f_kb, c0);
      advance();
    }
    if (group + NG < total) {
      fetch(f_kb, c1);
      advance();
    }
    const bool k_tail = p.K % BK != 0;
    int g = group, d_kb = group % nkb;
    bool dead = false;
    auto step = [&](int S, const uint4 (&cur)[IPT], uint4 (&fut)[IPT]) -> void {
      if (g + 2 * NG < total) {
        fetch(f_kb, fut);
        advance();
      }
      const bool tail = k_tail && d_kb == nkb - 1;
      const uint32_t n = (uint32_t)(g / OS);
      // after a timed-out wait (error recorded) keep stepping without waiting
      if constexpr (AHEAD) {
        uint4 dec[IPT][CPM];
        if (tail) decode_regs(true, cur, d_kb, dec);
        else decode_regs(false, cur, d_kb, dec);
        if (n > 0 && !dead && !mbar_wait(&op_empty[S], (n - 1) & 1u, p.err)) dead = true;
        store(S, dec);
      } else {
        if (n > 0 && !dead && !mbar_wait(&op_empty[S], (n - 1) & 1u, p.err)) dead = true;
        if (tail) decode_store(S, true, cur, d_kb);
        else decode_store(S, false, cur, d_kb);
      }
      // this warp's tiles -> visible to the async proxy, then one arrival
      // per warp on this CTA's `full` barrier (the odd CTA forwards it)
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&op_full[S]);
      d_kb += NG;
      while (d_kb >= nkb) d_kb -= nkb;
      g += NG;
    };
    if constexpr (NG == 1) {
      while (g < total) {
        step(0, c0, c2);
        if (g >= total) break;
        step(1, c1, c0);
        if (g >= total) break;
        step(2, c2, c1);
        if (g >= total) break;
        step(3, c0, c2);
        if (g >= total) break;
        step(4, c1, c0);
        if (g >= total) break;
        step(5, c2, c1);
      }
    } else {
      // group 0 fills stages 0, 2, 4 and group 1 stages 1, 3, 5
      auto run = [&](int s0) {
        while (g < total) {
          step(s0, c0, c2);
          if (g >= total) break;
          step(s0 + 2, c1, c0);
          if (g >= total) break;
          step(s0 + 4, c2, c1);
        }
      };
      if (group == 0) run(0);
      else run(1);
    }
  } else if (A_TMA && warp == TMA_WARP) {
    // ------------------------------------------------ A tiles by TMA (fused call)
    if (lane == 0) {
      int s = 0, kb = 0, tile = 0;
      uint32_t n = 0;
      auto a_row0 = [&](int tile_i) {
        return (int32_t)(((pair + (int64_t)tile_i * npairs) / p.n_tiles) * (2 * RM) + rank * RM);
      };
      int32_t m0 = a_row0(0);
      for (int g = 0; g < total; ++g) {
        if (n > 0 && !mbar_wait(&op_empty[s], (n - 1) & 1u, p.err)) break;
        // rows past M and columns past K arrive as zeros
        mbar_arrive_expect_tx(&op_full[s], (uint32_t)A_TILE);
        tma_load_2d(smem + s * STAGE_BYTES, &p.a_map, kb * BK, m0, &op_full[s]);
        if (++s == OS) {
          s = 0;
          ++n;
        }
        if (++kb == nkb) {
          kb = 0;
          m0 = a_row0(++tile);
        }
      }
    }
    __syncwarp();
  } else if (warp >= EPI_WARP0 && warp < EPI_WARP0 + 4) {
    // ------------------------------------------------ epilogue (both CTAs)
    // Each warp drains its 32 TMEM lanes (rows) in chunks of 32 columns,
    // scales them, stages the 32 x 32 box in shared memory (128B swizzle,
    // conflict-free) and writes it with one TMA store: full-line writes and
    // a handful of instructions per chunk.  Rows past M are clipped by TMA.
    const int q = warp & 3;
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
      // the descriptors of all stages share their high word; the low word is
      // the start address / 16 (plus the constant leading-offset field), so
      // one descriptor per stage and K step is one 32-bit add (this thread
      // shares its sub-partition with busy decoder warps: every instruction
      // it saves is issue latency off the MMA's critical path)
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
          // probe the next stage while this one's MMAs issue (a barrier check
          // costs ~200 cycles even when the phase is long complete)
          int s1 = s + 1;
          uint32_t n1 = n;
          if (s1 == OS) {
            s1 = 0;
            ++n1;
          }
          const bool more = kb + 1 < nkb || i + 1 < my_tiles;
          const uint32_t a_lo = a_lo0 + (uint32_t)s * (uint32_t)(STAGE_BYTES >> 4);
          const bool rdy1 = tc_kblock_4mma<2, F8>(d_tmem, a_lo, a_lo + (A_TILE >> 4), d_hi, idesc, kb > 0 ? 1u : 0u,
                                                  &op_empty[s], (uint16_t)0x3, &op_full[s1], n1 & 1u, more ? 1u : 0u);
          s = s1;
          n = n1;
          rdy = rdy1;
        }
        tc_commit_pair_mc(&acc_full[a], (uint16_t)0x3);
      }
    }
    __syncwarp();
  }

  if ((warp == MMA_WARP || warp == FWD2_WARP) && rank == 1) {
    // ------------------------------------------------ forwarders (odd CTA)
    // one cluster-scope release per stage instead of one per decoder warp; a
    // release at cluster scope takes longer than the MMAs of one K block, so
    // two threads take alternate K blocks (even and odd stages)
    if (lane == 0) {
      for (int g = (warp == MMA_WARP) ? 0 : 1; g < total; g += 2) {
        const int s = g % OS;
        if (!mbar_wait(&op_full[s], (uint32_t)(g / OS) & 1u, p.err)) break;
        mbar_arrive_cluster(mapa_shared(smem_u32(&op_full[s]), 0));
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

template <int A_BITS, int B_BITS, bool A_TMA, bool F8 = false>
oq_status launch_pair(const PairParams& kp_in, void* stream) {
  PairParams kp = kp_in;
  auto kern = gemm_pair_kernel<A_BITS, B_BITS, A_TMA, F8>;
  const size_t smem = 1024 + (size_t)OS * STAGE_BYTES + EPI_BYTES + 512 + 8 * (2 * OS + 4) + 16;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) {
    set_error(std::string("cudaFuncSetAttribute(gemm pair): ") + cudaGetErrorString(e));
    return OQ_ERR_CUDA;
  }
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  kp.n_tiles = kp.N / PN;
  kp.nkb = (kp.K + (F8 ? DEC_BK_F8 : BK) - 1) / (F8 ? DEC_BK_F8 : BK);
  kp.tiles = ((kp.M + 2 * RM - 1) / (2 * RM)) * (int64_t)kp.n_tiles;
  const int64_t grid = std::min<int64_t>(2 * kp.tiles, (int64_t)(sms & ~1));
  // K-block counters are 32-bit
  if (((kp.tiles + grid / 2 - 1) / (grid / 2)) * (int64_t)kp.nkb >= (int64_t)1 << 31) return OQ_ERR_UNSUPPORTED;
  kern<<<(unsigned)grid, A_TMA ? NTHREADS + 32 : NTHREADS, smem, static_cast<cudaStream_t>(stream)>>>(kp);
  e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error(std::string("gemm pair launch: ") + cudaGetErrorString(e));
    return OQ_ERR_CUDA;
  }
  return OQ_OK;
}

template <int A_BITS, bool A_TMA>
oq_status launch_pair_b(const PairParams& kp, int b_bits, void* stream) {
  switch (b_bits) {
    case 2: return launch_pair<A_BITS, 2, A_TMA>(kp, stream);
    case 3: return launch_pair<A_BITS, 3, A_TMA>(kp, stream);
    case 4: return launch_pair<A_BITS, 4, A_TMA>(kp, stream);
    default: return OQ_ERR_UNSUPPORTED;
  }
}

}  // namespace

oq_status gemm_pair_launch(const GemmArgs& g, void* stream) {
  if (g.M == 0) return OQ_OK;
  if (g.N % PN != 0) return OQ_ERR_UNSUPPORTED;
  PairParams kp;
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
  if (g.fp8) {
    // e4m3 bytes of the eight positive levels (codes 8..15) in two words
    for (int w = 0; w < 2; ++w) {
      kp.a_tab[w] = kp.b_tab[w] = 0u;
      for (int b = 0; b < 4; ++b) {
        kp.a_tab[w] |= (uint32_t)g.a_levels8[8 + 4 * w + b] << (8 * b);
        kp.b_tab[w] |= (uint32_t)g.b_levels8[8 + 4 * w + b] << (8 * b);
      }
    }
  } else {
    make_decode_tables(g.a_bits, g.a_levels_host, kp.a_tab);
    make_decode_tables(g.b_bits, g.b_levels_host, kp.b_tab);
  }
  kp.kc = make_deck();
  kp.a_lut8 = g.a_levels;
  kp.err = g.err;
  if (reinterpret_cast<uintptr_t>(g.y) & 15) return OQ_ERR_UNSUPPORTED;
  {
    const oq_status st = encode_y_map(&kp.y_map, g.y, g.M, g.N, g.y_bf16);
    if (st != OQ_OK) return st;
  }
  if (g.fp8) {
    if (g.a_f16 || g.a_bits != 4 || g.b_bits != 4) return OQ_ERR_UNSUPPORTED;
    return launch_pair<4, 4, false, true>(kp, stream);
  }
  if (g.a_f16) {
    // fp16 A operand fetched by TMA: 16-byte aligned rows of K halves
    if ((reinterpret_cast<uintptr_t>(g.a_f16) & 15) || (g.K % 8)) return OQ_ERR_UNSUPPORTED;
    const oq_status st = encode_operand_map(&kp.a_map, g.a_f16, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, g.M, g.K, RM,
                                            "the fp16 A operand");
    if (st != OQ_OK) return st;
    return launch_pair_b<4, true>(kp, g.b_bits, stream);
  }
  switch (g.a_bits) {
    case 2: return launch_pair_b<2, false>(kp, g.b_bits, stream);
    case 3: return launch_pair_b<3, false>(kp, g.b_bits, stream);
    case 4: return launch_pair_b<4, false>(kp, g.b_bits, stream);
    case 8: return launch_pair_b<8, false>(kp, g.b_bits, stream);
    default: return OQ_ERR_UNSUPPORTED;
  }
}

}  // namespace oq
