// Inline-PTX helpers for sm_100a: mbarriers, bulk async copies, tcgen05.
// Every wait is bounded in wall-clock time: after OQ_WAIT_NS nanoseconds
// (read from %globaltimer) it gives up, records OQ_DEVERR_TIMEOUT in the
// caller's error word and returns false.
#pragma once

#include <cstdint>

#include "oq_internal.h"

#ifndef OQ_WAIT_NS
#define OQ_WAIT_NS 1000000000ull
#endif

namespace oq {

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(
                   smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Bounded wait for the phase with the given parity to complete (limit_ns:
// the bound, OQ_WAIT_NS unless a caller gives a shorter one).
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, int* err,
                                          uint64_t limit_ns = OQ_WAIT_NS) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 64; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (globaltimer_ns() - t0 > limit_ns) {
      if (err) atomicOr(err, OQ_DEVERR_TIMEOUT);
      return false;
    }
  }
}

// ---------------------------------------------------------------- bulk copy
// 1-D bulk async copy global -> shared, completion counted on `bar` in bytes.
// Both addresses 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst_smem, const void* src_gmem, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst_smem)),
      "l"(src_gmem), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// 2-D tiled TMA load (no multicast) of box (x, y) of a tensor map into this
// CTA's shared memory, completion counted in bytes on `bar`
__device__ __forceinline__ void tma_load_2d(void* dst_smem, const void* tmap, int32_t x, int32_t y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          smem_u32(dst_smem)),
      "l"(tmap), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

// The same load issued by either CTA of a pair whose MMAs run with
// cta_group::2: the box lands in the issuing CTA's shared memory and its bytes
// are counted on the barrier at `bar_cluster`, a shared::cluster address that
// may lie in the peer CTA (no multicast)
__device__ __forceinline__ void tma_load_2d_pair(void* dst_smem, const void* tmap, int32_t x, int32_t y,
                                                 uint32_t bar_cluster) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, "
      "%3}], [%4];" ::"r"(smem_u32(dst_smem)),
      "l"(tmap), "r"(x), "r"(y), "r"(bar_cluster)
      : "memory");
}

// 2-D tiled TMA store of a shared-memory box to (x, y) of a tensor map; boxes
// reaching past the tensor's bounds are clipped.  Tracked as a bulk group.
__device__ __forceinline__ void tma_store_2d(const void* tmap, int32_t x, int32_t y, const void* src_smem) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(tmap), "r"(x),
               "r"(y), "r"(smem_u32(src_smem))
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// wait until at most N committed bulk groups of this thread still read shared memory
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
template <int N>
__device__ __forceinline__ void bulk_wait() {
  asm volatile("cp.async.bulk.wait_group %0;" ::"n"(N) : "memory");
}

// ---------------------------------------------------------------- proxies
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
// generic-proxy accesses to global memory ordered with async-proxy (TMA) ones
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// ---------------------------------------------------------------- flags in global memory
__device__ __forceinline__ int ld_relaxed_gpu(const int* p) {
  int v;
  asm volatile("ld.relaxed.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ int ld_acquire_gpu(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release_gpu(int* p, int v) {
  asm volatile("st.release.gpu.global.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ void fence_acq_rel_gpu() { asm volatile("fence.acq_rel.gpu;" ::: "memory"); }

// named barrier over `nthreads` threads (a multiple of 32); returns whether
// any of them passed a non-zero `pred`
__device__ __forceinline__ int named_bar_or(int id, int nthreads, int pred) {
  int r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.s32 q, %1, 0;\n\t"
      "bar.red.or.pred p, %2, %3, q;\n\tselp.s32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"(pred), "r"(id), "r"(nthreads)
      : "memory");
  return r;
}
__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// ---------------------------------------------------------------- tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc]^T, kind::f16, issued by one thread
__device__ __forceinline__ void tc_mma_f16_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                              uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// arrive on `bar` once all previously issued tcgen05.mma of this thread complete
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns: thread i gets lane (base+i)
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]),
        "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]),
        "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor (tcgen05): K-major operand in the
// 128-byte-swizzled layout, 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= (uint64_t)((smem_addr >> 4) & 0x3FFF);        // start address
  d |= (uint64_t)1 << 16;                             // leading byte offset (unused for SW128 K-major)
  d |= (uint64_t)(1024 >> 4) << 32;                   // stride byte offset: 8 rows x 128 B
  d |= (uint64_t)1 << 46;                             // descriptor version (sm_100)
  d |= (uint64_t)2 << 61;                             // layout: SWIZZLE_128B
  return d;
}

// Instruction descriptor, kind::f16: fp16 A and B (K-major), fp32 D, M x N.
// the same with bf16 A and B (both operands of a kind::f16 MMA share a type)
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N);
__host__ __device__ constexpr uint32_t idesc_f16_f32(int M, int N) {
  return (1u << 4)                                   // D format f32
         | (0u << 7) | (0u << 10)                    // A, B format f16
         | (0u << 15) | (0u << 16)                   // A, B K-major
         | ((uint32_t)(N >> 3) << 17)                // N / 8
         | ((uint32_t)(M >> 4) << 24);               // M / 16
}
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N) {
  return idesc_f16_f32(M, N) | (1u << 7) | (1u << 10);   // A, B format bf16
}

// ---------------------------------------------------------------- clusters
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// shared::cluster address of the same variable in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t mapa_shared(uint32_t local_addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local_addr), "r"(rank));
  return r;
}

// arrive (release at cluster scope) on an mbarrier given by shared::cluster address
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// non-blocking probe (no suspension): has the phase with this parity completed?
__device__ __forceinline__ bool mbar_test_wait_cluster(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// bounded wait whose completion was signalled from another CTA of the cluster
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t* bar, uint32_t parity, int* err) {
  if (mbar_try_wait_cluster(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 64; ++i)
      if (mbar_try_wait_cluster(bar, parity)) return true;
    if (globaltimer_ns() - t0 > OQ_WAIT_NS) {
      if (err) atomicOr(err, OQ_DEVERR_TIMEOUT);
      return false;
    }
  }
}

// every thread of every CTA of the cluster (release / acquire)
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}

// generic-proxy writes to shared memory -> visible to async-proxy readers
// of any CTA of the cluster (the paired tensor core reads the peer's tiles)
__device__ __forceinline__ void fence_proxy_async_all() { asm volatile("fence.proxy.async;" ::: "memory"); }

__device__ __forceinline__ void st_shared_v4(uint32_t addr, const uint4& v) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

// One K block of 64 (four kind::f16 MMAs of K 16; the smem descriptors
// {lo, hi} advance by 2 in their low word per K step), the commit of its
// completion to `bar`, and -- when `probe` is set -- a non-blocking check of
// phase `next_parity` of `next_bar` (.acquire.cluster).  The probe is issued
// before the MMAs and its answer is only read after them, so the ~200-cycle
// latency of a barrier check overlaps the MMA issue.  `accumulate` applies to
// the first MMA; the other three always accumulate.
// F8: the same with kind::f8f6f4 MMAs (K 32 e4m3 per MMA: 128 K per call;
// the descriptors advance by the same 32 bytes per MMA).
#define OQ_KBLOCK_ASM(CGS, KIND, WAITSCOPE, COMMIT)                                                             \
  "{\n\t.reg .pred pa, pt, pp, pn;\n\t.reg .b64 da, db;\n\t.reg .b32 al, bl;\n\t"                                \
  "setp.ne.b32 pa, %5, 0;\n\tsetp.eq.b32 pt, 0, 0;\n\tsetp.ne.b32 pp, %10, 0;\n\t"                                  \
  "setp.ne.b32 pn, 0, 0;\n\t"                                                                                    \
  "@pp mbarrier.test_wait.parity.acquire." WAITSCOPE ".shared::cta.b64 pn, [%8], %9;\n\t"                         \
  "mov.b64 da, {%2, %4};\n\tmov.b64 db, {%3, %4};\n\t"                                                          \
  "tcgen05.mma.cta_group::" CGS ".kind::" KIND " [%1], da, db, %6, pa;\n\t"                                      \
  "add.u32 al, %2, 2;\n\tadd.u32 bl, %3, 2;\n\tmov.b64 da, {al, %4};\n\tmov.b64 db, {bl, %4};\n\t"              \
  "tcgen05.mma.cta_group::" CGS ".kind::" KIND " [%1], da, db, %6, pt;\n\t"                                      \
  "add.u32 al, %2, 4;\n\tadd.u32 bl, %3, 4;\n\tmov.b64 da, {al, %4};\n\tmov.b64 db, {bl, %4};\n\t"              \
  "tcgen05.mma.cta_group::" CGS ".kind::" KIND " [%1], da, db, %6, pt;\n\t"                                      \
  "add.u32 al, %2, 6;\n\tadd.u32 bl, %3, 6;\n\tmov.b64 da, {al, %4};\n\tmov.b64 db, {bl, %4};\n\t"              \
  "tcgen05.mma.cta_group::" CGS ".kind::" KIND " [%1], da, db, %6, pt;\n\t" COMMIT                              \
  "selp.u32 %0, 1, 0, pn;\n\t}"

template <int CG, bool F8>
__device__ __forceinline__ bool tc_kblock_4mma(uint32_t d_tmem, uint32_t a_lo, uint32_t b_lo, uint32_t d_hi,
                                               uint32_t idesc, uint32_t accumulate, uint64_t* bar, uint16_t mask,
                                               uint64_t* next_bar, uint32_t next_parity, uint32_t probe) {
  uint32_t ready;
#define OQ_KBLOCK_ARGS                                                                                        \
  : "=r"(ready)                                                                                               \
  : "r"(d_tmem), "r"(a_lo), "r"(b_lo), "r"(d_hi), "r"(accumulate), "r"(idesc), "r"(smem_u32(bar)),              \
    "r"(smem_u32(next_bar)), "r"(next_parity), "r"(probe), "h"(mask)                                            \
  : "memory"
  if constexpr (CG == 2 && F8) {
    asm volatile(OQ_KBLOCK_ASM("2", "f8f6f4", "cluster",
                               "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::"
                               "cluster.b64 [%7], %11;\n\t") OQ_KBLOCK_ARGS);
  } else if constexpr (CG == 2) {
    asm volatile(OQ_KBLOCK_ASM("2", "f16", "cluster",
                               "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::"
                               "cluster.b64 [%7], %11;\n\t") OQ_KBLOCK_ARGS);
  } else {
    static_assert(!F8, "one-CTA FP8 K blocks are not used");
    asm volatile(OQ_KBLOCK_ASM("1", "f16", "cta",
                               "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%7];\n\t")
                     OQ_KBLOCK_ARGS);
  }
#undef OQ_KBLOCK_ARGS
  return ready != 0;
}
#undef OQ_KBLOCK_ASM

template <int CG>
__device__ __forceinline__ bool tc_kblock64_f16(uint32_t d_tmem, uint32_t a_lo, uint32_t b_lo, uint32_t d_hi,
                                                uint32_t idesc, uint32_t accumulate, uint64_t* bar, uint16_t mask,
                                                uint64_t* next_bar, uint32_t next_parity, uint32_t probe) {
  uint32_t ready;
  if constexpr (CG == 2) {
    asm volatile(
        "{\n\t.reg .pred pa, pt, pp, pn;\n\t.reg .b64 da, db;\n\t.reg .b32 al, bl;\n\t"
        "setp.ne.b32 pa, %5, 0;\n\tsetp.eq.b32 pt, 0, 0;\n\tsetp.ne.b32 pp, %10, 0;\n\t"
        "setp.ne.b32 pn, 0, 0;\n\t"
        "@pp mbarrier.test_wait.parity.acquire.cluster.shared::cta.b64 pn, [%8], %9;\n\t"
        "mov.b64 da, {%2, %4};\n\tmov.b64 db, {%3, %4};\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%1], da, db, %6, pa;\n\t"
        "add.u32 al, %2, 2;\n\tadd.u32 bl, %3, 2;\n\tmov.b64 da, {al, %4};\n\tmov.b64 db, {bl, %4};\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%1], da, db, %6, pt;\n\t"
        "add.u32 al, %2, 4;\n\tadd.u32 bl, %3, 4;\n\tmov.b64 da, {al, %4};\n\tmov.b64 db, {bl, %4};\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%1], da, db, %6, pt;\n\t"
        "add.u32 al, %2, 6;\n\tadd.u32 bl, %3, 6;\n\tmov.b64 da, {al, %4};\n\tmov.b64 db, {bl, %4};\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%1], da, db, %6, pt;\n\t"
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%7], %11;\n\t"
        "selp.u32 %0, 1, 0, pn;\n\t}"
        : "=r"(ready)
        : "r"(d_tmem), "r"(a_lo), "r"(b_lo), "r"(d_hi), "r"(accumulate), "r"(idesc), "r"(smem_u32(bar)),
          "r"(smem_u32(next_bar)), "r"(next_parity), "r"(probe), "h"(mask)
        : "memory");
  } else {
    asm volatile(
        "{\n\t.reg .pred pa, pt, pp, pn;\n\t.reg .b64 da, db;\n\t.reg .b32 al, bl;\n\t"
        "setp.ne.b32 pa, %5, 0;\n\tsetp.eq.b32 pt, 0, 0;\n\tsetp.ne.b32 pp, %10, 0;\n\t"
        "setp.ne.b32 pn, 0, 0;\n\t"
        "@pp mbarrier.test_wait.parity.acquire.cta.shared::cta.b64 pn, [%8], %9;\n\t"
        "mov.b64 da, {%2, %4};\n\tmov.b64 db, {%3, %4};\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%1], da, db, %6, pa;\n\t"
        "add.u32 al, %2, 2;\n\tadd.u32 bl, %3, 2;\n\tmov.b64 da, {al, %4};\n\tmov.b64 db, {bl, %4};\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%1], da, db, %6, pt;\n\t"
        "add.u32 al, %2, 4;\n\tadd.u32 bl, %3, 4;\n\tmov.b64 da, {al, %4};\n\tmov.b64 db, {bl, %4};\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%1], da, db, %6, pt;\n\t"
        "add.u32 al, %2, 6;\n\tadd.u32 bl, %3, 6;\n\tmov.b64 da, {al, %4};\n\tmov.b64 db, {bl, %4};\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%1], da, db, %6, pt;\n\t"
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%7];\n\t"
        "selp.u32 %0, 1, 0, pn;\n\t}"
        : "=r"(ready)
        : "r"(d_tmem), "r"(a_lo), "r"(b_lo), "r"(d_hi), "r"(accumulate), "r"(idesc), "r"(smem_u32(bar)),
          "r"(smem_u32(next_bar)), "r"(next_parity), "r"(probe), "h"(mask)
        : "memory");
  }
  return ready != 0;
}

// ---------------------------------------------------------------- tcgen05, CTA pair
__device__ __forceinline__ void tmem_alloc_pair(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// paired MMA issued by one thread of the even CTA: A rows split over the two
// CTAs, B rows (N) split over the two CTAs, D rows split over the two CTAs
__device__ __forceinline__ void tc_mma_f16_ss_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                                   uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// arrive on the mbarrier at this shared offset in every CTA of `mask` once
// the pair's previously issued MMAs complete
__device__ __forceinline__ void tc_commit_pair_mc(uint64_t* bar, uint16_t mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"(mask)
      : "memory");
}

}  // namespace oq
