// fia_device.cuh -- sm_100a device primitives used by the attention kernels:
// bounded mbarrier waits, TMA tile loads, tcgen05 (TMEM / UMMA) wrappers,
// legacy mma.sync + ldmatrix for the decode kernels, and small numeric helpers.
//
// Every wait on an mbarrier is bounded by wall-clock time (%globaltimer).  A
// wait that runs out records an error code in the kernel's error word and
// raises the CTA-wide abort flag; the kernels then leave their loops, meet at
// the final barrier and release TMEM.
#pragma once

#include <atomic>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace fia {

// Error codes written to the error word.
enum : uint32_t {
    kErrNone = 0,
    kErrWaitTimeout = 1,
};

constexpr uint64_t kWaitLimitNs = 2000000000ull;   // 2 s per wait (the default limit)
// After a role has given up, each copy or MMA still in flight is waited for
// (up to this long) before the CTA releases its shared memory and TMEM.
constexpr uint64_t kDrainLimitNs = 100000000ull;   // 100 ms

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------------------
// mbarrier
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}"
                 ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}"
                 ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}

// try_wait (the hardware may briefly park the warp; no explicit suspend hint:
// a measured hint woke the waiter later than plain polling did).
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
    return ok != 0;
}

// Non-blocking probe of the same phase (no suspend): cheaper than try_wait
// when the phase has usually completed long before.
__device__ __forceinline__ bool mbar_test_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
    return ok != 0;
}

// Waits for the phase of `bar` with parity `parity` to complete.  Returns
// false (after recording the error and raising `abort`) when the wait runs
// past `limit_ns`, or when another role has already raised `abort`.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, volatile int *abort,
                                          uint32_t *err, uint32_t where, uint64_t limit_ns) {
    if (mbar_test_wait(bar, parity)) return true;
    uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 0;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 63u) == 63u) {
            if (*abort) return false;
            if (globaltimer_ns() - t0 > limit_ns) {
                *abort = 1;
                if (err) atomicCAS(err, 0u, (where << 8) | kErrWaitTimeout);
                return false;
            }
        }
    }
}

// Error exit only: waits (up to kDrainLimitNs, ignoring `abort`) for the
// phase of `bar` with parity `parity`, i.e. for the copies or MMAs that will
// complete it, so that none of them still writes into shared memory or TMEM
// after the CTA has released them.
__device__ __forceinline__ bool mbar_wait_drain(uint64_t *bar, uint32_t parity) {
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 0;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 63u) == 63u && globaltimer_ns() - t0 > kDrainLimitNs) return false;
    }
}

// Error region layout (uint32 words): [0] error word, [1] trail count,
// [4 + 8k .. 4 + 8k + 7] trail record k (k < kTrailMax): where, block, thread,
// three caller values, the waited barrier's raw 64-bit state.
constexpr uint32_t kTrailMax = 31;
constexpr uint32_t kErrRegionBytes = (4 + 8 * kTrailMax) * 4;

static __device__ __noinline__ void fail_trail(uint32_t *err, uint32_t where, uint32_t x0, uint32_t x1,
                                        uint32_t x2, const uint64_t *bar) {
    if (!err) return;
    const uint32_t k = atomicAdd(err + 1, 1u);
    if (k >= kTrailMax) return;
    uint64_t st = 0;
    if (bar) asm volatile("ld.shared.b64 %0, [%1];" : "=l"(st) : "r"(smem_u32(bar)));
    uint32_t *r = err + 4 + 8 * k;
    r[0] = where; r[1] = blockIdx.x; r[2] = threadIdx.x;
    r[3] = x0; r[4] = x1; r[5] = x2;
    r[6] = (uint32_t)st; r[7] = (uint32_t)(st >> 32);
}

// ---------------------------------------------------------------------------
// TMA (cp.async.bulk.tensor), no multicast.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap *m) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}

__device__ __forceinline__ void tma_load_3d(void *smem_dst, const CUtensorMap *m, uint64_t *bar,
                                            int c0, int c1, int c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];"
        ::"r"(smem_u32(smem_dst)), "l"(reinterpret_cast<uint64_t>(m)), "r"(c0), "r"(c1), "r"(c2),
          "r"(smem_u32(bar))
        : "memory");
}

// Plain bulk copy global -> shared (no tensor map, no multicast); both
// addresses 16-byte aligned, `bytes` a multiple of 16.
__device__ __forceinline__ void bulk_load(void *smem_dst, const void *gsrc, uint32_t bytes,
                                          uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(smem_u32(smem_dst)), "l"(reinterpret_cast<uint64_t>(gsrc)), "r"(bytes),
          "r"(smem_u32(bar))
        : "memory");
}

// Generic-proxy shared-memory writes -> visible to the async proxy (TMA, UMMA).
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------------------
// tcgen05: TMEM allocation, UMMA issue, commit, TMEM <-> register moves.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t *smem_slot, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(smem_u32(smem_slot)), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem], kind::f16, one CTA.
__device__ __forceinline__ void umma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                        uint32_t idesc, uint32_t accumulate) {
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
                 ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
                 : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem], kind::f16, one CTA.  A is 128 lanes (rows)
// x K 16-bit elements packed two per 32-bit column.
__device__ __forceinline__ void umma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                        uint32_t idesc, uint32_t accumulate) {
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
                 ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
                 : "memory");
}

// Eight UMMA K-steps of one block from a single asm statement, with every
// descriptor prepared beforehand: one instruction per MMA on the issuing
// thread.  The issuing warp shares its SM sub-partition with busy softmax
// warps, and each instruction it issues competes with theirs.
// `acc_first` != 0 accumulates into D at the first step; the other steps
// always accumulate.
__device__ __forceinline__ void umma_ss_x8(uint32_t d_tmem, const uint64_t (&a)[8],
                                           const uint64_t (&b)[8], uint32_t idesc,
                                           uint32_t acc_first) {
    asm volatile("{\n\t.reg .pred p, t;\n\t"
                 "setp.ne.b32 p, %18, 0;\n\t"
                 "setp.eq.b32 t, %17, %17;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %9, %17, p;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f16 [%0], %2, %10, %17, t;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f16 [%0], %3, %11, %17, t;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f16 [%0], %4, %12, %17, t;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f16 [%0], %5, %13, %17, t;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f16 [%0], %6, %14, %17, t;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f16 [%0], %7, %15, %17, t;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f16 [%0], %8, %16, %17, t;\n\t}"
                 ::"r"(d_tmem), "l"(a[0]), "l"(a[1]), "l"(a[2]), "l"(a[3]), "l"(a[4]),
                   "l"(a[5]), "l"(a[6]), "l"(a[7]), "l"(b[0]), "l"(b[1]), "l"(b[2]),
                   "l"(b[3]), "l"(b[4]), "l"(b[5]), "l"(b[6]), "l"(b[7]), "r"(idesc),
                   "r"(acc_first)
                 : "memory");
}
// Four K-steps (a 64-wide contraction), same conventions.
__device__ __forceinline__ void umma_ss_x4(uint32_t d_tmem, const uint64_t (&a)[4],
                                           const uint64_t (&b)[4], uint32_t idesc,
                                           uint32_t acc_first) {
    asm volatile("{\n\t.reg .pred p, t;\n\t"
                 "setp.ne.b32 p, %10, 0;\n\t"
                 "setp.eq.b32 t, %9, %9;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %5, %9, p;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f16 [%0], %2, %6, %9, t;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f16 [%0], %3, %7, %9, t;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f16 [%0], %4, %8, %9, t;\n\t}"
                 ::"r"(d_tmem), "l"(a[0]), "l"(a[1]), "l"(a[2]), "l"(a[3]), "l"(b[0]),
                   "l"(b[1]), "l"(b[2]), "l"(b[3]), "r"(idesc), "r"(acc_first)
                 : "memory");
}
// The same with A read from TMEM (a[k]: TMEM address of K-step k).
__device__ __forceinline__ void umma_ts_x8(uint32_t d_tmem, const uint32_t (&a)[8],
                                           const uint64_t (&b)[8], uint32_t idesc,
                                           uint32_t acc_first) {
    asm volatile("{\n\t.reg .pred p, t;\n\t"
                 "setp.ne.b32 p, %18, 0;\n\t"
                 "setp.eq.b32 t, %17, %17;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %9, %17, p;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f16 [%0], [%2], %10, %17, t;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f16 [%0], [%3], %11, %17, t;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f16 [%0], [%4], %12, %17, t;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f16 [%0], [%5], %13, %17, t;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f16 [%0], [%6], %14, %17, t;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f16 [%0], [%7], %15, %17, t;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f16 [%0], [%8], %16, %17, t;\n\t}"
                 ::"r"(d_tmem), "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(a[4]),
                   "r"(a[5]), "r"(a[6]), "r"(a[7]), "l"(b[0]), "l"(b[1]), "l"(b[2]),
                   "l"(b[3]), "l"(b[4]), "l"(b[5]), "l"(b[6]), "l"(b[7]), "r"(idesc),
                   "r"(acc_first)
                 : "memory");
}

// One tile's PV(j) and QK^T(j + 1) from a single asm statement, each
// descriptor derived inside it from its base: a thread issues a tcgen05.mma
// about every 63 cycles (measured on B200, for any N), about as long as a
// 128x128x16 step runs, so the adds issue while the thread waits for its next
// MMA slot instead of lengthening the issue path.
//   PV: O[o_col] (+)= P V, P at TMEM column p_col + 8k, V descriptor
//       v0 + 128k (16-key steps of 2048 bytes), 8 steps, accumulating from
//       the first step unless acc == 0;
//   QK: S[s_col] = Q K^T, Q and K descriptors q0 / k0 + 2k within a 64-column
//       group and + 1024 for the second group (128-row tiles), 8 steps;
//   then one commit on `bar`.
__device__ __forceinline__ void umma_pv_qk(uint32_t o_col, uint32_t p_col, uint64_t v0,
                                           uint32_t idesc_pv, uint32_t acc, uint32_t s_col,
                                           uint64_t q0, uint64_t k0, uint32_t idesc_qk,
                                           uint64_t *bar) {
    asm volatile(
        "{\n\t.reg .pred p, t, z;\n\t.reg .b64 v, q, k;\n\t.reg .b32 pa;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "setp.eq.b32 t, %4, %4;\n\t"
        "setp.ne.b32 z, %4, %4;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t"
        "add.s32 pa, %1, 8;\n\tadd.s64 v, %2, 128;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [pa], v, %3, t;\n\t"
        "add.s32 pa, %1, 16;\n\tadd.s64 v, %2, 256;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [pa], v, %3, t;\n\t"
        "add.s32 pa, %1, 24;\n\tadd.s64 v, %2, 384;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [pa], v, %3, t;\n\t"
        "add.s32 pa, %1, 32;\n\tadd.s64 v, %2, 512;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [pa], v, %3, t;\n\t"
        "add.s32 pa, %1, 40;\n\tadd.s64 v, %2, 640;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [pa], v, %3, t;\n\t"
        "add.s32 pa, %1, 48;\n\tadd.s64 v, %2, 768;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [pa], v, %3, t;\n\t"
        "add.s32 pa, %1, 56;\n\tadd.s64 v, %2, 896;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [pa], v, %3, t;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%5], %6, %7, %8, z;\n\t"
        "add.s64 q, %6, 2;\n\tadd.s64 k, %7, 2;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%5], q, k, %8, t;\n\t"
        "add.s64 q, %6, 4;\n\tadd.s64 k, %7, 4;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%5], q, k, %8, t;\n\t"
        "add.s64 q, %6, 6;\n\tadd.s64 k, %7, 6;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%5], q, k, %8, t;\n\t"
        "add.s64 q, %6, 1024;\n\tadd.s64 k, %7, 1024;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%5], q, k, %8, t;\n\t"
        "add.s64 q, %6, 1026;\n\tadd.s64 k, %7, 1026;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%5], q, k, %8, t;\n\t"
        "add.s64 q, %6, 1028;\n\tadd.s64 k, %7, 1028;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%5], q, k, %8, t;\n\t"
        "add.s64 q, %6, 1030;\n\tadd.s64 k, %7, 1030;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%5], q, k, %8, t;\n\t"
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%9];\n\t}"
        ::"r"(o_col), "r"(p_col), "l"(v0), "r"(idesc_pv), "r"(acc), "r"(s_col), "l"(q0), "l"(k0),
          "r"(idesc_qk), "r"(smem_u32(bar))
        : "memory");
}

// umma_pv_qk with one more QK^T K-step (descriptors qx / kx, accumulating)
// before the commit: the ALiBi bias step.
__device__ __forceinline__ void umma_pv_qk_x(uint32_t o_col, uint32_t p_col, uint64_t v0,
                                             uint32_t idesc_pv, uint32_t acc, uint32_t s_col,
                                             uint64_t q0, uint64_t k0, uint32_t idesc_qk,
                                             uint64_t qx, uint64_t kx, uint64_t *bar) {
    asm volatile(
        "{\n\t.reg .pred p, t, z;\n\t.reg .b64 v, q, k;\n\t.reg .b32 pa;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "setp.eq.b32 t, %4, %4;\n\t"
        "setp.ne.b32 z, %4, %4;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t"
        "add.s32 pa, %1, 8;\n\tadd.s64 v, %2, 128;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [pa], v, %3, t;\n\t"
        "add.s32 pa, %1, 16;\n\tadd.s64 v, %2, 256;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [pa], v, %3, t;\n\t"
        "add.s32 pa, %1, 24;\n\tadd.s64 v, %2, 384;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [pa], v, %3, t;\n\t"
        "add.s32 pa, %1, 32;\n\tadd.s64 v, %2, 512;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [pa], v, %3, t;\n\t"
        "add.s32 pa, %1, 40;\n\tadd.s64 v, %2, 640;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [pa], v, %3, t;\n\t"
        "add.s32 pa, %1, 48;\n\tadd.s64 v, %2, 768;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [pa], v, %3, t;\n\t"
        "add.s32 pa, %1, 56;\n\tadd.s64 v, %2, 896;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [pa], v, %3, t;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%5], %6, %7, %8, z;\n\t"
        "add.s64 q, %6, 2;\n\tadd.s64 k, %7, 2;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%5], q, k, %8, t;\n\t"
        "add.s64 q, %6, 4;\n\tadd.s64 k, %7, 4;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%5], q, k, %8, t;\n\t"
        "add.s64 q, %6, 6;\n\tadd.s64 k, %7, 6;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%5], q, k, %8, t;\n\t"
        "add.s64 q, %6, 1024;\n\tadd.s64 k, %7, 1024;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%5], q, k, %8, t;\n\t"
        "add.s64 q, %6, 1026;\n\tadd.s64 k, %7, 1026;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%5], q, k, %8, t;\n\t"
        "add.s64 q, %6, 1028;\n\tadd.s64 k, %7, 1028;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%5], q, k, %8, t;\n\t"
        "add.s64 q, %6, 1030;\n\tadd.s64 k, %7, 1030;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%5], q, k, %8, t;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%5], %10, %11, %8, t;\n\t"
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%9];\n\t}"
        ::"r"(o_col), "r"(p_col), "l"(v0), "r"(idesc_pv), "r"(acc), "r"(s_col), "l"(q0), "l"(k0),
          "r"(idesc_qk), "r"(smem_u32(bar)), "l"(qx), "l"(kx)
        : "memory");
}

// Arrive (once) on `bar` when every tcgen05 op this thread issued so far is done.
__device__ __forceinline__ void umma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 ::"r"(smem_u32(bar)) : "memory");
}

// 16x32bx2 shape: the warp reads 16 TMEM lanes; threads 0-15 take lane
// (base + t) at columns [c, c + n), threads 16-31 take lane (base + t - 16) at
// columns [c + SPLIT, c + SPLIT + n).  The two column halves of one row sit in
// lanes t and t + 16 of the same warp.
template <int SPLIT>
__device__ __forceinline__ void tmem_ld16x2_32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.16x32bx2.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32], %33;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr), "n"(SPLIT));
}
template <int SPLIT>
__device__ __forceinline__ void tmem_st16x2_32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.16x32bx2.x32.b32 [%0], %33, "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};"
        ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]),
          "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]),
          "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]),
          "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]),
          "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31]), "n"(SPLIT)
        : "memory");
}
template <int SPLIT>
__device__ __forceinline__ void tmem_st16x2_16(uint32_t taddr, const uint32_t *r) {
    asm volatile(
        "tcgen05.st.sync.aligned.16x32bx2.x16.b32 [%0], %17, "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
        ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]),
          "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]),
          "r"(r[13]), "r"(r[14]), "r"(r[15]), "n"(SPLIT)
        : "memory");
}

__device__ __forceinline__ void tmem_ld_wait() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// tcgen05.ld writes its destination registers asynchronously; they are only
// defined after tcgen05.wait::ld.  The compiler does not know that, so after
// the wait every loaded register is passed through an empty volatile asm:
// no use of it can then be scheduled above the wait.
__device__ __forceinline__ void reg_fence32(uint32_t (&r)[32]) {
    asm volatile(""
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]),
                   "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]),
                   "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]),
                   "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]),
                   "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]),
                   "+r"(r[30]), "+r"(r[31])
                 :
                 : "memory");
}
__device__ __forceinline__ void tmem_st_wait() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor for UMMA (sm_100 layout: start>>4 in
// [0,14), leading-byte-offset>>4 in [16,30), stride-byte-offset>>4 in
// [32,46), version 1 in [46,48), swizzle mode in [61,64); 2 = 128-byte swizzle).
__host__ __device__ __forceinline__ constexpr uint64_t umma_desc_sw128(uint32_t smem_addr,
                                                                      uint32_t lbo_bytes,
                                                                      uint32_t sbo_bytes) {
    return (uint64_t)((smem_addr >> 4) & 0x3FFFu)
           | (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16
           | (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32
           | (uint64_t)1u << 46
           | (uint64_t)2u << 61;
}
// The same descriptor as two 32-bit words.  The low word (start address,
// leading byte offset) is the one that moves along K; adding (bytes >> 4) to
// it advances the start address as long as the address stays below 256 KB
// (always true for shared memory), so the per-step cost is one 32-bit add.
__host__ __device__ __forceinline__ constexpr uint32_t umma_desc_lo(uint32_t smem_addr,
                                                                   uint32_t lbo_bytes) {
    return ((smem_addr >> 4) & 0x3FFFu) | (((lbo_bytes >> 4) & 0x3FFFu) << 16);
}
__host__ __device__ __forceinline__ constexpr uint32_t umma_desc_hi_sw128(uint32_t sbo_bytes) {
    return ((sbo_bytes >> 4) & 0x3FFFu) | (1u << 14) | (2u << 29);
}
// High word for an unswizzled K-major operand (layout type 0): 8-row x
// 16-byte core matrices, `sbo_bytes` between 8-row groups along M / N; the
// low word's leading byte offset is the step between the two core matrices
// of a 16-wide K-step.
__host__ __device__ __forceinline__ constexpr uint32_t umma_desc_hi_none(uint32_t sbo_bytes) {
    return ((sbo_bytes >> 4) & 0x3FFFu) | (1u << 14);
}
static_assert(umma_desc_sw128(0x2A400u + 0x460u, 16384u, 1024u) ==
                  (((uint64_t)umma_desc_hi_sw128(1024u) << 32) |
                   (umma_desc_lo(0x2A400u, 16384u) + (0x460u >> 4))),
              "split UMMA descriptor words disagree with the 64-bit form");

// Instruction descriptor for kind::f16 with an f32 accumulator.
//   ab_bf16: operands are bf16 (else f16); a_mn / b_mn: operand is MN-major.
__host__ __device__ constexpr uint32_t umma_idesc_f16(bool ab_bf16, bool a_mn, bool b_mn, int M,
                                                      int N) {
    return (1u << 4)                                  // D format: f32
           | ((ab_bf16 ? 1u : 0u) << 7)               // A format
           | ((ab_bf16 ? 1u : 0u) << 10)              // B format
           | ((a_mn ? 1u : 0u) << 15)                 // A major
           | ((b_mn ? 1u : 0u) << 16)                 // B major
           | ((uint32_t)(N >> 3) << 17)               // N / 8
           | ((uint32_t)(M >> 4) << 24);              // M / 16
}

// ---------------------------------------------------------------------------
// Legacy warp-level tensor core ops (decode kernels).
// ---------------------------------------------------------------------------
template <typename T> struct MmaType;
template <> struct MmaType<__nv_bfloat16> { static constexpr bool bf16 = true; };
template <> struct MmaType<__half> { static constexpr bool bf16 = false; };

template <bool BF16>
__device__ __forceinline__ void mma_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                          uint32_t b1) {
    if constexpr (BF16) {
        asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
                     "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
                     : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
                     : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
    } else {
        asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
                     "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
                     : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
                     : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
    }
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2,
                                        uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2,
                                          uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}

__device__ __forceinline__ void lds128(uint32_t addr, uint32_t (&v)[4]) {
    asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]) : "r"(addr));
}
__device__ __forceinline__ uint2 lds64(uint32_t addr) {
    uint2 v;
    asm volatile("ld.shared.v2.b32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
    return v;
}
__device__ __forceinline__ void sts128(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                       uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
                 "r"(d)
                 : "memory");
}
// Transpose of an 8x8 16-bit matrix held in the usual fragment layout
// (thread t: row t/4, columns 2(t%4), 2(t%4)+1).
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
    uint32_t y;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
    return y;
}
__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
}

// ---------------------------------------------------------------------------
// Host-side launch helper.
// ---------------------------------------------------------------------------
// Dynamic shared-memory opt-in for kernel KERN, set once per device: it is a
// per-context setting, and setting it on every run costs host time on the
// launch path (and is best kept out of a stream capture).  One instance of
// the flag word per kernel (KERN is a template argument).
template <auto KERN>
static cudaError_t ensure_smem_attr(int smem) {
    static std::atomic<uint64_t> done{0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const uint64_t bit = (dev >= 0 && dev < 64) ? (uint64_t(1) << dev) : 0;
    if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
    e = cudaFuncSetAttribute(KERN, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_release);
    return e;
}

// ---------------------------------------------------------------------------
// Numerics.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// ---- packed fp32 pairs (Blackwell f32x2 FMA/ADD on a 64-bit register pair) ----
// ---- per-thread asynchronous global -> shared copies (cp.async) ----
__device__ __forceinline__ void cp_async4(uint32_t dst, const void *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;" ::: "memory");
}
// wait until at most N of this thread's committed groups are still in flight
template <int N> __device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ uint64_t f2pack(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f2unpack(uint64_t v, float &lo, float &hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t fadd2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t fmul2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

template <typename T> __device__ __forceinline__ uint32_t pack2(float lo, float hi);
template <> __device__ __forceinline__ uint32_t pack2<__nv_bfloat16>(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}
template <> __device__ __forceinline__ uint32_t pack2<__half>(float lo, float hi) {
    __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

template <typename T> __device__ __forceinline__ float to_f32(T v);
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) {
    return __bfloat162float(v);
}
template <> __device__ __forceinline__ float to_f32<__half>(__half v) { return __half2float(v); }

// v rounded (to nearest even) to T and back
template <typename T> __device__ __forceinline__ float round_to(float v);
template <> __device__ __forceinline__ float round_to<__nv_bfloat16>(float v) {
    return __bfloat162float(__float2bfloat16_rn(v));
}
template <> __device__ __forceinline__ float round_to<__half>(float v) {
    return __half2float(__float2half_rn(v));
}

// 128-byte swizzle (16-byte chunk index XOR row-in-8) for a 1024-aligned region
// of 128-byte rows.
__device__ __forceinline__ uint32_t swz128(uint32_t row, uint32_t chunk16) {
    return row * 128u + ((chunk16 ^ (row & 7u)) << 4);
}

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

}  // namespace fia
