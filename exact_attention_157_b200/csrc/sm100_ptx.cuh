// sm100_ptx.cuh -- thin inline-PTX wrappers for the sm_100a features the
// attention kernel uses: mbarriers with bounded waits, TMA tiled loads/stores
// (never with cluster multicast), and the tcgen05 tensor-memory family
// (alloc / mma / commit / ld / st / fences).  Written from the public PTX ISA.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <stdint.h>

namespace attn_sm100 {

// --------------------------------------------------------------------------
// Device-side error word (bits 0-7 code, 8-15 role, 16-31 site).  The library
// is a single translation unit, so the word lives here.
// --------------------------------------------------------------------------
static __device__ unsigned int g_error_word = 0u;

enum : unsigned int { kErrTimeout = 5u, kErrDevice = 6u };

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void record_error(unsigned int code, unsigned int role, unsigned int site) {
    atomicCAS(&g_error_word, 0u, (code & 0xffu) | ((role & 0xffu) << 8) | ((site & 0xffffu) << 16));
}

// ------------------------------------------------------------------ mbarrier
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("{\n\t.reg .b64 st;\n\t"
                 "mbarrier.arrive.release.cta.shared::cta.b64 st, [%0];\n\t}"
                 :: "r"(bar) : "memory");
}

// One thread arriving on behalf of `count` expected arrivals.
__device__ __forceinline__ void mbar_arrive_cnt(uint32_t bar, uint32_t count) {
    asm volatile("{\n\t.reg .b64 st;\n\t"
                 "mbarrier.arrive.release.cta.shared::cta.b64 st, [%0], %1;\n\t}"
                 :: "r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("{\n\t.reg .b64 st;\n\t"
                 "mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 st, [%0], %1;\n\t}"
                 :: "r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
    return ok != 0;
}

// Non-blocking probe of a phase (acquire on success).
__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.test_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
    return ok != 0;
}

// Launch-wide abort: the first role of a launch whose wait expires stores the
// launch's epoch here, and every other wait of the same launch gives up at its
// next poll.  A later launch carries a new epoch and is not affected.
static __device__ unsigned int g_abort_epoch = 0u;

__device__ __forceinline__ bool launch_aborted(unsigned int epoch) {
    return *reinterpret_cast<volatile unsigned int*>(&g_abort_epoch) == epoch;
}

// Bounded wait for the phase of parity `parity` to complete.  Gives up when
// `*abort` (this CTA) becomes non-zero, when this launch was aborted, or after
// `limit_ns` of wall clock, in which case it records a timeout for
// (role, site) and aborts the CTA and the launch.  Returns true on success.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, uint64_t limit_ns,
                                          volatile int* abort, unsigned int epoch,
                                          unsigned int role, unsigned int site) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t n = 1;; ++n) {
        if (mbar_try_wait(bar, parity)) return true;
        // The slow checks run rarely, so that a phase completing meanwhile is seen
        // at once: this CTA's abort flag and the clock every 256 polls, the
        // launch-wide abort word (a global-memory read) only after 1 ms of waiting.
        if ((n & 255u) == 0u) {
            if (*abort) return false;
            const uint64_t waited = globaltimer_ns() - t0;
            if (waited > 1000000ull && launch_aborted(epoch)) {
                *abort = 1;
                return false;
            }
            if (waited > limit_ns) {
                record_error(kErrTimeout, role, site);
                *abort = 1;
                atomicExch(&g_abort_epoch, epoch);
                return false;
            }
        }
    }
}

// mbar_wait executed by every lane of a converged warp; the result is the same
// in every lane.
__device__ __forceinline__ bool mbar_wait_warp(uint32_t bar, uint32_t parity, uint64_t limit_ns,
                                               volatile int* abort, unsigned int epoch,
                                               unsigned int role, unsigned int site) {
    const bool r = mbar_wait(bar, parity, limit_ns, abort, epoch, role, site);
    return __all_sync(0xffffffffu, r);
}

// Wait used only while tearing down: lets copies or MMAs this thread already
// issued finish.  They complete in microseconds when the pipeline is sound, so
// the bound is short and independent of any abort.
constexpr uint64_t kDrainLimitNs = 20000000ull;  // 20 ms

__device__ __forceinline__ void mbar_drain(uint32_t bar, uint32_t parity, unsigned int role, unsigned int site) {
    if (mbar_try_wait(bar, parity)) return;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t n = 1;; ++n) {
        if (mbar_try_wait(bar, parity)) return;
        if ((n & 255u) == 0u && globaltimer_ns() - t0 > kDrainLimitNs) {
            record_error(kErrTimeout, role, site);
            return;
        }
    }
}

// ---------------------------------------------------------------------- TMA
__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" :: "l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 3-D tiled load global -> shared, completion counted on `bar` (no multicast).
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int x, int y, int z) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];"
        :: "r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y), "r"(z)
        : "memory");
}

// 3-D tiled store shared -> global (rows outside the tensor are not written).
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, uint32_t src, int x, int y, int z) {
    asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %4}], [%1];"
                 :: "l"(reinterpret_cast<uint64_t>(map)), "r"(src), "r"(x), "r"(y), "r"(z)
                 : "memory");
}

__device__ __forceinline__ void bulk_commit_group() {
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

__device__ __forceinline__ void bulk_wait_group_read0() {
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}

__device__ __forceinline__ void bulk_wait_group0() {
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// Make this thread's generic-proxy shared-memory writes visible to the async proxy.
__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" :: "r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void named_barrier_sync(uint32_t id, uint32_t nthreads) {
    asm volatile("bar.sync %0, %1;" :: "r"(id), "r"(nthreads) : "memory");
}

// ------------------------------------------------------------------ tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 :: "r"(dst_smem), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc]
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
                 :: "r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate) : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem desc]
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
                 :: "r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate) : "memory");
}

// Warp-collective forms: the whole (converged) warp executes them with
// warp-uniform operands and one lane chosen by elect.sync issues the
// instruction.  Keeping the issuing warp's control flow uniform lets the
// compiler hold the descriptors in uniform registers; issuing from a branch
// that only lane 0 takes costs about twice the cycles per MMA.
__device__ __forceinline__ void mma_ss_warp(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
    asm volatile("{\n\t.reg .pred p, e;\n\t"
                 "elect.sync _|e, 0xffffffff;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
                 :: "r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate) : "memory");
}

__device__ __forceinline__ void mma_ts_warp(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
    asm volatile("{\n\t.reg .pred p, e;\n\t"
                 "elect.sync _|e, 0xffffffff;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
                 :: "r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate) : "memory");
}

// kind::f8f6f4 (FP8 E4M3 operands), the same warp-collective issue
__device__ __forceinline__ void mma_ss_f8_warp(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                               uint32_t idesc, uint32_t accumulate) {
    asm volatile("{\n\t.reg .pred p, e;\n\t"
                 "elect.sync _|e, 0xffffffff;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "@e tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}"
                 :: "r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate) : "memory");
}

__device__ __forceinline__ void mma_ts_f8_warp(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                               uint32_t idesc, uint32_t accumulate) {
    asm volatile("{\n\t.reg .pred p, e;\n\t"
                 "elect.sync _|e, 0xffffffff;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "@e tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t}"
                 :: "r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate) : "memory");
}

// Batches of N MMAs into one accumulator under one elected lane, followed by up
// to two commits (a barrier address of 0 means none): one elect and one
// predicate set-up for the whole batch.  MMA i reads A at a0 + i * kAStep and B
// at b0 + i * kBStep (descriptor units of 16 bytes, or TMEM columns for a TS-form
// A); the first accumulates iff acc0 != 0, the others always.  kind::f16 (bf16)
// or kind::f8f6f4 (E4M3).
template <bool F8, int N, int kAStep, int kBStep>
__device__ __forceinline__ void mma_ss_batch_warp(uint32_t d, uint64_t a0, uint64_t b0, uint32_t idesc,
                                                  uint32_t acc0, uint32_t bar_a = 0u, uint32_t bar_b = 0u) {
    static_assert(N == 2 || N == 4, "batch size");
    if constexpr (F8 && N == 4) {
        asm volatile("{\n\t.reg .pred p, e, t, ca, cb;\n\t"
                     ".reg .b64 a;\n\t.reg .b64 b;\n\t"
                     "elect.sync _|e, 0xffffffff;\n\t"
                     "setp.ne.b32 p, %4, 0;\n\t"
                     "setp.eq.b32 t, %3, %3;\n\t"
                     "mov.b64 a, %1;\n\tmov.b64 b, %2;\n\t"
                     "@e tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], a, b, %3, p;\n\t"
                     "add.s64 a, a, %7;\n\tadd.s64 b, b, %8;\n\t"
                     "@e tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], a, b, %3, t;\n\t"
                     "add.s64 a, a, %7;\n\tadd.s64 b, b, %8;\n\t"
                     "@e tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], a, b, %3, t;\n\t"
                     "add.s64 a, a, %7;\n\tadd.s64 b, b, %8;\n\t"
                     "@e tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], a, b, %3, t;\n\t"
                     "setp.ne.b32 ca, %5, 0;\n\tand.pred ca, ca, e;\n\t"
                     "@ca tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%5];\n\t"
                     "setp.ne.b32 cb, %6, 0;\n\tand.pred cb, cb, e;\n\t"
                     "@cb tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%6];\n\t}"
                     :: "r"(d), "l"(a0), "l"(b0), "r"(idesc), "r"(acc0), "r"(bar_a), "r"(bar_b), "n"(kAStep), "n"(kBStep) : "memory");
    } else if constexpr (F8) {
        asm volatile("{\n\t.reg .pred p, e, t, ca, cb;\n\t"
                     ".reg .b64 a;\n\t.reg .b64 b;\n\t"
                     "elect.sync _|e, 0xffffffff;\n\t"
                     "setp.ne.b32 p, %4, 0;\n\t"
                     "setp.eq.b32 t, %3, %3;\n\t"
                     "mov.b64 a, %1;\n\tmov.b64 b, %2;\n\t"
                     "@e tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], a, b, %3, p;\n\t"
                     "add.s64 a, a, %7;\n\tadd.s64 b, b, %8;\n\t"
                     "@e tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], a, b, %3, t;\n\t"
                     "setp.ne.b32 ca, %5, 0;\n\tand.pred ca, ca, e;\n\t"
                     "@ca tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%5];\n\t"
                     "setp.ne.b32 cb, %6, 0;\n\tand.pred cb, cb, e;\n\t"
                     "@cb tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%6];\n\t}"
                     :: "r"(d), "l"(a0), "l"(b0), "r"(idesc), "r"(acc0), "r"(bar_a), "r"(bar_b), "n"(kAStep), "n"(kBStep) : "memory");
    } else if constexpr (N == 4) {
        asm volatile("{\n\t.reg .pred p, e, t, ca, cb;\n\t"
                     ".reg .b64 a;\n\t.reg .b64 b;\n\t"
                     "elect.sync _|e, 0xffffffff;\n\t"
                     "setp.ne.b32 p, %4, 0;\n\t"
                     "setp.eq.b32 t, %3, %3;\n\t"
                     "mov.b64 a, %1;\n\tmov.b64 b, %2;\n\t"
                     "@e tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %3, p;\n\t"
                     "add.s64 a, a, %7;\n\tadd.s64 b, b, %8;\n\t"
                     "@e tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %3, t;\n\t"
                     "add.s64 a, a, %7;\n\tadd.s64 b, b, %8;\n\t"
                     "@e tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %3, t;\n\t"
                     "add.s64 a, a, %7;\n\tadd.s64 b, b, %8;\n\t"
                     "@e tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %3, t;\n\t"
                     "setp.ne.b32 ca, %5, 0;\n\tand.pred ca, ca, e;\n\t"
                     "@ca tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%5];\n\t"
                     "setp.ne.b32 cb, %6, 0;\n\tand.pred cb, cb, e;\n\t"
                     "@cb tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%6];\n\t}"
                     :: "r"(d), "l"(a0), "l"(b0), "r"(idesc), "r"(acc0), "r"(bar_a), "r"(bar_b), "n"(kAStep), "n"(kBStep) : "memory");
    } else {
        asm volatile("{\n\t.reg .pred p, e, t, ca, cb;\n\t"
                     ".reg .b64 a;\n\t.reg .b64 b;\n\t"
                     "elect.sync _|e, 0xffffffff;\n\t"
                     "setp.ne.b32 p, %4, 0;\n\t"
                     "setp.eq.b32 t, %3, %3;\n\t"
                     "mov.b64 a, %1;\n\tmov.b64 b, %2;\n\t"
                     "@e tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %3, p;\n\t"
                     "add.s64 a, a, %7;\n\tadd.s64 b, b, %8;\n\t"
                     "@e tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %3, t;\n\t"
                     "setp.ne.b32 ca, %5, 0;\n\tand.pred ca, ca, e;\n\t"
                     "@ca tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%5];\n\t"
                     "setp.ne.b32 cb, %6, 0;\n\tand.pred cb, cb, e;\n\t"
                     "@cb tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%6];\n\t}"
                     :: "r"(d), "l"(a0), "l"(b0), "r"(idesc), "r"(acc0), "r"(bar_a), "r"(bar_b), "n"(kAStep), "n"(kBStep) : "memory");
    }
}

// kind::f16 with A (P as bf16 pairs) in tensor memory, four MMAs
template <int kAStep, int kBStep>
__device__ __forceinline__ void mma_ts4_batch_warp(uint32_t d, uint32_t a0, uint64_t b0, uint32_t idesc,
                                                   uint32_t acc0, uint32_t bar_a = 0u, uint32_t bar_b = 0u) {
    asm volatile("{\n\t.reg .pred p, e, t, ca, cb;\n\t"
                     ".reg .b32 a;\n\t.reg .b64 b;\n\t"
                     "elect.sync _|e, 0xffffffff;\n\t"
                     "setp.ne.b32 p, %4, 0;\n\t"
                     "setp.eq.b32 t, %3, %3;\n\t"
                     "mov.b32 a, %1;\n\tmov.b64 b, %2;\n\t"
                     "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %3, p;\n\t"
                     "add.u32 a, a, %7;\n\tadd.s64 b, b, %8;\n\t"
                     "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %3, t;\n\t"
                     "add.u32 a, a, %7;\n\tadd.s64 b, b, %8;\n\t"
                     "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %3, t;\n\t"
                     "add.u32 a, a, %7;\n\tadd.s64 b, b, %8;\n\t"
                     "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %3, t;\n\t"
                     "setp.ne.b32 ca, %5, 0;\n\tand.pred ca, ca, e;\n\t"
                     "@ca tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%5];\n\t"
                     "setp.ne.b32 cb, %6, 0;\n\tand.pred cb, cb, e;\n\t"
                     "@cb tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%6];\n\t}"
                 :: "r"(d), "r"(a0), "l"(b0), "r"(idesc), "r"(acc0), "r"(bar_a), "r"(bar_b), "n"(kAStep), "n"(kBStep) : "memory");
}

// Up to two commits under one elected lane (0: none).
__device__ __forceinline__ void mma_commit2_warp(uint32_t bar_a, uint32_t bar_b) {
    asm volatile("{\n\t.reg .pred e, ca, cb;\n\t"
                 "elect.sync _|e, 0xffffffff;\n\t"
                 "setp.ne.b32 ca, %0, 0;\n\tand.pred ca, ca, e;\n\t"
                 "@ca tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t"
                 "setp.ne.b32 cb, %1, 0;\n\tand.pred cb, cb, e;\n\t"
                 "@cb tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%1];\n\t}"
                 :: "r"(bar_a), "r"(bar_b) : "memory");
}

__device__ __forceinline__ void mma_commit_warp(uint32_t bar) {
    asm volatile("{\n\t.reg .pred e;\n\t"
                 "elect.sync _|e, 0xffffffff;\n\t"
                 "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}"
                 :: "r"(bar) : "memory");
}

// Arrive once on `bar` when every tcgen05 operation this thread issued so far completes.
__device__ __forceinline__ void mma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 :: "r"(bar) : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_wait_st() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Each thread of the warp reads 32 consecutive 32-bit columns of its own lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}

// Each thread of the warp reads 16 consecutive 32-bit columns of its own lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* r) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};"
        :: "r"(taddr),
           "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
           "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
        "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};"
        :: "r"(taddr),
           "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
           "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]),
           "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]),
           "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}

// ------------------------------------------------------- UMMA descriptors
// Shared-memory matrix descriptor (tcgen05 "matrix descriptor"): start address,
// leading / stride byte offsets (all >> 4), version 1, swizzle mode in [61,64).
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
    uint64_t desc = 0;
    desc |= static_cast<uint64_t>((saddr >> 4) & 0x3fffu);
    desc |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3fffu) << 16;
    desc |= static_cast<uint64_t>((sbo_bytes >> 4) & 0x3fffu) << 32;
    desc |= static_cast<uint64_t>(1u) << 46;  // descriptor version for tcgen05
    desc |= static_cast<uint64_t>(2u) << 61;  // 128-byte swizzle
    return desc;
}

// Instruction descriptor for kind::f16 with bf16 A/B and fp32 accumulation.
// b_mn_major: B stored with N contiguous (V tile) instead of K contiguous.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, bool b_mn_major) {
    return (1u << 4)                      // D format: f32
         | (1u << 7)                      // A format: bf16
         | (1u << 10)                     // B format: bf16
         | ((b_mn_major ? 1u : 0u) << 16) // B major-ness
         | (static_cast<uint32_t>(N >> 3) << 17)
         | (static_cast<uint32_t>(M >> 4) << 24);
}

// Instruction descriptor for kind::f8f6f4 with E4M3 A/B (format code 0) and fp32 accumulation.
__host__ __device__ constexpr uint32_t idesc_e4m3_f32(int M, int N, bool b_mn_major) {
    return (1u << 4)                      // D format: f32
         | ((b_mn_major ? 1u : 0u) << 16) // B major-ness
         | (static_cast<uint32_t>(N >> 3) << 17)
         | (static_cast<uint32_t>(M >> 4) << 24);
}

// ------------------------------------------------------------------- math
__device__ __forceinline__ float rcp_approx(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}

// Four values as E4M3 codes (round to nearest, saturating to +-448), the first in the low byte.
__device__ __forceinline__ uint32_t pack_e4m3x4(float a0, float a1, float a2, float a3) {
    const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(a0, a1), __NV_SATFINITE, __NV_E4M3);
    const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(a2, a3), __NV_SATFINITE, __NV_E4M3);
    return (lo & 0xffffu) | (hi << 16);
}

}  // namespace attn_sm100
