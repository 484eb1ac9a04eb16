// tc_primitives.cuh -- sm_100a building blocks as inline PTX: mbarriers with
// bounded waits, TMA tile loads and stores, tcgen05 tensor-memory allocation,
// MMA issue, commit, loads and stores, and the shared-memory and instruction
// descriptors of tcgen05.mma (kind::f16, bfloat16 operands, float32 accumulate).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "monarch_common.cuh"

namespace monarch {
namespace tc {

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return done != 0;
}

// Everything a bounded wait needs: the poll limit, the device status word and
// the CTA's shared abort flag (set by the first wait that gives up, so that
// the other roles stop waiting on work that will never come).
struct WaitCtx {
    long long limit;
    int *status;
    volatile int *abort;
};

// One arrival for the whole (converged) warp, on barriers that count warps:
// the lanes synchronise first, so lane 0's arrival (a release) also orders the
// other lanes' earlier writes, and the barrier takes one shared-memory atomic
// per warp instead of 32.
__device__ __forceinline__ void mbar_arrive_warp(uint64_t *bar) {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
}

// Waits for the phase with `parity` of `bar` to complete.  Returns false when
// the CTA is aborting or after `limit` polls (then it records
// MONARCH_ERR_TIMEOUT and raises the abort flag).  Never traps, never spins
// without bound.
__device__ __forceinline__ bool wait_phase(uint64_t *bar, uint32_t parity, const WaitCtx &w) {
    if (mbar_try_wait(bar, parity)) return true;
    for (long long i = 1;; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 63) == 0) {
            if (*w.abort) return false;
            if (i >= w.limit) {
                record_status(w.status, MONARCH_ERR_TIMEOUT);
                *w.abort = 1;
                return false;
            }
        }
    }
}

// Waits with a fixed poll limit and no abort shortcut (clean-up paths).
__device__ __forceinline__ bool wait_phase_cleanup(uint64_t *bar, uint32_t parity,
                                                   long long limit) {
    for (long long i = 0; i < limit; ++i)
        if (mbar_try_wait(bar, parity)) return true;
    return false;
}

// ---------------------------------------------------------------- TMA
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int x, int y,
                                            uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}
__device__ __forceinline__ void tma_load_3d(void *dst, const CUtensorMap *map, int x, int y, int z,
                                            uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
        : "memory");
}
__device__ __forceinline__ void tma_load_4d(void *dst, const CUtensorMap *map, int x, int y, int z,
                                            int w, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(w), "r"(smem_u32(bar))
        : "memory");
}
__device__ __forceinline__ void tma_load_5d(void *dst, const CUtensorMap *map, int x, int y, int z,
                                            int w, int u, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.5d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4, %5, %6}], [%7];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(w), "r"(u),
        "r"(smem_u32(bar))
        : "memory");
}
// Bulk prefetch of a tile into L2 (no shared memory, no completion tracking).
__device__ __forceinline__ void tma_prefetch_5d(const CUtensorMap *map, int x, int y, int z, int w,
                                                int u) {
    asm volatile("cp.async.bulk.prefetch.tensor.5d.L2.global [%0, {%1, %2, %3, %4, %5}];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(x), "r"(y), "r"(z), "r"(w), "r"(u)
                 : "memory");
}
__device__ __forceinline__ void tma_prefetch_2d(const CUtensorMap *map, int x, int y) {
    asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global [%0, {%1, %2}];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(x), "r"(y)
                 : "memory");
}
__device__ __forceinline__ void tma_prefetch_3d(const CUtensorMap *map, int x, int y, int z) {
    asm volatile("cp.async.bulk.prefetch.tensor.3d.L2.global [%0, {%1, %2, %3}];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(x), "r"(y), "r"(z)
                 : "memory");
}
// Bulk copy of `bytes` (multiple of 16, both addresses 16-byte aligned) from
// global to shared memory, completing on an mbarrier transaction count.
__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes,
                                          uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
            "r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}
__device__ __forceinline__ void tma_store_4d(const CUtensorMap *map, const void *src, int x, int y,
                                             int z, int w) {
    asm volatile(
        "cp.async.bulk.tensor.4d.global.shared::cta.bulk_group [%0, {%2, %3, %4, %5}], [%1];" ::
            "l"(reinterpret_cast<uint64_t>(map)),
        "r"(smem_u32(src)), "r"(x), "r"(y), "r"(z), "r"(w)
        : "memory");
}
__device__ __forceinline__ void tma_store_5d(const CUtensorMap *map, const void *src, int x, int y,
                                             int z, int w, int u) {
    asm volatile(
        "cp.async.bulk.tensor.5d.global.shared::cta.bulk_group [%0, {%2, %3, %4, %5, %6}], [%1];" ::
            "l"(reinterpret_cast<uint64_t>(map)),
        "r"(smem_u32(src)), "r"(x), "r"(y), "r"(z), "r"(w), "r"(u)
        : "memory");
}
__device__ __forceinline__ void tma_store_commit() {
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
__device__ __forceinline__ void tma_store_wait_read_all() {
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// Waits until at most one of this thread's bulk store groups still reads its
// shared-memory source (the older ones are done reading).
__device__ __forceinline__ void tma_store_wait_read_le1() {
    asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}
__device__ __forceinline__ void tma_store_wait_all() {
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}
// Makes generic-proxy writes to shared memory visible to the async proxy (TMA).
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------- tcgen05
// Allocation is warp-wide; the base column address is written to *slot.
__device__ __forceinline__ void tmem_alloc(uint32_t *slot, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(slot)),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t base, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(base), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T-ish per the descriptors.
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// D[tmem] (+)= A[tmem] * B[smem].
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// The mbarrier receives one arrive once every MMA issued so far by this thread is done.
__device__ __forceinline__ void mma_commit(uint64_t *bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            smem_u32(bar))
        : "memory");
}

// Warp-collective forms of the three calls above: every lane of a converged
// warp executes them with the same (warp-uniform) operands and elect.sync
// picks the lane that issues.  Keeping the issuing warp convergent lets the
// operands live in uniform registers; an MMA issued from a one-lane divergent
// branch costs several times more issue slots, which the softmax warps sharing
// the SM sub-partition then take away (measured: 209 instead of 97 clocks per
// M128 N128 K16 MMA next to FMA-bound warps, against 64 on a quiet SM).
__device__ __forceinline__ void mma_ss_warp(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p, e;\n\tsetp.ne.b32 p, %4, 0;\n\telect.sync _|e, 0xffffffff;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
__device__ __forceinline__ void mma_ts_warp(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p, e;\n\tsetp.ne.b32 p, %4, 0;\n\telect.sync _|e, 0xffffffff;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
__device__ __forceinline__ void mma_commit_warp(uint64_t *bar) {
    asm volatile(
        "{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\t"
        "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(
            smem_u32(bar))
        : "memory");
}

// One K-group of up to eight MMAs (K = 16 each) from one elect.sync region:
// D (+)= sum over k < n of A_k B_k, the first product accumulating into D only
// when acc0 != 0.  The descriptors come precomputed (loop invariants of the
// caller), so the issuing warp spends about one instruction per MMA; with
// per-MMA descriptor arithmetic the same sequence issued at 97 clocks per
// M128 N128 K16 MMA next to FMA-bound warps, grouped and precomputed at 66.
__device__ __forceinline__ void mma_group_ss(uint32_t d_tmem, const uint64_t (&a)[8],
                                             const uint64_t (&b)[8], uint32_t idesc,
                                             uint32_t acc0, uint32_t n) {
    asm volatile(
        "{\n\t.reg .pred e, p0, q1, q2, q3, q4, q5, q6, q7;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "setp.ne.and.b32 p0, %17, 0, e;\n\t"
        "setp.gt.and.u32 q1, %19, 1, e;\n\tsetp.gt.and.u32 q2, %19, 2, e;\n\t"
        "setp.gt.and.u32 q3, %19, 3, e;\n\tsetp.gt.and.u32 q4, %19, 4, e;\n\t"
        "setp.gt.and.u32 q5, %19, 5, e;\n\tsetp.gt.and.u32 q6, %19, 6, e;\n\t"
        "setp.gt.and.u32 q7, %19, 7, e;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %9, %18, p0;\n\t"
        "@q1 tcgen05.mma.cta_group::1.kind::f16 [%0], %2, %10, %18, 1;\n\t"
        "@q2 tcgen05.mma.cta_group::1.kind::f16 [%0], %3, %11, %18, 1;\n\t"
        "@q3 tcgen05.mma.cta_group::1.kind::f16 [%0], %4, %12, %18, 1;\n\t"
        "@q4 tcgen05.mma.cta_group::1.kind::f16 [%0], %5, %13, %18, 1;\n\t"
        "@q5 tcgen05.mma.cta_group::1.kind::f16 [%0], %6, %14, %18, 1;\n\t"
        "@q6 tcgen05.mma.cta_group::1.kind::f16 [%0], %7, %15, %18, 1;\n\t"
        "@q7 tcgen05.mma.cta_group::1.kind::f16 [%0], %8, %16, %18, 1;\n\t}" ::"r"(d_tmem),
        "l"(a[0]), "l"(a[1]), "l"(a[2]), "l"(a[3]), "l"(a[4]), "l"(a[5]), "l"(a[6]), "l"(a[7]),
        "l"(b[0]), "l"(b[1]), "l"(b[2]), "l"(b[3]), "l"(b[4]), "l"(b[5]), "l"(b[6]), "l"(b[7]),
        "r"(acc0), "r"(idesc), "r"(n)
        : "memory");
}
// The same with A in TMEM: K-step k reads columns a_tmem + 8k (bf16 pairs).
__device__ __forceinline__ void mma_group_ts(uint32_t d_tmem, uint32_t a_tmem,
                                             const uint64_t (&b)[8], uint32_t idesc,
                                             uint32_t acc0, uint32_t n) {
    asm volatile(
        "{\n\t.reg .pred e, p0, q1, q2, q3, q4, q5, q6, q7;\n\t"
        ".reg .b32 a1, a2, a3, a4, a5, a6, a7;\n\t"
        "add.u32 a1, %1, 8;\n\tadd.u32 a2, %1, 16;\n\tadd.u32 a3, %1, 24;\n\t"
        "add.u32 a4, %1, 32;\n\tadd.u32 a5, %1, 40;\n\tadd.u32 a6, %1, 48;\n\t"
        "add.u32 a7, %1, 56;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "setp.ne.and.b32 p0, %10, 0, e;\n\t"
        "setp.gt.and.u32 q1, %12, 1, e;\n\tsetp.gt.and.u32 q2, %12, 2, e;\n\t"
        "setp.gt.and.u32 q3, %12, 3, e;\n\tsetp.gt.and.u32 q4, %12, 4, e;\n\t"
        "setp.gt.and.u32 q5, %12, 5, e;\n\tsetp.gt.and.u32 q6, %12, 6, e;\n\t"
        "setp.gt.and.u32 q7, %12, 7, e;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %11, p0;\n\t"
        "@q1 tcgen05.mma.cta_group::1.kind::f16 [%0], [a1], %3, %11, 1;\n\t"
        "@q2 tcgen05.mma.cta_group::1.kind::f16 [%0], [a2], %4, %11, 1;\n\t"
        "@q3 tcgen05.mma.cta_group::1.kind::f16 [%0], [a3], %5, %11, 1;\n\t"
        "@q4 tcgen05.mma.cta_group::1.kind::f16 [%0], [a4], %6, %11, 1;\n\t"
        "@q5 tcgen05.mma.cta_group::1.kind::f16 [%0], [a5], %7, %11, 1;\n\t"
        "@q6 tcgen05.mma.cta_group::1.kind::f16 [%0], [a6], %8, %11, 1;\n\t"
        "@q7 tcgen05.mma.cta_group::1.kind::f16 [%0], [a7], %9, %11, 1;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b[0]), "l"(b[1]), "l"(b[2]), "l"(b[3]), "l"(b[4]), "l"(b[5]),
        "l"(b[6]), "l"(b[7]), "r"(acc0), "r"(idesc), "r"(n)
        : "memory");
}

// Eight K-steps (K = 128) of D (+)= A B^T with both operands 128-deep, K-major,
// 128-byte swizzled tiles of two 64-column panels (16 KB apart): K-step k starts
// (k & 3) * 32 bytes into panel k >> 2, i.e. the base descriptors plus
// (k >> 2) * 1024 + (k & 3) * 2 in 16-byte units.  The warp stays convergent;
// elect.sync picks the issuing lane, and the seven offset descriptors are formed
// inside the asm block, so the issuing warp needs no registers for them.
__device__ __forceinline__ void mma8_ss_k128(uint32_t d_tmem, uint64_t a, uint64_t b,
                                             uint32_t idesc, uint32_t acc0) {
    asm volatile(
        "{\n\t.reg .pred e, p0;\n\t"
        ".reg .b64 a1, a2, a3, a4, a5, a6, a7, b1, b2, b3, b4, b5, b6, b7;\n\t"
        "add.s64 a1, %1, 2;\n\tadd.s64 a2, %1, 4;\n\tadd.s64 a3, %1, 6;\n\t"
        "add.s64 a4, %1, 1024;\n\tadd.s64 a5, %1, 1026;\n\tadd.s64 a6, %1, 1028;\n\t"
        "add.s64 a7, %1, 1030;\n\t"
        "add.s64 b1, %2, 2;\n\tadd.s64 b2, %2, 4;\n\tadd.s64 b3, %2, 6;\n\t"
        "add.s64 b4, %2, 1024;\n\tadd.s64 b5, %2, 1026;\n\tadd.s64 b6, %2, 1028;\n\t"
        "add.s64 b7, %2, 1030;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "setp.ne.and.b32 p0, %4, 0, e;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p0;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], a1, b1, %3, 1;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], a2, b2, %3, 1;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], a3, b3, %3, 1;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], a4, b4, %3, 1;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], a5, b5, %3, 1;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], a6, b6, %3, 1;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], a7, b7, %3, 1;\n\t}" ::"r"(d_tmem),
        "l"(a), "l"(b), "r"(idesc), "r"(acc0)
        : "memory");
}
// Eight K-steps (K = 128) of D (+)= A B with A in tensor memory (bfloat16 pairs,
// K-step k at columns a_tmem + 8k) and B an MN-major 128-byte swizzled tile
// whose K-step k starts 16 rows = 2048 bytes further (descriptor + 128k).
__device__ __forceinline__ void mma8_ts_mn128(uint32_t d_tmem, uint32_t a_tmem, uint64_t b,
                                              uint32_t idesc, uint32_t acc0) {
    asm volatile(
        "{\n\t.reg .pred e, p0;\n\t"
        ".reg .b32 a1, a2, a3, a4, a5, a6, a7;\n\t"
        ".reg .b64 b1, b2, b3, b4, b5, b6, b7;\n\t"
        "add.u32 a1, %1, 8;\n\tadd.u32 a2, %1, 16;\n\tadd.u32 a3, %1, 24;\n\t"
        "add.u32 a4, %1, 32;\n\tadd.u32 a5, %1, 40;\n\tadd.u32 a6, %1, 48;\n\t"
        "add.u32 a7, %1, 56;\n\t"
        "add.s64 b1, %2, 128;\n\tadd.s64 b2, %2, 256;\n\tadd.s64 b3, %2, 384;\n\t"
        "add.s64 b4, %2, 512;\n\tadd.s64 b5, %2, 640;\n\tadd.s64 b6, %2, 768;\n\t"
        "add.s64 b7, %2, 896;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "setp.ne.and.b32 p0, %4, 0, e;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p0;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a1], b1, %3, 1;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a2], b2, %3, 1;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a3], b3, %3, 1;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a4], b4, %3, 1;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a5], b5, %3, 1;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a6], b6, %3, 1;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a7], b7, %3, 1;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b), "r"(idesc), "r"(acc0)
        : "memory");
}

// One K-step (K = 16) of D += A B^T, both operands one 32-byte-swizzled K atom.
// D (+)= A * B over K = 64: A (M = 128 x 64, bfloat16) in tensor memory, B an
// MN-major SW128 shared-memory operand; four K-steps of 16 (A advances 8
// columns, B 16 rows = 2 KB per step).
__device__ __forceinline__ void mma4_ts_mn64(uint32_t d_tmem, uint32_t a_tmem, uint64_t b,
                                             uint32_t idesc, uint32_t acc0) {
    asm volatile(
        "{\n\t.reg .pred e, p0;\n\t"
        ".reg .b32 a1, a2, a3;\n\t"
        ".reg .b64 b1, b2, b3;\n\t"
        "add.u32 a1, %1, 8;\n\tadd.u32 a2, %1, 16;\n\tadd.u32 a3, %1, 24;\n\t"
        "add.s64 b1, %2, 128;\n\tadd.s64 b2, %2, 256;\n\tadd.s64 b3, %2, 384;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "setp.ne.and.b32 p0, %4, 0, e;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p0;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a1], b1, %3, 1;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a2], b2, %3, 1;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a3], b3, %3, 1;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b), "r"(idesc), "r"(acc0)
        : "memory");
}

__device__ __forceinline__ void mma1_ss_acc(uint32_t d_tmem, uint64_t a, uint64_t b,
                                            uint32_t idesc) {
    asm volatile(
        "{\n\t.reg .pred e;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, 1;\n\t}" ::"r"(d_tmem),
        "l"(a), "l"(b), "r"(idesc)
        : "memory");
}

// Warpgroup register reallocation (all four warps of a warpgroup execute the
// same call): dec returns registers to the CTA's pool, inc waits until the pool
// can give the warp N registers per thread.  The pool is what the block was
// launched with, so the warpgroups' final counts must sum to at most that.
template <int N> __device__ __forceinline__ void regs_dec() {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N> __device__ __forceinline__ void regs_inc() {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}

// Warp-collective loads/stores of 32 lanes x N consecutive 32-bit columns:
// lane i of the warp reads/writes TMEM lane (32*(warp%4) + i).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
        "%28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr));
}
// Same load into float registers (the bits are reinterpreted, not converted).
__device__ __forceinline__ void tmem_ld32f(uint32_t taddr, float *r) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
        "%28, %29, %30, %31}, [%32];"
        : "=f"(r[0]), "=f"(r[1]), "=f"(r[2]), "=f"(r[3]), "=f"(r[4]), "=f"(r[5]), "=f"(r[6]),
          "=f"(r[7]), "=f"(r[8]), "=f"(r[9]), "=f"(r[10]), "=f"(r[11]), "=f"(r[12]),
          "=f"(r[13]), "=f"(r[14]), "=f"(r[15]), "=f"(r[16]), "=f"(r[17]), "=f"(r[18]),
          "=f"(r[19]), "=f"(r[20]), "=f"(r[21]), "=f"(r[22]), "=f"(r[23]), "=f"(r[24]),
          "=f"(r[25]), "=f"(r[26]), "=f"(r[27]), "=f"(r[28]), "=f"(r[29]), "=f"(r[30]),
          "=f"(r[31])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_st32f(uint32_t taddr, const float *r) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
        "%28, %29, %30, %31, %32};" ::"r"(taddr),
        "f"(r[0]), "f"(r[1]), "f"(r[2]), "f"(r[3]), "f"(r[4]), "f"(r[5]), "f"(r[6]), "f"(r[7]),
        "f"(r[8]), "f"(r[9]), "f"(r[10]), "f"(r[11]), "f"(r[12]), "f"(r[13]), "f"(r[14]),
        "f"(r[15]), "f"(r[16]), "f"(r[17]), "f"(r[18]), "f"(r[19]), "f"(r[20]), "f"(r[21]),
        "f"(r[22]), "f"(r[23]), "f"(r[24]), "f"(r[25]), "f"(r[26]), "f"(r[27]), "f"(r[28]),
        "f"(r[29]), "f"(r[30]), "f"(r[31])
        : "memory");
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld16f(uint32_t taddr, float *r) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15}, [%16];"
        : "=f"(r[0]), "=f"(r[1]), "=f"(r[2]), "=f"(r[3]), "=f"(r[4]), "=f"(r[5]), "=f"(r[6]),
          "=f"(r[7]), "=f"(r[8]), "=f"(r[9]), "=f"(r[10]), "=f"(r[11]), "=f"(r[12]),
          "=f"(r[13]), "=f"(r[14]), "=f"(r[15])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
        "%28, %29, %30, %31, %32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
        "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
        "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(
            taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
        : "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// ---------------------------------------------------------------- descriptors
// Shared-memory matrix descriptor of tcgen05 for the 128-byte swizzle: start
// address, leading and stride byte offsets (16-byte units), descriptor
// version 1 (bits 46-47) and layout type 2 = SWIZZLE_128B (bits 61-63).
//  K-major operand (rows of 64 bf16 = 128 B along K, 8-row atoms of 1024 B):
//    SBO = 1024 (next 8-row group); LBO unused; a K step of 16 elements
//    advances the start address by 32 B inside the atom.
//  MN-major operand (64 MN-contiguous elements per 128-B row, rows along K):
//    LBO = byte distance between consecutive 64-element MN groups,
//    SBO = 1024 (next group of 8 K rows); a K step of 16 rows advances 2048 B.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((addr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}

// The same for the 32-byte swizzle (layout type 6): K-major rows of 16
// bfloat16 (32 bytes), 8-row atoms of 256 bytes (SBO); the tile base must be
// 256-byte aligned.
__device__ __forceinline__ uint64_t smem_desc_sw32(uint32_t addr) {
    uint64_t d = 0;
    d |= (uint64_t)((addr >> 4) & 0x3FFFu);
    d |= (uint64_t)1 << 16;                       // LBO: unused for one K atom
    d |= (uint64_t)((256u >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)6 << 61;
    return d;
}

// The start-address field holds (address >> 4) in 14 bits; shared memory is
// below 256 KB, so adding (bytes >> 4) to a descriptor never carries out of the
// field: descriptors for K steps are a base descriptor plus a constant.
__device__ __forceinline__ uint64_t desc_plus(uint64_t desc, uint32_t bytes) {
    return desc + (uint64_t)(bytes >> 4);
}

// Instruction descriptor, kind::f16: D float32 (bits 4-5 = 1), A and B
// bfloat16 (bits 7-9 = 1, 10-12 = 1), A/B major (bits 15/16: 0 = K, 1 = MN),
// N >> 3 in bits 17-22, M >> 4 in bits 24-28.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, int a_mn_major, int b_mn_major) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)a_mn_major << 15) |
           ((uint32_t)b_mn_major << 16) | ((uint32_t)(N >> 3) << 17) |
           ((uint32_t)(M >> 4) << 24);
}

// ---------------------------------------------------------------- packed float32 pairs
// sm_100 executes fma/add/mul on two float32 values held in one 64-bit register.
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float &lo, float &hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}
// Non-suspending poll of an mbarrier phase (for the single MMA-issuing thread).
__device__ __forceinline__ bool mbar_test_wait(uint64_t *bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return done != 0;
}
// Bounded spin with test_wait: lowest wake-up latency, for one thread only.
__device__ __forceinline__ bool spin_phase(uint64_t *bar, uint32_t parity, const WaitCtx &w) {
    for (long long i = 0;; ++i) {
        if (mbar_test_wait(bar, parity)) return true;
        if ((i & 255) == 255) {
            if (*w.abort) return false;
            if (i >= 16 * w.limit) {
                record_status(w.status, MONARCH_ERR_TIMEOUT);
                *w.abort = 1;
                return false;
            }
        }
    }
}

// spin_phase for a whole warp: every lane polls, and the warp takes one decision.
__device__ __forceinline__ bool spin_warp(uint64_t *bar, uint32_t parity, const WaitCtx &w) {
    const bool ok = spin_phase(bar, parity, w);
    return __all_sync(0xffffffffu, ok);
}

// ---------------------------------------------------------------- math
// 2^d for a packed pair of float32 values d <= 0 (finite), on the FMA and
// integer pipes instead of the MUFU.  Range reduction after Cody and Waite:
// d = j + f with j = floor(d) (the round-down addition of 1.5 * 2^23 leaves j in
// the low mantissa bits) and f in [0, 1); 2^f is the degree-3 polynomial that
// minimises the maximum relative error on [0, 1) (Remez exchange; 7.5e-5 in
// float32), and 2^j enters by adding j << 23 to the polynomial's bit pattern.
// j is clamped to -126: the polynomial lies in [0.99992, 2), so the exponent
// field of the result never goes below zero, and results below 2^-126 come out
// as values of at most 2^-125 (zero after the bfloat16 rounding of P would be
// no more accurate: such terms vanish next to the row maximum's 2^0).
__device__ __forceinline__ uint64_t exp2_poly_x2(uint64_t d) {
    const uint64_t magic = f2_pack(12582912.f, 12582912.f);
    const uint64_t neg_magic = f2_pack(-12582912.f, -12582912.f);
    const uint64_t neg_one = f2_pack(-1.f, -1.f);
    uint64_t t, jf, f, p;
    asm("add.rm.f32x2 %0, %1, %2;" : "=l"(t) : "l"(d), "l"(magic));   // magic + floor(d)
    jf = f2_add(t, neg_magic);                                        // floor(d), exact
    f = f2_fma(jf, neg_one, d);                                       // d - floor(d)
    p = f2_fma(f, f2_pack(0.07802452147006989f, 0.07802452147006989f),
               f2_pack(0.22606715559959412f, 0.22606715559959412f));
    p = f2_fma(p, f, f2_pack(0.6958335638046265f, 0.6958335638046265f));
    p = f2_fma(p, f, f2_pack(0.9999251961708069f, 0.9999251961708069f));
    uint32_t tlo, thi, plo, phi;
    asm("mov.b64 {%0, %1}, %2;" : "=r"(tlo), "=r"(thi) : "l"(t));
    asm("mov.b64 {%0, %1}, %2;" : "=r"(plo), "=r"(phi) : "l"(p));
    const int lo_min = 0x4B400000 - 126;
    tlo = (uint32_t)max((int)tlo, lo_min);
    thi = (uint32_t)max((int)thi, lo_min);
    // (magic + j) << 23 == j << 23 (mod 2^32): the magic's set bits shift out
    plo = tlo * 8388608u + plo;
    phi = thi * 8388608u + phi;
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(plo), "r"(phi));
    return r;
}

__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float fast_log2(float x) {
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
// Two floats -> packed bfloat16 pair (lo in bits 0-15), round to nearest even.
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

}  // namespace tc
}  // namespace monarch
