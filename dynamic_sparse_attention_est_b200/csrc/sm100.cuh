// sm100.cuh -- thin inline-PTX wrappers for the Blackwell (sm_100a) pieces the
// kernels use: mbarriers with bounded waits, TMA tiled loads, tcgen05 MMA with
// TMEM accumulators, TMEM loads/stores, and the shared-memory matrix descriptor.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

namespace minf {

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
// try_wait with a suspend-time hint: a thread whose phase is not yet complete may
// be suspended for up to `ns` nanoseconds, woken early when the phase completes.
__device__ __forceinline__ bool mbar_try_wait_hint(uint32_t bar, uint32_t parity, uint32_t ns) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(ns)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}
// Arrives on `bar` once all cp.async of this thread issued so far have landed.
__device__ __forceinline__ void cp_async_mbar_arrive(uint32_t bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}

// Shared abort/timeout state of one CTA.  Every wait in the kernels is
// bounded: after `limit_ns` it records MINF_ERR_TIMEOUT (-4) in the global
// status word, raises the CTA-local abort flag so that the other roles stop
// waiting too, and returns false.
struct WaitCtl {
    volatile int *abort_flag;  // shared memory
    int *status;               // global status word; status[1] records the site
    uint64_t limit_ns;
};

// Records a wait that gave up: sets the CTA's abort flag and the status word.
__device__ __forceinline__ void wait_gave_up(const WaitCtl &w, int site) {
    *w.abort_flag = 1;
    if (w.status) {
        atomicExch(w.status, -4);
        atomicCAS(w.status + 1, 0, site | 0x40000000);
    }
    __threadfence();
}

// `site` identifies the wait (role << 24 | barrier << 16 | tile) for diagnosis.
__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity, const WaitCtl &w, int site = 0) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (;;) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*w.abort_flag) return false;
        if (globaltimer_ns() - t0 > w.limit_ns) {
            wait_gave_up(w, site);
            return false;
        }
    }
}

// wait_bounded with suspended waiting (see mbar_try_wait_hint): far fewer
// instructions issued while a warp waits, for kernels whose waits are long.
__device__ __forceinline__ bool wait_bounded_sleep(uint32_t bar, uint32_t parity, const WaitCtl &w, int site = 0) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (;;) {
        if (mbar_try_wait_hint(bar, parity, 20000u)) return true;
        if (*w.abort_flag) return false;
        if (globaltimer_ns() - t0 > w.limit_ns) {
            wait_gave_up(w, site);
            return false;
        }
    }
}

__host__ __device__ constexpr int wait_site(int role, int barrier, int tile) {
    return (role << 24) | (barrier << 16) | (tile & 0xFFFF);
}

// --------------------------------------------------------------------- TMA
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const void *tmap, uint32_t bar, int x, int y,
                                            int z) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
        "l"(tmap), "r"(bar), "r"(x), "r"(y), "r"(z)
        : "memory");
}
// Warp-wide load of a 128-row K or V stage (two 64-row halves, each two 64-column
// boxes of a 3-D tensor map {128, n, heads}): every lane of a converged warp
// calls it with the same operands, and one lane, picked by elect.sync, adds the
// expected bytes to `bar` and issues the TMA loads of the halves flagged in
// `halves` (bit 0: rows y0 into dst, bit 1: rows y1 into dst + 8192).  Callers
// order their own arrive on `bar` after it with __syncwarp.
__device__ __forceinline__ void tma_load_stage_warp(uint32_t dst, const void *tmap, uint32_t bar, uint32_t bytes,
                                                    int y0, int y1, int z, uint32_t halves) {
    asm volatile(
        "{\n\t.reg .pred e, h0, h1;\n\t.reg .b32 f0, f1;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "and.b32 f0, %7, 1;\n\t"
        "and.b32 f1, %7, 2;\n\t"
        "setp.ne.and.b32 h0, f0, 0, e;\n\t"
        "setp.ne.and.b32 h1, f1, 0, e;\n\t"
        "@e mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%2], %3;\n\t"
        "@h0 cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
        "[%0], [%1, {0, %4, %6}], [%2];\n\t"
        "@h0 cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
        "[%8], [%1, {64, %4, %6}], [%2];\n\t"
        "@h1 cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
        "[%9], [%1, {0, %5, %6}], [%2];\n\t"
        "@h1 cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
        "[%10], [%1, {64, %5, %6}], [%2];\n\t}\n" ::"r"(dst),
        "l"(tmap), "r"(bar), "r"(bytes), "r"(y0), "r"(y1), "r"(z), "r"(halves),
        "r"(dst + 16384), "r"(dst + 8192), "r"(dst + 16384 + 8192)
        : "memory");
}
// TMA store of one box from shared memory into a 3-D tensor (bulk-group completion:
// bulk_commit closes the group, bulk_wait_read<N> waits until at most N groups of
// this thread still read shared memory, bulk_wait<N> until at most N are
// outstanding at all).  Elements outside the tensor are not written.
__device__ __forceinline__ void tma_store_3d(const void *tmap, uint32_t src, int x, int y, int z) {
    asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(tmap),
                 "r"(src), "r"(x), "r"(y), "r"(z)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
template <int N>
__device__ __forceinline__ void bulk_wait() {
    asm volatile("cp.async.bulk.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void tma_prefetch_desc(const void *tmap) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(tmap) : "memory");
}

// 16-byte cp.async (L2 only) of one chunk into shared memory.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
// Makes this thread's generic-proxy shared-memory writes visible to the async
// proxy (TMA, tensor cores).
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------------------------ tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
                 "r"(ncols)
                 : "memory");
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
// D[tmem] (+)= A[smem] * B[smem]^T, kind::f16 (bf16 in, fp32 accumulate).
__device__ __forceinline__ void umma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                        uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// D[tmem] (+)= A[tmem] * B[smem]^T, kind::f16.
__device__ __forceinline__ void umma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                        uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// One 128x128x128 tile as eight K = 16 steps in a single asm block (fewer
// instructions for the issuing thread than eight separate calls).  a0/b0 are the
// step-0 shared-memory descriptors of two K-major 128B-swizzled operands; step kk
// sits 32 bytes further within a 64-element chunk and the second chunk 16 KB on,
// i.e. +2 and +1024 in the descriptors' address field (16-byte units).  The first
// step accumulates into D iff acc_first.
__device__ __forceinline__ void umma_ss_tile(uint32_t d, uint64_t a0, uint64_t b0, uint32_t idesc,
                                             uint32_t acc_first) {
    asm volatile(
        "{\n\t.reg .pred p, t;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "setp.eq.b32 t, %3, %3;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %5, %6, %3, t;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %7, %8, %3, t;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %9, %10, %3, t;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %11, %12, %3, t;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %13, %14, %3, t;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %15, %16, %3, t;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %17, %18, %3, t;\n\t}\n" ::"r"(d),
        "l"(a0), "l"(b0), "r"(idesc), "r"(acc_first), "l"(a0 + 2), "l"(b0 + 2), "l"(a0 + 4), "l"(b0 + 4),
        "l"(a0 + 6), "l"(b0 + 6), "l"(a0 + 1024), "l"(b0 + 1024), "l"(a0 + 1026), "l"(b0 + 1026),
        "l"(a0 + 1028), "l"(b0 + 1028), "l"(a0 + 1030), "l"(b0 + 1030)
        : "memory");
}

// The P.V tile: A = P from TMEM (a_tmem, 8 columns per K = 16 step), B = an
// N-major 128B-swizzled operand whose step kk sits 2 KB further (+128 in the
// descriptor).  The first step accumulates into D iff acc_first.
__device__ __forceinline__ void umma_ts_tile(uint32_t d, uint32_t a_tmem, uint64_t b0, uint32_t idesc,
                                             uint32_t acc_first) {
    asm volatile(
        "{\n\t.reg .pred p, t;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "setp.eq.b32 t, %3, %3;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%5], %6, %3, t;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%7], %8, %3, t;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%9], %10, %3, t;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%11], %12, %3, t;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%13], %14, %3, t;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%15], %16, %3, t;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%17], %18, %3, t;\n\t}\n" ::"r"(d),
        "r"(a_tmem), "l"(b0), "r"(idesc), "r"(acc_first), "r"(a_tmem + 8), "l"(b0 + 128), "r"(a_tmem + 16),
        "l"(b0 + 256), "r"(a_tmem + 24), "l"(b0 + 384), "r"(a_tmem + 32), "l"(b0 + 512), "r"(a_tmem + 40),
        "l"(b0 + 640), "r"(a_tmem + 48), "l"(b0 + 768), "r"(a_tmem + 56), "l"(b0 + 896)
        : "memory");
}

// Warp-wide forms of umma_ss_tile / umma_ts_tile / umma_commit: every lane of a
// converged warp calls them with the same (warp-uniform) operands and
// elect.sync lets one lane issue, so the operands need not come from a
// single-lane branch.
__device__ __forceinline__ void umma_ss_tile_warp(uint32_t d, uint64_t a0, uint64_t b0, uint32_t idesc,
                                                  uint32_t acc_first) {
    asm volatile(
        "{\n\t.reg .pred p, t, e;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "setp.eq.b32 t, %3, %3;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %5, %6, %3, t;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %7, %8, %3, t;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %9, %10, %3, t;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %11, %12, %3, t;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %13, %14, %3, t;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %15, %16, %3, t;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %17, %18, %3, t;\n\t}\n" ::"r"(d),
        "l"(a0), "l"(b0), "r"(idesc), "r"(acc_first), "l"(a0 + 2), "l"(b0 + 2), "l"(a0 + 4), "l"(b0 + 4),
        "l"(a0 + 6), "l"(b0 + 6), "l"(a0 + 1024), "l"(b0 + 1024), "l"(a0 + 1026), "l"(b0 + 1026),
        "l"(a0 + 1028), "l"(b0 + 1028), "l"(a0 + 1030), "l"(b0 + 1030)
        : "memory");
}

__device__ __forceinline__ void umma_ts_tile_warp(uint32_t d, uint32_t a_tmem, uint64_t b0, uint32_t idesc,
                                                  uint32_t acc_first) {
    asm volatile(
        "{\n\t.reg .pred p, t, e;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "setp.eq.b32 t, %3, %3;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%5], %6, %3, t;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%7], %8, %3, t;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%9], %10, %3, t;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%11], %12, %3, t;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%13], %14, %3, t;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%15], %16, %3, t;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%17], %18, %3, t;\n\t}\n" ::"r"(d),
        "r"(a_tmem), "l"(b0), "r"(idesc), "r"(acc_first), "r"(a_tmem + 8), "l"(b0 + 128), "r"(a_tmem + 16),
        "l"(b0 + 256), "r"(a_tmem + 24), "l"(b0 + 384), "r"(a_tmem + 32), "l"(b0 + 512), "r"(a_tmem + 40),
        "l"(b0 + 640), "r"(a_tmem + 48), "l"(b0 + 768), "r"(a_tmem + 56), "l"(b0 + 896)
        : "memory");
}

__device__ __forceinline__ void umma_commit_warp(uint32_t bar) {
    asm volatile(
        "{\n\t.reg .pred e;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}\n" ::"r"(bar)
        : "memory");
}

// Arrives once on `bar` when every tcgen05 operation issued so far by this
// thread has completed.
__device__ __forceinline__ void umma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

// Instruction descriptor, kind::f16: fp32 D, bf16 A and B, M = 128, N = n.
// b_mn_major selects an N-major B operand (V in the P.V product).
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int n, bool b_mn_major) {
    return (1u << 4)                      // D format: fp32
           | (1u << 7)                    // A format: bf16
           | (1u << 10)                   // B format: bf16
           | ((b_mn_major ? 1u : 0u) << 16)
           | ((uint32_t)(n >> 3) << 17)   // N / 8
           | ((uint32_t)(128 >> 4) << 24);  // M / 16
}

// Shared-memory matrix descriptor for a 128-byte-swizzled operand (the layout
// TMA writes with CU_TENSOR_MAP_SWIZZLE_128B).  lbo/sbo in bytes.
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;  // descriptor version for sm_100
    d |= (uint64_t)2 << 61;  // SWIZZLE_128B
    return d;
}

// TMEM loads/stores of 32 consecutive 32-bit columns for this warp's 32 lanes
// (shape 32x32b: lane i of the warp reads TMEM lane base+i).
#define MINF_R32(r)                                                                             \
    "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),          \
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),  \
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),            \
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),            \
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
#define MINF_RW32(r)                                                                            \
    "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),          \
        "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]),  \
        "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]),            \
        "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]),            \
        "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
#define MINF_IN32(r)                                                                            \
    "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),      \
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),        \
        "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),      \
        "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),      \
        "r"(r[29]), "r"(r[30]), "r"(r[31])

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : MINF_R32(r)
        : "r"(taddr)
        : "memory");
}
// Waits for this thread's outstanding TMEM loads; the registers are tied to the
// wait so that no use of them can be scheduled before it.
__device__ __forceinline__ void tmem_ld_wait(uint32_t (&r)[32]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;" : MINF_RW32(r) : : "memory");
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        MINF_IN32(r)
        : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Packed fp32 pairs (sm_100 f32x2 arithmetic).
__device__ __forceinline__ uint64_t f32x2_pack(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f32x2_unpack(uint64_t v, float &lo, float &hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f32x2_splat(float x) { return f32x2_pack(x, x); }
__device__ __forceinline__ uint64_t f32x2_fma(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}
__device__ __forceinline__ uint64_t f32x2_add(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t f32x2_sub(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t f32x2_mul(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
// Three-input maximum (sm_100).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// Register reallocation between warpgroups (all four warps of a warpgroup execute it).
template <int N>
__device__ __forceinline__ void setmaxnreg_inc() {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void setmaxnreg_dec() {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}

__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// Named barrier over nthreads threads that also returns the OR of `v` over them.
__device__ __forceinline__ bool named_bar_or(int id, int nthreads, bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}\n"
        : "=r"(r)
        : "r"((uint32_t)v), "r"(id), "r"(nthreads)
        : "memory");
    return r != 0;
}

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

}  // namespace minf
