// diag.cu -- Vertical-Slash attention over sparse slash groups, on the CUDA cores.
//
// A slash line is the diagonal of the attention matrix at a fixed offset o:
// query i meets key i - o (AICon talk "以 KV 缓存为中心的高效长文本方法", the
// vertical and slash observation).  Where the estimated offsets are dense, the
// tensor-core kernel computes their key ranges as whole 128x128 tiles and masks
// them (news article "单卡A100实现百万token推理…", Figure 4: slashes as dense
// blocks).  Where they are sparse -- an offset alone, or a few within 128 of one
// another -- a 128-row query tile meets each offset in only one key per row, and
// a 128x128 tile wastes 127 of every 128 products and exponentials.  This kernel
// takes those groups instead: for each query tile it stages the groups' key
// ranges in 128-key chunks (K and V, by TMA, as the tile kernel does), and each
// query row computes only its in-mask pairs, one dot product, one exponential
// and one V update per offset (fp32 sums of products of bf16 operands).
//
// It produces a partial softmax state per query row over exactly those pairs
// (each slash pair whose key is not a vertical key; verticals belong to the tile
// kernel) -- the running max m and sum l in the log2 domain and the unnormalised
// O -- which the tile kernel merges into its own in its epilogue.
//
// Roles (384 threads, one persistent CTA per SM striding over the work items):
//   warp 0      TMA producer: one 128-key chunk of K and V per stage, 3 stages
//   warps 1..3  idle (they give their registers to the consumers and exit)
//   warps 4..11 consumers: two threads per query row (lane l of warp 4 + w holds
//               row 16 w + (l & 15) and head dims [64 (l >> 4), 64 (l >> 4) + 64))
// A chunk stays until every consumer warp has moved past it; each warp releases
// chunks in order, after it has seen them full.
#include <algorithm>
#include <climits>

#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace minf {

namespace {

constexpr int kConsumerWarps = 8;
constexpr int kDiagThreads = 384;  // warpgroup 0: producer (warp 0) + 3 idle warps; warpgroups 1-2: consumers
// Register split after setmaxnreg: the launch gives 384 threads x 168 registers (three
// warps per SM sub-partition); warpgroup 0 drops to 40, the consumers rise to 232
// (128 x 40 + 256 x 232 = 384 x 168).
constexpr int kDiagRegsLaunch = 168;
constexpr int kDiagRegsProducer = 40;
constexpr int kDiagRegsConsumer = 232;
static_assert(128 * kDiagRegsProducer + 256 * kDiagRegsConsumer <= kDiagThreads * kDiagRegsLaunch, "register split");
constexpr int kDiagStages = 3;
constexpr int kChunkKeys = 128;
constexpr uint32_t kChunkBytes = 65536;  // 128 keys x 128 dims x 2 B, K then V
constexpr uint32_t kDiagSmem = kDiagStages * kChunkBytes + 256 + 1024;  // + barriers + alignment slack

// (acc0, acc1) += (lo(a) lo(b), hi(a) hi(b)): bf16 operands, fp32 products and
// sums (one rounding per fused multiply-add, as an fp32 FMA of the widened
// operands); two independent accumulators.
__device__ __forceinline__ void dot2_bf16(uint32_t a, uint32_t b, float &acc0, float &acc1) {
    asm("{\n\t.reg .b16 al, ah, bl, bh;\n\t"
        "mov.b32 {al, ah}, %2;\n\t"
        "mov.b32 {bl, bh}, %3;\n\t"
        "fma.rn.f32.bf16 %0, al, bl, %0;\n\t"
        "fma.rn.f32.bf16 %1, ah, bh, %1;\n\t}"
        : "+f"(acc0), "+f"(acc1)
        : "r"(a), "r"(b));
}

// (o0, o1) += p * (lo(v), hi(v)) with p and v bf16, o fp32.
__device__ __forceinline__ void axpy2_bf16(uint32_t v, uint16_t p, float &o0, float &o1) {
    asm("{\n\t.reg .b16 vl, vh;\n\t"
        "mov.b32 {vl, vh}, %2;\n\t"
        "fma.rn.f32.bf16 %0, %3, vl, %0;\n\t"
        "fma.rn.f32.bf16 %1, %3, vh, %1;\n\t}"
        : "+f"(o0), "+f"(o1)
        : "r"(v), "h"(p));
}

__device__ __forceinline__ uint16_t bf16_bits(float x) {
    uint16_t r;
    asm("cvt.rn.bf16.f32 %0, %1;" : "=h"(r) : "f"(x));
    return r;
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr) : "memory");
    return v;
}

// Warp-wide TMA load of one chunk: keys [y, y + 128) of kv-head z, K into
// dst[0, 32K) and V into dst[32K, 64K).  Each of the two 64-column halves of K
// (and of V) is 128 rows of 128 bytes, 128B-swizzled, loaded as two 64-row
// boxes.  Every lane calls it with the same operands; elect.sync picks the lane
// that adds the 64 KB to `bar` and issues the eight loads.
__device__ __forceinline__ void tma_load_kv_chunk_warp(uint32_t dst, const void *tmap_k, const void *tmap_v,
                                                       uint32_t bar, int y, int z) {
    asm volatile(
        "{\n\t.reg .pred e;\n\t.reg .b32 y1;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "add.s32 y1, %4, 64;\n\t"
        "@e mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%2], 65536;\n\t"
        "@e cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
        "[%0], [%1, {0, %4, %5}], [%2];\n\t"
        "@e cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
        "[%6], [%1, {0, y1, %5}], [%2];\n\t"
        "@e cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
        "[%7], [%1, {64, %4, %5}], [%2];\n\t"
        "@e cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
        "[%8], [%1, {64, y1, %5}], [%2];\n\t"
        "@e cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
        "[%9], [%3, {0, %4, %5}], [%2];\n\t"
        "@e cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
        "[%10], [%3, {0, y1, %5}], [%2];\n\t"
        "@e cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
        "[%11], [%3, {64, %4, %5}], [%2];\n\t"
        "@e cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
        "[%12], [%3, {64, y1, %5}], [%2];\n\t}\n" ::"r"(dst),
        "l"(tmap_k), "r"(bar), "l"(tmap_v), "r"(y), "r"(z), "r"(dst + 8192), "r"(dst + 16384), "r"(dst + 24576),
        "r"(dst + 32768), "r"(dst + 40960), "r"(dst + 49152), "r"(dst + 57344)
        : "memory");
}

__global__ void __launch_bounds__(kDiagThreads, 1) vs_diag_kernel(const __grid_constant__ DiagParams P) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t ring = smem_u32(smem);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kDiagStages * kChunkBytes);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(bars + 2 * kDiagStages);
    // per stage: bit u of its two words set iff key (chunk start + u) is a vertical key
    // (written by the producer before it arrives on the stage's full barrier)
    uint64_t *vmask = bars + 2 * kDiagStages + 1;
    auto full_bar = [&](int s) { return smem_u32(bars + s); };
    auto empty_bar = [&](int s) { return smem_u32(bars + kDiagStages + s); };
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kDiagStages; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), kConsumerWarps);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    const WaitCtl wc{abort_flag, P.hdr ? &P.hdr->status : nullptr, P.wait_limit_ns};
    const int n_items = P.n_heads * P.n_qtiles;

    if (warp < 4) {
        setmaxnreg_dec<kDiagRegsProducer>();
        if (warp != 0) return;
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            tma_prefetch_desc(&P.tmap_k);
            tma_prefetch_desc(&P.tmap_v);
        }
        __syncwarp();
        int c = 0;  // chunks issued by this CTA, over all its work items
        bool ok = true;
        for (int it = blockIdx.x; ok && it < n_items; it += gridDim.x) {
            // heaviest query tiles first (a tile meets every offset at or below its last row)
            const int t = P.n_qtiles - 1 - it / P.n_heads, hp = it % P.n_heads;
            const int ng = P.ngroups[hp];
            const int4 *groups = P.groups + (size_t)hp * P.gstride;
            const int g = P.head_ids[hp] / P.group;
            const uint32_t *bv = P.bits_v + (size_t)hp * P.bit_stride;
            const int r0 = t * kTileM, rmax = min(r0 + kTileM - 1, P.n - 1);
            int2 gwin = make_int2(0, 0);
            for (int gi = 0; ok && gi < ng; ++gi) {
                // first and last offsets of 32 groups at a time, broadcast by shuffle
                if ((gi & 31) == 0) {
                    const int4 w = gi + lane < ng ? __ldg(groups + gi + lane) : make_int4(INT_MAX, 0, 0, 0);
                    gwin = make_int2(w.x, w.y);
                }
                const int gx = __shfl_sync(0xffffffffu, gwin.x, gi & 31), gy = __shfl_sync(0xffffffffu, gwin.y, gi & 31);
                if (gx > rmax) break;  // groups ascend: no row of this tile reaches the rest
                const int a = max(0, r0 - gy), b = rmax - gx;
                const int nc = (b - a + kChunkKeys) / kChunkKeys;
                for (int j = 0; j < nc; ++j, ++c) {
                    const int s = c % kDiagStages;
                    const bool got = wait_bounded_sleep(empty_bar(s), ((c / kDiagStages) & 1) ^ 1, wc, wait_site(8, s, c));
                    if (!__all_sync(0xffffffffu, got)) {
                        ok = false;
                        break;
                    }
                    tma_load_kv_chunk_warp(ring + s * kChunkBytes, &P.tmap_k, &P.tmap_v, full_bar(s),
                                           a + j * kChunkKeys, g);
                    if (lane == 0) {
                        vmask[2 * s] = bits64_at(bv, P.n >> 5, a + j * kChunkKeys);
                        vmask[2 * s + 1] = bits64_at(bv, P.n >> 5, a + j * kChunkKeys + 64);
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(full_bar(s));
                }
            }
        }
        if (*abort_flag && lane == 0) {
            // drain: let the loads already issued land before the CTA exits
            volatile int no_abort = 0;
            const WaitCtl drain{&no_abort, nullptr, 50000000ull};
            for (int j = max(0, c - kDiagStages); j < c; ++j)
                wait_bounded(full_bar(j % kDiagStages), (j / kDiagStages) & 1, drain);
        }
        return;
    }

    // ---------------------------------------------------------------- consumers
    setmaxnreg_inc<kDiagRegsConsumer>();
    const int rw = (warp - 4) * 16;     // first row of this warp
    const int r = rw + (lane & 15);     // query row in the tile
    const int hf = lane >> 4;           // head-dimension half
    const float sl2 = P.scale_log2;
    const uint32_t kbase = ring + hf * 16384;  // this thread's K half of a stage; its V half is 32 KB further
    const uint32_t *vmask32 = reinterpret_cast<const uint32_t *>(vmask);
    int win_lo = -1, st_lo = 0;  // first chunk of the current window and its stage
    int c_base = 0;  // sequence number of the current group's first chunk
    int got = 0;     // chunks [0, got) seen full by this warp
    int rel = 0;     // chunks [0, rel) released by this warp
    bool ok = true;
    unsigned long long pairs = 0;
    auto see = [&]() -> bool {  // waits for chunk `got` to be full (warp-uniform)
        const int s = got % kDiagStages;
        const bool gfull = wait_bounded_sleep(full_bar(s), (got / kDiagStages) & 1, wc, wait_site(9, s, got));
        if (!__all_sync(0xffffffffu, gfull)) return false;
        ++got;
        return true;
    };
    auto release = [&]() {  // chunk `rel`, seen full and no longer needed
        __syncwarp();
        if (lane == 0) mbar_arrive(empty_bar(rel % kDiagStages));
        ++rel;
    };
    // From now on this warp needs chunks [lo, hi] (at most two; hi < lo at a group's
    // end).  Everything below lo is released first -- chunks not seen yet are seen
    // and released one by one -- so a warp never waits for a chunk while holding one
    // it no longer needs; the ring then always has room for the chunk awaited by
    // the warp that is furthest behind.
    auto need = [&](int lo, int hi) -> bool {
        while (rel < lo && rel < got) release();
        while (got < lo) {
            if (!see()) return false;
            release();
        }
        while (got <= hi)
            if (!see()) return false;
        return true;
    };
    for (int it = blockIdx.x; ok && it < n_items; it += gridDim.x) {
        const int t = P.n_qtiles - 1 - it / P.n_heads, hp = it % P.n_heads;
        const int ng = P.ngroups[hp];
        if (ng == 0) continue;  // the tile kernel reads no state for this head
        const int h = P.head_ids[hp];
        const int4 *groups = P.groups + (size_t)hp * P.gstride;
        const int *offs = P.offs + (size_t)hp * P.ostride;
        const int r0 = t * kTileM, rmax = min(r0 + kTileM - 1, P.n - 1);
        const int qi = r0 + r;
        const bool row_ok = qi <= rmax;
        const int last_r = rmax - r0;  // last valid row of the tile
        uint32_t qv[32];  // this thread's 64 query dims, bf16 pairs
        {
            const uint4 *src =
                reinterpret_cast<const uint4 *>(P.q + ((size_t)h * P.n + min(qi, P.n - 1)) * kD + hf * 64);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const uint4 x = row_ok ? __ldg(src + i) : make_uint4(0, 0, 0, 0);
                qv[4 * i] = x.x;
                qv[4 * i + 1] = x.y;
                qv[4 * i + 2] = x.z;
                qv[4 * i + 3] = x.w;
            }
        }
        float o[64];  // unnormalised O over this thread's 64 dims
#pragma unroll
        for (int e = 0; e < 64; ++e) o[e] = 0.f;
        float m = -INFINITY, l = 0.f;
        // group descriptors 32 at a time: lane l holds group gw + l, broadcast by shuffle,
        // so that no group waits on a load of its own descriptor
        int4 gwin = make_int4(0, 0, 0, 0);
        for (int gi = 0; ok && gi < ng; ++gi) {
            if ((gi & 31) == 0) gwin = gi + lane < ng ? __ldg(groups + gi + lane) : make_int4(INT_MAX, 0, 0, 0);
            int4 G;
            G.x = __shfl_sync(0xffffffffu, gwin.x, gi & 31);
            G.y = __shfl_sync(0xffffffffu, gwin.y, gi & 31);
            G.z = __shfl_sync(0xffffffffu, gwin.z, gi & 31);
            G.w = __shfl_sync(0xffffffffu, gwin.w, gi & 31);
            if (G.x > rmax) break;
            const int a = max(0, r0 - G.y), b = rmax - G.x;
            const int nc = (b - a + kChunkKeys) / kChunkKeys;
            // offsets of the group from the largest down (the key ranges move forward),
            // 32 at a time: lane l holds the l-th of the batch, broadcast by shuffle (a
            // lone offset is the descriptor's own first offset: nothing to load)
            for (int top = G.w - 1; ok && top >= 0; top -= 32) {
                const int cnt = min(32, top + 1);
                const int my_off = G.w == 1 ? G.x : (lane < cnt ? __ldg(offs + G.z + top - lane) : 0);
                for (int jj = 0; jj < cnt; ++jj) {
                    const int off = __shfl_sync(0xffffffffu, my_off, jj);
                    const int u0 = r0 - off - a;  // range position of row 0's key
                    const int ulo = max(0, u0 + rw), uhi = min(u0 + rw + 15, u0 + last_r);
                    if (ulo > uhi) continue;  // no valid row of this warp meets a key of this offset
                    const int clo = c_base + (ulo >> 7), chi = c_base + (uhi >> 7);
                    if (clo != win_lo || chi >= got) {  // the window moved: release below it, see it full
                        if (!need(clo, chi)) {
                            ok = false;
                            break;
                        }
                        win_lo = clo;
                        st_lo = clo % kDiagStages;
                    }
                    const int u = u0 + r;
                    const bool in = row_ok && u >= 0;
                    const int uc = max(u, 0);
                    // the row's chunk is the window's first or second (the 16 rows span at most two)
                    int st = st_lo + ((uc >> 7) - (ulo >> 7));
                    if (st >= kDiagStages) st -= kDiagStages;
                    const int ur = uc & 127;
                    // in the mask unless the key is a vertical (those are the tile kernel's)
                    const bool use = in && !((vmask32[4 * st + (ur >> 5)] >> (ur & 31)) & 1u);
                    // row ur of the stage; its 16-byte chunk i sits at chunk i ^ (ur & 7) (128B swizzle)
                    const uint32_t ka = kbase + (uint32_t)st * kChunkBytes + (uint32_t)ur * 128 + ((ur & 7) << 4);
                    float s;
                    // no branch on `use`: every lane computes, and a lane outside the mask
                    // adds P = 0.  Its address always lies in the ring: rows inside the tile read
                    // a chunk of the window (real, finite K and V); rows past the tile's end may
                    // read the stage after it, and their state is never stored.
                    {
                        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};  // eight chains of 8
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            const uint4 kk = lds128(ka ^ (i << 4));
                            dot2_bf16(kk.x, qv[4 * i], acc[0], acc[1]);
                            dot2_bf16(kk.y, qv[4 * i + 1], acc[2], acc[3]);
                            dot2_bf16(kk.z, qv[4 * i + 2], acc[4], acc[5]);
                            dot2_bf16(kk.w, qv[4 * i + 3], acc[6], acc[7]);
                        }
                        s = ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));
                    }
                    s += __shfl_xor_sync(0xffffffffu, s, 16);  // the two halves of the row's dot product
                    const float x = s * sl2;
                    // the running max moves only when it grows by more than 2^8; the rescale
                    // of O is a branch the whole warp takes or skips together
                    const bool grow = use && x > m + 8.0f;
                    if (__any_sync(0xffffffffu, grow)) {
                        const float alpha = grow ? ex2_approx(m - x) : 1.f;  // 0 while m = -inf
#pragma unroll
                        for (int e = 0; e < 64; ++e) o[e] *= alpha;
                        l *= alpha;
                        m = grow ? x : m;
                    }
                    {
                        const float p = use ? ex2_approx(x - m) : 0.f;
                        l += p;
                        const uint16_t pb = bf16_bits(p);  // P enters P V in bf16, as on the tensor cores
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            const uint4 vvi = lds128((ka + 32768) ^ (i << 4));
                            axpy2_bf16(vvi.x, pb, o[8 * i], o[8 * i + 1]);
                            axpy2_bf16(vvi.y, pb, o[8 * i + 2], o[8 * i + 3]);
                            axpy2_bf16(vvi.z, pb, o[8 * i + 4], o[8 * i + 5]);
                            axpy2_bf16(vvi.w, pb, o[8 * i + 6], o[8 * i + 7]);
                        }
                        pairs += use ? 1u : 0u;  // counted by both threads of the row, halved at the end
                    }
                }
            }
            if (!ok) break;
            // the group's remaining chunks: seen full, then released
            if (!need(c_base + nc, c_base + nc - 1)) {
                ok = false;
                break;
            }
            c_base += nc;
        }
        // the row's partial softmax state: (m, l) and the unnormalised O
        if (ok && row_ok) {
            const size_t row = (size_t)hp * P.n + qi;
            if (hf == 0) P.ml[row] = make_float2(m, l);
            if (l > 0.f) {
                float4 *dst = reinterpret_cast<float4 *>(P.o + row * kD + hf * 64);
#pragma unroll
                for (int i = 0; i < 16; ++i) dst[i] = make_float4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
            }
        }
    }
    if (P.hdr) {
#pragma unroll
        for (int sft = 16; sft > 0; sft >>= 1) pairs += __shfl_xor_sync(0xffffffffu, pairs, sft);
        pairs >>= 1;  // both threads of each row counted its pairs
        if (lane == 0 && pairs) {
            atomicAdd(&P.hdr->pairs, pairs);
            atomicAdd(&P.hdr->diag_pairs, pairs);
        }
    }
}

}  // namespace

cudaError_t run_vs_diag(const DiagParams &P, cudaStream_t st) {
    cudaError_t e = cudaFuncSetAttribute(vs_diag_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kDiagSmem);
    if (e != cudaSuccess) return e;
    // setmaxnreg.inc waits for registers the launch reserved: refuse to launch a
    // build whose register count at entry would make the split wait forever
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, vs_diag_kernel);
    if (e != cudaSuccess) return e;
    if (fa.numRegs < kDiagRegsLaunch) return cudaErrorInvalidConfiguration;
    int dev = 0, sms = 0;
    e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    // persistent: one CTA per SM, each striding over the work items heaviest first
    const int items = P.n_heads * P.n_qtiles;
    const int grid = std::min(items, std::max(1, sms));
    if (grid == 0) return cudaSuccess;
    ProfScope prof("vs_diag_kernel", st);
    vs_diag_kernel<<<grid, kDiagThreads, kDiagSmem, st>>>(P);
    return cudaGetLastError();
}

}  // namespace minf
