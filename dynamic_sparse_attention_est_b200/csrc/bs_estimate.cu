// bs_estimate.cu -- Block-Sparse index estimation on sm_100a.
//
// News article "单卡A100实现百万token推理，速度快10倍，这是微软官方的大模型推理加速",
// section 方法介绍: Q and K are mean-pooled and the pooled matrices multiplied;
// because mean pooling commutes with the product, the pooled score estimates the
// block-mean of the attention logits, and the best key blocks of each query
// block are kept.  Here:
//   pool    Qp[h][b] = mean of the 64 rows of block b (fp32 sums), Kp[g][b]
//           likewise, each stored as three bf16 parts hi + mid + lo that add up
//           to the fp32 mean within 2^-24 of it;
//   score   s_ij = Qp_i . Kp_j for j <= i on the tensor cores (tcgen05, fp32
//           accumulation in TMEM) as the six part products down to 2^-16 relative
//           size (split-bf16 products in the manner of Henry, Tang and Heinecke,
//           "Leveraging the bfloat16 artificial intelligence datatype for
//           higher-precision computations", 2019), smallest first;
//   top-k   diagonal block i always kept, the best topk-1 of j < i by radix
//           select (ties to the lower j), ascending.
#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"
#include "topk.cuh"

namespace minf {

namespace {

struct HeadList {
    int ids[MINF_MAX_HEADS];
};

struct ScoreParams {
    CUtensorMap tmap_q;  // pooled Q parts [n_heads * 3][nb][128] bf16 (slot hp, part p at z = 3 hp + p)
    CUtensorMap tmap_k;  // pooled K parts [hkv * 3][nb][128]
    HeadList hl;         // q-head of each slot
    float *scores;       // [hbn][nb][nb]
    WsHeader *hdr;
    unsigned long long wait_limit_ns;
    int group, nb, n_rt, hp0, hbn;
};

// One warp per 64-row block: lane l sums columns 4l..4l+3 in fp32, takes the
// mean and stores it as three bf16 parts.  out is [slot][3][nb][128] (part 0 hi,
// 1 mid, 2 lo).  With `listed`, slot s pools q-head hl.ids[s]; otherwise slot s
// pools head s.
__global__ void pool_split_kernel(const __nv_bfloat16 *x, const __grid_constant__ HeadList hl, bool listed,
                                  int n_rows_heads, int n, __nv_bfloat16 *out) {
    const int warp_global = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    const int nb = n / kBlock;
    if (warp_global >= n_rows_heads * nb) return;
    const int slot = warp_global / nb, b = warp_global % nb;
    const int head = listed ? hl.ids[slot] : slot;
    const __nv_bfloat16 *src = x + ((size_t)head * n + (size_t)b * kBlock) * kD + lane * 4;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int r = 0; r < kBlock; ++r) {
        const uint2 raw = *reinterpret_cast<const uint2 *>(src + (size_t)r * kD);
        const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162 *>(&raw.x);
        const __nv_bfloat162 c = *reinterpret_cast<const __nv_bfloat162 *>(&raw.y);
        acc[0] += __low2float(a);
        acc[1] += __high2float(a);
        acc[2] += __low2float(c);
        acc[3] += __high2float(c);
    }
    // x = hi + r1 exactly (r1 = x - hi is representable in fp32), r1 = mid + r2
    // likewise, lo = bf16(r2): |x - hi - mid - lo| <= 2^-24 |x|
    uint32_t part[3][2];
#pragma unroll
    for (int e = 0; e < 4; e += 2) {
        float x0 = acc[e] * (1.f / kBlock), x1 = acc[e + 1] * (1.f / kBlock);
#pragma unroll
        for (int p = 0; p < 3; ++p) {
            const __nv_bfloat162 v = __floats2bfloat162_rn(x0, x1);
            part[p][e >> 1] = *reinterpret_cast<const uint32_t *>(&v);
            x0 -= __low2float(v);
            x1 -= __high2float(v);
        }
    }
    const size_t plane = (size_t)nb * kD;
    __nv_bfloat16 *dst = out + (size_t)slot * 3 * plane + (size_t)b * kD + lane * 4;
#pragma unroll
    for (int p = 0; p < 3; ++p)
        *reinterpret_cast<uint2 *>(dst + p * plane) = make_uint2(part[p][0], part[p][1]);
}

// ---------------------------------------------------------------- pooled scores
// One CTA per (query row tile it, head): D(jt) = Qp[it] Kp[jt]^T for jt = 0..it,
// 128 x 128 each, accumulated in TMEM from the part products
//   hi.lo, mid.mid, hi.mid, lo.hi, mid.hi, hi.hi   (Q part . K part)
// in that order (K parts lo, mid, hi are streamed one 32 KB stage at a time).
// Dropped: mid.lo, lo.mid, lo.lo, each below 2^-24 of |Qp||Kp| per term.
// Warps: 0 TMA producer, 1 TMEM allocator + MMA issue (elect.sync picks the
// lane), 2..5 epilogue (TMEM lane quarter = warp % 4: row = quarter * 32 + lane).
// Two TMEM accumulators let tile jt's epilogue overlap tile jt + 1's products.
constexpr int kScThreads = 192;
constexpr int kScSlots = 4;                  // K part stages
constexpr uint32_t kScPart = 32768;          // 128 rows x 128 bf16
constexpr uint32_t kScA = 0;                 // Q parts hi, mid, lo
constexpr uint32_t kScB = 3 * kScPart;
constexpr uint32_t kScBar = kScB + kScSlots * kScPart;
constexpr uint32_t kScSmem = kScBar + 256 + 1024;
enum : int { SB_A = 0, SB_FULL = 1, SB_EMPTY = 5, SB_DFULL = 9, SB_DEMPTY = 11, SB_DONE = 13, SB_COUNT = 14 };
constexpr uint32_t kIdescScore = idesc_bf16_f32(128, false);

__global__ void __launch_bounds__(kScThreads, 1) pooled_scores_tc_kernel(const __grid_constant__ ScoreParams P) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kScBar);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(bars + SB_COUNT);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + SB_COUNT + 1);
    auto bar = [&](int i) { return smem_u32(bars + i); };
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // heaviest row tiles first, the batch's heads side by side
    const int it = P.n_rt - 1 - (int)blockIdx.x / P.hbn;
    const int hb = (int)blockIdx.x % P.hbn;
    const int hp = P.hp0 + hb;
    const int g = P.hl.ids[hp] / P.group;
    const int T = it + 1;

    if (threadIdx.x == 0) {
        mbar_init(bar(SB_A), 1);
        for (int s = 0; s < kScSlots; ++s) {
            mbar_init(bar(SB_FULL + s), 1);
            mbar_init(bar(SB_EMPTY + s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar(SB_DFULL + b), 1);
            mbar_init(bar(SB_DEMPTY + b), 128);
        }
        mbar_init(bar(SB_DONE), 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&P.tmap_q);
        tma_prefetch_desc(&P.tmap_k);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const WaitCtl wc{abort_flag, P.hdr ? &P.hdr->status : nullptr, P.wait_limit_ns};

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        const int r0 = it * 128;
        for (int p = 0; p < 3; ++p)
            tma_load_stage_warp(sbase + kScA + p * kScPart, &P.tmap_q, bar(SB_A), kScPart, r0, r0 + 64, hp * 3 + p,
                                3u);
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(SB_A));
        int issued = 0;
        for (int c = 0; c < 3 * T; ++c) {
            const int jt = c / 3, part = 2 - c % 3;  // K parts lo, mid, hi
            const int s = c % kScSlots;
            const bool got = wait_bounded(bar(SB_EMPTY + s), ((c / kScSlots) & 1) ^ 1, wc, wait_site(10, SB_EMPTY + s, c));
            if (__any_sync(0xffffffffu, !got)) break;
            tma_load_stage_warp(sbase + kScB + s * kScPart, &P.tmap_k, bar(SB_FULL + s), kScPart, jt * 128,
                                jt * 128 + 64, g * 3 + part, 3u);
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(SB_FULL + s));
            issued = c + 1;
        }
        if (lane == 0) {
            // the Q parts and the last stages must land before the CTA exits (abort path)
            volatile int no_abort = 0;
            const WaitCtl drain{&no_abort, nullptr, 50000000ull};
            if (*abort_flag) {
                wait_bounded(bar(SB_A), 0, drain);
                for (int c = max(0, issued - kScSlots); c < issued; ++c)
                    wait_bounded(bar(SB_FULL + c % kScSlots), (c / kScSlots) & 1, drain);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issue
        uint64_t da[3];
#pragma unroll
        for (int p = 0; p < 3; ++p) da[p] = sdesc_sw128(sbase + kScA + p * kScPart, 16, 1024);
        const uint64_t db0 = sdesc_sw128(sbase + kScB, 16, 1024);
        bool ok = __all_sync(0xffffffffu, wait_bounded(bar(SB_A), 0, wc, wait_site(11, SB_A, 0)));
        for (int jt = 0; ok && jt < T; ++jt) {
            const int b = jt & 1;
            ok = __all_sync(0xffffffffu,
                            wait_bounded(bar(SB_DEMPTY + b), ((jt >> 1) & 1) ^ 1, wc, wait_site(11, SB_DEMPTY + b, jt)));
            if (!ok) break;
            const uint32_t d = tmem + b * 128;
            for (int k = 0; k < 3; ++k) {  // K part lo, mid, hi
                const int c = 3 * jt + k, s = c % kScSlots;
                ok = __all_sync(0xffffffffu,
                                wait_bounded(bar(SB_FULL + s), (c / kScSlots) & 1, wc, wait_site(11, SB_FULL + s, c)));
                if (!ok) break;
                tc_fence_after();
                const uint64_t db = db0 + (uint64_t)((s * kScPart) >> 4);
                if (k == 0) {
                    umma_ss_tile_warp(d, da[0], db, kIdescScore, 0u);       // hi . lo
                } else if (k == 1) {
                    umma_ss_tile_warp(d, da[1], db, kIdescScore, 1u);       // mid . mid
                    umma_ss_tile_warp(d, da[0], db, kIdescScore, 1u);       // hi . mid
                } else {
                    umma_ss_tile_warp(d, da[2], db, kIdescScore, 1u);       // lo . hi
                    umma_ss_tile_warp(d, da[1], db, kIdescScore, 1u);       // mid . hi
                    umma_ss_tile_warp(d, da[0], db, kIdescScore, 1u);       // hi . hi
                }
                umma_commit_warp(bar(SB_EMPTY + s));
            }
            if (!ok) break;
            umma_commit_warp(bar(SB_DFULL + b));
        }
        // every product issued has completed before TMEM is freed
        umma_commit_warp(bar(SB_DONE));
        volatile int no_abort = 0;
        const WaitCtl drain{&no_abort, nullptr, 50000000ull};
        wait_bounded(bar(SB_DONE), 0, drain);
    } else {
        // ------------------------------------------------------------ epilogue
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;
        const int gi = it * 128 + r;
        float *srow = P.scores + ((size_t)hb * P.nb + (size_t)min(gi, P.nb - 1)) * P.nb;
        const bool vec = (P.nb & 3) == 0;
        for (int jt = 0; jt < T; ++jt) {
            const int b = jt & 1;
            const bool got = wait_bounded(bar(SB_DFULL + b), (jt >> 1) & 1, wc, wait_site(12, SB_DFULL + b, jt));
            if (__any_sync(0xffffffffu, !got)) break;  // the TMEM loads below are warp-wide
            tc_fence_after();
            uint32_t v[4][32];
            const uint32_t ta = tmem + ((uint32_t)(quarter * 32) << 16) + b * 128;
#pragma unroll
            for (int c = 0; c < 4; ++c) tmem_ld32(ta + c * 32, v[c]);
#pragma unroll
            for (int c = 0; c < 4; ++c) tmem_ld_wait(v[c]);
            tc_fence_before();
            mbar_arrive(bar(SB_DEMPTY + b));
            if (gi < P.nb) {
                const int j0 = jt * 128;
                if (vec && j0 + 128 <= P.nb) {
                    float4 *dst = reinterpret_cast<float4 *>(srow + j0);
#pragma unroll
                    for (int c = 0; c < 4; ++c)
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            dst[c * 8 + e] = make_float4(__uint_as_float(v[c][4 * e]), __uint_as_float(v[c][4 * e + 1]),
                                                         __uint_as_float(v[c][4 * e + 2]),
                                                         __uint_as_float(v[c][4 * e + 3]));
                } else {
#pragma unroll
                    for (int c = 0; c < 4; ++c)
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            if (j0 + c * 32 + e < P.nb) srow[j0 + c * 32 + e] = __uint_as_float(v[c][e]);
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, 256);
}

// ---------------------------------------------------------------- per-row top-k
// One warp per score row (query block i of one head): the diagonal block plus the
// best topk-1 blocks j < i.  Radix select over the order-preserving 32-bit keys,
// eight bits per pass with a 256-bin histogram in shared memory; the first pass
// (sign and exponent, where a row's keys crowd into a few bins) adds each group
// of equal bins once via match.any.  The passes stop as soon as the bin holding
// the k-th key is taken whole, since no tie inside it then needs splitting.  The
// final sweep takes the keys above the selected prefix and the first `rem` keys
// equal to it, in index order, so the output is ascending.
constexpr int kTopkWarps = 8;

__global__ void __launch_bounds__(kTopkWarps * 32) block_topk_warp_kernel(const float *scores, int nb, int topk,
                                                                          int hp0, int rows, int *blk_idx,
                                                                          int *blk_cnt) {
    __shared__ unsigned hist_all[kTopkWarps][256];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int row = (int)blockIdx.x * kTopkWarps + warp;
    if (row >= rows) return;  // whole warps only: no block-wide barrier below
    const int hb = row / nb, i = row % nb;
    const int hp = hp0 + hb;
    const float *src = scores + ((size_t)hb * nb + i) * nb;
    int *o = blk_idx + ((size_t)hp * nb + i) * topk;
    unsigned *hist = hist_all[warp];
    const unsigned lt = (1u << lane) - 1u;
    const int take = min(topk - 1, i);
    if (take == i) {
        for (int j = lane; j < i; j += 32) o[j] = j;
    } else if (take > 0) {
        uint32_t prefix = 0, pmask = 0;
        int rem = take;
#pragma unroll 1
        for (int pass = 0; pass < 4; ++pass) {
            const int shift = 24 - 8 * pass;
            for (int b = lane; b < 256; b += 32) hist[b] = 0u;
            __syncwarp();
#pragma unroll 4
            for (int j0 = 0; j0 < i; j0 += 32) {
                const int j = j0 + lane;
                const uint32_t u = j < i ? topk_key<true>(__ldg(src + j)) : 0u;
                const bool hit = j < i && (u & pmask) == prefix;
                const uint32_t bin = (u >> shift) & 255u;
                if (pass == 0) {
                    const unsigned peers = __match_any_sync(0xffffffffu, hit ? bin : 0xffffffffu);
                    if (hit && (peers & lt) == 0u) atomicAdd(&hist[bin], (unsigned)__popc(peers));
                } else if (hit) {
                    atomicAdd(&hist[bin], 1u);
                }
            }
            __syncwarp();
            // lane L owns bins 255-8L .. 248-8L; a scan from the top finds the bin
            // that holds the rem-th largest key among those matching the prefix
            int c[8], sum = 0;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                c[e] = (int)hist[255 - 8 * lane - e];
                sum += c[e];
            }
            int incl = sum;
#pragma unroll
            for (int s = 1; s < 32; s <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, incl, s);
                if (lane >= s) incl += y;
            }
            int cum = incl - sum;
            const bool mine = cum < rem && incl >= rem;
            int digit = 0, left = 0, in_bin = 0;
            if (mine) {
                int d = 255 - 8 * lane;
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    if (cum + c[e] >= rem) {
                        in_bin = c[e];
                        break;
                    }
                    cum += c[e];
                    --d;
                }
                digit = d;
                left = rem - cum;
            }
            const int who = __ffs(__ballot_sync(0xffffffffu, mine)) - 1;
            digit = __shfl_sync(0xffffffffu, digit, who);
            rem = __shfl_sync(0xffffffffu, left, who);
            in_bin = __shfl_sync(0xffffffffu, in_bin, who);
            prefix |= (uint32_t)digit << shift;
            pmask |= 255u << shift;
            __syncwarp();  // every lane has read the histogram before the next pass clears it
            if (in_bin == rem) break;
        }
        int base = 0, eq_seen = 0;
        for (int j0 = 0; j0 < i; j0 += 32) {
            const int j = j0 + lane;
            const uint32_t u = j < i ? (topk_key<true>(__ldg(src + j)) & pmask) : 0u;
            const bool gt = j < i && u > prefix;
            const bool eq = j < i && u == prefix;
            const unsigned eqm = __ballot_sync(0xffffffffu, eq);
            const bool tk = gt || (eq && eq_seen + __popc(eqm & lt) < rem);
            const unsigned tm = __ballot_sync(0xffffffffu, tk);
            if (tk) o[base + __popc(tm & lt)] = j;
            base += __popc(tm);
            eq_seen += __popc(eqm);
        }
    }
    if (lane == 0) {
        o[take] = i;
        blk_cnt[(size_t)hp * nb + i] = take + 1;
    }
    for (int j = take + 1 + lane; j < topk; j += 32) o[j] = -1;
}

}  // namespace

cudaError_t run_block_estimate(const BsEstArgs &a, const BsEstBufs &b, cudaStream_t st) {
    const int nb = a.n / kBlock;
    ScoreParams P;
    memset(&P, 0, sizeof(P));
    for (int i = 0; i < MINF_MAX_HEADS; ++i) P.hl.ids[i] = i < a.n_heads ? a.head_ids[i] : 0;
    P.group = a.hq / a.hkv;
    P.nb = nb;
    P.n_rt = (nb + 127) / 128;
    P.hdr = reinterpret_cast<WsHeader *>(a.hdr);
    P.wait_limit_ns = a.wait_limit_ns;
    cudaError_t e = make_tmap_3d(&P.tmap_q, b.qs, 3 * a.n_heads, nb);
    if (e == cudaSuccess) e = make_tmap_3d(&P.tmap_k, b.ks, 3 * a.hkv, nb);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(pooled_scores_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kScSmem);
    if (e != cudaSuccess) return e;
    {
        // pooled Q of the listed heads, pooled K of every kv-head
        ProfScope prof("bs_estimate: pool", st);
        const int warps = a.n_heads * nb;
        pool_split_kernel<<<(warps + 7) / 8, 256, 0, st>>>(reinterpret_cast<const __nv_bfloat16 *>(a.q), P.hl,
                                                           true, a.n_heads, a.n, b.qs);
        const int warps_k = a.hkv * nb;
        pool_split_kernel<<<(warps_k + 7) / 8, 256, 0, st>>>(reinterpret_cast<const __nv_bfloat16 *>(a.k), P.hl,
                                                             false, a.hkv, a.n, b.ks);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    // scores of every head straight into the caller's buffer, or a batch of heads
    // at a time through the workspace followed by the row selection
    const int batch = a.scores_out ? a.n_heads : b.head_batch;
    for (int hp0 = 0; hp0 < a.n_heads; hp0 += batch) {
        P.hp0 = hp0;
        P.hbn = min(batch, a.n_heads - hp0);
        P.scores = a.scores_out ? a.scores_out : b.scores;
        {
            ProfScope prof("bs_estimate: scores", st);
            pooled_scores_tc_kernel<<<P.n_rt * P.hbn, kScThreads, kScSmem, st>>>(P);
        }
        if (!a.scores_out) {
            ProfScope prof("bs_estimate: top-k", st);
            const int rows = P.hbn * nb;
            block_topk_warp_kernel<<<(rows + kTopkWarps - 1) / kTopkWarps, kTopkWarps * 32, 0, st>>>(
                b.scores, nb, a.topk, hp0, rows, a.blk_idx, a.blk_cnt);
        }
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace minf
