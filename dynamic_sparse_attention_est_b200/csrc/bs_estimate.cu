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
//   top-k   diagonal block i always kept, the best topk-1 of j < i (ties to
//           the lower j), ascending: a histogram of value bins finds the
//           threshold bin, an exact selection settles it.
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
    CUtensorMap tmap_s;  // the scores [hbn][nb][nb] fp32, box {32, 32, 1}, 128B swizzle (when tma_store)
    HeadList hl;         // q-head of each slot
    float *scores;       // [hbn][nb][nb]
    WsHeader *hdr;
    unsigned long long wait_limit_ns;
    int group, nb, n_rt, hp0, hbn;
    int tma_store;       // 1: stores through shared memory by TMA; 0: plain per-row stores
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
// The epilogue writes each warp's 32 x 32 pieces into a swizzled shared-memory box
// (two per warp, alternating) and stores it with one TMA instruction, so that the
// scattered per-row stores do not throttle the load/store unit.
constexpr int kScThreads = 192;
constexpr int kScSlots = 3;                  // K part stages
constexpr uint32_t kScPart = 32768;          // 128 rows x 128 bf16
constexpr uint32_t kScA = 0;                 // Q parts hi, mid, lo
constexpr uint32_t kScB = 3 * kScPart;
constexpr uint32_t kScBox = 4096;            // 32 rows x 32 fp32
constexpr uint32_t kScStage = kScB + kScSlots * kScPart;  // 4 warps x 2 boxes
constexpr uint32_t kScBar = kScStage + 8 * kScBox;
constexpr uint32_t kScSmem = kScBar + 256 + 1024;
enum : int { SB_A = 0, SB_FULL = 1, SB_EMPTY = 5, SB_DFULL = 9, SB_DEMPTY = 11, SB_DONE = 13, SB_COUNT = 14 };
static_assert(kScSlots <= 4, "barrier slots");
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
        const uint32_t box0 = sbase + kScStage + (uint32_t)(warp - 2) * 2 * kScBox;
        int nbox = 0;  // boxes this warp has handed to TMA
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
            const int j0 = jt * 128;
            if (P.tma_store) {
#pragma unroll
                for (int c = 0; c < 4; ++c, ++nbox) {
                    const uint32_t box = box0 + (uint32_t)(nbox & 1) * kScBox;
                    // the store that used this box two boxes ago has read it
                    if (lane == 0) bulk_wait_read<1>();
                    __syncwarp();
                    // row `lane` of the box; its 16-byte chunk k sits at chunk k ^ (lane & 7)
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const uint32_t dst = box + (uint32_t)lane * 128 + ((uint32_t)(k ^ (lane & 7)) << 4);
                        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(v[c][4 * k]),
                                     "r"(v[c][4 * k + 1]), "r"(v[c][4 * k + 2]), "r"(v[c][4 * k + 3])
                                     : "memory");
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    // a box that starts past the last row or column holds nothing to write
                    const int bx = j0 + c * 32, by = it * 128 + quarter * 32;
                    if (lane == 0) {
                        if (bx < P.nb && by < P.nb) tma_store_3d(&P.tmap_s, box, bx, by, hb);
                        bulk_commit();  // one group per box, empty or not, so the wait above counts boxes
                    }
                }
            } else if (gi < P.nb) {
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
        // the boxes are read and the scores written before the CTA exits
        if (lane == 0) bulk_wait<0>();
        __syncwarp();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, 256);
}

// ---------------------------------------------------------------- per-row top-k
// One warp per score row (query block i of one head): the diagonal block plus the
// best topk-1 blocks j < i, ties to the lower j.  Two stages:
//  1. coarse: the row's scores fall into 256 bins linear in value between the
//     row's minimum and maximum (a monotone map: a higher bin means a higher
//     score); a scan from the top finds the bin b* that holds the k-th best, and
//     every score in a higher bin is taken;
//  2. exact, inside b*: up to 32 candidates are ranked against one another
//     (score descending, index ascending); more go through a radix select over
//     their order-preserving keys (eight bits per pass, starting below the bits
//     they all share, stopping once the digit holding the k-th is taken whole).
// Rows up to kRowSmem scores are copied once into the warp's shared-memory row by
// cp.async (the whole row in flight); longer rows are re-read (L1/L2) by every
// sweep.  After the histogram one sweep compacts the indices of bin b* and above
// into a list (candidates flagged) -- in place of a staged row, else in the
// histogram's words -- and the output is taken from the list.  Bins of more than
// 32 candidates (and, for long rows, budgets above 224) sweep the row again for
// the output.  -0 is read as +0, so that equal scores have equal keys.
constexpr int kTopkWarps = 8;
constexpr int kRowSmem = 2048;

struct DigitPick {
    int digit, left, in_bin;
};

// After a histogram pass: the bin holding the rem-th largest of the counted keys,
// the rank left inside it and its count.  Lane L owns bins 255-8L .. 248-8L.
__device__ __forceinline__ DigitPick pick_digit(const unsigned *hist, int rem, int lane) {
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
    DigitPick d{0, 0, 0};
    if (mine) {
        int dg = 255 - 8 * lane;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            if (cum + c[e] >= rem) {
                d.in_bin = c[e];
                break;
            }
            cum += c[e];
            --dg;
        }
        d.digit = dg;
        d.left = rem - cum;
    }
    const int who = __ffs(__ballot_sync(0xffffffffu, mine)) - 1;
    d.digit = __shfl_sync(0xffffffffu, d.digit, who);
    d.left = __shfl_sync(0xffffffffu, d.left, who);
    d.in_bin = __shfl_sync(0xffffffffu, d.in_bin, who);
    return d;
}

__device__ __forceinline__ float warp_min(float v) {
#pragma unroll
    for (int s = 16; s > 0; s >>= 1) v = fminf(v, __shfl_xor_sync(0xffffffffu, v, s));
    return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int s = 16; s > 0; s >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, s));
    return v;
}

// The row's scores in index order, 32 at a time (one per lane; lanes past the end
// get j >= i): fn(j, x) is called by every lane of the warp together.  `xs` is the
// row in shared memory (STAGED) or in global memory.
template <bool STAGED, class F>
__device__ __forceinline__ void row_sweep(const float *xs, int i, int lane, F &&fn) {
#pragma unroll 4
    for (int j0 = 0; j0 < i; j0 += 32) {
        const int j = j0 + lane;
        float x = 0.f;
        if (j < i) x = STAGED ? xs[j] : __ldg(xs + j) + 0.f;
        fn(j, x);
    }
}

template <bool STAGED>
__device__ __forceinline__ void select_row(const float *src, float *row, int i, int nb_of_row, int take, int *o,
                                           unsigned *hist, float2 *cand, int lane) {
    const unsigned lt = (1u << lane) - 1u;
    float xmin = INFINITY, xmax = -INFINITY;
    bool copied = false;
    if constexpr (STAGED) {
        // the whole row in flight at once: 16-byte cp.async per lane and chunk (the
        // row and the staging buffer are 16-byte aligned when nb % 4 == 0; the
        // rounded-up tail stays inside the row's nb scores and the buffer)
        if ((reinterpret_cast<uintptr_t>(src) & 15) == 0 && (reinterpret_cast<uintptr_t>(row) & 15) == 0 &&
            (nb_of_row & 3) == 0) {
            for (int c = lane; c < (i + 3) >> 2; c += 32) cp_async16(smem_u32(row + 4 * c), src + 4 * c);
            cp_async_wait_all();
            __syncwarp();
            copied = true;
        }
    }
#pragma unroll 4
    for (int j = lane; j < i; j += 32) {
        const float x = (copied ? row[j] : __ldg(src + j)) + 0.f;
        if constexpr (STAGED) row[j] = x;
        xmin = fminf(xmin, x);
        xmax = fmaxf(xmax, x);
    }
    const float *xs = STAGED ? row : src;
    __syncwarp();
    xmin = warp_min(xmin);
    xmax = warp_max(xmax);
    // ---- stage 1: 256 bins linear in value (all in bin 0 when the span is zero or too small to scale)
    float scale = 256.f / (xmax - xmin);
    if (!(scale < 3.0e38f)) scale = 0.f;
    auto bin_of = [&](float x) { return min(255, (int)((x - xmin) * scale)); };
    for (int b = lane; b < 256; b += 32) hist[b] = 0u;
    __syncwarp();
    row_sweep<STAGED>(xs, i, lane, [&](int j, float x) {
        if (j < i) atomicAdd(&hist[bin_of(x)], 1u);
    });
    __syncwarp();
    const DigitPick d = pick_digit(hist, take, lane);
    const int bstar = d.digit, rem = d.left, in_bin = d.in_bin;
    __syncwarp();  // the histogram is read before it is reused below
    const bool all_of_bin = rem == in_bin;
    const bool ranked = !all_of_bin && in_bin <= 32;
    // the list holds take - rem + in_bin <= take + 31 indices: staged rows keep it in
    // place of the row, the others in the (no longer needed) histogram's 256 words
    if ((all_of_bin || ranked) && (STAGED || take + 32 <= 256)) {
        // ---- one sweep: the indices of bin b* and above, compacted into the list (as
        // float bits; bit 31 flags a candidate of b*), candidates also to `cand`
        float *list = STAGED ? row : reinterpret_cast<float *>(hist);
        int base = 0, cbase = 0;
        row_sweep<STAGED>(xs, i, lane, [&](int j, float x) {
            const int b = j < i ? bin_of(x) : -1;
            const bool ge = b >= bstar, isc = b == bstar && !all_of_bin;
            const unsigned gm = __ballot_sync(0xffffffffu, ge), cm = __ballot_sync(0xffffffffu, isc);
            // staged: every lane has read its score before any lane writes (the ballots
            // above depend on all the reads), and positions written are <= this chunk's own
            if (ge) list[base + __popc(gm & lt)] = __int_as_float(j | (isc ? (int)0x80000000 : 0));
            if (isc) cand[cbase + __popc(cm & lt)] = make_float2(x, __int_as_float(j));
            base += __popc(gm);
            cbase += __popc(cm);
        });
        __syncwarp();
        unsigned sel = 0u;  // slot bits of the taken candidates
        if (ranked) {
            bool mine = false;
            if (lane < in_bin) {
                const float2 me = cand[lane];
                const int jm = __float_as_int(me.y);
                int rank = 0;
                for (int c = 0; c < in_bin; ++c) {
                    const float2 o2 = cand[c];
                    rank += (o2.x > me.x || (o2.x == me.x && __float_as_int(o2.y) < jm)) ? 1 : 0;
                }
                mine = rank < rem;
            }
            sel = __ballot_sync(0xffffffffu, mine);
        }
        // the output from the list (take - rem + in_bin entries, ascending)
        int obase = 0, cslot = 0;
        for (int e0 = 0; e0 < base; e0 += 32) {
            const int e = e0 + lane;
            const int v = e < base ? __float_as_int(list[e]) : 0;
            const bool isc = e < base && v < 0;
            const unsigned cm = __ballot_sync(0xffffffffu, isc);
            const bool tk = e < base && (!isc || ((sel >> (cslot + __popc(cm & lt))) & 1u));
            const unsigned tm = __ballot_sync(0xffffffffu, tk);
            if (tk) o[obase + __popc(tm & lt)] = v & 0x7fffffff;
            obase += __popc(tm);
            cslot += __popc(cm);
        }
        return;
    }
    // ---- stage 2 over the row again: which `rem` of the `in_bin` scores of bin b* are taken
    unsigned sel = 0u;               // candidates ranked: slot bits of the taken ones
    uint32_t prefix = 0u, pmask = 0u;  // radix: keys above prefix (under pmask) taken...
    int rem2 = 0;                    // ...and the first rem2 equal to it
    if (ranked) {
        int base = 0;
        row_sweep<STAGED>(xs, i, lane, [&](int j, float x) {
            const bool c = j < i && bin_of(x) == bstar;
            const unsigned m = __ballot_sync(0xffffffffu, c);
            if (c) cand[base + __popc(m & lt)] = make_float2(x, __int_as_float(j));
            base += __popc(m);
        });
        __syncwarp();
        bool mine = false;
        if (lane < in_bin) {
            const float2 me = cand[lane];
            const int jm = __float_as_int(me.y);
            int rank = 0;
            for (int c = 0; c < in_bin; ++c) {
                const float2 o2 = cand[c];
                rank += (o2.x > me.x || (o2.x == me.x && __float_as_int(o2.y) < jm)) ? 1 : 0;
            }
            mine = rank < rem;
        }
        sel = __ballot_sync(0xffffffffu, mine);
        __syncwarp();
    } else if (!all_of_bin) {
        uint32_t kmin = 0xffffffffu, kmax = 0u;
        row_sweep<STAGED>(xs, i, lane, [&](int j, float x) {
            if (j < i && bin_of(x) == bstar) {
                const uint32_t u = topk_key<true>(x);
                kmin = min(kmin, u);
                kmax = max(kmax, u);
            }
        });
        kmin = __reduce_min_sync(0xffffffffu, kmin);
        kmax = __reduce_max_sync(0xffffffffu, kmax);
        const uint32_t diff = kmin ^ kmax;
        int top = diff ? 31 - __clz((int)diff) : -1;
        pmask = top < 0 ? 0xffffffffu : (top == 31 ? 0u : ~((2u << top) - 1u));
        prefix = kmax & pmask;
        rem2 = rem;
        while (top >= 0) {
            const int w = min(8, top + 1), shift = top + 1 - w;
            const uint32_t dm = (1u << w) - 1u;
            for (int b = lane; b < 256; b += 32) hist[b] = 0u;
            __syncwarp();
            row_sweep<STAGED>(xs, i, lane, [&](int j, float x) {
                const uint32_t u = topk_key<true>(x);
                if (j < i && bin_of(x) == bstar && (u & pmask) == prefix) atomicAdd(&hist[(u >> shift) & dm], 1u);
            });
            __syncwarp();
            const DigitPick r = pick_digit(hist, rem2, lane);
            prefix |= (uint32_t)r.digit << shift;
            pmask |= dm << shift;
            rem2 = r.left;
            top -= w;
            __syncwarp();
            if (r.in_bin == rem2) break;
        }
    }
    // ---- the taken indices, ascending
    int base = 0, cslot = 0, eq_seen = 0;
    row_sweep<STAGED>(xs, i, lane, [&](int j, float x) {
        const int b = j < i ? bin_of(x) : -1;
        const bool inb = b == bstar;
        bool tk = b > bstar || (inb && all_of_bin);
        if (ranked) {
            const unsigned cm = __ballot_sync(0xffffffffu, inb);
            tk = tk || (inb && ((sel >> (cslot + __popc(cm & lt))) & 1u));
            cslot += __popc(cm);
        } else if (!all_of_bin) {
            const uint32_t u = topk_key<true>(x) & pmask;
            const bool eq = inb && u == prefix;
            const unsigned eqm = __ballot_sync(0xffffffffu, eq);
            tk = tk || (inb && u > prefix) || (eq && eq_seen + __popc(eqm & lt) < rem2);
            eq_seen += __popc(eqm);
        }
        const unsigned tm = __ballot_sync(0xffffffffu, tk);
        if (tk) o[base + __popc(tm & lt)] = j;
        base += __popc(tm);
    });
}

__global__ void __launch_bounds__(kTopkWarps * 32) block_topk_warp_kernel(const float *scores, int nb, int topk,
                                                                          int hp0, int rows, int *blk_idx,
                                                                          int *blk_cnt) {
    __shared__ unsigned hist_all[kTopkWarps][256];
    __shared__ float2 cand_all[kTopkWarps][32];
    extern __shared__ __align__(16) float row_all[];  // kTopkWarps rows of min(nb, kRowSmem) scores
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int row = (int)blockIdx.x * kTopkWarps + warp;
    if (row >= rows) return;  // whole warps only: no block-wide barrier below
    const int hb = row / nb, i = row % nb;
    const int hp = hp0 + hb;
    const float *src = scores + ((size_t)hb * nb + i) * nb;
    int *o = blk_idx + ((size_t)hp * nb + i) * topk;
    const int take = min(topk - 1, i);
    if (take == i) {
        for (int j = lane; j < i; j += 32) o[j] = j;
    } else if (take > 0) {
        // staged rows have i <= stride elements: i < nb when nb <= kRowSmem, else i <= kRowSmem
        const int stride = min(nb, kRowSmem);
        if (i <= kRowSmem)  // uniform over the warp
            select_row<true>(src, row_all + (size_t)warp * stride, i, nb, take, o, hist_all[warp], cand_all[warp],
                             lane);
        else
            select_row<false>(src, nullptr, i, nb, take, o, hist_all[warp], cand_all[warp], lane);
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
    // kTopkWarps staged rows of min(nb, kRowSmem) scores
    const int topk_smem = kTopkWarps * std::min(nb, kRowSmem) * (int)sizeof(float);
    e = cudaFuncSetAttribute(block_topk_warp_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, topk_smem);
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
        // TMA stores need 16-byte rows and a 16-byte aligned base; otherwise plain stores
        P.tma_store = (nb % 4 == 0 && (reinterpret_cast<uintptr_t>(P.scores) & 15) == 0 &&
                       make_tmap_f32_3d(&P.tmap_s, P.scores, nb, nb, P.hbn) == cudaSuccess)
                          ? 1
                          : 0;
        {
            ProfScope prof("bs_estimate: scores", st);
            pooled_scores_tc_kernel<<<P.n_rt * P.hbn, kScThreads, kScSmem, st>>>(P);
        }
        if (!a.scores_out) {
            ProfScope prof("bs_estimate: top-k", st);
            const int rows = P.hbn * nb;
            block_topk_warp_kernel<<<(rows + kTopkWarps - 1) / kTopkWarps, kTopkWarps * 32, topk_smem, st>>>(
                b.scores, nb, a.topk, hp0, rows, a.blk_idx, a.blk_cnt);
        }
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace minf
