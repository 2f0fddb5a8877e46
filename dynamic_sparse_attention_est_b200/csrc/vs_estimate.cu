// vs_estimate.cu -- Vertical-Slash index estimation on sm_100a.
//
// News article "单卡A100实现百万token推理，速度快10倍，这是微软官方的大模型推理加速",
// section 方法介绍: the vertical and slash indices of a head are estimated from
// the attention of its last queries against all keys.  Here, per q-head:
//   pass 1  lse_i  = log-sum-exp over keys k <= i of scale * q_i . k_k, for the
//           last 64 rows i (split over key chunks, then combined);
//   pass 2  A_ik   = exp(scale * q_i . k_k - lse_i), summed along columns
//           (vertical score of key k) and along diagonals (slash score of the
//           offset o = i - k);
//   top-k   the best keys and offsets (radix select, ties to the lower index),
//           offset 0 forced.
// Both passes run S = Q K^T on the tensor cores: one CTA holds the last 64 rows
// of two q-heads of the same kv-head as one M=128 tile (TMEM lanes 0-63 and
// 64-127) and streams 128-key tiles of K through TMA.  Pass 2 writes each
// tile's softmax weights to a row-major shared-memory tile and sums it along
// columns and along diagonals (both read patterns are bank-conflict-free), so
// that the sums come out deterministic and without atomics.  The grid is one
// wave of one CTA per SM: head pairs x key chunks.
#include <cfloat>
#include <cstring>

#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace minf {

namespace {

constexpr int kThreads = 384;  // warp 0 TMA, warp 1 MMA, warps 4-11 compute
constexpr int kStages = 3;
constexpr uint32_t kTileBytes = 32768;
constexpr int kDiagW = 191;          // offsets one 128-key tile touches for 64 rows
// Row stride (floats) of the weight tile: rows start 16 bytes apart modulo the
// 32 banks, so a warp's 16-byte row stores take the minimum four wavefronts.
constexpr int kPStride = 132;
constexpr uint32_t kSmemQ = 0;
constexpr uint32_t kSmemK = kTileBytes;
constexpr uint32_t kSmemP = kSmemK + kStages * kTileBytes;  // 128 x kPStride floats
constexpr uint32_t kSmemBar = (kSmemP + 128 * kPStride * 4 + 255) & ~255u;
constexpr uint32_t kSmemBytes = kSmemBar + 256 + 1024;

enum : int { B_Q = 0, B_KF = 1, B_KE = 4, B_SF = 7, B_SE = 9, B_DONE = 11, B_COUNT = 12 };

constexpr uint32_t kIdescQK = idesc_bf16_f32(128, false);

struct EstParams {
    CUtensorMap tmap_q, tmap_k;
    int4 pairs[MINF_MAX_HEADS];  // (hp0, hp1, h0, h1); hp1 = -1 when the second half is empty
    int n_pairs, n, group, last_q, n_ktiles, chunk_tiles, n_chunks;
    float scale_log2;
    float2 *part;
    const float *lse2;
    float *vert, *diag;
    int *status;
    unsigned long long wait_limit_ns;
};

template <int MODE>  // 0: per-row (max, sum) partials; 1: column and diagonal sums
__global__ void __launch_bounds__(kThreads, 1) vs_est_kernel(const __grid_constant__ EstParams P) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sQ = smem_u32(smem) + kSmemQ, sK = smem_u32(smem) + kSmemK;
    float *ptile = reinterpret_cast<float *>(smem + kSmemP);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kSmemBar);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(bars + B_COUNT);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + B_COUNT + 1);
    auto bar = [&](int i) { return smem_u32(bars + i); };

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int pair = blockIdx.x % P.n_pairs, chunk = blockIdx.x / P.n_pairs;
    const int4 pr = P.pairs[pair];
    const int g = pr.z / P.group;
    const int kt0 = chunk * P.chunk_tiles;
    const int T = max(0, min(P.chunk_tiles, P.n_ktiles - kt0));

    if (threadIdx.x == 0) {
        mbar_init(bar(B_Q), 1);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(bar(B_KF + s), 1);
            mbar_init(bar(B_KE + s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar(B_SF + b), 1);
            mbar_init(bar(B_SE + b), 256);
        }
        mbar_init(bar(B_DONE), 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const WaitCtl wc{abort_flag, P.status, P.wait_limit_ns};

    if (warp == 0) {
        if (T > 0) {
            if (lane == 0) {
                const int q0 = P.n - 64;
                const int h1 = pr.y >= 0 ? pr.w : pr.z;
                mbar_expect_tx(bar(B_Q), 4 * 8192);
                tma_load_3d(sQ, &P.tmap_q, bar(B_Q), 0, q0, pr.z);
                tma_load_3d(sQ + 16384, &P.tmap_q, bar(B_Q), 64, q0, pr.z);
                tma_load_3d(sQ + 8192, &P.tmap_q, bar(B_Q), 0, q0, h1);
                tma_load_3d(sQ + 16384 + 8192, &P.tmap_q, bar(B_Q), 64, q0, h1);
                mbar_arrive(bar(B_Q));
            }
            // K tiles: the whole warp runs the loop (warp-uniform operands), one elected
            // lane issues each stage's loads
            int issued = 0;
            for (int j = 0; j < T; ++j) {
                const int s = j % kStages;
                const bool got = wait_bounded(bar(B_KE + s), ((j / kStages) & 1) ^ 1, wc, wait_site(5, B_KE + s, j));
                if (!__all_sync(0xffffffffu, got)) break;
                const int key0 = (kt0 + j) * 128;
                tma_load_stage_warp(sK + s * kTileBytes, &P.tmap_k, bar(B_KF + s), kTileBytes, key0, key0 + 64, g, 3u);
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(B_KF + s));
                issued = j + 1;
            }
            if (*abort_flag && lane == 0) {
                // drain: let the Q load and the K loads already issued land before the CTA exits
                volatile int no_abort = 0;
                const WaitCtl drain{&no_abort, nullptr, 50000000ull};
                wait_bounded(bar(B_Q), 0, drain);
                for (int j = max(0, issued - kStages); j < issued; ++j)
                    wait_bounded(bar(B_KF + j % kStages), (j / kStages) & 1, drain);
            }
        }
    } else if (warp == 1) {
        if (T > 0) {
            // the whole warp runs the issue loop; elect.sync picks the issuing lane
            const uint64_t dq = sdesc_sw128(sQ, 16, 1024), dk0 = sdesc_sw128(sK, 16, 1024);
            bool ok = __all_sync(0xffffffffu, wait_bounded(bar(B_Q), 0, wc, wait_site(6, B_Q, 0)));
            if (ok) tc_fence_after();
            for (int j = 0; ok && j < T; ++j) {
                const int s = j % kStages, b = j & 1;
                bool got = wait_bounded(bar(B_KF + s), (j / kStages) & 1, wc, wait_site(6, B_KF + s, j));
                if (!__all_sync(0xffffffffu, got)) break;
                got = wait_bounded(bar(B_SE + b), ((j >> 1) & 1) ^ 1, wc, wait_site(6, B_SE + b, j));
                if (!__all_sync(0xffffffffu, got)) break;
                tc_fence_after();
                umma_ss_tile_warp(tmem + b * 128, dq, dk0 + (uint64_t)((s * kTileBytes) >> 4), kIdescQK, 0u);
                umma_commit_warp(bar(B_KE + s));
                umma_commit_warp(bar(B_SF + b));
            }
            if (*abort_flag) {
                // the MMAs already issued complete before TMEM is freed
                umma_commit_warp(bar(B_DONE));
                volatile int no_abort = 0;
                const WaitCtl drain{&no_abort, nullptr, 50000000ull};
                wait_bounded(bar(B_DONE), 0, drain);
            }
        }
    } else if (warp >= 4) {
        // Eight compute warps: thread t holds columns [64 * half, 64 * half + 64) of
        // row r (TMEM lane r: rows 0-63 are the first head's last 64 queries,
        // rows 64-127 the second head's).
        const int t = threadIdx.x - 128;
        const int half = t >> 7, r = t & 127;
        const int rr = r & 63, hh = r >> 6;
        const int i = P.n - 64 + rr;  // query position of this row
        const bool head_ok = hh == 0 || pr.y >= 0;
        const bool row_ok = head_ok && rr >= 64 - P.last_q;
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        const float sl2 = P.scale_log2;
        float m_run = -INFINITY, l_run = 0.f;
        float lse2 = 0.f;
        if constexpr (MODE == 1) lse2 = row_ok ? P.lse2[pair * 128 + r] : 0.f;
        if (MODE == 1 && !(lse2 > -INFINITY)) lse2 = 0.f;
        for (int j = 0; j < T; ++j) {
            const int b = j & 1;
            const int kt = kt0 + j;
            const bool got = wait_bounded(bar(B_SF + b), (j >> 1) & 1, wc, wait_site(7, B_SF + b, j));
            // one decision for all compute threads: they meet at named barriers below
            if (named_bar_or(1, 256, !got || *abort_flag)) break;
            tc_fence_after();
            uint32_t sr[2][32];
#pragma unroll
            for (int c = 0; c < 2; ++c) tmem_ld32(tmem + lane_off + b * 128 + half * 64 + c * 32, sr[c]);
#pragma unroll
            for (int c = 0; c < 2; ++c) tmem_ld_wait(sr[c]);
            tc_fence_before();
            mbar_arrive(bar(B_SE + b));
            // causal limit: columns c <= cmax are keys <= i (every column of the tiles
            // below the last rows); rows outside the estimate take none
            const int cmax = (row_ok ? i - kt * 128 : -1) - half * 64;
            if (cmax < 63) {
#pragma unroll
                for (int c = 0; c < 2; ++c)
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        if (c * 32 + e > cmax) sr[c][e] = 0xff800000u;  // -inf
            }
            if constexpr (MODE == 0) {
                float mc[2];
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    mc[c] = fmaxf(__uint_as_float(sr[c][0]), __uint_as_float(sr[c][1]));
#pragma unroll
                    for (int e = 2; e < 32; e += 2)
                        mc[c] = fmax3(mc[c], __uint_as_float(sr[c][e]), __uint_as_float(sr[c][e + 1]));
                }
                const float m_new = fmaxf(m_run, fmaxf(mc[0], mc[1]) * sl2);
                if (m_new > -INFINITY) {
                    const uint64_t sl2x2 = f32x2_splat(sl2), negm = f32x2_splat(-m_new);
                    uint64_t acc[4] = {0, 0, 0, 0};
#pragma unroll
                    for (int c = 0; c < 2; ++c)
#pragma unroll
                        for (int e = 0; e < 16; ++e) {
                            float p0, p1;
                            f32x2_unpack(f32x2_fma(f32x2_pack(__uint_as_float(sr[c][2 * e]),
                                                              __uint_as_float(sr[c][2 * e + 1])),
                                                   sl2x2, negm),
                                         p0, p1);
                            acc[e & 3] = f32x2_add(acc[e & 3], f32x2_pack(ex2_approx(p0), ex2_approx(p1)));
                        }
                    float a[8];
#pragma unroll
                    for (int u = 0; u < 4; ++u) f32x2_unpack(acc[u], a[2 * u], a[2 * u + 1]);
                    const float tile_sum = ((a[0] + a[1]) + (a[2] + a[3])) + ((a[4] + a[5]) + (a[6] + a[7]));
                    l_run = l_run * ex2_approx(m_run - m_new) + tile_sum;
                    m_run = m_new;
                }
            } else {
                // normalised weights of this half row, then the whole tile in shared memory
                named_bar_sync(1, 256);  // the previous tile's readers are done
                float4 *dst = reinterpret_cast<float4 *>(ptile + r * kPStride + half * 64);
                const uint64_t sl2x2 = f32x2_splat(sl2), negl = f32x2_splat(-lse2);
#pragma unroll
                for (int c = 0; c < 2; ++c)
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        float w[4];
#pragma unroll
                        for (int h2 = 0; h2 < 2; ++h2) {
                            float x0, x1;
                            f32x2_unpack(f32x2_fma(f32x2_pack(__uint_as_float(sr[c][4 * e + 2 * h2]),
                                                              __uint_as_float(sr[c][4 * e + 2 * h2 + 1])),
                                                   sl2x2, negl),
                                         x0, x1);
                            w[2 * h2] = ex2_approx(x0);
                            w[2 * h2 + 1] = ex2_approx(x1);
                        }
                        dst[c * 8 + e] = make_float4(w[0], w[1], w[2], w[3]);
                    }
                named_bar_sync(1, 256);
                // column sums: thread t owns key column t & 127 of head t >> 7 (a warp
                // reads 32 consecutive floats of one row per step)
                {
                    const int h2 = t >> 7, c = t & 127;
                    const float *col = ptile + h2 * 64 * kPStride + c;
                    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll 16
                    for (int r2 = 0; r2 < 64; ++r2) acc[r2 & 7] += col[r2 * kPStride];
                    const int hp2 = h2 == 0 ? pr.x : pr.y;
                    const int key = kt * 128 + c;
                    if (hp2 >= 0 && key < P.n)
                        P.vert[(size_t)hp2 * P.n + key] =
                            ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));
                }
                // diagonal sums: task u = (head, x), x = row - column + 127 in [0, 191),
                // row rr in [x - 127, x] of that head; a warp takes 32 consecutive tasks,
                // so each row read is 32 consecutive floats
#pragma unroll 1
                for (int u = t; u < 2 * kDiagW; u += 256) {
                    const int h2 = u >= kDiagW ? 1 : 0, x = u - h2 * kDiagW;
                    const float *base = ptile + h2 * 64 * kPStride + 127 - x;
                    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll 16
                    for (int r2 = 0; r2 < 64; ++r2)
                        if (r2 <= x && r2 >= x - 127) acc[r2 & 7] += base[r2 * (kPStride + 1)];
                    const int hp2 = h2 == 0 ? pr.x : pr.y;
                    if (hp2 >= 0)
                        P.diag[((size_t)hp2 * P.n_ktiles + kt) * kDiagW + x] =
                            ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));
                }
            }
        }
        if constexpr (MODE == 0) {
            // merge the two column halves of each row (the weight tile is unused in this pass)
            float2 *xch = reinterpret_cast<float2 *>(ptile);
            if (half == 1) xch[r] = make_float2(m_run, l_run);
            named_bar_sync(1, 256);
            if (half == 0) {
                const float2 o = xch[r];
                const float m = fmaxf(m_run, o.x);
                const float l = m > -INFINITY ? l_run * ex2_approx(m_run - m) + o.y * ex2_approx(o.x - m) : 0.f;
                P.part[((size_t)pair * P.n_chunks + chunk) * 128 + r] = make_float2(m, l);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, 256);
}

// lse2[pair][row] = log2 sum over chunks of the partial (max, sum) pairs.
__global__ void lse_combine_kernel(const float2 *part, int n_pairs, int n_chunks, float *lse2) {
    const int x = blockIdx.x * blockDim.x + threadIdx.x;
    if (x >= n_pairs * 128) return;
    const int pair = x / 128, r = x % 128;
    float m = -INFINITY;
    for (int c = 0; c < n_chunks; ++c) m = fmaxf(m, part[((size_t)pair * n_chunks + c) * 128 + r].x);
    float l = 0.f;
    if (m > -INFINITY)
        for (int c = 0; c < n_chunks; ++c) {
            const float2 p = part[((size_t)pair * n_chunks + c) * 128 + r];
            if (p.x > -INFINITY) l += p.y * exp2f(p.x - m);
        }
    lse2[x] = l > 0.f ? m + log2f(l) : -INFINITY;
}

// slash[hp][o] = sum of the (at most two) key tiles' diagonal partials that
// cover offset o, in increasing tile order; offset 0 is forced to +inf.
__global__ void slash_combine_kernel(const float *diag, int n, int n_ktiles, float *slash, float *diag0) {
    const int hp = blockIdx.y;
    const int o = blockIdx.x * blockDim.x + threadIdx.x;
    if (o >= n) return;
    float s = 0.f;
    const int hi = min(n_ktiles - 1, (n - 1 - o) >> 7);  // last tile whose keys can sit o before a row
    for (int kt = max(0, hi - 2); kt <= hi; ++kt) {
        const int rel = o - (n - kDiagW - kt * 128);
        if (rel >= 0 && rel < kDiagW) s += diag[((size_t)hp * n_ktiles + kt) * kDiagW + rel];
    }
    slash[(size_t)hp * n + o] = o == 0 ? INFINITY : s;  // offset 0 is forced
    if (o == 0) diag0[hp] = s;                           // its mass, for top-p budgets
}

}  // namespace

cudaError_t run_vs_estimate(const VsEstArgs &a, const VsEstBufs &b, cudaStream_t st) {
    EstParams P;
    memset(&P, 0, sizeof(P));
    cudaError_t e = make_tmap_3d(&P.tmap_q, a.q, a.hq, a.n);
    if (e == cudaSuccess) e = make_tmap_3d(&P.tmap_k, a.k, a.hkv, a.n);
    if (e != cudaSuccess) return e;
    const int group = a.hq / a.hkv;
    // pair the listed heads that share a kv-head: M = 128 rows = 2 x 64 rows
    int np = 0;
    for (int g = 0; g < a.hkv; ++g) {
        int pending = -1;
        for (int hp = 0; hp < a.n_heads; ++hp) {
            const int h = a.head_ids[hp];
            if (h / group != g) continue;
            if (pending < 0) {
                pending = hp;
            } else {
                P.pairs[np++] = make_int4(pending, hp, a.head_ids[pending], h);
                pending = -1;
            }
        }
        if (pending >= 0) P.pairs[np++] = make_int4(pending, -1, a.head_ids[pending], a.head_ids[pending]);
    }
    P.n_pairs = np;
    P.n = a.n;
    P.group = group;
    P.last_q = a.last_q;
    P.n_ktiles = b.n_ktiles;
    P.chunk_tiles = b.chunk_tiles;
    P.n_chunks = b.n_chunks;
    P.scale_log2 = a.scale_log2;
    P.part = b.part;
    P.lse2 = b.lse2;
    P.vert = b.vert;
    P.diag = b.diag;
    P.status = a.hdr ? &reinterpret_cast<WsHeader *>(a.hdr)->status : nullptr;
    P.wait_limit_ns = a.wait_limit_ns;
    if (np == 0) return cudaSuccess;

    e = cudaFuncSetAttribute(vs_est_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(vs_est_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    const int grid = np * b.n_chunks;
    {
        ProfScope prof("vs_estimate (vs_est_kernel x2 + combines)", st);
        vs_est_kernel<0><<<grid, kThreads, kSmemBytes, st>>>(P);
        lse_combine_kernel<<<(np * 128 + 255) / 256, 256, 0, st>>>(b.part, np, b.n_chunks, b.lse2);
        vs_est_kernel<1><<<grid, kThreads, kSmemBytes, st>>>(P);
        dim3 sg((a.n + 255) / 256, a.n_heads);
        slash_combine_kernel<<<sg, 256, 0, st>>>(b.diag, a.n, b.n_ktiles, b.slash, b.diag0);
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    ProfScope prof("vs_topk", st);
    const int *kv = nullptr, *ks = nullptr;
    if (a.topp) {
        // top-p: per-row counts by mass, then the same ordered selection with those counts
        int *cv = a.v_cnt ? a.v_cnt : b.counts, *cs = a.s_cnt ? a.s_cnt : b.counts + a.n_heads;
        e = run_topp_counts2(b.vert, a.n_heads, false, nullptr, a.p_vertical, a.n_vertical, cv, b.slash, a.n_heads,
                             true, b.diag0, a.p_slash, a.n_slash, cs, a.n, b.topp_scratch, st);
        if (e != cudaSuccess) return e;
        kv = cv;
        ks = cs;
    }
    return run_topk_rows2(TopkRows{b.vert, a.n_heads, a.n_vertical, a.v_idx, kv},
                          TopkRows{b.slash, a.n_heads, a.n_slash, a.s_idx, ks}, a.n, b.topk_scratch, st);
}

}  // namespace minf
