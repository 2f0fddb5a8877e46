// attention.cu -- causal sparse FlashAttention on sm_100a (tcgen05 + TMEM + TMA).
//
// One CTA computes one work item: 128 query rows of one q-head against the key
// tiles its pattern selects.  A key tile is 128 keys made of two 64-key halves;
// each half is a contiguous key range loaded by TMA or a list of gathered keys
// (vertical lines), so every tile is one dense M=128, N=128 contraction on the
// tensor cores whatever the pattern (the index-shifting idea of the AICon talk
// "以 KV 缓存为中心的高效长文本方法": turn verticals and slashes into dense blocks;
// news article "单卡A100实现百万token推理…", Figure 4: slashes as dense blocks,
// verticals as 1x64 pieces).  The pattern's exact mask is applied per element
// inside each tile, so the result is the token-exact masked softmax.
//
// Warp roles (384 threads, one CTA per SM):
//   warp 0       TMA producer for Q and K (+ cp.async gathers of vertical keys)
//   warp 1       TMEM allocator; runs the tcgen05.mma issue loop (elect.sync picks the issuing lane)
//   warp 2       TMA producer for V (+ gathers)
//   warp 3       idle
//   warps 4..7   softmax warpgroup 0: even key tiles
//   warps 8..11  softmax warpgroup 1: odd key tiles
// Thread r of a softmax warpgroup owns query row r (TMEM lane r).  TMEM
// columns: S0 [0,128) S1 [128,256) O0 [256,384) O1 [384,512); each warpgroup
// keeps its own running max, sum and O over its half of the key tiles, and
// the two halves are merged in the epilogue.  S = Q K^T (SS MMA); P = exp(S-m)
// as bf16 overwrites the first 64 columns of its S buffer and feeds O += P V
// straight from TMEM (TS MMA).  The running max only moves when a row's max
// grows by more than 2^8.  A build-time share of the exponentials can run on
// the FMA pipe (polynomial) instead of the MUFU unit.
#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"
#include "topk.cuh"

namespace minf {

namespace {

constexpr int kThreads = 384;
constexpr int kStages = 3;                 // K ring and V ring depth
constexpr uint32_t kTileBytes = 32768;  // 128 rows x 128 bf16
constexpr uint32_t kSmemQ = 0;
constexpr uint32_t kSmemK = kSmemQ + kTileBytes;
constexpr uint32_t kSmemV = kSmemK + kStages * kTileBytes;
constexpr uint32_t kSmemBar = kSmemV + kStages * kTileBytes;
constexpr uint32_t kSmemBytes = kSmemBar + 256 + 1024;  // barriers + alignment slack
// Register split after setmaxnreg: the launch gives 384 threads x 168 registers;
// the load/MMA warpgroup drops to 56, the two softmax warpgroups rise to 224
// (128 x 56 + 256 x 224 = 384 x 168).
constexpr int kRegsLaunch = 168;
#ifndef MINF_REGS_LOAD
#define MINF_REGS_LOAD 56
#define MINF_REGS_SOFTMAX 224
#endif
constexpr int kRegsLoad = MINF_REGS_LOAD;
constexpr int kRegsSoftmax = MINF_REGS_SOFTMAX;
static_assert(128 * kRegsLoad + 256 * kRegsSoftmax <= kThreads * kRegsLaunch, "register split");
// Every kEmuEvery-th column pair takes its exponential from the FMA-pipe
// polynomial instead of MUFU ex2 (0 disables it).  Off by default: on B200 the
// softmax is issue-bound rather than MUFU-bound (measured: dense 32K 7.97 ms
// with 0, 8.41 ms with every 4th pair, 9.20 ms with every 2nd).
#ifndef MINF_EMU_EVERY
#define MINF_EMU_EVERY 0
#endif
constexpr int kEmuEvery = MINF_EMU_EVERY;

enum : int {
    B_Q_FULL = 0, B_K_FULL = 1, B_K_EMPTY = 4, B_V_FULL = 7, B_V_EMPTY = 10,
    B_S_FULL = 13, B_P_FULL = 15, B_ALL_DONE = 17, B_COUNT = 18
};

constexpr uint32_t kIdescQK = idesc_bf16_f32(128, false);
constexpr uint32_t kIdescPV = idesc_bf16_f32(128, true);

// ------------------------------------------------------------------ tile plans
// Every role walks the same deterministic sequence of half-tiles.
template <int PAT>
struct TileGen {
    int r0, rmax, total, emitted;
    // A-shape
    int sink_h, w_lo, split;
    // Block-Sparse
    const int *plan;
    // Vertical-Slash
    const int2 *groups;
    int2 gnext;     // groups[gi], loaded one group ahead
    int ng, gi, cur_a, cur_b, nsh, nvert, nle;

    __device__ void init(const AttnParams &P, int hp, int t) {
        r0 = t * kTileM;
        rmax = min(r0 + kTileM - 1, P.n - 1);
        emitted = 0;
        const int nb64 = P.n / kHalf;
        const int hi = min(2 * t + 1, nb64 - 1);
        if constexpr (PAT == PAT_DENSE) {
            total = hi + 1;
        } else if constexpr (PAT == PAT_ASHAPE) {
            sink_h = min((P.n_sink + kHalf - 1) / kHalf, nb64);
            w_lo = max(0, r0 - P.window + 1) / kHalf;
            // a tile holding dense tail rows (Tri-shape) needs every causal key
            split = w_lo > sink_h && rmax < P.n - P.n_last;
            total = split ? sink_h + (hi - w_lo + 1) : hi + 1;
        } else if constexpr (PAT == PAT_BLOCK) {
            const int w = hp * P.n_qtiles + t;
            plan = P.bs_plan + (size_t)w * P.bs_stride;
            total = P.bs_cnt[w];
        } else {
            const int w = hp * P.n_qtiles + t;
            groups = P.vs_groups + (size_t)hp * P.vs_gstride;
            ng = P.vs_ngroups[hp];
            gi = 0;
            gnext = ng > 0 ? __ldg(groups) : make_int2(0, 0);
            cur_a = 1;
            cur_b = 0;
            nsh = P.vs_nsh[w];
            nvert = P.vs_nvert[w];
            nle = P.vs_nle[w];
            total = nsh + (nvert + kHalf - 1) / kHalf;
        }
    }

    __device__ int tiles() const { return (total + 1) >> 1; }

    // Moves past two halves without describing them (the other softmax
    // warpgroup's tile): only Vertical-Slash keeps state beyond the count, and two
    // slash halves inside the current group just advance its cursor.
    __device__ void skip2(const AttnParams &P) {
        if constexpr (PAT == PAT_VS) {
            if (emitted + 2 <= nsh && cur_a + kHalf <= cur_b) {
                emitted += 2;
                cur_a += 2 * kHalf;
            } else {
                next(P);
                next(P);
            }
        } else {
            emitted += 2;
        }
    }

    __device__ HalfDesc next(const AttnParams &P) {
        HalfDesc h{HALF_EMPTY, 0, 0, 0};
        if (emitted >= total) {
            ++emitted;
            return h;
        }
        const int i = emitted++;
        if constexpr (PAT == PAT_DENSE) {
            h.kind = HALF_RANGE;
            h.ks = i * kHalf;
            h.len = kHalf;
            h.flags = HF_ROWS0 | HF_ROWS1 | (h.ks + kHalf - 1 <= r0 ? HF_FULL : 0);
        } else if constexpr (PAT == PAT_ASHAPE) {
            const int blk = (!split || i < sink_h) ? i : w_lo + (i - sink_h);
            h.kind = HALF_RANGE;
            h.ks = blk * kHalf;
            h.len = kHalf;
            const bool full = (h.ks + kHalf - 1 <= r0) &&
                              (h.ks + kHalf - 1 < P.n_sink || (r0 + kTileM - 1) - h.ks < P.window ||
                               r0 >= P.n - P.n_last);
            h.flags = HF_ROWS0 | HF_ROWS1 | (full ? HF_FULL : 0);
        } else if constexpr (PAT == PAT_BLOCK) {
            const int e = __ldg(plan + i);
            const int rows = e & 3;
            h.kind = HALF_RANGE;
            h.ks = (e >> 2) * kHalf;
            h.len = kHalf;
            h.flags = (rows << 1) | ((rows == 3 && h.ks + kHalf - 1 <= r0) ? HF_FULL : 0);
        } else {
            if (i < nsh) {
                if (cur_a > cur_b) {
                    while (gi < ng) {
                        const int2 g = gnext;
                        ++gi;
                        if (gi < ng) gnext = __ldg(groups + gi);  // in flight until the next group is needed
                        const int a = max(0, r0 - g.y);
                        const int b = min(r0 + kTileM - 1 - g.x, rmax);
                        if (b >= a) {
                            cur_a = a;
                            cur_b = b;
                            break;
                        }
                    }
                }
                if (cur_a <= cur_b) {
                    h.kind = HALF_RANGE;
                    h.ks = cur_a;
                    h.len = min(kHalf, cur_b - cur_a + 1);
                    // whole slash tiles: a full half below the tile's first row needs no mask
                    const bool full = P.vs_tiles && h.len == kHalf && h.ks + kHalf - 1 <= r0;
                    h.flags = HF_ROWS0 | HF_ROWS1 | (full ? HF_FULL : 0);
                    cur_a += kHalf;
                }
            } else {
                const int m = i - nsh;
                h.kind = HALF_GATHER;
                h.ks = m * kHalf;
                h.len = min(kHalf, nvert - m * kHalf);
                // every gathered key precedes the tile's first row: no element mask
                const bool full = h.len == kHalf && h.ks + kHalf <= nle;
                h.flags = HF_ROWS0 | HF_ROWS1 | (full ? HF_FULL : 0);
            }
        }
        return h;
    }
};

// Bitmap words a Vertical-Slash range half needs for one row.  They are loaded
// right after a softmax warpgroup hands over its P, while it waits for its next S.
struct MaskWords {
    uint32_t s[3], v[3];
};

template <int PAT>
__device__ __forceinline__ void mask_fetch(const AttnParams &P, const HalfDesc &h, int q,
                                           const uint32_t *bits_s, const uint32_t *bits_v,
                                           MaskWords &mw) {
    if constexpr (PAT == PAT_VS) {
        if (h.kind != HALF_RANGE || P.vs_tiles) return;
        // q - ks - 63 >= -190 (ks <= r0 + 127) and ks <= n - 1: the windows stay
        // within the guard words on either side of the bitmaps
        const uint32_t *ps = bits_s + ((q - h.ks - 63) >> 5), *pv = bits_v + (h.ks >> 5);
#pragma unroll
        for (int i = 0; i < 3; ++i) {
            mw.s[i] = __ldg(ps + i);
            mw.v[i] = __ldg(pv + i);
        }
    }
}

// Element mask of one half for query row q (= r0 + r): bit c set iff key c of
// the half is inside the pattern's mask for q.
template <int PAT>
__device__ __forceinline__ uint64_t half_mask(const AttnParams &P, const HalfDesc &h, int q, int r,
                                              const int *vlist, const MaskWords &mw) {
    if (h.kind == HALF_EMPTY) return 0ull;
    if (h.flags & HF_FULL) return ~0ull;
    const uint64_t causal = low_bits(q - h.ks + 1);
    if constexpr (PAT == PAT_DENSE) {
        return causal;
    } else if constexpr (PAT == PAT_ASHAPE) {
        const uint64_t sink = low_bits(P.n_sink - h.ks);
        const int c0 = q - h.ks - P.window + 1;  // first column inside the window
        const uint64_t win = c0 <= 0 ? ~0ull : (c0 >= 64 ? 0ull : (~0ull << c0));
        const uint64_t tail = q >= P.n - P.n_last ? ~0ull : 0ull;  // Tri-shape dense rows
        return causal & (sink | win | tail);
    } else if constexpr (PAT == PAT_BLOCK) {
        const int half_row = r >> 6;
        return (h.flags & (HF_ROWS0 << half_row)) ? causal : 0ull;
    } else {
        const uint64_t lenm = low_bits(h.len);
        if (h.kind == HALF_RANGE && P.vs_tiles) return causal & lenm;  // whole slash tiles
        if (h.kind == HALF_RANGE) {
            // slash: offset q - (ks + c) in S; vertical: key ks + c in V (words prefetched)
            const int ss = (q - h.ks - 63) & 31, sv = h.ks & 31;
            const uint64_t ws = (uint64_t)__funnelshift_r(mw.s[0], mw.s[1], ss) |
                                ((uint64_t)__funnelshift_r(mw.s[1], mw.s[2], ss) << 32);
            const uint64_t wv = (uint64_t)__funnelshift_r(mw.v[0], mw.v[1], sv) |
                                ((uint64_t)__funnelshift_r(mw.v[1], mw.v[2], sv) << 32);
            return causal & lenm & (__brevll(ws) | wv);
        }
        // gathered verticals, ascending: keep those <= q
        const int *lst = vlist + h.ks;
        int lo = 0, hi = h.len;  // first index with key > q
        while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (__ldg(lst + mid) <= q) lo = mid + 1;
            else hi = mid;
        }
        return low_bits(lo) & lenm;
    }
}

// Loads the two halves of one K or V tile into a 128-row, 128B-swizzled stage.
template <int PAT>
__device__ __forceinline__ void load_tile(uint32_t stage, uint32_t bar, const HalfDesc (&hd)[2],
                                          const CUtensorMap *map, const __nv_bfloat16 *raw,
                                          int g, int n, const int *vlist, int lane) {
    uint32_t tma_bytes = 0;
#pragma unroll
    for (int s = 0; s < 2; ++s)
        if (hd[s].kind != HALF_GATHER) tma_bytes += 2 * 8192;
    // the whole warp: warp-uniform operands, one elected lane adds the bytes and issues
    const uint32_t halves = (hd[0].kind != HALF_GATHER ? 1u : 0u) | (hd[1].kind != HALF_GATHER ? 2u : 0u);
    tma_load_stage_warp(stage, map, bar, tma_bytes, hd[0].kind == HALF_RANGE ? hd[0].ks : 0,
                        hd[1].kind == HALF_RANGE ? hd[1].ks : 0, g, halves);
    bool gathered = false;
#pragma unroll
    for (int s = 0; s < 2; ++s) {
        if (hd[s].kind != HALF_GATHER) continue;
        gathered = true;
        const int *lst = vlist + hd[s].ks;
        for (int rr = lane; rr < kHalf; rr += 32) {
            const int key = __ldg(lst + min(rr, hd[s].len - 1));
            const __nv_bfloat16 *src = raw + ((size_t)g * n + key) * kD;
            const int row = s * kHalf + rr;
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const uint32_t dst = stage + (u >> 3) * 16384 + row * 128 + (((u & 7) ^ (row & 7)) << 4);
                cp_async16(dst, src + u * 8);
            }
        }
    }
    if (gathered) {
        cp_async_wait_all();
        fence_proxy_async_smem();
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(bar);
}

// Exponential of a pair of arguments on the FMA pipe (Cody-Waite reduction for
// base 2: x = n + f with n = rint(x), f in [-1/2, 1/2]; 2^f from a degree-3
// minimax polynomial derived by csrc/exp2_poly.py, max relative error 7.5e-5;
// 2^n assembled in the exponent bits).  Arguments at or below -127 give 0.
__device__ __forceinline__ void exp2_poly_pair(float &a, float &b) {
    const uint64_t magic = f32x2_splat(12582912.0f);  // 1.5 * 2^23: rounds to an integer in the low bits
    uint64_t x = f32x2_pack(fmaxf(a, -127.f), fmaxf(b, -127.f));
    const uint64_t t = f32x2_add(x, magic);
    const uint64_t rn = f32x2_sub(t, magic);
    const uint64_t f = f32x2_sub(x, rn);
    uint64_t p = f32x2_fma(f, f32x2_splat(5.517166853e-02f), f32x2_splat(2.426111251e-01f));
    p = f32x2_fma(p, f, f32x2_splat(6.932609677e-01f));
    p = f32x2_fma(p, f, f32x2_splat(9.999280572e-01f));
    float t0, t1;
    f32x2_unpack(t, t0, t1);
    // bits(2^n) = (n + 127) << 23 = bits(t) * 2^23 + 0x3F800000 (mod 2^32): n = -127 gives +0
    const uint32_t s0 = __float_as_uint(t0) * (1u << 23) + 0x3F800000u;
    const uint32_t s1 = __float_as_uint(t1) * (1u << 23) + 0x3F800000u;
    p = f32x2_mul(p, f32x2_pack(__uint_as_float(s0), __uint_as_float(s1)));
    f32x2_unpack(p, a, b);
}

template <int PAT>
__global__ void __launch_bounds__(kThreads, 1) attn_kernel(const __grid_constant__ AttnParams P) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t sQ = sbase + kSmemQ, sK = sbase + kSmemK, sV = sbase + kSmemV;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kSmemBar);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(bars + B_COUNT);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + B_COUNT + 1);
    auto bar = [&](int i) { return smem_u32(bars + i); };

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // groups of heads one after the other; within a group the heaviest query tiles first,
    // its heads side by side
    int gi = 0;
    while (gi + 1 < P.n_kvgroups && (int)blockIdx.x >= P.kv_start[gi + 1] * P.n_qtiles) ++gi;
    const int gh = P.kv_start[gi + 1] - P.kv_start[gi];
    const int local = (int)blockIdx.x - P.kv_start[gi] * P.n_qtiles;
    const int t = P.n_qtiles - 1 - local / gh;
    const int hp = P.kv_order[P.kv_start[gi] + local % gh];
    const int h = P.head_ids[hp];
    const int g = h / P.group;
    const int w_item = hp * P.n_qtiles + t;

    if (threadIdx.x == 0) {
        mbar_init(bar(B_Q_FULL), 1);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(bar(B_K_FULL + s), 1);
            mbar_init(bar(B_K_EMPTY + s), 1);
            mbar_init(bar(B_V_FULL + s), 1);
            mbar_init(bar(B_V_EMPTY + s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar(B_S_FULL + b), 1);
            mbar_init(bar(B_P_FULL + b), 128);
        }
        mbar_init(bar(B_ALL_DONE), 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&P.tmap_q);
        tma_prefetch_desc(&P.tmap_k);
        tma_prefetch_desc(&P.tmap_v);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const WaitCtl wc{abort_flag, P.hdr ? &P.hdr->status : nullptr, P.wait_limit_ns};

    TileGen<PAT> gen;
    gen.init(P, hp, t);
    const int T = gen.tiles();
    const int *vlist = nullptr;
    if constexpr (PAT == PAT_VS) vlist = P.vs_vert + (size_t)w_item * P.vs_vstride;

    if (warp < 4) {
        // ---------------------------------------------------------- load / MMA warpgroup
        setmaxnreg_dec<kRegsLoad>();
        if (warp == 0 || warp == 2) {
            const bool is_k = warp == 0;
            const CUtensorMap *map = is_k ? &P.tmap_k : &P.tmap_v;
            const __nv_bfloat16 *raw = is_k ? P.k : P.v;
            const uint32_t stage0 = is_k ? sK : sV;
            const int full0 = is_k ? B_K_FULL : B_V_FULL, empty0 = is_k ? B_K_EMPTY : B_V_EMPTY;
            if (is_k && T > 0) {
                const int r0 = t * kTileM;
                tma_load_stage_warp(sQ, &P.tmap_q, bar(B_Q_FULL), 4 * 8192, r0, r0 + 64, h, 3u);
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(B_Q_FULL));
            }
            int issued = 0;
            for (int j = 0; j < T; ++j) {
                const int s = j % kStages;
                const uint32_t ph = (j / kStages) & 1;
                HalfDesc hd[2];
                hd[0] = gen.next(P);
                hd[1] = gen.next(P);
                // one decision per warp: every lane takes the same path through load_tile
                const bool got = wait_bounded(bar(empty0 + s), ph ^ 1, wc, wait_site(is_k ? 1 : 2, empty0 + s, j));
                if (__any_sync(0xffffffffu, !got)) break;
                load_tile<PAT>(stage0 + s * kTileBytes, bar(full0 + s), hd, map, raw, g, P.n, vlist, lane);
                issued = j + 1;
            }
            if (*abort_flag && lane == 0) {
                // drain: let the loads already issued land before the CTA exits
                volatile int no_abort = 0;
                const WaitCtl drain{&no_abort, nullptr, 50000000ull};
                for (int j = max(0, issued - kStages); j < issued; ++j)
                    wait_bounded(bar(full0 + j % kStages), (j / kStages) & 1, drain);
            }
        } else if (warp == 1 && T > 0) {
            // tcgen05 issue: S(j) = Q K(j)^T into S[j % 2]; O[j % 2] += P(j) V(j) with P(j)
            // read from the first 64 columns of S[j % 2]; S(j + 2) is issued after P(j) V(j)
            // and the tensor pipe runs them in order, so P(j) is consumed before it is overwritten.
            // The whole warp runs this loop (waits, counters and descriptors stay warp-uniform,
            // every decision is taken by the warp as one); elect.sync picks the lane that issues.
            // step-0 descriptors of Q, K stage 0 and V stage 0; a stage adds its offset / 16
            const uint64_t dq = sdesc_sw128(sQ, 16, 1024), dk0 = sdesc_sw128(sK, 16, 1024);
            const uint64_t dv0 = sdesc_sw128(sV, 16384, 1024);
            auto issue_s = [&](int j) -> bool {
                const int s = j % kStages;
                const bool got = wait_bounded(bar(B_K_FULL + s), (j / kStages) & 1, wc, wait_site(3, B_K_FULL + s, j));
                if (!__all_sync(0xffffffffu, got)) return false;
                tc_fence_after();
                umma_ss_tile_warp(tmem + (j & 1) * 128, dq, dk0 + (uint64_t)((s * kTileBytes) >> 4), kIdescQK, 0u);
                umma_commit_warp(bar(B_K_EMPTY + s));
                umma_commit_warp(bar(B_S_FULL + (j & 1)));
                return true;
            };
            bool ok = __all_sync(0xffffffffu, wait_bounded(bar(B_Q_FULL), 0, wc, wait_site(3, B_Q_FULL, 0)));
            if (ok) {
                tc_fence_after();
                ok = issue_s(0);
                if (ok && T > 1) ok = issue_s(1);
            }
            for (int j = 0; ok && j < T; ++j) {
                const int b = j & 1, s = j % kStages;
                bool got = wait_bounded(bar(B_P_FULL + b), (j >> 1) & 1, wc, wait_site(3, B_P_FULL + b, j));
                if (!__all_sync(0xffffffffu, got)) break;
                got = wait_bounded(bar(B_V_FULL + s), (j / kStages) & 1, wc, wait_site(3, B_V_FULL + s, j));
                if (!__all_sync(0xffffffffu, got)) break;
                tc_fence_after();
                umma_ts_tile_warp(tmem + 256 + b * 128, tmem + b * 128, dv0 + (uint64_t)((s * kTileBytes) >> 4),
                                  kIdescPV, j >= 2 ? 1u : 0u);
                umma_commit_warp(bar(B_V_EMPTY + s));
                if (j + 2 < T && !issue_s(j + 2)) break;
            }
            umma_commit_warp(bar(B_ALL_DONE));  // always close: the epilogue (or the abort path) waits on it
            if (P.hdr && lane == 0) {
                atomicAdd(&P.hdr->tiles, (unsigned long long)T);
                atomicAdd(&P.hdr->pat_tiles[PAT], (unsigned long long)T);
            }
        }
    } else {
        // ---------------------------------------------------------- softmax warpgroups
        setmaxnreg_inc<kRegsSoftmax>();
        const int wg = (warp - 4) >> 2;          // 0: even tiles, 1: odd tiles
        const int r = (threadIdx.x - 128) & 127; // query row = TMEM lane
        const int q = t * kTileM + r;
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        const uint32_t tS = tmem + lane_off + wg * 128;
        const uint32_t tO = tmem + lane_off + 256 + wg * 128;
        const float sl2 = P.scale_log2;
        const uint32_t *bits_s = nullptr, *bits_v = nullptr;
        if constexpr (PAT == PAT_VS) {
            bits_s = P.vs_bits_s + (size_t)hp * P.bit_stride;
            bits_v = P.vs_bits_v + (size_t)hp * P.bit_stride;
        }
        float m_run = -INFINITY, l_run = 0.f;
        unsigned long long pairs = 0;
        bool ok = true;
        if (wg == 1) gen.skip2(P);  // tile 0 belongs to the other warpgroup
        // element masks of this warpgroup's next tile: described, their bitmap words
        // loaded and combined while the warpgroup waits for that tile's S, so that
        // only the two 64-bit masks stay live through the softmax
        uint64_t mk0 = 0, mk1 = 0;
        bool full = false;
        auto prepare = [&]() {
            const HalfDesc d0 = gen.next(P), d1 = gen.next(P);
            MaskWords w0, w1;
            mask_fetch<PAT>(P, d0, q, bits_s, bits_v, w0);
            mask_fetch<PAT>(P, d1, q, bits_s, bits_v, w1);
            mk0 = half_mask<PAT>(P, d0, q, r, vlist, w0);
            mk1 = half_mask<PAT>(P, d1, q, r, vlist, w1);
            full = (d0.flags & d1.flags & HF_FULL) != 0;  // uniform over the CTA
        };
        prepare();
        for (int j = wg; j < T; j += 2) {
            if (q < P.n) pairs += __popcll(mk0) + __popcll(mk1);
            const bool got = wait_bounded(bar(B_S_FULL + wg), (j >> 1) & 1, wc, wait_site(4 + wg, B_S_FULL + wg, j));
            if (__any_sync(0xffffffffu, !got)) { ok = false; break; }  // tcgen05.ld below is warp-wide
            tc_fence_after();
            uint32_t sr[4][32];
#pragma unroll
            for (int c = 0; c < 4; ++c) tmem_ld32(tS + c * 32, sr[c]);
#pragma unroll
            for (int c = 0; c < 4; ++c) tmem_ld_wait(sr[c]);
            if (!full) {
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const uint32_t mw = (uint32_t)((c < 2 ? mk0 : mk1) >> ((c & 1) * 32));
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        if (!((mw >> e) & 1u)) sr[c][e] = 0xff800000u;  // -inf
                }
            }
            // row max over the 128 columns: four independent three-input max chains
            float mc[4];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                mc[c] = fmaxf(__uint_as_float(sr[c][0]), __uint_as_float(sr[c][1]));
#pragma unroll
                for (int e = 2; e < 32; e += 2)
                    mc[c] = fmax3(mc[c], __uint_as_float(sr[c][e]), __uint_as_float(sr[c][e + 1]));
            }
            float mx = fmax3(mc[0], mc[1], fmaxf(mc[2], mc[3]));
            mx *= sl2;
            const float m_new = fmaxf(m_run, mx);
            const bool want = m_new > m_run + 8.0f;  // includes m_run = -inf with a finite m_new
            const float alpha = want ? ex2_approx(m_run - m_new) : 1.f;  // 0 when m_run = -inf
            // O[wg] holds this warpgroup's tiles < j, all complete (S(j) was issued after their P.V):
            // rescale it in TMEM with the whole warp (lanes that keep their max use alpha = 1)
            if (j >= 2 && __any_sync(0xffffffffu, want && m_run != -INFINITY)) {
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint32_t o[32];
                    tmem_ld32(tO + c * 32, o);
                    tmem_ld_wait(o);
#pragma unroll
                    for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                    tmem_st32(tO + c * 32, o);
                }
            }
            if (want) {
                l_run *= alpha;
                m_run = m_new;
            }
            const float m_use = m_run == -INFINITY ? 0.f : m_run;
            const uint64_t sl2x2 = f32x2_splat(sl2), negm = f32x2_splat(-m_use);
            uint64_t acc0 = 0, acc1 = 0;  // two running (sum, sum) pairs
            uint32_t pp[2][32];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const uint64_t x = f32x2_fma(f32x2_pack(__uint_as_float(sr[c][2 * e]), __uint_as_float(sr[c][2 * e + 1])),
                                                 sl2x2, negm);
                    float p0, p1;
                    f32x2_unpack(x, p0, p1);
                    if (kEmuEvery > 0 && (e % kEmuEvery) == kEmuEvery - 1) {
                        exp2_poly_pair(p0, p1);
                    } else {
                        p0 = ex2_approx(p0);
                        p1 = ex2_approx(p1);
                    }
                    if (e & 1) acc1 = f32x2_add(acc1, f32x2_pack(p0, p1));
                    else acc0 = f32x2_add(acc0, f32x2_pack(p0, p1));
                    pp[c >> 1][(c & 1) * 16 + e] = pack_bf16x2(p0, p1);
                }
                if (c == 1) tmem_st32(tS, pp[0]);  // P(j) columns 0-31 of S[wg], stored while 32-63 are computed
            }
            float a0, a1, b0, b1;
            f32x2_unpack(acc0, a0, a1);
            f32x2_unpack(acc1, b0, b1);
            l_run += (a0 + a1) + (b0 + b1);
            tmem_st32(tS + 32, pp[1]);
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(bar(B_P_FULL + wg));
            gen.skip2(P);  // the other warpgroup's tile j + 1
            prepare();     // tile j + 2
        }
        // ------------------------------------------------------------ epilogue
        ok = __all_sync(0xffffffffu, ok);
        if (ok && T > 0) ok = wait_bounded(bar(B_ALL_DONE), 0, wc, wait_site(4 + wg, B_ALL_DONE, T));
        ok = __all_sync(0xffffffffu, ok);  // the TMEM loads below are warp-wide
        // exchange (max, sum) of the two halves of the key stream through shared memory
        // (the K stages are idle once every MMA has completed)
        float2 *ex = reinterpret_cast<float2 *>(smem + kSmemK);
        ex[wg * 128 + r] = make_float2(m_run, l_run);
        named_bar_sync(1, 256);
        if (ok) {
            tc_fence_after();
            const float2 s0 = ex[r], s1 = ex[128 + r];
            // a third partial state: the row's sparse-slash pairs, from the CUDA-core pass
            float2 s2 = make_float2(-INFINITY, 0.f);
            if constexpr (PAT == PAT_VS) {
                if (P.vs_diag_ml && q < P.n && P.vs_ndgroups[hp] > 0) s2 = P.vs_diag_ml[(size_t)hp * P.n + q];
            }
            const bool has2 = s2.y > 0.f;
            const float m = fmaxf(fmaxf(s0.x, s1.x), has2 ? s2.x : -INFINITY);
            const float a0 = s0.x == -INFINITY ? 0.f : ex2_approx(s0.x - m);
            const float a1 = (T < 2 || s1.x == -INFINITY) ? 0.f : ex2_approx(s1.x - m);
            const float a2 = has2 ? ex2_approx(s2.x - m) : 0.f;
            const float l = s0.y * a0 + s1.y * a1 + s2.y * a2;
            const float inv_l = l > 0.f ? 1.f / l : 0.f;
            const float w0 = a0 * inv_l, w1 = a1 * inv_l, w2 = a2 * inv_l;
            const float4 *o2 = has2 ? reinterpret_cast<const float4 *>(P.vs_diag_o + ((size_t)hp * P.n + q) * kD + wg * 64)
                                    : nullptr;
            const size_t orow = (size_t)P.out_slot[hp] * P.n + min(q, P.n - 1);
            uint4 *dst = reinterpret_cast<uint4 *>(P.out + orow * kD + wg * 64);
            const uint32_t tO0 = tmem + lane_off + 256 + wg * 64, tO1 = tmem + lane_off + 384 + wg * 64;
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                uint32_t o0[32], o1[32];
                if (T > 0) {  // uniform over the CTA
                    tmem_ld32(tO0 + c * 32, o0);
                    tmem_ld_wait(o0);
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e) o0[e] = 0u;
                }
                if (T > 1) {
                    tmem_ld32(tO1 + c * 32, o1);
                    tmem_ld_wait(o1);
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e) o1[e] = 0u;
                }
                if (q < P.n) {
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        o0[e] = __float_as_uint(__uint_as_float(o0[e]) * w0 + __uint_as_float(o1[e]) * w1);
                    if (o2) {
#pragma unroll
                        for (int i = 0; i < 8; ++i) {  // columns 32 c + 4 i .. + 3 of this warpgroup's 64
                            const float4 x = __ldg(o2 + c * 8 + i);
                            o0[4 * i] = __float_as_uint(fmaf(x.x, w2, __uint_as_float(o0[4 * i])));
                            o0[4 * i + 1] = __float_as_uint(fmaf(x.y, w2, __uint_as_float(o0[4 * i + 1])));
                            o0[4 * i + 2] = __float_as_uint(fmaf(x.z, w2, __uint_as_float(o0[4 * i + 2])));
                            o0[4 * i + 3] = __float_as_uint(fmaf(x.w, w2, __uint_as_float(o0[4 * i + 3])));
                        }
                    }
                    uint32_t pk[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        pk[e] = pack_bf16x2(__uint_as_float(o0[2 * e]), __uint_as_float(o0[2 * e + 1]));
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        dst[c * 4 + e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
                }
            }
            if (wg == 0 && q < P.n && P.lse)
                P.lse[orow] = l > 0.f ? (m + __log2f(l)) * 0.69314718055994531f : -INFINITY;
        }
        if (P.hdr) {
#pragma unroll
            for (int s = 16; s > 0; s >>= 1) pairs += __shfl_xor_sync(0xffffffffu, pairs, s);
            if (lane == 0) atomicAdd(&P.hdr->pairs, pairs);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, 512);
}

// ------------------------------------------------------------------ planners
// Block-Sparse: per work item (two 64-row query blocks), merge the two
// ascending block lists into one list of half entries (block << 2 | rows).
__global__ void bs_plan_kernel(const int *blk_idx, const int *blk_cnt, int topk, int n_heads,
                               int n_qtiles, int nb, int *plan, int *cnt, int stride) {
    const int w = blockIdx.x * blockDim.x + threadIdx.x;
    if (w >= n_heads * n_qtiles) return;
    const int hp = w / n_qtiles, t = w % n_qtiles;
    const int b0 = 2 * t, b1 = 2 * t + 1;
    const int *l0 = blk_idx + ((size_t)hp * nb + b0) * topk;
    const int *l1 = b1 < nb ? blk_idx + ((size_t)hp * nb + b1) * topk : nullptr;
    const int c0 = min(max(blk_cnt[(size_t)hp * nb + b0], 0), topk);
    const int c1 = l1 ? min(max(blk_cnt[(size_t)hp * nb + b1], 0), topk) : 0;
    int i0 = 0, i1 = 0, last0 = -1, last1 = -1, out = 0;
    int *dst = plan + (size_t)w * stride;
    // entries that are negative, in the future of their block, or not above the
    // previous entry of their list are skipped
    auto next0 = [&]() -> int {
        while (i0 < c0) {
            const int j = l0[i0];
            if (j > last0 && j >= 0 && j <= b0) return j;
            ++i0;
        }
        return INT_MAX;
    };
    auto next1 = [&]() -> int {
        while (i1 < c1) {
            const int j = l1[i1];
            if (j > last1 && j >= 0 && j <= b1) return j;
            ++i1;
        }
        return INT_MAX;
    };
    for (;;) {
        const int j0 = next0(), j1 = next1();
        if (j0 == INT_MAX && j1 == INT_MAX) break;
        const int j = min(j0, j1);
        int rows = 0;
        if (j0 == j) { rows |= 1; last0 = j; ++i0; }
        if (j1 == j) { rows |= 2; last1 = j; ++i1; }
        dst[out++] = (j << 2) | rows;
    }
    cnt[w] = out;
}

// Vertical-Slash: mark the index rows into per-head bitmaps (order-free,
// duplicates merge, out-of-range entries ignored).
__global__ void vs_mark_kernel(const int *v_idx, int n_vertical, const int *s_idx, int n_slash, int n,
                               uint32_t *bits_v, uint32_t *bits_s, int stride) {
    const int hp = blockIdx.x;
    for (int i = threadIdx.x; i < n_vertical; i += blockDim.x) {
        const int x = v_idx[(size_t)hp * n_vertical + i];
        if (x >= 0 && x < n) atomicOr(bits_v + (size_t)hp * stride + (x >> 5), 1u << (x & 31));
    }
    for (int i = threadIdx.x; i < n_slash; i += blockDim.x) {
        const int x = s_idx[(size_t)hp * n_slash + i];
        if (x >= 0 && x < n) atomicOr(bits_s + (size_t)hp * stride + (x >> 5), 1u << (x & 31));
    }
}

// Ordered extraction of the set bits of a bitmap by the NT threads of a block:
// each thread takes 8 consecutive words per sweep and a block scan gives its
// output position.
constexpr int kExtractThreads = 1024;

template <int NT>
__device__ int block_extract_bits(const uint32_t *bm, int words, int *out, int cap, TopkShared &sh) {
    int base = 0;
    for (int w0 = 0; w0 < words; w0 += NT * 8) {
        const int wb = w0 + (int)threadIdx.x * 8;
        uint32_t wd[8];
        int c = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            wd[e] = (wb + e < words) ? bm[wb + e] : 0u;
            c += __popc(wd[e]);
        }
        int tot;
        int pos = base + block_excl_scan<NT>(c, &tot, sh);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            uint32_t word = wd[e];
            while (word) {
                const int b = __ffs(word) - 1;
                if (pos < cap) out[pos] = (wb + e) * 32 + b;
                ++pos;
                word &= word - 1;
            }
        }
        base += tot;
    }
    return min(base, cap);
}

// Per head: sorted distinct verticals, and slash offsets merged into groups
// whose 128-row key ranges touch (consecutive offsets at most 128 apart).  A
// group starts at an offset more than 128 past its predecessor and ends at
// one more than 128 short of its successor; the j-th start and the j-th end
// bound group j.  Each group then goes to one of two paths: the tile kernel
// (dense 128x128 tiles over the group's key range, masked per element) or the
// CUDA-core pass (one pair per row and offset), whichever computes it for less:
// a tile half costs about `diag_ratio` offsets of the CUDA-core pass, so a
// group of m offsets whose range needs H halves goes there when
// m < diag_ratio * H (0 sends every group to the tile kernel).  The offsets of
// those groups are cleared from the slash bitmap, which from then on masks the
// tile kernel's ranges.
__global__ void __launch_bounds__(kExtractThreads) vs_extract_kernel(const uint32_t *bits_v, uint32_t *bits_s,
                                                                     int words, int stride, int *vsorted, int *nvs,
                                                                     int vcap, int *soff, int scap, int2 *groups,
                                                                     int *ngroups, int4 *dgroups, int *ndgroups,
                                                                     float diag_ratio) {
    __shared__ TopkShared sh;
    const int hp = blockIdx.x;
    const int cv = block_extract_bits<kExtractThreads>(bits_v + (size_t)hp * stride, words,
                                                       vsorted + (size_t)hp * vcap, vcap, sh);
    const int cs = block_extract_bits<kExtractThreads>(bits_s + (size_t)hp * stride, words,
                                                       soff + (size_t)hp * scap, scap, sh);
    __syncthreads();  // the offsets written above are read by other threads below
    const int *so = soff + (size_t)hp * scap;
    int4 *all = dgroups + (size_t)hp * scap;  // every group: (first offset, last offset, first index, last index)
    int n_start = 0, n_end = 0;
    for (int e0 = 0; e0 < cs; e0 += kExtractThreads) {
        const int e = e0 + (int)threadIdx.x;
        int start = 0, end = 0, x = 0;
        if (e < cs) {
            x = so[e];
            start = (e == 0) || (x - so[e - 1] > kTileM);
            end = (e == cs - 1) || (so[e + 1] - x > kTileM);
        }
        int tot;
        const int packed = block_excl_scan<kExtractThreads>(start | (end << 16), &tot, sh);
        if (start) {
            all[n_start + (packed & 0xffff)].x = x;
            all[n_start + (packed & 0xffff)].z = e;
        }
        if (end) {
            all[n_end + (packed >> 16)].y = x;
            all[n_end + (packed >> 16)].w = e;
        }
        n_start += tot & 0xffff;
        n_end += tot >> 16;
    }
    __syncthreads();  // every group's four fields are written
    int2 *tg = groups + (size_t)hp * scap;
    uint32_t *bs = bits_s + (size_t)hp * stride;
    int n_tile = 0, n_diag = 0;
    for (int i0 = 0; i0 < n_start; i0 += kExtractThreads) {
        const int i = i0 + (int)threadIdx.x;
        int4 gd = make_int4(0, 0, 0, 0);
        int to_tile = 0, to_diag = 0;
        if (i < n_start) {
            gd = all[i];
            const int m = gd.w - gd.z + 1;
            const int halves = (gd.y - gd.x + kTileM + kHalf - 1) / kHalf;
            to_diag = diag_ratio > 0.f && (float)m < diag_ratio * (float)halves;
            to_tile = !to_diag;
        }
        int tot;
        // every read of this sweep happens before the scan's barriers, and the
        // CUDA-core groups are compacted in place towards lower indices
        const int packed = block_excl_scan<kExtractThreads>(to_tile | (to_diag << 16), &tot, sh);
        if (to_tile) tg[n_tile + (packed & 0xffff)] = make_int2(gd.x, gd.y);
        if (to_diag) {
            all[n_diag + (packed >> 16)] = make_int4(gd.x, gd.y, gd.z, gd.w - gd.z + 1);
            for (int j = gd.z; j <= gd.w; ++j) {
                const int x = so[j];
                atomicAnd(bs + (x >> 5), ~(1u << (x & 31)));
            }
        }
        n_tile += tot & 0xffff;
        n_diag += tot >> 16;
    }
    if (threadIdx.x == 0) {
        nvs[hp] = cv;
        ngroups[hp] = n_tile;
        ndgroups[hp] = n_diag;
    }
}

__device__ __forceinline__ bool any_bits(const uint32_t *bm, int lo, int hi) {
    for (int w = lo >> 5; w <= (hi >> 5); ++w) {
        uint32_t m = 0xffffffffu;
        if (w == (lo >> 5)) m &= 0xffffffffu << (lo & 31);
        if (w == (hi >> 5)) m &= 0xffffffffu >> (31 - (hi & 31));
        if (bm[w] & m) return true;
    }
    return false;
}

// Per work item (one warp): number of slash half-tiles, the ascending list of
// vertical keys that no slash range of this 128-row tile covers, and how many
// of those precede the tile's first row (their halves need no element mask).
__global__ void vs_workitem_kernel(const int *vsorted, const int *nvs, int vcap, const int2 *groups,
                                   const int *ngroups, int gstride, const uint32_t *bits_s, int stride, int n,
                                   int n_heads, int n_qtiles, int *nsh, int *nvert, int *nle, int *vlist) {
    const int w = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (w >= n_heads * n_qtiles) return;
    const int hp = w / n_qtiles, t = w % n_qtiles;
    const int r0 = t * kTileM, rmax = min(r0 + kTileM - 1, n - 1);
    const int2 *gr = groups + (size_t)hp * gstride;
    const int ng = ngroups[hp];
    int halves = 0;
    for (int i = lane; i < ng; i += 32) {
        const int2 gg = gr[i];
        const int a = max(0, r0 - gg.y), b = min(r0 + kTileM - 1 - gg.x, rmax);
        if (b >= a) halves += (b - a + kHalf) / kHalf;
    }
#pragma unroll
    for (int s = 16; s > 0; s >>= 1) halves += __shfl_xor_sync(0xffffffffu, halves, s);
    const int *vs = vsorted + (size_t)hp * vcap;
    const uint32_t *bs = bits_s + (size_t)hp * stride;
    int *dst = vlist + (size_t)w * vcap;
    const int cv = nvs[hp];
    int out = 0, le = 0;
    for (int e0 = 0; e0 < cv; e0 += 32) {
        const int e = e0 + lane;
        bool keep = false;
        if (e < cv) {
            const int x = vs[e];
            if (x <= rmax) {
                const int lo = max(0, r0 - x), hi = min(r0 + kTileM - 1 - x, n - 1);
                keep = !any_bits(bs, lo, hi);
            }
        }
        const uint32_t bal = __ballot_sync(0xffffffffu, keep);
        if (keep) dst[out + __popc(bal & ((1u << lane) - 1u))] = vs[e];
        out += __popc(bal);
        le += __popc(__ballot_sync(0xffffffffu, keep && vs[e] <= r0));
    }
    if (lane == 0) {
        nsh[w] = halves;
        nvert[w] = out;
        nle[w] = le;
    }
}

template <int PAT>
cudaError_t launch_attn(const AttnParams &P, cudaStream_t st) {
    cudaError_t e = cudaFuncSetAttribute(attn_kernel<PAT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    // setmaxnreg.inc waits for registers the launch reserved: refuse to launch a
    // build whose register count at entry would make the split wait forever
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, attn_kernel<PAT>);
    if (e != cudaSuccess) return e;
    if (fa.numRegs < kRegsLaunch) return cudaErrorInvalidConfiguration;
    const int grid = P.n_heads * P.n_qtiles;
    if (grid == 0) return cudaSuccess;
    static const char *const names[] = {"attn_kernel<DENSE>", "attn_kernel<VS>", "attn_kernel<BLOCK>",
                                        "attn_kernel<ASHAPE>"};
    ProfScope prof(names[PAT], st);
    attn_kernel<PAT><<<grid, kThreads, kSmemBytes, st>>>(P);
    return cudaGetLastError();
}

// Applies the attention kernel's two exponential paths to x: the FMA-pipe
// polynomial and the MUFU ex2 (self-test of the polynomial against the hardware).
__global__ void exp2_selftest_kernel(const float *x, float *y_poly, float *y_hw, int n) {
    const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
    if (i >= n) return;
    float a = x[i], b = i + 1 < n ? x[i + 1] : 0.f;
    y_hw[i] = ex2_approx(a);
    if (i + 1 < n) y_hw[i + 1] = ex2_approx(b);
    exp2_poly_pair(a, b);
    y_poly[i] = a;
    if (i + 1 < n) y_poly[i + 1] = b;
}

}  // namespace

cudaError_t run_exp2_selftest(const float *x, float *y_poly, float *y_hw, int n, cudaStream_t st) {
    const int pairs = (n + 1) / 2;
    if (pairs == 0) return cudaSuccess;
    exp2_selftest_kernel<<<(pairs + 255) / 256, 256, 0, st>>>(x, y_poly, y_hw, n);
    return cudaGetLastError();
}

cudaError_t run_attention(int pattern, const AttnParams &P, cudaStream_t st) {
    switch (pattern) {
    case PAT_DENSE: return launch_attn<PAT_DENSE>(P, st);
    case PAT_ASHAPE: return launch_attn<PAT_ASHAPE>(P, st);
    case PAT_BLOCK: return launch_attn<PAT_BLOCK>(P, st);
    case PAT_VS: return launch_attn<PAT_VS>(P, st);
    }
    return cudaErrorInvalidValue;
}

cudaError_t run_bs_plan(const int *blk_idx, const int *blk_cnt, int topk, int n_heads, int n_qtiles, int nb,
                        int *plan, int *cnt, int stride, cudaStream_t st) {
    const int nw = n_heads * n_qtiles;
    ProfScope prof("bs_plan", st);
    bs_plan_kernel<<<(nw + 127) / 128, 128, 0, st>>>(blk_idx, blk_cnt, topk, n_heads, n_qtiles, nb, plan, cnt,
                                                     stride);
    return cudaGetLastError();
}

cudaError_t run_vs_plan(const VsPlanBufs &b, const int *v_idx, int n_vertical, const int *s_idx, int n_slash,
                        int n, int n_heads, int n_qtiles, float diag_ratio, cudaStream_t st) {
    ProfScope prof("vs_plan", st);
    // the guards are cleared with the bitmaps
    const size_t bytes = sizeof(uint32_t) * (size_t)n_heads * b.stride;
    cudaError_t e = cudaMemsetAsync(b.bits_v - kBitGuard, 0, bytes, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(b.bits_s - kBitGuard, 0, bytes, st);
    if (e != cudaSuccess) return e;
    vs_mark_kernel<<<n_heads, 256, 0, st>>>(v_idx, n_vertical, s_idx, n_slash, n, b.bits_v, b.bits_s, b.stride);
    vs_extract_kernel<<<n_heads, kExtractThreads, 0, st>>>(b.bits_v, b.bits_s, b.words, b.stride, b.vsorted, b.nvs,
                                                           b.vcap, b.soff, b.scap, b.groups, b.ngroups, b.dgroups,
                                                           b.ndgroups, diag_ratio);
    const int nw = n_heads * n_qtiles;
    vs_workitem_kernel<<<(nw + 3) / 4, 128, 0, st>>>(b.vsorted, b.nvs, b.vcap, b.groups, b.ngroups, b.scap,
                                                     b.bits_s, b.stride, n, n_heads, n_qtiles, b.nsh, b.nvert,
                                                     b.nle, b.vlist);
    return cudaGetLastError();
}

}  // namespace minf
