// topk.cu -- radix select: the k largest of a row (ties to the lower index),
// written as ascending indices.  Used for the vertical keys and slash offsets
// of Vertical-Slash (rows of n floats) and, through topk.cuh, for the
// per-query-block rows of Block-Sparse.
//
// A float maps to an unsigned key with the same order (non-negative floats as
// their bits).  Four 8-bit digit passes find the k-th largest key t and how
// many keys equal to t are needed; an ordered compaction then keeps every key
// above t and the first needed keys equal to t.
//
// Rows of up to kSmemRow floats are handled by one 1024-thread block with the
// row held in shared memory.  Longer rows (up to 1M keys and beyond) are split
// into chunks of kChunk keys over many blocks: per-chunk histograms are added
// into a per-row global histogram, one small block per row picks the digit,
// and the compaction uses per-chunk counts scanned per row.
#include "common.cuh"
#include "internal.h"
#include "topk.cuh"

namespace minf {

namespace {

constexpr int kTopkThreads = 1024;
constexpr int kSmemRow = 48 * 1024;  // floats held in shared memory by the one-block path
constexpr int kChunk = 8192;         // keys per block in the multi-block path
constexpr int kChunkThreads = 256;

// One block per row; blocks [0, a.n_rows) take the rows of a, the rest those of b
// (two independent row sets of the same length in one launch).
__global__ void __launch_bounds__(kTopkThreads) topk_rows_smem_kernel(const TopkRows a, const TopkRows b, int len) {
    extern __shared__ float row[];
    __shared__ TopkShared sh;
    const bool second = (int)blockIdx.x >= a.n_rows;
    const int r = second ? (int)blockIdx.x - a.n_rows : (int)blockIdx.x;
    const float *x = (second ? b.scores : a.scores) + (size_t)r * len;
    const int k = second ? b.k : a.k;
    const int *k_row = second ? b.k_row : a.k_row;
    for (int i = threadIdx.x * 4; i < len; i += kTopkThreads * 4) {
        if (i + 3 < len) {
            *reinterpret_cast<float4 *>(row + i) = __ldg(reinterpret_cast<const float4 *>(x + i));
        } else {
            for (int j = i; j < len; ++j) row[j] = x[j];
        }
    }
    __syncthreads();
    int *o = (second ? b.out : a.out) + (size_t)r * k;
    const int kr = k_row ? max(0, min(k_row[r], k)) : k;
    block_topk_ascending<kTopkThreads, false>(row, len, kr, o, 0, sh);
    for (int j = min(kr, len) + (int)threadIdx.x; j < k; j += kTopkThreads) o[j] = -1;
}

// ---- multi-block path --------------------------------------------------------
struct RowState {
    uint32_t prefix, mask;
    int remaining;  // keys equal to the threshold still to take
    int k;          // this row's count, at most the row stride
};

__global__ void topk_init_kernel(RowState *st, uint32_t *hist, int rows, int len, int k, const int *k_row) {
    const int r = blockIdx.x;
    for (int b = threadIdx.x; b < 256; b += blockDim.x) hist[(size_t)r * 256 + b] = 0u;
    const int kr = k_row ? max(0, min(k_row[r], k)) : k;
    if (threadIdx.x == 0) st[r] = RowState{0u, 0u, min(kr, len), kr};
}

__global__ void __launch_bounds__(kChunkThreads) topk_hist_kernel(const float *scores, int len,
                                                                  const RowState *st, uint32_t *hist,
                                                                  int shift) {
    __shared__ unsigned h[256];
    const int r = blockIdx.y;
    const RowState s = st[r];
    if (s.remaining <= 0) return;
    for (int b = threadIdx.x; b < 256; b += kChunkThreads) h[b] = 0u;
    __syncthreads();
    const float *x = scores + (size_t)r * len;
    const int c0 = blockIdx.x * kChunk, c1 = min(len, c0 + kChunk);
    for (int i0 = c0; i0 < c1; i0 += kChunkThreads) {
        const int i = i0 + threadIdx.x;
        const bool in = i < c1;
        const uint32_t u = in ? __float_as_uint(__ldg(x + i)) : 0u;
        const bool hit = in && (u & s.mask) == s.prefix;
        const uint32_t bin = (u >> shift) & 255u;
        if (hit) atomicAdd(&h[bin], 1u);
    }
    __syncthreads();
    for (int b = threadIdx.x; b < 256; b += kChunkThreads)
        if (h[b]) atomicAdd(hist + (size_t)r * 256 + b, h[b]);
}

// One block of 256 threads per row: digit with the remaining count inside it,
// found from the top of the histogram by a suffix scan.
__global__ void topk_digit_kernel(RowState *st, uint32_t *hist, int shift) {
    __shared__ int suffix[256];
    const int r = blockIdx.x, b = threadIdx.x;
    const RowState s = st[r];
    const int hb = (int)hist[(size_t)r * 256 + b];
    // inclusive suffix sum over bins b..255 (Hillis-Steele)
    suffix[b] = hb;
    __syncthreads();
    for (int off = 1; off < 256; off <<= 1) {
        const int add = b + off < 256 ? suffix[b + off] : 0;
        __syncthreads();
        suffix[b] += add;
        __syncthreads();
    }
    const int above = suffix[b] - hb;  // keys in bins > b
    if (s.remaining > 0 && above < s.remaining && suffix[b] >= s.remaining) {
        RowState n = s;
        n.prefix |= (uint32_t)b << shift;
        n.mask |= 255u << shift;
        n.remaining = s.remaining - above;
        st[r] = n;
    }
    hist[(size_t)r * 256 + b] = 0u;
}

// Per chunk: keys above the threshold and keys equal to it.
__global__ void __launch_bounds__(kChunkThreads) topk_count_kernel(const float *scores, int len, const RowState *st,
                                                                   int2 *cnt, int n_chunks) {
    __shared__ int red[2][kChunkThreads / 32];
    const int r = blockIdx.y;
    // a row with nothing to take: every key counts as below the threshold
    const uint32_t t = st[r].k > 0 ? st[r].prefix : 0xffffffffu;
    const float *x = scores + (size_t)r * len;
    const int c0 = blockIdx.x * kChunk, c1 = min(len, c0 + kChunk);
    int gt = 0, eq = 0;
    for (int i = c0 + threadIdx.x; i < c1; i += kChunkThreads) {
        const uint32_t u = __float_as_uint(__ldg(x + i));
        gt += u > t;
        eq += u == t;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        gt += __shfl_xor_sync(0xffffffffu, gt, o);
        eq += __shfl_xor_sync(0xffffffffu, eq, o);
    }
    if ((threadIdx.x & 31) == 0) {
        red[0][threadIdx.x >> 5] = gt;
        red[1][threadIdx.x >> 5] = eq;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int a = 0, b = 0;
        for (int w = 0; w < kChunkThreads / 32; ++w) {
            a += red[0][w];
            b += red[1][w];
        }
        cnt[(size_t)r * n_chunks + blockIdx.x] = make_int2(a, b);
    }
}

// Per row: for each chunk, the equal keys before it and its output offset.
__global__ void topk_offsets_kernel(const RowState *st, const int2 *cnt, int2 *off, int n_chunks) {
    const int r = blockIdx.x;
    if (threadIdx.x != 0) return;
    const int need = st[r].remaining;
    int eq_before = 0, out_before = 0;
    for (int c = 0; c < n_chunks; ++c) {
        const int2 v = cnt[(size_t)r * n_chunks + c];
        off[(size_t)r * n_chunks + c] = make_int2(eq_before, out_before);
        const int take_eq = max(0, min(v.y, need - eq_before));
        out_before += v.x + take_eq;
        eq_before += v.y;
    }
}

__global__ void __launch_bounds__(kChunkThreads) topk_write_kernel(const float *scores, int len, int k,
                                                                   const RowState *st, const int2 *off,
                                                                   int n_chunks, int *out) {
    __shared__ TopkShared sh;
    const int r = blockIdx.y;
    const uint32_t t = st[r].k > 0 ? st[r].prefix : 0xffffffffu;
    const int need = st[r].remaining;
    const int2 base = off[(size_t)r * n_chunks + blockIdx.x];
    const float *x = scores + (size_t)r * len;
    int *o = out + (size_t)r * k;
    const int c0 = blockIdx.x * kChunk, c1 = min(len, c0 + kChunk);
    int eq_seen = base.x, pos0 = base.y;
    for (int start = c0; start < c1; start += kChunkThreads * 4) {
        const int i0 = start + threadIdx.x * 4;
        uint32_t keys[4];
        int n_eq = 0;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            keys[e] = (i0 + e < c1) ? __float_as_uint(__ldg(x + i0 + e)) : 0u;
            n_eq += (i0 + e < c1 && keys[e] == t) ? 1 : 0;
        }
        int eq_tot;
        const int eq_before = eq_seen + block_excl_scan<kChunkThreads>(n_eq, &eq_tot, sh);
        bool take[4];
        int n_take = 0, eq_r = 0;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const bool valid = i0 + e < c1;
            const bool eq = valid && keys[e] == t;
            take[e] = valid && (keys[e] > t || (eq && eq_before + eq_r < need));
            eq_r += eq ? 1 : 0;
            n_take += take[e] ? 1 : 0;
        }
        int take_tot;
        int pos = pos0 + block_excl_scan<kChunkThreads>(n_take, &take_tot, sh);
#pragma unroll
        for (int e = 0; e < 4; ++e)
            if (take[e]) o[pos++] = i0 + e;
        pos0 += take_tot;
        eq_seen += eq_tot;
    }
    if (blockIdx.x == 0)
        for (int j = min(st[r].k, len) + (int)threadIdx.x; j < k; j += kChunkThreads) o[j] = -1;
}

// ---- top-p counts -------------------------------------------------------------
// For each row: the fewest keys, best first (ties to the lower index), whose
// scores sum to at least p of the row's mass.  With skip0, key 0 is left out
// (it holds a forced entry) and extra0[row], that entry's own score, is counted
// first.  Masses are summed exactly in 2^-32 fixed point (a score is at most
// 64, so a row of 2^20 keys stays below 2^58): the count does not depend on
// the order of the additions.  The threshold is found like the top-k one, on
// histograms of mass instead of counts, over 8K-key chunks of the row.
constexpr int kToppChunk = 8192;

struct ToppState {
    uint32_t prefix, mask;
    unsigned long long rem;  // mass still needed from keys at or below the current prefix
    int above;               // keys already known to be above the threshold
    int eq;                  // keys in the chosen bin of the last pass
    int done;                // nothing (more) needed
    int pad;
};

__device__ __forceinline__ unsigned long long fixed_mass(float x) {
    return __float2ull_rz(x * 4294967296.0f);
}

__device__ __forceinline__ unsigned long long shfl_up_u64(unsigned long long v, int d) {
    const uint32_t lo = __shfl_up_sync(0xffffffffu, (uint32_t)v, d);
    const uint32_t hi = __shfl_up_sync(0xffffffffu, (uint32_t)(v >> 32), d);
    return ((unsigned long long)hi << 32) | lo;
}

__global__ void __launch_bounds__(kChunkThreads) topp_total_kernel(const float *scores, int len, int skip0,
                                                                  unsigned long long *total) {
    __shared__ unsigned long long red[kChunkThreads / 32];
    const int r = blockIdx.y, lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const float *x = scores + (size_t)r * len;
    const int c0 = max(blockIdx.x * kToppChunk, skip0), c1 = min(len, (int)(blockIdx.x + 1) * kToppChunk);
    unsigned long long part = 0;
    for (int i = c0 + threadIdx.x; i < c1; i += kChunkThreads) part += fixed_mass(__ldg(x + i));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
    if (lane == 0) red[wid] = part;
    __syncthreads();
    if (threadIdx.x == 0) {
        unsigned long long t = 0;
        for (int w = 0; w < kChunkThreads / 32; ++w) t += red[w];
        atomicAdd(total + r, t);  // integer: the sum is exact in any order
    }
}

__global__ void topp_init_kernel(const unsigned long long *total, int skip0, const float *extra0, float p,
                                 ToppState *st, uint32_t *hcnt, unsigned long long *hmass) {
    const int r = blockIdx.x;
    for (int b = threadIdx.x; b < 256; b += blockDim.x) {
        hcnt[(size_t)r * 256 + b] = 0u;
        hmass[(size_t)r * 256 + b] = 0ull;
    }
    if (threadIdx.x == 0) {
        const unsigned long long m0 = skip0 ? fixed_mass(extra0[r]) : 0ull, all = total[r] + m0;
        unsigned long long target = (unsigned long long)ceil((double)p * (double)all);
        target = min(target, all);
        ToppState s;
        s.prefix = 0u;
        s.mask = 0u;
        s.rem = target > m0 ? target - m0 : 0ull;
        s.above = 0;
        s.eq = 0;
        s.done = s.rem == 0ull;
        s.pad = 0;
        st[r] = s;
    }
}

__global__ void __launch_bounds__(kChunkThreads) topp_hist_kernel(const float *scores, int len, int skip0,
                                                                 const ToppState *st, uint32_t *hcnt,
                                                                 unsigned long long *hmass, int shift) {
    __shared__ unsigned long long sm[256];
    __shared__ uint32_t sc[256];
    const int r = blockIdx.y, lane = threadIdx.x & 31;
    const ToppState s = st[r];
    if (s.done) return;
    for (int b = threadIdx.x; b < 256; b += kChunkThreads) {
        sm[b] = 0ull;
        sc[b] = 0u;
    }
    __syncthreads();
    const float *x = scores + (size_t)r * len;
    const int c0 = max(blockIdx.x * kToppChunk, skip0), c1 = min(len, (int)(blockIdx.x + 1) * kToppChunk);
    for (int i0 = c0; i0 < c1; i0 += kChunkThreads) {
        const int i = i0 + threadIdx.x;
        uint32_t u = 0u;
        bool valid = false;
        if (i < c1) {
            u = __float_as_uint(__ldg(x + i));
            valid = (u & s.mask) == s.prefix;
        }
        const uint32_t bin = (u >> shift) & 255u;
        const unsigned long long m = valid ? fixed_mass(__uint_as_float(u)) : 0ull;
        // one shared atomic per distinct bin per warp: exact sums of <= 2^16 / 2^16 / 2^6 parts
        unsigned todo = __ballot_sync(0xffffffffu, valid);
        while (todo) {
            const int leader = __ffs(todo) - 1;
            const uint32_t lb = __shfl_sync(0xffffffffu, bin, leader);
            const bool mine = valid && bin == lb;
            const unsigned grp = __ballot_sync(0xffffffffu, mine);
            const uint32_t a = __reduce_add_sync(0xffffffffu, mine ? (uint32_t)(m & 0xffffu) : 0u);
            const uint32_t b = __reduce_add_sync(0xffffffffu, mine ? (uint32_t)((m >> 16) & 0xffffu) : 0u);
            const uint32_t c = __reduce_add_sync(0xffffffffu, mine ? (uint32_t)(m >> 32) : 0u);
            if (lane == leader) {
                atomicAdd(&sc[lb], (uint32_t)__popc(grp));
                atomicAdd(&sm[lb], ((unsigned long long)c << 32) + ((unsigned long long)b << 16) + a);
            }
            todo &= ~grp;
        }
    }
    __syncthreads();
    for (int b = threadIdx.x; b < 256; b += kChunkThreads)
        if (sc[b]) {
            atomicAdd(hcnt + (size_t)r * 256 + b, sc[b]);
            atomicAdd(hmass + (size_t)r * 256 + b, sm[b]);
        }
}

// One warp per row: lane L owns bins 255-8L .. 248-8L; a scan from the top finds
// the bin where the mass still needed is reached.  The histogram is cleared for
// the next pass.
__global__ void topp_digit_kernel(ToppState *st, uint32_t *hcnt, unsigned long long *hmass, int shift) {
    const int r = blockIdx.x, lane = threadIdx.x;
    ToppState s = st[r];
    unsigned long long ms[8], sum = 0;
    uint32_t cs[8], csum = 0;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        const size_t at = (size_t)r * 256 + 255 - 8 * lane - e;
        ms[e] = hmass[at];
        cs[e] = hcnt[at];
        hmass[at] = 0ull;
        hcnt[at] = 0u;
        sum += ms[e];
        csum += cs[e];
    }
    if (s.done) return;
    unsigned long long incl = sum;
    uint32_t cincl = csum;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const unsigned long long y = shfl_up_u64(incl, d);
        const uint32_t cy = __shfl_up_sync(0xffffffffu, cincl, d);
        if (lane >= d) {
            incl += y;
            cincl += cy;
        }
    }
    unsigned long long cum = incl - sum;
    uint32_t ccum = cincl - csum;
    if (cum < s.rem && incl >= s.rem) {
        int e = 0;
        for (; e < 7; ++e) {
            if (cum + ms[e] >= s.rem) break;
            cum += ms[e];
            ccum += cs[e];
        }
        s.prefix |= (uint32_t)(255 - 8 * lane - e) << shift;
        s.mask |= 255u << shift;
        s.rem -= cum;
        s.above += (int)ccum;
        s.eq = (int)cs[e];
        st[r] = s;
    }
}

__global__ void topp_final_kernel(const ToppState *st, int skip0, int cap, int *count) {
    const int r = blockIdx.x * blockDim.x + threadIdx.x;
    if (r >= gridDim.x * blockDim.x) return;
    const ToppState s = st[r];
    int c = 0;
    if (!s.done) {
        // keys above the threshold, then as many of its ties (each of the same mass) as the rest needs
        const unsigned long long mt = fixed_mass(__uint_as_float(s.prefix));
        long long need = mt ? (long long)((s.rem + mt - 1) / mt) : (long long)s.eq;
        need = min(need, (long long)s.eq);
        c = s.above + (int)need;
    }
    count[r] = min(c + skip0, cap);
}

// Rows of up to kSmemRow floats: one 1024-thread block per row does the whole
// top-p count (total, four mass-histogram digit passes, final count) with the
// row in shared memory, and blocks [0, a.n_rows) take row set a, the rest row
// set b.  The arithmetic is that of the multi-block kernels above: the same
// fixed-point masses, exact integer sums, the same digit search and final count.
struct ToppRows {
    const float *scores;
    int n_rows, skip0, cap;
    const float *extra0;
    float p;
    int *count;
};

__global__ void __launch_bounds__(kTopkThreads) topp_rows_smem_kernel(const ToppRows a, const ToppRows b, int len) {
    extern __shared__ float row[];
    __shared__ unsigned long long hm[256];
    __shared__ uint32_t hc[256];
    __shared__ unsigned long long red[kTopkThreads / 32];
    __shared__ ToppState sst;
    const bool second = (int)blockIdx.x >= a.n_rows;
    const ToppRows &g = second ? b : a;
    const int r = second ? (int)blockIdx.x - a.n_rows : (int)blockIdx.x;
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const float *x = g.scores + (size_t)r * len;
    for (int i = threadIdx.x * 4; i < len; i += kTopkThreads * 4) {
        if (i + 3 < len) {
            *reinterpret_cast<float4 *>(row + i) = __ldg(reinterpret_cast<const float4 *>(x + i));
        } else {
            for (int j = i; j < len; ++j) row[j] = x[j];
        }
    }
    __syncthreads();
    // total mass of the keys from skip0 on (exact: integer sums)
    unsigned long long part = 0;
    for (int i = g.skip0 + (int)threadIdx.x; i < len; i += kTopkThreads) part += fixed_mass(row[i]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
    if (lane == 0) red[wid] = part;
    __syncthreads();
    if (threadIdx.x == 0) {
        unsigned long long total = 0;
        for (int w = 0; w < kTopkThreads / 32; ++w) total += red[w];
        const unsigned long long m0 = g.skip0 ? fixed_mass(g.extra0[r]) : 0ull, all = total + m0;
        unsigned long long target = (unsigned long long)ceil((double)g.p * (double)all);
        target = min(target, all);
        ToppState st0;
        st0.prefix = 0u;
        st0.mask = 0u;
        st0.rem = target > m0 ? target - m0 : 0ull;
        st0.above = 0;
        st0.eq = 0;
        st0.done = st0.rem == 0ull;
        st0.pad = 0;
        sst = st0;
    }
    __syncthreads();
#pragma unroll 1
    for (int pass = 0; pass < 4; ++pass) {
        const ToppState s = sst;
        if (s.done) break;  // uniform: every thread read the same state
        const int shift = 24 - 8 * pass;
        for (int bb = threadIdx.x; bb < 256; bb += kTopkThreads) {
            hm[bb] = 0ull;
            hc[bb] = 0u;
        }
        __syncthreads();
        for (int i0 = g.skip0; i0 < len; i0 += kTopkThreads) {
            const int i = i0 + threadIdx.x;
            uint32_t u = 0u;
            bool valid = false;
            if (i < len) {
                u = __float_as_uint(row[i]);
                valid = (u & s.mask) == s.prefix;
            }
            const uint32_t bin = (u >> shift) & 255u;
            const unsigned long long m = valid ? fixed_mass(__uint_as_float(u)) : 0ull;
            // one shared atomic per distinct bin per warp: exact sums of <= 2^16 / 2^16 / 2^6 parts
            unsigned todo = __ballot_sync(0xffffffffu, valid);
            while (todo) {
                const int leader = __ffs(todo) - 1;
                const uint32_t lb = __shfl_sync(0xffffffffu, bin, leader);
                const bool mine = valid && bin == lb;
                const unsigned grp = __ballot_sync(0xffffffffu, mine);
                const uint32_t a0 = __reduce_add_sync(0xffffffffu, mine ? (uint32_t)(m & 0xffffu) : 0u);
                const uint32_t a1 = __reduce_add_sync(0xffffffffu, mine ? (uint32_t)((m >> 16) & 0xffffu) : 0u);
                const uint32_t a2 = __reduce_add_sync(0xffffffffu, mine ? (uint32_t)(m >> 32) : 0u);
                if (lane == leader) {
                    atomicAdd(&hc[lb], (uint32_t)__popc(grp));
                    atomicAdd(&hm[lb], ((unsigned long long)a2 << 32) + ((unsigned long long)a1 << 16) + a0);
                }
                todo &= ~grp;
            }
        }
        __syncthreads();
        if (wid == 0) {
            // lane L owns bins 255-8L .. 248-8L; a scan from the top finds the bin where
            // the mass still needed is reached
            unsigned long long ms[8], sum = 0;
            uint32_t cs[8], csum = 0;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                ms[e] = hm[255 - 8 * lane - e];
                cs[e] = hc[255 - 8 * lane - e];
                sum += ms[e];
                csum += cs[e];
            }
            unsigned long long incl = sum;
            uint32_t cincl = csum;
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                const unsigned long long y = shfl_up_u64(incl, d);
                const uint32_t cy = __shfl_up_sync(0xffffffffu, cincl, d);
                if (lane >= d) {
                    incl += y;
                    cincl += cy;
                }
            }
            unsigned long long cum = incl - sum;
            uint32_t ccum = cincl - csum;
            if (cum < s.rem && incl >= s.rem) {
                int e = 0;
                for (; e < 7; ++e) {
                    if (cum + ms[e] >= s.rem) break;
                    cum += ms[e];
                    ccum += cs[e];
                }
                ToppState n = s;
                n.prefix |= (uint32_t)(255 - 8 * lane - e) << shift;
                n.mask |= 255u << shift;
                n.rem -= cum;
                n.above += (int)ccum;
                n.eq = (int)cs[e];
                sst = n;
            }
        }
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        const ToppState s = sst;
        int c = 0;
        if (!s.done) {
            // keys above the threshold, then as many of its ties (each of the same mass) as the rest needs
            const unsigned long long mt = fixed_mass(__uint_as_float(s.prefix));
            long long need = mt ? (long long)((s.rem + mt - 1) / mt) : (long long)s.eq;
            need = min(need, (long long)s.eq);
            c = s.above + (int)need;
        }
        g.count[r] = min(c + g.skip0, g.cap);
    }
}

}  // namespace

cudaError_t run_topp_counts2(const float *scores_a, int n_rows_a, bool skip0_a, const float *extra0_a, float p_a,
                             int cap_a, int *count_a, const float *scores_b, int n_rows_b, bool skip0_b,
                             const float *extra0_b, float p_b, int cap_b, int *count_b, int len, void *scratch,
                             cudaStream_t st) {
    if (len <= kSmemRow && n_rows_a + n_rows_b > 0) {
        const int smem = len * (int)sizeof(float);
        cudaError_t e = cudaFuncSetAttribute(topp_rows_smem_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        const ToppRows A{scores_a, max(n_rows_a, 0), skip0_a ? 1 : 0, cap_a, extra0_a, p_a, count_a};
        const ToppRows B{scores_b, max(n_rows_b, 0), skip0_b ? 1 : 0, cap_b, extra0_b, p_b, count_b};
        topp_rows_smem_kernel<<<A.n_rows + B.n_rows, kTopkThreads, smem, st>>>(A, B, len);
        return cudaGetLastError();
    }
    cudaError_t e = run_topp_counts(scores_a, n_rows_a, len, skip0_a, extra0_a, p_a, cap_a, count_a, scratch, st);
    if (e != cudaSuccess) return e;
    return run_topp_counts(scores_b, n_rows_b, len, skip0_b, extra0_b, p_b, cap_b, count_b, scratch, st);
}

size_t topp_scratch_bytes(int n_rows) {
    return (size_t)n_rows * (sizeof(unsigned long long) + sizeof(ToppState) + 256 * (4 + 8)) + 1024;
}

cudaError_t run_topp_counts(const float *scores, int n_rows, int len, bool skip0, const float *extra0, float p,
                            int cap, int *count, void *scratch, cudaStream_t st) {
    if (n_rows <= 0) return cudaSuccess;
    if (!scratch) return cudaErrorInvalidValue;
    char *q = static_cast<char *>(scratch);
    auto align = [](size_t x) { return (x + 255) & ~size_t(255); };
    size_t off = 0;
    unsigned long long *total = reinterpret_cast<unsigned long long *>(q + off);
    off = align(off + n_rows * sizeof(unsigned long long));
    ToppState *state = reinterpret_cast<ToppState *>(q + off);
    off = align(off + n_rows * sizeof(ToppState));
    uint32_t *hcnt = reinterpret_cast<uint32_t *>(q + off);
    off = align(off + (size_t)n_rows * 256 * sizeof(uint32_t));
    unsigned long long *hmass = reinterpret_cast<unsigned long long *>(q + off);
    const int sk = skip0 ? 1 : 0;
    const int n_chunks = (len + kToppChunk - 1) / kToppChunk;
    const dim3 grid(n_chunks, n_rows);
    cudaError_t e = cudaMemsetAsync(total, 0, n_rows * sizeof(unsigned long long), st);
    if (e != cudaSuccess) return e;
    topp_total_kernel<<<grid, kChunkThreads, 0, st>>>(scores, len, sk, total);
    topp_init_kernel<<<n_rows, 256, 0, st>>>(total, sk, extra0, p, state, hcnt, hmass);
    for (int pass = 0; pass < 4; ++pass) {
        const int shift = 24 - 8 * pass;
        topp_hist_kernel<<<grid, kChunkThreads, 0, st>>>(scores, len, sk, state, hcnt, hmass, shift);
        topp_digit_kernel<<<n_rows, 32, 0, st>>>(state, hcnt, hmass, shift);
    }
    topp_final_kernel<<<n_rows, 1, 0, st>>>(state, sk, cap, count);
    return cudaGetLastError();
}

size_t topk_scratch_bytes(int n_rows, int len) {
    if (len <= kSmemRow) return 0;
    const int n_chunks = (len + kChunk - 1) / kChunk;
    return (size_t)n_rows * (sizeof(RowState) + 256 * sizeof(uint32_t) + 2 * (size_t)n_chunks * sizeof(int2)) + 1024;
}

// Rows longer than kSmemRow: chunked radix select over many blocks.
static cudaError_t run_topk_rows_long(const TopkRows &t, int len, void *scratch, cudaStream_t st) {
    const float *scores = t.scores;
    const int n_rows = t.n_rows, k = t.k;
    const int *k_row = t.k_row;
    int *out = t.out;
    if (!scratch) return cudaErrorInvalidValue;
    const int n_chunks = (len + kChunk - 1) / kChunk;
    char *p = static_cast<char *>(scratch);
    auto align = [](size_t x) { return (x + 255) & ~size_t(255); };
    size_t off = 0;
    RowState *state = reinterpret_cast<RowState *>(p + off);
    off = align(off + n_rows * sizeof(RowState));
    uint32_t *hist = reinterpret_cast<uint32_t *>(p + off);
    off = align(off + (size_t)n_rows * 256 * sizeof(uint32_t));
    int2 *cnt = reinterpret_cast<int2 *>(p + off);
    off = align(off + (size_t)n_rows * n_chunks * sizeof(int2));
    int2 *offs = reinterpret_cast<int2 *>(p + off);
    topk_init_kernel<<<n_rows, 256, 0, st>>>(state, hist, n_rows, len, k, k_row);
    const dim3 grid(n_chunks, n_rows);
    for (int pass = 0; pass < 4; ++pass) {
        const int shift = 24 - 8 * pass;
        topk_hist_kernel<<<grid, kChunkThreads, 0, st>>>(scores, len, state, hist, shift);
        topk_digit_kernel<<<n_rows, 256, 0, st>>>(state, hist, shift);
    }
    topk_count_kernel<<<grid, kChunkThreads, 0, st>>>(scores, len, state, cnt, n_chunks);
    topk_offsets_kernel<<<n_rows, 32, 0, st>>>(state, cnt, offs, n_chunks);
    topk_write_kernel<<<grid, kChunkThreads, 0, st>>>(scores, len, k, state, offs, n_chunks, out);
    return cudaGetLastError();
}

cudaError_t run_topk_rows(const float *scores, int n_rows, int len, int k, int *out, void *scratch,
                          cudaStream_t st, const int *k_row) {
    return run_topk_rows2(TopkRows{scores, n_rows, k, out, k_row}, TopkRows{nullptr, 0, 0, nullptr, nullptr}, len,
                          scratch, st);
}

cudaError_t run_topk_rows2(const TopkRows &a, const TopkRows &b, int len, void *scratch, cudaStream_t st) {
    const TopkRows A = (a.n_rows > 0 && a.k > 0) ? a : TopkRows{nullptr, 0, 0, nullptr, nullptr};
    const TopkRows B = (b.n_rows > 0 && b.k > 0) ? b : TopkRows{nullptr, 0, 0, nullptr, nullptr};
    if (A.n_rows + B.n_rows == 0) return cudaSuccess;
    if (len <= kSmemRow) {
        const int smem = len * (int)sizeof(float);
        cudaError_t e = cudaFuncSetAttribute(topk_rows_smem_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        topk_rows_smem_kernel<<<A.n_rows + B.n_rows, kTopkThreads, smem, st>>>(A, B, len);
        return cudaGetLastError();
    }
    if (!scratch) return cudaErrorInvalidValue;
    // long rows: the row sets one after the other, sharing the scratch
    for (const TopkRows *t : {&A, &B}) {
        if (t->n_rows == 0) continue;
        cudaError_t e = run_topk_rows_long(*t, len, scratch, st);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace minf
