// topk.cuh -- device routines of the block-wide radix select (see topk.cu).
#pragma once

#include <cstdint>

namespace minf {

struct TopkShared {
    unsigned hist[256];
    int scan[33];
    int digit;
    int remaining;
};

// Order-preserving map of a float to an unsigned key.
template <bool SIGNED>
__device__ __forceinline__ uint32_t topk_key(float f) {
    const uint32_t u = __float_as_uint(f);
    if constexpr (SIGNED) return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    return u;
}

// Exclusive prefix sum of v over the NT threads of the block; *total gets the sum.
template <int NT>
__device__ __forceinline__ int block_excl_scan(int v, int *total, TopkShared &sh) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    int incl = v;
#pragma unroll
    for (int s = 1; s < 32; s <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, s);
        if (lane >= s) incl += y;
    }
    if (lane == 31) sh.scan[wid] = incl;
    __syncthreads();
    if (wid == 0) {
        const int w = lane < NT / 32 ? sh.scan[lane] : 0;
        int winc = w;
#pragma unroll
        for (int s = 1; s < 32; s <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, winc, s);
            if (lane >= s) winc += y;
        }
        if (lane < NT / 32) sh.scan[lane] = winc - w;
        if (lane == 31) sh.scan[32] = winc;
    }
    __syncthreads();
    const int res = sh.scan[wid] + incl - v;
    *total = sh.scan[32];
    __syncthreads();
    return res;
}

// Writes the indices (+ add) of the min(k, len) largest entries of x[0..len),
// ties to the lower index, ascending, to out[0..min(k, len)).  All NT threads
// of the block must call it.
template <int NT, bool SIGNED>
__device__ void block_topk_ascending(const float *x, int len, int k, int *out, int add, TopkShared &sh) {
    const int tid = threadIdx.x;
    const int kk = min(k, len);
    if (kk <= 0) return;
    if (kk == len) {
        for (int j = tid; j < len; j += NT) out[j] = j + add;
        return;
    }
    uint32_t prefix = 0, pmask = 0;
    int rem = kk;
#pragma unroll 1
    for (int pass = 0; pass < 4; ++pass) {
        const int shift = 24 - 8 * pass;
        for (int b = tid; b < 256; b += NT) sh.hist[b] = 0;
        __syncthreads();
        for (int i0 = 0; i0 < len; i0 += NT) {
            const int i = i0 + tid;
            const bool in = i < len;
            const uint32_t u = in ? topk_key<SIGNED>(x[i]) : 0u;
            const bool hit = in && (u & pmask) == prefix;
            const uint32_t bin = (u >> shift) & 255u;
            // plain shared-memory atomics: measured faster than aggregating equal bins
            // with match.any on score rows, whose first digits spread over a few bins
            if (hit) atomicAdd(&sh.hist[bin], 1u);
        }
        __syncthreads();
        if (tid < 32) {
            // lane L owns bins 255-8L .. 248-8L; a scan over lanes from the top
            // finds the lane whose bins hold the rem-th largest key.
            int c[8], sum = 0;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                c[e] = (int)sh.hist[255 - 8 * tid - e];
                sum += c[e];
            }
            int incl = sum;
#pragma unroll
            for (int s = 1; s < 32; s <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, incl, s);
                if (tid >= s) incl += y;
            }
            int cum = incl - sum;
            if (cum < rem && incl >= rem) {
                int d = 255 - 8 * tid;
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    if (cum + c[e] >= rem) break;
                    cum += c[e];
                    --d;
                }
                sh.digit = d;
                sh.remaining = rem - cum;
            }
        }
        __syncthreads();
        prefix |= (uint32_t)sh.digit << shift;
        pmask |= 255u << shift;
        rem = sh.remaining;
        __syncthreads();
    }
    // keys > prefix are all taken; keys == prefix: the first `rem` in index order
    int base = 0, eq_seen = 0;
#pragma unroll 1
    for (int start = 0; start < len; start += NT * 4) {
        const int i0 = start + tid * 4;
        uint32_t keys[4];
        int n_eq = 0;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            keys[e] = (i0 + e < len) ? topk_key<SIGNED>(x[i0 + e]) : 0u;
            n_eq += (i0 + e < len && keys[e] == prefix) ? 1 : 0;
        }
        int eq_tot;
        const int eq_before = eq_seen + block_excl_scan<NT>(n_eq, &eq_tot, sh);
        bool take[4];
        int n_take = 0, eq_r = 0;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const bool valid = i0 + e < len;
            const bool eq = valid && keys[e] == prefix;
            take[e] = valid && (keys[e] > prefix || (eq && eq_before + eq_r < rem));
            eq_r += eq ? 1 : 0;
            n_take += take[e] ? 1 : 0;
        }
        int take_tot;
        int pos = base + block_excl_scan<NT>(n_take, &take_tot, sh);
#pragma unroll
        for (int e = 0; e < 4; ++e)
            if (take[e]) out[pos++] = i0 + e + add;
        base += take_tot;
        eq_seen += eq_tot;
    }
}

}  // namespace minf
