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

__global__ void __launch_bounds__(kTopkThreads) topk_rows_smem_kernel(const float *scores, int len, int k,
                                                                      int *out) {
    extern __shared__ float row[];
    __shared__ TopkShared sh;
    const float *x = scores + (size_t)blockIdx.x * len;
    for (int i = threadIdx.x * 4; i < len; i += kTopkThreads * 4) {
        if (i + 3 < len) {
            *reinterpret_cast<float4 *>(row + i) = __ldg(reinterpret_cast<const float4 *>(x + i));
        } else {
            for (int j = i; j < len; ++j) row[j] = x[j];
        }
    }
    __syncthreads();
    int *o = out + (size_t)blockIdx.x * k;
    block_topk_ascending<kTopkThreads, false>(row, len, k, o, 0, sh);
    for (int j = min(k, len) + (int)threadIdx.x; j < k; j += kTopkThreads) o[j] = -1;
}

// ---- multi-block path --------------------------------------------------------
struct RowState {
    uint32_t prefix, mask;
    int remaining;  // keys equal to the threshold still to take
    int pad;
};

__global__ void topk_init_kernel(RowState *st, uint32_t *hist, int rows, int len, int k) {
    const int r = blockIdx.x;
    for (int b = threadIdx.x; b < 256; b += blockDim.x) hist[(size_t)r * 256 + b] = 0u;
    if (threadIdx.x == 0) st[r] = RowState{0u, 0u, min(k, len), 0};
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
        const uint32_t active = __ballot_sync(0xffffffffu, hit);
        if (hit) {
            const uint32_t peers = __match_any_sync(active, bin);
            if ((int)(threadIdx.x & 31) == __ffs(peers) - 1) atomicAdd(&h[bin], __popc(peers));
        }
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
    const uint32_t t = st[r].prefix;
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
    const uint32_t t = st[r].prefix;
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
        for (int j = min(k, len) + (int)threadIdx.x; j < k; j += kChunkThreads) o[j] = -1;
}

}  // namespace

size_t topk_scratch_bytes(int n_rows, int len) {
    if (len <= kSmemRow) return 0;
    const int n_chunks = (len + kChunk - 1) / kChunk;
    return (size_t)n_rows * (sizeof(RowState) + 256 * sizeof(uint32_t) + 2 * (size_t)n_chunks * sizeof(int2)) + 1024;
}

cudaError_t run_topk_rows(const float *scores, int n_rows, int len, int k, int *out, void *scratch,
                          cudaStream_t st) {
    if (n_rows <= 0 || k <= 0) return cudaSuccess;
    if (len <= kSmemRow) {
        const int smem = len * (int)sizeof(float);
        cudaError_t e = cudaFuncSetAttribute(topk_rows_smem_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        topk_rows_smem_kernel<<<n_rows, kTopkThreads, smem, st>>>(scores, len, k, out);
        return cudaGetLastError();
    }
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
    topk_init_kernel<<<n_rows, 256, 0, st>>>(state, hist, n_rows, len, k);
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

}  // namespace minf
