// bs_estimate.cu -- Block-Sparse index estimation on sm_100a.
//
// News article "单卡A100实现百万token推理，速度快10倍，这是微软官方的大模型推理加速",
// section 方法介绍: Q and K are mean-pooled and the pooled matrices multiplied;
// because mean pooling commutes with the product, the pooled score estimates the
// block-mean of the attention logits, and the best key blocks of each query
// block are kept.  Here:
//   pool    Qp[h][b] = mean of the 64 rows of block b (fp32), Kp[g][b] likewise;
//   score   s_ij = Qp_i . Kp_j for j <= i, fp32 FMA (bf16 tensor cores would
//           round the pooled values and move indices across ties);
//   top-k   diagonal block i always kept, the best topk-1 of j < i by radix
//           select (ties to the lower j), ascending.
#include "common.cuh"
#include "internal.h"
#include "topk.cuh"

namespace minf {

namespace {

struct HeadList {
    int ids[MINF_MAX_HEADS];
};

// One warp per 64-row block: lane l sums columns 4l..4l+3 in fp32.  With
// `listed`, slot s pools q-head hl.ids[s]; otherwise slot s pools head s.
__global__ void pool_kernel(const __nv_bfloat16 *x, const __grid_constant__ HeadList hl, bool listed,
                            int n_rows_heads, int n, float *out) {
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
    float4 res = make_float4(acc[0] * (1.f / kBlock), acc[1] * (1.f / kBlock), acc[2] * (1.f / kBlock),
                             acc[3] * (1.f / kBlock));
    *reinterpret_cast<float4 *>(out + ((size_t)slot * nb + b) * kD + lane * 4) = res;
}

// Pooled-score tiles: 128 x 128 (i, j) per CTA, lower triangle only (the CTA's
// index enumerates the tiles jt <= it), 256 threads with an 8 x 8 register
// tile each (rows ty*4+u and 64+ty*4+u, columns tx*4+v and 64+tx*4+v), d in
// chunks of 32 staged transposed in shared memory.  Per d step a thread reads
// four 16-byte vectors for 64 FMAs, one byte per FMA: the shared-memory
// bandwidth matches the fp32 FMA rate.
constexpr int kSt = 128;        // tile edge
constexpr int kDc = 32;         // d per stage
constexpr int kLd = kSt + 4;    // padded row of the transposed tiles (4 mod 32 banks)

__global__ void __launch_bounds__(256) pooled_scores_kernel(const float *qp, const float *kp,
                                                            const __grid_constant__ HeadList hl, int group,
                                                            int hp0, int nb, float *scores) {
    // tile t of the lower triangle: it (it + 1) / 2 <= t < (it + 1) (it + 2) / 2
    const int t = blockIdx.x, hb = blockIdx.y;
    int it = (int)((sqrtf(8.f * (float)t + 1.f) - 1.f) * 0.5f);
    while ((it + 1) * (it + 2) / 2 <= t) ++it;
    while (it * (it + 1) / 2 > t) --it;
    const int jt = t - it * (it + 1) / 2;
    __shared__ __align__(16) float As[kDc * kLd];
    __shared__ __align__(16) float Bs[kDc * kLd];
    const int hp = hp0 + hb;
    const float *A = qp + (size_t)hp * nb * kD;
    const float *B = kp + (size_t)(hl.ids[hp] / group) * nb * kD;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;
    float acc[8][8];
#pragma unroll
    for (int u = 0; u < 8; ++u)
#pragma unroll
        for (int v = 0; v < 8; ++v) acc[u][v] = 0.f;
    for (int d0 = 0; d0 < kD; d0 += kDc) {
        // a warp stores a 4-row x 8-d patch: its 32 words land in 32 different banks
        // (4 d + row mod 32), and each row's 8 floats are one 32-byte sector in global memory
        for (int patch = warp; patch < (kSt / 4) * (kDc / 8); patch += 8) {
            const int row = (patch / (kDc / 8)) * 4 + (lane & 3), d = (patch % (kDc / 8)) * 8 + (lane >> 2);
            const int gi = it * kSt + row, gj = jt * kSt + row;
            As[d * kLd + row] = gi < nb ? A[(size_t)gi * kD + d0 + d] : 0.f;
            Bs[d * kLd + row] = gj < nb ? B[(size_t)gj * kD + d0 + d] : 0.f;
        }
        __syncthreads();
#pragma unroll 4
        for (int d = 0; d < kDc; ++d) {
            const float4 a0 = *reinterpret_cast<const float4 *>(As + d * kLd + ty * 4);
            const float4 a1 = *reinterpret_cast<const float4 *>(As + d * kLd + 64 + ty * 4);
            const float4 b0 = *reinterpret_cast<const float4 *>(Bs + d * kLd + tx * 4);
            const float4 b1 = *reinterpret_cast<const float4 *>(Bs + d * kLd + 64 + tx * 4);
            const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
            const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
            for (int u = 0; u < 8; ++u)
#pragma unroll
                for (int v = 0; v < 8; ++v) acc[u][v] = fmaf(av[u], bv[v], acc[u][v]);
        }
        __syncthreads();
    }
    float *S = scores + (size_t)hb * nb * nb;
    const bool vec = (nb & 3) == 0;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
        const int gi = it * kSt + (u >> 2) * 64 + ty * 4 + (u & 3);
        if (gi >= nb) continue;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int gj = jt * kSt + h * 64 + tx * 4;
            float *dst = S + (size_t)gi * nb + gj;
            if (vec && gj + 3 < nb) {
                *reinterpret_cast<float4 *>(dst) =
                    make_float4(acc[u][4 * h], acc[u][4 * h + 1], acc[u][4 * h + 2], acc[u][4 * h + 3]);
            } else {
#pragma unroll
                for (int v = 0; v < 4; ++v)
                    if (gj + v < nb) dst[v] = acc[u][4 * h + v];
            }
        }
    }
}

constexpr int kRowThreads = 256;

// Row i of one head: the diagonal block plus the best topk-1 blocks j < i.
__global__ void __launch_bounds__(kRowThreads) block_topk_kernel(const float *scores, int nb, int topk, int hp0,
                                                                 int *blk_idx, int *blk_cnt) {
    extern __shared__ float row[];
    __shared__ TopkShared sh;
    const int i = blockIdx.x, hb = blockIdx.y;
    const int hp = hp0 + hb;
    const float *src = scores + ((size_t)hb * nb + i) * nb;
    for (int j = threadIdx.x; j < i; j += kRowThreads) row[j] = src[j];
    __syncthreads();
    int *o = blk_idx + ((size_t)hp * nb + i) * topk;
    const int take = min(topk - 1, i);
    block_topk_ascending<kRowThreads, true>(row, i, topk - 1, o, 0, sh);
    __syncthreads();
    if (threadIdx.x == 0) {
        o[take] = i;
        blk_cnt[(size_t)hp * nb + i] = take + 1;
    }
    for (int j = take + 1 + (int)threadIdx.x; j < topk; j += kRowThreads) o[j] = -1;
}

}  // namespace

cudaError_t run_block_estimate(const BsEstArgs &a, const BsEstBufs &b, cudaStream_t st) {
    const int nb = a.n / kBlock;
    const int group = a.hq / a.hkv;
    HeadList hl;
    for (int i = 0; i < MINF_MAX_HEADS; ++i) hl.ids[i] = i < a.n_heads ? a.head_ids[i] : 0;
    // pooled Q of the listed heads, pooled K of every kv-head
    ProfScope prof("bs_estimate (pool, scores, top-k)", st);
    const int warps = a.n_heads * nb;
    pool_kernel<<<(warps + 7) / 8, 256, 0, st>>>(reinterpret_cast<const __nv_bfloat16 *>(a.q), hl, true, a.n_heads,
                                                 a.n, b.qp);
    const int warps_k = a.hkv * nb;
    pool_kernel<<<(warps_k + 7) / 8, 256, 0, st>>>(reinterpret_cast<const __nv_bfloat16 *>(a.k), hl, false, a.hkv,
                                                   a.n, b.kp);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int smem_row = nb * (int)sizeof(float);
    e = cudaFuncSetAttribute(block_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_row);
    if (e != cudaSuccess) return e;
    const int tiles = (nb + kSt - 1) / kSt;
    const int tri = tiles * (tiles + 1) / 2;
    for (int hp0 = 0; hp0 < a.n_heads; hp0 += b.head_batch) {
        const int hbn = min(b.head_batch, a.n_heads - hp0);
        pooled_scores_kernel<<<dim3(tri, hbn), 256, 0, st>>>(b.qp, b.kp, hl, group, hp0, nb, b.scores);
        block_topk_kernel<<<dim3(nb, hbn), kRowThreads, smem_row, st>>>(b.scores, nb, a.topk, hp0, a.blk_idx,
                                                                       a.blk_cnt);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace minf
