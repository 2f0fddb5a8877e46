// topk.cu -- block-wide radix select: the k largest of a row (ties to the lower
// index), written as ascending indices.  Used for the vertical keys and slash
// offsets of Vertical-Slash (rows of n floats in HBM) and, through the same
// device routines, for the per-query-block rows of Block-Sparse.
//
// A float maps to an unsigned key with the same order (non-negative floats as
// their bits; signed floats with the usual sign flip).  Four 8-bit digit passes
// find the k-th largest key t and how many keys equal to t are needed; a final
// ordered compaction keeps every key > t and the first needed keys == t.
#include "common.cuh"
#include "internal.h"
#include "topk.cuh"

namespace minf {

namespace {

constexpr int kTopkThreads = 1024;

__global__ void __launch_bounds__(kTopkThreads) topk_rows_kernel(const float *scores, int len, int k,
                                                                 int *out) {
    __shared__ TopkShared sh;
    const float *x = scores + (size_t)blockIdx.x * len;
    int *o = out + (size_t)blockIdx.x * k;
    block_topk_ascending<kTopkThreads, false>(x, len, k, o, 0, sh);
    for (int j = min(k, len) + (int)threadIdx.x; j < k; j += kTopkThreads) o[j] = -1;
}

}  // namespace

cudaError_t run_topk_rows(const float *scores, int n_rows, int len, int k, int *out, cudaStream_t st) {
    if (n_rows <= 0) return cudaSuccess;
    topk_rows_kernel<<<n_rows, kTopkThreads, 0, st>>>(scores, len, k, out);
    return cudaGetLastError();
}

}  // namespace minf
