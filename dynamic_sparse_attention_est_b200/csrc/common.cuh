// common.cuh -- definitions shared by the kernels and the host launchers.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "minf.h"

namespace minf {

constexpr int kD = 128;        // head dimension
constexpr int kTileM = 128;    // query rows per tile
constexpr int kHalf = 64;      // keys per half-tile (a tile is two halves)
constexpr int kBlock = 64;     // Block-Sparse block size / Vertical-Slash row granularity
// Zero words on each side of a head's Vertical-Slash bitmap, so that a 64-bit
// window starting up to 6 words before the first word or ending 2 words past the
// last one reads zeros without a bounds check.
constexpr int kBitGuard = 8;

// Workspace header: status word + counters, first 256 bytes of every workspace.
struct WsHeader {
    int status;
    int site;  // where the first bounded wait gave up: role << 24 | barrier << 16 | tile
    unsigned long long tiles;
    unsigned long long pairs;
    unsigned long long pat_tiles[4];  // tiles by attention kernel pattern (PAT_*)
    unsigned long long diag_pairs;    // pairs of the CUDA-core sparse-slash pass (included in pairs)
};
static_assert(sizeof(WsHeader) <= MINF_STATUS_BYTES, "header fits the status block");

enum : int { PAT_DENSE = MINF_PATTERN_DENSE, PAT_VS = MINF_PATTERN_VS, PAT_BLOCK = MINF_PATTERN_BLOCK,
             PAT_ASHAPE = MINF_PATTERN_ASHAPE };

// One half-tile of 64 keys: a contiguous key range (TMA), a list of gathered
// keys (vertical lines outside every slash range), or nothing.
enum : int { HALF_EMPTY = 0, HALF_RANGE = 1, HALF_GATHER = 2 };
enum : int { HF_FULL = 1, HF_ROWS0 = 2, HF_ROWS1 = 4 };

struct HalfDesc {
    int kind;
    int ks;     // first key (range) or offset into the work item's vertical list (gather)
    int len;    // valid keys, 1..64
    int flags;  // HF_*
};

struct AttnParams {
    CUtensorMap tmap_q;  // [hq][n][128] bf16, box {64, 64, 1}, 128B swizzle
    CUtensorMap tmap_k;  // [hkv][n][128]
    CUtensorMap tmap_v;
    const __nv_bfloat16 *k;
    const __nv_bfloat16 *v;
    __nv_bfloat16 *out;
    float *lse;
    WsHeader *hdr;
    unsigned long long wait_limit_ns;
    int n, hq, hkv, group;
    int n_heads, n_qtiles;
    float scale_log2;
    // A-shape / Tri-shape (n_last > 0: the last n_last query rows attend densely)
    int n_sink, window, n_last;
    // Block-Sparse plan: per work item (hp * n_qtiles + t), up to bs_stride half entries
    const int *bs_plan;
    const int *bs_cnt;
    int bs_stride;
    // Vertical-Slash plan
    const int2 *vs_groups;    // per head: merged slash-offset groups (lo, hi), ascending
    const int *vs_ngroups;    // per head
    int vs_gstride;
    const int *vs_vert;       // per work item: gathered vertical keys, ascending
    const int *vs_nvert;      // per work item
    const int *vs_nsh;        // per work item: number of slash half-tiles
    const int *vs_nle;        // per work item: gathered keys at or before the tile's first row
    int vs_tiles;             // 1: slash ranges attended whole (causal mask only)
    int vs_vstride;
    const uint32_t *vs_bits_s;  // per head: bitmap of slash offsets (head hp at hp * bit_stride)
    const uint32_t *vs_bits_v;  // per head: bitmap of vertical keys
    int bit_stride;             // words per head, kBitGuard zero words on each side included
    // Vertical-Slash pairs of the sparse slash groups, computed beforehand on the
    // CUDA cores (null: none): per query row of each listed head, (m, l) in the
    // log2 domain and the unnormalised O, merged in the epilogue
    const int *vs_ndgroups;     // per head: its number of such groups (0: nothing to merge)
    const float2 *vs_diag_ml;   // [n_heads][n]
    const float *vs_diag_o;     // [n_heads][n][128], read only where l > 0
    int head_ids[MINF_MAX_HEADS];
    int out_slot[MINF_MAX_HEADS];  // output row block of each listed head (its position, or its id)
    // Launch order: the listed heads in n_kvgroups groups, taken one group after
    // the other; inside a group the heaviest query tiles first, its heads side by
    // side.  Grouped by kv-head, the CTAs in flight share that kv-head's K and V
    // in L2; a single group is the plain heaviest-first order.
    int n_kvgroups;
    int kv_order[MINF_MAX_HEADS];       // head positions sorted by kv-head
    int kv_start[MINF_MAX_HEADS + 1];   // kv_order index where each group starts
};

// The CUDA-core pass over the sparse slash groups of Vertical-Slash.
struct DiagParams {
    CUtensorMap tmap_k;  // [hkv][n][128], box {64, 64, 1}, 128B swizzle
    CUtensorMap tmap_v;
    const __nv_bfloat16 *q;
    const int4 *groups;       // per head: (first offset, last offset, index of the first in offs, count), ascending
    const int *ngroups;       // per head
    int gstride;
    const int *offs;          // per head: the sorted distinct slash offsets
    int ostride;
    const uint32_t *bits_v;   // per head: bitmap of vertical keys
    int bit_stride;
    float2 *ml;               // [n_heads][n] (m, l), log2 domain
    float *o;                 // [n_heads][n][128] unnormalised, written where l > 0
    WsHeader *hdr;
    unsigned long long wait_limit_ns;
    int n, group, n_heads, n_qtiles;
    float scale_log2;
    int head_ids[MINF_MAX_HEADS];
};

// Bits [start, start + 64) of a bitmap of nbits bits; positions outside
// [0, nbits) read as 0.
__device__ __forceinline__ uint64_t bits64_at(const uint32_t *bm, int nwords, int start) {
    const int w0 = start >> 5;  // floor division (arithmetic shift)
    const int sh = start & 31;
    uint32_t w[3];
#pragma unroll
    for (int i = 0; i < 3; ++i) {
        const int wi = w0 + i;
        w[i] = (wi >= 0 && wi < nwords) ? __ldg(bm + wi) : 0u;
    }
    const uint32_t lo = __funnelshift_r(w[0], w[1], sh);
    const uint32_t hi = __funnelshift_r(w[1], w[2], sh);
    return (uint64_t)lo | ((uint64_t)hi << 32);
}

// Mask with bits [0, x) set, clamped to [0, 64].
__device__ __forceinline__ uint64_t low_bits(int x) {
    return x <= 0 ? 0ull : (x >= 64 ? ~0ull : ((1ull << x) - 1ull));
}

}  // namespace minf
