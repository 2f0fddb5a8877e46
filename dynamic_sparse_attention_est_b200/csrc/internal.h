// internal.h -- host-side declarations shared by the library's translation units.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>

namespace minf {

struct AttnParams;

// Launch timing (minf_profile_enable): while enabled, an event pair around the
// scope's launches on `st`, read back by minf_profile_read.
class ProfScope {
  public:
    ProfScope(const char *name, cudaStream_t st);
    ~ProfScope();
    ProfScope(const ProfScope &) = delete;
    ProfScope &operator=(const ProfScope &) = delete;

  private:
    cudaStream_t st_;
    cudaEvent_t end_;
};

// Device buffers of the Vertical-Slash tile plan (all inside the workspace).
struct VsPlanBufs {
    uint32_t *bits_v, *bits_s;  // head hp's n bits at + hp * stride, kBitGuard zero words on each side
    int words, stride;          // n / 32, words + 2 * kBitGuard
    int *vsorted, *nvs;         // [n_heads][vcap], [n_heads]
    int vcap;
    int *soff;                  // [n_heads][scap]
    int2 *groups;               // [n_heads][scap] slash groups of the tile kernel
    int *ngroups;               // [n_heads]
    int4 *dgroups;              // [n_heads][scap] slash groups of the CUDA-core pass
    int *ndgroups;              // [n_heads]
    int scap;
    int *nsh, *nvert, *nle;     // [n_work]
    int *vlist;                 // [n_work][vcap]
    float2 *diag_ml;            // [n_heads][n] partial (m, l) of the CUDA-core pass
    float *diag_o;              // [n_heads][n][128] its unnormalised O
};

// 3D TMA map over a bf16 [heads][n][128] tensor: box {64, 64, 1}, 128B swizzle.
cudaError_t make_tmap_3d(CUtensorMap *map, const void *base, int heads, int n);
cudaError_t make_tmap_f32_3d(CUtensorMap *map, const void *base, int x, int y, int z);

cudaError_t run_attention(int pattern, const AttnParams &P, cudaStream_t st);
cudaError_t run_bs_plan(const int *blk_idx, const int *blk_cnt, int topk, int n_heads, int n_qtiles, int nb,
                        int *plan, int *cnt, int stride, cudaStream_t st);
cudaError_t run_vs_plan(const VsPlanBufs &b, const int *v_idx, int n_vertical, const int *s_idx, int n_slash,
                        int n, int n_heads, int n_qtiles, float diag_ratio, cudaStream_t st);
struct DiagParams;
cudaError_t run_vs_diag(const DiagParams &P, cudaStream_t st);

// Vertical-Slash estimation.
struct VsEstBufs {
    float2 *part;   // [n_pairs][n_chunks][128] running (max, sum) per row, log2 domain
    float *lse2;    // [n_pairs][128]
    float *diag;    // [n_heads][n_ktiles][191] per key-tile diagonal partial sums
    float *vert;    // [n_heads][n]
    float *slash;   // [n_heads][n]
    void *topk_scratch;  // topk_scratch_bytes(n_heads, n)
    float *diag0;   // [n_heads] mass of offset 0 (its slash entry is forced to +inf)
    int *counts;    // [2][n_heads] top-p counts when the caller keeps none
    void *topp_scratch;  // topp_scratch_bytes(n_heads)
    int n_chunks, chunk_tiles, n_ktiles;
};

struct VsEstArgs {
    const void *q, *k;     // bf16
    int hq, hkv, n, last_q, n_heads;
    float scale_log2;
    const int *head_ids;   // host, n_heads entries
    int n_vertical, n_slash;
    int *v_idx, *s_idx;
    bool topp;             // budgets by mass: p_vertical / p_slash, n_vertical / n_slash as caps
    float p_vertical, p_slash;
    int *v_cnt, *s_cnt;    // device, nullable: the top-p counts
    void *hdr;             // WsHeader*
    unsigned long long wait_limit_ns;
};

cudaError_t run_vs_estimate(const VsEstArgs &a, const VsEstBufs &b, cudaStream_t st);

// Block-Sparse estimation.
struct BsEstBufs {
    __nv_bfloat16 *qs;  // [n_heads][3][nb][128] pooled Q as hi, mid, lo bf16 parts
    __nv_bfloat16 *ks;  // [hkv][3][nb][128]
    float *scores;      // [head_batch][nb][nb]
    int head_batch;
};

struct BsEstArgs {
    const void *q, *k;
    int hq, hkv, n, n_heads, topk;
    const int *head_ids;  // host
    int *blk_idx, *blk_cnt;
    float *scores_out;    // when set: the pooled scores of every listed head go here, no selection
    void *hdr;            // WsHeader*
    unsigned long long wait_limit_ns;
};

cudaError_t run_block_estimate(const BsEstArgs &a, const BsEstBufs &b, cudaStream_t st);

// Self-test of the attention kernel's exponentials (polynomial and MUFU).
cudaError_t run_exp2_selftest(const float *x, float *y_poly, float *y_hw, int n, cudaStream_t st);

// Self-test of the bounded wait.
cudaError_t run_wait_timeout_check(void *hdr, unsigned long long limit_ns, cudaStream_t st);

// Top-k (largest first, ties to the lower index) of n_rows rows of `len`
// non-negative floats each; writes min(k, len) indices ascending, -1 padded to k.
// Rows longer than the one-block limit need topk_scratch_bytes(n_rows, len)
// bytes of device scratch (256-byte aligned); shorter rows need none.
// With k_row (device, n_rows entries) row r keeps min(k_row[r], k) keys.
size_t topk_scratch_bytes(int n_rows, int len);
cudaError_t run_topk_rows(const float *scores, int n_rows, int len, int k, int *out, void *scratch,
                          cudaStream_t st, const int *k_row = nullptr);
// Two row sets of the same length (each with its own k, k_row and output) in
// one launch when the rows fit the one-block path, else one after the other.
struct TopkRows {
    const float *scores;
    int n_rows, k;
    int *out;
    const int *k_row;
};
cudaError_t run_topk_rows2(const TopkRows &a, const TopkRows &b, int len, void *scratch, cudaStream_t st);

// Top-p counts (device, n_rows entries, each at most cap): the fewest keys of a
// row, best first, whose scores reach p of the row's mass; with skip0 key 0 is
// left out and extra0[r] counts first (the count then includes that entry).
// scratch: topp_scratch_bytes(n_rows) bytes of device memory, 256-byte aligned.
size_t topp_scratch_bytes(int n_rows);
cudaError_t run_topp_counts(const float *scores, int n_rows, int len, bool skip0, const float *extra0, float p,
                            int cap, int *count, void *scratch, cudaStream_t st);
// Two row sets of the same length in one launch when the rows fit the
// one-block path (same counts as run_topp_counts), else one after the other.
cudaError_t run_topp_counts2(const float *scores_a, int n_rows_a, bool skip0_a, const float *extra0_a, float p_a,
                             int cap_a, int *count_a, const float *scores_b, int n_rows_b, bool skip0_b,
                             const float *extra0_b, float p_b, int cap_b, int *count_b, int len, void *scratch,
                             cudaStream_t st);

}  // namespace minf
