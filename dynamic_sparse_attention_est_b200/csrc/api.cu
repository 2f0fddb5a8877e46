// api.cu -- the extern "C" entry points of minf.h: argument checks, workspace
// carving, TMA descriptors, and the launch sequence of each operation.
#include <cudaTypedefs.h>

#include <atomic>
#include <cstdarg>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace minf {

namespace {

thread_local std::string g_last_error;
std::atomic<unsigned long long> g_wait_limit_ns{2000000000ull};
// Vertical-Slash routing of sparse slash groups to the CUDA-core pass: a tile
// half is taken to cost this many offsets of that pass (0: tile kernel only).
std::atomic<float> g_vs_diag_ratio{1.0f};

int fail(int code, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return code;
}

int cuda_fail(cudaError_t e, const char *what) {
    return fail(MINF_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// ------------------------------------------------------------------ workspace
constexpr size_t kAlign = 256;

struct Carver {
    char *base;
    size_t off;
    explicit Carver(void *b, size_t start) : base(static_cast<char *>(b)), off(start) {}
    template <class T>
    T *take(size_t count) {
        off = (off + kAlign - 1) & ~(kAlign - 1);
        T *p = base ? reinterpret_cast<T *>(base + off) : nullptr;
        off += count * sizeof(T);
        return p;
    }
};

int qtiles(int n) { return (n + kTileM - 1) / kTileM; }

// Vertical-Slash tile kernel launch order: kv-head-major from this length on.
constexpr int kVsKvMajorFrom = 1 << 18;

// Vertical-Slash estimate: key chunking for one wave of one CTA per SM (148 SMs;
// the kernel's shared memory allows one CTA per SM), whole chunks per head pair.
void vs_est_geometry(int n, int n_pairs, int *n_chunks, int *chunk_tiles, int *n_ktiles) {
    const int kt = (n + 127) / 128;
    int want = 148 / std::max(1, n_pairs);
    want = std::max(1, std::min(want, kt));
    const int ct = (kt + want - 1) / want;
    *n_ktiles = kt;
    *chunk_tiles = ct;
    *n_chunks = (kt + ct - 1) / ct;
}

VsEstBufs carve_vs_est(Carver &c, int n, int n_heads, int n_pairs) {
    VsEstBufs b{};
    vs_est_geometry(n, n_pairs, &b.n_chunks, &b.chunk_tiles, &b.n_ktiles);
    int maxc = 0, ct, kt;
    vs_est_geometry(n, 1, &maxc, &ct, &kt);  // upper bound of n_chunks over pairings
    b.part = c.take<float2>((size_t)n_heads * maxc * 128);
    b.lse2 = c.take<float>((size_t)n_heads * 128);
    b.diag = c.take<float>((size_t)n_heads * b.n_ktiles * 191);
    b.vert = c.take<float>((size_t)n_heads * n);
    b.slash = c.take<float>((size_t)n_heads * n);
    b.topk_scratch = c.take<char>(topk_scratch_bytes(n_heads, n));
    b.diag0 = c.take<float>(n_heads);
    b.counts = c.take<int>(2 * (size_t)n_heads);
    b.topp_scratch = c.take<char>(topp_scratch_bytes(n_heads));
    return b;
}

VsPlanBufs carve_vs_plan(Carver &c, int n, int n_heads, int n_vertical, int n_slash) {
    VsPlanBufs b{};
    b.words = n / 32;
    b.stride = b.words + 2 * kBitGuard;
    b.vcap = std::min(n_vertical, n);
    b.scap = std::min(n_slash, n);
    const size_t nw = (size_t)n_heads * qtiles(n);
    b.bits_v = c.take<uint32_t>((size_t)n_heads * b.stride) + kBitGuard;
    b.bits_s = c.take<uint32_t>((size_t)n_heads * b.stride) + kBitGuard;
    b.vsorted = c.take<int>((size_t)n_heads * b.vcap);
    b.nvs = c.take<int>(n_heads);
    b.soff = c.take<int>((size_t)n_heads * b.scap);
    b.groups = c.take<int2>((size_t)n_heads * b.scap);
    b.ngroups = c.take<int>(n_heads);
    b.nsh = c.take<int>(nw);
    b.nvert = c.take<int>(nw);
    b.nle = c.take<int>(nw);
    b.vlist = c.take<int>(nw * b.vcap);
    b.dgroups = c.take<int4>((size_t)n_heads * b.scap);
    b.ndgroups = c.take<int>(n_heads);
    b.diag_ml = c.take<float2>((size_t)n_heads * n);
    b.diag_o = c.take<float>((size_t)n_heads * n * kD);
    return b;
}

int bs_head_batch(int n, int n_heads) {
    const size_t nb = (size_t)n / kBlock;
    const size_t per = nb * nb * sizeof(float);
    size_t hb = ((size_t)1 << 30) / std::max<size_t>(per, 1);
    hb = std::max<size_t>(1, std::min<size_t>(hb, (size_t)n_heads));
    return (int)hb;
}

BsEstBufs carve_bs_est(Carver &c, int hkv, int n, int n_heads) {
    BsEstBufs b{};
    const size_t nb = (size_t)n / kBlock;
    b.head_batch = bs_head_batch(n, n_heads);
    b.qs = c.take<__nv_bfloat16>((size_t)n_heads * 3 * nb * kD);
    b.ks = c.take<__nv_bfloat16>((size_t)hkv * 3 * nb * kD);
    b.scores = c.take<float>((size_t)b.head_batch * nb * nb);
    return b;
}

struct BsPlanBufs {
    int *plan, *cnt;
    int stride;
};

BsPlanBufs carve_bs_plan(Carver &c, int n, int n_heads, int topk) {
    BsPlanBufs b{};
    const int nb = n / kBlock;
    b.stride = 2 * std::min(topk, nb);
    const size_t nw = (size_t)n_heads * qtiles(n);
    b.plan = c.take<int>(nw * b.stride);
    b.cnt = c.take<int>(nw);
    return b;
}

// ------------------------------------------------------------------ devices
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;
std::mutex g_dev_mutex;
int g_dev_ok[64] = {0};  // 0 unknown, 1 sm_100, -1 other

int select_device(const void *ptr) {
    cudaPointerAttributes attr;
    cudaError_t e = cudaPointerGetAttributes(&attr, ptr);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return fail(MINF_ERR_CUDA, "cudaPointerGetAttributes: %s", cudaGetErrorString(e));
    }
    if (attr.type != cudaMemoryTypeDevice && attr.type != cudaMemoryTypeManaged)
        return fail(MINF_ERR_INVALID, "tensor pointer is not device memory");
    const int dev = attr.device;
    e = cudaSetDevice(dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaSetDevice");
    std::lock_guard<std::mutex> lk(g_dev_mutex);
    if (dev >= 0 && dev < 64 && g_dev_ok[dev] == 0) {
        cudaDeviceProp prop;
        e = cudaGetDeviceProperties(&prop, dev);
        if (e != cudaSuccess) return cuda_fail(e, "cudaGetDeviceProperties");
        g_dev_ok[dev] = prop.major == 10 ? 1 : -1;
    }
    if (dev < 0 || dev >= 64 || g_dev_ok[dev] != 1)
        return fail(MINF_ERR_UNSUPPORTED, "device %d is not an sm_100 (B200-class) GPU", dev);
    return MINF_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ------------------------------------------------------------------ checks
struct Common {
    int hq, hkv, n, n_heads;
    int ids[MINF_MAX_HEADS];
};

int check_common(const void *q, const void *k, int hq, int hkv, int n, int d, const int32_t *head_ids,
                 int n_heads, Common &c) {
    if (!q || !k) return fail(MINF_ERR_INVALID, "null q or k");
    if (hq <= 0 || hkv <= 0 || hq % hkv != 0) return fail(MINF_ERR_INVALID, "bad head counts hq=%d hkv=%d", hq, hkv);
    if (d != kD) return fail(MINF_ERR_UNSUPPORTED, "head dimension %d (only 128)", d);
    if (n <= 0 || n % kBlock != 0) return fail(MINF_ERR_UNSUPPORTED, "sequence length %d (positive multiple of 64)", n);
    if (n > (1 << 26)) return fail(MINF_ERR_UNSUPPORTED, "sequence length %d too large", n);
    if (!aligned16(q) || !aligned16(k)) return fail(MINF_ERR_INVALID, "q/k not 16-byte aligned");
    if (head_ids) {
        if (n_heads <= 0 || n_heads > MINF_MAX_HEADS) return fail(MINF_ERR_INVALID, "n_heads=%d", n_heads);
        for (int i = 0; i < n_heads; ++i) {
            if (head_ids[i] < 0 || head_ids[i] >= hq) return fail(MINF_ERR_INVALID, "head id %d out of range", head_ids[i]);
            c.ids[i] = head_ids[i];
        }
    } else {
        if (hq > MINF_MAX_HEADS) return fail(MINF_ERR_INVALID, "hq=%d above %d", hq, MINF_MAX_HEADS);
        n_heads = hq;
        for (int i = 0; i < hq; ++i) c.ids[i] = i;
    }
    c.hq = hq;
    c.hkv = hkv;
    c.n = n;
    c.n_heads = n_heads;
    return MINF_OK;
}

int check_scale(float scale) {
    if (!(scale > 0.f) || !std::isfinite(scale)) return fail(MINF_ERR_INVALID, "scale must be finite and > 0");
    return MINF_OK;
}

// One non-blocking side stream per device for the mixed layer, created on first use.
cudaError_t side_stream(cudaStream_t *out) {
    static std::mutex mu;
    static cudaStream_t streams[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (!streams[dev]) {
        e = cudaStreamCreateWithFlags(&streams[dev], cudaStreamNonBlocking);
        if (e != cudaSuccess) return e;
    }
    *out = streams[dev];
    return cudaSuccess;
}

int check_ws(void *ws, size_t ws_bytes, size_t need) {
    if (!ws) return fail(MINF_ERR_INVALID, "null workspace");
    if ((reinterpret_cast<uintptr_t>(ws) & (kAlign - 1)) != 0) return fail(MINF_ERR_INVALID, "workspace not 256-byte aligned");
    if (ws_bytes < need) return fail(MINF_ERR_WORKSPACE, "workspace %zu bytes, need %zu", ws_bytes, need);
    return MINF_OK;
}

// ------------------------------------------------------------------ ops
size_t bytes_vs_est(int hkv, int n, int n_heads) {
    Carver c(nullptr, MINF_STATUS_BYTES);
    carve_vs_est(c, n, n_heads, 1);
    (void)hkv;
    return c.off;
}
size_t bytes_vs_attn(int n, int n_heads, int nv, int ns) {
    Carver c(nullptr, MINF_STATUS_BYTES);
    carve_vs_plan(c, n, n_heads, nv, ns);
    return c.off;
}
size_t bytes_bs_est(int hkv, int n, int n_heads) {
    Carver c(nullptr, MINF_STATUS_BYTES);
    carve_bs_est(c, hkv, n, n_heads);
    return c.off;
}
size_t bytes_bs_attn(int n, int n_heads, int topk) {
    Carver c(nullptr, MINF_STATUS_BYTES);
    carve_bs_plan(c, n, n_heads, topk);
    return c.off;
}

void fill_attn_common(AttnParams &P, const Common &c, float scale, const void *k, const void *v, void *out,
                      float *lse, void *ws, bool slot_is_id, bool kv_major = false) {
    P.k = reinterpret_cast<const __nv_bfloat16 *>(k);
    P.v = reinterpret_cast<const __nv_bfloat16 *>(v);
    P.out = reinterpret_cast<__nv_bfloat16 *>(out);
    P.lse = lse;
    P.hdr = reinterpret_cast<WsHeader *>(ws);
    P.wait_limit_ns = g_wait_limit_ns.load();
    P.n = c.n;
    P.hq = c.hq;
    P.hkv = c.hkv;
    P.group = c.hq / c.hkv;
    P.n_heads = c.n_heads;
    P.n_qtiles = qtiles(c.n);
    P.scale_log2 = scale * 1.4426950408889634f;
    for (int i = 0; i < MINF_MAX_HEADS; ++i) {
        P.head_ids[i] = i < c.n_heads ? c.ids[i] : 0;
        P.out_slot[i] = i < c.n_heads ? (slot_is_id ? c.ids[i] : i) : 0;
    }
    // Launch order.  kv-head-major (the listed heads grouped by kv-head, stable) keeps
    // one kv-head's K and V in L2 while its tiles run: it takes the Block-Sparse 128K
    // layer from 79 GB of DRAM reads per launch to 2 GB (27.1 -> 24.5 ms).  The other
    // patterns measured no better (Vertical-Slash 32K about 5 % slower), so they keep
    // one group: every listed head side by side, heaviest query tiles first.
    int ng = 0, pos = 0;
    if (kv_major) {
        const int group = c.hq / c.hkv;
        for (int g = 0; g < c.hkv; ++g) {
            const int start = pos;
            for (int i = 0; i < c.n_heads; ++i)
                if (c.ids[i] / group == g) P.kv_order[pos++] = i;
            if (pos > start) P.kv_start[ng++] = start;
        }
    } else {
        for (int i = 0; i < c.n_heads; ++i) P.kv_order[pos++] = i;
        P.kv_start[ng++] = 0;
    }
    P.kv_start[ng] = pos;
    P.n_kvgroups = ng;
}

cudaError_t encode_attn_maps(AttnParams &P, const void *q, const void *k, const void *v, const Common &c) {
    cudaError_t e = make_tmap_3d(&P.tmap_q, q, c.hq, c.n);
    if (e == cudaSuccess) e = make_tmap_3d(&P.tmap_k, k, c.hkv, c.n);
    if (e == cudaSuccess) e = make_tmap_3d(&P.tmap_v, v, c.hkv, c.n);
    return e;
}

int reset_counters(void *ws, cudaStream_t st) {
    cudaError_t e = cudaMemsetAsync(static_cast<char *>(ws) + offsetof(WsHeader, tiles), 0,
                                    sizeof(WsHeader) - offsetof(WsHeader, tiles), st);
    return e == cudaSuccess ? MINF_OK : cuda_fail(e, "cudaMemsetAsync");
}

// The bodies below assume checked arguments; `scratch` is the workspace past
// the status header (or a sub-area of it in the mixed layer).
int do_vs_estimate(const Common &c, const void *q, const void *k, int last_q, int nv, int ns, float scale,
                   int32_t *v_idx, int32_t *s_idx, void *ws, char *scratch, cudaStream_t st, float p_v = 0.f,
                   float p_s = 0.f, int32_t *v_cnt = nullptr, int32_t *s_cnt = nullptr) {
    // count the pairs the estimate kernel will form
    const int group = c.hq / c.hkv;
    int n_pairs = 0;
    for (int g = 0; g < c.hkv; ++g) {
        int cnt = 0;
        for (int i = 0; i < c.n_heads; ++i) cnt += (c.ids[i] / group == g);
        n_pairs += (cnt + 1) / 2;
    }
    Carver cv(scratch, 0);
    VsEstBufs b = carve_vs_est(cv, c.n, c.n_heads, n_pairs);
    VsEstArgs a{};
    a.q = q;
    a.k = k;
    a.hq = c.hq;
    a.hkv = c.hkv;
    a.n = c.n;
    a.last_q = last_q;
    a.n_heads = c.n_heads;
    a.scale_log2 = scale * 1.4426950408889634f;
    a.head_ids = c.ids;
    a.n_vertical = nv;
    a.n_slash = ns;
    a.v_idx = v_idx;
    a.s_idx = s_idx;
    a.topp = p_v > 0.f;
    a.p_vertical = p_v;
    a.p_slash = p_s;
    a.v_cnt = v_cnt;
    a.s_cnt = s_cnt;
    a.hdr = ws;
    a.wait_limit_ns = g_wait_limit_ns.load();
    cudaError_t e = run_vs_estimate(a, b, st);
    return e == cudaSuccess ? MINF_OK : cuda_fail(e, "vs_estimate launch");
}

int do_vs_attention(const Common &c, const void *q, const void *k, const void *v, float scale, const int32_t *v_idx,
                    int nv, const int32_t *s_idx, int ns, void *out, float *lse, void *ws, char *scratch,
                    bool slot_is_id, cudaStream_t st, bool tiles = false) {
    Carver cv(scratch, 0);
    VsPlanBufs b = carve_vs_plan(cv, c.n, c.n_heads, nv, ns);
    // whole slash tiles attend every key of a computed range: no CUDA-core pass
    const float ratio = tiles ? 0.f : g_vs_diag_ratio.load();
    cudaError_t e = run_vs_plan(b, v_idx, nv, s_idx, ns, c.n, c.n_heads, qtiles(c.n), ratio, st);
    if (e != cudaSuccess) return cuda_fail(e, "vs plan launch");
    AttnParams P;
    memset(&P, 0, sizeof(P));
    // long sequences launch kv-head-major (one kv-head's q-heads side by side), so that
    // the CTAs in flight share that kv-head's K and V in L2 (at 32K heads side by side
    // measured faster)
    fill_attn_common(P, c, scale, k, v, out, lse, ws, slot_is_id, c.n >= kVsKvMajorFrom);
    e = encode_attn_maps(P, q, k, v, c);
    if (e != cudaSuccess) return cuda_fail(e, "tensor map");
    if (ratio > 0.f) {
        // the sparse slash groups first, on the CUDA cores; the tile kernel merges their state
        DiagParams D;
        memset(&D, 0, sizeof(D));
        D.tmap_k = P.tmap_k;
        D.tmap_v = P.tmap_v;
        D.q = reinterpret_cast<const __nv_bfloat16 *>(q);
        D.groups = b.dgroups;
        D.ngroups = b.ndgroups;
        D.gstride = b.scap;
        D.offs = b.soff;
        D.ostride = b.scap;
        D.bits_v = b.bits_v;
        D.bit_stride = b.stride;
        D.ml = b.diag_ml;
        D.o = b.diag_o;
        D.hdr = P.hdr;
        D.wait_limit_ns = P.wait_limit_ns;
        D.n = c.n;
        D.group = c.hq / c.hkv;
        D.n_heads = c.n_heads;
        D.n_qtiles = qtiles(c.n);
        D.scale_log2 = P.scale_log2;
        for (int i = 0; i < MINF_MAX_HEADS; ++i) D.head_ids[i] = P.head_ids[i];
        e = run_vs_diag(D, st);
        if (e != cudaSuccess) return cuda_fail(e, "vs sparse-slash launch");
        P.vs_ndgroups = b.ndgroups;
        P.vs_diag_ml = b.diag_ml;
        P.vs_diag_o = b.diag_o;
    }
    P.vs_groups = b.groups;
    P.vs_ngroups = b.ngroups;
    P.vs_gstride = b.scap;
    P.vs_vert = b.vlist;
    P.vs_nvert = b.nvert;
    P.vs_nsh = b.nsh;
    P.vs_nle = b.nle;
    P.vs_vstride = b.vcap;
    P.vs_bits_s = b.bits_s;
    P.vs_bits_v = b.bits_v;
    P.bit_stride = b.stride;
    P.vs_tiles = tiles ? 1 : 0;
    e = run_attention(PAT_VS, P, st);
    return e == cudaSuccess ? MINF_OK : cuda_fail(e, "vs attention launch");
}

int do_block_estimate(const Common &c, const void *q, const void *k, int topk, int32_t *blk_idx, int32_t *blk_cnt,
                      float *scores_out, void *ws, char *scratch, cudaStream_t st) {
    Carver cv(scratch, 0);
    BsEstBufs b = carve_bs_est(cv, c.hkv, c.n, c.n_heads);
    BsEstArgs a{};
    a.q = q;
    a.k = k;
    a.hq = c.hq;
    a.hkv = c.hkv;
    a.n = c.n;
    a.n_heads = c.n_heads;
    a.topk = topk;
    a.head_ids = c.ids;
    a.blk_idx = blk_idx;
    a.blk_cnt = blk_cnt;
    a.scores_out = scores_out;
    a.hdr = ws;
    a.wait_limit_ns = g_wait_limit_ns.load();
    cudaError_t e = run_block_estimate(a, b, st);
    return e == cudaSuccess ? MINF_OK : cuda_fail(e, "block_estimate launch");
}

int do_block_attention(const Common &c, const void *q, const void *k, const void *v, float scale,
                       const int32_t *blk_idx, const int32_t *blk_cnt, int topk, void *out, float *lse, void *ws,
                       char *scratch, bool slot_is_id, cudaStream_t st) {
    Carver cv(scratch, 0);
    BsPlanBufs b = carve_bs_plan(cv, c.n, c.n_heads, topk);
    cudaError_t e = run_bs_plan(blk_idx, blk_cnt, topk, c.n_heads, qtiles(c.n), c.n / kBlock, b.plan, b.cnt,
                                b.stride, st);
    if (e != cudaSuccess) return cuda_fail(e, "block plan launch");
    AttnParams P;
    memset(&P, 0, sizeof(P));
    fill_attn_common(P, c, scale, k, v, out, lse, ws, slot_is_id, true);
    e = encode_attn_maps(P, q, k, v, c);
    if (e != cudaSuccess) return cuda_fail(e, "tensor map");
    P.bs_plan = b.plan;
    P.bs_cnt = b.cnt;
    P.bs_stride = b.stride;
    e = run_attention(PAT_BLOCK, P, st);
    return e == cudaSuccess ? MINF_OK : cuda_fail(e, "block attention launch");
}

int do_static_attention(int pattern, const Common &c, const void *q, const void *k, const void *v, float scale,
                        int n_sink, int window, int n_last, void *out, float *lse, void *ws, bool slot_is_id,
                        cudaStream_t st) {
    AttnParams P;
    memset(&P, 0, sizeof(P));
    fill_attn_common(P, c, scale, k, v, out, lse, ws, slot_is_id);
    cudaError_t e = encode_attn_maps(P, q, k, v, c);
    if (e != cudaSuccess) return cuda_fail(e, "tensor map");
    P.n_sink = n_sink;
    P.window = window;
    P.n_last = n_last;
    e = run_attention(pattern, P, st);
    return e == cudaSuccess ? MINF_OK : cuda_fail(e, "attention launch");
}

}  // namespace

// The driver's tensor-map encoder, looked up once.
PFN_cuTensorMapEncodeTiled_v12000 tmap_encoder() {
    std::call_once(g_encode_once, [] {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult qres;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &qres) ==
                cudaSuccess &&
            qres == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    });
    return g_encode;
}

// TMA descriptor of a bf16 [heads][n][128] tensor, box {64, 64, 1}, 128-byte swizzle.
cudaError_t make_tmap_3d(CUtensorMap *map, const void *base, int heads, int n) {
    if (!tmap_encoder()) return cudaErrorNotSupported;
    const cuuint64_t dims[3] = {(cuuint64_t)kD, (cuuint64_t)n, (cuuint64_t)heads};
    const cuuint64_t strides[2] = {(cuuint64_t)kD * 2, (cuuint64_t)n * kD * 2};
    const cuuint32_t box[3] = {64, 64, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides,
                                box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// TMA descriptor of an fp32 [z][y][x] tensor (row stride x floats, a multiple of
// 4), box {32, 32, 1}, 128-byte swizzle: the score tiles' store path.
cudaError_t make_tmap_f32_3d(CUtensorMap *map, const void *base, int x, int y, int z) {
    if (!tmap_encoder()) return cudaErrorNotSupported;
    const cuuint64_t dims[3] = {(cuuint64_t)x, (cuuint64_t)y, (cuuint64_t)z};
    const cuuint64_t strides[2] = {(cuuint64_t)x * 4, (cuuint64_t)x * y * 4};
    const cuuint32_t box[3] = {32, 32, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void *>(base), dims, strides,
                                box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                                CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

namespace {
__global__ void wait_timeout_kernel(WsHeader *hdr, unsigned long long limit_ns) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bar), 1);  // nothing ever arrives on it
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        const WaitCtl wc{&abort_flag, &hdr->status, limit_ns};
        wait_bounded(smem_u32(&bar), 0, wc);
    }
}
}  // namespace

cudaError_t run_wait_timeout_check(void *hdr, unsigned long long limit_ns, cudaStream_t st) {
    wait_timeout_kernel<<<1, 32, 0, st>>>(reinterpret_cast<WsHeader *>(hdr), limit_ns);
    return cudaGetLastError();
}

}  // namespace minf

using namespace minf;

extern "C" {

size_t minf_workspace_bytes(int op, int hq, int hkv, int n, int n_heads, int p1, int p2, int p3) {
    if (hq <= 0 || hkv <= 0 || hq % hkv || n <= 0 || n % kBlock) return 0;
    if (n_heads <= 0) n_heads = hq;
    switch (op) {
    case MINF_OP_VS_ESTIMATE:
        return bytes_vs_est(hkv, n, n_heads);
    case MINF_OP_VS_ATTENTION:
        if (p1 < 1 || p2 < 1) return 0;
        return bytes_vs_attn(n, n_heads, p1, p2);
    case MINF_OP_BLOCK_ESTIMATE:
        return bytes_bs_est(hkv, n, n_heads);
    case MINF_OP_BLOCK_ATTENTION:
        if (p1 < 1) return 0;
        return bytes_bs_attn(n, n_heads, p1);
    case MINF_OP_ASHAPE_ATTENTION:
    case MINF_OP_TRISHAPE_ATTENTION:
    case MINF_OP_DENSE_ATTENTION:
        return MINF_STATUS_BYTES;
    case MINF_OP_MIXED_LAYER: {
        if (p1 < 1 || p2 < 1 || p3 < 1) return 0;
        const int nb = n / kBlock;
        Carver c(nullptr, MINF_STATUS_BYTES);
        c.take<int>((size_t)hq * p1);
        c.take<int>((size_t)hq * p2);
        c.take<int>((size_t)hq * nb * p3);
        c.take<int>((size_t)hq * nb);
        // Vertical-Slash and Block-Sparse work run side by side: one scratch region each
        c.take<char>(std::max(bytes_vs_est(hkv, n, hq), bytes_vs_attn(n, hq, p1, p2)));
        c.take<char>(std::max(bytes_bs_est(hkv, n, hq), bytes_bs_attn(n, hq, p3)));
        return c.off;
    }
    }
    return 0;
}

int minf_vs_estimate(const minf_bf16 *q, const minf_bf16 *k, int hq, int hkv, int n, int d, int last_q,
                     int n_vertical, int n_slash, float scale, const int32_t *head_ids, int n_heads,
                     int32_t *v_idx, int32_t *s_idx, void *ws, size_t ws_bytes, minf_stream_t stream) {
    Common c;
    int rc = check_common(q, k, hq, hkv, n, d, head_ids, n_heads, c);
    if (rc) return rc;
    if ((rc = check_scale(scale))) return rc;
    if (!v_idx || !s_idx) return fail(MINF_ERR_INVALID, "null v_idx or s_idx");
    if (n_vertical < 1 || n_slash < 1) return fail(MINF_ERR_INVALID, "budgets must be >= 1");
    if (last_q < 1) return fail(MINF_ERR_INVALID, "last_q must be >= 1");
    if (last_q > 64) return fail(MINF_ERR_UNSUPPORTED, "last_q %d above 64", last_q);
    if ((rc = check_ws(ws, ws_bytes, bytes_vs_est(hkv, n, c.n_heads)))) return rc;
    if ((rc = select_device(q))) return rc;
    return do_vs_estimate(c, q, k, last_q, n_vertical, n_slash, scale, v_idx, s_idx, ws,
                          static_cast<char *>(ws) + MINF_STATUS_BYTES, (cudaStream_t)stream);
}

int minf_vs_estimate_topp(const minf_bf16 *q, const minf_bf16 *k, int hq, int hkv, int n, int d, int last_q,
                          int n_vertical, int n_slash, float p_vertical, float p_slash, float scale,
                          const int32_t *head_ids, int n_heads, int32_t *v_idx, int32_t *s_idx, int32_t *v_cnt,
                          int32_t *s_cnt, void *ws, size_t ws_bytes, minf_stream_t stream) {
    Common c;
    int rc = check_common(q, k, hq, hkv, n, d, head_ids, n_heads, c);
    if (rc) return rc;
    if ((rc = check_scale(scale))) return rc;
    if (!v_idx || !s_idx) return fail(MINF_ERR_INVALID, "null v_idx or s_idx");
    if (n_vertical < 1 || n_slash < 1) return fail(MINF_ERR_INVALID, "caps must be >= 1");
    if (!(p_vertical > 0.f && p_vertical <= 1.f) || !(p_slash > 0.f && p_slash <= 1.f))
        return fail(MINF_ERR_INVALID, "p must be in (0, 1]");
    if (last_q < 1) return fail(MINF_ERR_INVALID, "last_q must be >= 1");
    if (last_q > 64) return fail(MINF_ERR_UNSUPPORTED, "last_q %d above 64", last_q);
    if (n > (1 << 20)) return fail(MINF_ERR_UNSUPPORTED, "top-p rows above 2^20 keys");
    if ((rc = check_ws(ws, ws_bytes, bytes_vs_est(hkv, n, c.n_heads)))) return rc;
    if ((rc = select_device(q))) return rc;
    return do_vs_estimate(c, q, k, last_q, n_vertical, n_slash, scale, v_idx, s_idx, ws,
                          static_cast<char *>(ws) + MINF_STATUS_BYTES, (cudaStream_t)stream, p_vertical, p_slash,
                          v_cnt, s_cnt);
}

static int vs_attention_entry(const minf_bf16 *q, const minf_bf16 *k, const minf_bf16 *v, int hq, int hkv,
                              int n, int d, float scale, const int32_t *head_ids, int n_heads,
                              const int32_t *v_idx, int n_vertical, const int32_t *s_idx, int n_slash,
                              minf_bf16 *out, float *lse, void *ws, size_t ws_bytes, minf_stream_t stream,
                              bool tiles) {
    Common c;
    int rc = check_common(q, k, hq, hkv, n, d, head_ids, n_heads, c);
    if (rc) return rc;
    if ((rc = check_scale(scale))) return rc;
    if (!v || !out || !v_idx || !s_idx) return fail(MINF_ERR_INVALID, "null v, out or index rows");
    if (!aligned16(v) || !aligned16(out)) return fail(MINF_ERR_INVALID, "v/out not 16-byte aligned");
    if (n_vertical < 1 || n_slash < 1) return fail(MINF_ERR_INVALID, "budgets must be >= 1");
    if ((rc = check_ws(ws, ws_bytes, bytes_vs_attn(n, c.n_heads, n_vertical, n_slash)))) return rc;
    if ((rc = select_device(q))) return rc;
    if ((rc = reset_counters(ws, (cudaStream_t)stream))) return rc;
    return do_vs_attention(c, q, k, v, scale, v_idx, n_vertical, s_idx, n_slash, out, lse, ws,
                           static_cast<char *>(ws) + MINF_STATUS_BYTES, false, (cudaStream_t)stream, tiles);
}

int minf_vs_attention(const minf_bf16 *q, const minf_bf16 *k, const minf_bf16 *v, int hq, int hkv, int n, int d,
                      float scale, const int32_t *head_ids, int n_heads, const int32_t *v_idx, int n_vertical,
                      const int32_t *s_idx, int n_slash, minf_bf16 *out, float *lse, void *ws, size_t ws_bytes,
                      minf_stream_t stream) {
    return vs_attention_entry(q, k, v, hq, hkv, n, d, scale, head_ids, n_heads, v_idx, n_vertical, s_idx, n_slash,
                              out, lse, ws, ws_bytes, stream, false);
}

int minf_vs_attention_tiles(const minf_bf16 *q, const minf_bf16 *k, const minf_bf16 *v, int hq, int hkv, int n,
                            int d, float scale, const int32_t *head_ids, int n_heads, const int32_t *v_idx,
                            int n_vertical, const int32_t *s_idx, int n_slash, minf_bf16 *out, float *lse, void *ws,
                            size_t ws_bytes, minf_stream_t stream) {
    return vs_attention_entry(q, k, v, hq, hkv, n, d, scale, head_ids, n_heads, v_idx, n_vertical, s_idx, n_slash,
                              out, lse, ws, ws_bytes, stream, true);
}

int minf_block_estimate(const minf_bf16 *q, const minf_bf16 *k, int hq, int hkv, int n, int d, int block, int topk,
                        const int32_t *head_ids, int n_heads, int32_t *blk_idx, int32_t *blk_cnt, void *ws,
                        size_t ws_bytes, minf_stream_t stream) {
    Common c;
    int rc = check_common(q, k, hq, hkv, n, d, head_ids, n_heads, c);
    if (rc) return rc;
    if (block != kBlock) return fail(MINF_ERR_UNSUPPORTED, "block %d (only 64)", block);
    if (!blk_idx || !blk_cnt) return fail(MINF_ERR_INVALID, "null blk_idx or blk_cnt");
    if (topk < 1) return fail(MINF_ERR_INVALID, "topk must be >= 1");
    if (n / kBlock > 32768) return fail(MINF_ERR_UNSUPPORTED, "more than 32768 blocks");
    if ((rc = check_ws(ws, ws_bytes, bytes_bs_est(hkv, n, c.n_heads)))) return rc;
    if ((rc = select_device(q))) return rc;
    return do_block_estimate(c, q, k, topk, blk_idx, blk_cnt, nullptr, ws,
                             static_cast<char *>(ws) + MINF_STATUS_BYTES, (cudaStream_t)stream);
}

int minf_block_scores(const minf_bf16 *q, const minf_bf16 *k, int hq, int hkv, int n, int d, int block,
                      const int32_t *head_ids, int n_heads, float *scores, void *ws, size_t ws_bytes,
                      minf_stream_t stream) {
    Common c;
    int rc = check_common(q, k, hq, hkv, n, d, head_ids, n_heads, c);
    if (rc) return rc;
    if (block != kBlock) return fail(MINF_ERR_UNSUPPORTED, "block %d (only 64)", block);
    if (!scores) return fail(MINF_ERR_INVALID, "null scores");
    if (n / kBlock > 32768) return fail(MINF_ERR_UNSUPPORTED, "more than 32768 blocks");
    if ((rc = check_ws(ws, ws_bytes, bytes_bs_est(hkv, n, c.n_heads)))) return rc;
    if ((rc = select_device(q))) return rc;
    return do_block_estimate(c, q, k, 1, nullptr, nullptr, scores, ws, static_cast<char *>(ws) + MINF_STATUS_BYTES,
                             (cudaStream_t)stream);
}

int minf_block_attention(const minf_bf16 *q, const minf_bf16 *k, const minf_bf16 *v, int hq, int hkv, int n, int d,
                         float scale, const int32_t *head_ids, int n_heads, const int32_t *blk_idx,
                         const int32_t *blk_cnt, int topk, minf_bf16 *out, float *lse, void *ws, size_t ws_bytes,
                         minf_stream_t stream) {
    Common c;
    int rc = check_common(q, k, hq, hkv, n, d, head_ids, n_heads, c);
    if (rc) return rc;
    if ((rc = check_scale(scale))) return rc;
    if (!v || !out || !blk_idx || !blk_cnt) return fail(MINF_ERR_INVALID, "null v, out or block rows");
    if (!aligned16(v) || !aligned16(out)) return fail(MINF_ERR_INVALID, "v/out not 16-byte aligned");
    if (topk < 1) return fail(MINF_ERR_INVALID, "topk must be >= 1");
    if ((rc = check_ws(ws, ws_bytes, bytes_bs_attn(n, c.n_heads, topk)))) return rc;
    if ((rc = select_device(q))) return rc;
    if ((rc = reset_counters(ws, (cudaStream_t)stream))) return rc;
    return do_block_attention(c, q, k, v, scale, blk_idx, blk_cnt, topk, out, lse, ws,
                              static_cast<char *>(ws) + MINF_STATUS_BYTES, false, (cudaStream_t)stream);
}

int minf_ashape_attention(const minf_bf16 *q, const minf_bf16 *k, const minf_bf16 *v, int hq, int hkv, int n, int d,
                          float scale, const int32_t *head_ids, int n_heads, int n_sink, int window, minf_bf16 *out,
                          float *lse, void *ws, size_t ws_bytes, minf_stream_t stream) {
    Common c;
    int rc = check_common(q, k, hq, hkv, n, d, head_ids, n_heads, c);
    if (rc) return rc;
    if ((rc = check_scale(scale))) return rc;
    if (!v || !out) return fail(MINF_ERR_INVALID, "null v or out");
    if (!aligned16(v) || !aligned16(out)) return fail(MINF_ERR_INVALID, "v/out not 16-byte aligned");
    if (n_sink < 0 || window < 1) return fail(MINF_ERR_INVALID, "n_sink >= 0 and window >= 1 required");
    if ((rc = check_ws(ws, ws_bytes, MINF_STATUS_BYTES))) return rc;
    if ((rc = select_device(q))) return rc;
    if ((rc = reset_counters(ws, (cudaStream_t)stream))) return rc;
    return do_static_attention(PAT_ASHAPE, c, q, k, v, scale, n_sink, window, 0, out, lse, ws, false,
                               (cudaStream_t)stream);
}

int minf_trishape_attention(const minf_bf16 *q, const minf_bf16 *k, const minf_bf16 *v, int hq, int hkv, int n,
                            int d, float scale, const int32_t *head_ids, int n_heads, int n_sink, int window,
                            int n_last, minf_bf16 *out, float *lse, void *ws, size_t ws_bytes,
                            minf_stream_t stream) {
    Common c;
    int rc = check_common(q, k, hq, hkv, n, d, head_ids, n_heads, c);
    if (rc) return rc;
    if ((rc = check_scale(scale))) return rc;
    if (!v || !out) return fail(MINF_ERR_INVALID, "null v or out");
    if (!aligned16(v) || !aligned16(out)) return fail(MINF_ERR_INVALID, "v/out not 16-byte aligned");
    if (n_sink < 0 || window < 1 || n_last < 0)
        return fail(MINF_ERR_INVALID, "n_sink >= 0, window >= 1 and n_last >= 0 required");
    if ((rc = check_ws(ws, ws_bytes, MINF_STATUS_BYTES))) return rc;
    if ((rc = select_device(q))) return rc;
    if ((rc = reset_counters(ws, (cudaStream_t)stream))) return rc;
    return do_static_attention(PAT_ASHAPE, c, q, k, v, scale, n_sink, window, n_last, out, lse, ws, false,
                               (cudaStream_t)stream);
}

int minf_dense_attention(const minf_bf16 *q, const minf_bf16 *k, const minf_bf16 *v, int hq, int hkv, int n, int d,
                         float scale, const int32_t *head_ids, int n_heads, minf_bf16 *out, float *lse, void *ws,
                         size_t ws_bytes, minf_stream_t stream) {
    Common c;
    int rc = check_common(q, k, hq, hkv, n, d, head_ids, n_heads, c);
    if (rc) return rc;
    if ((rc = check_scale(scale))) return rc;
    if (!v || !out) return fail(MINF_ERR_INVALID, "null v or out");
    if (!aligned16(v) || !aligned16(out)) return fail(MINF_ERR_INVALID, "v/out not 16-byte aligned");
    if ((rc = check_ws(ws, ws_bytes, MINF_STATUS_BYTES))) return rc;
    if ((rc = select_device(q))) return rc;
    if ((rc = reset_counters(ws, (cudaStream_t)stream))) return rc;
    return do_static_attention(PAT_DENSE, c, q, k, v, scale, 0, 1, 0, out, lse, ws, false, (cudaStream_t)stream);
}

int minf_mixed_layer(const minf_bf16 *q, const minf_bf16 *k, const minf_bf16 *v, int hq, int hkv, int n, int d,
                     float scale, const int8_t *head_pattern, int last_q, int n_vertical, int n_slash, int topk,
                     int n_sink, int window, minf_bf16 *out, float *lse, void *ws, size_t ws_bytes,
                     minf_stream_t stream) {
    Common all;
    int rc = check_common(q, k, hq, hkv, n, d, nullptr, hq, all);
    if (rc) return rc;
    if ((rc = check_scale(scale))) return rc;
    if (!v || !out || !head_pattern) return fail(MINF_ERR_INVALID, "null v, out or head_pattern");
    if (!aligned16(v) || !aligned16(out)) return fail(MINF_ERR_INVALID, "v/out not 16-byte aligned");
    if (n_vertical < 1 || n_slash < 1 || topk < 1 || last_q < 1 || n_sink < 0 || window < 1)
        return fail(MINF_ERR_INVALID, "bad pattern parameters");
    if (last_q > 64) return fail(MINF_ERR_UNSUPPORTED, "last_q %d above 64", last_q);
    if (n / kBlock > 32768) return fail(MINF_ERR_UNSUPPORTED, "more than 32768 blocks");
    Common sub[5];
    for (int p = 0; p < 5; ++p) {
        sub[p] = all;
        sub[p].n_heads = 0;
    }
    for (int h = 0; h < hq; ++h) {
        const int p = head_pattern[h];
        if (p < 0 || p > 4) return fail(MINF_ERR_INVALID, "head %d: pattern code %d", h, p);
        sub[p].ids[sub[p].n_heads++] = h;
    }
    const size_t need = minf_workspace_bytes(MINF_OP_MIXED_LAYER, hq, hkv, n, hq, n_vertical, n_slash, topk);
    if ((rc = check_ws(ws, ws_bytes, need))) return rc;
    if ((rc = select_device(q))) return rc;
    cudaStream_t st = (cudaStream_t)stream;
    if ((rc = reset_counters(ws, st))) return rc;
    const int nb = n / kBlock;
    Carver c(ws, MINF_STATUS_BYTES);
    int32_t *v_idx = c.take<int32_t>((size_t)hq * n_vertical);
    int32_t *s_idx = c.take<int32_t>((size_t)hq * n_slash);
    int32_t *blk_idx = c.take<int32_t>((size_t)hq * nb * topk);
    int32_t *blk_cnt = c.take<int32_t>((size_t)hq * nb);
    char *scratch_vs = c.take<char>(std::max(bytes_vs_est(hkv, n, hq), bytes_vs_attn(n, hq, n_vertical, n_slash)));
    char *scratch_bs = c.take<char>(std::max(bytes_bs_est(hkv, n, hq), bytes_bs_attn(n, hq, topk)));
    // Two streams (the caller's and a library side stream that starts after the
    // work already queued on it): Vertical-Slash estimate and attention, then
    // A-shape and Tri-shape on the caller's; Block-Sparse estimate and attention,
    // then dense on the side stream, so each group's estimate overlaps the other
    // group's attention.  The caller's stream waits for the side stream at the end.
    cudaStream_t side = nullptr;
    cudaEvent_t ev_start = nullptr, ev_side = nullptr;
    const bool two = (sub[PAT_BLOCK].n_heads || sub[PAT_DENSE].n_heads) &&
                     (sub[PAT_VS].n_heads || sub[PAT_ASHAPE].n_heads || sub[MINF_PATTERN_TRISHAPE].n_heads);
    if (two) {
        cudaError_t e = side_stream(&side);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ev_start, cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ev_side, cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventRecord(ev_start, st);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(side, ev_start, 0);
        if (e != cudaSuccess) {
            if (ev_start) cudaEventDestroy(ev_start);
            if (ev_side) cudaEventDestroy(ev_side);
            return cuda_fail(e, "side stream");
        }
    }
    cudaStream_t st2 = two ? side : st;
    int rc2 = MINF_OK;
    if (sub[PAT_VS].n_heads) {
        rc = do_vs_estimate(sub[PAT_VS], q, k, last_q, n_vertical, n_slash, scale, v_idx, s_idx, ws, scratch_vs, st);
        if (!rc)
            rc = do_vs_attention(sub[PAT_VS], q, k, v, scale, v_idx, n_vertical, s_idx, n_slash, out, lse, ws,
                                 scratch_vs, true, st);
    }
    if (sub[PAT_BLOCK].n_heads) {
        rc2 = do_block_estimate(sub[PAT_BLOCK], q, k, topk, blk_idx, blk_cnt, nullptr, ws, scratch_bs, st2);
        if (!rc2)
            rc2 = do_block_attention(sub[PAT_BLOCK], q, k, v, scale, blk_idx, blk_cnt, topk, out, lse, ws,
                                     scratch_bs, true, st2);
    }
    if (!rc && sub[PAT_ASHAPE].n_heads)
        rc = do_static_attention(PAT_ASHAPE, sub[PAT_ASHAPE], q, k, v, scale, n_sink, window, 0, out, lse, ws, true,
                                 st);
    if (!rc && sub[MINF_PATTERN_TRISHAPE].n_heads)
        rc = do_static_attention(PAT_ASHAPE, sub[MINF_PATTERN_TRISHAPE], q, k, v, scale, n_sink, window, last_q, out,
                                 lse, ws, true, st);
    if (!rc2 && sub[PAT_DENSE].n_heads)
        rc2 = do_static_attention(PAT_DENSE, sub[PAT_DENSE], q, k, v, scale, 0, 1, 0, out, lse, ws, true, st2);
    if (two) {
        // join even after a failed launch: nothing may stay queued behind the caller's back
        cudaError_t e = cudaEventRecord(ev_side, side);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(st, ev_side, 0);
        cudaEventDestroy(ev_start);
        cudaEventDestroy(ev_side);
        if (e != cudaSuccess && !rc && !rc2) return cuda_fail(e, "side stream join");
    }
    return rc ? rc : rc2;
}

int minf_status(void *ws, minf_stream_t stream) {
    if (!ws) return fail(MINF_ERR_INVALID, "null workspace");
    cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    int st[2] = {0, 0};
    e = cudaMemcpy(st, ws, sizeof(st), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy status");
    if (st[0] != 0) {
        fail(st[0], "device wait gave up at site 0x%08x (role %d, barrier %d, tile %d)", st[1],
             (st[1] >> 24) & 0x3f, (st[1] >> 16) & 0xff, st[1] & 0xffff);
        e = cudaMemset(ws, 0, sizeof(st));
        if (e != cudaSuccess) return cuda_fail(e, "cudaMemset status");
    }
    return st[0];
}

int minf_stats(void *ws, minf_stream_t stream, uint64_t *tiles, uint64_t *pairs) {
    if (!ws || !tiles || !pairs) return fail(MINF_ERR_INVALID, "null argument");
    cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    WsHeader h;
    e = cudaMemcpy(&h, ws, sizeof(h), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy stats");
    *tiles = h.tiles;
    *pairs = h.pairs;
    return MINF_OK;
}

int minf_stats_detail(void *ws, minf_stream_t stream, uint64_t *out, int n_out) {
    if (!ws || !out || n_out < 0) return fail(MINF_ERR_INVALID, "null argument");
    cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    WsHeader h;
    e = cudaMemcpy(&h, ws, sizeof(h), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy stats");
    const uint64_t v[7] = {h.tiles, h.pairs, h.pat_tiles[PAT_DENSE], h.pat_tiles[PAT_VS], h.pat_tiles[PAT_BLOCK],
                           h.pat_tiles[PAT_ASHAPE], h.diag_pairs};
    const int n = n_out < 7 ? n_out : 7;
    for (int i = 0; i < n; ++i) out[i] = v[i];
    return n;
}

void minf_set_wait_limit_ns(uint64_t ns) { g_wait_limit_ns.store(ns ? ns : 2000000000ull); }

void minf_set_vs_diag_ratio(float ratio) { g_vs_diag_ratio.store(ratio > 0.f ? ratio : 0.f); }

int minf_check_wait_timeout(void *ws, size_t ws_bytes, uint64_t limit_ns, minf_stream_t stream) {
    int rc = check_ws(ws, ws_bytes, MINF_STATUS_BYTES);
    if (rc) return rc;
    if ((rc = select_device(ws))) return rc;
    cudaError_t e = run_wait_timeout_check(ws, limit_ns, (cudaStream_t)stream);
    return e == cudaSuccess ? MINF_OK : cuda_fail(e, "wait check launch");
}

int minf_selftest_exp2(const float *x, float *y_poly, float *y_hw, int n, minf_stream_t stream) {
    if (!x || !y_poly || !y_hw || n < 0) return fail(MINF_ERR_INVALID, "bad self-test arguments");
    int rc = select_device(x);
    if (rc) return rc;
    cudaError_t e = run_exp2_selftest(x, y_poly, y_hw, n, (cudaStream_t)stream);
    return e == cudaSuccess ? MINF_OK : cuda_fail(e, "exp2 self-test launch");
}

const char *minf_version(void) { return "minf-b200 0.1.0 (sm_100a)"; }

const char *minf_last_error(void) { return g_last_error.c_str(); }

}  // extern "C"

// ---------------------------------------------------------------------------
// Vertical-Slash estimate without a caller workspace.
//
// Some callers cannot allocate device memory at the point where they estimate
// indices -- for example code running inside a caller's own memory-managed
// runtime or a capture region where cudaMalloc is not allowed, or an embedding
// that has no allocator at all.  For them this entry point takes its scratch
// from one file-scope device array of kNoAllocScratchBytes, which every GPU
// that loads the library holds until the process exits.  Requests whose
// scratch would exceed it are rejected with MINF_ERR_WORKSPACE.
//
// The array's device address is looked up by the first call made on a device
// in a given CUDA context (with that device current) and kept for that
// context; a call from another context, or after the context was reset, looks
// it up again, since the module and its array may then sit elsewhere.  Make
// the first call before any stream capture.  Every call shares the array:
// calls whose work overlaps on the GPU (different streams, or different host
// threads, with no ordering between them) race on it.  The status block at
// its start is cleared by each call and read back (and cleared) by
// minf_vs_estimate_noalloc_status.
namespace minf {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;  // 32 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Context identity through driver entry points (the library links no libcuda).
PFN_cuCtxGetCurrent_v4000 g_ctx_current = nullptr;
PFN_cuCtxGetId_v12000 g_ctx_id = nullptr;
std::once_flag g_ctx_once;

// Id of the context current on this thread, or 0 if it cannot be told.
unsigned long long current_ctx_id() {
    std::call_once(g_ctx_once, [] {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult qres;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &fn, 4000, cudaEnableDefault, &qres) ==
                cudaSuccess &&
            qres == cudaDriverEntryPointSuccess)
            g_ctx_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(fn);
        fn = nullptr;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &fn, 12000, cudaEnableDefault, &qres) == cudaSuccess &&
            qres == cudaDriverEntryPointSuccess)
            g_ctx_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(fn);
    });
    if (!g_ctx_current || !g_ctx_id) return 0;
    CUcontext ctx = nullptr;
    if (g_ctx_current(&ctx) != CUDA_SUCCESS || !ctx) return 0;
    unsigned long long id = 0;
    return g_ctx_id(ctx, &id) == CUDA_SUCCESS ? id : 0;
}

struct NoAllocSlot {
    unsigned long long ctx;  // context the address belongs to (0: none cached)
    void *ptr;
};
std::mutex g_noalloc_mutex;
NoAllocSlot g_noalloc[64] = {};

// Device address of the built-in array on device `dev`, which must be current.
int noalloc_scratch(int dev, void **out) {
    std::lock_guard<std::mutex> lk(g_noalloc_mutex);
    if (dev < 0 || dev >= 64) return fail(MINF_ERR_UNSUPPORTED, "device %d out of range", dev);
    const unsigned long long ctx = current_ctx_id();
    NoAllocSlot &slot = g_noalloc[dev];
    if (ctx == 0 || slot.ctx != ctx || !slot.ptr) {
        void *p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(scratch)");
        slot.ctx = ctx;  // 0 (context unknown) caches nothing: the next call looks it up again
        slot.ptr = p;
    }
    *out = slot.ptr;
    return MINF_OK;
}

// Makes `device` current and returns the built-in array on it.
int noalloc_on_device(int device, void **out) {
    int count = 0;
    cudaError_t e = cudaGetDeviceCount(&count);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDeviceCount");
    if (device < 0 || device >= count) return fail(MINF_ERR_INVALID, "device %d out of range", device);
    e = cudaSetDevice(device);
    if (e != cudaSuccess) return cuda_fail(e, "cudaSetDevice");
    return noalloc_scratch(device, out);
}

}  // namespace
}  // namespace minf

extern "C" int minf_vs_estimate_noalloc(const minf_bf16 *q, const minf_bf16 *k, int hq, int hkv, int n, int d,
                                        int last_q, int n_vertical, int n_slash, float scale,
                                        const int32_t *head_ids, int n_heads, int32_t *v_idx, int32_t *s_idx,
                                        minf_stream_t stream) {
    Common c;
    int rc = check_common(q, k, hq, hkv, n, d, head_ids, n_heads, c);
    if (rc) return rc;
    if ((rc = check_scale(scale))) return rc;
    if (!v_idx || !s_idx) return fail(MINF_ERR_INVALID, "null v_idx or s_idx");
    if (n_vertical < 1 || n_slash < 1) return fail(MINF_ERR_INVALID, "budgets must be >= 1");
    if (last_q < 1) return fail(MINF_ERR_INVALID, "last_q must be >= 1");
    if (last_q > 64) return fail(MINF_ERR_UNSUPPORTED, "last_q %d above 64", last_q);
    const size_t need = bytes_vs_est(hkv, n, c.n_heads);
    if (need > kNoAllocScratchBytes)
        return fail(MINF_ERR_WORKSPACE, "needs %zu bytes of scratch; the built-in area holds %zu", need,
                    kNoAllocScratchBytes);
    if ((rc = select_device(q))) return rc;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    void *ws = nullptr;
    if ((rc = noalloc_scratch(dev, &ws))) return rc;
    cudaStream_t st = (cudaStream_t)stream;
    e = cudaMemsetAsync(ws, 0, MINF_STATUS_BYTES, st);  // status block starts at zero
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(status)");
    return do_vs_estimate(c, q, k, last_q, n_vertical, n_slash, scale, v_idx, s_idx, ws,
                          static_cast<char *>(ws) + MINF_STATUS_BYTES, st);
}

extern "C" int minf_vs_estimate_noalloc_status(int device, minf_stream_t stream) {
    void *ws = nullptr;
    int rc = noalloc_on_device(device, &ws);
    if (rc) return rc;
    return minf_status(ws, stream);  // waits for `stream`, reads and clears the status word
}

extern "C" int minf_vs_estimate_noalloc_check_timeout(int device, uint64_t limit_ns, minf_stream_t stream) {
    void *ws = nullptr;
    int rc = noalloc_on_device(device, &ws);
    if (rc) return rc;
    const cudaError_t e = run_wait_timeout_check(ws, limit_ns, (cudaStream_t)stream);
    return e == cudaSuccess ? MINF_OK : cuda_fail(e, "wait check launch");
}
