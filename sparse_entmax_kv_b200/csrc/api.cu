// api.cu -- the C ABI declared in include/entmaxkv.h: argument checks (all on
// the host, before any CUDA call), workspace carving, TMA descriptor set-up,
// and the per-device status word.
#include <cudaTypedefs.h>

#include <cmath>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "internal.h"

using namespace ekv;

namespace {

__device__ int g_status;  // ENTMAXKV_STATUS_* bits, one word per device

constexpr int MAX_DEV = 64;
std::mutex g_mu;
DevInfo g_dev[MAX_DEV];
bool g_dev_ok[MAX_DEV];

int device_info(DevInfo *out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEV) return ENTMAXKV_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_dev_ok[dev]) {
        DevInfo d{};
        if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return ENTMAXKV_ERR_CUDA;
        if (cudaGetSymbolAddress(reinterpret_cast<void **>(&d.status), g_status) != cudaSuccess)
            return ENTMAXKV_ERR_CUDA;
        g_dev[dev] = d;
        g_dev_ok[dev] = true;
    }
    *out = g_dev[dev];
    return ENTMAXKV_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

int get_encoder() {
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_encode) return ENTMAXKV_OK;
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || fn == nullptr)
        return ENTMAXKV_ERR_CUDA;
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    return ENTMAXKV_OK;
}

// 2-D view of a paged cache: rows = num_blocks*Hkv*P tokens, d bf16 columns;
// box = 64 columns x P rows, 128-byte swizzle (conflict-free ldmatrix reads).
// The last few descriptors are kept, keyed by (address, geometry): a cache
// passed again gets its descriptor without a driver call.
struct MapEntry {
    const void *base;
    int d, rows, P;
    CUtensorMap map;
};
MapEntry g_maps[16];
int g_nmaps = 0, g_next_map = 0;

int make_kv_map_uncached(CUtensorMap *m, const void *base, const entmaxkv_shape *s);

int make_kv_map(CUtensorMap *m, const void *base, const entmaxkv_shape *s) {
    const int rows = s->num_blocks * s->Hkv * s->page_size;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        for (int i = 0; i < g_nmaps; ++i)
            if (g_maps[i].base == base && g_maps[i].d == s->d && g_maps[i].rows == rows &&
                g_maps[i].P == s->page_size) {
                *m = g_maps[i].map;
                return ENTMAXKV_OK;
            }
    }
    int rc = make_kv_map_uncached(m, base, s);
    if (rc) return rc;
    std::lock_guard<std::mutex> lk(g_mu);
    MapEntry &e = g_maps[g_next_map];
    e.base = base;
    e.d = s->d;
    e.rows = rows;
    e.P = s->page_size;
    e.map = *m;
    g_next_map = (g_next_map + 1) % 16;
    if (g_nmaps < 16) ++g_nmaps;
    return ENTMAXKV_OK;
}

int make_kv_map_uncached(CUtensorMap *m, const void *base, const entmaxkv_shape *s) {
    int rc = get_encoder();
    if (rc) return rc;
    cuuint64_t dims[2] = {(cuuint64_t)s->d, (cuuint64_t)s->num_blocks * s->Hkv * s->page_size};
    cuuint64_t strides[1] = {(cuuint64_t)s->d * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)s->page_size};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? ENTMAXKV_OK : ENTMAXKV_ERR_CUDA;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

constexpr int MAX_SEL_PAGES = 196608;

int check_shape(const entmaxkv_shape *s) {
    if (!s) return ENTMAXKV_ERR_NULL;
    if (s->B < 1 || s->Hq < 1 || s->Hkv < 1 || s->max_pages < 1 || s->num_blocks < 1) return ENTMAXKV_ERR_SHAPE;
    if (s->Hq % s->Hkv) return ENTMAXKV_ERR_SHAPE;
    const int G = s->Hq / s->Hkv;
    if (G != 1 && G != 2 && G != 4 && G != 8) return ENTMAXKV_ERR_SHAPE;
    if (s->d != 64 && s->d != 128) return ENTMAXKV_ERR_SHAPE;
    if (s->page_size != 16 && s->page_size != 32 && s->page_size != 64) return ENTMAXKV_ERR_SHAPE;
    if ((long long)s->max_pages * s->page_size >= (1ll << 31)) return ENTMAXKV_ERR_SHAPE;
    if ((long long)s->num_blocks * s->Hkv * s->page_size >= (1ll << 31)) return ENTMAXKV_ERR_SHAPE;
    if (s->B > 65535 || s->Hq > 65535 || (long long)s->B * s->Hq >= (1ll << 31)) return ENTMAXKV_ERR_SHAPE;
    if (s->kv_begin < 0 || s->kv_begin >= s->Hkv || s->kv_count < 0 || s->kv_begin + s->kv_count > s->Hkv)
        return ENTMAXKV_ERR_SHAPE;
    return ENTMAXKV_OK;
}

// The call's kv-head range [kv0, kv0 + nk) (check_shape has accepted s).
void kv_range(const entmaxkv_shape *s, int *kv0, int *nk) {
    *kv0 = s->kv_begin;
    *nk = s->kv_count ? s->kv_count : s->Hkv - s->kv_begin;
}

// 1/(alpha-1) when it is an integer in 1..8, else 0.
int integer_r(float alpha) {
    const double r = 1.0 / ((double)alpha - 1.0);
    const double ri = std::floor(r + 0.5);
    if (ri >= 1.0 && ri <= 8.0 && std::fabs(r - ri) <= 1e-5 * ri) return (int)ri;
    return 0;
}

int cuda_rc(cudaError_t e) { return e == cudaSuccess ? ENTMAXKV_OK : ENTMAXKV_ERR_CUDA; }

// Thread 0 waits on an mbarrier of its own that nothing arrives at (no copy
// is in flight), through the bounded wait every pipelined kernel uses, with
// the given limit; it sets ENTMAXKV_STATUS_TIMEOUT when the limit passes.
__global__ void wait_selftest_kernel(unsigned long long limit_ns, int *status) {
    __shared__ uint64_t bar;
    if (threadIdx.x != 0) return;
    mbar_init(&bar, 1);
    mbar_fence_init();
    mbar_wait_for(&bar, 0, status, limit_ns);
}

}  // namespace

extern "C" {

const char *entmaxkv_strerror(int code) {
    switch (code) {
        case ENTMAXKV_OK: return "ok";
        case ENTMAXKV_ERR_NULL: return "a required pointer is NULL";
        case ENTMAXKV_ERR_SHAPE: return "shape out of range or inconsistent";
        case ENTMAXKV_ERR_ALPHA: return "alpha out of range for this call";
        case ENTMAXKV_ERR_POLICY: return "unknown selection policy, k < 1, or delta not finite";
        case ENTMAXKV_ERR_WORKSPACE: return "workspace missing or too small";
        case ENTMAXKV_ERR_CUDA: return "CUDA runtime or driver error";
        case ENTMAXKV_ERR_UNSUPPORTED: return "valid arguments that the library does not support";
        case ENTMAXKV_ERR_ALIGN: return "pointer not 16-byte aligned";
        case ENTMAXKV_ERR_TOO_LARGE:
            return "problem needs more scratch than the fixed array of entmaxkv_decode_sparse_static";
        default: return "unknown error code";
    }
}

int entmaxkv_version(void) { return 100; }

size_t entmaxkv_meta_bytes(const entmaxkv_shape *s) {
    if (check_shape(s)) return 0;
    return (size_t)s->B * s->Hkv * meta_tiles(s->max_pages) * META_TILE * 12 * s->d;
}

size_t entmaxkv_workspace_size(const entmaxkv_shape *s, int call) {
    if (check_shape(s)) return (size_t)-1;
    switch (call) {
        case ENTMAXKV_CALL_SELECT: return 0;
        case ENTMAXKV_CALL_DECODE_SPARSE:
        case ENTMAXKV_CALL_DECODE_DENSE:
            return decode_ws_bytes(call == ENTMAXKV_CALL_DECODE_DENSE, s->B, s->Hq, s->Hkv, s->d, s->page_size,
                                   s->max_pages, nullptr, nullptr);
        case ENTMAXKV_CALL_DECODE_STEP:
            return decode_ws_bytes(false, s->B, s->Hq, s->Hkv, s->d, s->page_size, s->max_pages, nullptr, nullptr,
                                   true);
        default: return (size_t)-1;
    }
}

int entmaxkv_get_status(int32_t *status_out, int clear, void *stream) {
    if (!status_out) return ENTMAXKV_ERR_NULL;
    DevInfo di;
    int rc = device_info(&di);
    if (rc) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int v = 0;
    if (cudaMemcpyAsync(&v, di.status, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess)
        return ENTMAXKV_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return ENTMAXKV_ERR_CUDA;
    if (clear && cudaMemsetAsync(di.status, 0, sizeof(int), st) != cudaSuccess) return ENTMAXKV_ERR_CUDA;
    *status_out = v;
    return ENTMAXKV_OK;
}

int entmaxkv_selftest_wait(uint64_t limit_ns, void *stream) {
    if (limit_ns == 0 || limit_ns > WAIT_LIMIT_NS) return ENTMAXKV_ERR_SHAPE;
    DevInfo di;
    int rc = device_info(&di);
    if (rc) return rc;
    wait_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(limit_ns, di.status);
    return cuda_rc(cudaGetLastError());
}

int entmaxkv_build_meta(const entmaxkv_shape *s, const void *k_cache, const int32_t *page_table,
                        const int32_t *seq_lens, int32_t first_page, int32_t n_pages, void *meta, void *stream) {
    int rc = check_shape(s);
    if (rc) return rc;
    if (!k_cache || !page_table || !seq_lens || !meta) return ENTMAXKV_ERR_NULL;
    if (!aligned16(k_cache) || !aligned16(meta)) return ENTMAXKV_ERR_ALIGN;
    if (first_page < 0 || first_page > s->max_pages || n_pages < -1) return ENTMAXKV_ERR_SHAPE;
    int n = n_pages < 0 ? s->max_pages - first_page : n_pages;
    if (first_page + n > s->max_pages) n = s->max_pages - first_page;
    DevInfo di;
    if ((rc = device_info(&di))) return rc;
    MetaArgs a{};
    a.k = static_cast<const uint16_t *>(k_cache);
    a.page_table = page_table;
    a.seq_lens = seq_lens;
    a.meta = static_cast<uint8_t *>(meta);
    a.n_tiles = meta_tiles(s->max_pages);
    a.n_tiles_total = (long long)s->B * s->Hkv * a.n_tiles;
    a.B = s->B;
    a.Hkv = s->Hkv;
    a.d = s->d;
    a.P = s->page_size;
    a.max_pages = s->max_pages;
    a.num_blocks = s->num_blocks;
    a.first_page = first_page;
    a.n_pages = n;
    kv_range(s, &a.kv0, &a.nk);
    a.status = di.status;
    return cuda_rc(launch_build_meta(a, static_cast<cudaStream_t>(stream)));
}

int entmaxkv_append(const entmaxkv_shape *s, const void *k_new, const void *v_new, const int32_t *page_table,
                    const int32_t *seq_lens, void *k_cache, void *v_cache, void *meta, const void *q_in,
                    void *q_out, void *stream) {
    int rc = check_shape(s);
    if (rc) return rc;
    if (!k_new || !v_new || !page_table || !seq_lens || !k_cache || !v_cache || !meta) return ENTMAXKV_ERR_NULL;
    if ((q_in == nullptr) != (q_out == nullptr)) return ENTMAXKV_ERR_NULL;
    if (!aligned16(k_cache) || !aligned16(v_cache) || !aligned16(meta)) return ENTMAXKV_ERR_ALIGN;
    DevInfo di;
    if ((rc = device_info(&di))) return rc;
    AppendArgs a{};
    a.m.page_table = page_table;
    a.m.seq_lens = seq_lens;
    a.m.meta = static_cast<uint8_t *>(meta);
    a.m.n_tiles = meta_tiles(s->max_pages);
    a.m.n_tiles_total = (long long)s->B * s->Hkv * a.m.n_tiles;
    a.m.B = s->B;
    a.m.Hkv = s->Hkv;
    a.m.d = s->d;
    a.m.P = s->page_size;
    a.m.max_pages = s->max_pages;
    a.m.num_blocks = s->num_blocks;
    kv_range(s, &a.m.kv0, &a.m.nk);
    a.m.status = di.status;
    a.k_cache = static_cast<uint16_t *>(k_cache);
    a.v_cache = static_cast<uint16_t *>(v_cache);
    a.m.k = a.k_cache;
    a.k_new = static_cast<const uint16_t *>(k_new);
    a.v_new = static_cast<const uint16_t *>(v_new);
    a.q_in = static_cast<const uint16_t *>(q_in);
    a.q_out = static_cast<uint16_t *>(q_out);
    a.Hq = s->Hq;
    return cuda_rc(launch_append(a, static_cast<cudaStream_t>(stream)));
}

int entmaxkv_score_pages(const entmaxkv_shape *s, const void *q, const void *meta, const int32_t *seq_lens,
                         float *bbox, float *mu, float *sigma, void *stream) {
    int rc = check_shape(s);
    if (rc) return rc;
    if (!q || !meta || !seq_lens || !bbox) return ENTMAXKV_ERR_NULL;
    if ((mu == nullptr) != (sigma == nullptr)) return ENTMAXKV_ERR_NULL;
    if (!aligned16(q) || !aligned16(meta)) return ENTMAXKV_ERR_ALIGN;
    DevInfo di;
    if ((rc = device_info(&di))) return rc;
    ScoreArgs a{};
    a.q = static_cast<const uint16_t *>(q);
    a.meta = static_cast<const uint8_t *>(meta);
    a.seq_lens = seq_lens;
    a.bbox = bbox;
    a.mu = mu;
    a.sigma = sigma;
    a.n_tiles = meta_tiles(s->max_pages);
    a.n_tiles_total = (long long)s->B * s->Hkv * a.n_tiles;
    a.B = s->B;
    a.Hq = s->Hq;
    a.Hkv = s->Hkv;
    a.d = s->d;
    a.P = s->page_size;
    a.max_pages = s->max_pages;
    kv_range(s, &a.kv0, &a.nk);
    a.status = di.status;
    return cuda_rc(launch_score_pages(a, static_cast<cudaStream_t>(stream)));
}

int entmaxkv_select(const entmaxkv_shape *s, const int32_t *seq_lens, const float *bbox, const float *mu,
                    const float *sigma, int32_t policy, int32_t k, float alpha, float delta, int32_t *sel,
                    int32_t *cnt, float *tau_hat, void *workspace, size_t ws_bytes, void *stream) {
    (void)workspace;
    (void)ws_bytes;
    int rc = check_shape(s);
    if (rc) return rc;
    if (s->max_pages > MAX_SEL_PAGES) return ENTMAXKV_ERR_SHAPE;
    if (!seq_lens || !bbox || !sel || !cnt) return ENTMAXKV_ERR_NULL;
    SelectArgs a{};
    if (policy == ENTMAXKV_TOPK) {
        if (k < 1) return ENTMAXKV_ERR_POLICY;
    } else if (policy == ENTMAXKV_GAUSS || policy == ENTMAXKV_GAUSS_EST) {
        if (!mu || !sigma) return ENTMAXKV_ERR_NULL;
        if (!std::isfinite(delta)) return ENTMAXKV_ERR_POLICY;
        if (!std::isfinite(alpha) || !(alpha > 1.f)) return ENTMAXKV_ERR_ALPHA;
        a.r_int = integer_r(alpha);
        if (a.r_int == 0) return ENTMAXKV_ERR_UNSUPPORTED;
    } else {
        return ENTMAXKV_ERR_POLICY;
    }
    DevInfo di;
    if ((rc = device_info(&di))) return rc;
    a.seq_lens = seq_lens;
    a.bbox = bbox;
    a.mu = mu;
    a.sigma = sigma;
    a.sel = sel;
    a.cnt = cnt;
    a.tau_hat = tau_hat;
    a.B = s->B;
    a.Hq = s->Hq;
    a.P = s->page_size;
    a.max_pages = s->max_pages;
    a.policy = policy;
    a.k = k;
    a.alpha = alpha;
    a.delta = delta;
    {
        int kv0, nk;
        kv_range(s, &kv0, &nk);
        const int G = s->Hq / s->Hkv;
        a.h0 = kv0 * G;
        a.nh = nk * G;
    }
    a.sms = di.sms;
    a.status = di.status;
    return cuda_rc(launch_select(a, static_cast<cudaStream_t>(stream)));
}

// Shared argument checks and set-up of the decode calls.  out may be NULL only
// where the call writes no output (need_out false: the sharded begin and
// candidates phases).
static int fill_decode(bool dense, const entmaxkv_shape *s, const void *q, const void *k_cache, const void *v_cache,
                       const int32_t *page_table, const int32_t *seq_lens, float alpha, float *out, float *tau_out,
                       float *p_out, void *workspace, size_t ws_bytes, DecodeArgs *a, bool need_out = true) {
    int rc = check_shape(s);
    if (rc) return rc;
    if (!q || !k_cache || !v_cache || !page_table || !seq_lens || (need_out && !out)) return ENTMAXKV_ERR_NULL;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache)) return ENTMAXKV_ERR_ALIGN;
    if (!std::isfinite(alpha)) return ENTMAXKV_ERR_ALPHA;
    const size_t need =
        decode_ws_bytes(dense, s->B, s->Hq, s->Hkv, s->d, s->page_size, s->max_pages, nullptr, nullptr);
    if (!workspace || ws_bytes < need) return ENTMAXKV_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return ENTMAXKV_ERR_ALIGN;
    DevInfo di;
    if ((rc = device_info(&di))) return rc;
    std::memset(a, 0, sizeof(*a));
    a->q = static_cast<const uint16_t *>(q);
    a->k = static_cast<const uint16_t *>(k_cache);
    a->v = static_cast<const uint16_t *>(v_cache);
    a->page_table = page_table;
    a->seq_lens = seq_lens;
    a->out = out;
    a->tau_out = tau_out;
    a->p_out = p_out;
    decode_ws_bytes(dense, s->B, s->Hq, s->Hkv, s->d, s->page_size, s->max_pages, &a->ws, workspace);
    a->B = s->B;
    a->Hq = s->Hq;
    a->Hkv = s->Hkv;
    a->d = s->d;
    a->P = s->page_size;
    a->max_pages = s->max_pages;
    a->num_blocks = s->num_blocks;
    a->alpha = alpha;
    a->r_int = alpha > 1.f ? integer_r(alpha) : 0;
    a->sms = di.sms;
    kv_range(s, &a->kv0, &a->nk);
    a->sel_stride = s->max_pages;  // single-device call: sel rows are this shape's
    a->status = di.status;
    return ENTMAXKV_OK;
}

int entmaxkv_decode_sparse(const entmaxkv_shape *s, const void *q, const void *k_cache, const void *v_cache,
                           const int32_t *page_table, const int32_t *seq_lens, const int32_t *sel,
                           const int32_t *cnt, float alpha, float *out, float *tau_out, float *p_out,
                           void *workspace, size_t ws_bytes, void *stream) {
    if (!sel || !cnt) return ENTMAXKV_ERR_NULL;
    if (!(alpha >= 1.f)) return ENTMAXKV_ERR_ALPHA;
    if (alpha == 1.f && p_out) return ENTMAXKV_ERR_NULL;
    if (s && s->max_pages > MAX_SEL_PAGES) return ENTMAXKV_ERR_SHAPE;
    DecodeArgs a;
    int rc = fill_decode(false, s, q, k_cache, v_cache, page_table, seq_lens, alpha, out, tau_out, p_out, workspace,
                         ws_bytes, &a);
    if (rc) return rc;
    a.sel = sel;
    a.cnt = cnt;
    if ((rc = make_kv_map(&a.kmap, k_cache, s))) return rc;
    if (alpha == 1.f && (rc = make_kv_map(&a.vmap, v_cache, s))) return rc;
    return cuda_rc(launch_decode_sparse(a, static_cast<cudaStream_t>(stream)));
}

int entmaxkv_decode_step(const entmaxkv_shape *s, const void *q, const void *meta, const void *k_cache,
                         const void *v_cache, const int32_t *page_table, const int32_t *seq_lens, int32_t policy,
                         int32_t k, float alpha, float delta, float *bbox, float *mu, float *sigma, int32_t *sel,
                         int32_t *cnt, float *tau_hat, float *out, float *tau_out, float *p_out, void *workspace,
                         size_t ws_bytes, void *stream) {
    int rc = check_shape(s);
    if (rc) return rc;
    if (s->max_pages > MAX_SEL_PAGES) return ENTMAXKV_ERR_SHAPE;
    if (!meta || !bbox || !sel || !cnt) return ENTMAXKV_ERR_NULL;
    if ((mu == nullptr) != (sigma == nullptr)) return ENTMAXKV_ERR_NULL;
    if (!std::isfinite(alpha) || !(alpha > 1.f)) return ENTMAXKV_ERR_ALPHA;
    SelectArgs la{};
    if (policy == ENTMAXKV_TOPK) {
        if (k < 1) return ENTMAXKV_ERR_POLICY;
    } else if (policy == ENTMAXKV_GAUSS || policy == ENTMAXKV_GAUSS_EST) {
        if (!mu) return ENTMAXKV_ERR_NULL;
        if (!std::isfinite(delta)) return ENTMAXKV_ERR_POLICY;
        la.r_int = integer_r(alpha);
        if (la.r_int == 0) return ENTMAXKV_ERR_UNSUPPORTED;
    } else {
        return ENTMAXKV_ERR_POLICY;
    }
    if (!aligned16(meta)) return ENTMAXKV_ERR_ALIGN;
    const size_t need =
        decode_ws_bytes(false, s->B, s->Hq, s->Hkv, s->d, s->page_size, s->max_pages, nullptr, nullptr, true);
    if (!workspace || ws_bytes < need) return ENTMAXKV_ERR_WORKSPACE;
    DecodeArgs da;
    if ((rc = fill_decode(false, s, q, k_cache, v_cache, page_table, seq_lens, alpha, out, tau_out, p_out,
                          workspace, ws_bytes, &da)))
        return rc;
    decode_ws_bytes(false, s->B, s->Hq, s->Hkv, s->d, s->page_size, s->max_pages, &da.ws, workspace, true);
    da.sel = sel;
    da.cnt = cnt;
    if ((rc = make_kv_map(&da.kmap, k_cache, s))) return rc;

    const int G = s->Hq / s->Hkv;
    la.seq_lens = seq_lens;
    la.bbox = bbox;
    la.mu = mu;
    la.sigma = sigma;
    la.sel = sel;
    la.cnt = cnt;
    la.tau_hat = tau_hat;
    la.B = s->B;
    la.Hq = s->Hq;
    la.P = s->page_size;
    la.max_pages = s->max_pages;
    la.policy = policy;
    la.k = k;
    la.alpha = alpha;
    la.delta = delta;
    la.h0 = da.kv0 * G;
    la.nh = da.nk * G;
    la.sms = da.sms;
    la.status = da.status;
    la.Hkv = s->Hkv;
    la.num_blocks = s->num_blocks;
    const bool fused = select_marks_union(la);
    if (fused) {
        la.umap = da.ws.umap;
        la.uwords = da.ws.uwords;
        la.union_e = da.ws.union_e;
        la.union_blk = da.ws.union_blk;
        la.union_cnt = da.ws.union_cnt;
        la.zmax = da.ws.zmax;
        la.page_table = page_table;
    }

    ScoreArgs sa{};
    sa.q = static_cast<const uint16_t *>(q);
    sa.meta = static_cast<const uint8_t *>(meta);
    sa.seq_lens = seq_lens;
    sa.bbox = bbox;
    sa.mu = mu;
    sa.sigma = sigma;
    sa.n_tiles = meta_tiles(s->max_pages);
    sa.n_tiles_total = (long long)s->B * s->Hkv * sa.n_tiles;
    sa.B = s->B;
    sa.Hq = s->Hq;
    sa.Hkv = s->Hkv;
    sa.d = s->d;
    sa.P = s->page_size;
    sa.max_pages = s->max_pages;
    sa.kv0 = da.kv0;
    sa.nk = da.nk;
    sa.status = da.status;
    if (fused && G > 1) {  // the union marks of the call's groups
        sa.umap = da.ws.umap;
        sa.uwords = da.ws.uwords;
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e = launch_score_pages(sa, st);
    if (e == cudaSuccess) e = launch_select(la, st);
    if (e == cudaSuccess) e = fused ? launch_decode_step_tail(da, st) : launch_decode_sparse(da, st);
    return cuda_rc(e);
}

int entmaxkv_decode_step_kernels(const entmaxkv_shape *s, int32_t policy, float alpha) {
    int rc = check_shape(s);
    if (rc) return rc;
    if (!std::isfinite(alpha) || !(alpha > 1.f)) return ENTMAXKV_ERR_ALPHA;
    if (policy != ENTMAXKV_TOPK && policy != ENTMAXKV_GAUSS && policy != ENTMAXKV_GAUSS_EST)
        return ENTMAXKV_ERR_POLICY;
    if ((rc = entmaxkv_decode_sparse_kernels(s, alpha)) < 0) return rc;
    SelectArgs la{};
    la.policy = policy;
    la.max_pages = s->max_pages;
    if (!select_marks_union(la)) return 2 + rc;  // score, select, then the separate decode
    DecodeArgs da{};
    da.Hq = s->Hq;
    da.Hkv = s->Hkv;
    return 2 + decode_step_tail_kernels(da);
}

int entmaxkv_decode_sparse_kernels(const entmaxkv_shape *s, float alpha) {
    int rc = check_shape(s);
    if (rc) return rc;
    if (!(alpha >= 1.f)) return ENTMAXKV_ERR_ALPHA;
    DevInfo di;
    if ((rc = device_info(&di))) return rc;
    DecodeArgs a;
    std::memset(&a, 0, sizeof(a));
    a.B = s->B;
    a.Hq = s->Hq;
    a.Hkv = s->Hkv;
    a.d = s->d;
    a.P = s->page_size;
    a.max_pages = s->max_pages;
    a.alpha = alpha;
    a.sms = di.sms;
    kv_range(s, &a.kv0, &a.nk);
    return decode_sparse_kernels(a);
}

int entmaxkv_decode_sparse_begin(const entmaxkv_shape *s, const void *q, const void *k_cache, const void *v_cache,
                                 const int32_t *page_table, const int32_t *seq_lens, const int32_t *sel,
                                 const int32_t *cnt, int32_t sel_max_pages, int32_t page_begin, float alpha,
                                 float *zmax_out, void *workspace, size_t ws_bytes, void *stream) {
    if (!sel || !cnt || !zmax_out) return ENTMAXKV_ERR_NULL;
    if (!(alpha > 1.f)) return ENTMAXKV_ERR_ALPHA;
    // (the last shard's page range may reach past the global page count: its
    // token count keeps those pages empty)
    if (s && (s->max_pages > MAX_SEL_PAGES || page_begin < 0 || sel_max_pages < 1 || page_begin >= sel_max_pages))
        return ENTMAXKV_ERR_SHAPE;
    DecodeArgs a;
    int rc = fill_decode(false, s, q, k_cache, v_cache, page_table, seq_lens, alpha, nullptr, nullptr, nullptr,
                         workspace, ws_bytes, &a, false);
    if (rc) return rc;
    a.sel = sel;
    a.cnt = cnt;
    a.sharded = 1;
    a.page_begin = page_begin;
    a.sel_stride = sel_max_pages;
    a.zmax_out = zmax_out;
    if ((rc = make_kv_map(&a.kmap, k_cache, s))) return rc;
    return cuda_rc(launch_decode_sparse_begin(a, static_cast<cudaStream_t>(stream)));
}

int entmaxkv_decode_sparse_candidates(const entmaxkv_shape *s, const void *q, const void *k_cache,
                                      const void *v_cache, const int32_t *page_table, const int32_t *seq_lens,
                                      float alpha, const float *zmax_in, int32_t cap, float *cand_z,
                                      int32_t *cand_n, void *workspace, size_t ws_bytes, void *stream) {
    if (!zmax_in || !cand_z || !cand_n) return ENTMAXKV_ERR_NULL;
    if (!(alpha > 1.f)) return ENTMAXKV_ERR_ALPHA;
    if (cap < 1) return ENTMAXKV_ERR_SHAPE;
    DecodeArgs a;
    int rc = fill_decode(false, s, q, k_cache, v_cache, page_table, seq_lens, alpha, nullptr, nullptr, nullptr,
                         workspace, ws_bytes, &a, false);
    if (rc) return rc;
    a.zmax_in = zmax_in;
    a.cand_z = cand_z;
    a.cand_n = cand_n;
    a.cap = cap;
    return cuda_rc(launch_decode_sparse_candidates(a, static_cast<cudaStream_t>(stream)));
}

int entmaxkv_entmax_threshold(const entmaxkv_shape *s, int32_t n_shards, int32_t cap, const float *cand_z,
                              const int32_t *cand_n, const float *zmax_in, float alpha, float *tau_out,
                              void *stream) {
    int rc = check_shape(s);
    if (rc) return rc;
    if (!cand_z || !cand_n || !zmax_in || !tau_out) return ENTMAXKV_ERR_NULL;
    if (!std::isfinite(alpha) || !(alpha > 1.f)) return ENTMAXKV_ERR_ALPHA;
    if (n_shards < 1 || cap < 1 || (long long)n_shards * cap * 4 > (200ll << 10)) return ENTMAXKV_ERR_SHAPE;
    DevInfo di;
    if ((rc = device_info(&di))) return rc;
    ThresholdArgs a{};
    a.cand_z = cand_z;
    a.cand_n = cand_n;
    a.zmax = zmax_in;
    a.tau = tau_out;
    a.S = n_shards;
    a.cap = cap;
    a.B = s->B;
    a.Hq = s->Hq;
    a.Hkv = s->Hkv;
    kv_range(s, &a.kv0, &a.nk);
    a.alpha = alpha;
    a.r_int = integer_r(alpha);
    a.status = di.status;
    return cuda_rc(launch_entmax_threshold(a, static_cast<cudaStream_t>(stream)));
}

int entmaxkv_decode_sparse_finish(const entmaxkv_shape *s, const void *q, const void *k_cache, const void *v_cache,
                                  const int32_t *page_table, const int32_t *seq_lens, float alpha,
                                  const float *zmax_in, const float *tau_in, float *out, float *p_out,
                                  void *workspace, size_t ws_bytes, void *stream) {
    if (!zmax_in || !tau_in) return ENTMAXKV_ERR_NULL;
    if (!(alpha > 1.f)) return ENTMAXKV_ERR_ALPHA;
    DecodeArgs a;
    int rc = fill_decode(false, s, q, k_cache, v_cache, page_table, seq_lens, alpha, out, nullptr, p_out, workspace,
                         ws_bytes, &a);
    if (rc) return rc;
    a.zmax_in = zmax_in;
    a.tau_in = tau_in;
    return cuda_rc(launch_decode_sparse_finish(a, static_cast<cudaStream_t>(stream)));
}

int entmaxkv_decode_dense(const entmaxkv_shape *s, const void *q, const void *k_cache, const void *v_cache,
                          const int32_t *page_table, const int32_t *seq_lens, float alpha, float *out,
                          float *tau_out, float *p_out, void *workspace, size_t ws_bytes, void *stream) {
    if (!(alpha >= 1.f)) return ENTMAXKV_ERR_ALPHA;
    if (alpha == 1.f && p_out) return ENTMAXKV_ERR_NULL;
    DecodeArgs a;
    int rc = fill_decode(true, s, q, k_cache, v_cache, page_table, seq_lens, alpha, out, tau_out, p_out, workspace,
                         ws_bytes, &a);
    if (rc) return rc;
    if ((rc = make_kv_map(&a.kmap, k_cache, s))) return rc;
    if ((rc = make_kv_map(&a.vmap, v_cache, s))) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    return cuda_rc(alpha == 1.f ? launch_decode_dense_softmax(a, st) : launch_decode_dense_entmax(a, st));
}

}  // extern "C"

// ------------------------------------------------ allocation-free decode
//
// entmaxkv_decode_sparse_static: the sparse decode with its scratch in a
// fixed file-scope device array instead of a caller-provided workspace, for
// callers that cannot allocate device memory at decode time.  In host code
// g_static_scratch names a host-side stand-in, not device memory, so the
// device address is looked up once per device (with that device current) and
// that pointer is what the kernels receive.
namespace {

__device__ __align__(256) unsigned char g_static_scratch[ENTMAXKV_STATIC_SCRATCH_BYTES];

void *g_static_ptr[MAX_DEV];
bool g_static_ok[MAX_DEV];

int static_scratch(void **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEV) return ENTMAXKV_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_static_ok[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr) return ENTMAXKV_ERR_CUDA;
        g_static_ptr[dev] = p;
        g_static_ok[dev] = true;
    }
    *out = g_static_ptr[dev];
    return ENTMAXKV_OK;
}

}  // namespace

extern "C" int entmaxkv_decode_sparse_static(const entmaxkv_shape *s, const void *q, const void *k_cache,
                                             const void *v_cache, const int32_t *page_table,
                                             const int32_t *seq_lens, const int32_t *sel, const int32_t *cnt,
                                             float alpha, float *out, float *tau_out, float *p_out, void *stream) {
    int rc = check_shape(s);
    if (rc) return rc;
    const size_t need =
        decode_ws_bytes(false, s->B, s->Hq, s->Hkv, s->d, s->page_size, s->max_pages, nullptr, nullptr);
    if (need > ENTMAXKV_STATIC_SCRATCH_BYTES) return ENTMAXKV_ERR_TOO_LARGE;
    void *ws = nullptr;
    if ((rc = static_scratch(&ws))) return rc;
    return entmaxkv_decode_sparse(s, q, k_cache, v_cache, page_table, seq_lens, sel, cnt, alpha, out, tau_out,
                                  p_out, ws, ENTMAXKV_STATIC_SCRATCH_BYTES, stream);
}
