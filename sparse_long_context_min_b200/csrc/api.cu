// extern "C" entry points of the EntmaxKV library: argument validation,
// workspace layout, TMA descriptors, and dispatch to the kernels.
#include <cudaTypedefs.h>

#include <atomic>
#include <mutex>

#include "common.cuh"
#include "kernels.cuh"

namespace ekv {

// ------------------------------------------------------------------ devices
int num_sms()
{
    static int cache[64] = {0};
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) != cudaSuccess) return n;
    if (dev >= 0 && dev < 64 && cache[dev] > 0) return cache[dev];
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) n = 148;
    if (dev >= 0 && dev < 64) cache[dev] = n;
    return n;
}

int ensure_smem(const void* func, int bytes)
{
    // one flag per (kernel, device); a small table of seen pairs
    static std::mutex mu;
    static const void* seen_f[1024];
    static int seen_d[1024];
    static int nseen = 0;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 1;
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < nseen; ++i)
        if (seen_f[i] == func && seen_d[i] == dev) return 0;
    if (cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess) return 1;
    if (nseen < 1024) {
        seen_f[nseen] = func;
        seen_d[nseen] = dev;
        ++nseen;
    }
    return 0;
}

int ensure_cluster_kernel(const void* func, int smem)
{
    static std::mutex mu;
    static const void* seen_f[256];
    static int seen_d[256];
    static int nseen = 0;
    if (ensure_smem(func, smem)) return 1;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 1;
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < nseen; ++i)
        if (seen_f[i] == func && seen_d[i] == dev) return 0;
    if (cudaFuncSetAttribute(func, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess) return 1;
    if (nseen < 256) {
        seen_f[nseen] = func;
        seen_d[nseen] = dev;
        ++nseen;
    }
    return 0;
}

int max_active_clusters(const void* func, int cluster, int threads, int smem)
{
    struct Entry {
        const void* f;
        int dev, cluster, threads, smem, n;
    };
    static std::mutex mu;
    static Entry seen[256];
    static int nseen = 0;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < nseen; ++i)
        if (seen[i].f == func && seen[i].dev == dev && seen[i].cluster == cluster && seen[i].threads == threads &&
            seen[i].smem == smem)
            return seen[i].n;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(cluster, 1, 1);
    cfg.blockDim = dim3(threads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = cluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, func, &cfg) != cudaSuccess) {
        cudaGetLastError();   // clear the error: the caller tries a smaller cluster
        n = 0;
    }
    if (nseen < 256) seen[nseen++] = Entry{func, dev, cluster, threads, smem, n};
    return n;
}

// ------------------------------------------------------------------ TMA descriptors
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    static std::once_flag once;
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// 2-D view [num_phys * H_kv * ps rows][d cols] of a bf16 pool, 64 x ps boxes,
// 128-byte swizzle.
static int make_pool_map(CUtensorMap* map, const entmaxkv_pool& pool, void* base)
{
    auto fn = encode_fn();
    if (!fn) return ENTMAXKV_CUDA_ERROR;
    const cuuint64_t rows = (cuuint64_t)pool.num_phys_pages * pool.H_kv * pool.ps;
    cuuint64_t dims[2] = {(cuuint64_t)pool.d, rows};
    cuuint64_t strides[1] = {(cuuint64_t)pool.d * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)pool.ps};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? ENTMAXKV_OK : ENTMAXKV_CUDA_ERROR;
}

// ------------------------------------------------------------------ validation
static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static int check_pool(const entmaxkv_pool* pool, bool need_kv, bool need_meta)
{
    if (!pool) return ENTMAXKV_INVALID_ARG;
    if (pool->num_phys_pages <= 0 || pool->H_kv <= 0) return ENTMAXKV_INVALID_ARG;
    if (pool->d != 64 && pool->d != 128) return ENTMAXKV_UNSUPPORTED;
    if (pool->ps != 16 && pool->ps != 64) return ENTMAXKV_UNSUPPORTED;
    if (pool->dtype != ENTMAXKV_F32 && pool->dtype != ENTMAXKV_BF16) return ENTMAXKV_UNSUPPORTED;
    if ((long long)pool->num_phys_pages * pool->H_kv * pool->ps >= (1ll << 31)) return ENTMAXKV_UNSUPPORTED;
    if (need_kv && (!pool->k_pool || !pool->v_pool || !aligned16(pool->k_pool) || !aligned16(pool->v_pool)))
        return ENTMAXKV_INVALID_ARG;
    if (need_meta && (!pool->kmin || !pool->kmax || !pool->mean || !pool->m2 || !pool->count ||
                      !aligned16(pool->kmin) || !aligned16(pool->kmax) || !aligned16(pool->mean) ||
                      !aligned16(pool->m2)))
        return ENTMAXKV_INVALID_ARG;
    return ENTMAXKV_OK;
}

static int check_heads(int H_q, int H_kv)
{
    if (H_q <= 0 || H_kv <= 0 || H_q % H_kv) return ENTMAXKV_INVALID_ARG;
    const int G = H_q / H_kv;
    if (G != 1 && G != 2 && G != 4 && G != 8) return ENTMAXKV_UNSUPPORTED;
    return ENTMAXKV_OK;
}

// Exact attention takes any alpha in (1, 16] (other than 1.5 and 2 by a
// safeguarded Newton solve of the threshold and powf weights).  The Gaussian
// selector has closed forms at 1.5 and 2 and integrates numerically for any
// other alpha in [1.05, 16] (r = 1/(alpha-1) up to 20: the rule follows the
// integrand's peak, and float32 powers stay finite).
static bool alpha_gauss_ok(float alpha) { return alpha == 1.5f || alpha == 2.0f || (alpha >= 1.05f && alpha <= 16.0f); }
static bool alpha_attend_ok(float alpha) { return alpha > 1.0f && alpha <= 16.0f; }

// ------------------------------------------------------------------ workspace
static size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

static int num_splits(int B, int H_kv, int list_pages)
{
    const long long units = (long long)B * H_kv;
    long long S = (2ll * num_sms() + units - 1) / (units > 0 ? units : 1);
    if (S > list_pages) S = list_pages;
    if (S > 1024) S = 1024;
    if (S < 1) S = 1;
    return (int)S;
}

struct AttnLayout {
    int S;
    size_t xbuf, cmax, opart, mlpart, lmax, tau, counters, cval, cidx, total;
};

// attention ops over a caller's page list / with softmax weights
static bool is_sparse(int op) { return op == ENTMAXKV_OP_SPARSE_ATTEND || op == ENTMAXKV_OP_SPARSE_SOFTMAX; }
static bool is_softmax(int op) { return op == ENTMAXKV_OP_FULL_SOFTMAX || op == ENTMAXKV_OP_SPARSE_SOFTMAX; }

static AttnLayout attn_layout(int op, int B, int H_q, int H_kv, int max_pages, int k_max, int ps, int d)
{
    AttnLayout L{};
    const bool soft = is_softmax(op);
    const int list = is_sparse(op) ? k_max : max_pages;
    L.S = num_splits(B, H_kv, list);
    size_t off = 0;
    L.xbuf = off;
    if (!soft) off += round256((size_t)B * H_q * list * ps * sizeof(float));
    L.cmax = off;
    if (!soft) off += round256((size_t)B * H_q * list * ((ps + 15) / 16) * sizeof(float));
    L.opart = off;
    off += round256((size_t)B * H_q * L.S * d * sizeof(float));
    L.mlpart = off;
    if (soft) off += round256((size_t)B * H_q * L.S * 2 * sizeof(float));
    L.lmax = off;
    if (!soft) off += round256((size_t)B * H_q * L.S * sizeof(float));
    L.tau = off;
    off += round256((size_t)B * H_q * sizeof(float));
    L.counters = off;
    off += round256((size_t)B * H_kv * sizeof(int32_t));
    // candidate slots of the clustered bf16 entmax kernel
    const size_t rows = soft ? 0 : (size_t)B * H_q * kFusedMaxSplits;
    L.cval = off;
    off += round256(rows * kFusedCandCap * sizeof(float));
    L.cidx = off;
    off += round256(rows * kFusedCandCap * sizeof(int32_t));
    L.total = off;
    return L;
}

int attend_check(int op, const entmaxkv_pool* pool, const float* q, int H_q, const int32_t* page_table,
                 int max_pages, const int32_t* seq_lens, int B, const int32_t* sel, const int32_t* sel_count,
                 int k_max, float alpha, float scale, const float* out, const int32_t* status)
{
    int rc = check_pool(pool, true, false);
    if (rc) return rc;
    if ((rc = check_heads(H_q, pool->H_kv))) return rc;
    if (B < 0 || max_pages <= 0) return ENTMAXKV_INVALID_ARG;
    if (!is_softmax(op) && !alpha_attend_ok(alpha)) return ENTMAXKV_UNSUPPORTED;
    if (!(scale > 0.f) || !std::isfinite(scale)) return ENTMAXKV_INVALID_ARG;
    if (is_sparse(op) && (!sel || !sel_count || k_max <= 0)) return ENTMAXKV_INVALID_ARG;
    if (B == 0) return ENTMAXKV_OK;
    if (!q || !page_table || !seq_lens || !out || !status) return ENTMAXKV_INVALID_ARG;
    return ENTMAXKV_OK;
}

static int attend_common(int op, const entmaxkv_pool* pool, const float* q, int H_q, const int32_t* page_table,
                         int max_pages, const int32_t* seq_lens, int B, const int32_t* sel,
                         const int32_t* sel_count, int k_max, float alpha, float scale, float* out,
                         float* tau_out, int32_t* v_pages, void* workspace, size_t ws_bytes, int32_t* status,
                         void* stream)
{
    int rc = attend_check(op, pool, q, H_q, page_table, max_pages, seq_lens, B, sel, sel_count, k_max, alpha,
                          scale, out, status);
    if (rc || B == 0) return rc;
    const AttnLayout lay = attn_layout(op, B, H_q, pool->H_kv, max_pages, k_max, pool->ps, pool->d);
    if (!workspace || ws_bytes < lay.total || !aligned16(workspace)) return ENTMAXKV_WORKSPACE;

    AttnArgs a{};
    a.q = q;
    a.H_q = H_q;
    a.H_kv = pool->H_kv;
    a.G = H_q / pool->H_kv;
    a.page_table = page_table;
    a.max_pages = max_pages;
    a.seq_lens = seq_lens;
    a.sel = is_sparse(op) ? sel : nullptr;
    a.sel_count = is_sparse(op) ? sel_count : nullptr;
    a.k_max = is_sparse(op) ? k_max : max_pages;
    a.num_phys = pool->num_phys_pages;
    a.S = lay.S;
    a.alpha = alpha;
    a.xscale = is_softmax(op) ? scale : (alpha - 1.0f) * scale;
    char* ws = static_cast<char*>(workspace);
    a.xbuf = reinterpret_cast<float*>(ws + lay.xbuf);
    a.cmax = reinterpret_cast<float*>(ws + lay.cmax);
    a.opart = reinterpret_cast<float*>(ws + lay.opart);
    a.mlpart = reinterpret_cast<float*>(ws + lay.mlpart);
    a.lmax = reinterpret_cast<float*>(ws + lay.lmax);
    a.vpages = v_pages;
    a.tau = reinterpret_cast<float*>(ws + lay.tau);
    a.counters = reinterpret_cast<int32_t*>(ws + lay.counters);
    a.cval = reinterpret_cast<float*>(ws + lay.cval);
    a.cidx = reinterpret_cast<int32_t*>(ws + lay.cidx);
    a.out = out;
    a.tau_out = tau_out;
    a.status = status;

    CUtensorMap kmap, vmap;
    if (pool->dtype == ENTMAXKV_BF16) {
        if ((rc = make_pool_map(&kmap, *pool, pool->k_pool))) return rc;
        if ((rc = make_pool_map(&vmap, *pool, pool->v_pool))) return rc;
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (is_softmax(op)) return launch_softmax_attend(*pool, a, B, &kmap, &vmap, st);
    return launch_entmax_attend(*pool, a, B, &kmap, &vmap, st);
}

}  // namespace ekv

using namespace ekv;

extern "C" {

int entmaxkv_append_metadata(const entmaxkv_pool* pool, const void* k_new, const void* v_new, int32_t n_new,
                             const int32_t* page_table, int32_t max_pages, int32_t* seq_lens, int32_t B,
                             int32_t* status, void* stream)
{
    int rc = check_pool(pool, true, true);
    if (rc) return rc;
    if (n_new < 0 || B < 0 || max_pages <= 0) return ENTMAXKV_INVALID_ARG;
    if (n_new == 0 || B == 0) return ENTMAXKV_OK;
    if (!k_new || !v_new || !page_table || !seq_lens || !status) return ENTMAXKV_INVALID_ARG;
    if ((long long)n_new > (long long)max_pages * pool->ps) return ENTMAXKV_INVALID_ARG;
    return launch_append(*pool, k_new, v_new, n_new, page_table, max_pages, seq_lens, B, status,
                         static_cast<cudaStream_t>(stream));
}

int entmaxkv_score_pages(const entmaxkv_pool* pool, const float* q, int32_t H_q, const int32_t* page_table,
                         int32_t max_pages, const int32_t* seq_lens, int32_t B, int32_t mode, float scale,
                         float* ub, float* m, float* v, float* est_max, int32_t* status, void* stream)
{
    int rc = check_pool(pool, false, true);
    if (rc) return rc;
    if ((rc = check_heads(H_q, pool->H_kv))) return rc;
    if (B < 0 || max_pages <= 0) return ENTMAXKV_INVALID_ARG;
    if (mode != ENTMAXKV_SCORE_BBOX && mode != ENTMAXKV_SCORE_GAUSS) return ENTMAXKV_INVALID_ARG;
    if (!std::isfinite(scale)) return ENTMAXKV_INVALID_ARG;
    if (B == 0) return ENTMAXKV_OK;
    if (!q || !page_table || !seq_lens || !status) return ENTMAXKV_INVALID_ARG;
    if (mode == ENTMAXKV_SCORE_BBOX && !ub) return ENTMAXKV_INVALID_ARG;
    if (mode == ENTMAXKV_SCORE_GAUSS && (!m || !v || !est_max)) return ENTMAXKV_INVALID_ARG;
    return launch_score(*pool, q, H_q, page_table, max_pages, seq_lens, B, mode, scale, ub, m, v, est_max,
                        status, static_cast<cudaStream_t>(stream));
}

int entmaxkv_append_score_pages(const entmaxkv_pool* pool, const void* k_new, const void* v_new, int32_t n_new,
                                const float* q, int32_t H_q, const int32_t* page_table, int32_t max_pages,
                                int32_t* seq_lens, int32_t B, float scale, float* ub, int32_t* status, void* stream)
{
    int rc = check_pool(pool, true, true);
    if (rc) return rc;
    if ((rc = check_heads(H_q, pool->H_kv))) return rc;
    if (n_new < 0 || B < 0 || max_pages <= 0) return ENTMAXKV_INVALID_ARG;
    if (!std::isfinite(scale)) return ENTMAXKV_INVALID_ARG;
    if ((long long)n_new > (long long)max_pages * pool->ps) return ENTMAXKV_INVALID_ARG;
    if (B == 0) return ENTMAXKV_OK;
    if (!q || !page_table || !seq_lens || !ub || !status) return ENTMAXKV_INVALID_ARG;
    if (n_new > 0 && (!k_new || !v_new)) return ENTMAXKV_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (n_new == 0)
        return launch_score(*pool, q, H_q, page_table, max_pages, seq_lens, B, ENTMAXKV_SCORE_BBOX, scale, ub,
                            nullptr, nullptr, nullptr, status, st);
    return launch_append_score(*pool, k_new, v_new, n_new, q, H_q, page_table, max_pages, seq_lens, B, scale, ub,
                               status, st);
}

int entmaxkv_select(int32_t mode, const float* ub, const float* m, const float* v, const float* est_max,
                    const int32_t* seq_lens, int32_t ps, int32_t B, int32_t H_q, int32_t H_kv, int32_t max_pages,
                    int32_t budget, float budget_frac, float alpha, float delta, int32_t k_max, int32_t* sel,
                    int32_t* sel_count, float* tau_hat, void* workspace, size_t ws_bytes, int32_t* status,
                    void* stream)
{
    (void)workspace;
    (void)ws_bytes;
    int rc = check_heads(H_q, H_kv);
    if (rc) return rc;
    if (ps <= 0 || B < 0 || max_pages <= 0 || k_max <= 0) return ENTMAXKV_INVALID_ARG;
    if (mode == ENTMAXKV_SELECT_TOPK) {
        if (budget >= 0) {
            if (budget > k_max) return ENTMAXKV_INVALID_ARG;
        } else {
            if (!(budget_frac >= 0.f) || budget_frac > 1.f) return ENTMAXKV_INVALID_ARG;
            if ((long long)std::ceil((double)budget_frac * (double)max_pages) > k_max) return ENTMAXKV_INVALID_ARG;
        }
        if (B == 0) return ENTMAXKV_OK;
        if (!ub || !seq_lens || !sel || !sel_count || !status) return ENTMAXKV_INVALID_ARG;
    } else if (mode == ENTMAXKV_SELECT_GAUSS) {
        if (!alpha_gauss_ok(alpha)) return ENTMAXKV_UNSUPPORTED;
        if (!std::isfinite(delta) || k_max < max_pages) return ENTMAXKV_INVALID_ARG;
        if (B == 0) return ENTMAXKV_OK;
        if (!m || !v || !est_max || !seq_lens || !sel || !sel_count || !tau_hat || !status)
            return ENTMAXKV_INVALID_ARG;
    } else {
        return ENTMAXKV_INVALID_ARG;
    }
    return launch_select(mode, ub, m, v, est_max, seq_lens, ps, B, H_q, H_kv, max_pages, budget, budget_frac,
                         alpha, delta, k_max, sel, sel_count, tau_hat, status, static_cast<cudaStream_t>(stream));
}

int entmaxkv_sparse_attend(const entmaxkv_pool* pool, const float* q, int32_t H_q, const int32_t* page_table,
                           int32_t max_pages, const int32_t* seq_lens, int32_t B, const int32_t* sel,
                           const int32_t* sel_count, int32_t k_max, float alpha, float scale, float* out,
                           float* tau_out, int32_t* v_pages, void* workspace, size_t ws_bytes, int32_t* status,
                           void* stream)
{
    return attend_common(ENTMAXKV_OP_SPARSE_ATTEND, pool, q, H_q, page_table, max_pages, seq_lens, B, sel,
                         sel_count, k_max, alpha, scale, out, tau_out, v_pages, workspace, ws_bytes, status,
                         stream);
}

int entmaxkv_full_entmax_decode(const entmaxkv_pool* pool, const float* q, int32_t H_q,
                                const int32_t* page_table, int32_t max_pages, const int32_t* seq_lens, int32_t B,
                                float alpha, float scale, float* out, float* tau_out, int32_t* v_pages,
                                void* workspace, size_t ws_bytes, int32_t* status, void* stream)
{
    return attend_common(ENTMAXKV_OP_FULL_ENTMAX, pool, q, H_q, page_table, max_pages, seq_lens, B, nullptr,
                         nullptr, max_pages, alpha, scale, out, tau_out, v_pages, workspace, ws_bytes, status,
                         stream);
}

int entmaxkv_full_softmax_decode(const entmaxkv_pool* pool, const float* q, int32_t H_q,
                                 const int32_t* page_table, int32_t max_pages, const int32_t* seq_lens, int32_t B,
                                 float scale, float* out, void* workspace, size_t ws_bytes, int32_t* status,
                                 void* stream)
{
    return attend_common(ENTMAXKV_OP_FULL_SOFTMAX, pool, q, H_q, page_table, max_pages, seq_lens, B, nullptr,
                         nullptr, max_pages, 1.5f, scale, out, nullptr, nullptr, workspace, ws_bytes, status,
                         stream);
}

int entmaxkv_sparse_softmax_attend(const entmaxkv_pool* pool, const float* q, int32_t H_q,
                                   const int32_t* page_table, int32_t max_pages, const int32_t* seq_lens, int32_t B,
                                   const int32_t* sel, const int32_t* sel_count, int32_t k_max, float scale,
                                   float* out, void* workspace, size_t ws_bytes, int32_t* status, void* stream)
{
    return attend_common(ENTMAXKV_OP_SPARSE_SOFTMAX, pool, q, H_q, page_table, max_pages, seq_lens, B, sel,
                         sel_count, k_max, 1.5f, scale, out, nullptr, nullptr, workspace, ws_bytes, status, stream);
}

size_t entmaxkv_workspace_size(int32_t op, int32_t B, int32_t H_q, int32_t H_kv, int32_t max_pages, int32_t k_max,
                               int32_t ps, int32_t d)
{
    if (B <= 0 || H_q <= 0 || H_kv <= 0 || max_pages <= 0 || ps <= 0 || d <= 0) return 0;
    if (op == ENTMAXKV_OP_SELECT) return 0;
    if (is_sparse(op) && k_max <= 0) return 0;
    if (!is_sparse(op) && op != ENTMAXKV_OP_FULL_ENTMAX && op != ENTMAXKV_OP_FULL_SOFTMAX) return 0;
    return attn_layout(op, B, H_q, H_kv, max_pages, k_max, ps, d).total;
}

const char* entmaxkv_status_string(int32_t code)
{
    switch (code) {
        case ENTMAXKV_OK: return "ok";
        case ENTMAXKV_INVALID_ARG: return "invalid argument";
        case ENTMAXKV_UNSUPPORTED: return "unsupported configuration (d, ps, dtype, group size or alpha)";
        case ENTMAXKV_CUDA_ERROR: return "CUDA runtime error";
        case ENTMAXKV_TIMEOUT: return "bounded device wait timed out";
        case ENTMAXKV_DEVICE_BOUNDS: return "device index check failed (page id, list entry or count out of range)";
        case ENTMAXKV_WORKSPACE: return "workspace missing, misaligned or too small";
        case ENTMAXKV_STATIC_LIMIT: return "problem needs more scratch than the built-in buffer holds";
        default: return "unknown status";
    }
}

int entmaxkv_selftest_timeout(int64_t limit_ns, int32_t* status, void* stream)
{
    if (!status || limit_ns < 0 || limit_ns > 2000000000ll) return ENTMAXKV_INVALID_ARG;
    return launch_selftest_timeout(limit_ns, status, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
