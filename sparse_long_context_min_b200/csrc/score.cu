// Query-aware page scoring from per-page metadata.
//
// EntmaxKV (German technical summary, section 2.A): before any key or value is
// loaded, every page is scored from its metadata -- the bounding box
// (coordinatewise k_min / k_max) bounds q.k for every key of the page; the
// Gaussian statistics (mean, variance) model the page's token scores.
//
// One thread scores one logical page of one (sequence, kv head) for every
// query head of the group.  The query group sits in shared memory and is read
// as a broadcast; each thread streams its page's metadata rows with 16-byte
// loads.  The arithmetic order is the canonical one of entmaxkv.h (fused
// multiply-adds in ascending d from 0, explicit round-to-nearest intrinsics so
// nothing else is contracted), because selection decisions are taken on these
// fp32 values.
#include "common.cuh"
#include "kernels.cuh"

namespace ekv {

constexpr int kScoreThreads = 128;

// 16-byte vector of metadata: 8 bf16 or 4 fp32 values, widened to fp32.
template <typename T>
struct Vec16;
template <>
struct Vec16<uint16_t> {
    static constexpr int N = 8;
    EKV_DEV static void load(const uint16_t* p, float (&f)[8])
    {
        const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            f[2 * i] = __uint_as_float(w[i] << 16);
            f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
        }
    }
};
template <>
struct Vec16<float> {
    static constexpr int N = 4;
    EKV_DEV static void load(const float* p, float (&f)[4])
    {
        const float4 u = __ldg(reinterpret_cast<const float4*>(p));
        f[0] = u.x; f[1] = u.y; f[2] = u.z; f[3] = u.w;
    }
};

template <typename T, int D, int G>
__global__ void __launch_bounds__(kScoreThreads)
score_bbox_kernel(const T* __restrict__ kmin, const T* __restrict__ kmax, const float* __restrict__ q,
                  int H_q, int H_kv, int ps, int num_phys, const int32_t* __restrict__ page_table,
                  int max_pages, const int32_t* __restrict__ seq_lens, float scale, float* __restrict__ ub,
                  int32_t* status)
{
    __shared__ float qs[G * D];
    const int b = blockIdx.z, g = blockIdx.y;
    const int p = blockIdx.x * kScoreThreads + threadIdx.x;
    for (int i = threadIdx.x; i < G * D; i += kScoreThreads)
        qs[i] = q[((size_t)b * H_q + (size_t)g * G) * D + i];
    __syncthreads();
    if (p >= max_pages) return;
    const int L = seq_lens[b];
    const int P = pages_of(L, ps, max_pages, status);
    float* dst = ub + ((size_t)b * H_kv + g) * max_pages + p;
    if (p >= P) {
        *dst = -INFINITY;
        return;
    }
    const int phys = page_table[(size_t)b * max_pages + p];
    if (phys < 0 || phys >= num_phys) {
        report(status, ENTMAXKV_DEVICE_BOUNDS);
        *dst = -INFINITY;
        return;
    }
    const size_t row = ((size_t)phys * H_kv + g) * D;
    const T* lo = kmin + row;
    const T* hi = kmax + row;
    constexpr int N = Vec16<T>::N;
    float acc[G];
#pragma unroll
    for (int h = 0; h < G; ++h) acc[h] = 0.f;
#pragma unroll 4
    for (int j = 0; j < D; j += N) {
        float a[N], c[N];
        Vec16<T>::load(lo + j, a);
        Vec16<T>::load(hi + j, c);
#pragma unroll
        for (int e = 0; e < N; ++e) {
#pragma unroll
            for (int h = 0; h < G; ++h) {
                const float qv = qs[h * D + j + e];
                acc[h] = __fmaf_rn(qv, qv >= 0.f ? c[e] : a[e], acc[h]);
            }
        }
    }
    float best = 0.f;
#pragma unroll
    for (int h = 0; h < G; ++h) {
        const float u = __fmul_rn(acc[h], scale);
        if (h == 0 || u > best) best = u;
    }
    if (best == 0.f) best = 0.f;
    *dst = best;
}

struct ZTable {
    float z[65];
};

template <int D, int G>
__global__ void __launch_bounds__(kScoreThreads)
score_gauss_kernel(const float* __restrict__ mean, const float* __restrict__ m2, const float* __restrict__ q,
                   int H_q, int H_kv, int ps, int num_phys, const int32_t* __restrict__ page_table,
                   int max_pages, const int32_t* __restrict__ seq_lens, float scale, const ZTable zt,
                   float* __restrict__ m_out, float* __restrict__ v_out, float* __restrict__ e_out,
                   int32_t* status)
{
    __shared__ float qs[G * D];
    const int b = blockIdx.z, g = blockIdx.y;
    const int p = blockIdx.x * kScoreThreads + threadIdx.x;
    for (int i = threadIdx.x; i < G * D; i += kScoreThreads)
        qs[i] = q[((size_t)b * H_q + (size_t)g * G) * D + i];
    __syncthreads();
    if (p >= max_pages) return;
    const int L = seq_lens[b];
    const int P = pages_of(L, ps, max_pages, status);
    const size_t out0 = ((size_t)b * H_q + (size_t)g * G) * max_pages + p;
    int phys = -1;
    if (p < P) {
        phys = page_table[(size_t)b * max_pages + p];
        if (phys < 0 || phys >= num_phys) {
            report(status, ENTMAXKV_DEVICE_BOUNDS);
            phys = -1;
        }
    }
    if (phys < 0) {
#pragma unroll
        for (int h = 0; h < G; ++h) {
            m_out[out0 + (size_t)h * max_pages] = -INFINITY;
            v_out[out0 + (size_t)h * max_pages] = 0.f;
            e_out[out0 + (size_t)h * max_pages] = -INFINITY;
        }
        return;
    }
    const int n = min(ps, L - p * ps);
    const size_t row = ((size_t)phys * H_kv + g) * D;
    const float* mu = mean + row;
    const float* sq = m2 + row;
    float ma[G], va[G];
#pragma unroll
    for (int h = 0; h < G; ++h) ma[h] = va[h] = 0.f;
#pragma unroll 4
    for (int j = 0; j < D; j += 4) {
        float a[4], c[4];
        Vec16<float>::load(mu + j, a);
        Vec16<float>::load(sq + j, c);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
#pragma unroll
            for (int h = 0; h < G; ++h) {
                const float qv = qs[h * D + j + e];
                ma[h] = __fmaf_rn(qv, a[e], ma[h]);
                va[h] = __fmaf_rn(__fmul_rn(qv, qv), c[e], va[h]);
            }
        }
    }
    const float scale2 = __fmul_rn(scale, scale);
    const float zn = zt.z[n];
#pragma unroll
    for (int h = 0; h < G; ++h) {
        const float mm = __fmul_rn(ma[h], scale);
        const float vv = __fmul_rn(__fdiv_rn(va[h], (float)n), scale2);
        m_out[out0 + (size_t)h * max_pages] = mm;
        v_out[out0 + (size_t)h * max_pages] = vv;
        e_out[out0 + (size_t)h * max_pages] = __fmaf_rn(__fsqrt_rn(vv), zn, mm);
    }
}

template <typename T, int D>
static void bbox_dispatch_g(int G, dim3 grid, cudaStream_t st, const entmaxkv_pool& pool, const float* q,
                            int H_q, const int32_t* pt, int max_pages, const int32_t* sl, float scale,
                            float* ub, int32_t* status)
{
#define EKV_BBOX(GG)                                                                                     \
    score_bbox_kernel<T, D, GG><<<grid, kScoreThreads, 0, st>>>(                                         \
        (const T*)pool.kmin, (const T*)pool.kmax, q, H_q, pool.H_kv, pool.ps, pool.num_phys_pages, pt, \
        max_pages, sl, scale, ub, status)
    switch (G) {
        case 1: EKV_BBOX(1); break;
        case 2: EKV_BBOX(2); break;
        case 4: EKV_BBOX(4); break;
        default: EKV_BBOX(8); break;
    }
#undef EKV_BBOX
}

template <int D>
static void gauss_dispatch_g(int G, dim3 grid, cudaStream_t st, const entmaxkv_pool& pool, const float* q,
                             int H_q, const int32_t* pt, int max_pages, const int32_t* sl, float scale,
                             const ZTable& zt, float* m, float* v, float* e, int32_t* status)
{
#define EKV_GAUSS(GG)                                                                                      \
    score_gauss_kernel<D, GG><<<grid, kScoreThreads, 0, st>>>(pool.mean, pool.m2, q, H_q, pool.H_kv,     \
                                                              pool.ps, pool.num_phys_pages, pt, max_pages, \
                                                              sl, scale, zt, m, v, e, status)
    switch (G) {
        case 1: EKV_GAUSS(1); break;
        case 2: EKV_GAUSS(2); break;
        case 4: EKV_GAUSS(4); break;
        default: EKV_GAUSS(8); break;
    }
#undef EKV_GAUSS
}

int launch_score(const entmaxkv_pool& pool, const float* q, int H_q, const int32_t* page_table,
                 int max_pages, const int32_t* seq_lens, int B, int mode, float scale, float* ub, float* m,
                 float* v, float* est, int32_t* status, cudaStream_t stream)
{
    const int G = H_q / pool.H_kv;
    dim3 grid((max_pages + kScoreThreads - 1) / kScoreThreads, pool.H_kv, B);
    if (mode == ENTMAXKV_SCORE_BBOX) {
        if (pool.dtype == ENTMAXKV_BF16) {
            if (pool.d == 128) bbox_dispatch_g<uint16_t, 128>(G, grid, stream, pool, q, H_q, page_table, max_pages, seq_lens, scale, ub, status);
            else bbox_dispatch_g<uint16_t, 64>(G, grid, stream, pool, q, H_q, page_table, max_pages, seq_lens, scale, ub, status);
        } else {
            if (pool.d == 128) bbox_dispatch_g<float, 128>(G, grid, stream, pool, q, H_q, page_table, max_pages, seq_lens, scale, ub, status);
            else bbox_dispatch_g<float, 64>(G, grid, stream, pool, q, H_q, page_table, max_pages, seq_lens, scale, ub, status);
        }
    } else {
        // z_n = fp32(sqrt(2 ln n)), n >= 2; z_0 = z_1 = 0 (Gaussian expected
        // maximum of n draws, in units of the standard deviation)
        ZTable zt;
        for (int n = 0; n <= 64; ++n) zt.z[n] = n >= 2 ? (float)std::sqrt(2.0 * std::log((double)n)) : 0.0f;
        if (pool.d == 128) gauss_dispatch_g<128>(G, grid, stream, pool, q, H_q, page_table, max_pages, seq_lens, scale, zt, m, v, est, status);
        else gauss_dispatch_g<64>(G, grid, stream, pool, q, H_q, page_table, max_pages, seq_lens, scale, zt, m, v, est, status);
    }
    return cudaGetLastError() == cudaSuccess ? ENTMAXKV_OK : ENTMAXKV_CUDA_ERROR;
}

}  // namespace ekv
