// KV append fused with the per-page metadata update.
//
// EntmaxKV (German technical summary, section 2.A): pages carry lightweight
// metadata -- the coordinatewise minimum and maximum key and the first and
// second moments of the keys -- which the decode loop keeps current as tokens
// are appended.  One CTA handles one (logical page touched, kv head, sequence);
// thread j owns coordinate j and walks the page's new tokens in order, so the
// Welford recurrence runs in token order exactly as specified in entmaxkv.h.
#include "common.cuh"
#include "kernels.cuh"

#include <algorithm>

namespace ekv {

template <typename T>
EKV_DEV float kv_to_f32(T v);
template <>
EKV_DEV float kv_to_f32<float>(float v) { return v; }
template <>
EKV_DEV float kv_to_f32<uint16_t>(uint16_t v) { return bf16_bits_to_f32(v); }

template <typename T>
__global__ void append_kernel(T* __restrict__ k_pool, T* __restrict__ v_pool, T* __restrict__ kmin,
                              T* __restrict__ kmax, float* __restrict__ mean, float* __restrict__ m2,
                              int32_t* __restrict__ count, int num_phys, int H_kv, int ps, int d,
                              const T* __restrict__ k_new, const T* __restrict__ v_new, int n_new,
                              const int32_t* __restrict__ page_table, int max_pages,
                              const int32_t* __restrict__ seq_lens, int32_t* status)
{
    pdl_enter();
    const int b = blockIdx.z, g = blockIdx.y, j = threadIdx.x;
    const int base = seq_lens[b];
    if (base < 0) {
        if (j == 0 && g == 0 && blockIdx.x == 0) report(status, ENTMAXKV_DEVICE_BOUNDS);
        return;
    }
    const int lp = base / ps + (int)blockIdx.x;
    const int t0 = max(base, lp * ps);
    const int t1 = min(base + n_new, (lp + 1) * ps);
    if (t0 >= t1) return;
    if (lp >= max_pages) {
        if (j == 0) report(status, ENTMAXKV_DEVICE_BOUNDS);
        return;
    }
    const int phys = page_table[(size_t)b * max_pages + lp];
    if (phys < 0 || phys >= num_phys) {
        if (j == 0) report(status, ENTMAXKV_DEVICE_BOUNDS);
        return;
    }
    const size_t row = (size_t)phys * H_kv + g;
    const size_t meta = row * d + j;

    float mu = 0.f, s = 0.f, lof = 0.f, hif = 0.f;
    T lo = T(0), hi = T(0);
    if (t0 - lp * ps > 0) {   // resume a partially filled page
        mu = mean[meta];
        s = m2[meta];
        lo = kmin[meta];
        hi = kmax[meta];
        lof = kv_to_f32<T>(lo);
        hif = kv_to_f32<T>(hi);
    }
    const size_t src0 = ((size_t)b * H_kv + g) * n_new;
    for (int t = t0; t < t1; ++t) {
        const int slot = t - lp * ps;
        const size_t src = (src0 + (t - base)) * d + j;
        const T kx = k_new[src];
        const T vx = v_new[src];
        const size_t dst = (row * ps + slot) * d + j;
        k_pool[dst] = kx;
        v_pool[dst] = vx;
        const float x = kv_to_f32<T>(kx);
        if (slot == 0) {
            mu = x;
            s = 0.f;
            lo = hi = kx;
            lof = hif = x;
        } else {
            const float n = (float)(slot + 1);
            const float d1 = __fsub_rn(x, mu);
            mu = __fadd_rn(mu, __fdiv_rn(d1, n));
            const float d2 = __fsub_rn(x, mu);
            s = __fmaf_rn(d1, d2, s);
            if (x < lof) { lo = kx; lof = x; }
            if (x > hif) { hi = kx; hif = x; }
        }
    }
    mean[meta] = mu;
    m2[meta] = s;
    kmin[meta] = lo;
    kmax[meta] = hi;
    if (g == 0 && j == 0) count[phys] = t1 - lp * ps;
}

// Decode-sized appends (n_new <= ps): one block per sequence walks every
// (touched page, kv head, coordinate) of its new tokens and then advances
// seq_lens itself -- no other block reads that sequence's length, so no second
// kernel is needed.
template <typename T>
__global__ void __launch_bounds__(1024) append_small_kernel(T* __restrict__ k_pool, T* __restrict__ v_pool, T* __restrict__ kmin,
                                    T* __restrict__ kmax, float* __restrict__ mean, float* __restrict__ m2,
                                    int32_t* __restrict__ count, int num_phys, int H_kv, int ps, int d,
                                    const T* __restrict__ k_new, const T* __restrict__ v_new, int n_new,
                                    const int32_t* __restrict__ page_table, int max_pages,
                                    int32_t* __restrict__ seq_lens, int32_t* status)
{
    pdl_enter();
    const int b = blockIdx.x;
    // the first new token of this thread's first (kv head, coordinate) does not
    // depend on the sequence length: load it before the length and page id
    const int w0 = threadIdx.x;
    T pk = T(0), pv = T(0);
    if (n_new > 0 && w0 < H_kv * d) {
        const size_t src = ((size_t)b * H_kv + w0 / d) * n_new * d + w0 % d;
        pk = k_new[src];
        pv = v_new[src];
    }
    const int base = seq_lens[b];
    __syncthreads();                      // every thread has read the length
    if (base < 0) {
        if (threadIdx.x == 0) report(status, ENTMAXKV_DEVICE_BOUNDS);
        return;
    }
    for (int lp = base / ps; lp * ps < base + n_new; ++lp) {
        const int t0 = max(base, lp * ps);
        const int t1 = min(base + n_new, (lp + 1) * ps);
        if (lp >= max_pages) {
            if (threadIdx.x == 0) report(status, ENTMAXKV_DEVICE_BOUNDS);
            break;
        }
        const int phys = page_table[(size_t)b * max_pages + lp];
        if (phys < 0 || phys >= num_phys) {
            if (threadIdx.x == 0) report(status, ENTMAXKV_DEVICE_BOUNDS);
            continue;
        }
        for (int w = threadIdx.x; w < H_kv * d; w += blockDim.x) {
            const int g = w / d, j = w % d;
            const size_t row = (size_t)phys * H_kv + g;
            const size_t meta = row * d + j;
            float mu = 0.f, s = 0.f, lof = 0.f, hif = 0.f;
            T lo = T(0), hi = T(0);
            if (t0 - lp * ps > 0) {
                mu = mean[meta];
                s = m2[meta];
                lo = kmin[meta];
                hi = kmax[meta];
                lof = kv_to_f32<T>(lo);
                hif = kv_to_f32<T>(hi);
            }
            const size_t src0 = ((size_t)b * H_kv + g) * n_new;
            for (int t = t0; t < t1; ++t) {
                const int slot = t - lp * ps;
                const size_t src = (src0 + (t - base)) * d + j;
                const bool pre = w == w0 && t == base;
                const T kx = pre ? pk : k_new[src];
                const size_t dst = (row * ps + slot) * d + j;
                k_pool[dst] = kx;
                v_pool[dst] = pre ? pv : v_new[src];
                const float x = kv_to_f32<T>(kx);
                if (slot == 0) {
                    mu = x;
                    s = 0.f;
                    lo = hi = kx;
                    lof = hif = x;
                } else {
                    const float n = (float)(slot + 1);
                    const float d1 = __fsub_rn(x, mu);
                    mu = __fadd_rn(mu, __fdiv_rn(d1, n));
                    const float d2 = __fsub_rn(x, mu);
                    s = __fmaf_rn(d1, d2, s);
                    if (x < lof) { lo = kx; lof = x; }
                    if (x > hif) { hi = kx; hif = x; }
                }
            }
            mean[meta] = mu;
            m2[meta] = s;
            kmin[meta] = lo;
            kmax[meta] = hi;
        }
        if (threadIdx.x == 0) count[phys] = t1 - lp * ps;
    }
    if (threadIdx.x == 0) seq_lens[b] = base + n_new;
}

__global__ void advance_kernel(int32_t* seq_lens, int B, int n_new)
{
    pdl_enter();
    const int b = blockIdx.x * blockDim.x + threadIdx.x;
    if (b < B) seq_lens[b] += n_new;
}

int launch_advance(int32_t* seq_lens, int B, int n_new, cudaStream_t stream)
{
    launch_pdl(advance_kernel, dim3((B + 127) / 128), dim3(128), 0, stream, seq_lens, B, n_new);
    return cudaGetLastError() == cudaSuccess ? ENTMAXKV_OK : ENTMAXKV_CUDA_ERROR;
}

int launch_append(const entmaxkv_pool& pool, const void* k_new, const void* v_new, int n_new,
                  const int32_t* page_table, int max_pages, int32_t* seq_lens, int B, int32_t* status,
                  cudaStream_t stream)
{
    if (n_new <= pool.ps) {
        const int threads = std::min(1024, pool.H_kv * pool.d);
        cudaError_t e;
        if (pool.dtype == ENTMAXKV_BF16)
            e = launch_pdl(append_small_kernel<uint16_t>, dim3(B), dim3(threads), 0, stream, (uint16_t*)pool.k_pool,
                           (uint16_t*)pool.v_pool, (uint16_t*)pool.kmin, (uint16_t*)pool.kmax, pool.mean, pool.m2,
                           pool.count, pool.num_phys_pages, pool.H_kv, pool.ps, pool.d, (const uint16_t*)k_new,
                           (const uint16_t*)v_new, n_new, page_table, max_pages, seq_lens, status);
        else
            e = launch_pdl(append_small_kernel<float>, dim3(B), dim3(threads), 0, stream, (float*)pool.k_pool,
                           (float*)pool.v_pool, (float*)pool.kmin, (float*)pool.kmax, pool.mean, pool.m2, pool.count,
                           pool.num_phys_pages, pool.H_kv, pool.ps, pool.d, (const float*)k_new,
                           (const float*)v_new, n_new, page_table, max_pages, seq_lens, status);
        return e == cudaSuccess ? ENTMAXKV_OK : ENTMAXKV_CUDA_ERROR;
    }
    dim3 grid((n_new + pool.ps - 1) / pool.ps + 1, pool.H_kv, B);
    if (pool.dtype == ENTMAXKV_BF16) {
        launch_pdl(append_kernel<uint16_t>, dim3(grid), dim3(pool.d), 0, stream, (uint16_t*)pool.k_pool, (uint16_t*)pool.v_pool, (uint16_t*)pool.kmin, (uint16_t*)pool.kmax,
            pool.mean, pool.m2, pool.count, pool.num_phys_pages, pool.H_kv, pool.ps, pool.d,
            (const uint16_t*)k_new, (const uint16_t*)v_new, n_new, page_table, max_pages, seq_lens, status);
    } else {
        launch_pdl(append_kernel<float>, dim3(grid), dim3(pool.d), 0, stream, (float*)pool.k_pool, (float*)pool.v_pool, (float*)pool.kmin, (float*)pool.kmax, pool.mean,
            pool.m2, pool.count, pool.num_phys_pages, pool.H_kv, pool.ps, pool.d, (const float*)k_new,
            (const float*)v_new, n_new, page_table, max_pages, seq_lens, status);
    }
    if (cudaGetLastError() != cudaSuccess) return ENTMAXKV_CUDA_ERROR;
    launch_pdl(advance_kernel, dim3((B + 127) / 128), dim3(128), 0, stream, seq_lens, B, n_new);
    if (cudaGetLastError() != cudaSuccess) return ENTMAXKV_CUDA_ERROR;
    return ENTMAXKV_OK;
}

}  // namespace ekv
