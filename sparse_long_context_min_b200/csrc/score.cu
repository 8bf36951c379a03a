// Query-aware page scoring from per-page metadata.
//
// EntmaxKV (German technical summary, section 2.A): before any key or value is
// loaded, every page is scored from its metadata -- the bounding box
// (coordinatewise k_min / k_max) bounds q.k for every key of the page; the
// Gaussian statistics (mean, variance) model the page's token scores.
//
// Streaming kernel: eight threads share a metadata row (one page, one kv
// head), thread k owning the k-th of 8 consecutive d-slices with its slice of
// the query group held in registers.  Each thread reads its slice with 16-byte
// loads, prefetching the next row while it computes the current one, forms
// its slice sum as a chain of fp32 fused multiply-adds in ascending d, and the
// 8 slice sums are combined by a fixed xor-shuffle tree
// ((S0+S1)+(S2+S3))+((S4+S5)+(S6+S7)).  No shared memory, no block barrier:
// at this size (tens of MB per call) fixed per-stage overheads cost more than
// they hide.
// That is the canonical order of entmaxkv.h: selection is decided on these
// fp32 values, so nothing else may be fused or reordered (explicit
// round-to-nearest intrinsics throughout).
#include <type_traits>

#include "common.cuh"
#include "kernels.cuh"

namespace ekv {

constexpr int kScoreCTA = 512;

struct ZTable {
    float z[65];
};

template <typename T, int D, int G, bool GAUSS>
struct ScoreShape {
    static constexpr int ELT = GAUSS ? 4 : (int)sizeof(T);
    static constexpr int ROWB = D * ELT;                   // bytes of one metadata vector
    static constexpr int SW = D / 8;                       // slice width (coordinates)
    static constexpr int SLB = SW * ELT;                   // slice bytes (16, 32 or 64)
    static constexpr int NV = SLB / 16;                    // 16-byte loads per slice and vector
    static constexpr int HS = (G * SW + 63) / 64;          // head split: <= 64 query registers
    static constexpr int HPT = G / HS;                     // query heads per thread
    static constexpr int TPR = 8 * HS;                     // threads per row group
    static constexpr int CTA = (GAUSS || NV > 2) ? 256 : kScoreCTA;
    static constexpr int RG = CTA / TPR;                   // row groups per CTA
};

template <typename T>
struct RowVec;
template <>
struct RowVec<uint16_t> {   // 16 bytes = 8 bf16, widened exactly
    static constexpr int N = 8;
    EKV_DEV static void widen(const uint4& u, float (&f)[8])
    {
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            f[2 * i] = __uint_as_float(w[i] << 16);
            f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
        }
    }
};
template <>
struct RowVec<float> {      // 16 bytes = 4 fp32
    static constexpr int N = 4;
    EKV_DEV static void widen(const uint4& u, float (&f)[4])
    {
        f[0] = __uint_as_float(u.x); f[1] = __uint_as_float(u.y);
        f[2] = __uint_as_float(u.z); f[3] = __uint_as_float(u.w);
    }
};

struct ScoreArgs {
    const void* row_a;      // kmin (bbox) or mean (gauss)
    const void* row_b;      // kmax (bbox) or m2 (gauss)
    const float* q;
    int H_q, H_kv, ps, num_phys;
    const int32_t* page_table;
    int max_pages;
    const int32_t* seq_lens;
    int B;
    float scale;
    float* ub;              // bbox
    float* m_out;           // gauss
    float* v_out;
    float* e_out;
    int32_t* status;
};

// sum over the 8 slice lanes of a row: ((S0+S1)+(S2+S3))+((S4+S5)+(S6+S7))
EKV_DEV float slice_tree(float v)
{
    v = __fadd_rn(v, __shfl_xor_sync(0xffffffffu, v, 1));
    v = __fadd_rn(v, __shfl_xor_sync(0xffffffffu, v, 2));
    v = __fadd_rn(v, __shfl_xor_sync(0xffffffffu, v, 4));
    return v;
}

// Streaming kernel without shared memory or block barriers.  A row group of
// 8 (or 16) threads owns one kv head g for the whole launch and walks the
// (sequence, page) items j = first, first + step, ... of that head; thread k
// of the group owns d-slice k.  The page id and the metadata slices of the
// next item are loaded while the current one is computed.
template <typename T, int D, int G, bool GAUSS>
__global__ void __launch_bounds__(ScoreShape<T, D, G, GAUSS>::CTA, 1)
score_kernel(const ScoreArgs a, const ZTable zt)
{
    pdl_enter();
    using S = ScoreShape<T, D, G, GAUSS>;
    using E = typename std::conditional<GAUSS, float, T>::type;
    using V = RowVec<E>;
    const int tid = threadIdx.x;
    const int w = tid % S::TPR, ks = w & 7, hs = w >> 3;
    const int rg = blockIdx.x * S::RG + tid / S::TPR;      // global row group
    const int nrg = gridDim.x * S::RG;
    const int g = rg % a.H_kv;                             // kv head of this row group
    const int step = nrg / a.H_kv;                         // row groups per kv head
    const bool valid_rg = rg < step * a.H_kv;              // leftover groups only join the shuffles
    const int first = rg / a.H_kv;
    const int items = a.B * a.max_pages;                   // (sequence, page) pairs

    const float scale = a.scale;
    const float scale2 = __fmul_rn(scale, scale);
    const uint8_t* basea = static_cast<const uint8_t*>(a.row_a) + (size_t)g * S::ROWB + ks * S::SLB;
    const uint8_t* baseb = static_cast<const uint8_t*>(a.row_b) + (size_t)g * S::ROWB + ks * S::SLB;
    const size_t pstride = (size_t)a.H_kv * S::ROWB;       // bytes between physical pages

    float qreg[S::HPT][S::SW];
    int qb = -1;
    // item j -> (b, p, n, phys); phys < 0 for absent pages
    auto info = [&](int j, int& b, int& p, int& n, int& phys) {
        b = j / a.max_pages;
        p = j - b * a.max_pages;
        const int L = __ldg(&a.seq_lens[b]);
        const int P = pages_of(L, a.ps, a.max_pages, a.status);
        n = 0;
        phys = -1;
        if (p < P) {
            phys = __ldg(&a.page_table[(size_t)b * a.max_pages + p]);
            if (phys < 0 || phys >= a.num_phys) {
                if (w == 0) report(a.status, ENTMAXKV_DEVICE_BOUNDS);
                phys = -1;
            } else {
                n = min(a.ps, L - p * a.ps);
            }
        }
    };
    auto fetch = [&](int phys, uint4 (&ra)[S::NV], uint4 (&rb)[S::NV]) {
        if (phys >= 0) {
            const uint4* pa = reinterpret_cast<const uint4*>(basea + (size_t)phys * pstride);
            const uint4* pb = reinterpret_cast<const uint4*>(baseb + (size_t)phys * pstride);
#pragma unroll
            for (int c = 0; c < S::NV; ++c) {
                ra[c] = __ldg(pa + c);
                rb[c] = __ldg(pb + c);
            }
        }
    };

    int b = 0, p = 0, n = 0, phys = -1;
    uint4 ca[S::NV], cb[S::NV];
    if (valid_rg && first < items) {
        info(first, b, p, n, phys);
        fetch(phys, ca, cb);
    }
    // the trip count is uniform per warp (the shuffles below need every lane)
    for (int j = first;; j += step) {
        const bool live = valid_rg && j < items;
        if (!__any_sync(0xffffffffu, live)) break;
        // prefetch the next item
        int b2 = 0, p2 = 0, n2 = 0, phys2 = -1;
        uint4 na[S::NV], nb[S::NV];
        if (valid_rg && j + step < items) {
            info(j + step, b2, p2, n2, phys2);
            fetch(phys2, na, nb);
        }
        if (!live) n = 0;
        if (live && b != qb) {
            const float* qg = a.q + ((size_t)b * a.H_q + (size_t)g * G + hs * S::HPT) * D + ks * S::SW;
#pragma unroll
            for (int i = 0; i < S::HPT; ++i)
#pragma unroll
                for (int e = 0; e < S::SW; e += 4) {
                    const float4 f = __ldg(reinterpret_cast<const float4*>(qg + (size_t)i * D + e));
                    qreg[i][e] = f.x; qreg[i][e + 1] = f.y; qreg[i][e + 2] = f.z; qreg[i][e + 3] = f.w;
                }
            qb = b;
        }
        float acc[S::HPT], acc2[S::HPT];
#pragma unroll
        for (int i = 0; i < S::HPT; ++i) acc[i] = acc2[i] = 0.f;
        if (n > 0) {
#pragma unroll
            for (int c = 0; c < S::NV; ++c) {
                float fa[V::N], fb[V::N];
                V::widen(ca[c], fa);
                V::widen(cb[c], fb);
#pragma unroll
                for (int e = 0; e < V::N; ++e) {
#pragma unroll
                    for (int i = 0; i < S::HPT; ++i) {
                        const float qv = qreg[i][c * V::N + e];
                        if (!GAUSS) {
                            acc[i] = __fmaf_rn(qv, qv >= 0.f ? fb[e] : fa[e], acc[i]);
                        } else {
                            acc[i] = __fmaf_rn(qv, fa[e], acc[i]);
                            acc2[i] = __fmaf_rn(__fmul_rn(qv, qv), fb[e], acc2[i]);
                        }
                    }
                }
            }
        }
#pragma unroll
        for (int i = 0; i < S::HPT; ++i) {
            acc[i] = slice_tree(acc[i]);
            if (GAUSS) acc2[i] = slice_tree(acc2[i]);
        }
        if (!GAUSS) {
            float best = -INFINITY;
#pragma unroll
            for (int i = 0; i < S::HPT; ++i) {
                const float u = __fmul_rn(acc[i], scale);
                if (i == 0 || u > best) best = u;
            }
            if (S::HS > 1) best = fmaxf(best, __shfl_xor_sync(0xffffffffu, best, 8));
            if (best == 0.f) best = 0.f;   // -0 -> +0
            if (live && w == 0) a.ub[((size_t)b * a.H_kv + g) * a.max_pages + p] = n > 0 ? best : -INFINITY;
        } else if (live && ks == 0) {
            const float zn = zt.z[n];
#pragma unroll
            for (int i = 0; i < S::HPT; ++i) {
                const int h = hs * S::HPT + i;
                const size_t o = ((size_t)b * a.H_q + (size_t)g * G + h) * a.max_pages + p;
                if (n > 0) {
                    const float mm = __fmul_rn(acc[i], scale);
                    const float vv = __fmul_rn(__fdiv_rn(acc2[i], (float)n), scale2);
                    a.m_out[o] = mm;
                    a.v_out[o] = vv;
                    a.e_out[o] = __fmaf_rn(__fsqrt_rn(vv), zn, mm);
                } else {
                    a.m_out[o] = -INFINITY;
                    a.v_out[o] = 0.f;
                    a.e_out[o] = -INFINITY;
                }
            }
        }
        b = b2; p = p2; n = n2; phys = phys2;
#pragma unroll
        for (int c = 0; c < S::NV; ++c) {
            ca[c] = na[c];
            cb[c] = nb[c];
        }
    }
}

template <typename T, int D, int G, bool GAUSS>
static int launch_score_t(const ScoreArgs& a, const ZTable& zt, cudaStream_t stream)
{
    using S = ScoreShape<T, D, G, GAUSS>;
    static int occ[64] = {0};                              // resident CTAs per SM, per device
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) dev = 0;
    if (occ[dev] == 0) {
        int n = 1;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, score_kernel<T, D, G, GAUSS>, S::CTA, 0) !=
                cudaSuccess || n < 1)
            n = 1;
        occ[dev] = n;
    }
    const long long rows = (long long)a.B * a.max_pages * a.H_kv;
    const long long want = (rows + S::RG - 1) / S::RG;
    const int grid = (int)std::max<long long>(1, std::min<long long>(want, (long long)occ[dev] * num_sms()));
    if ((long long)grid * S::RG < a.H_kv) return ENTMAXKV_UNSUPPORTED;   // at least one group per kv head
    launch_pdl(score_kernel<T, D, G, GAUSS>, dim3(grid), dim3(S::CTA), 0, stream, a, zt);
    return cudaGetLastError() == cudaSuccess ? ENTMAXKV_OK : ENTMAXKV_CUDA_ERROR;
}

template <typename T, int D, bool GAUSS>
static int dispatch_g(int G, const ScoreArgs& a, const ZTable& zt, cudaStream_t st)
{
    switch (G) {
        case 1: return launch_score_t<T, D, 1, GAUSS>(a, zt, st);
        case 2: return launch_score_t<T, D, 2, GAUSS>(a, zt, st);
        case 4: return launch_score_t<T, D, 4, GAUSS>(a, zt, st);
        default: return launch_score_t<T, D, 8, GAUSS>(a, zt, st);
    }
}

int launch_score(const entmaxkv_pool& pool, const float* q, int H_q, const int32_t* page_table,
                 int max_pages, const int32_t* seq_lens, int B, int mode, float scale, float* ub, float* m,
                 float* v, float* est, int32_t* status, cudaStream_t stream)
{
    const int G = H_q / pool.H_kv;
    ScoreArgs a{};
    a.q = q;
    a.H_q = H_q;
    a.H_kv = pool.H_kv;
    a.ps = pool.ps;
    a.num_phys = pool.num_phys_pages;
    a.page_table = page_table;
    a.max_pages = max_pages;
    a.seq_lens = seq_lens;
    a.B = B;
    a.scale = scale;
    a.ub = ub;
    a.m_out = m;
    a.v_out = v;
    a.e_out = est;
    a.status = status;
    // z_n = fp32(sqrt(2 ln n)), n >= 2; z_0 = z_1 = 0 (Gaussian expected
    // maximum of n draws, in units of the standard deviation)
    ZTable zt;
    for (int n = 0; n <= 64; ++n) zt.z[n] = n >= 2 ? (float)std::sqrt(2.0 * std::log((double)n)) : 0.0f;
    if (mode == ENTMAXKV_SCORE_BBOX) {
        a.row_a = pool.kmin;
        a.row_b = pool.kmax;
        if (pool.dtype == ENTMAXKV_BF16)
            return pool.d == 128 ? dispatch_g<uint16_t, 128, false>(G, a, zt, stream)
                                 : dispatch_g<uint16_t, 64, false>(G, a, zt, stream);
        return pool.d == 128 ? dispatch_g<float, 128, false>(G, a, zt, stream)
                             : dispatch_g<float, 64, false>(G, a, zt, stream);
    }
    a.row_a = pool.mean;
    a.row_b = pool.m2;
    return pool.d == 128 ? dispatch_g<float, 128, true>(G, a, zt, stream)
                         : dispatch_g<float, 64, true>(G, a, zt, stream);
}

}  // namespace ekv
