// Candidate page selection.
//
// EntmaxKV (German technical summary, section 2.B):
//  policy 1, top-k: a fixed budget of the k pages with the highest
//    bounding-box bounds;
//  policy 2, Gaussian-aware entmax selection: estimate the entmax threshold
//    tau_hat from page statistics by solving an approximate normalisation
//    equation, then keep the pages whose estimated maximum score clears
//    tau_hat minus a safety margin Delta.
//
// Top-k runs one CTA per (sequence, kv head).  It finds the k-th key in the
// order (key desc, page asc) by value bucketing: a histogram over a linear
// map of [min, max] (monotone, so buckets keep the key order), the bucket
// holding the k-th key is narrowed until it holds few enough keys to rank
// them exactly.  The kept pages are then emitted in page order with a block
// scan, so the list comes out sorted.
#include "common.cuh"
#include "kernels.cuh"

namespace ekv {

constexpr int kSelThreads = 1024;
constexpr int kBins = 2048;
constexpr int kRankCap = 1024;

// Inclusive block scan (sum) of one int per thread, 1024 threads.
EKV_DEV int block_scan_incl(int v, int* wsum)
{
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += t;
    }
    __syncthreads();
    if (lane == 31) wsum[w] = v;
    __syncthreads();
    if (w == 0) {
        int t = lane < (int)(blockDim.x >> 5) ? wsum[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int u = __shfl_up_sync(0xffffffffu, t, o);
            if (lane >= o) t += u;
        }
        wsum[lane] = t;
    }
    __syncthreads();
    return v + (w > 0 ? wsum[w - 1] : 0);
}

struct TopkShared {
    int hist[kBins];
    unsigned long long cand[kRankCap];
    int wsum[32];
    float redf[32];
    int ncand;
    int bucket;
    int need;
    unsigned int thr_key;
    int thr_idx;
};

__global__ void __launch_bounds__(kSelThreads)
topk_kernel(const float* __restrict__ ub, const int32_t* __restrict__ seq_lens, int ps, int H_kv,
            int max_pages, int budget, float budget_frac, int k_max, int32_t* __restrict__ sel,
            int32_t* __restrict__ sel_count, int32_t* status)
{
    pdl_enter();
    __shared__ TopkShared sh;
    const int b = blockIdx.y, g = blockIdx.x, tid = threadIdx.x;
    const int L = seq_lens[b];
    const int P = pages_of(L, ps, max_pages, status);
    int k = budget >= 0 ? budget : (int)ceil((double)budget_frac * (double)P);
    k = min(k, P);
    if (k > k_max) {
        if (tid == 0) report(status, ENTMAXKV_DEVICE_BOUNDS);
        k = k_max;
    }
    const float* keys = ub + ((size_t)b * H_kv + g) * max_pages;
    int32_t* out = sel + ((size_t)b * H_kv + g) * k_max;
    if (k <= 0 || k >= P) {
        const int n = k <= 0 ? 0 : P;
        for (int i = tid; i < n; i += kSelThreads) out[i] = i;
        if (tid == 0) sel_count[(size_t)b * H_kv + g] = n;
        return;
    }

    // --- find the k-th key (thr_key, thr_idx) in the order (key desc, index asc)
    float lo_v = -INFINITY, hi_v = INFINITY;   // current value range [lo_v, hi_v]
    int need = k;
    bool done = false;
    unsigned int thr_key = 0;
    int thr_idx = 0;
    for (int round = 0; round < 8 && !done; ++round) {
        float mn = INFINITY, mx = -INFINITY;
        for (int i = tid; i < P; i += kSelThreads) {
            float v = keys[i];
            if (v == 0.f) v = 0.f;
            if (v >= lo_v && v <= hi_v) { mn = fminf(mn, v); mx = fmaxf(mx, v); }
        }
        mn = block_min(mn, sh.redf);
        mx = block_max(mx, sh.redf);
        if (mn == mx) {
            // every key in range is equal: the need-th lowest index among them
            thr_key = ordered_key(mn);
            const int per = (P + kSelThreads - 1) / kSelThreads;
            const int i0 = tid * per, i1 = min(P, i0 + per);
            int c = 0;
            for (int i = i0; i < i1; ++i) {
                float v = keys[i];
                if (v == 0.f) v = 0.f;
                c += (v == mn);
            }
            const int incl = block_scan_incl(c, sh.wsum);
            int before = incl - c;
            for (int i = i0; i < i1; ++i) {
                float v = keys[i];
                if (v == 0.f) v = 0.f;
                if (v == mn) {
                    if (before == need - 1) sh.thr_idx = i;
                    ++before;
                }
            }
            __syncthreads();
            thr_idx = sh.thr_idx;
            done = true;
            break;
        }
        const float w = (float)kBins / (mx - mn);
        for (int i = tid; i < kBins; i += kSelThreads) sh.hist[i] = 0;
        __syncthreads();
        for (int i = tid; i < P; i += kSelThreads) {
            float v = keys[i];
            if (v == 0.f) v = 0.f;
            if (v >= mn && v <= mx) {
                const int bk = (int)fminf((v - mn) * w, (float)(kBins - 1));
                atomicAdd(&sh.hist[bk], 1);
            }
        }
        __syncthreads();
        // suffix counts: thread t owns bins kBins-1-2t and kBins-2-2t (descending)
        const int bA = kBins - 1 - 2 * tid, bB = bA - 1;
        const int cA = sh.hist[bA], cB = sh.hist[bB];
        const int incl = block_scan_incl(cA + cB, sh.wsum);
        const int above = incl - cA - cB;   // keys in bins > bA
        if (above < need && need <= above + cA) {
            sh.bucket = bA;
            sh.need = need - above;
        } else if (above + cA < need && need <= above + cA + cB) {
            sh.bucket = bB;
            sh.need = need - above - cA;
        }
        __syncthreads();
        const int T = sh.bucket;
        need = sh.need;
        // value range of bucket T
        float bmn = INFINITY, bmx = -INFINITY;
        for (int i = tid; i < P; i += kSelThreads) {
            float v = keys[i];
            if (v == 0.f) v = 0.f;
            if (v >= mn && v <= mx && (int)fminf((v - mn) * w, (float)(kBins - 1)) == T) {
                bmn = fminf(bmn, v);
                bmx = fmaxf(bmx, v);
            }
        }
        bmn = block_min(bmn, sh.redf);
        bmx = block_max(bmx, sh.redf);
        lo_v = bmn;
        hi_v = bmx;
        const int cnt = sh.hist[T];
        if (cnt <= kRankCap && bmn != bmx) {
            if (tid == 0) sh.ncand = 0;
            __syncthreads();
            for (int i = tid; i < P; i += kSelThreads) {
                float v = keys[i];
                if (v == 0.f) v = 0.f;
                if (v >= lo_v && v <= hi_v) {
                    const int slot = atomicAdd(&sh.ncand, 1);
                    if (slot < kRankCap)
                        sh.cand[slot] = ((unsigned long long)ordered_key(v) << 32) |
                                        (unsigned long long)(0xFFFFFFFFu - (unsigned)i);
                }
            }
            __syncthreads();
            const int nc = min(sh.ncand, kRankCap);
            if (tid < nc) {
                const unsigned long long me = sh.cand[tid];
                int rank = 0;
                for (int j = 0; j < nc; ++j) rank += (sh.cand[j] > me);
                if (rank == need - 1) {
                    sh.thr_key = (unsigned)(me >> 32);
                    sh.thr_idx = (int)(0xFFFFFFFFu - (unsigned)(me & 0xFFFFFFFFull));
                }
            }
            __syncthreads();
            thr_key = sh.thr_key;
            thr_idx = sh.thr_idx;
            done = true;
        }
        __syncthreads();
    }
    if (!done) {   // cannot happen for finite keys; keep the output well formed
        if (tid == 0) report(status, ENTMAXKV_DEVICE_BOUNDS);
        thr_key = 0xFFFFFFFFu;
        thr_idx = -1;
    }

    // --- emit kept pages in page order
    const int per = (P + kSelThreads - 1) / kSelThreads;
    const int i0 = tid * per, i1 = min(P, i0 + per);
    int c = 0;
    for (int i = i0; i < i1; ++i) {
        const unsigned kk = ordered_key(keys[i]);
        c += (kk > thr_key) || (kk == thr_key && i <= thr_idx);
    }
    const int incl = block_scan_incl(c, sh.wsum);
    int pos = incl - c;
    for (int i = i0; i < i1; ++i) {
        const unsigned kk = ordered_key(keys[i]);
        if ((kk > thr_key) || (kk == thr_key && i <= thr_idx)) {
            if (pos < k_max) out[pos] = i;
            ++pos;
        }
    }
    if (tid == kSelThreads - 1) {
        if (incl != k) report(status, ENTMAXKV_DEVICE_BOUNDS);
        sel_count[(size_t)b * H_kv + g] = min(incl, k_max);
    }
}

// Register-resident variant: thread t holds keys [t*KPT, (t+1)*KPT) (ordered
// integer form, -0 as +0); the same bucket narrowing and index-ordered
// emission as topk_kernel, without returning to memory between passes.
template <int KPT>
__global__ void __launch_bounds__(kSelThreads, 1)
topk_reg_kernel(const float* __restrict__ ub, const int32_t* __restrict__ seq_lens, int ps, int H_kv,
                int max_pages, int budget, float budget_frac, int k_max, int32_t* __restrict__ sel,
                int32_t* __restrict__ sel_count, int32_t* status)
{
    pdl_enter();
    __shared__ TopkShared sh;
    const int b = blockIdx.y, g = blockIdx.x, tid = threadIdx.x;
    const int L = seq_lens[b];
    const int P = pages_of(L, ps, max_pages, status);
    int k = budget >= 0 ? budget : (int)ceil((double)budget_frac * (double)P);
    k = min(k, P);
    if (k > k_max) {
        if (tid == 0) report(status, ENTMAXKV_DEVICE_BOUNDS);
        k = k_max;
    }
    const float* keys = ub + ((size_t)b * H_kv + g) * max_pages;
    int32_t* out = sel + ((size_t)b * H_kv + g) * k_max;
    if (k <= 0 || k >= P) {
        const int n = k <= 0 ? 0 : P;
        for (int i = tid; i < n; i += kSelThreads) out[i] = i;
        if (tid == 0) sel_count[(size_t)b * H_kv + g] = n;
        return;
    }
    // keys of this thread (absent entries become the smallest float)
    const int i0 = tid * KPT;
    float kv[KPT];
#pragma unroll
    for (int e = 0; e < KPT; ++e) {
        const int i = i0 + e;
        float v = i < P ? __ldg(keys + i) : -INFINITY;
        if (v == 0.f) v = 0.f;
        kv[e] = v;
    }
    auto inr = [&](int e, float lo, float hi) { return i0 + e < P && kv[e] >= lo && kv[e] <= hi; };

    float lo_v = -INFINITY, hi_v = INFINITY;
    int need = k;
    bool done = false;
    unsigned int thr_key = 0;
    int thr_idx = 0;
    for (int round = 0; round < 8 && !done; ++round) {
        float mn = INFINITY, mx = -INFINITY;
#pragma unroll
        for (int e = 0; e < KPT; ++e)
            if (inr(e, lo_v, hi_v)) {
                mn = fminf(mn, kv[e]);
                mx = fmaxf(mx, kv[e]);
            }
        mn = block_min(mn, sh.redf);
        mx = block_max(mx, sh.redf);
        if (mn == mx) {
            thr_key = ordered_key(mn);
            int c = 0;
#pragma unroll
            for (int e = 0; e < KPT; ++e) c += inr(e, mn, mn);
            const int incl = block_scan_incl(c, sh.wsum);
            int before = incl - c;
#pragma unroll
            for (int e = 0; e < KPT; ++e)
                if (inr(e, mn, mn)) {
                    if (before == need - 1) sh.thr_idx = i0 + e;
                    ++before;
                }
            __syncthreads();
            thr_idx = sh.thr_idx;
            done = true;
            break;
        }
        const float w = (float)kBins / (mx - mn);
        for (int i = tid; i < kBins; i += kSelThreads) sh.hist[i] = 0;
        __syncthreads();
        // bucket of key e in this round (-1 when outside the range); recomputed, not stored
        auto bucket = [&](int e) { return inr(e, mn, mx) ? (int)fminf((kv[e] - mn) * w, (float)(kBins - 1)) : -1; };
#pragma unroll
        for (int e = 0; e < KPT; ++e) {
            const int bk = bucket(e);
            if (bk >= 0) atomicAdd(&sh.hist[bk], 1);
        }
        __syncthreads();
        const int bA = kBins - 1 - 2 * tid, bB = bA - 1;
        const int cA = sh.hist[bA], cB = sh.hist[bB];
        const int incl = block_scan_incl(cA + cB, sh.wsum);
        const int above = incl - cA - cB;
        if (above < need && need <= above + cA) {
            sh.bucket = bA;
            sh.need = need - above;
        } else if (above + cA < need && need <= above + cA + cB) {
            sh.bucket = bB;
            sh.need = need - above - cA;
        }
        __syncthreads();
        const int T = sh.bucket;
        need = sh.need;
        float bmn = INFINITY, bmx = -INFINITY;
#pragma unroll
        for (int e = 0; e < KPT; ++e)
            if (bucket(e) == T) {
                bmn = fminf(bmn, kv[e]);
                bmx = fmaxf(bmx, kv[e]);
            }
        bmn = block_min(bmn, sh.redf);
        bmx = block_max(bmx, sh.redf);
        lo_v = bmn;
        hi_v = bmx;
        const int cnt = sh.hist[T];
        if (cnt <= kRankCap && bmn != bmx) {
            if (tid == 0) sh.ncand = 0;
            __syncthreads();
#pragma unroll
            for (int e = 0; e < KPT; ++e)
                if (bucket(e) == T) {
                    const int slot = atomicAdd(&sh.ncand, 1);
                    if (slot < kRankCap)
                        sh.cand[slot] = ((unsigned long long)ordered_key(kv[e]) << 32) |
                                        (unsigned long long)(0xFFFFFFFFu - (unsigned)(i0 + e));
                }
            __syncthreads();
            const int nc = min(sh.ncand, kRankCap);
            if (tid < nc) {
                const unsigned long long me = sh.cand[tid];
                int rank = 0;
                for (int j = 0; j < nc; ++j) rank += (sh.cand[j] > me);
                if (rank == need - 1) {
                    sh.thr_key = (unsigned)(me >> 32);
                    sh.thr_idx = (int)(0xFFFFFFFFu - (unsigned)(me & 0xFFFFFFFFull));
                }
            }
            __syncthreads();
            thr_key = sh.thr_key;
            thr_idx = sh.thr_idx;
            done = true;
        }
        __syncthreads();
    }
    if (!done) {
        if (tid == 0) report(status, ENTMAXKV_DEVICE_BOUNDS);
        thr_key = 0xFFFFFFFFu;
        thr_idx = -1;
    }
    int c = 0;
#pragma unroll
    for (int e = 0; e < KPT; ++e) {
        const unsigned kk = ordered_key(kv[e]);
        c += (i0 + e < P) && ((kk > thr_key) || (kk == thr_key && i0 + e <= thr_idx));
    }
    const int incl = block_scan_incl(c, sh.wsum);
    int pos = incl - c;
#pragma unroll
    for (int e = 0; e < KPT; ++e) {
        const unsigned kk = ordered_key(kv[e]);
        if ((i0 + e < P) && ((kk > thr_key) || (kk == thr_key && i0 + e <= thr_idx))) {
            if (pos < k_max) out[pos] = i0 + e;
            ++pos;
        }
    }
    if (tid == kSelThreads - 1) {
        if (incl != k) report(status, ENTMAXKV_DEVICE_BOUNDS);
        sel_count[(size_t)b * H_kv + g] = min(incl, k_max);
    }
}

// ---------------------------------------------------------------- Gaussian
//
// tau_hat per (sequence, query head): root of
//   F(tau) = sum_p n_p E[((alpha-1) s_p - tau)_+^(1/(alpha-1))] - 1,
// s_p ~ N(m_p, v_p), by bracketed Newton steps (F is convex and decreasing,
// so a Newton step from the left never passes the root); a step that leaves
// the bracket is replaced by bisection.

constexpr int kTauThreads = 512;

EKV_DEV void gauss_term(float mp, float sp, float tau, bool a2, float& g, float& dg)
{
    const float u = mp - tau;
    if (sp > 0.f) {
        const float z = u / sp;
        if (z < -12.f) { g = 0.f; dg = 0.f; return; }
        const float Phi = normcdff(z);
        const float phi = 0.3989422804014327f * expf(-0.5f * z * z);
        if (a2) {            // E[(X - tau)_+], d/dtau = -Phi
            g = fmaf(u, Phi, sp * phi);
            dg = Phi;
        } else {             // E[(X - tau)_+^2], d/dtau = -2 E[(X - tau)_+]
            g = fmaf(fmaf(u, u, sp * sp), Phi, u * sp * phi);
            dg = 2.f * fmaf(u, Phi, sp * phi);
        }
    } else {
        const float up = fmaxf(u, 0.f);
        g = a2 ? up : up * up;
        dg = a2 ? (u > 0.f ? 1.f : 0.f) : 2.f * up;
    }
}

__global__ void __launch_bounds__(kTauThreads)
gauss_tau_kernel(const float* __restrict__ m, const float* __restrict__ v, const int32_t* __restrict__ seq_lens,
                 int ps, int H_q, int max_pages, float alpha, float* __restrict__ tau_hat)
{
    pdl_enter();
    __shared__ double red[kTauThreads / 32];
    __shared__ float redf[kTauThreads / 32];
    const int b = blockIdx.y, h = blockIdx.x, tid = threadIdx.x;
    const int L = seq_lens[b];
    const int P = pages_of(L, ps, max_pages, nullptr);
    const float am1 = alpha - 1.0f;
    const bool a2 = alpha == 2.0f;
    const float* mh = m + ((size_t)b * H_q + h) * max_pages;
    const float* vh = v + ((size_t)b * H_q + h) * max_pages;
    if (P == 0) {
        if (tid == 0) tau_hat[(size_t)b * H_q + h] = INFINITY;
        return;
    }
    float mx = -INFINITY;
    for (int p = tid; p < P; p += kTauThreads) mx = fmaxf(mx, am1 * mh[p]);
    mx = block_max(mx, redf);
    double lo = (double)mx - 1.0;   // F(lo) >= 1 (Jensen: the top page alone gives >= 1)
    double hi = INFINITY;
    double tau = lo;
    for (int it = 0; it < 60; ++it) {
        double F = 0.0, dF = 0.0;
        const float tf = (float)tau;
        for (int p = tid; p < P; p += kTauThreads) {
            const float mp = am1 * mh[p];
            const float sp = am1 * sqrtf(fmaxf(vh[p], 0.f));
            const int n = min(ps, L - p * ps);
            float gv, dg;
            gauss_term(mp, sp, tf, a2, gv, dg);
            F += (double)n * gv;
            dF += (double)n * dg;
        }
        F = block_sum(F, red);
        dF = block_sum(dF, red);
        if (F >= 1.0) lo = tau; else hi = tau;
        if (fabs(F - 1.0) < 1e-7 || (hi - lo) < 1e-7 * fmax(1.0, fabs(tau))) break;
        double nt = dF > 0.0 ? tau + (F - 1.0) / dF : INFINITY;
        if (!(nt > lo && nt < hi)) nt = isinf(hi) ? lo + fmax(1.0, 2.0 * (tau - lo + 0.5)) : 0.5 * (lo + hi);
        tau = nt;
    }
    if (tid == 0) tau_hat[(size_t)b * H_q + h] = (float)tau;
}

template <int G>
__global__ void __launch_bounds__(kSelThreads)
gauss_keep_kernel(const float* __restrict__ est, const float* __restrict__ tau_hat,
                  const int32_t* __restrict__ seq_lens, int ps, int H_q, int H_kv, int max_pages,
                  float alpha, float delta, int k_max, int32_t* __restrict__ sel, int32_t* __restrict__ sel_count,
                  int32_t* status)
{
    pdl_enter();
    __shared__ int wsum[32];
    const int b = blockIdx.y, g = blockIdx.x, tid = threadIdx.x;
    const int L = seq_lens[b];
    const int P = pages_of(L, ps, max_pages, status);
    const float am1 = alpha - 1.0f;
    float rhs[G];
#pragma unroll
    for (int h = 0; h < G; ++h) rhs[h] = __fsub_rn(tau_hat[(size_t)b * H_q + g * G + h], delta);
    const float* e0 = est + ((size_t)b * H_q + (size_t)g * G) * max_pages;
    const int per = (P + kSelThreads - 1) / kSelThreads;
    const int i0 = tid * per, i1 = min(P, i0 + per);
    int c = 0;
    for (int i = i0; i < i1; ++i) {
        bool keep = false;
#pragma unroll
        for (int h = 0; h < G; ++h) keep |= __fmul_rn(am1, e0[(size_t)h * max_pages + i]) >= rhs[h];
        c += keep;
    }
    const int incl = block_scan_incl(c, wsum);
    int pos = incl - c;
    int32_t* out = sel + ((size_t)b * H_kv + g) * k_max;
    for (int i = i0; i < i1; ++i) {
        bool keep = false;
#pragma unroll
        for (int h = 0; h < G; ++h) keep |= __fmul_rn(am1, e0[(size_t)h * max_pages + i]) >= rhs[h];
        if (keep) {
            if (pos < k_max) out[pos] = i;
            ++pos;
        }
    }
    if (tid == kSelThreads - 1) {
        if (incl > k_max) report(status, ENTMAXKV_DEVICE_BOUNDS);
        sel_count[(size_t)b * H_kv + g] = min(incl, k_max);
    }
}

int launch_select(int mode, const float* ub, const float* m, const float* v, const float* est,
                  const int32_t* seq_lens, int ps, int B, int H_q, int H_kv, int max_pages, int budget,
                  float budget_frac, float alpha, float delta, int k_max, int32_t* sel, int32_t* sel_count,
                  float* tau_hat, int32_t* status, cudaStream_t stream)
{
    if (mode == ENTMAXKV_SELECT_TOPK) {
        // every sequence has at most max_pages pages: pick the register width from it
        const dim3 grid(H_kv, B), block(kSelThreads);
        if (max_pages <= 4 * kSelThreads)
            launch_pdl(topk_reg_kernel<4>, grid, block, 0, stream, ub, seq_lens, ps, H_kv, max_pages, budget,
                       budget_frac, k_max, sel, sel_count, status);
        else if (max_pages <= 8 * kSelThreads)
            launch_pdl(topk_reg_kernel<8>, grid, block, 0, stream, ub, seq_lens, ps, H_kv, max_pages, budget,
                       budget_frac, k_max, sel, sel_count, status);
        else if (max_pages <= 16 * kSelThreads)
            launch_pdl(topk_reg_kernel<16>, grid, block, 0, stream, ub, seq_lens, ps, H_kv, max_pages, budget,
                       budget_frac, k_max, sel, sel_count, status);
        else if (max_pages <= 20 * kSelThreads)
            launch_pdl(topk_reg_kernel<20>, grid, block, 0, stream, ub, seq_lens, ps, H_kv, max_pages, budget,
                       budget_frac, k_max, sel, sel_count, status);
        else
            launch_pdl(topk_kernel, grid, block, 0, stream, ub, seq_lens, ps, H_kv, max_pages, budget, budget_frac,
                       k_max, sel, sel_count, status);
    } else {
        launch_pdl(gauss_tau_kernel, dim3(dim3(H_q, B)), dim3(kTauThreads), 0, stream, m, v, seq_lens, ps, H_q, max_pages, alpha,
                                                                   tau_hat);
        if (cudaGetLastError() != cudaSuccess) return ENTMAXKV_CUDA_ERROR;
        const int G = H_q / H_kv;
#define EKV_KEEP(GG)                                                                                    \
    launch_pdl(gauss_keep_kernel<GG>, dim3(dim3(H_kv, B)), dim3(kSelThreads), 0, stream, est, tau_hat, seq_lens, ps, H_q, \
                                                                     H_kv, max_pages, alpha, delta,    \
                                                                     k_max, sel, sel_count, status)
        switch (G) {
            case 1: EKV_KEEP(1); break;
            case 2: EKV_KEEP(2); break;
            case 4: EKV_KEEP(4); break;
            default: EKV_KEEP(8); break;
        }
#undef EKV_KEEP
    }
    return cudaGetLastError() == cudaSuccess ? ENTMAXKV_OK : ENTMAXKV_CUDA_ERROR;
}

}  // namespace ekv
