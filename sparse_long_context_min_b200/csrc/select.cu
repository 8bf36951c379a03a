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
    unsigned int redk[32];
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

    // --- find the k-th key (thr_key, thr_idx) in the order (key desc, index asc),
    // on ordered 32-bit keys (monotone in the float order, -0 as +0, infinities
    // included); buckets are a float multiple of the offset from the minimum
    auto key_at = [&](int i) { return ordered_key(keys[i]); };
    auto bmin = [&](unsigned int v) {
        v = __reduce_min_sync(0xffffffffu, v);
        __syncthreads();
        if ((tid & 31) == 0) sh.redk[tid >> 5] = v;
        __syncthreads();
        return __reduce_min_sync(0xffffffffu, sh.redk[tid & 31]);
    };
    auto bmax = [&](unsigned int v) {
        v = __reduce_max_sync(0xffffffffu, v);
        __syncthreads();
        if ((tid & 31) == 0) sh.redk[tid >> 5] = v;
        __syncthreads();
        return __reduce_max_sync(0xffffffffu, sh.redk[tid & 31]);
    };
    unsigned int lo_k = 0u, hi_k = 0xFFFFFFFFu;   // current key range [lo_k, hi_k]
    int need = k;
    bool done = false;
    unsigned int thr_key = 0;
    int thr_idx = 0;
    for (int round = 0; round < 8 && !done; ++round) {
        unsigned int mn = 0xFFFFFFFFu, mx = 0u;
        for (int i = tid; i < P; i += kSelThreads) {
            const unsigned int v = key_at(i);
            if (v >= lo_k && v <= hi_k) { mn = min(mn, v); mx = max(mx, v); }
        }
        mn = bmin(mn);
        mx = bmax(mx);
        if (mn == mx) {
            // every key in range is equal: the need-th lowest index among them
            thr_key = mn;
            const int per = (P + kSelThreads - 1) / kSelThreads;
            const int i0 = tid * per, i1 = min(P, i0 + per);
            int c = 0;
            for (int i = i0; i < i1; ++i) c += (key_at(i) == mn);
            const int incl = block_scan_incl(c, sh.wsum);
            int before = incl - c;
            for (int i = i0; i < i1; ++i)
                if (key_at(i) == mn) {
                    if (before == need - 1) sh.thr_idx = i;
                    ++before;
                }
            __syncthreads();
            thr_idx = sh.thr_idx;
            done = true;
            break;
        }
        const float w = (float)kBins / ((float)(mx - mn) + 1.0f);
        auto bucket_of = [&](unsigned int v) { return min((int)((float)(v - mn) * w), kBins - 1); };
        for (int i = tid; i < kBins; i += kSelThreads) sh.hist[i] = 0;
        __syncthreads();
        for (int i = tid; i < P; i += kSelThreads) {
            const unsigned int v = key_at(i);
            if (v >= mn && v <= mx) atomicAdd(&sh.hist[bucket_of(v)], 1);
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
        // key range of bucket T
        unsigned int bmn = 0xFFFFFFFFu, bmx = 0u;
        for (int i = tid; i < P; i += kSelThreads) {
            const unsigned int v = key_at(i);
            if (v >= mn && v <= mx && bucket_of(v) == T) {
                bmn = min(bmn, v);
                bmx = max(bmx, v);
            }
        }
        bmn = bmin(bmn);
        bmx = bmax(bmx);
        lo_k = bmn;
        hi_k = bmx;
        const int cnt = sh.hist[T];
        if (cnt <= kRankCap && bmn != bmx) {
            if (tid == 0) sh.ncand = 0;
            __syncthreads();
            for (int i = tid; i < P; i += kSelThreads) {
                const unsigned int v = key_at(i);
                if (v >= lo_k && v <= hi_k) {
                    const int slot = atomicAdd(&sh.ncand, 1);
                    if (slot < kRankCap)
                        sh.cand[slot] = ((unsigned long long)v << 32) |
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
    if (!done) {   // cannot happen (a few rounds reach one value); keep the output well formed
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

// Cluster variant: the keys of one (sequence, kv head) are spread over a
// cluster of kTopkCTAs CTAs, thread t of CTA r holding keys
// [(r*kCThreads + t)*KPT, ... + KPT) in registers, so that every pass over the
// keys runs on kTopkCTAs SMs.  Each round publishes per-CTA partial results
// (range, histogram, candidates, counts) in shared memory and every CTA reads
// all of them through distributed shared memory, so all CTAs take identical
// decisions and meet the same cluster barriers.
//  round: [min, max] of the keys in play (as ordered 32-bit keys); if equal,
//         the keys in play are tied and the `need` lowest indices among them
//         are kept; otherwise a 512-bin histogram over a linear map of
//         [min, max] gives the
//         bucket T holding the need-th key; if T holds at most kCCap keys
//         they are gathered and ranked exactly (all pairs compared), else
//         the next round narrows to T.
//  The keys are read coalesced into shared memory, then each thread takes
//  its KPT consecutive ones.
//  emit:  kept pages in page order, offset by the kept counts of the CTAs
//         of lower rank.
constexpr int kTopkCTAs = 8;
constexpr int kCThreads = 512;
constexpr int kCBins = kCThreads; // one bin per thread
constexpr int kCCap = 128;      // exact ranking is quadratic: larger buckets narrow once more
constexpr int kCRounds = 40;     // each round shrinks the key range about 512-fold: a few rounds reach one value

struct TopkClusterShared {
    __align__(16) int hist[kCBins];          // this CTA's histogram of the round
    int tot[kCBins / kTopkCTAs];             // cluster totals of this CTA's slice of the bins
    unsigned long long lc[kCCap];            // this CTA's keys of the threshold bucket
    unsigned long long mc[kCCap];            // the whole cluster's, merged
    int wsum[32];
    unsigned int redk[2][32];
    unsigned int pub_mm[2];                  // this CTA's range of the keys in play (ordered keys)
    unsigned int g_mm[2];
    int lcn;                                 // entries of lc
    int pub_tie;                             // this CTA's tied keys (tie round)
    int pub_kept;                            // this CTA's kept keys
    int mc_off[kTopkCTAs + 1];
    int before, total;
    int T, need, cT;
    unsigned int thr_key;
    int thr_idx;
};

template <int KPT>
__global__ void __launch_bounds__(kCThreads)
topk_cluster_kernel(const float* __restrict__ ub, const int32_t* __restrict__ seq_lens, int ps, int H_kv,
                    int max_pages, int budget, float budget_frac, int k_max, int32_t* __restrict__ sel,
                    int32_t* __restrict__ sel_count, int32_t* status)
{
    pdl_enter();
    __shared__ TopkClusterShared sh;
    constexpr int C = kTopkCTAs;
    const int r = (int)cluster_rank();
    const int b = blockIdx.y, g = blockIdx.x / C, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int L = seq_lens[b];
    const int P = pages_of(L, ps, max_pages, r == 0 ? status : nullptr);
    int k = budget >= 0 ? budget : (int)ceil((double)budget_frac * (double)P);
    k = min(k, P);
    if (k > k_max) {
        if (tid == 0 && r == 0) report(status, ENTMAXKV_DEVICE_BOUNDS);
        k = k_max;
    }
    const float* keys = ub + ((size_t)b * H_kv + g) * max_pages;
    int32_t* out = sel + ((size_t)b * H_kv + g) * k_max;
    if (k <= 0 || k >= P) {   // the same on every CTA of the cluster: no barrier is met
        const int n = k <= 0 ? 0 : P;
        for (int i = r * kCThreads + tid; i < n; i += C * kCThreads) out[i] = i;
        if (tid == 0 && r == 0) sel_count[(size_t)b * H_kv + g] = n;
        return;
    }
    const int i0 = (r * kCThreads + tid) * KPT;
    __shared__ unsigned int kst[kCThreads * KPT];
#pragma unroll
    for (int e = 0; e < KPT; ++e) {
        const int i = r * kCThreads * KPT + e * kCThreads + tid;
        kst[e * kCThreads + tid] = i < P ? ordered_key(__ldg(keys + i)) : 0u;
    }
    __syncthreads();
    unsigned int kv[KPT];                 // ordered keys (-0 as +0), page order
#pragma unroll
    for (int e = 0; e < KPT; ++e) kv[e] = kst[tid * KPT + e];
    // keys in play: valid, inside [lo_k, hi_k] and in bucket pT of the previous
    // round's map (plo, pw); round 0 takes every valid key.  Buckets are a
    // float multiple of the ordered-key offset: monotone, so they keep the key
    // order, and infinities need no special case.
    unsigned int lo_k = 0u, hi_k = 0xFFFFFFFFu, plo = 0u;
    float pw = 0.f;
    int pT = -1;
    auto bucket_of = [](unsigned int v, unsigned int lo, float w) {
        return min((int)((float)(v - lo) * w), kCBins - 1);
    };
    auto inplay = [&](int e) {
        if (!(i0 + e < P && kv[e] >= lo_k && kv[e] <= hi_k)) return false;
        return pT < 0 || bucket_of(kv[e], plo, pw) == pT;
    };
    int need = k;
    int mode = 0;           // 0 searching, 1 threshold (thr_key, thr_idx), 2 tie (thr_idx per thread)
    unsigned int thr_key = 0xFFFFFFFFu;
    int thr_idx = -1;
    for (int round = 0; round < kCRounds && mode == 0; ++round) {
        // --- range of the keys in play, over the cluster
        unsigned int mn = 0xFFFFFFFFu, mx = 0u;
#pragma unroll
        for (int e = 0; e < KPT; ++e)
            if (inplay(e)) {
                mn = min(mn, kv[e]);
                mx = max(mx, kv[e]);
            }
        mn = __reduce_min_sync(0xffffffffu, mn);
        mx = __reduce_max_sync(0xffffffffu, mx);
        if (lane == 0) {
            sh.redk[0][warp] = mn;
            sh.redk[1][warp] = mx;
        }
        __syncthreads();
        if (warp == 0) {
            const unsigned int a = __reduce_min_sync(0xffffffffu, lane < kCThreads / 32 ? sh.redk[0][lane] : 0xFFFFFFFFu);
            const unsigned int c = __reduce_max_sync(0xffffffffu, lane < kCThreads / 32 ? sh.redk[1][lane] : 0u);
            if (lane == 0) {
                sh.pub_mm[0] = a;
                sh.pub_mm[1] = c;
            }
        }
        cluster_sync();
        if (warp == 0) {
            const unsigned int va = lane < C ? (unsigned)ld_dsmem_s32(dsmem(&sh.pub_mm[0], lane)) : 0xFFFFFFFFu;
            const unsigned int vc = lane < C ? (unsigned)ld_dsmem_s32(dsmem(&sh.pub_mm[1], lane)) : 0u;
            const unsigned int a = __reduce_min_sync(0xffffffffu, va);
            const unsigned int c = __reduce_max_sync(0xffffffffu, vc);
            if (lane == 0) {
                sh.g_mm[0] = a;
                sh.g_mm[1] = c;
            }
        }
        __syncthreads();
        mn = sh.g_mm[0];
        mx = sh.g_mm[1];
        if (mn == mx) {
            // every key in play equals mn: keep the `need` lowest indices of them
            thr_key = mn;
            int c = 0;
#pragma unroll
            for (int e = 0; e < KPT; ++e) c += inplay(e);
            const int incl = block_scan_incl(c, sh.wsum);
            if (tid == kCThreads - 1) sh.pub_tie = incl;
            cluster_sync();
            if (warp == 0) {
                int v = lane < r ? ld_dsmem_s32(dsmem(&sh.pub_tie, lane)) : 0;
                v = warp_sum(v);
                if (lane == 0) sh.before = v;
            }
            __syncthreads();
            int rk = sh.before + incl - c;
#pragma unroll
            for (int e = 0; e < KPT; ++e)
                if (inplay(e)) {
                    if (rk < need) thr_idx = i0 + e;   // ascending: the last kept one
                    ++rk;
                }
            mode = 2;
            break;
        }
        // --- histogram; this CTA's is read by the cluster after the barrier
        const float w = (float)kCBins / ((float)(mx - mn) + 1.0f);
        for (int i = tid; i < kCBins; i += kCThreads) sh.hist[i] = 0;
        __syncthreads();
#pragma unroll
        for (int e = 0; e < KPT; ++e)
            if (inplay(e)) atomicAdd(&sh.hist[bucket_of(kv[e], mn, w)], 1);
        cluster_sync();
        // cluster totals in two steps (distributed shared memory is slow for
        // many small reads): CTA r totals its slice of kCBins / C bins over the
        // cluster, then thread t reads the total of bin jb = NB - 1 - t (thread
        // 0 the top bin) from the CTA that holds it
        constexpr int SL = kCBins / C;
        if (tid < SL) {
            int v[C];                        // every read goes out before the first add
#pragma unroll
            for (int q = 0; q < C; ++q) v[q] = ld_dsmem_s32(dsmem(&sh.hist[r * SL + tid], q));
            int t = 0;
#pragma unroll
            for (int q = 0; q < C; ++q) t += v[q];
            sh.tot[tid] = t;
        }
        cluster_sync();
        const int jb = kCBins - 1 - tid;
        const int hsum = ld_dsmem_s32(dsmem(&sh.tot[jb % SL], jb / SL));
        const int incl = block_scan_incl(hsum, sh.wsum);
        const int above = incl - hsum;   // keys in the bins above jb
        if (above < need && need <= above + hsum) {
            sh.T = jb;
            sh.need = need - above;
            sh.cT = hsum;
        }
        __syncthreads();
        const int T = sh.T;
        need = sh.need;
        const int cT = sh.cT;
        if (cT <= kCCap) {
            // --- gather bucket T's keys from the cluster and rank them exactly
            if (tid == 0) sh.lcn = 0;
            __syncthreads();
#pragma unroll
            for (int e = 0; e < KPT; ++e)
                if (inplay(e) && bucket_of(kv[e], mn, w) == T) {
                    const int slot = atomicAdd(&sh.lcn, 1);
                    sh.lc[slot] = ((unsigned long long)kv[e] << 32) |
                                  (unsigned long long)(0xFFFFFFFFu - (unsigned)(i0 + e));
                }
            cluster_sync();
            if (warp == 0) {
                const int n = lane < C ? ld_dsmem_s32(dsmem(&sh.lcn, lane)) : 0;
                int x = n;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int t = __shfl_up_sync(0xffffffffu, x, o);
                    if (lane >= o) x += t;
                }
                if (lane < C) sh.mc_off[lane + 1] = x;
                if (lane == 0) sh.mc_off[0] = 0;
            }
            __syncthreads();
            const int nc = sh.mc_off[C];
            for (int j = tid; j < nc; j += kCThreads) {   // one read per thread, all at once
                int q = 0;
#pragma unroll
                for (int u = 1; u < C; ++u) q += j >= sh.mc_off[u];
                sh.mc[j] = ld_dsmem_u64(dsmem(&sh.lc[j - sh.mc_off[q]], q));
            }
            __syncthreads();
            for (int j = tid; j < nc; j += kCThreads) {
                const unsigned long long me = sh.mc[j];
                int rank = 0;
                for (int jj = 0; jj < nc; ++jj) rank += (sh.mc[jj] > me);
                if (rank == need - 1) {
                    sh.thr_key = (unsigned)(me >> 32);
                    sh.thr_idx = (int)(0xFFFFFFFFu - (unsigned)(me & 0xFFFFFFFFull));
                }
            }
            __syncthreads();
            thr_key = sh.thr_key;
            thr_idx = sh.thr_idx;
            mode = 1;
        } else {
            lo_k = mn;
            hi_k = mx;
            plo = mn;
            pw = w;
            pT = T;
        }
    }
    if (mode == 0 && tid == 0 && r == 0) report(status, ENTMAXKV_DEVICE_BOUNDS);   // keeps nothing

    // --- emit the kept pages in page order
    int c = 0;
#pragma unroll
    for (int e = 0; e < KPT; ++e) {
        const unsigned kk = kv[e];
        c += (i0 + e < P) && ((kk > thr_key) || (kk == thr_key && i0 + e <= thr_idx));
    }
    const int incl = block_scan_incl(c, sh.wsum);
    if (tid == kCThreads - 1) sh.pub_kept = incl;
    cluster_sync();
    if (warp == 0) {
        const int v = lane < C ? ld_dsmem_s32(dsmem(&sh.pub_kept, lane)) : 0;
        const int before = warp_sum(lane < r ? v : 0);
        const int total = warp_sum(v);
        if (lane == 0) {
            sh.before = before;
            sh.total = total;
        }
    }
    __syncthreads();
    cluster_arrive();   // this CTA reads no other CTA's shared memory from here on
    int pos = sh.before + incl - c;
#pragma unroll
    for (int e = 0; e < KPT; ++e) {
        const unsigned kk = kv[e];
        if ((i0 + e < P) && ((kk > thr_key) || (kk == thr_key && i0 + e <= thr_idx))) {
            if (pos < k_max) out[pos] = i0 + e;
            ++pos;
        }
    }
    if (tid == 0 && r == 0) {
        if (sh.total != k) report(status, ENTMAXKV_DEVICE_BOUNDS);
        sel_count[(size_t)b * H_kv + g] = min(sh.total, k_max);
    }
    cluster_wait();     // no CTA leaves while another may still read its shared memory
}

// ---------------------------------------------------------------- Gaussian
//
// tau_hat per (sequence, query head): root of
//   F(tau) = sum_p n_p E[((alpha-1) s_p - tau)_+^(1/(alpha-1))] = 1,
// s_p ~ N(m_p, v_p), by safeguarded Newton steps on log F (each term is
// log-concave in tau, so the steps behave like Newton on a near-quadratic
// function even where F spans many orders of magnitude); every evaluation
// narrows a bracket [lo, hi] with F(lo) >= 1 > F(hi), and a step that leaves
// it is replaced by bisection (or by doubling while no upper end is known).

constexpr int kTauThreads = 512;
constexpr int kGLNodes = 32;

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

// The pages of one (sequence, query head) are split over a cluster of
// kGaussTauCTAs CTAs; every evaluation of F and F' is summed per CTA, the
// per-CTA sums are exchanged through distributed shared memory (double
// buffered by iteration parity) and added in rank order by every CTA, so all
// CTAs hold the same values and take the same steps.
constexpr int kGaussTauCTAs = 8;
constexpr int kGaussTauReg = 4;      // pages per thread whose terms' inputs stay in registers

// Any other alpha (r = 1/(alpha-1) not 1 or 2): E[(X - tau)_+^r] for
// X ~ N(m', s'^2), with u = m' - tau and z = u / s', is s'^r times
// I(z) = int_0^inf y^r phi(y - z) dy.  The log of the integrand,
// r ln y - (y - z)^2 / 2, is concave with its peak at y* = (z + sqrt(z^2 + 4r)) / 2
// and second derivative -(1 + r / y^2): below y* it falls at least as fast as
// a Gaussian of width w = 1 / sqrt(1 + r / y*^2), above y* at least as fast as
// one of width w' = 1 / sqrt(1 + r / (y* + 10)^2), so [y* - 10 w, y* + 10 w']
// holds all but about exp(-50) of it.  A 32-node Gauss-Legendre rule covers
// that interval in y when it starts above 0, else [0, y* + 10 w'] in t with
// y = t^2 (which removes the y^r endpoint behaviour at 0).  Terms are formed
// as powf(s' y, r), so s'^r y^r never overflows where the product is small.
// g is the expectation and dg = -d/dtau of it (r times the same integral of
// the (r-1)-th power).
struct GLTable {
    float x[kGLNodes], w[kGLNodes];   // nodes and weights on [-1, 1]
};

EKV_DEV void gauss_term_any(float mp, float sp, float tau, float r, const GLTable& gl, float& g, float& dg)
{
    const float u = mp - tau;
    if (!(sp > 0.f)) {
        const float up = fmaxf(u, 0.f);
        g = up > 0.f ? powf(up, r) : 0.f;
        dg = up > 0.f ? r * powf(up, r - 1.f) : 0.f;
        return;
    }
    const float z = u / sp;
    g = dg = 0.f;
    const float ys = 0.5f * (z + sqrtf(fmaf(z, z, 4.f * r)));
    const float w = rsqrtf(1.f + r / (ys * ys));
    const float yh = ys + 10.f;
    const float hi = ys + 10.f * rsqrtf(1.f + r / (yh * yh));
    if (hi <= 0.f) return;
    const float lo = ys - 10.f * w;
    const float c = 0.3989422804014327f;
    float s0 = 0.f, s1 = 0.f;
    if (lo > 0.f) {
        const float half = 0.5f * (hi - lo), mid = 0.5f * (hi + lo);
#pragma unroll 8
        for (int k = 0; k < kGLNodes; ++k) {
            const float y = fmaf(half, gl.x[k], mid);
            const float e = y - z;
            const float ph = c * expf(-0.5f * e * e) * half * gl.w[k];
            const float yr = powf(sp * y, r);
            s0 = fmaf(yr, ph, s0);
            s1 = fmaf(yr / (sp * y), ph, s1);
        }
    } else {
        const float T = sqrtf(hi);
#pragma unroll 8
        for (int k = 0; k < kGLNodes; ++k) {
            const float t = 0.5f * T * (gl.x[k] + 1.f);
            const float y = t * t;
            const float e = y - z;
            const float ph = c * expf(-0.5f * e * e) * t * T * gl.w[k];   // phi * 2t * (T/2) w
            const float yr = powf(sp * y, r);
            s0 = fmaf(yr, ph, s0);
            s1 = fmaf(y > 0.f ? yr / (sp * y) : 0.f, ph, s1);
        }
    }
    g = s0;
    dg = r * s1;
}

__global__ void __launch_bounds__(kTauThreads)
gauss_tau_kernel(const float* __restrict__ m, const float* __restrict__ v, const float* __restrict__ est,
                 const int32_t* __restrict__ seq_lens, int ps, int H_q, int max_pages, float alpha,
                 float* __restrict__ tau_hat, const GLTable gl)
{
    pdl_enter();
    constexpr int C = kGaussTauCTAs, NW = kTauThreads / 32, KR = kGaussTauReg;
    __shared__ double red[2][NW];
    __shared__ float redf[2][NW];
    __shared__ double pub[2][2];          // this CTA's (F, F') of the iterations of each parity
    __shared__ float pub_mx[2];
    __shared__ double gsum[2];
    __shared__ float gmx[2];
    const int r = (int)cluster_rank();
    const int b = blockIdx.y, h = blockIdx.x / C, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int L = seq_lens[b];
    const int P = pages_of(L, ps, max_pages, nullptr);
    const float am1 = alpha - 1.0f;
    const bool a2 = alpha == 2.0f;
    const bool any = !a2 && alpha != 1.5f;
    const float rexp = 1.0f / am1;
    const float* mh = m + ((size_t)b * H_q + h) * max_pages;
    const float* vh = v + ((size_t)b * H_q + h) * max_pages;
    const float* eh = est + ((size_t)b * H_q + h) * max_pages;
    if (P == 0) {   // the same on every CTA of the cluster: no barrier is met
        if (tid == 0 && r == 0) tau_hat[(size_t)b * H_q + h] = INFINITY;
        return;
    }
    const int chunk = (P + C - 1) / C;
    const int p0 = min(P, r * chunk), p1 = min(P, p0 + chunk);
    // inputs of this thread's first KR pages, kept for every iteration: m', s', tokens
    float rm[KR], rs[KR];
    int rn[KR];
    float mx = -INFINITY, emx = -INFINITY;
#pragma unroll
    for (int k = 0; k < KR; ++k) {
        const int p = p0 + tid + k * kTauThreads;
        rn[k] = 0;
        rm[k] = rs[k] = 0.f;
        if (p < p1) {
            rm[k] = am1 * mh[p];
            rs[k] = am1 * sqrtf(fmaxf(vh[p], 0.f));
            rn[k] = min(ps, L - p * ps);
            mx = fmaxf(mx, rm[k]);
            emx = fmaxf(emx, am1 * eh[p]);
        }
    }
    for (int p = p0 + tid + KR * kTauThreads; p < p1; p += kTauThreads) {
        mx = fmaxf(mx, am1 * mh[p]);
        emx = fmaxf(emx, am1 * eh[p]);
    }
    mx = warp_max(mx);
    emx = warp_max(emx);
    if (lane == 0) {
        redf[0][warp] = mx;
        redf[1][warp] = emx;
    }
    __syncthreads();
    if (warp == 0) {
        float a = lane < NW ? redf[0][lane] : -INFINITY;
        float c = lane < NW ? redf[1][lane] : -INFINITY;
        a = warp_max(a);
        c = warp_max(c);
        if (lane == 0) {
            pub_mx[0] = a;
            pub_mx[1] = c;
        }
    }
    cluster_sync();
    if (warp == 0) {
        float a = lane < C ? ld_dsmem_f32(dsmem(&pub_mx[0], lane)) : -INFINITY;
        float c = lane < C ? ld_dsmem_f32(dsmem(&pub_mx[1], lane)) : -INFINITY;
        a = warp_max(a);
        c = warp_max(c);
        if (lane == 0) {
            gmx[0] = a;
            gmx[1] = c;
        }
    }
    __syncthreads();
    double lo = (double)gmx[0] - 1.0;   // F(lo) >= 1 (Jensen: the top page alone gives >= 1)
    double hi = INFINITY;
    // first guess half a unit below the largest estimated page maximum: the
    // threshold sits just under the top scores, so this usually starts a step
    // or two from the root (the bracket keeps any start safe)
    double tau = fmax(lo, (double)gmx[1] - 0.5);
    for (int it = 0; it < 60; ++it) {
        double F = 0.0, dF = 0.0;
        const float tf = (float)tau;
#pragma unroll
        for (int k = 0; k < KR; ++k) {
            if (rn[k] == 0) continue;
            float gv, dg;
            if (any) gauss_term_any(rm[k], rs[k], tf, rexp, gl, gv, dg);
            else gauss_term(rm[k], rs[k], tf, a2, gv, dg);
            F += (double)rn[k] * gv;
            dF += (double)rn[k] * dg;
        }
        for (int p = p0 + tid + KR * kTauThreads; p < p1; p += kTauThreads) {
            const float mp = am1 * mh[p];
            const float sp = am1 * sqrtf(fmaxf(vh[p], 0.f));
            const int n = min(ps, L - p * ps);
            float gv, dg;
            if (any) gauss_term_any(mp, sp, tf, rexp, gl, gv, dg);
            else gauss_term(mp, sp, tf, a2, gv, dg);
            F += (double)n * gv;
            dF += (double)n * dg;
        }
        F = warp_sum(F);
        dF = warp_sum(dF);
        if (lane == 0) {
            red[0][warp] = F;
            red[1][warp] = dF;
        }
        __syncthreads();
        const int par = it & 1;
        if (tid == 0) {
            double f = 0.0, df = 0.0;
            for (int w = 0; w < NW; ++w) {
                f += red[0][w];
                df += red[1][w];
            }
            pub[par][0] = f;
            pub[par][1] = df;
        }
        cluster_sync();
        if (tid == 0) {
            double f = 0.0, df = 0.0;
            for (int q = 0; q < C; ++q) {   // rank order: the same sums on every CTA
                f += __longlong_as_double((long long)ld_dsmem_u64(dsmem(&pub[par][0], q)));
                df += __longlong_as_double((long long)ld_dsmem_u64(dsmem(&pub[par][1], q)));
            }
            gsum[0] = f;
            gsum[1] = df;
        }
        __syncthreads();
        F = gsum[0];
        dF = gsum[1];
        if (F >= 1.0) lo = tau; else hi = tau;
        if (fabs(F - 1.0) < 1e-7 || (hi - lo) < 1e-7 * fmax(1.0, fabs(tau))) break;
        // Newton step on log F: far left of the root F is exponential-like and a
        // step on F itself would gain one e-fold at a time
        double nt = (F > 0.0 && dF > 0.0) ? tau + F * log(F) / dF : INFINITY;
        if (!(nt > lo && nt < hi)) {
            nt = isinf(hi) ? lo + fmax(1.0, 2.0 * (tau - lo + 0.5)) : 0.5 * (lo + hi);
        } else if (fabs(nt - tau) < 1e-6 * fmax(1.0, fabs(tau))) {
            // the terms are evaluated in float: F is not known to better than
            // about 1e-6 relative, so a smaller step is converged
            tau = nt;
            break;
        }
        tau = nt;
    }
    if (tid == 0 && r == 0) tau_hat[(size_t)b * H_q + h] = (float)tau;
    cluster_sync();   // no CTA leaves while another may still read its shared memory
}

// Keep rule: page p is kept when (alpha-1) * est_p >= tau_hat_h - delta for
// some query head h of the group (fp32, as entmaxkv.h states).  The pages of
// one (sequence, kv head) are split over a cluster of kTopkCTAs CTAs; kept
// counts are exchanged through distributed shared memory so that each CTA
// writes its kept pages at the right offset, in page order.  Flags of a tile
// are computed with coalesced loads, then each thread emits 8 consecutive
// pages.
constexpr int kKeepThreads = 256;

template <int G>
__global__ void __launch_bounds__(kKeepThreads)
gauss_keep_kernel(const float* __restrict__ est, const float* __restrict__ tau_hat,
                  const int32_t* __restrict__ seq_lens, int ps, int H_q, int H_kv, int max_pages,
                  float alpha, float delta, int k_max, int32_t* __restrict__ sel, int32_t* __restrict__ sel_count,
                  int32_t* status)
{
    pdl_enter();
    constexpr int C = kTopkCTAs, TILE = kKeepThreads * 8;
    __shared__ __align__(16) uint8_t flags[TILE];
    __shared__ int wsum[32];
    __shared__ int pub_cnt;
    __shared__ int s_before, s_total, s_tile;
    const int r = (int)cluster_rank();
    const int b = blockIdx.y, g = blockIdx.x / C, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int L = seq_lens[b];
    const int P = pages_of(L, ps, max_pages, r == 0 ? status : nullptr);
    const float am1 = alpha - 1.0f;
    float rhs[G];
#pragma unroll
    for (int h = 0; h < G; ++h) rhs[h] = __fsub_rn(tau_hat[(size_t)b * H_q + g * G + h], delta);
    const float* e0 = est + ((size_t)b * H_q + (size_t)g * G) * max_pages;
    auto keep = [&](int p) {
        bool k = false;
#pragma unroll
        for (int h = 0; h < G; ++h) k |= __fmul_rn(am1, e0[(size_t)h * max_pages + p]) >= rhs[h];
        return k;
    };
    const int chunk = (P + C - 1) / C;
    const int p0 = min(P, r * chunk), p1 = min(P, p0 + chunk);

    int c = 0;
    for (int t0 = p0; t0 < p1; t0 += TILE)
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const int p = t0 + e * kKeepThreads + tid;
            if (p < p1) c += keep(p);
        }
    c = block_sum(c, wsum);
    if (tid == 0) pub_cnt = c;
    cluster_sync();
    if (warp == 0) {
        const int x = lane < C ? ld_dsmem_s32(dsmem(&pub_cnt, lane)) : 0;
        const int before = warp_sum(lane < r ? x : 0);
        const int total = warp_sum(x);
        if (lane == 0) {
            s_before = before;
            s_total = total;
        }
    }
    __syncthreads();
    cluster_arrive();   // this CTA reads no other CTA's shared memory from here on
    int32_t* out = sel + ((size_t)b * H_kv + g) * k_max;
    int pos = s_before;
    for (int t0 = p0; t0 < p1; t0 += TILE) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const int p = t0 + e * kKeepThreads + tid;
            flags[e * kKeepThreads + tid] = p < p1 && keep(p);
        }
        __syncthreads();
        const uint2 f8 = *reinterpret_cast<const uint2*>(&flags[tid * 8]);
        const int n = __popc(f8.x) + __popc(f8.y);   // flags are 0 or 1
        const int incl = block_scan_incl(n, wsum);
        if (tid == kKeepThreads - 1) s_tile = incl;
        int q = pos + incl - n;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const uint32_t word = e < 4 ? f8.x : f8.y;
            if ((word >> (8 * (e & 3))) & 1u) {
                if (q < k_max) out[q] = t0 + tid * 8 + e;
                ++q;
            }
        }
        __syncthreads();
        pos += s_tile;
    }
    if (tid == 0 && r == 0) {
        if (s_total > k_max) report(status, ENTMAXKV_DEVICE_BOUNDS);
        sel_count[(size_t)b * H_kv + g] = min(s_total, k_max);
    }
    cluster_wait();     // no CTA leaves while another may still read its shared memory
}

// Gauss-Legendre nodes and weights on [-1, 1]: roots of P_n by Newton steps
// from the Chebyshev-like guess cos(pi (i + 3/4) / (n + 1/2)), weights
// 2 / ((1 - x^2) P_n'(x)^2); float64, computed once.
static const GLTable& gl_table()
{
    static const GLTable t = [] {
        GLTable r{};
        const int n = kGLNodes;
        for (int i = 0; i < n; ++i) {
            double x = std::cos(M_PI * (i + 0.75) / (n + 0.5)), dp = 0.0;
            for (int it = 0; it < 100; ++it) {
                double p0 = 1.0, p1 = x;            // P_0, P_1
                for (int k = 2; k <= n; ++k) {
                    const double p2 = ((2.0 * k - 1.0) * x * p1 - (k - 1.0) * p0) / k;
                    p0 = p1;
                    p1 = p2;
                }
                dp = n * (x * p1 - p0) / (x * x - 1.0);   // P_n'(x)
                const double dx = p1 / dp;
                x -= dx;
                if (std::fabs(dx) < 1e-16) break;
            }
            r.x[i] = (float)x;
            r.w[i] = (float)(2.0 / ((1.0 - x * x) * dp * dp));
        }
        return r;
    }();
    return t;
}

int launch_select(int mode, const float* ub, const float* m, const float* v, const float* est,
                  const int32_t* seq_lens, int ps, int B, int H_q, int H_kv, int max_pages, int budget,
                  float budget_frac, float alpha, float delta, int k_max, int32_t* sel, int32_t* sel_count,
                  float* tau_hat, int32_t* status, cudaStream_t stream)
{
    if (mode == ENTMAXKV_SELECT_TOPK) {
        // every sequence has at most max_pages pages: pick the register width from it
        const dim3 grid(H_kv * kTopkCTAs, B), block(kCThreads);
        constexpr int per = kTopkCTAs * kCThreads;
#define EKV_TOPK(KPT) \
    launch_pdl_cluster(topk_cluster_kernel<KPT>, grid, block, kTopkCTAs, 0, stream, ub, seq_lens, ps, H_kv, max_pages, \
                       budget, budget_frac, k_max, sel, sel_count, status)
        if (max_pages <= per) EKV_TOPK(1);
        else if (max_pages <= 2 * per) EKV_TOPK(2);
        else if (max_pages <= 4 * per) EKV_TOPK(4);
        else if (max_pages <= 8 * per) EKV_TOPK(8);
        else if (max_pages <= 16 * per) EKV_TOPK(16);
#undef EKV_TOPK
        else
            launch_pdl(topk_kernel, dim3(H_kv, B), dim3(kSelThreads), 0, stream, ub, seq_lens, ps, H_kv, max_pages, budget, budget_frac,
                       k_max, sel, sel_count, status);
    } else {
        launch_pdl_cluster(gauss_tau_kernel, dim3(H_q * kGaussTauCTAs, B), dim3(kTauThreads), kGaussTauCTAs, 0, stream,
                           m, v, est, seq_lens, ps, H_q, max_pages, alpha, tau_hat, gl_table());
        if (cudaGetLastError() != cudaSuccess) return ENTMAXKV_CUDA_ERROR;
        const int G = H_q / H_kv;
#define EKV_KEEP(GG)                                                                                            \
    launch_pdl_cluster(gauss_keep_kernel<GG>, dim3(H_kv * kTopkCTAs, B), dim3(kKeepThreads), kTopkCTAs, 0, stream, \
                       est, tau_hat, seq_lens, ps, H_q, H_kv, max_pages, alpha, delta, k_max, sel, sel_count, status)
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
