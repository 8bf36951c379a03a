// Exact alpha-entmax attention over gathered pages, and the full-cache
// softmax (flash-decode) baseline.
//
// EntmaxKV (German technical summary, section 2.C): once candidate pages are
// chosen, only their keys and values are loaded and alpha-entmax is computed
// over that reduced set; the result is exact when the set holds the support.
// Section 4 compares against full-cache entmax and full-cache softmax
// (FlashDecoding) decoding.
//
// The threshold tau needs every candidate score before any weight is known.
// With a bf16 cache one launch does everything (entmax_bf16_kernel): the
// split-KV CTAs of a (sequence, kv head) form a thread-block cluster and
// cluster barriers separate
//   K pass:    gather key pages through the page table (TMA tile loads into
//              128-byte-swizzled shared memory, mbarrier pipeline), score the
//              GQA head group with mma.sync (keys bf16, query split into a
//              bf16 high and low part so the product keeps ~16 mantissa bits),
//              write x = (alpha-1) * scale * q.k per listed token;
//   threshold: a lower bound of tau from the chunk maxima, the scores above it
//              as candidates, Newton steps from the left and the closed form
//              on the final support in float64;
//   V pass:    gather the value pages holding weight, turn x into
//              p = [x - tau]_+^(1/(alpha-1)) (split bf16 high + low) and
//              accumulate P.V with mma.sync in fp32; the partials are added
//              in a fixed order (deterministic).
// fp32 caches (small configurations) take three plain CUDA-core kernels with
// the same split structure (qk_f32_kernel, tau_kernel, pv_f32_kernel).
// The softmax baseline does K and V in one pass with an online softmax and a
// log-sum-exp merge of the splits.
#include "common.cuh"
#include "kernels.cuh"

namespace ekv {

constexpr int kStagesQK = 4;
constexpr int kStagesPV = 4;
constexpr int kStagesSM = 3;
constexpr int kPsPad = 8;   // padding (bf16 elements) of a row of the P tile

struct Range {
    int start, end;
};

EKV_DEV Range split_range(int cnt, int S, int s)
{
    const int per = (cnt + S - 1) / S;
    const int start = min(cnt, s * per);
    return {start, min(cnt, start + per)};
}


EKV_DEV int list_count(const AttnArgs& a, int b, int g, int P)
{
    if (!a.sel_count) return P;
    int c = a.sel_count[(size_t)b * a.H_kv + g];
    if (c < 0 || c > a.k_max) {
        report(a.status, ENTMAXKV_DEVICE_BOUNDS);
        c = max(0, min(c, a.k_max));
    }
    return c;
}

// Physical page of list entry idx of (b, g), or -1 when the entry or its page
// id is out of range (reported when `rep`).
EKV_DEV int resolve_g(const AttnArgs& a, int b, int g, int idx, int P, int& lp, bool rep)
{
    lp = a.sel ? a.sel[((size_t)b * a.H_kv + g) * a.k_max + idx] : idx;
    if (lp < 0 || lp >= P) {
        if (rep) report(a.status, ENTMAXKV_DEVICE_BOUNDS);
        return -1;
    }
    const int phys = a.page_table[(size_t)b * a.max_pages + lp];
    if (phys < 0 || phys >= a.num_phys) {
        if (rep) report(a.status, ENTMAXKV_DEVICE_BOUNDS);
        return -1;
    }
    return phys;
}

// Page ids of a CTA's split, resolved once into shared memory so that the
// copy pipeline never waits on a dependent chain of global loads (list entry,
// then page table) before issuing a stage.  Every attention kernel calls
// tab_fill first; splits longer than the table resolve from global memory.
constexpr int kTabCap = 1024;
__shared__ int tab_phys[kTabCap];
__shared__ int tab_lp[kTabCap];
__shared__ int tab_base, tab_n;

EKV_DEV void tab_fill(const AttnArgs& a, int b, int g, Range r, int P)
{
    const int n = r.end > r.start ? r.end - r.start : 0;
    if (threadIdx.x == 0) {
        tab_base = r.start;
        tab_n = n <= kTabCap ? n : 0;
    }
    if (n <= kTabCap)
        for (int i = threadIdx.x; i < n; i += blockDim.x) {
            int lp;
            const int ph = resolve_g(a, b, g, r.start + i, P, lp, true);
            tab_phys[i] = ph;
            tab_lp[i] = lp;
        }
    __syncthreads();
}

// tab_fill for a split whose first list entries were loaded ahead (thread t
// holds entry rs.start + t and its page-table entry, or -1): used where the
// split is the one they were loaded for, with the same checks as resolve_g.
EKV_DEV void tab_fill_ahead(const AttnArgs& a, int b, int g, Range r, int P, Range rs, int ahead_lp,
                            int ahead_phys)
{
    const int n = r.end > r.start ? r.end - r.start : 0;
    if (threadIdx.x == 0) {
        tab_base = r.start;
        tab_n = n <= kTabCap ? n : 0;
    }
    const bool same = a.sel != nullptr && r.start == rs.start && r.end == rs.end;
    if (n <= kTabCap)
        for (int i = threadIdx.x; i < n; i += blockDim.x) {
            int lp, ph;
            if (same && i == (int)threadIdx.x) {
                lp = ahead_lp;
                ph = ahead_phys;
                if (lp < 0 || lp >= P || ph < 0 || ph >= a.num_phys) {
                    report(a.status, ENTMAXKV_DEVICE_BOUNDS);
                    ph = -1;
                }
            } else {
                ph = resolve_g(a, b, g, r.start + i, P, lp, true);
            }
            tab_phys[i] = ph;
            tab_lp[i] = lp;
        }
    __syncthreads();
}

EKV_DEV int resolve(const AttnArgs& a, int b, int g, int idx, int P, int& lp, bool rep)
{
    const int j = idx - tab_base;
    if (j >= 0 && j < tab_n) {
        lp = tab_lp[j];
        return tab_phys[j];
    }
    return resolve_g(a, b, g, idx, P, lp, rep);
}

// Issue the TMA loads of pipeline stage `st` (pages start + st*PPS ...) of one
// tensor into `dst`; returns the bytes expected.  Called by one thread.
template <int D, int PS>
EKV_DEV uint32_t issue_stage(const AttnArgs& a, const CUtensorMap* map, uint8_t* dst, uint64_t* bar, int b,
                             int g, Range r, int st, int P)
{
    constexpr int PPS = kStageTok / PS;
    int phys[PPS];
    uint32_t bytes = 0;
#pragma unroll
    for (int i = 0; i < PPS; ++i) {
        const int idx = r.start + st * PPS + i;
        int lp;
        phys[i] = idx < r.end ? resolve(a, b, g, idx, P, lp, true) : -1;
        if (phys[i] >= 0) bytes += PS * D * 2;
    }
    mbar_arrive_expect_tx(bar, bytes);
#pragma unroll
    for (int i = 0; i < PPS; ++i) {
        if (phys[i] < 0) continue;
        const int y = (phys[i] * a.H_kv + g) * PS;
#pragma unroll
        for (int h = 0; h < D / 64; ++h) tma_load_2d(dst + h * (kStageTok * 128) + i * PS * 128, map, bar, h * 64, y);
    }
    return bytes;
}

// Query fragments (B operand of m16n8k16, k = head dim, n = 2*head + part).
template <int D, int NT>
EKV_DEV void load_q_frags(const AttnArgs& a, int b, int g, float mul, uint32_t (&bq)[NT][D / 16][2])
{
    const int lane = threadIdx.x & 31;
    const int n = lane >> 2, c = lane & 3;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const int head = 4 * nt + (n >> 1);
        const int part = n & 1;
        const float* qh = a.q + ((size_t)b * a.H_q + (size_t)g * a.G + head) * D;
#pragma unroll
        for (int j = 0; j < D / 16; ++j) {
            uint32_t bits[4];
            const int ks[4] = {16 * j + 2 * c, 16 * j + 2 * c + 1, 16 * j + 2 * c + 8, 16 * j + 2 * c + 9};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float v = head < a.G ? qh[ks[e]] * mul : 0.f;
                uint32_t hi, lo;
                split_bf16(v, hi, lo);
                bits[e] = part ? lo : hi;
            }
            bq[nt][j][0] = pack2(bits[0], bits[1]);
            bq[nt][j][1] = pack2(bits[2], bits[3]);
        }
    }
}

// Zero the shared-memory rows of stage tokens that hold no valid token, so a
// zero weight never meets a non-finite value.
template <int D, int PS>
EKV_DEV void zero_invalid_rows(const AttnArgs& a, uint8_t* stage, int b, int g, Range r, int st, int P, int L)
{
    const int tid = threadIdx.x;
    const int t = tid & (kStageTok - 1);
    const int half = tid >> 6;
    if (half >= D / 64) return;
    const int i = t / PS;
    const int idx = r.start + st * (kStageTok / PS) + i;
    bool valid = false;
    if (idx < r.end) {
        int lp;
        const int phys = resolve(a, b, g, idx, P, lp, false);
        valid = phys >= 0 && lp * PS + (t % PS) < L;
    }
    if (!valid) {
        uint4* row = reinterpret_cast<uint4*>(stage + half * (kStageTok * 128) + t * 128);
#pragma unroll
        for (int k = 0; k < 8; ++k) row[k] = make_uint4(0, 0, 0, 0);
        fence_proxy_async();
    }
}

// ====================================================================== K pass
// Per-head maximum over lanes with equal (lane & 3): xor over lane bits 2..4.
EKV_DEV float group_lane_max(float v)
{
    v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 4));
    v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 8));
    v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 16));
    return v;
}

// Write this split's maximum score of every head of the group (all threads
// call; `wm` is shared [4][8]).
EKV_DEV void write_split_max(const AttnArgs& a, int b, int g, int s, const float* run, int NT, float (*wm)[8])
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, c = lane & 3;
    for (int nt = 0; nt < NT; ++nt) {
        const float m = group_lane_max(run[nt]);
        if (lane < 4) wm[warp][4 * nt + c] = m;
    }
    __syncthreads();
    if (threadIdx.x < a.G) {
        const int h = threadIdx.x;
        const float m = fmaxf(fmaxf(wm[0][h], wm[1][h]), fmaxf(wm[2][h], wm[3][h]));
        a.lmax[((size_t)b * a.H_q + (size_t)g * a.G + h) * a.S + s] = m;
    }
}

template <int D, int PS, int NT>
__global__ void __launch_bounds__(kThreads) qk_bf16_kernel(const __grid_constant__ CUtensorMap kmap, const AttnArgs a)
{
    pdl_enter();
    constexpr int STAGE = kStageTok * D * 2;
    constexpr int PPS = kStageTok / PS;
    constexpr int KS = D / 16;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_align<1024>(smem_raw);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStagesQK * STAGE);
    __shared__ int abort_flag;
    __shared__ float wm[4][8];

    const int b = blockIdx.z, g = blockIdx.y, s = blockIdx.x;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int L = a.seq_lens[b];
    const int P = pages_of(L, PS, a.max_pages, a.status);
    const int cnt = list_count(a, b, g, P);
    if (s == 0 && tid == 0) a.counters[(size_t)b * a.H_kv + g] = 0;
    const Range r = split_range(cnt, a.S, s);
    const int nst = r.end > r.start ? (r.end - r.start + PPS - 1) / PPS : 0;
    tab_fill(a, b, g, r, P);

    // start the key loads first; the query fragments are prepared meanwhile
    if (tid == 0) {
        abort_flag = 0;
        if (nst > 0) {
            prefetch_tmap(&kmap);
            for (int i = 0; i < kStagesQK; ++i) mbar_init(&bars[i], 1);
            fence_mbar_init();
            for (int st = 0; st < min(kStagesQK, nst); ++st)
                issue_stage<D, PS>(a, &kmap, smem + st * STAGE, &bars[st], b, g, r, st, P);
        }
    }
    float run[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) run[nt] = -INFINITY;
    if (nst == 0) {
        write_split_max(a, b, g, s, run, NT, wm);
        return;
    }
    uint32_t bq[NT][KS][2];
    load_q_frags<D, NT>(a, b, g, a.xscale, bq);
    __syncthreads();

    const uint32_t sbase = smem_addr(smem);
    const size_t xstride = (size_t)a.k_max * PS;
    const size_t cstride = (size_t)a.k_max * (PS / 16);
    for (int st = 0; st < nst; ++st) {
        const int slot = st % kStagesQK;
        if (!mbar_wait(&bars[slot], (st / kStagesQK) & 1, kWaitLimitNs)) {
            abort_flag = 1;
            report(a.status, ENTMAXKV_TIMEOUT);
        }
        __syncthreads();
        if (abort_flag) {
            if (tid == 0)
                for (int k = st; k < min(st + kStagesQK, nst); ++k)
                    mbar_wait(&bars[k % kStagesQK], (k / kStagesQK) & 1, kWaitLimitNs);
            return;
        }
        const uint32_t base = sbase + slot * STAGE;
        const int row0 = warp * 16;
        float acc[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
        const int arow = row0 + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
        for (int j = 0; j < KS; ++j) {
            uint32_t af[4];
            ldsm_x4(swz_addr(base, arow, 2 * j + (lane >> 4)), af);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) mma_bf16(acc[nt], af, bq[nt][j][0], bq[nt][j][1]);
        }
        // the warp's 16 rows lie in one page (16 divides PS): one list entry
        const int gi = lane >> 2, c = lane & 3;
        const int idx = r.start + st * PPS + row0 / PS;
        if (idx < r.end) {
            int lp;
            const int phys = resolve(a, b, g, idx, P, lp, false);
            float cm[NT];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) cm[nt] = -INFINITY;
#pragma unroll
            for (int rr = 0; rr < 2; ++rr) {
                const int prow = (row0 + gi + 8 * rr) % PS;
                const bool valid = phys >= 0 && lp * PS + prow < L;
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const int head = 4 * nt + c;
                    const float x = valid ? acc[nt][2 * rr] + acc[nt][2 * rr + 1] : -INFINITY;
                    cm[nt] = fmaxf(cm[nt], x);
                    if (head < a.G)
                        a.xbuf[((size_t)b * a.H_q + (size_t)g * a.G + head) * xstride + (size_t)idx * PS + prow] = x;
                }
            }
            // chunk maxima: the V pass decides from these which pages hold weight
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const float m = group_lane_max(cm[nt]);
                run[nt] = fmaxf(run[nt], m);
                const int head = 4 * nt + c;
                if (gi == 0 && head < a.G)
                    a.cmax[((size_t)b * a.H_q + (size_t)g * a.G + head) * cstride + (size_t)idx * (PS / 16) +
                           (row0 % PS) / 16] = m;
            }
        }
        __syncthreads();
        if (tid == 0 && st + kStagesQK < nst)
            issue_stage<D, PS>(a, &kmap, smem + slot * STAGE, &bars[slot], b, g, r, st + kStagesQK, P);
    }
    write_split_max(a, b, g, s, run, NT, wm);
}

// fp32 cache: each thread scores (token, head) pairs of a page with a float64
// dot product.
template <int D>
__global__ void __launch_bounds__(kThreads) qk_f32_kernel(const float* __restrict__ k_pool, int ps, const AttnArgs a)
{
    pdl_enter();
    __shared__ unsigned int hmax[8];
    const int b = blockIdx.z, g = blockIdx.y, s = blockIdx.x, tid = threadIdx.x;
    const int L = a.seq_lens[b];
    const int P = pages_of(L, ps, a.max_pages, a.status);
    const int cnt = list_count(a, b, g, P);
    if (s == 0 && tid == 0) a.counters[(size_t)b * a.H_kv + g] = 0;
    if (tid < 8) hmax[tid] = ordered_key(-INFINITY);
    const Range r = split_range(cnt, a.S, s);
    tab_fill(a, b, g, r, P);
    const size_t xstride = (size_t)a.k_max * ps;
    const double xs = (double)a.xscale;
    for (int idx = r.start; idx < r.end; ++idx) {
        int lp;
        const int phys = resolve(a, b, g, idx, P, lp, tid == 0);
        for (int w = tid; w < ps * a.G; w += kThreads) {
            const int t = w % ps, head = w / ps;
            float x = -INFINITY;
            if (phys >= 0 && lp * ps + t < L) {
                const float* kr = k_pool + (((size_t)phys * a.H_kv + g) * ps + t) * D;
                const float* qh = a.q + ((size_t)b * a.H_q + (size_t)g * a.G + head) * D;
                double dot = 0.0;
                for (int j = 0; j < D; ++j) dot = fma((double)qh[j], (double)kr[j], dot);
                x = (float)(dot * xs);
                atomicMax(&hmax[head], ordered_key(x));
            }
            a.xbuf[((size_t)b * a.H_q + (size_t)g * a.G + head) * xstride + (size_t)idx * ps + t] = x;
        }
    }
    __syncthreads();
    if (tid < a.G) {
        const unsigned int k = hmax[tid];
        const float m = __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
        a.lmax[((size_t)b * a.H_q + (size_t)g * a.G + tid) * a.S + s] = m;
    }
}

// ====================================================================== tau
// One CTA per (sequence, query head).  The maximum score M comes from the
// split maxima of the K pass; tau >= M - 1 (the top score alone has mass
// >= 1 there), so only scores above M - 1 can carry weight.  They are
// compacted in one vectorised pass.  A 2048-bin histogram of them over
// [M - 1, M] then brackets tau: at every bin edge t the counts give a lower
// and an upper bound of F(t) = sum (x - t)_+^(1/(alpha-1)) (each value lies
// within its bin), so tau lies between the last edge with F_lower >= 1 and
// the first edge with F_upper < 1, a few bins apart.  Newton steps from that
// lower edge (never past the root: F is convex and decreasing) then shrink
// the support {x > tau} until the closed form on it is consistent, usually
// in one to three passes.
constexpr int kTauBlock = 512;
constexpr int kTauWarps = kTauBlock / 32;
constexpr int kTauBins = 2048;
constexpr int kTauCap = 32768;                         // candidates kept in shared memory
constexpr int kTauSmem = kTauCap * 4 + kTauBins * 4 + 64;

// block-wide sum of 3 doubles and min/max of 2 floats; double-buffered scratch
struct TauRed {
    double d[2][kTauWarps][3];
    float f[2][kTauWarps][2];
};

EKV_DEV void tau_reduce(TauRed& R, int it, double (&v)[3], float& mn, float& mx)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, bb = it & 1;
#pragma unroll
    for (int i = 0; i < 3; ++i) v[i] = warp_sum(v[i]);
    mn = warp_min(mn);
    mx = warp_max(mx);
    if (lane == 0) {
        R.d[bb][warp][0] = v[0];
        R.d[bb][warp][1] = v[1];
        R.d[bb][warp][2] = v[2];
        R.f[bb][warp][0] = mn;
        R.f[bb][warp][1] = mx;
    }
    __syncthreads();
    v[0] = v[1] = v[2] = 0.0;
    mn = INFINITY;
    mx = -INFINITY;
#pragma unroll
    for (int w = 0; w < kTauWarps; ++w) {
        v[0] += R.d[bb][w][0];
        v[1] += R.d[bb][w][1];
        v[2] += R.d[bb][w][2];
        mn = fminf(mn, R.f[bb][w][0]);
        mx = fmaxf(mx, R.f[bb][w][1]);
    }
}

__global__ void __launch_bounds__(kTauBlock) tau_kernel(int ps, const AttnArgs a)
{
    pdl_enter();
    extern __shared__ uint8_t tau_smem[];
    float* cand = reinterpret_cast<float*>(tau_smem);
    int* hist = reinterpret_cast<int*>(tau_smem + kTauCap * 4);
    __shared__ int ncand;
    __shared__ float redm[kTauWarps];
    __shared__ TauRed R;
    __shared__ double scan[kTauWarps][3];
    __shared__ double brk[1][kTauWarps];
    const int b = blockIdx.y, h = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = h / a.G;
    const int L = a.seq_lens[b];
    const int P = pages_of(L, ps, a.max_pages, a.status);
    const int cnt = list_count(a, b, g, P);
    const int n = cnt * ps;
    const size_t row = (size_t)b * a.H_q + h;
    const float* x = a.xbuf + row * (size_t)a.k_max * ps;
    const bool a2 = a.alpha == 2.0f;
    const bool gen = !a2 && a.alpha != 1.5f;          // any other alpha: no closed form

    float M = -INFINITY;
    for (int s = tid; s < a.S; s += kTauBlock) M = fmaxf(M, a.lmax[row * a.S + s]);
    M = block_max(M, redm);
    if (!(M > -INFINITY)) {
        if (tid == 0) {
            a.tau[row] = INFINITY;
            if (a.tau_out) a.tau_out[row] = INFINITY;
        }
        return;
    }
    const double thr = (double)M - 1.0;
    // float prefilter at or below thr: most scores fail it without a float64 step
    const float thr_f = nextafterf((float)thr, -INFINITY);
    if (tid == 0) ncand = 0;
    for (int i = tid; i < kTauBins; i += kTauBlock) hist[i] = 0;
    __syncthreads();
    // --- compaction of {x > M - 1} + histogram.  Every thread issues all its
    // loads of a round (8 float4) before using any of them.
    const float4* x4 = reinterpret_cast<const float4*>(x);
    const int n4 = n >> 2;
    constexpr int U = 8;
    for (int base = warp * 32 * U; base < n4; base += kTauBlock * U) {
        float v[4 * U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int i = base + u * 32 + lane;
            const float4 f = i < n4 ? x4[i] : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
            v[4 * u] = f.x; v[4 * u + 1] = f.y; v[4 * u + 2] = f.z; v[4 * u + 3] = f.w;
        }
        int c = 0;
#pragma unroll
        for (int e = 0; e < 4 * U; ++e) {
            if (!(v[e] > thr_f)) continue;
            const double d = (double)v[e] - thr;
            if (d > 0.0) {
                ++c;
                atomicAdd(&hist[min(kTauBins - 1, (int)(d * kTauBins))], 1);
            }
        }
        int incl = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int t = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += t;
        }
        const int tot = __shfl_sync(0xffffffffu, incl, 31);
        if (tot == 0) continue;
        int wbase = 0;
        if (lane == 31) wbase = atomicAdd(&ncand, tot);
        wbase = __shfl_sync(0xffffffffu, wbase, 31);
        int pos = wbase + incl - c;
#pragma unroll
        for (int e = 0; e < 4 * U; ++e)
            if (v[e] > thr_f && (double)v[e] > thr) {
                if (pos < kTauCap) cand[pos] = v[e];
                ++pos;
            }
    }
    __syncthreads();
    // --- lower bracket of tau from the histogram.  Bin j holds values in
    // [e_j, e_{j+1}], e_j = thr + j / NB (exact: x and thr are floats, the
    // difference and the scaling by a power of two are exact in double), so
    //   F(e_i) >= sum_{j > i} c_j (e_j - eps - e_i)^r = F_lower(e_i)
    // expanded in suffix sums of c_j, c_j a_j, c_j a_j^2 with a_j = e_j - eps.
    // tau >= the largest edge with F_lower >= 1 (and >= thr).
    constexpr int BPT = kTauBins / kTauBlock;            // bins per thread (4)
    const double w = 1.0 / kTauBins;
    const double eps = 4e-7 * fmax(1.0, fabs((double)M));
    double loc[3] = {0, 0, 0};
    const int j0 = tid * BPT;
#pragma unroll
    for (int k = 0; k < BPT; ++k) {
        const int j = j0 + k;
        const double c = (double)hist[j];
        const double lo = thr + j * w - eps;
        loc[0] += c;
        loc[1] += c * lo;
        loc[2] += c * lo * lo;
    }
    double suf[3];
#pragma unroll
    for (int i = 0; i < 3; ++i) {
        double v = loc[i];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const double t = __shfl_down_sync(0xffffffffu, v, o);
            if (lane + o < 32) v += t;
        }
        suf[i] = v;
    }
    if (lane == 0)
#pragma unroll
        for (int i = 0; i < 3; ++i) scan[warp][i] = suf[i];
    __syncthreads();
#pragma unroll
    for (int i = 0; i < 3; ++i) {
        double above = 0.0;
        for (int ww = warp + 1; ww < kTauWarps; ++ww) above += scan[ww][i];
        suf[i] = suf[i] - loc[i] + above;                // bins of the threads above mine
    }
    double best_lo = thr;
    if (!gen) {
        double S0 = suf[0], S1 = suf[1], S2 = suf[2];     // sums over bins > my last bin
        for (int k = BPT - 1; k >= 0; --k) {
            const int j = j0 + k;
            const double e = thr + j * w;
            const double flo = a2 ? (S1 - e * S0) : (S2 - 2.0 * e * S1 + e * e * S0);
            if (flo >= 1.0) best_lo = fmax(best_lo, e);
            const double c = (double)hist[j];
            const double lo = e - eps;
            S0 += c;
            S1 += c * lo;
            S2 += c * lo * lo;
        }
    }
    best_lo = warp_max_d(best_lo);
    if (lane == 0) brk[0][warp] = best_lo;
    __syncthreads();
    double lo_t = thr;
    for (int ww = 0; ww < kTauWarps; ++ww) lo_t = fmax(lo_t, brk[0][ww]);
    const bool spill = ncand > kTauCap;
    const float* src = spill ? x : cand;
    const int len = spill ? n : ncand;

    double tau = lo_t;
    if (gen) {
        // --- any alpha: Newton steps on G(t) = F(t)^(1/r) - 1, F(t) = sum (x - t)_+^r,
        // inside the bracket [M - 1, M] (F(M - 1) >= 1 > F(M) = 0), bisection
        // where a step leaves it.  For r >= 1, F^(1/r) is the r-norm of (x - t)_+:
        // convex, decreasing and close to linear, so steps from the left never
        // pass the root and converge in a few iterations (exactly in one when a
        // single value is above t).  Terms in float (powf), sums in float64.
        const double r = 1.0 / ((double)a.alpha - 1.0);
        const float rf = (float)r;
        double lo = thr, hi = (double)M;
        for (int it = 0; it < 100; ++it) {
            double v[3] = {0.0, 0.0, 0.0};
            float unused0 = INFINITY, unused1 = -INFINITY;
            for (int i = tid; i < len; i += kTauBlock) {
                const double vd = (double)src[i];
                if (vd > tau) {
                    const float u = (float)(vd - tau);
                    const float pu = powf(u, rf);
                    v[0] += (double)pu;
                    v[1] += (double)pu / (double)u;
                }
            }
            tau_reduce(R, it, v, unused0, unused1);
            const double F = v[0], S1 = r * v[1];          // F and -dF/dt
            if (F >= 1.0) lo = tau; else hi = tau;
            if (F == 1.0 || hi - lo <= 1e-13 * fmax(1.0, fabs(tau))) break;
            double nt = (F > 0.0 && S1 > 0.0) ? tau + r * F * (1.0 - pow(F, -1.0 / r)) / S1 : 0.5 * (lo + hi);
            if (!(nt > lo && nt < hi)) nt = 0.5 * (lo + hi);
            // the float terms fix F to about 1e-7 relative, tau to about 1e-8
            if (fabs(nt - tau) <= 1e-8 * fmax(1.0, fabs(tau))) {
                tau = nt;
                break;
            }
            tau = nt;
        }
    } else
    // --- Newton / closed form over {x > lo_t}
    for (int it = 0; it < 100; ++it) {
        double v[3] = {0.0, 0.0, 0.0};
        float minS = INFINITY, maxN = -INFINITY;
        for (int i = tid; i < len; i += kTauBlock) {
            const float f = src[i];
            const double vd = (double)f;
            if (!(vd > lo_t)) continue;
            if (vd > tau) {
                v[0] += 1.0;
                v[1] += vd;
                v[2] = fma(vd, vd, v[2]);
                minS = fminf(minS, f);
            } else {
                maxN = fmaxf(maxN, f);
            }
        }
        tau_reduce(R, it, v, minS, maxN);
        const double k = v[0], sx = v[1], sxx = v[2];
        double tcf;
        bool ok;
        if (a2) {
            tcf = (sx - 1.0) / k;
            ok = true;
        } else {
            const double mean = sx / k, msq = sxx / k;
            const double disc = mean * mean - msq + 1.0 / k;
            ok = disc >= 0.0;
            tcf = ok ? mean - sqrt(disc) : 0.0;
        }
        // consistent support: every kept value above tcf, every dropped one at or
        // below it (values at or below lo_t are below tau as well)
        if (ok && tcf < (double)minS && (double)maxN <= tcf && tcf >= lo_t) {
            tau = tcf;
            break;
        }
        double nt;
        if (a2) {
            nt = tcf;
        } else {
            const double s1 = sx - k * tau;
            const double s2 = sxx - 2.0 * tau * sx + k * tau * tau;
            nt = tau + (s2 - 1.0) / (2.0 * s1);
        }
        if (!(nt != tau) || !isfinite(nt)) break;
        tau = nt;
    }
    if (tid == 0) {
        a.tau[row] = (float)tau;
        if (a.tau_out) a.tau_out[row] = (float)tau;
    }
}

// ====================================================================== split reduction
// Each CTA has written its partial for (b, g); the last one to arrive sums the
// partials in split order.
template <int D, bool SOFTMAX>
EKV_DEV void reduce_splits(const AttnArgs& a, int b, int g)
{
    __shared__ int is_last;
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        const int t = atomicAdd(&a.counters[(size_t)b * a.H_kv + g], 1);
        is_last = (t == a.S - 1);
    }
    __syncthreads();
    if (!is_last) return;
    __threadfence();
    if (!SOFTMAX) {
        // four outputs per thread; up to 16 partials in flight, added in split
        // order (deterministic)
        for (int i = threadIdx.x; i < a.G * D / 4; i += blockDim.x) {
            const int head = 4 * i / D, dd = 4 * i % D;
            const size_t row = (size_t)b * a.H_q + (size_t)g * a.G + head;
            const float4* src = reinterpret_cast<const float4*>(a.opart + row * a.S * D + dd);
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int s0 = 0; s0 < a.S; s0 += 16) {
                float4 t[16];
#pragma unroll
                for (int u = 0; u < 16; ++u)
                    if (s0 + u < a.S) t[u] = __ldcg(src + (size_t)(s0 + u) * (D / 4));
#pragma unroll
                for (int u = 0; u < 16; ++u)
                    if (s0 + u < a.S) {
                        acc.x += t[u].x;
                        acc.y += t[u].y;
                        acc.z += t[u].z;
                        acc.w += t[u].w;
                    }
            }
            float* o = a.out + row * D + dd;
            o[0] = acc.x;
            o[1] = acc.y;
            o[2] = acc.z;
            o[3] = acc.w;
        }
    } else {
        for (int i = threadIdx.x; i < a.G * D; i += blockDim.x) {
            const int head = i / D, dd = i % D;
            const size_t row = (size_t)b * a.H_q + (size_t)g * a.G + head;
            float acc = 0.f;
            float Mx = -INFINITY;
            for (int s = 0; s < a.S; ++s) Mx = fmaxf(Mx, __ldcg(&a.mlpart[(row * a.S + s) * 2]));
            float l = 0.f;
            if (Mx != -INFINITY) {
                for (int s = 0; s < a.S; ++s) {
                    const float ms = __ldcg(&a.mlpart[(row * a.S + s) * 2]);
                    if (ms == -INFINITY) continue;
                    const float w = expf(ms - Mx);
                    l += w * __ldcg(&a.mlpart[(row * a.S + s) * 2 + 1]);
                    acc += w * __ldcg(&a.opart[(row * a.S + s) * D + dd]);
                }
            }
            a.out[row * D + dd] = l > 0.f ? acc / l : 0.f;
        }
    }
    if (threadIdx.x == 0) a.counters[(size_t)b * a.H_kv + g] = 0;
}

// ====================================================================== V pass
// Only pages holding a token with p > 0 for some head of the group are
// loaded: p = [x - tau]_+^(1/(alpha-1)) is exactly zero elsewhere, so the
// result is unchanged (support-aware value loading).  The split's pages are
// scanned in windows; each window's active pages are compacted into a list
// that feeds the TMA pipeline.
constexpr int kActWin = 512;

template <int D, int PS, int NT>
__global__ void __launch_bounds__(kThreads) pv_bf16_kernel(const __grid_constant__ CUtensorMap vmap, const AttnArgs a)
{
    pdl_enter();
    constexpr int STAGE = kStageTok * D * 2;
    constexpr int PPS = kStageTok / PS;
    constexpr int MTW = D / 64;           // 16-row m-tiles (head-dim rows) per warp
    constexpr int PROW = kStageTok + kPsPad;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_align<1024>(smem_raw);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStagesPV * STAGE);
    uint16_t* ps_tile = reinterpret_cast<uint16_t*>(smem + kStagesPV * STAGE + 64);   // [8*NT][PROW]
    __shared__ int abort_flag;
    __shared__ int act[kActWin];
    __shared__ unsigned char flag[kActWin];
    __shared__ int nact;
    __shared__ float tau_s[8];

    const int b = blockIdx.z, g = blockIdx.y, s = blockIdx.x;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int L = a.seq_lens[b];
    const int P = pages_of(L, PS, a.max_pages, a.status);
    const int cnt = list_count(a, b, g, P);
    const Range r = split_range(cnt, a.S, s);
    const bool a2 = a.alpha == 2.0f;
    const bool a15 = a.alpha == 1.5f;
    const float rexp = 1.0f / (a.alpha - 1.0f);   // weight exponent for any other alpha
    const size_t xstride = (size_t)a.k_max * PS;
    const size_t row0h = (size_t)b * a.H_q + (size_t)g * a.G;

    float acc[NT][MTW][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int m = 0; m < MTW; ++m) acc[nt][m][0] = acc[nt][m][1] = acc[nt][m][2] = acc[nt][m][3] = 0.f;

    tab_fill(a, b, g, r, P);
    if (tid < 8) tau_s[tid] = tid < a.G ? a.tau[row0h + tid] : INFINITY;
    if (tid == 0) {
        abort_flag = 0;
        prefetch_tmap(&vmap);
        for (int i = 0; i < kStagesPV; ++i) mbar_init(&bars[i], 1);
        fence_mbar_init();
    }
    for (int i = tid; i < 8 * NT * PROW; i += kThreads) ps_tile[i] = 0;
    __syncthreads();
    const uint32_t sbase = smem_addr(smem);
    const uint32_t pbase = smem_addr(ps_tile);
    int gst = 0;          // stages issued so far (barrier phase bookkeeping)
    int loaded = 0;

    for (int w0 = r.start; w0 < r.end; w0 += kActWin) {
        const int wn = min(kActWin, r.end - w0);
        // --- which pages of the window hold weight
        for (int i = tid; i < wn; i += kThreads) flag[i] = 0;
        __syncthreads();
        {
            constexpr int C = PS / 16;          // 16-token chunk maxima per page
            const size_t cstride = (size_t)a.k_max * C;
            const int items = wn * a.G;
            for (int it = tid; it < items; it += kThreads) {
                const int j = it / a.G, h = it % a.G;
                const float* cp = a.cmax + (row0h + h) * cstride + (size_t)(w0 + j) * C;
                float m = -INFINITY;
                if constexpr (C % 4 == 0) {
#pragma unroll
                    for (int k = 0; k < C; k += 4) {
                        const float4 v = *reinterpret_cast<const float4*>(cp + k);
                        m = fmaxf(m, fmaxf(fmaxf(v.x, v.y), fmaxf(v.z, v.w)));
                    }
                } else {
#pragma unroll
                    for (int k = 0; k < C; ++k) m = fmaxf(m, cp[k]);
                }
                if (m > tau_s[h]) flag[j] = 1;
            }
        }
        __syncthreads();
        if (warp == 0) {   // ordered compaction of the flags
            int base = 0;
            for (int i0 = 0; i0 < wn; i0 += 32) {
                const bool f = (i0 + lane < wn) && flag[i0 + lane];
                const unsigned m = __ballot_sync(0xffffffffu, f);
                if (f) act[base + __popc(m & ((1u << lane) - 1u))] = w0 + i0 + lane;
                base += __popc(m);
            }
            if (lane == 0) nact = base;
        }
        __syncthreads();
        const int na = nact;
        loaded += na;
        const int nst = (na + PPS - 1) / PPS;
        if (nst == 0) continue;
        // --- pipeline over the active pages
        auto issue = [&](int st, int slot_) {
            uint8_t* dst = smem + slot_ * STAGE;
            int phys[PPS];
            uint32_t bytes = 0;
#pragma unroll
            for (int i = 0; i < PPS; ++i) {
                const int ai = st * PPS + i;
                int lp;
                phys[i] = ai < na ? resolve(a, b, g, act[ai], P, lp, true) : -1;
                if (phys[i] >= 0) bytes += PS * D * 2;
            }
            mbar_arrive_expect_tx(&bars[slot_], bytes);
#pragma unroll
            for (int i = 0; i < PPS; ++i) {
                if (phys[i] < 0) continue;
                const int y = (phys[i] * a.H_kv + g) * PS;
#pragma unroll
                for (int hh = 0; hh < D / 64; ++hh)
                    tma_load_2d(dst + hh * (kStageTok * 128) + i * PS * 128, &vmap, &bars[slot_], hh * 64, y);
            }
        };
        if (tid == 0)
            for (int st = 0; st < min(kStagesPV, nst); ++st) issue(st, (gst + st) % kStagesPV);
        for (int st = 0; st < nst; ++st) {
            const int gs = gst + st;
            const int slot = gs % kStagesPV;
            // weights of this stage: token tid % 64, heads (tid / 64) * 2 * NT ...
            {
                const int t = tid & (kStageTok - 1);
                const int ai = st * PPS + t / PS;
                const int prow = t % PS;
                int idx = -1;
                bool valid = false;
                if (ai < na) {
                    idx = act[ai];
                    int lp;
                    const int phys = resolve(a, b, g, idx, P, lp, false);
                    valid = phys >= 0 && lp * PS + prow < L;
                }
                const int hbase = (tid >> 6) * 2 * NT;
#pragma unroll
                for (int k = 0; k < 2 * NT; ++k) {
                    const int head = hbase + k;
                    float p = 0.f;
                    if (head < a.G && valid) {
                        const float xv = a.xbuf[(row0h + head) * xstride + (size_t)idx * PS + prow];
                        const float u = fmaxf(xv - tau_s[head], 0.f);
                        p = a2 ? u : (a15 ? u * u : powf(u, rexp));
                    }
                    uint32_t hi, lo;
                    split_bf16(p, hi, lo);
                    ps_tile[(2 * head) * PROW + t] = (uint16_t)hi;
                    ps_tile[(2 * head + 1) * PROW + t] = (uint16_t)lo;
                }
            }
            if (!mbar_wait(&bars[slot], (gs / kStagesPV) & 1, kWaitLimitNs)) {
                abort_flag = 1;
                report(a.status, ENTMAXKV_TIMEOUT);
            }
            __syncthreads();
            if (abort_flag) {
                if (tid == 0)
                    for (int k = st; k < min(st + kStagesPV, nst); ++k)
                        mbar_wait(&bars[(gst + k) % kStagesPV], ((gst + k) / kStagesPV) & 1, kWaitLimitNs);
                return;
            }
            // rows without a valid token are zeroed so zero weights never meet garbage
            {
                const int t = tid & (kStageTok - 1);
                const int half = tid >> 6;
                if (half < D / 64) {
                    const int ai = st * PPS + t / PS;
                    bool valid = false;
                    if (ai < na) {
                        int lp;
                        const int phys = resolve(a, b, g, act[ai], P, lp, false);
                        valid = phys >= 0 && lp * PS + (t % PS) < L;
                    }
                    if (!valid) {
                        uint4* rowp = reinterpret_cast<uint4*>(smem + slot * STAGE + half * (kStageTok * 128) + t * 128);
#pragma unroll
                        for (int k = 0; k < 8; ++k) rowp[k] = make_uint4(0, 0, 0, 0);
                        fence_proxy_async();
                    }
                }
            }
            __syncthreads();
            const uint32_t base = sbase + slot * STAGE;
            const int n = lane >> 2, c = lane & 3;
#pragma unroll
            for (int kk = 0; kk < kStageTok / 16; ++kk) {
                uint32_t b0[NT], b1[NT];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const uint32_t pr = pbase + ((8 * nt + n) * PROW + 16 * kk + 2 * c) * 2;
                    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(b0[nt]) : "r"(pr));
                    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(b1[nt]) : "r"(pr + 16));
                }
                const int mi = lane >> 3;
                const int trow = 16 * kk + (lane & 7) + 8 * (mi >> 1);
#pragma unroll
                for (int m = 0; m < MTW; ++m) {
                    const int d0 = 16 * (warp * MTW + m);
                    uint32_t af[4];
                    ldsm_x4_t(swz_addr(base, trow, d0 / 8 + (mi & 1)), af);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) mma_bf16(acc[nt][m], af, b0[nt], b1[nt]);
                }
            }
            __syncthreads();
            if (tid == 0 && st + kStagesPV < nst) issue(st + kStagesPV, (gs + kStagesPV) % kStagesPV);
        }
        gst += nst;
    }
    if (tid == 0 && a.vpages) atomicAdd(&a.vpages[(size_t)b * a.H_kv + g], loaded);
    // partial output of this split: o[head 4nt + c][d]
    {
        const int c = lane & 3, gi = lane >> 2;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int head = 4 * nt + c;
            if (head >= a.G) continue;
            const size_t row = (row0h + head) * a.S + s;
#pragma unroll
            for (int m = 0; m < MTW; ++m) {
                const int d = 16 * (warp * MTW + m) + gi;
                a.opart[row * D + d] = acc[nt][m][0] + acc[nt][m][1];
                a.opart[row * D + d + 8] = acc[nt][m][2] + acc[nt][m][3];
            }
        }
    }
    reduce_splits<D, false>(a, b, g);
}

template <int D>
__global__ void __launch_bounds__(kThreads) pv_f32_kernel(const float* __restrict__ v_pool, int ps, const AttnArgs a)
{
    pdl_enter();
    const int b = blockIdx.z, g = blockIdx.y, s = blockIdx.x, tid = threadIdx.x;
    const int L = a.seq_lens[b];
    const int P = pages_of(L, ps, a.max_pages, a.status);
    const int cnt = list_count(a, b, g, P);
    const Range r = split_range(cnt, a.S, s);
    tab_fill(a, b, g, r, P);
    const size_t xstride = (size_t)a.k_max * ps;
    const bool a2 = a.alpha == 2.0f;
    const bool a15 = a.alpha == 1.5f;
    const double rexp = 1.0 / ((double)a.alpha - 1.0);
    for (int w = tid; w < a.G * D; w += kThreads) {
        const int head = w / D, dd = w % D;
        const size_t row = (size_t)b * a.H_q + (size_t)g * a.G + head;
        const float tau = a.tau[row];
        double acc = 0.0;
        for (int idx = r.start; idx < r.end; ++idx) {
            int lp;
            const int phys = resolve(a, b, g, idx, P, lp, false);
            if (phys < 0) continue;
            for (int t = 0; t < ps && lp * ps + t < L; ++t) {
                const float xv = a.xbuf[row * xstride + (size_t)idx * ps + t];
                const double u = fmax((double)xv - (double)tau, 0.0);
                if (u > 0.0) {
                    const double p = a2 ? u : (a15 ? u * u : pow(u, rexp));
                    acc = fma(p, (double)v_pool[(((size_t)phys * a.H_kv + g) * ps + t) * D + dd], acc);
                }
            }
        }
        a.opart[(row * a.S + s) * D + dd] = (float)acc;
    }
    if (tid == 0 && a.vpages) {   // pages of this split holding weight for some head
        int n = 0;
        for (int idx = r.start; idx < r.end; ++idx) {
            int lp;
            if (resolve(a, b, g, idx, P, lp, false) < 0) continue;
            bool any = false;
            for (int head = 0; head < a.G && !any; ++head) {
                const size_t row = (size_t)b * a.H_q + (size_t)g * a.G + head;
                const float tau = a.tau[row];
                for (int t = 0; t < ps && lp * ps + t < L; ++t)
                    if (a.xbuf[row * xstride + (size_t)idx * ps + t] > tau) { any = true; break; }
            }
            n += any;
        }
        atomicAdd(&a.vpages[(size_t)b * a.H_kv + g], n);
    }
    reduce_splits<D, false>(a, b, g);
}

// ====================================================================== fused entmax (bf16 cache)
// One launch runs the K pass, the threshold and the V pass.  The S splits of
// a (sequence, kv head) form one thread-block cluster, whose CTAs are
// scheduled together, so cluster barriers (about 0.2 us on B200) separate the
// phases:
//   K pass      each split scores its pages and writes x and the 16-token
//               chunk maxima to the workspace;
//   local       each split, one warp per query head, finds a lower bound t_s
//               of tau from its own chunk maxima (split_bound) and writes its
//               scores above t_s, with their list positions, to its slots in
//               the workspace (local_candidates); t_s, its largest score and
//               its candidate count stay in shared memory;
//   barrier 1
//   threshold   every CTA reads the splits' bounds and counts (distributed
//               shared memory) and their candidates (global memory); the
//               largest bound is a lower bound of tau for the whole group, so
//               the candidates above it hold every score that can carry
//               weight (gather_candidates); tau of every query head is solved
//               from them, one warp per head, with the same operations in the
//               same order in every CTA, so all splits hold the same tau; the
//               candidates above tau mark the value pages that hold weight,
//               and CTA s takes every S-th of them in list order, their page
//               ids read from the owning split's table;
//   V pass      each CTA accumulates P.V over its value pages and keeps its
//               partial output in shared memory;
//   barrier 2
//   merge       CTA r adds the partials of the output elements
//               [r E / S, (r + 1) E / S) in CTA order (deterministic);
//   barrier 3   no CTA leaves while another may still read its memory.
// Bulk data crosses CTAs through global memory (written before the barrier
// behind a fence, read through L2 with ld.global.cg), a few words per CTA
// through distributed shared memory.  Where a split has more candidates than
// its slots hold, every CTA instead solves over all the group's scores and
// loads the value pages of its own split.  No CTA leaves before the last
// barrier, whatever happens (a timed-out copy only skips work).
constexpr int kFusedStages = 5;
constexpr int kCandCap = kFusedCandCap;   // candidate slots per (split, query head) in the workspace
constexpr int kBitWords = 128;            // weighted-page bitmap: lists of up to 4096 pages (the clustered
                                          // kernel's longest: 16 splits of 4096 tokens in pages of 16)
constexpr int kFusedMaxSplitTokens = 4096; // listed tokens per split (per query head) the fused kernel takes

// Warp-wide sum of three doubles and min / max of two floats (xor butterfly:
// every lane ends with the same values).
EKV_DEV void warp_red5(double (&v)[3], float& mn, float& mx)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
#pragma unroll
        for (int i = 0; i < 3; ++i) v[i] += __shfl_xor_sync(0xffffffffu, v[i], o);
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    }
}

// Warp-wide sums of three floats (xor butterfly, every lane the same values).
EKV_DEV void warp_sum3(float& a, float& b, float& c)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        a += __shfl_xor_sync(0xffffffffu, a, o);
        b += __shfl_xor_sync(0xffffffffu, b, o);
        c += __shfl_xor_sync(0xffffffffu, c, o);
    }
}

// Where the candidates of a head's threshold are read from.
struct TauSrc {
    const float* cand;  // the candidate scores (shared)
    int ncand;
    double lo;          // every candidate is > lo; every other score is <= lo <= tau
};

// f(x) for every candidate x of the head; lane l takes every 32nd one.
template <typename Fn>
EKV_DEV void for_candidates(const TauSrc& s, Fn&& f)
{
    const int lane = threadIdx.x & 31;
    for (int i = lane; i < s.ncand; i += 32) f(s.cand[i]);
}

// Lower bound of tau from one split's chunk maxima, by one warp.  cm: the
// maxima of the split's own chunks [c0, c1) (cm[c - c0]); m_s the split's largest
// score.  Every chunk maximum is the score of a distinct token, so for any
// subset of the head's tokens sum_i (x_i - t)_+^r >= sum over the subset's
// chunk maxima, and the root of the latter is at or below tau.  Up to three
// Newton steps from m_s - 1 on that sum (convex and decreasing for r >= 1, so
// the steps stay at or below its root; r < 1 keeps m_s - 1).  The chunks
// above m_s - 1 (the only ones that can matter) are kept in (lc, lcv); *nlc
// is their number (more than cap: the list is unusable).
EKV_DEV float split_bound(const float* cm, int c0, int c1, float m_s, float r, bool a2, bool a15, int* lc,
                          float* lcv, int cap, int* nlc)
{
    const int lane = threadIdx.x & 31;
    const unsigned below = (1u << lane) - 1u;
    if (!(m_s > -INFINITY)) {
        *nlc = 0;
        return -INFINITY;
    }
    const float thr = __fsub_rd(m_s, 1.0f);
    int n = 0;
    constexpr int U = 8;
    for (int i0 = c0; i0 < c1; i0 += 32 * U) {
        float v[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int i = i0 + u * 32 + lane;
            v[u] = i < c1 ? cm[i - c0] : -INFINITY;
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const bool keep = v[u] > thr;
            const unsigned m = __ballot_sync(0xffffffffu, keep);
            const int pos = n + __popc(m & below);
            if (keep && pos < cap) {
                lc[pos] = i0 + u * 32 + lane;
                lcv[pos] = v[u];
            }
            n += __popc(m);
        }
    }
    __syncwarp();
    *nlc = n;
    float t = thr;
    if (n <= cap && r >= 1.0f) {
        for (int it = 0; it < 3; ++it) {
            float F = 0.f, dF = 0.f, unused = 0.f;
            for (int j = lane; j < n; j += 32) {
                const float u = lcv[j] - t;
                if (u > 0.f) {
                    const float p1 = a2 ? 1.f : (a15 ? u : powf(u, r - 1.f));
                    F = fmaf(p1, u, F);
                    dF = fmaf(r, p1, dF);
                }
            }
            warp_sum3(F, dF, unused);
            if (!(F > 1.f) || !(dF > 0.f)) break;      // at (or by rounding past) the root
            t += (F - 1.f) / dF;
        }
        t -= 1e-5f * fmaxf(1.f, fabsf(t));             // the float steps may have rounded past the root
    }
    return fmaxf(t, thr);                              // at least m_s - 1 (rounded down), itself a bound
}

// One split's candidates of one head, by one warp: its scores above t with
// their list positions, to oval / oidx (global, at most kCandCap kept);
// returns how many there are.  The chunks to read: those of split_bound's
// list above t (the list holds every chunk above m_s - 1 <= t), or all the
// split's chunks [c0, c1) when the list overflowed.
EKV_DEV int local_candidates(const float* x, int c0, int c1, int* lc, const float* lcv, int nlc, int cap, float t,
                             float* oval, int* oidx)
{
    const int lane = threadIdx.x & 31;
    const unsigned below = (1u << lane) - 1u;
    constexpr int U = 8;
    int nf = 0;
    const bool listed = nlc <= cap;
    if (listed) {                                      // chunks above t, compacted in place (order kept)
        for (int j0 = 0; j0 < nlc; j0 += 32) {
            const int j = j0 + lane;
            const bool keep = j < nlc && lcv[j] > t;
            const int c = keep ? lc[j] : 0;
            const unsigned m = __ballot_sync(0xffffffffu, keep);
            __syncwarp();
            if (keep) lc[nf + __popc(m & below)] = c;
            nf += __popc(m);
            __syncwarp();
        }
    }
    const int nk = listed ? nf * 16 : (c1 - c0) * 16;
    int nc = 0;
    for (int k0 = 0; k0 < nk; k0 += 32 * U) {
        float v[U];
        int pos[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int k = k0 + u * 32 + lane;
            pos[u] = k < nk ? (listed ? lc[k >> 4] * 16 + (k & 15) : c0 * 16 + k) : 0;
            v[u] = k < nk ? x[pos[u]] : -INFINITY;
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const bool keep = v[u] > t;
            const unsigned m = __ballot_sync(0xffffffffu, keep);
            const int q = nc + __popc(m & below);
            if (keep && q < kCandCap) {
                oval[q] = v[u];
                oidx[q] = pos[u];
            }
            nc += __popc(m);
        }
    }
    return nc;
}

// The group's candidates of one head (every one above the group's bound),
// gathered by one warp from the S splits' slots (global: split q's n_q of them
// at cval + q * kCandCap, lane q holding n_q) into (cv, ci) in one round trip:
// 16-byte asynchronous copies, split q's at the next 4-entry boundary, the up
// to three entries past its count set to -inf (no candidate).  Returns the
// entries written, gaps included (-1 when more than cap).  pre: per-warp
// shared scratch of S + 1 ints.
EKV_DEV int gather_candidates(const float* cval, const int* cidx, int nq, int S, float* cv, int* ci, int cap,
                              int* pre)
{
    const int lane = threadIdx.x & 31;
    const int n4 = lane < S ? (nq + 3) & ~3 : 0;
    int incl = n4;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
    }
    if (lane < S) pre[lane + 1] = incl;
    if (lane == 0) pre[0] = 0;
    const int total = __shfl_sync(0xffffffffu, incl, 31);
    __syncwarp();
    if (total > cap) return -1;
    const uint32_t vbase = smem_addr(cv), ibase = smem_addr(ci);
    for (int q = 0; q < S; ++q) {
        const int o = pre[q], chunks = (pre[q + 1] - o) >> 2;
        for (int c = lane; c < chunks; c += 32) {
            cp_async16(vbase + 4u * (uint32_t)(o + 4 * c), cval + (size_t)q * kCandCap + 4 * c);
            cp_async16(ibase + 4u * (uint32_t)(o + 4 * c), cidx + (size_t)q * kCandCap + 4 * c);
        }
    }
    cp_async_commit();
    cp_async_wait<0>();
    __syncwarp();
    if (lane < S)
        for (int j = nq; j < n4; ++j) cv[pre[lane] + j] = -INFINITY;
    __syncwarp();
    return total;
}

// The exact closed form of tau on the support {x > t} of the candidates
// (float64, one warp, every lane the same): alpha = 2 gives (sum x - 1) / k,
// alpha = 1.5 the smaller root of sum (x - tau)^2 = 1.  NaN unless the support
// is consistent with it (every kept value above, every dropped one at or
// below, and at least the bound); *next: the next iterate from t (the fixed
// point for 2, a Newton step on sum (x - t)^2 = 1 for 1.5).
EKV_DEV double closed_form(const TauSrc& src, bool a2, double t, double* next)
{
    double v[3] = {0.0, 0.0, 0.0};
    float minS = INFINITY, maxN = -INFINITY;
    for_candidates(src, [&](float f) {
        const double vd = (double)f;
        if (vd > t) {
            v[0] += 1.0;
            v[1] += vd;
            v[2] = fma(vd, vd, v[2]);
            minS = fminf(minS, f);
        } else {
            maxN = fmaxf(maxN, f);
        }
    });
    warp_red5(v, minS, maxN);
    const double k = v[0], sx = v[1], sxx = v[2];
    double tcf;
    bool ok;
    if (a2) {
        tcf = (sx - 1.0) / k;
        ok = true;
        *next = tcf;
    } else {
        const double mean = sx / k, msq = sxx / k;
        const double disc = mean * mean - msq + 1.0 / k;
        ok = disc >= 0.0;
        tcf = ok ? mean - sqrt(disc) : 0.0;
        const double s1 = sx - k * t;
        const double s2 = sxx - 2.0 * t * sx + k * t * t;
        *next = t + (s2 - 1.0) / (2.0 * s1);
    }
    return (ok && tcf < (double)minS && (double)maxN <= tcf && tcf >= src.lo) ? tcf : NAN;
}

// tau of solve_tau for any alpha other than 1.5 and 2: safeguarded Newton
// steps on F^(1/r) inside [src.lo, M] (kept out of line: the alpha = 1.5 and
// 2 path does not fetch its code).
__device__ __noinline__ double solve_tau_general(const TauSrc src, float M, float alpha)
{
    // Newton on G(t) = F(t)^(1/r) - 1 inside [lo, hi] (F(lo) >= 1 > F(M) = 0),
    // bisection where a step leaves it; terms in float (powf), sums in float64
    double tau = src.lo;
    const double r = 1.0 / ((double)alpha - 1.0);
    const float rf = (float)r;
    double lo = src.lo, hi = (double)M;
    for (int it = 0; it < 100; ++it) {
        double v[3] = {0.0, 0.0, 0.0};
        float u0 = INFINITY, u1 = -INFINITY;
        for_candidates(src, [&](float f) {
            const double vd = (double)f;
            if (vd > tau) {
                const float u = (float)(vd - tau);
                const float pu = powf(u, rf);
                v[0] += (double)pu;
                v[1] += (double)pu / (double)u;
            }
        });
        warp_red5(v, u0, u1);
        const double F = v[0], S1 = r * v[1];
        if (F >= 1.0) lo = tau; else hi = tau;
        if (F == 1.0 || hi - lo <= 1e-13 * fmax(1.0, fabs(tau))) break;
        double nt = (F > 0.0 && S1 > 0.0) ? tau + r * F * (1.0 - pow(F, -1.0 / r)) / S1 : 0.5 * (lo + hi);
        if (!(nt > lo && nt < hi)) nt = 0.5 * (lo + hi);
        if (fabs(nt - tau) <= 1e-8 * fmax(1.0, fabs(tau))) {
            tau = nt;
            break;
        }
        tau = nt;
    }
    return tau;
}

__device__ __noinline__ double solve_tau_refine(const TauSrc src, bool a2, float t);

// tau from the candidates of src, one warp, every lane returns it.
//  alpha = 2 and 1.5: steps in float from the bound src.lo -- Newton on
//  sum (x - t)^2 = 1 for 1.5, the fixed point t = (sum x - 1) / k for 2, both
//  from the left over the current support {x > t} -- until the support holds
//  for a step; then the closed form on that support in float64, accepted when
//  the support is consistent with it (every kept value above, every dropped
//  one at or below).  Should rounding in float leave the support
//  inconsistent, the same iteration runs in float64 (solve_tau_refine).
//  Any other alpha: solve_tau_general.
EKV_DEV double solve_tau(const TauSrc& src, float M, float alpha)
{
    const bool a2 = alpha == 2.0f;
    const bool a15 = alpha == 1.5f;
    if (!a2 && !a15) return solve_tau_general(src, M, alpha);
    // float iteration to the support
    float t = (float)src.lo;
    float kprev = -1.f;
    for (int it = 0; it < 64; ++it) {
        float k = 0.f, s1 = 0.f, s2 = 0.f;
        for_candidates(src, [&](float f) {
            const float u = f - t;
            if (u > 0.f) {
                k += 1.f;
                s1 += a2 ? f : u;
                s2 = fmaf(u, u, s2);
            }
        });
        warp_sum3(k, s1, s2);
        if (k == kprev) break;
        kprev = k;
        const float nt = a2 ? (s1 - 1.f) / k : t + (s2 - 1.f) / (2.f * s1);
        if (!(nt > t)) break;
        t = nt;
    }
    double next = 0.0;
    const double tc = closed_form(src, a2, (double)t, &next);
    if (tc == tc) return tc;
    return solve_tau_refine(src, a2, t);
}

// The float64 iteration of solve_tau for when the float iterate's support was
// not consistent with its closed form (kept out of line: rarely taken).
__device__ __noinline__ double solve_tau_refine(const TauSrc src, bool a2, float t)
{
    double next = 0.0;
    // float64 steps from just below the float iterate (rounding left the float
    // support off by a value or two); should that start lie right of the root
    // (a step that does not move right), from the bound itself
    double tau = fmax(src.lo, (double)t - 1e-4 * fmax(1.0, fabs((double)t)));
    bool restarted = tau == src.lo;
    for (int it = 0; it < 100; ++it) {
        const double c = closed_form(src, a2, tau, &next);
        if (c == c) return c;
        if (!(next > tau) || !isfinite(next)) {
            if (restarted) break;
            tau = src.lo;
            restarted = true;
            continue;
        }
        tau = next;
    }
    return tau;
}

// tau of every head by the whole cluster, for when a head's candidates do not
// fit the slots: each iteration every CTA sums its own split's scores of the
// head at the current iterate (one warp per head, heads h and h + 4 on warp
// h % 4), the S partial sums go through distributed shared memory, and every
// CTA adds them in split order (lane q holds split q; the xor butterfly gives
// every lane, and so every CTA, the same bits) and takes the same step, so
// all CTAs hold the same iterates and leave the loop after the same barrier.
//  alpha = 2 and 1.5: from the group bound, the closed form on the current
//  support {x > t}; accepted when the support is consistent with it, else t
//  moves to the next iterate from the left (t = (sum x - 1) / k for 2, a
//  Newton step on sum (x - t)^2 = 1 for 1.5).
//  Any other alpha: safeguarded Newton steps on F^(1/r) inside [bound, max].
// x: score row of head 0 (heads xstride apart); [t0, t1): this split's
// tokens; skip: this CTA adds nothing (it gave up on a copy); part, mm:
// shared [2][8][3] doubles and [2][8][2] floats; pub_t, pub_m: every split's
// bound and largest score per head (read through distributed shared memory);
// tau_h: tau per head, out (every CTA).
__device__ __noinline__ void cluster_tau(const float* x, size_t xstride, int t0, int t1, const float* pub_t,
                                        const float* pub_m,
                         int G, int S, float alpha, bool skip, double* part, float* mm, double* tau_h)
{
    constexpr int kMaxIt = 48;
    constexpr int U = 8;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const bool a2 = alpha == 2.0f, a15 = alpha == 1.5f, gen = !a2 && !a15;
    const double r = 1.0 / ((double)alpha - 1.0);
    const float rm1 = (float)(r - 1.0);
    double t[2], lo[2], hi[2], res[2];
    bool dn[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const int h = warp + 4 * k;
        dn[k] = true;
        t[k] = lo[k] = hi[k] = res[k] = INFINITY;
        if (h < G) {
            float tb = lane < S ? ld_dsmem_f32(dsmem(&pub_t[h], lane)) : -INFINITY;
            float mx = lane < S ? ld_dsmem_f32(dsmem(&pub_m[h], lane)) : -INFINITY;
            tb = warp_max(tb);
            mx = warp_max(mx);
            dn[k] = !(mx > -INFINITY);           // no scores: tau = +inf, nothing is kept
            t[k] = lo[k] = (double)tb;
            hi[k] = (double)mx;
        }
    }
    for (int it = 0; it < kMaxIt; ++it) {
        const int bf = it & 1;
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            const int h = warp + 4 * k;
            if (h >= G) continue;
            double v[3] = {0.0, 0.0, 0.0};
            float mnS = INFINITY, mxN = -INFINITY;
            if (!dn[k] && !skip) {
                const float* xr = x + (size_t)h * xstride;
                const double tk = t[k];
                for (int i0 = t0; i0 < t1; i0 += 32 * U) {
                    float f[U];
#pragma unroll
                    for (int u = 0; u < U; ++u) {
                        const int i = i0 + u * 32 + lane;
                        f[u] = i < t1 ? __ldcg(xr + i) : -INFINITY;
                    }
#pragma unroll
                    for (int u = 0; u < U; ++u) {
                        const double vd = (double)f[u];
                        if (vd > tk) {
                            if (gen) {
                                const float uu = (float)(vd - tk);
                                if (uu > 0.f) {
                                    const float p1 = powf(uu, rm1);
                                    v[0] += (double)(p1 * uu);
                                    v[1] += (double)p1;
                                }
                            } else {
                                v[0] += 1.0;
                                v[1] += vd;
                                v[2] = fma(vd, vd, v[2]);
                                mnS = fminf(mnS, f[u]);
                            }
                        } else if (f[u] > -INFINITY) {
                            mxN = fmaxf(mxN, f[u]);
                        }
                    }
                }
            }
            warp_red5(v, mnS, mxN);
            if (lane == 0) {
                double* pp = part + (bf * 8 + h) * 3;
                pp[0] = v[0];
                pp[1] = v[1];
                pp[2] = v[2];
                mm[(bf * 8 + h) * 2] = mnS;
                mm[(bf * 8 + h) * 2 + 1] = mxN;
            }
        }
        __syncthreads();
        cluster_sync();
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            const int h = warp + 4 * k;
            if (h >= G || dn[k]) continue;
            double w[3] = {0.0, 0.0, 0.0};
            float mnS = INFINITY, mxN = -INFINITY;
            if (lane < S) {
                const double* pp = part + (bf * 8 + h) * 3;
#pragma unroll
                for (int j = 0; j < 3; ++j) w[j] = __longlong_as_double((long long)ld_dsmem_u64(dsmem(pp + j, lane)));
                mnS = ld_dsmem_f32(dsmem(&mm[(bf * 8 + h) * 2], lane));
                mxN = ld_dsmem_f32(dsmem(&mm[(bf * 8 + h) * 2 + 1], lane));
            }
            warp_red5(w, mnS, mxN);
            const double tk = t[k];
            if (gen) {
                const double F = w[0], S1 = r * w[1];     // F and -dF/dt
                if (F >= 1.0) lo[k] = tk; else hi[k] = tk;
                if (F == 1.0 || hi[k] - lo[k] <= 1e-13 * fmax(1.0, fabs(tk))) {
                    dn[k] = true;
                    res[k] = tk;
                } else {
                    double nt = (F > 0.0 && S1 > 0.0) ? tk + r * F * (1.0 - pow(F, -1.0 / r)) / S1
                                                      : 0.5 * (lo[k] + hi[k]);
                    if (!(nt > lo[k] && nt < hi[k])) nt = 0.5 * (lo[k] + hi[k]);
                    if (fabs(nt - tk) <= 1e-8 * fmax(1.0, fabs(tk))) {
                        dn[k] = true;
                        res[k] = nt;
                    }
                    t[k] = nt;
                }
            } else {
                const double kk = w[0], sx = w[1], sxx = w[2];
                if (!(kk > 0.0)) {
                    dn[k] = true;
                    res[k] = tk;
                } else {
                    double tcf, next;
                    bool ok;
                    if (a2) {
                        tcf = (sx - 1.0) / kk;
                        ok = true;
                        next = tcf;
                    } else {
                        const double mean = sx / kk, msq = sxx / kk;
                        const double disc = mean * mean - msq + 1.0 / kk;
                        ok = disc >= 0.0;
                        tcf = ok ? mean - sqrt(disc) : 0.0;
                        const double s1 = sx - kk * tk;
                        const double s2 = sxx - 2.0 * tk * sx + kk * tk * tk;
                        next = tk + (s2 - 1.0) / (2.0 * s1);
                    }
                    if (ok && tcf < (double)mnS && (double)mxN <= tcf && tcf >= lo[k]) {
                        dn[k] = true;
                        res[k] = tcf;
                    } else if (!(next > tk) || !isfinite(next)) {
                        dn[k] = true;
                        res[k] = ok ? tcf : tk;
                    } else {
                        t[k] = next;
                    }
                }
            }
        }
        // the same in every CTA: every head's iterates are
        if (__syncthreads_and(dn[0] && dn[1])) break;
    }
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const int h = warp + 4 * k;
        if (h < G && lane == 0) tau_h[h] = dn[k] ? res[k] : t[k];
    }
    __syncthreads();
}

// List position j of (b, g) -> physical page (and logical page in lp), read
// from the page table of the split that owns j (distributed shared memory;
// splits of `per` positions), or from global memory when that split resolved
// none.
EKV_DEV int resolve_peer(const AttnArgs& a, int b, int g, int j, int P, int per, int& lp)
{
    const int q = j / per;
    const int li = j - q * per;          // < per <= kTabCap: the three reads go out together
    const int n = ld_dsmem_s32(dsmem(&tab_n, q));
    const int l = ld_dsmem_s32(dsmem(&tab_lp[li], q));
    const int ph = ld_dsmem_s32(dsmem(&tab_phys[li], q));
    if (li < n) {
        lp = l;
        return ph;
    }
    return resolve_g(a, b, g, j, P, lp, true);
}

template <int D, int PS, int NT>
__global__ void __launch_bounds__(kThreads, 2) entmax_bf16_kernel(const __grid_constant__ CUtensorMap kmap,
                                                               const __grid_constant__ CUtensorMap vmap,
                                                               const AttnArgs a)
{
    pdl_enter();
    constexpr int NSTG = kFusedStages;
    constexpr int STAGE = kStageTok * D * 2;
    constexpr int PPS = kStageTok / PS;
    constexpr int KS = D / 16;
    constexpr int MTW = D / 64;            // 16-row m-tiles (head-dim rows) per warp in the V pass
    constexpr int PROW = kStageTok + kPsPad;
    constexpr int C = PS / 16;             // 16-token chunks per page
    constexpr int WSCR = NSTG * STAGE / 4; // per-warp scratch (in the stage buffers) between the passes
    constexpr int LC_CAP = WSCR / (8 * NT);// chunk-list entries per head (index + value)
    constexpr int CAND_CAP = WSCR / 8;     // gathered candidates of the head being solved (value + position)
    static_assert(kFusedMaxSplits <= 31, "split counts are held one per lane");
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_align<1024>(smem_raw);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + NSTG * STAGE);
    uint16_t* ps_tile = reinterpret_cast<uint16_t*>(smem + NSTG * STAGE + 64);   // [8*NT][PROW]
    float* part = reinterpret_cast<float*>(smem);                                // [G][D] after the V pass
    __shared__ int abort_flag;
    __shared__ float wm[4][8];
    __shared__ float smax[8];
    __shared__ float tau_s[8];
    __shared__ int fallback;
    __shared__ int wsum[4];
    __shared__ int pre[4][kFusedMaxSplits + 1];
    __shared__ int act[kActWin];
    __shared__ int act_phys[kActWin];
    __shared__ int act_lp[kActWin];
    __shared__ unsigned char flag[kActWin];
    __shared__ int nact;
    __shared__ unsigned int bits[kBitWords];      // weighted pages of the heads this CTA solved
    __shared__ unsigned int vbits[kBitWords];     // weighted pages of every head
    __shared__ float tau_pub[8];                  // tau of the heads this CTA solved
    __shared__ int fb_all;
    __shared__ int nlc_s[8];
    __shared__ int wbase[kBitWords];
    // this split's bound, largest score and candidate count per head (read by
    // the other CTAs through distributed shared memory)
    __shared__ float pub_t[8], pub_m[8];
    __shared__ int pub_n[8];
    // every split's bound, largest score and candidate count per head, as the
    // splits stored them into this CTA before the barriers (read locally)
    __shared__ float all_t[kFusedMaxSplits][8], all_m[kFusedMaxSplits][8];
    __shared__ int all_n[kFusedMaxSplits][8];
    // the largest score of every 16-token chunk of this split, per head
    __shared__ float cm_s[4 * NT][kFusedMaxSplitTokens / 16];
    // the cluster-wide threshold solve: partial sums per iteration parity and head
    __shared__ double ct_part[2 * 8 * 3];
    __shared__ float ct_mm[2 * 8 * 2];
    __shared__ double ct_tau[8];
    __shared__ int over_all;

    const int b = blockIdx.z, g = blockIdx.y, s = blockIdx.x;   // s = rank in the cluster
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // A full list (every top-k list once the sequence has k_max pages) fixes
    // this split's range before its count arrives: its first entries and their
    // page-table entries load together with the length and the count.
    const Range rs = split_range(a.k_max, a.S, s);
    const bool ahead = a.sel != nullptr && tid < rs.end - rs.start;
    const int L = a.seq_lens[b];
    const int ahead_lp = ahead ? a.sel[((size_t)b * a.H_kv + g) * a.k_max + rs.start + tid] : -1;
    const int ahead_phys =
        ahead_lp >= 0 && ahead_lp < a.max_pages ? a.page_table[(size_t)b * a.max_pages + ahead_lp] : -1;
    const int P = pages_of(L, PS, a.max_pages, a.status);
    const int cnt = list_count(a, b, g, P);
    const Range r = split_range(cnt, a.S, s);
    const int per_split = (cnt + a.S - 1) / a.S;
    const int nst = r.end > r.start ? (r.end - r.start + PPS - 1) / PPS : 0;
    const size_t row0h = (size_t)b * a.H_q + (size_t)g * a.G;
    const size_t xstride = (size_t)a.k_max * PS;
    const uint32_t sbase = smem_addr(smem);
    const bool a2 = a.alpha == 2.0f;
    const bool a15 = a.alpha == 1.5f;
    const float rpow = a2 ? 1.0f : (a15 ? 2.0f : 1.0f / (a.alpha - 1.0f));
    const size_t seg = (size_t)kFusedMaxSplits * kCandCap;   // candidate slots of one head row
    // the query first: its load overlaps the page-table lookups instead of
    // queueing behind the first key tiles
    uint32_t bq[NT][KS][2];
    load_q_frags<D, NT>(a, b, g, a.xscale, bq);
    tab_fill_ahead(a, b, g, r, P, rs, ahead_lp, ahead_phys);

    // ------------------------------------------------------------ K pass
    if (tid == 0) {
        abort_flag = 0;
        fallback = 0;
        fb_all = 0;
        prefetch_tmap(&kmap);
        prefetch_tmap(&vmap);
        for (int i = 0; i < NSTG; ++i) mbar_init(&bars[i], 1);
        fence_mbar_init();
        for (int st = 0; st < min(NSTG, nst); ++st)
            issue_stage<D, PS>(a, &kmap, smem + st * STAGE, &bars[st], b, g, r, st, P);
    }
    for (int i = tid; i < kBitWords; i += kThreads) bits[i] = 0;
    if (tid < 8) {
        pub_t[tid] = -INFINITY;
        pub_m[tid] = -INFINITY;
        pub_n[tid] = 0;
    }
    float run[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) run[nt] = -INFINITY;
    __syncthreads();
    int kst = 0;
    for (; kst < nst; ++kst) {
        const int st = kst;
        const int slot = st % NSTG;
        if (!mbar_wait(&bars[slot], (st / NSTG) & 1, kWaitLimitNs)) {
            abort_flag = 1;
            report(a.status, ENTMAXKV_TIMEOUT);
        }
        __syncthreads();
        if (abort_flag) break;
        const uint32_t base = sbase + slot * STAGE;
        const int row0 = warp * 16;
        float acc[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
        const int arow = row0 + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
        for (int j = 0; j < KS; ++j) {
            uint32_t af[4];
            ldsm_x4(swz_addr(base, arow, 2 * j + (lane >> 4)), af);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) mma_bf16(acc[nt], af, bq[nt][j][0], bq[nt][j][1]);
        }
        // the warp's 16 rows lie in one page (16 divides PS): one list entry, one chunk
        const int gi = lane >> 2, c = lane & 3;
        const int idx = r.start + st * PPS + row0 / PS;
        if (idx < r.end) {
            int lp;
            const int phys = resolve(a, b, g, idx, P, lp, false);
            float cmx[NT];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) cmx[nt] = -INFINITY;
#pragma unroll
            for (int rr = 0; rr < 2; ++rr) {
                const int prow = (row0 + gi + 8 * rr) % PS;
                const bool valid = phys >= 0 && lp * PS + prow < L;
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const int head = 4 * nt + c;
                    const float xv = valid ? acc[nt][2 * rr] + acc[nt][2 * rr + 1] : -INFINITY;
                    cmx[nt] = fmaxf(cmx[nt], xv);
                    if (head < a.G) a.xbuf[(row0h + head) * xstride + (size_t)idx * PS + prow] = xv;
                }
            }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const float m = group_lane_max(cmx[nt]);
                run[nt] = fmaxf(run[nt], m);
                const int head = 4 * nt + c;
                if (gi == 0 && head < a.G) cm_s[head][(idx - r.start) * C + (row0 % PS) / 16] = m;
            }
        }
        __syncthreads();
        if (tid == 0 && st + NSTG < nst)
            issue_stage<D, PS>(a, &kmap, smem + slot * STAGE, &bars[slot], b, g, r, st + NSTG, P);
    }
    if (abort_flag && tid == 0)   // copies still in flight must land before the buffers are reused
        for (int k = kst; k < min(kst + NSTG, nst); ++k) mbar_wait(&bars[k % NSTG], (k / NSTG) & 1, kWaitLimitNs);
    // this split's largest score per head
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const float m = group_lane_max(run[nt]);
        if (lane < 4) wm[warp][4 * nt + (lane & 3)] = m;
    }
    __syncthreads();
    if (tid < 8) smax[tid] = tid < a.G ? fmaxf(fmaxf(wm[0][tid], wm[1][tid]), fmaxf(wm[2][tid], wm[3][tid])) : -INFINITY;
    __syncthreads();

    // ------------------------------------------------------------ local bound, then candidates
    // above the group's bound (the largest of the splits' bounds)
    const int c0 = r.start * C, c1 = r.end * C;
    if (!abort_flag) {
        for (int h = warp, k = 0; h < a.G; h += 4, ++k) {
            int* lc = reinterpret_cast<int*>(smem + warp * WSCR + k * LC_CAP * 8);
            float* lcv = reinterpret_cast<float*>(smem + warp * WSCR + k * LC_CAP * 8 + LC_CAP * 4);
            int nlc;
            const float t = split_bound(cm_s[h], c0, c1, smax[h], rpow, a2, a15, lc, lcv, LC_CAP, &nlc);
            if (lane == 0) {
                pub_t[h] = t;
                pub_m[h] = smax[h];
                nlc_s[h] = nlc;
            }
        }
    }
    __syncthreads();
    if (tid < a.S * 8) {   // this split's bound and largest score per head into every CTA
        const int q = tid >> 3, h = tid & 7;
        st_dsmem_f32(dsmem(&all_t[s][h], q), pub_t[h]);
        st_dsmem_f32(dsmem(&all_m[s][h], q), pub_m[h]);
    }
    cluster_sync();
    if (!abort_flag) {
        for (int h = warp, k = 0; h < a.G; h += 4, ++k) {
            const size_t row = row0h + h;
            int* lc = reinterpret_cast<int*>(smem + warp * WSCR + k * LC_CAP * 8);
            float* lcv = reinterpret_cast<float*>(smem + warp * WSCR + k * LC_CAP * 8 + LC_CAP * 4);
            float tlb = lane < a.S ? all_t[lane][h] : -INFINITY;
            tlb = warp_max(tlb);
            const int n = local_candidates(a.xbuf + row * xstride, c0, c1, lc, lcv, nlc_s[h], LC_CAP, tlb,
                                           a.cval + row * seg + (size_t)s * kCandCap,
                                           a.cidx + row * seg + (size_t)s * kCandCap);
            if (lane == 0) pub_n[h] = n;
        }
    }
    __threadfence();   // candidates and scores in global memory are read by the other splits
    __syncthreads();
    if (tid < a.S * 8)     // this split's candidate count per head into every CTA
        st_dsmem_s32(dsmem(&all_n[s][tid & 7], tid >> 3), pub_n[tid & 7]);
    cluster_sync();

    // ------------------------------------------------------------ threshold
    // Every CTA reads every split's candidate counts.  When some split's
    // candidates of a head outgrew its slots, or a head's outgrow what one warp
    // gathers, the whole cluster solves every head (cluster_tau; the same
    // decision in every CTA) and the V pass takes each split's own pages.
    // Otherwise query head h is solved by CTA h % S, on its warp (h / S) % 4;
    // the owner keeps tau and the head's weighted pages for the others.
    const bool bitmap_ok = cnt <= kBitWords * 32;
    if (tid < 32) {
        int nh[8];                                            // every read goes out before the first use
#pragma unroll
        for (int h = 0; h < 8; ++h) nh[h] = h < a.G && lane < a.S ? all_n[lane][h] : 0;
        bool o = false;
#pragma unroll
        for (int h = 0; h < 8; ++h) {
            const int tot = warp_sum((nh[h] + 3) & ~3);       // as gathered: 4-entry aligned per split
            o = o || __any_sync(0xffffffffu, nh[h] > kCandCap) || tot > CAND_CAP;
        }
        if (tid == 0) over_all = o;
    }
    __syncthreads();
    if (over_all) {
        cluster_tau(a.xbuf + row0h * xstride, xstride, r.start * PS, r.end * PS, pub_t, pub_m, a.G, a.S, a.alpha,
                    abort_flag != 0, ct_part, ct_mm, ct_tau);
        if (tid < a.G) {
            tau_pub[tid] = (float)ct_tau[tid];
            if (a.tau_out && tid % a.S == s) a.tau_out[row0h + tid] = (float)ct_tau[tid];
        }
        if (tid == 0) fallback = 1;
    } else if (!abort_flag) {
        float* cv = reinterpret_cast<float*>(smem + warp * WSCR);
        int* ci = reinterpret_cast<int*>(smem + warp * WSCR + CAND_CAP * 4);
        for (int h = s + warp * a.S; h < a.G; h += 4 * a.S) {
            const size_t row = row0h + h;
            float M = -INFINITY, tlb = -INFINITY;
            int nq = 0;
            if (lane < a.S) {
                M = all_m[lane][h];
                tlb = all_t[lane][h];
                nq = all_n[lane][h];
            }
            M = warp_max(M);
            tlb = warp_max(tlb);
            double tau = INFINITY;
            if (M > -INFINITY) {
                // at most CAND_CAP entries in all (over_all is false)
                const int nc = gather_candidates(a.cval + row * seg, a.cidx + row * seg, nq, a.S, cv, ci, CAND_CAP,
                                                 pre[warp]);
                TauSrc src{cv, max(nc, 0), (double)tlb};
                tau = solve_tau(src, M, a.alpha);
                // value pages holding weight: the pages of the candidates above tau
                if (bitmap_ok)
                    for (int k = lane; k < nc; k += 32)
                        if ((double)cv[k] > tau) {
                            const int pg = ci[k] / PS;
                            atomicOr(&bits[pg >> 5], 1u << (pg & 31));
                        }
            }
            if (lane == 0) {
                tau_pub[h] = (float)tau;
                if (a.tau_out) a.tau_out[row] = (float)tau;
            }
            __syncwarp();
        }
    }
    fence_proxy_async();   // the scratch writes above come before the V copies into the same buffers
    __syncthreads();
    cluster_sync();        // every owner's tau, flag and page bits are complete
    const int owners = min(a.S, a.G);
    const int words = (cnt + 31) / 32;
    if (!abort_flag) {
        if (tid < 8) tau_s[tid] = tid < a.G ? ld_dsmem_f32(dsmem(&tau_pub[tid], tid % a.S)) : INFINITY;
        if (tid < 32) {
            const int f = tid < owners ? ld_dsmem_s32(dsmem(&fallback, tid)) : 0;
            const bool any = __any_sync(0xffffffffu, f != 0);
            if (tid == 0) fb_all = any;
        }
        if (bitmap_ok)
            for (int w = tid; w < words; w += kThreads) {
                unsigned v[8];                   // owners <= 8: every read goes out before the first use
#pragma unroll
                for (int q = 0; q < 8; ++q) v[q] = q < owners ? (unsigned)ld_dsmem_s32(dsmem(&bits[w], q)) : 0u;
                unsigned u = 0;
#pragma unroll
                for (int q = 0; q < 8; ++q) u |= v[q];
                vbits[w] = u;
            }
    }
    __syncthreads();
    const bool balanced = !fb_all && bitmap_ok;

    // ------------------------------------------------------------ V pass
    const float rexp = 1.0f / (a.alpha - 1.0f);
    float acc[NT][MTW][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int m = 0; m < MTW; ++m) acc[nt][m][0] = acc[nt][m][1] = acc[nt][m][2] = acc[nt][m][3] = 0.f;
    for (int i = tid; i < 8 * NT * PROW; i += kThreads) ps_tile[i] = 0;
    int gst = nst;        // stages through the barriers so far (phase bookkeeping)
    int loaded = 0;
    const uint32_t pbase = smem_addr(ps_tile);
    // balanced: the weighted pages in list order, CTA s taking ranks s, s + S, ...
    // (windows of kActWin of them); otherwise the weighted pages of its own split
    int nw = 0, share = 0;
    if (balanced) {
        // rank of the first weighted page of every bitmap word (warp 0, 32 words a step)
        if (warp == 0) {
            int base = 0;
            for (int w0 = 0; w0 < words; w0 += 32) {
                const int c = w0 + lane < words ? __popc(vbits[w0 + lane]) : 0;
                int incl = c;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int t = __shfl_up_sync(0xffffffffu, incl, o);
                    if (lane >= o) incl += t;
                }
                if (w0 + lane < words) wbase[w0 + lane] = base + incl - c;
                base += __shfl_sync(0xffffffffu, incl, 31);
            }
            if (lane == 0) wsum[0] = base;
        }
        __syncthreads();
        const int tot = wsum[0];
        share = tot > s ? (tot - s + a.S - 1) / a.S : 0;
        nw = (share + kActWin - 1) / kActWin;
    } else {
        nw = (r.end - r.start + kActWin - 1) / kActWin;
    }
    for (int win = 0; win < nw && !abort_flag; ++win) {
        if (balanced) {
            // this CTA's entries [win * kActWin, ...) of its share: list positions of
            // the weighted pages of rank s + j S
            if (tid == 0) nact = min(kActWin, share - win * kActWin);
            for (int w = tid; w < words; w += kThreads) {
                unsigned m = vbits[w];
                int rk = wbase[w];
                while (m) {
                    const int bit = __ffs(m) - 1;
                    m &= m - 1;
                    if (rk >= s && (rk - s) % a.S == 0) {
                        const int j = (rk - s) / a.S - win * kActWin;
                        if (j >= 0 && j < kActWin) act[j] = w * 32 + bit;
                    }
                    ++rk;
                }
            }
            __syncthreads();
            for (int i = tid; i < nact; i += kThreads) {
                int lp;
                act_phys[i] = resolve_peer(a, b, g, act[i], P, per_split, lp);
                act_lp[i] = lp;
            }
        } else {
            const int w0 = r.start + win * kActWin;
            const int wn = min(kActWin, r.end - w0);
            for (int i = tid; i < wn; i += kThreads) flag[i] = 0;
            __syncthreads();
            for (int it = tid; it < wn * a.G; it += kThreads) {
                const int j = it / a.G, h = it % a.G;
                const float* cp = cm_s[h] + (w0 + j - r.start) * C;
                float m = -INFINITY;
#pragma unroll
                for (int k = 0; k < C; ++k) m = fmaxf(m, cp[k]);
                if (m > tau_s[h]) flag[j] = 1;
            }
            __syncthreads();
            if (warp == 0) {   // ordered compaction of the flags
                int base = 0;
                for (int i0 = 0; i0 < wn; i0 += 32) {
                    const bool f = (i0 + lane < wn) && flag[i0 + lane];
                    const unsigned m = __ballot_sync(0xffffffffu, f);
                    if (f) act[base + __popc(m & ((1u << lane) - 1u))] = w0 + i0 + lane;
                    base += __popc(m);
                }
                if (lane == 0) nact = base;
            }
            __syncthreads();
            for (int i = tid; i < nact; i += kThreads) {
                int lp;
                act_phys[i] = resolve(a, b, g, act[i], P, lp, true);
                act_lp[i] = lp;
            }
        }
        __syncthreads();
        const int na = nact;
        loaded += na;
        const int nsv = (na + PPS - 1) / PPS;
        auto issue = [&](int st, int slot_) {
            uint8_t* dst = smem + slot_ * STAGE;
            uint32_t bytes = 0;
#pragma unroll
            for (int i = 0; i < PPS; ++i) {
                const int ai = st * PPS + i;
                if (ai < na && act_phys[ai] >= 0) bytes += PS * D * 2;
            }
            mbar_arrive_expect_tx(&bars[slot_], bytes);
#pragma unroll
            for (int i = 0; i < PPS; ++i) {
                const int ai = st * PPS + i;
                if (ai >= na || act_phys[ai] < 0) continue;
                const int y = (act_phys[ai] * a.H_kv + g) * PS;
#pragma unroll
                for (int hh = 0; hh < D / 64; ++hh)
                    tma_load_2d(dst + hh * (kStageTok * 128) + i * PS * 128, &vmap, &bars[slot_], hh * 64, y);
            }
        };
        if (tid == 0)
            for (int st = 0; st < min(NSTG, nsv); ++st) issue(st, (gst + st) % NSTG);
        int st = 0;
        for (; st < nsv; ++st) {
            const int gs = gst + st;
            const int slot = gs % NSTG;
            const int t = tid & (kStageTok - 1);
            const int ai = st * PPS + t / PS;
            const bool valid = ai < na && act_phys[ai] >= 0 && act_lp[ai] * PS + (t % PS) < L;
            {   // weights of this stage: token tid % 64, heads (tid / 64) * 2 * NT ...
                const int hbase = (tid >> 6) * 2 * NT;
#pragma unroll
                for (int k = 0; k < 2 * NT; ++k) {
                    const int head = hbase + k;
                    float p = 0.f;
                    if (head < a.G && valid) {
                        const float xv = __ldcg(a.xbuf + (row0h + head) * xstride + (size_t)act[ai] * PS + t % PS);
                        const float u = fmaxf(xv - tau_s[head], 0.f);
                        p = a2 ? u : (a15 ? u * u : powf(u, rexp));
                    }
                    uint32_t hi, lo;
                    split_bf16(p, hi, lo);
                    ps_tile[(2 * head) * PROW + t] = (uint16_t)hi;
                    ps_tile[(2 * head + 1) * PROW + t] = (uint16_t)lo;
                }
            }
            if (!mbar_wait(&bars[slot], (gs / NSTG) & 1, kWaitLimitNs)) {
                abort_flag = 1;
                report(a.status, ENTMAXKV_TIMEOUT);
            }
            __syncthreads();
            if (abort_flag) break;
            // rows without a valid token are zeroed so zero weights never meet garbage
            if ((tid >> 6) < D / 64 && !valid) {
                uint4* rowp = reinterpret_cast<uint4*>(smem + slot * STAGE + (tid >> 6) * (kStageTok * 128) + t * 128);
#pragma unroll
                for (int k = 0; k < 8; ++k) rowp[k] = make_uint4(0, 0, 0, 0);
                fence_proxy_async();
            }
            __syncthreads();
            const uint32_t base = sbase + slot * STAGE;
            const int n = lane >> 2, c = lane & 3;
#pragma unroll
            for (int kk = 0; kk < kStageTok / 16; ++kk) {
                uint32_t b0[NT], b1[NT];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const uint32_t pr = pbase + ((8 * nt + n) * PROW + 16 * kk + 2 * c) * 2;
                    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(b0[nt]) : "r"(pr));
                    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(b1[nt]) : "r"(pr + 16));
                }
                const int mi = lane >> 3;
                const int trow = 16 * kk + (lane & 7) + 8 * (mi >> 1);
#pragma unroll
                for (int m = 0; m < MTW; ++m) {
                    const int d0 = 16 * (warp * MTW + m);
                    uint32_t af[4];
                    ldsm_x4_t(swz_addr(base, trow, d0 / 8 + (mi & 1)), af);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) mma_bf16(acc[nt][m], af, b0[nt], b1[nt]);
                }
            }
            __syncthreads();
            if (tid == 0 && st + NSTG < nsv) issue(st + NSTG, (gs + NSTG) % NSTG);
        }
        if (abort_flag && tid == 0)   // copies still in flight must land before the CTA moves on
            for (int k = st; k < min(st + NSTG, nsv); ++k)
                mbar_wait(&bars[(gst + k) % NSTG], ((gst + k) / NSTG) & 1, kWaitLimitNs);
        gst += nsv;
        __syncthreads();   // act and nact are rebuilt by the next window
    }
    if (tid == 0 && a.vpages) atomicAdd(&a.vpages[(size_t)b * a.H_kv + g], loaded);
    const int E = a.G * D;
    const int per = (E + a.S - 1) / a.S;     // output elements [s per, (s + 1) per) are added by CTA s
    if (balanced) {
        // Every CTA stores its partial of each output element straight into the
        // shared memory of the element's owner, received as rb[split][element -
        // owner's first] in the chunk maxima (unused on this path after the
        // bounds); one cluster barrier, then each owner adds its elements'
        // partials locally in split order.  Nothing reads another CTA's shared
        // memory after that barrier, so no CTA waits for the others to leave.
        static_assert(4 * NT * (kFusedMaxSplitTokens / 16) >= 4 * NT * D + kFusedMaxSplits,
                      "the received partials fit the chunk-maximum array");
        float* rb = &cm_s[0][0];
        const int c = lane & 3, gi = lane >> 2;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int head = 4 * nt + c;
            if (head >= a.G) continue;
#pragma unroll
            for (int m = 0; m < MTW; ++m) {
                const int e0 = head * D + 16 * (warp * MTW + m) + gi, e1 = e0 + 8;
                const int o0 = e0 / per, o1 = e1 / per;
                st_dsmem_f32(dsmem(rb + s * per + (e0 - o0 * per), o0), acc[nt][m][0] + acc[nt][m][1]);
                st_dsmem_f32(dsmem(rb + s * per + (e1 - o1 * per), o1), acc[nt][m][2] + acc[nt][m][3]);
            }
        }
        cluster_sync();   // every split's partials have landed at their owners
        for (int e = s * per + tid; e < min(E, (s + 1) * per); e += kThreads) {
            const int j = e - s * per;
            float sum = 0.f;                     // in CTA order, as the loads below
            for (int q = 0; q < a.S; ++q) sum += rb[q * per + j];
            if (a.S < kFusedMaxSplits) sum += 0.f;   // the absent splits' +0 (turns a -0 sum into +0)
            a.out[(row0h + e / D) * D + e % D] = sum;
        }
        return;
    }
    // partial output of this CTA into shared memory (every copy has landed or
    // been waited out above): part[head 4nt + c][d]
    __syncthreads();
    {
        const int c = lane & 3, gi = lane >> 2;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int head = 4 * nt + c;
            if (head >= a.G) continue;
#pragma unroll
            for (int m = 0; m < MTW; ++m) {
                const int d = 16 * (warp * MTW + m) + gi;
                part[head * D + d] = acc[nt][m][0] + acc[nt][m][1];
                part[head * D + d + 8] = acc[nt][m][2] + acc[nt][m][3];
            }
        }
    }
    __syncthreads();
    cluster_sync();

    // ------------------------------------------------------------ merge
    for (int e = s * per + tid; e < min(E, (s + 1) * per); e += kThreads) {
        const int head = e / D, dd = e % D;
        float v[kFusedMaxSplits];            // every read goes out before the first add
#pragma unroll
        for (int q = 0; q < kFusedMaxSplits; ++q) v[q] = q < a.S ? ld_dsmem_f32(dsmem(part + e, q)) : 0.f;
        float sum = 0.f;                     // in CTA order; the +0 of absent splits changes nothing
#pragma unroll
        for (int q = 0; q < kFusedMaxSplits; ++q) sum += v[q];
        a.out[(row0h + head) * D + dd] = sum;
    }
    cluster_sync();       // no CTA leaves while another may still read its shared memory
}

// ====================================================================== softmax
template <int D, int PS, int NT>
__global__ void __launch_bounds__(kThreads) softmax_bf16_kernel(const __grid_constant__ CUtensorMap kmap,
                                                                const __grid_constant__ CUtensorMap vmap,
                                                                const AttnArgs a)
{
    pdl_enter();
    constexpr int STAGE = kStageTok * D * 2;
    constexpr int PPS = kStageTok / PS;
    constexpr int KS = D / 16;
    constexpr int MTW = D / 64;
    constexpr int PROW = kStageTok + kPsPad;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_align<1024>(smem_raw);
    // stage i: K tile at 2i*STAGE, V tile at (2i+1)*STAGE
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + 2 * kStagesSM * STAGE);
    uint16_t* ps_tile = reinterpret_cast<uint16_t*>(smem + 2 * kStagesSM * STAGE + 64);
    __shared__ float wmax[4][4 * NT];
    __shared__ int abort_flag;

    const int b = blockIdx.z, g = blockIdx.y, s = blockIdx.x;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int gi = lane >> 2, c = lane & 3;
    const int L = a.seq_lens[b];
    const int P = pages_of(L, PS, a.max_pages, a.status);
    const int cnt = list_count(a, b, g, P);
    const Range r = split_range(cnt, a.S, s);
    const int nst = r.end > r.start ? (r.end - r.start + PPS - 1) / PPS : 0;
    tab_fill(a, b, g, r, P);

    float acc[NT][MTW][4];
    float mrun[NT], lrun[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        mrun[nt] = -INFINITY;
        lrun[nt] = 0.f;
#pragma unroll
        for (int m = 0; m < MTW; ++m) acc[nt][m][0] = acc[nt][m][1] = acc[nt][m][2] = acc[nt][m][3] = 0.f;
    }

    if (nst > 0) {
        uint32_t bq[NT][KS][2];
        load_q_frags<D, NT>(a, b, g, a.xscale, bq);
        if (tid == 0) {
            prefetch_tmap(&kmap);
            prefetch_tmap(&vmap);
            for (int i = 0; i < kStagesSM; ++i) mbar_init(&bars[i], 1);
            fence_mbar_init();
            abort_flag = 0;
        }
        for (int i = tid; i < 8 * NT * PROW; i += kThreads) ps_tile[i] = 0;
        __syncthreads();
        auto issue = [&](int st) {
            const int slot = st % kStagesSM;
            // one barrier for both tiles: expect the sum of their bytes
            constexpr int PPS_ = PPS;
            int phys[PPS_];
            uint32_t bytes = 0;
#pragma unroll
            for (int i = 0; i < PPS_; ++i) {
                const int idx = r.start + st * PPS_ + i;
                int lp;
                phys[i] = idx < r.end ? resolve(a, b, g, idx, P, lp, true) : -1;
                if (phys[i] >= 0) bytes += 2 * PS * D * 2;
            }
            mbar_arrive_expect_tx(&bars[slot], bytes);
#pragma unroll
            for (int i = 0; i < PPS_; ++i) {
                if (phys[i] < 0) continue;
                const int y = (phys[i] * a.H_kv + g) * PS;
#pragma unroll
                for (int h = 0; h < D / 64; ++h) {
                    tma_load_2d(smem + (2 * slot) * STAGE + h * (kStageTok * 128) + i * PS * 128, &kmap, &bars[slot], h * 64, y);
                    tma_load_2d(smem + (2 * slot + 1) * STAGE + h * (kStageTok * 128) + i * PS * 128, &vmap, &bars[slot], h * 64, y);
                }
            }
        };
        if (tid == 0)
            for (int st = 0; st < min(kStagesSM, nst); ++st) issue(st);
        const uint32_t sbase = smem_addr(smem);
        const uint32_t pbase = smem_addr(ps_tile);
        for (int st = 0; st < nst; ++st) {
            const int slot = st % kStagesSM;
            if (!mbar_wait(&bars[slot], (st / kStagesSM) & 1, kWaitLimitNs)) {
                abort_flag = 1;
                report(a.status, ENTMAXKV_TIMEOUT);
            }
            __syncthreads();
            if (abort_flag) {
                if (tid == 0)
                    for (int k = st; k < min(st + kStagesSM, nst); ++k)
                        mbar_wait(&bars[k % kStagesSM], (k / kStagesSM) & 1, kWaitLimitNs);
                return;
            }
            const uint32_t kbase = sbase + (2 * slot) * STAGE;
            const uint32_t vbase = sbase + (2 * slot + 1) * STAGE;
            // scores of tokens row0+gi (+8), head 4nt + c
            const int row0 = warp * 16;
            float sc[NT][2];
            {
                float qa[NT][4];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) qa[nt][0] = qa[nt][1] = qa[nt][2] = qa[nt][3] = 0.f;
                const int arow = row0 + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
                for (int j = 0; j < KS; ++j) {
                    uint32_t af[4];
                    ldsm_x4(swz_addr(kbase, arow, 2 * j + (lane >> 4)), af);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) mma_bf16(qa[nt], af, bq[nt][j][0], bq[nt][j][1]);
                }
#pragma unroll
                for (int rr = 0; rr < 2; ++rr) {
                    const int t = row0 + gi + 8 * rr;
                    const int idx = r.start + st * PPS + t / PS;
                    bool valid = false;
                    if (idx < r.end) {
                        int lp;
                        const int phys = resolve(a, b, g, idx, P, lp, false);
                        valid = phys >= 0 && lp * PS + t % PS < L;
                    }
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
                        sc[nt][rr] = (valid && 4 * nt + c < a.G) ? qa[nt][2 * rr] + qa[nt][2 * rr + 1] : -INFINITY;
                }
            }
            // stage maximum per head (lanes with equal c share a head)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                float mloc = fmaxf(sc[nt][0], sc[nt][1]);
                mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, 4));
                mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, 8));
                mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, 16));
                if (gi == 0) wmax[warp][4 * nt + c] = mloc;
            }
            zero_invalid_rows<D, PS>(a, smem + (2 * slot + 1) * STAGE, b, g, r, st, P, L);
            __syncthreads();
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const int hh = 4 * nt + c;
                const float smax = fmaxf(fmaxf(wmax[0][hh], wmax[1][hh]), fmaxf(wmax[2][hh], wmax[3][hh]));
                const float mnew = fmaxf(mrun[nt], smax);
                const float corr = (mnew == -INFINITY) ? 1.f : expf(mrun[nt] - mnew);
                mrun[nt] = mnew;
                lrun[nt] *= corr;
#pragma unroll
                for (int m = 0; m < MTW; ++m) {
                    acc[nt][m][0] *= corr; acc[nt][m][1] *= corr;
                    acc[nt][m][2] *= corr; acc[nt][m][3] *= corr;
                }
#pragma unroll
                for (int rr = 0; rr < 2; ++rr) {
                    const float p = (sc[nt][rr] == -INFINITY) ? 0.f : expf(sc[nt][rr] - mnew);
                    lrun[nt] += p;
                    uint32_t hi, lo;
                    split_bf16(p, hi, lo);
                    const int t = row0 + gi + 8 * rr;
                    ps_tile[(2 * hh) * PROW + t] = (uint16_t)hi;
                    ps_tile[(2 * hh + 1) * PROW + t] = (uint16_t)lo;
                }
            }
            __syncthreads();
#pragma unroll
            for (int kk = 0; kk < kStageTok / 16; ++kk) {
                uint32_t b0[NT], b1[NT];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const uint32_t pr = pbase + ((8 * nt + gi) * PROW + 16 * kk + 2 * c) * 2;
                    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(b0[nt]) : "r"(pr));
                    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(b1[nt]) : "r"(pr + 16));
                }
                const int mi = lane >> 3;
                const int trow = 16 * kk + (lane & 7) + 8 * (mi >> 1);
#pragma unroll
                for (int m = 0; m < MTW; ++m) {
                    const int d0 = 16 * (warp * MTW + m);
                    uint32_t af[4];
                    ldsm_x4_t(swz_addr(vbase, trow, d0 / 8 + (mi & 1)), af);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) mma_bf16(acc[nt][m], af, b0[nt], b1[nt]);
                }
            }
            __syncthreads();
            if (tid == 0 && st + kStagesSM < nst) issue(st + kStagesSM);
        }
    }
    // running sums: lanes with equal c, all warps
    __shared__ float lsum[4][4 * NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        float l = lrun[nt];
        l += __shfl_xor_sync(0xffffffffu, l, 4);
        l += __shfl_xor_sync(0xffffffffu, l, 8);
        l += __shfl_xor_sync(0xffffffffu, l, 16);
        if (gi == 0) lsum[warp][4 * nt + c] = l;
    }
    __syncthreads();
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const int head = 4 * nt + c;
        if (head >= a.G) continue;
        const size_t row = ((size_t)b * a.H_q + (size_t)g * a.G + head) * a.S + s;
#pragma unroll
        for (int m = 0; m < MTW; ++m) {
            const int d = 16 * (warp * MTW + m) + gi;
            a.opart[row * D + d] = acc[nt][m][0] + acc[nt][m][1];
            a.opart[row * D + d + 8] = acc[nt][m][2] + acc[nt][m][3];
        }
        if (warp == 0 && gi == 0) {
            a.mlpart[row * 2] = mrun[nt];
            a.mlpart[row * 2 + 1] = lsum[0][head] + lsum[1][head] + lsum[2][head] + lsum[3][head];
        }
    }
    reduce_splits<D, true>(a, b, g);
}

template <int D>
__global__ void __launch_bounds__(kThreads) softmax_f32_kernel(const float* __restrict__ k_pool,
                                                               const float* __restrict__ v_pool, int ps,
                                                               const AttnArgs a)
{
    pdl_enter();
    __shared__ float sc[64 * 8];
    const int b = blockIdx.z, g = blockIdx.y, s = blockIdx.x, tid = threadIdx.x;
    const int L = a.seq_lens[b];
    const int P = pages_of(L, ps, a.max_pages, a.status);
    const int cnt = list_count(a, b, g, P);
    const Range r = split_range(cnt, a.S, s);
    tab_fill(a, b, g, r, P);
    // thread w < G*D owns (head, d) pairs w, w + kThreads, ...
    constexpr int PER = (8 * D + kThreads - 1) / kThreads;
    float m[PER], l[PER];
    double o[PER];
    for (int k = 0; k < PER; ++k) { m[k] = -INFINITY; l[k] = 0.f; o[k] = 0.0; }
    for (int idx = r.start; idx < r.end; ++idx) {
        int lp;
        const int phys = resolve(a, b, g, idx, P, lp, tid == 0);
        __syncthreads();
        for (int w = tid; w < ps * a.G; w += kThreads) {
            const int t = w % ps, head = w / ps;
            float x = -INFINITY;
            if (phys >= 0 && lp * ps + t < L) {
                const float* kr = k_pool + (((size_t)phys * a.H_kv + g) * ps + t) * D;
                const float* qh = a.q + ((size_t)b * a.H_q + (size_t)g * a.G + head) * D;
                double dot = 0.0;
                for (int j = 0; j < D; ++j) dot = fma((double)qh[j], (double)kr[j], dot);
                x = (float)(dot * (double)a.xscale);
            }
            sc[head * 64 + t] = x;
        }
        __syncthreads();
        for (int k = 0; k < PER; ++k) {
            const int w = tid + k * kThreads;
            if (w >= a.G * D) break;
            const int head = w / D, dd = w % D;
            for (int t = 0; t < ps; ++t) {
                const float x = sc[head * 64 + t];
                if (x == -INFINITY) continue;
                const float mn = fmaxf(m[k], x);
                const float corr = m[k] == -INFINITY ? 0.f : expf(m[k] - mn);
                const float p = expf(x - mn);
                l[k] = l[k] * corr + p;
                o[k] = o[k] * corr + (double)p * (double)v_pool[(((size_t)phys * a.H_kv + g) * ps + t) * D + dd];
                m[k] = mn;
            }
        }
    }
    for (int k = 0; k < PER; ++k) {
        const int w = tid + k * kThreads;
        if (w >= a.G * D) break;
        const int head = w / D, dd = w % D;
        const size_t row = ((size_t)b * a.H_q + (size_t)g * a.G + head) * a.S + s;
        a.opart[row * D + dd] = (float)o[k];
        if (dd == 0) {
            a.mlpart[row * 2] = m[k];
            a.mlpart[row * 2 + 1] = l[k];
        }
    }
    reduce_splits<D, true>(a, b, g);
}

// ====================================================================== self test
__global__ void selftest_timeout_kernel(uint64_t limit_ns, int32_t* status)
{
    pdl_enter();
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 2);   // two arrivals expected, only one ever comes
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_arrive(&bar);
    if (!mbar_wait(&bar, 0, limit_ns)) {
        if (threadIdx.x == 0) report(status, ENTMAXKV_TIMEOUT);
    }
}

// ====================================================================== launch
// Long page lists: K pass, threshold and V pass as three kernels (the
// threshold kernel gives each query head a 512-thread CTA).
template <int D, int PS, int NT>
static int launch_entmax_bf16_split(const AttnArgs& a, int B, const CUtensorMap* kmap, const CUtensorMap* vmap,
                              cudaStream_t stream)
{
    dim3 grid(a.S, a.H_kv, B);
    const int qk_smem = kStagesQK * kStageTok * D * 2 + 1024 + 64;
    const int pv_smem = kStagesPV * kStageTok * D * 2 + 1024 + 64 + 8 * NT * (kStageTok + kPsPad) * 2;
    if (ensure_smem((const void*)qk_bf16_kernel<D, PS, NT>, qk_smem)) return ENTMAXKV_CUDA_ERROR;
    if (ensure_smem((const void*)pv_bf16_kernel<D, PS, NT>, pv_smem)) return ENTMAXKV_CUDA_ERROR;
    launch_pdl(qk_bf16_kernel<D, PS, NT>, dim3(grid), dim3(kThreads), qk_smem, stream, *kmap, a);
    if (cudaGetLastError() != cudaSuccess) return ENTMAXKV_CUDA_ERROR;
    if (ensure_smem((const void*)tau_kernel, kTauSmem)) return ENTMAXKV_CUDA_ERROR;
    launch_pdl(tau_kernel, dim3(dim3(a.H_q, B)), dim3(kTauBlock), kTauSmem, stream, PS, a);
    if (cudaGetLastError() != cudaSuccess) return ENTMAXKV_CUDA_ERROR;
    launch_pdl(pv_bf16_kernel<D, PS, NT>, dim3(grid), dim3(kThreads), pv_smem, stream, *vmap, a);
    return cudaGetLastError() == cudaSuccess ? ENTMAXKV_OK : ENTMAXKV_CUDA_ERROR;
}

// Splits of the fused kernel: the largest power of two up to 16 that the list
// length and two CTAs per SM allow, and that the device can place as one
// cluster with the kernel's resources.
static int fused_splits(const void* kern, int smem, int units, int list)
{
    int S = kFusedMaxSplits;
    while (S > 1 && (S > list || (long long)units * S > 2ll * num_sms())) S >>= 1;
    while (S > 1 && max_active_clusters(kern, S, kThreads, smem) < 1) S >>= 1;
    return S;
}

template <int D, int PS, int NT>
static int launch_entmax_bf16(const AttnArgs& a0, int B, const CUtensorMap* kmap, const CUtensorMap* vmap,
                              cudaStream_t stream)
{
    const void* kern = (const void*)entmax_bf16_kernel<D, PS, NT>;
    const int smem = kFusedStages * kStageTok * D * 2 + 1024 + 64 + 8 * NT * (kStageTok + kPsPad) * 2;
    if (ensure_cluster_kernel(kern, smem)) return ENTMAXKV_CUDA_ERROR;
    AttnArgs a = a0;
    a.S = fused_splits(kern, smem, B * a.H_kv, a.k_max);   // <= the workspace layout's split count
    // long lists (the full cache, the Gaussian selector's worst case): each
    // split's candidates would outgrow their slots, so the three-kernel path
    if ((long long)((a.k_max + a.S - 1) / a.S) * PS > kFusedMaxSplitTokens)
        return launch_entmax_bf16_split<D, PS, NT>(a0, B, kmap, vmap, stream);
    launch_pdl_cluster(entmax_bf16_kernel<D, PS, NT>, dim3(a.S, a.H_kv, B), dim3(kThreads), a.S, smem, stream,
                       *kmap, *vmap, a);
    return cudaGetLastError() == cudaSuccess ? ENTMAXKV_OK : ENTMAXKV_CUDA_ERROR;
}

template <int D>
static int launch_entmax_f32(const entmaxkv_pool& pool, const AttnArgs& a, int B, cudaStream_t stream)
{
    dim3 grid(a.S, a.H_kv, B);
    launch_pdl(qk_f32_kernel<D>, dim3(grid), dim3(kThreads), 0, stream, (const float*)pool.k_pool, pool.ps, a);
    if (cudaGetLastError() != cudaSuccess) return ENTMAXKV_CUDA_ERROR;
    if (ensure_smem((const void*)tau_kernel, kTauSmem)) return ENTMAXKV_CUDA_ERROR;
    launch_pdl(tau_kernel, dim3(dim3(a.H_q, B)), dim3(kTauBlock), kTauSmem, stream, pool.ps, a);
    if (cudaGetLastError() != cudaSuccess) return ENTMAXKV_CUDA_ERROR;
    launch_pdl(pv_f32_kernel<D>, dim3(grid), dim3(kThreads), 0, stream, (const float*)pool.v_pool, pool.ps, a);
    return cudaGetLastError() == cudaSuccess ? ENTMAXKV_OK : ENTMAXKV_CUDA_ERROR;
}

int launch_entmax_attend(const entmaxkv_pool& pool, const AttnArgs& a, int B, const CUtensorMap* kmap,
                         const CUtensorMap* vmap, cudaStream_t stream)
{
    if (pool.dtype == ENTMAXKV_F32) {
        return pool.d == 128 ? launch_entmax_f32<128>(pool, a, B, stream) : launch_entmax_f32<64>(pool, a, B, stream);
    }
    const bool g8 = a.G == 8;
    if (pool.d == 128) {
        if (pool.ps == 64) return g8 ? launch_entmax_bf16<128, 64, 2>(a, B, kmap, vmap, stream)
                                     : launch_entmax_bf16<128, 64, 1>(a, B, kmap, vmap, stream);
        return g8 ? launch_entmax_bf16<128, 16, 2>(a, B, kmap, vmap, stream)
                  : launch_entmax_bf16<128, 16, 1>(a, B, kmap, vmap, stream);
    }
    if (pool.ps == 64) return g8 ? launch_entmax_bf16<64, 64, 2>(a, B, kmap, vmap, stream)
                                 : launch_entmax_bf16<64, 64, 1>(a, B, kmap, vmap, stream);
    return g8 ? launch_entmax_bf16<64, 16, 2>(a, B, kmap, vmap, stream)
              : launch_entmax_bf16<64, 16, 1>(a, B, kmap, vmap, stream);
}

template <int D, int PS, int NT>
static int launch_softmax_bf16(const AttnArgs& a, int B, const CUtensorMap* kmap, const CUtensorMap* vmap,
                               cudaStream_t stream)
{
    dim3 grid(a.S, a.H_kv, B);
    const int smem = 2 * kStagesSM * kStageTok * D * 2 + 1024 + 64 + 8 * NT * (kStageTok + kPsPad) * 2;
    if (ensure_smem((const void*)softmax_bf16_kernel<D, PS, NT>, smem)) return ENTMAXKV_CUDA_ERROR;
    launch_pdl(softmax_bf16_kernel<D, PS, NT>, dim3(grid), dim3(kThreads), smem, stream, *kmap, *vmap, a);
    return cudaGetLastError() == cudaSuccess ? ENTMAXKV_OK : ENTMAXKV_CUDA_ERROR;
}

__global__ void zero_counters_kernel(int32_t* counters, int n)
{
    pdl_enter();
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) counters[i] = 0;
}

int launch_softmax_attend(const entmaxkv_pool& pool, const AttnArgs& a, int B, const CUtensorMap* kmap,
                          const CUtensorMap* vmap, cudaStream_t stream)
{
    const int n = B * a.H_kv;
    launch_pdl(zero_counters_kernel, dim3((n + 255) / 256), dim3(256), 0, stream, a.counters, n);
    if (cudaGetLastError() != cudaSuccess) return ENTMAXKV_CUDA_ERROR;
    if (pool.dtype == ENTMAXKV_F32) {
        dim3 grid(a.S, a.H_kv, B);
        if (pool.d == 128)
            launch_pdl(softmax_f32_kernel<128>, dim3(grid), dim3(kThreads), 0, stream, (const float*)pool.k_pool, (const float*)pool.v_pool, pool.ps, a);
        else
            launch_pdl(softmax_f32_kernel<64>, dim3(grid), dim3(kThreads), 0, stream, (const float*)pool.k_pool, (const float*)pool.v_pool, pool.ps, a);
        return cudaGetLastError() == cudaSuccess ? ENTMAXKV_OK : ENTMAXKV_CUDA_ERROR;
    }
    const bool g8 = a.G == 8;
    if (pool.d == 128) {
        if (pool.ps == 64) return g8 ? launch_softmax_bf16<128, 64, 2>(a, B, kmap, vmap, stream)
                                     : launch_softmax_bf16<128, 64, 1>(a, B, kmap, vmap, stream);
        return g8 ? launch_softmax_bf16<128, 16, 2>(a, B, kmap, vmap, stream)
                  : launch_softmax_bf16<128, 16, 1>(a, B, kmap, vmap, stream);
    }
    if (pool.ps == 64) return g8 ? launch_softmax_bf16<64, 64, 2>(a, B, kmap, vmap, stream)
                                 : launch_softmax_bf16<64, 64, 1>(a, B, kmap, vmap, stream);
    return g8 ? launch_softmax_bf16<64, 16, 2>(a, B, kmap, vmap, stream)
              : launch_softmax_bf16<64, 16, 1>(a, B, kmap, vmap, stream);
}

int launch_selftest_timeout(int64_t limit_ns, int32_t* status, cudaStream_t stream)
{
    launch_pdl(selftest_timeout_kernel, dim3(1), dim3(32), 0, stream, (uint64_t)limit_ns, status);
    return cudaGetLastError() == cudaSuccess ? ENTMAXKV_OK : ENTMAXKV_CUDA_ERROR;
}

}  // namespace ekv
