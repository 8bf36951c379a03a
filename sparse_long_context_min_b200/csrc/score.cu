// Query-aware page scoring from per-page metadata.
//
// EntmaxKV (German technical summary, section 2.A): before any key or value is
// loaded, every page is scored from its metadata -- the bounding box
// (coordinatewise k_min / k_max) bounds q.k for every key of the page; the
// Gaussian statistics (mean, variance) model the page's token scores.
//
// Streaming kernel: eight threads share a metadata row (one page, one kv
// head), thread k owning the k-th of 8 consecutive d-slices with its slice of
// the query group held in registers.  Each thread streams its own slices
// through a private ring of shared-memory stages filled by 16-byte cp.async
// copies kScoreStages - 1 rows ahead (the page-table entry of a row is loaded
// one row earlier still), so the copies in flight are not bounded by
// registers and no block barrier is ever needed.  A thread forms its slice
// sum as a chain of fp32 fused multiply-adds in ascending d, and the 8 slice
// sums are combined by a fixed xor-shuffle tree
// ((S0+S1)+(S2+S3))+((S4+S5)+(S6+S7)).
// That is the canonical order of entmaxkv.h: selection is decided on these
// fp32 values, so nothing else may be fused or reordered (explicit
// round-to-nearest intrinsics throughout).
#include <type_traits>

#include "common.cuh"
#include "kernels.cuh"

namespace ekv {

constexpr int kScoreCTA = 512;
constexpr int kScoreStages = 2;

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
    // shared memory: [stage][vector a|b][16-byte chunk][thread] + n[stage][thread]
    static constexpr int SMEM = kScoreStages * (2 * NV * CTA * 16 + CTA * 4);
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
    // appended tokens scored in the same launch (bf16 bounding boxes): n_new
    // tokens per sequence, written by the CTAs [0, napp) (napp = B, or 0 when
    // n_new = 0) while the nscore CTAs after them score every untouched page
    int n_new, napp, nscore;
    const uint16_t* k_new;  // [B][H_kv][n_new][d]
    const uint16_t* v_new;
    uint16_t* k_pool;       // [num_phys][H_kv][ps][d]
    uint16_t* v_pool;
    uint16_t* kmin_w;       // the metadata the appending CTAs update
    uint16_t* kmax_w;
    float* mean_w;
    float* m2_w;
    int32_t* count_w;
};

// sum over the 8 slice lanes of a row: ((S0+S1)+(S2+S3))+((S4+S5)+(S6+S7))
EKV_DEV float slice_tree(float v)
{
    v = __fadd_rn(v, __shfl_xor_sync(0xffffffffu, v, 1));
    v = __fadd_rn(v, __shfl_xor_sync(0xffffffffu, v, 2));
    v = __fadd_rn(v, __shfl_xor_sync(0xffffffffu, v, 4));
    return v;
}

// A row group of 8 (or 16) threads owns one kv head g for the whole launch
// and walks the (sequence, page) items j = first, first + step, ... of that
// head; thread k of the group owns d-slice k.  Item j is page j % max_pages of
// sequence j / max_pages, so its page-table entry is page_table[j].
template <typename T, int D, int G, bool GAUSS>
__global__ void __launch_bounds__(ScoreShape<T, D, G, GAUSS>::CTA, 1)
score_kernel(const ScoreArgs a, const ZTable zt)
{
    pdl_enter();
    using S = ScoreShape<T, D, G, GAUSS>;
    using E = typename std::conditional<GAUSS, float, T>::type;
    using V = RowVec<E>;
    constexpr int NST = kScoreStages;
    extern __shared__ uint4 score_smem[];
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
    const uint32_t sbase = smem_addr(score_smem);
    // 16-byte chunk c of vector v (0: a, 1: b) of stage `slot`, this thread
    auto chunk = [&](int slot, int v, int c) -> uint32_t {
        return sbase + (uint32_t)((((slot * 2 + v) * S::NV + c) * S::CTA + tid) * 16);
    };
    int* nrow = reinterpret_cast<int*>(score_smem + NST * 2 * S::NV * S::CTA);   // [NST][CTA]

    auto pt_load = [&](int j) -> int { return (valid_rg && j < items) ? __ldg(&a.page_table[j]) : -1; };
    // copy item j's slices into stage `slot` (pt = its page-table entry); one group per call
    auto issue = [&](int slot, int j, int pt) {
        int n = 0;
        if (valid_rg && j < items) {
            const int b = j / a.max_pages, p = j - b * a.max_pages;
            const int L = __ldg(&a.seq_lens[b]);
            const int P = pages_of(L, a.ps, a.max_pages, a.status);
            if (p < P) {
                if (pt < 0 || pt >= a.num_phys) {
                    if (w == 0) report(a.status, ENTMAXKV_DEVICE_BOUNDS);
                } else {
                    n = min(a.ps, L - p * a.ps);
                    const uint8_t* pa = basea + (size_t)pt * pstride;
                    const uint8_t* pb = baseb + (size_t)pt * pstride;
#pragma unroll
                    for (int c = 0; c < S::NV; ++c) {
                        cp_async16(chunk(slot, 0, c), pa + 16 * c);
                        cp_async16(chunk(slot, 1, c), pb + 16 * c);
                    }
                }
            }
        }
        nrow[slot * S::CTA + tid] = n;
        cp_async_commit();
    };

    // prologue: items 0 .. NST-2 in flight, the page-table entry of item NST-1 loading
#pragma unroll
    for (int t = 0; t < NST - 1; ++t) issue(t, first + t * step, pt_load(first + t * step));
    int pt_next = pt_load(first + (NST - 1) * step);

    float qreg[S::HPT][S::SW];
    int qb = -1;
    // the trip count is uniform per warp (the shuffles below need every lane)
    for (int t = 0;; ++t) {
        const int j = first + t * step;
        const bool live = valid_rg && j < items;
        if (!__any_sync(0xffffffffu, live)) break;
        const int slot = t % NST;
        {   // keep NST - 1 items in flight
            const int jn = j + (NST - 1) * step;
            const int pt = pt_next;
            pt_next = pt_load(jn + step);
            issue((t + NST - 1) % NST, jn, pt);
        }
        cp_async_wait<NST - 1>();                          // this item's copies have landed
        const int b = live ? j / a.max_pages : 0;
        const int p = j - b * a.max_pages;
        const int n = live ? nrow[slot * S::CTA + tid] : 0;
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
                V::widen(lds128(chunk(slot, 0, c)), fa);
                V::widen(lds128(chunk(slot, 1, c)), fb);
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
    }
    cp_async_wait<0>();   // nothing may still be writing this CTA's shared memory at exit
}

// ---------------------------------------------------------------- bf16 boxes
// Bounding-box scores of a bf16 cache, the scoring pass of every top-k decode
// step.  Same canonical order as score_kernel; the work is split by role.
//  * One producer warp walks the CTA's contiguous run of pages in chunks of
//    PPS pages: it resolves each page (page-table entries loaded 32 at a time,
//    ahead of use), writes (sequence, page, tokens) of the chunk's pages into
//    the stage header and copies each page's k_min and k_max blocks (all kv
//    heads, contiguous in the pool; one copy per run of consecutive physical
//    pages) with bulk copies (TMA) whose bytes complete the stage's `full`
//    mbarrier.  It refills a stage once all
//    consumer warps have arrived on its `empty` mbarrier.
//  * kWsConsumers consumer warps each own kWsRounds x RPW fixed (page slot,
//    kv head) rows of every stage, all of the same kv heads, so their query
//    registers never change within a sequence.
//    The head-dependent choice of k_max or k_min is a byte permute of the two
//    packed bf16 words (one selector per head and word, built when the query
//    is loaded), and two query heads advance their fma chains in one packed
//    f32x2 fma (each lane an IEEE fma with round-to-nearest, as fmaf).
// Every wait is bounded; a CTA meets one block barrier, after the barriers
// are initialised.
constexpr int kWsStages = 3;
constexpr int kWsConsumers = 8;
constexpr int kWsRounds = 4;    // row sets per stage and consumer warp

template <int D, int G>
struct BoxWsShape {
    static constexpr int SW = D / 8;                  // coordinates per slice
    static constexpr int WPS = SW / 2;                // packed bf16 words per slice
    static constexpr int NV = SW * 2 / 16;            // 16-byte chunks per slice and vector
    static constexpr int HPT = G >= 2 ? 2 : 1;        // query heads per thread
    static constexpr int HS = G / HPT;                // threads sharing a slice
    static constexpr int TPR = 8 * HS;                // threads per row (<= 32)
    static constexpr int RPW = 32 / TPR;              // rows per consumer warp
    static constexpr int SET = kWsConsumers * RPW;    // rows of one round of the consumer warps
    static constexpr int SLOTS = kWsRounds * SET;     // rows per stage (= pages per stage x H_kv)
    static constexpr int CTA = 32 * (kWsConsumers + 1);
    static constexpr int ROWB = D * 2;                // bytes of one metadata vector
    static constexpr int STAGEB = SLOTS * 2 * ROWB;   // k_min and k_max of every row of a stage
    static constexpr int DATA = kWsStages * STAGEB;
    // header per stage: SLOTS int4 {sequence or -1, page, tokens, 0}; then full[], empty[]
    static constexpr int SMEM = DATA + kWsStages * SLOTS * 16 + kWsStages * 16;
};

EKV_DEV uint64_t pack2(float lo, float hi)
{
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
EKV_DEV void unpack2(uint64_t v, float& lo, float& hi)
{
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
// two independent fmas, acc.lane = fma(x.lane, y.lane, acc.lane), round to nearest
EKV_DEV void fma2(uint64_t& acc, uint64_t x, uint64_t y)
{
    asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(acc) : "l"(x), "l"(y));
}

// Producer warp of the role-split scoring kernels: walks chunks k = 0..K-1
// (chunk c0 + k = pages (c0 + k) * PPS ...), lane i < PPS resolving page i of
// the chunk, and fills stage k % NST: header int4 {sequence or -1, page,
// tokens, 0} per page slot, and both metadata vectors of each present page
// (all kv heads, vecb bytes each) by bulk copies completing `full`.
template <int NST>
EKV_DEV void ws_produce(const ScoreArgs& a, uint8_t* data, int stageb, int slots, int4* info, uint64_t* full,
                        uint64_t* empty, int PPS, long long c0, int K, size_t vecb)
{
    const int lane = threadIdx.x & 31;
    const long long items = (long long)a.B * a.max_pages;
    const long long j0 = c0 * PPS;                       // first item of the CTA
    auto pt_load = [&](long long j) -> int {
        return j < items && j < (c0 + K) * PPS ? __ldg(&a.page_table[j]) : -1;
    };
    int cur = pt_load(j0 + lane);                        // entries of items j0 + 32m + lane
    int nxt = pt_load(j0 + 32 + lane);
    int lb = -1, lL = 0, lP = 0, lT = 0;
    const int per_batch = 32 / PPS;                      // chunks per batch of entries
    // lane i < PPS walks items j = (c0 + k) * PPS + i as (sequence bb, page pp)
    long long jl = c0 * PPS + lane;
    int bb = (int)(jl / a.max_pages), pp = (int)(jl - (long long)bb * a.max_pages);
    for (int k = 0; k < K; ++k) {
        const int s = k % NST;
        if (k >= NST && !mbar_wait(&empty[s], ((k / NST) - 1) & 1, kWaitLimitNs)) {
            if (lane == 0) report(a.status, ENTMAXKV_TIMEOUT);
            break;
        }
        const int kb = k % per_batch;
        const int pt = __shfl_sync(0xffffffffu, cur, kb * PPS + (lane < PPS ? lane : 0));
        if (kb == per_batch - 1) {
            cur = nxt;
            nxt = pt_load(j0 + (long long)(k + 1 + per_batch) * PPS + lane);
        }
        int n = 0;
        if (lane < PPS) {
            const bool in = jl < items;
            if (in) {
                if (bb != lb) {
                    lb = bb;
                    const int L0 = __ldg(&a.seq_lens[bb]);
                    lL = L0 + a.n_new;                           // the length after this launch's append
                    lP = pages_of(lL, a.ps, a.max_pages, a.status);
                    lT = a.n_new > 0 ? L0 / a.ps : lP;           // first page the append touches
                }
                if (pp >= lT && pp < lP) {
                    n = -1;                                      // scored by the appending CTA
                } else if (pp < lP) {
                    if (pt < 0 || pt >= a.num_phys) report(a.status, ENTMAXKV_DEVICE_BOUNDS);
                    else n = min(a.ps, lL - pp * a.ps);
                }
            }
            info[s * slots + lane] = make_int4(in ? bb : -1, pp, n, 0);
        }
        jl += PPS;
        pp += PPS;
        while (pp >= a.max_pages) {
            pp -= a.max_pages;
            ++bb;
        }
        // one copy per run of slots whose physical pages are consecutive (the
        // blocks of consecutive pages are contiguous in the pool and in the stage)
        const bool mem = lane < PPS && n > 0;
        const unsigned copies = __ballot_sync(0xffffffffu, mem);
        const int prev = __shfl_up_sync(0xffffffffu, pt, 1);
        const bool start = mem && (lane == 0 || !((copies >> (lane - 1)) & 1u) || pt != prev + 1);
        const unsigned starts = __ballot_sync(0xffffffffu, start);
        __syncwarp();                                    // header writes before the arrive
        if (lane == 0) mbar_arrive_expect_tx(&full[s], (uint32_t)(__popc(copies) * 2 * vecb));
        if (start) {
            const unsigned after = starts & ~((2u << lane) - 1u);            // later run starts
            const int stop = after ? __ffs(after) - 1 : PPS;
            const unsigned rest = ~(copies >> lane);                         // 0 bits: members from lane on
            const int gap = rest ? __ffs(rest) - 1 : 32 - lane;
            const int len = min(stop - lane, gap);
            uint8_t* dst = data + (size_t)s * stageb + (size_t)lane * vecb;
            const size_t off = (size_t)pt * vecb;
            bulk_load(dst, static_cast<const uint8_t*>(a.row_a) + off, (uint32_t)(len * vecb), &full[s]);
            bulk_load(dst + (size_t)PPS * vecb, static_cast<const uint8_t*>(a.row_b) + off, (uint32_t)(len * vecb),
                      &full[s]);
        }
    }
}

// An appending CTA of score_box16_kernel: appends the n_new tokens of
// sequence b exactly as append_small_kernel does (pool rows, then per page
// and coordinate the metadata in token order), and scores every page the
// append touched from the metadata it has just written, in the canonical
// order of entmaxkv.h (8 slices of D/8 coordinates, each a chain of fmaf in
// ascending d from 0, combined as ((S0+S1)+(S2+S3))+((S4+S5)+(S6+S7)), times
// scale, largest over the group's heads, -0 -> +0).  sm: shared scratch.
template <int D, int G>
EKV_DEV void append_and_score(const ScoreArgs& a, int b, uint8_t* sm)
{
    constexpr int SW = D / 8;
    const int Hk = a.H_kv, ps = a.ps, n_new = a.n_new;
    uint16_t* lo_s = reinterpret_cast<uint16_t*>(sm);                 // [H_kv][D] new k_min
    uint16_t* hi_s = lo_s + Hk * D;                                   // [H_kv][D] new k_max
    float* part = reinterpret_cast<float*>(sm + 4 * Hk * D);         // [H_kv][G][8] slice sums
    const int base = a.seq_lens[b];
    if (base < 0) {
        if (threadIdx.x == 0) report(a.status, ENTMAXKV_DEVICE_BOUNDS);
        return;
    }
    for (int lp = base / ps; lp * ps < base + n_new; ++lp) {
        const int t0 = max(base, lp * ps);
        const int t1 = min(base + n_new, (lp + 1) * ps);
        if (lp >= a.max_pages) {
            if (threadIdx.x == 0) report(a.status, ENTMAXKV_DEVICE_BOUNDS);
            break;
        }
        const int phys = a.page_table[(size_t)b * a.max_pages + lp];
        if (phys < 0 || phys >= a.num_phys) {
            if (threadIdx.x == 0) report(a.status, ENTMAXKV_DEVICE_BOUNDS);
            continue;
        }
        for (int w = threadIdx.x; w < Hk * D; w += blockDim.x) {
            const int g = w / D, j = w % D;
            const size_t row = (size_t)phys * Hk + g;
            const size_t meta = row * D + j;
            float mu = 0.f, s2 = 0.f, lof = 0.f, hif = 0.f;
            uint16_t lo = 0, hi = 0;
            if (t0 - lp * ps > 0) {                  // resume a partially filled page
                mu = a.mean_w[meta];
                s2 = a.m2_w[meta];
                lo = a.kmin_w[meta];
                hi = a.kmax_w[meta];
                lof = bf16_bits_to_f32(lo);
                hif = bf16_bits_to_f32(hi);
            }
            const size_t src0 = ((size_t)b * Hk + g) * n_new;
            for (int t = t0; t < t1; ++t) {
                const int slot = t - lp * ps;
                const size_t src = (src0 + (t - base)) * D + j;
                const uint16_t kx = a.k_new[src];
                const size_t dst = (row * ps + slot) * D + j;
                a.k_pool[dst] = kx;
                a.v_pool[dst] = a.v_new[src];
                const float x = bf16_bits_to_f32(kx);
                if (slot == 0) {
                    mu = x;
                    s2 = 0.f;
                    lo = hi = kx;
                    lof = hif = x;
                } else {
                    const float n = (float)(slot + 1);
                    const float d1 = __fsub_rn(x, mu);
                    mu = __fadd_rn(mu, __fdiv_rn(d1, n));
                    const float d2 = __fsub_rn(x, mu);
                    s2 = __fmaf_rn(d1, d2, s2);
                    if (x < lof) { lo = kx; lof = x; }
                    if (x > hif) { hi = kx; hif = x; }
                }
            }
            a.mean_w[meta] = mu;
            a.m2_w[meta] = s2;
            a.kmin_w[meta] = lo;
            a.kmax_w[meta] = hi;
            lo_s[w] = lo;
            hi_s[w] = hi;
        }
        if (threadIdx.x == 0) a.count_w[phys] = t1 - lp * ps;
        __syncthreads();
        // slice sums of every (kv head, query head, slice)
        for (int it = threadIdx.x; it < Hk * G * 8; it += blockDim.x) {
            const int g = it / (G * 8), h = (it / 8) % G, k = it % 8;
            const float* qh = a.q + ((size_t)b * a.H_q + (size_t)g * G + h) * D + k * SW;
            const uint16_t* lo_r = lo_s + g * D + k * SW;
            const uint16_t* hi_r = hi_s + g * D + k * SW;
            float acc = 0.f;
#pragma unroll
            for (int e = 0; e < SW; ++e) {
                const float qv = __ldg(qh + e);
                acc = __fmaf_rn(qv, bf16_bits_to_f32(qv >= 0.f ? hi_r[e] : lo_r[e]), acc);
            }
            part[it] = acc;
        }
        __syncthreads();
        for (int g = threadIdx.x; g < Hk; g += blockDim.x) {
            float best = -INFINITY;
#pragma unroll
            for (int h = 0; h < G; ++h) {
                const float* S = part + (g * G + h) * 8;
                const float t = __fadd_rn(__fadd_rn(__fadd_rn(S[0], S[1]), __fadd_rn(S[2], S[3])),
                                          __fadd_rn(__fadd_rn(S[4], S[5]), __fadd_rn(S[6], S[7])));
                const float u = __fmul_rn(t, a.scale);
                if (h == 0 || u > best) best = u;
            }
            if (best == 0.f) best = 0.f;   // -0 -> +0
            a.ub[((size_t)b * Hk + g) * a.max_pages + lp] = best;
        }
        __syncthreads();
    }
}

template <int D, int G>
__global__ void __launch_bounds__(BoxWsShape<D, G>::CTA, 2) score_box16_kernel(const ScoreArgs a)
{
    pdl_enter();
    using S = BoxWsShape<D, G>;
    constexpr int NST = kWsStages;
    extern __shared__ __align__(128) uint8_t box_smem[];
    // appending CTAs first, so that they start with the scoring CTAs rather
    // than in the slots the scoring CTAs leave at the end
    if ((int)blockIdx.x < a.napp) {                      // an appending CTA: no barriers below
        append_and_score<D, G>(a, blockIdx.x, box_smem);
        return;
    }
    const int cta = (int)blockIdx.x - a.napp;
    int4* info = reinterpret_cast<int4*>(box_smem + S::DATA);                     // [NST][SLOTS]
    uint64_t* full = reinterpret_cast<uint64_t*>(box_smem + S::DATA + NST * S::SLOTS * 16);
    uint64_t* empty = full + NST;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int PPS = S::SLOTS / a.H_kv;                   // pages per stage (host checks H_kv | SLOTS)
    const long long items = (long long)a.B * a.max_pages;
    const long long nchunks = (items + PPS - 1) / PPS;
    const long long per = (nchunks + a.nscore - 1) / a.nscore;
    const long long c0 = cta * per;
    const int K = (int)max(0ll, min(nchunks, c0 + per) - c0);   // chunks of this CTA
    const size_t vecb = (size_t)a.H_kv * S::ROWB;        // one page's block of one vector
    if (tid == 0) {
        for (int i = 0; i < NST; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], kWsConsumers);
        }
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == kWsConsumers) {
        ws_produce<NST>(a, box_smem, S::STAGEB, S::SLOTS, info, full, empty, PPS, c0, K, vecb);
        return;   // the consumers keep the CTA alive until every copy has been consumed
    }

    // ---------------------------------------------------- consumers
    const int w = lane % S::TPR, ks = w & 7, hs = w >> 3;
    const int rw = lane / S::TPR;
    const int slot = warp * S::RPW + rw;                 // row of round 0; round r adds r * SET
    const int g = slot % a.H_kv, pi = slot / a.H_kv;     // kv head and page of this row (round 0)
    const int ppr = S::SET / a.H_kv;                     // pages per round (host checks H_kv | SET)
    // stage layout: the k_min blocks of the stage's PPS pages, then their k_max blocks
    const uint32_t rowoff = (uint32_t)(pi * vecb + g * S::ROWB + ks * S::SW * 2);
    const uint32_t maxoff = (uint32_t)(PPS * vecb);
    const uint32_t sbase = smem_addr(box_smem);
    uint64_t qp[S::SW];                                  // (head 0, head 1) query pairs per coordinate
    float qs[S::SW];                                     // single head (HPT == 1)
    uint32_t sel[S::HPT][S::WPS];                        // byte-permute selectors
    int qb = -1;
    const float scale = a.scale;
    auto load_q = [&](int b) {
        const float* qg = a.q + ((size_t)b * a.H_q + (size_t)g * G + hs * S::HPT) * D + ks * S::SW;
        float qv[S::HPT][S::SW];
#pragma unroll
        for (int i = 0; i < S::HPT; ++i)
#pragma unroll
            for (int e = 0; e < S::SW; e += 4) {
                const float4 f = __ldg(reinterpret_cast<const float4*>(qg + (size_t)i * D + e));
                qv[i][e] = f.x; qv[i][e + 1] = f.y; qv[i][e + 2] = f.z; qv[i][e + 3] = f.w;
            }
#pragma unroll
        for (int i = 0; i < S::HPT; ++i)
#pragma unroll
            for (int kk = 0; kk < S::WPS; ++kk)   // k_max (second operand) where q >= 0, else k_min
                sel[i][kk] = (qv[i][2 * kk] >= 0.f ? 0x0054u : 0x0010u) | (qv[i][2 * kk + 1] >= 0.f ? 0x7600u : 0x3200u);
#pragma unroll
        for (int e = 0; e < S::SW; ++e) {
            if (S::HPT == 2) qp[e] = pack2(qv[0][e], qv[S::HPT - 1][e]);
            else qs[e] = qv[0][e];
        }
        qb = b;
    };
    // the query of the CTA's first sequence before the first chunk arrives: a
    // load issued after the chunk copies would queue behind them
    if (K > 0 && c0 * PPS < items) load_q((int)(c0 * PPS / a.max_pages));
    for (int k = 0; k < K; ++k) {
        const int s = k % NST;
        const bool ok = mbar_wait(&full[s], (k / NST) & 1, kWaitLimitNs);
        if (!__all_sync(0xffffffffu, ok)) {
            if (lane == 0) report(a.status, ENTMAXKV_TIMEOUT);
            break;
        }
#pragma unroll
        for (int r = 0; r < kWsRounds; ++r) {
            const int4 inf = info[s * S::SLOTS + pi + r * ppr];
            const int b = inf.x, p = inf.y, n = inf.z;
            if (b >= 0 && b != qb) load_q(b);
            float acc[S::HPT];
#pragma unroll
            for (int i = 0; i < S::HPT; ++i) acc[i] = 0.f;
            if (n > 0) {
                const uint32_t src = sbase + (uint32_t)(s * S::STAGEB) + rowoff + (uint32_t)(r * ppr * vecb);
                uint64_t acc2 = pack2(0.f, 0.f);
#pragma unroll
                for (int c = 0; c < S::NV; ++c) {
                    const uint4 va = lds128(src + 16 * c);
                    const uint4 vb = lds128(src + maxoff + 16 * c);
                    const uint32_t wa[4] = {va.x, va.y, va.z, va.w};
                    const uint32_t wb[4] = {vb.x, vb.y, vb.z, vb.w};
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const int wd = 4 * c + kk, e = 2 * wd;
                        if (S::HPT == 2) {
                            const uint32_t d0 = __byte_perm(wa[kk], wb[kk], sel[0][wd]);
                            const uint32_t d1 = __byte_perm(wa[kk], wb[kk], sel[S::HPT - 1][wd]);
                            fma2(acc2, qp[e], pack2(__uint_as_float(d0 << 16), __uint_as_float(d1 << 16)));
                            fma2(acc2, qp[e + 1],
                                 pack2(__uint_as_float(d0 & 0xFFFF0000u), __uint_as_float(d1 & 0xFFFF0000u)));
                        } else {
                            const uint32_t d0 = __byte_perm(wa[kk], wb[kk], sel[0][wd]);
                            acc[0] = __fmaf_rn(qs[e], __uint_as_float(d0 << 16), acc[0]);
                            acc[0] = __fmaf_rn(qs[e + 1], __uint_as_float(d0 & 0xFFFF0000u), acc[0]);
                        }
                    }
                }
                if (S::HPT == 2) unpack2(acc2, acc[0], acc[S::HPT - 1]);
            }
            float best = -INFINITY;
#pragma unroll
            for (int i = 0; i < S::HPT; ++i) {
                const float u = __fmul_rn(slice_tree(acc[i]), scale);
                if (i == 0 || u > best) best = u;
            }
            if (S::HS > 1) best = fmaxf(best, __shfl_xor_sync(0xffffffffu, best, 8));
            if (S::HS > 2) best = fmaxf(best, __shfl_xor_sync(0xffffffffu, best, 16));
            if (best == 0.f) best = 0.f;   // -0 -> +0
            if (b >= 0 && n >= 0 && w == 0) a.ub[((size_t)b * a.H_kv + g) * a.max_pages + p] = n > 0 ? best : -INFINITY;
        }
        __syncwarp();                                    // every lane is done with stage s
        if (lane == 0) mbar_arrive(&empty[s]);
    }
}

template <int D, int G>
static int launch_box16(const ScoreArgs& a, cudaStream_t stream)
{
    using S = BoxWsShape<D, G>;
    static int occ[64] = {0};                              // resident CTAs per SM, per device
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) dev = 0;
    if (ensure_smem((const void*)score_box16_kernel<D, G>, S::SMEM)) return ENTMAXKV_CUDA_ERROR;
    if (occ[dev] == 0) {
        int n = 1;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, score_box16_kernel<D, G>, S::CTA, S::SMEM) !=
                cudaSuccess || n < 1)
            n = 1;
        occ[dev] = n;
    }
    const int pps = S::SLOTS / a.H_kv;
    const long long chunks = ((long long)a.B * a.max_pages + pps - 1) / pps;
    const int appenders = a.n_new > 0 ? a.B : 0;
    // every CTA resident at once where the appending CTAs leave room
    const long long slots = std::max<long long>(1, (long long)occ[dev] * num_sms() - appenders);
    const int grid = (int)std::max<long long>(1, std::min<long long>(chunks, slots));
    ScoreArgs b = a;
    b.napp = appenders;
    b.nscore = grid;
    launch_pdl(score_box16_kernel<D, G>, dim3(grid + appenders), dim3(S::CTA), S::SMEM, stream, b);
    return cudaGetLastError() == cudaSuccess ? ENTMAXKV_OK : ENTMAXKV_CUDA_ERROR;
}

template <int D>
static int dispatch_box16(int G, const ScoreArgs& a, cudaStream_t st)
{
    switch (G) {
        case 1: return launch_box16<D, 1>(a, st);
        case 2: return launch_box16<D, 2>(a, st);
        case 4: return launch_box16<D, 4>(a, st);
        default: return launch_box16<D, 8>(a, st);
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
    if (ensure_smem((const void*)score_kernel<T, D, G, GAUSS>, S::SMEM)) return ENTMAXKV_CUDA_ERROR;
    if (occ[dev] == 0) {
        int n = 1;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, score_kernel<T, D, G, GAUSS>, S::CTA, S::SMEM) !=
                cudaSuccess || n < 1)
            n = 1;
        occ[dev] = n;
    }
    const long long rows = (long long)a.B * a.max_pages * a.H_kv;
    const long long want = (rows + S::RG - 1) / S::RG;
    const int grid = (int)std::max<long long>(1, std::min<long long>(want, (long long)occ[dev] * num_sms()));
    if ((long long)grid * S::RG < a.H_kv) return ENTMAXKV_UNSUPPORTED;   // at least one group per kv head
    launch_pdl(score_kernel<T, D, G, GAUSS>, dim3(grid), dim3(S::CTA), S::SMEM, stream, a, zt);
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

// The bf16 bounding-box scoring kernel with the role split covers this head
// layout: H_kv divides the rows of a round, and the pages per stage divide
// 32 (one producer lane per page; page-table entries come in batches of 32).
static bool box16_layout(int G, int H_kv)
{
    const int set = kWsConsumers * (32 / (8 * (G >= 2 ? G / 2 : 1)));
    const int pps = set % H_kv == 0 ? kWsRounds * set / H_kv : 0;
    return pps > 0 && pps <= 32 && 32 % pps == 0;
}

int launch_append_score(const entmaxkv_pool& pool, const void* k_new, const void* v_new, int n_new, const float* q,
                        int H_q, const int32_t* page_table, int max_pages, int32_t* seq_lens, int B, float scale,
                        float* ub, int32_t* status, cudaStream_t stream)
{
    const int G = H_q / pool.H_kv;
    if (pool.dtype != ENTMAXKV_BF16 || n_new > pool.ps || !box16_layout(G, pool.H_kv)) {
        // the two calls in turn
        int rc = launch_append(pool, k_new, v_new, n_new, page_table, max_pages, seq_lens, B, status, stream);
        if (rc) return rc;
        return launch_score(pool, q, H_q, page_table, max_pages, seq_lens, B, ENTMAXKV_SCORE_BBOX, scale, ub,
                            nullptr, nullptr, nullptr, status, stream);
    }
    ScoreArgs a{};
    a.row_a = pool.kmin;
    a.row_b = pool.kmax;
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
    a.status = status;
    a.n_new = n_new;
    a.k_new = static_cast<const uint16_t*>(k_new);
    a.v_new = static_cast<const uint16_t*>(v_new);
    a.k_pool = static_cast<uint16_t*>(pool.k_pool);
    a.v_pool = static_cast<uint16_t*>(pool.v_pool);
    a.kmin_w = static_cast<uint16_t*>(pool.kmin);
    a.kmax_w = static_cast<uint16_t*>(pool.kmax);
    a.mean_w = pool.mean;
    a.m2_w = pool.m2;
    a.count_w = pool.count;
    const int rc = pool.d == 128 ? dispatch_box16<128>(G, a, stream) : dispatch_box16<64>(G, a, stream);
    if (rc) return rc;
    // the lengths advance once every CTA of the scoring launch has read them
    return launch_advance(seq_lens, B, n_new, stream);
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
        if (pool.dtype == ENTMAXKV_BF16) {
            if (box16_layout(G, pool.H_kv))
                return pool.d == 128 ? dispatch_box16<128>(G, a, stream) : dispatch_box16<64>(G, a, stream);
            return pool.d == 128 ? dispatch_g<uint16_t, 128, false>(G, a, zt, stream)
                                 : dispatch_g<uint16_t, 64, false>(G, a, zt, stream);
        }
        return pool.d == 128 ? dispatch_g<float, 128, false>(G, a, zt, stream)
                             : dispatch_g<float, 64, false>(G, a, zt, stream);
    }
    a.row_a = pool.mean;
    a.row_b = pool.m2;
    return pool.d == 128 ? dispatch_g<float, 128, true>(G, a, zt, stream)
                         : dispatch_g<float, 64, true>(G, a, zt, stream);
}

}  // namespace ekv
