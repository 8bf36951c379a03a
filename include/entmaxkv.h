/*
 * entmaxkv.h -- C ABI of the EntmaxKV paged-decode library (sm_100a).
 *
 * One decode step of alpha-entmax attention over a paged KV cache, as in
 * "EntmaxKV: Support-Aware Decoding for Entmax Attention" (German technical
 * summary, section 2: query-aware page scoring, candidate selection, sparse
 * entmax attention; abstract: "combines query-aware page scoring,
 * support-aware candidate selection, and sparse entmax attention").
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Every pointer argument is CUDA device memory owned by the caller, unless
 *   the comment says "host".  The attention outputs (out, tau_out) may also be
 *   pinned host memory mapped into the device's address space: the kernels
 *   then store results straight to the host.  The library never allocates or
 *   frees memory and keeps no state between calls (the built-in scratch of
 *   entmaxkv_sparse_attend_static and per-device caches of the SM count and
 *   kernel attributes aside).
 * - Every call is asynchronous on `stream` (a cudaStream_t passed as void*;
 *   NULL is the legacy default stream).  Inputs must stay valid and outputs
 *   untouched until the stream reaches the work.
 * - Return value: an entmaxkv_status detected on the host before or at launch
 *   (argument validation, launch failure).  On a non-zero return nothing was
 *   launched by that call, except for ENTMAXKV_CUDA_ERROR where a launch may
 *   have failed part way.
 * - `status` (device, one int32): errors found by the kernels themselves
 *   (ENTMAXKV_TIMEOUT, ENTMAXKV_DEVICE_BOUNDS) are written there with an
 *   atomic compare-and-swap from 0, so the first error sticks.  The library
 *   never clears it: the caller zeroes it, runs its step, and reads it after
 *   synchronising.  A kernel that reports an error skips the offending access
 *   and leaves its outputs unspecified.
 * - Layouts are row-major, innermost index last.  Symbols: B batch, H_q query
 *   heads, H_kv kv heads, G = H_q / H_kv (query head h belongs to kv head
 *   h / G), d head dim, ps page size, P_b = ceil(seq_lens[b] / ps) pages of
 *   sequence b, max_pages the row length of page_table.
 * - Supported: d in {64, 128}; ps in {16, 64}; dtype F32 or BF16; G in
 *   {1, 2, 4, 8}.  alpha (German summary, section 2: alpha-entmax for any
 *   alpha > 1): the attention entry points take any alpha in (1, 16]; alpha
 *   = 1.5 and 2 have closed-form thresholds, any other alpha a threshold by
 *   safeguarded Newton steps in float64 and weights by powf.  The Gaussian
 *   selector takes alpha = 1.5 or 2 (closed-form expectations) and any alpha
 *   in [1.05, 16] (expectations by a 32-node Gauss-Legendre rule placed on
 *   the integrand's peak); other alpha return ENTMAXKV_UNSUPPORTED.
 * - page_table[b][p] (int32, [B][max_pages]) is the physical page holding
 *   logical page p of sequence b; entries p >= P_b are never read.  Physical
 *   ids out of [0, num_phys_pages) are reported as ENTMAXKV_DEVICE_BOUNDS.
 */
#ifndef ENTMAXKV_H
#define ENTMAXKV_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define ENTMAXKV_API __attribute__((visibility("default")))
#else
#define ENTMAXKV_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    ENTMAXKV_OK = 0,
    ENTMAXKV_INVALID_ARG = 1,    /* host validation failed */
    ENTMAXKV_UNSUPPORTED = 2,    /* d, ps, dtype, G or alpha outside the supported set */
    ENTMAXKV_CUDA_ERROR = 3,     /* a CUDA runtime call or launch failed */
    ENTMAXKV_TIMEOUT = 4,        /* a bounded device wait ran out (device status) */
    ENTMAXKV_DEVICE_BOUNDS = 5,  /* a page id or index failed its device check */
    ENTMAXKV_WORKSPACE = 6,      /* workspace pointer NULL or ws_bytes too small */
    ENTMAXKV_STATIC_LIMIT = 7    /* needs more scratch than the built-in buffer holds */
} entmaxkv_status;

typedef enum { ENTMAXKV_F32 = 0, ENTMAXKV_BF16 = 1 } entmaxkv_dtype;
typedef enum { ENTMAXKV_SCORE_BBOX = 0, ENTMAXKV_SCORE_GAUSS = 1 } entmaxkv_score_mode;
typedef enum { ENTMAXKV_SELECT_TOPK = 0, ENTMAXKV_SELECT_GAUSS = 1 } entmaxkv_select_mode;
typedef enum {
    ENTMAXKV_OP_SELECT = 0,
    ENTMAXKV_OP_SPARSE_ATTEND = 1,
    ENTMAXKV_OP_FULL_ENTMAX = 2,
    ENTMAXKV_OP_FULL_SOFTMAX = 3,
    ENTMAXKV_OP_SPARSE_SOFTMAX = 4
} entmaxkv_op;

/*
 * The shared paged pool and its per-page metadata (host struct holding device
 * pointers).  German summary, section 2.A: the cache is split into pages, each
 * with lightweight metadata -- the coordinatewise minimum and maximum key and
 * the first and second moments of its keys.
 *   k_pool, v_pool : [num_phys_pages][H_kv][ps][d]  dtype
 *   kmin, kmax     : [num_phys_pages][H_kv][d]      dtype (exact extremes)
 *   mean, m2       : [num_phys_pages][H_kv][d]      fp32 (Welford mean and sum
 *                                                    of squared deviations)
 *   count          : [num_phys_pages]               int32 tokens filled
 * All pointers must be 16-byte aligned.
 */
typedef struct {
    void* k_pool;
    void* v_pool;
    void* kmin;
    void* kmax;
    float* mean;
    float* m2;
    int32_t* count;
    int32_t num_phys_pages;
    int32_t H_kv;
    int32_t ps;
    int32_t d;
    int32_t dtype;   /* entmaxkv_dtype */
} entmaxkv_pool;

/*
 * Append n_new tokens per sequence to the cache and update the metadata of
 * every page they touch (German summary, section 2.A: metadata stored per
 * page; the append keeps it current).
 *   pool       : host pointer to the pool description.
 *   k_new,v_new: [B][H_kv][n_new][d] dtype; token j of sequence b goes to
 *                position seq_lens[b] + j.
 *   seq_lens   : [B] int32, read as the lengths before the append and advanced
 *                by n_new on the device after the write (stream ordered).
 *   page_table : the caller writes the physical id of every page the append
 *                reaches before calling; a page's metadata is reset when its
 *                first token is written.
 * Metadata update per page and coordinate, in token order, fp32:
 *   first token: mean = x, m2 = 0, kmin = kmax = x;
 *   token with n tokens filled after it: d1 = x - mean; mean += d1 / n;
 *   m2 = fma(d1, x - mean, m2); kmin = x < kmin ? x : kmin (same for kmax).
 *   count[phys] = tokens filled.  n_new = 0 is a no-op.
 */
ENTMAXKV_API int entmaxkv_append_metadata(const entmaxkv_pool* pool, const void* k_new, const void* v_new,
                             int32_t n_new, const int32_t* page_table, int32_t max_pages,
                             int32_t* seq_lens, int32_t B, int32_t* status, void* stream);

/*
 * Score every page of every sequence from its metadata (German summary,
 * section 2.A).
 *   q     : [B][H_q][d] fp32 query.
 *   scale : score scale (1/sqrt(d) for standard attention); s = scale * q.k.
 *   Every sum over d below is taken in one fixed fp32 order, because
 *   selection is decided on these values: d is cut into 8 consecutive slices
 *   of d/8 coordinates, each slice is a chain of fused multiply-adds from 0 in
 *   ascending d, and the slice sums are combined as
 *   ((S0 + S1) + (S2 + S3)) + ((S4 + S5) + (S6 + S7)).
 *   mode ENTMAXKV_SCORE_BBOX: ub [B][H_kv][max_pages] fp32, the bounding-box
 *     bound of the group, UBg = max over the group's heads of
 *     scale * sum_d q_d (q_d >= 0 ? kmax_d : kmin_d); -0 becomes +0.
 *     m, v, est_max are ignored (may be NULL).
 *   mode ENTMAXKV_SCORE_GAUSS: m, v, est_max [B][H_q][max_pages] fp32, the
 *     Gaussian page model of each query head: m = scale * sum_d q_d mean_d,
 *     v = ((sum_d (q_d*q_d) m2_d) / n) * scale^2, est_max = fma(sqrt(v), z_n, m)
 *     with z_n = fp32(sqrt(2 ln n)) for n >= 2 and z_1 = 0, n the page's
 *     tokens.  ub is ignored.
 *   Entries p >= P_b are written as -INFINITY (v as 0).
 */
ENTMAXKV_API int entmaxkv_score_pages(const entmaxkv_pool* pool, const float* q, int32_t H_q,
                         const int32_t* page_table, int32_t max_pages, const int32_t* seq_lens,
                         int32_t B, int32_t mode, float scale, float* ub, float* m, float* v,
                         float* est_max, int32_t* status, void* stream);

/*
 * entmaxkv_append_metadata followed by entmaxkv_score_pages(ENTMAXKV_SCORE_BBOX)
 * over the new lengths, as one call (German summary, section 2.A: the
 * metadata is kept current as tokens are appended, and every page is scored
 * from it).  The results -- pool rows, metadata, count, the advanced seq_lens
 * and ub -- equal those of the two calls made in turn, bit for bit.  With a
 * bf16 cache, n_new <= ps and a head layout the role-split scoring kernel
 * covers, the append runs inside the scoring launch: extra CTAs write the new
 * tokens, update the touched pages' metadata and score those pages (same
 * operation order) while the other CTAs score every untouched page; a small
 * trailing kernel then advances seq_lens.  Otherwise the two calls run in
 * turn.  Arguments as in those two calls; n_new = 0 only scores.
 */
ENTMAXKV_API int entmaxkv_append_score_pages(const entmaxkv_pool* pool, const void* k_new, const void* v_new,
                                int32_t n_new, const float* q, int32_t H_q, const int32_t* page_table,
                                int32_t max_pages, int32_t* seq_lens, int32_t B, float scale, float* ub,
                                int32_t* status, void* stream);

/*
 * Select candidate pages per (sequence, kv head) (German summary, section 2.B).
 *   Output sel [B][H_kv][k_max] int32 logical page ids sorted ascending, the
 *   first sel_count[b][g] entries valid; sel_count [B][H_kv] int32.
 *   mode ENTMAXKV_SELECT_TOPK (policy 1): keep k = min(budget, P_b) pages, or
 *     k = min(ceil(budget_frac * P_b), P_b) when budget < 0, with the largest
 *     ub; ties go to the lower page index.  Needs k_max >= budget (budget >= 0)
 *     or k_max >= ceil(budget_frac * max_pages).  m, v, est_max, tau_hat,
 *     alpha and delta are ignored.
 *   mode ENTMAXKV_SELECT_GAUSS (policy 2): per query head solve
 *     sum_p n_p E[((alpha-1) s - tau)_+^(1/(alpha-1))] = 1 for tau_hat, s ~
 *     N(m_p, v_p), by Newton steps on log F kept inside a bracket (bisection
 *     where a step leaves it; page terms in fp32, sums in float64; it stops
 *     when |F - 1| < 1e-7, the bracket or the step falls below the terms'
 *     accuracy, or after 60 steps); keep page p for kv head g when
 *     (alpha-1) * est_max[h][p] >= tau_hat[h] - delta for some h in g.
 *     tau_hat [B][H_q] fp32 is written.  Needs k_max >= max_pages.  ub,
 *     budget and budget_frac are ignored.
 *   seq_lens and ps give P_b and the token count n_p of each page.
 *   workspace: entmaxkv_workspace_size(ENTMAXKV_OP_SELECT, ...) bytes (may be
 *   0, then workspace may be NULL).
 */
ENTMAXKV_API int entmaxkv_select(int32_t mode, const float* ub, const float* m, const float* v,
                    const float* est_max, const int32_t* seq_lens, int32_t ps, int32_t B,
                    int32_t H_q, int32_t H_kv, int32_t max_pages, int32_t budget,
                    float budget_frac, float alpha, float delta, int32_t k_max, int32_t* sel,
                    int32_t* sel_count, float* tau_hat, void* workspace, size_t ws_bytes,
                    int32_t* status, void* stream);

/*
 * Exact alpha-entmax attention over the selected pages only (German summary,
 * section 2.C: only the selected entries are loaded; the weights are computed
 * over that reduced set, exactly when it holds the support).
 *   For every query head h of kv head g: x_i = (alpha-1) * scale * q_h . k_i
 *   over the valid tokens of pages sel[b][g][0 .. sel_count[b][g]), tau solved
 *   so that sum_i [x_i - tau]_+^(1/(alpha-1)) = 1, out[b][h] = sum_i p_i v_i.
 *   sel [B][H_kv][k_max] int32 holds distinct logical page ids in [0, pages
 *   of sequence b), in any order (entmaxkv_select emits them ascending); a
 *   page listed twice counts twice.  sel_count [B][H_kv] int32 in
 *   [0, k_max].  An entry or count out of range is skipped (count clamped)
 *   and reported as ENTMAXKV_DEVICE_BOUNDS.
 *   out [B][H_q][d] fp32; tau_out [B][H_q] fp32 (may be NULL).  A head with
 *   no valid token gets out = 0 and tau = +INFINITY.
 *   Value rows are loaded only for pages holding a token with p > 0 for some
 *   head of the group (the weights are exactly zero elsewhere, German summary
 *   section 3: tokens outside the support carry no mass).  v_pages
 *   [B][H_kv] int32 (may be NULL): the number of value pages loaded is ADDED
 *   to it (the caller zeroes it).
 *   workspace: entmaxkv_workspace_size(ENTMAXKV_OP_SPARSE_ATTEND, ...) bytes.
 */
ENTMAXKV_API int entmaxkv_sparse_attend(const entmaxkv_pool* pool, const float* q, int32_t H_q,
                           const int32_t* page_table, int32_t max_pages, const int32_t* seq_lens,
                           int32_t B, const int32_t* sel, const int32_t* sel_count, int32_t k_max,
                           float alpha, float scale, float* out, float* tau_out, int32_t* v_pages,
                           void* workspace, size_t ws_bytes, int32_t* status, void* stream);

/*
 * entmaxkv_sparse_attend for callers that cannot allocate device memory.  The
 * paper has no counterpart: this is a deployment convenience.  Some callers
 * may not call cudaMalloc when they decode -- code under CUDA stream capture
 * (allocation is not allowed while capturing), hosts whose own allocator owns
 * all device memory, latency-critical loops where an allocation or free would
 * synchronise the device.  This call takes its scratch memory from a buffer
 * built into the library (ENTMAXKV_STATIC_SCRATCH_BYTES, 16 MiB, held on every
 * GPU that loads the library until the process exits) instead of a workspace.
 *   Arguments, layouts and results are those of entmaxkv_sparse_attend, and
 *   its argument checks run first (a bad call returns the same code from
 *   both entry points, whatever its size).  Then it returns
 *   ENTMAXKV_STATIC_LIMIT, launching nothing, when
 *   entmaxkv_workspace_size(ENTMAXKV_OP_SPARSE_ATTEND, ...) exceeds the buffer
 *   (e.g. about 5 sequences of 2^20 tokens at a 1/64 budget with 32 query
 *   heads of 128 dims).
 *   The first call on a device looks up the buffer's device address on that
 *   device (make it before any stream capture).  All calls share the buffer,
 *   which keeps the last call's contents; the kernels reset what must start
 *   at zero themselves.  Calls whose work overlaps on the GPU (other streams,
 *   other threads) race on the buffer: serialise them.
 */
#define ENTMAXKV_STATIC_SCRATCH_BYTES ((size_t)16 << 20)
ENTMAXKV_API int entmaxkv_sparse_attend_static(const entmaxkv_pool* pool, const float* q, int32_t H_q,
                                  const int32_t* page_table, int32_t max_pages,
                                  const int32_t* seq_lens, int32_t B, const int32_t* sel,
                                  const int32_t* sel_count, int32_t k_max, float alpha, float scale,
                                  float* out, float* tau_out, int32_t* v_pages, int32_t* status,
                                  void* stream);

/*
 * Full-cache alpha-entmax decode: entmaxkv_sparse_attend over every page of
 * every sequence (German summary, section 4: the full-cache entmax decoding
 * baseline).  Every key is read; value pages are read where they hold weight,
 * as in entmaxkv_sparse_attend (v_pages likewise, may be NULL).
 * workspace: ENTMAXKV_OP_FULL_ENTMAX.
 */
ENTMAXKV_API int entmaxkv_full_entmax_decode(const entmaxkv_pool* pool, const float* q, int32_t H_q,
                                const int32_t* page_table, int32_t max_pages,
                                const int32_t* seq_lens, int32_t B, float alpha, float scale,
                                float* out, float* tau_out, int32_t* v_pages, void* workspace,
                                size_t ws_bytes, int32_t* status, void* stream);

/*
 * Full-cache softmax decode, split over the cache with a log-sum-exp merge
 * (German summary, section 4: full-cache softmax, FlashDecoding).
 *   out[b][h] = sum_i softmax(scale * q_h . k_i)_i v_i, [B][H_q][d] fp32.
 *   workspace: ENTMAXKV_OP_FULL_SOFTMAX.
 */
ENTMAXKV_API int entmaxkv_full_softmax_decode(const entmaxkv_pool* pool, const float* q, int32_t H_q,
                                 const int32_t* page_table, int32_t max_pages,
                                 const int32_t* seq_lens, int32_t B, float scale, float* out,
                                 void* workspace, size_t ws_bytes, int32_t* status, void* stream);

/*
 * Softmax attention over the caller's selected pages: the sparse softmax
 * decoding the pages compare EntmaxKV against at the same kept set / budget
 * (German summary, section 3 "Vergleich" and section 4
 * "Approximationsqualitaet": softmax has a dense tail, so any dropped token
 * loses mass delta > 0, and the output error is bounded by 2 B delta).
 *   out[b][h] = sum_{i in kept} softmax_kept(scale * q_h . k_i)_i v_i, the
 *   softmax renormalised over the valid tokens of the listed pages,
 *   [B][H_q][d] fp32; a kv head with an empty list gives zeros.
 * sel, sel_count, k_max as in entmaxkv_sparse_attend (any set of distinct
 * pages, e.g. the output of entmaxkv_select).  Split over the list with the
 * log-sum-exp merge of entmaxkv_full_softmax_decode.
 * workspace: entmaxkv_workspace_size(ENTMAXKV_OP_SPARSE_SOFTMAX, ...) bytes.
 * Errors: as entmaxkv_sparse_attend.
 */
ENTMAXKV_API int entmaxkv_sparse_softmax_attend(const entmaxkv_pool* pool, const float* q, int32_t H_q,
                                   const int32_t* page_table, int32_t max_pages,
                                   const int32_t* seq_lens, int32_t B, const int32_t* sel,
                                   const int32_t* sel_count, int32_t k_max, float scale, float* out,
                                   void* workspace, size_t ws_bytes, int32_t* status, void* stream);

/*
 * Bytes of device workspace an entry point needs (host only; uses the SM
 * count of the current device, so call it with the device that will run the
 * step current).  op: entmaxkv_op.  The workspace is scratch: its contents
 * need no initialisation and are unspecified afterwards; two calls that
 * overlap on the GPU must not share one.
 */
ENTMAXKV_API size_t entmaxkv_workspace_size(int32_t op, int32_t B, int32_t H_q, int32_t H_kv,
                               int32_t max_pages, int32_t k_max, int32_t ps, int32_t d);

/* Text for a status code (host only; static storage). */
ENTMAXKV_API const char* entmaxkv_status_string(int32_t code);

/*
 * Failure-detection self test (the pages have no counterpart; it exercises the
 * bounded device wait every pipelined kernel uses).  Launches one block that
 * waits on a shared-memory barrier nothing ever completes, gives up after
 * limit_ns nanoseconds and writes ENTMAXKV_TIMEOUT to *status.  No memory copy
 * is in flight while it waits.  limit_ns must lie in [0, 2e9].
 */
ENTMAXKV_API int entmaxkv_selftest_timeout(int64_t limit_ns, int32_t* status, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* ENTMAXKV_H */
