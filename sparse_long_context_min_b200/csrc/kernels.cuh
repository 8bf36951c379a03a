// Host-side launch entry points of the kernels (internal to the library).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <cmath>
#include <utility>

#include "entmaxkv.h"

namespace ekv {

// The fused bf16 entmax kernel runs at most kFusedMaxSplits splits per (sequence,
// kv head), each publishing up to kFusedCandCap threshold candidates per query head.
constexpr int kFusedMaxSplits = 16;
constexpr int kFusedCandCap = 256;

// Arguments shared by the attention kernels (passed by value).
struct AttnArgs {
    const float* q;                // [B][H_q][d]
    int H_q, H_kv, G;
    const int32_t* page_table;     // [B][max_pages]
    int max_pages;
    const int32_t* seq_lens;       // [B]
    const int32_t* sel;            // [B][H_kv][k_max], NULL = every page in order
    const int32_t* sel_count;      // [B][H_kv], NULL = P_b
    int k_max;                     // row length of sel and of the score buffer (in pages)
    int num_phys;
    int S;                         // splits per (sequence, kv head)
    float alpha;
    float xscale;                  // (alpha - 1) * scale, or scale for softmax
    float* xbuf;                   // [B][H_q][k_max * ps] scores x of the listed tokens
    float* cmax;                   // [B][H_q][k_max * ps / 16] largest x of each 16-token chunk (bf16 K pass)
    float* tau;                    // [B][H_q]
    float* opart;                  // [B][H_q][S][d] partial outputs
    float* mlpart;                 // [B][H_q][S][2] softmax running max and sum
    float* lmax;                   // [B][H_q][S] largest score of each split (K pass)
    int32_t* vpages;               // [B][H_kv] value pages loaded (V pass adds), or NULL
    int32_t* counters;             // [B][H_kv] arrival counters of the split reduction
    float* cval;                   // [B][H_q][S][kFusedCandCap] candidate scores (fused bf16 kernel)
    int32_t* cidx;                 // [B][H_q][S][kFusedCandCap] their list positions (fused bf16 kernel)
    float* out;                    // [B][H_q][d]
    float* tau_out;                // [B][H_q] or NULL
    int32_t* status;
};

int launch_append(const entmaxkv_pool& pool, const void* k_new, const void* v_new, int n_new,
                  const int32_t* page_table, int max_pages, int32_t* seq_lens, int B, int32_t* status,
                  cudaStream_t stream);

// seq_lens[b] += n_new for b < B (after the previous grid has completed)
int launch_advance(int32_t* seq_lens, int B, int n_new, cudaStream_t stream);

// append (n_new tokens per sequence) and bounding-box scoring over the new
// lengths in one launch where the layout allows, else the two in turn; the
// results equal launch_append followed by launch_score(BBOX)
int launch_append_score(const entmaxkv_pool& pool, const void* k_new, const void* v_new, int n_new, const float* q,
                        int H_q, const int32_t* page_table, int max_pages, int32_t* seq_lens, int B, float scale,
                        float* ub, int32_t* status, cudaStream_t stream);

int launch_score(const entmaxkv_pool& pool, const float* q, int H_q, const int32_t* page_table,
                 int max_pages, const int32_t* seq_lens, int B, int mode, float scale, float* ub, float* m,
                 float* v, float* est, int32_t* status, cudaStream_t stream);

int launch_select(int mode, const float* ub, const float* m, const float* v, const float* est,
                  const int32_t* seq_lens, int ps, int B, int H_q, int H_kv, int max_pages, int budget,
                  float budget_frac, float alpha, float delta, int k_max, int32_t* sel, int32_t* sel_count,
                  float* tau_hat, int32_t* status, cudaStream_t stream);

// entmax attention over the listed pages (sparse, or full when a.sel == NULL)
int launch_entmax_attend(const entmaxkv_pool& pool, const AttnArgs& a, int B, const CUtensorMap* kmap,
                         const CUtensorMap* vmap, cudaStream_t stream);

int launch_softmax_attend(const entmaxkv_pool& pool, const AttnArgs& a, int B, const CUtensorMap* kmap,
                          const CUtensorMap* vmap, cudaStream_t stream);

// Host-side argument checks of the attention entry points (op: entmaxkv_op),
// everything but the workspace; ENTMAXKV_OK when the call may proceed.
int attend_check(int op, const entmaxkv_pool* pool, const float* q, int H_q, const int32_t* page_table,
                 int max_pages, const int32_t* seq_lens, int B, const int32_t* sel, const int32_t* sel_count,
                 int k_max, float alpha, float scale, const float* out, const int32_t* status);

int launch_selftest_timeout(int64_t limit_ns, int32_t* status, cudaStream_t stream);

// set the dynamic shared memory limit of a kernel once per device
int ensure_smem(const void* func, int bytes);

// SM count of the current device
int num_sms();

// Dynamic shared memory limit and permission for clusters above 8 CTAs of a
// cluster kernel, once per device.
int ensure_cluster_kernel(const void* func, int smem);

// Clusters of `cluster` CTAs (threads, smem each) the current device can run
// at once (0 when none fits); cached per (kernel, size, device).
int max_active_clusters(const void* func, int cluster, int threads, int smem);

// Launch with programmatic stream serialization (the kernel calls pdl_enter()).
template <typename... KArgs, typename... Args>
static cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              Args&&... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// launch_pdl for a kernel whose CTAs form clusters of `cluster` along x
template <typename... KArgs, typename... Args>
static cudaError_t launch_pdl_cluster(void (*kern)(KArgs...), dim3 grid, dim3 block, int cluster, size_t smem,
                                      cudaStream_t st, Args&&... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = cluster;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

}  // namespace ekv
