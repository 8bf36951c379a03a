// entmaxkv_sparse_attend_static: sparse entmax attention for callers that
// cannot allocate device memory.
//
// Some callers may not call cudaMalloc when they decode: code running under
// CUDA stream capture (allocation is not allowed while capturing), hosts
// whose own allocator owns all device memory, and latency-critical loops
// where an allocation or free would synchronise the device.  This entry point
// takes the scratch memory sparse attention needs from a fixed buffer
// compiled into the library instead of a caller-provided workspace.
//
// The buffer is a file-scope __device__ array of kStaticScratchBytes; every
// GPU that loads the library holds it until the process exits.  In host code
// its name is only a host-side stand-in, so its device address is looked up
// once per device with cudaGetSymbolAddress (with that device current) and
// passed to the kernels.  All calls share the buffer and it keeps the last
// call's contents; the kernels clear what must start at zero (the split
// arrival counters) themselves, and calls that overlap on the GPU race.
#include <mutex>

#include "common.cuh"
#include "kernels.cuh"

namespace ekv {

constexpr size_t kStaticScratchBytes = ENTMAXKV_STATIC_SCRATCH_BYTES;

static __device__ __align__(256) uint8_t g_static_scratch[kStaticScratchBytes];

// Device address of the scratch buffer on the current device (looked up on the
// first call for that device); nullptr on failure.
static void* static_scratch_address()
{
    static std::mutex mu;
    static void* addr[64] = {nullptr};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess) return nullptr;
        addr[dev] = p;
    }
    return addr[dev];
}

}  // namespace ekv

extern "C" {

int entmaxkv_sparse_attend_static(const entmaxkv_pool* pool, const float* q, int32_t H_q,
                                  const int32_t* page_table, int32_t max_pages, const int32_t* seq_lens,
                                  int32_t B, const int32_t* sel, const int32_t* sel_count, int32_t k_max,
                                  float alpha, float scale, float* out, float* tau_out, int32_t* v_pages,
                                  int32_t* status, void* stream)
{
    // the argument checks of entmaxkv_sparse_attend come first, so a bad call
    // gets the same code from both entry points whatever its size
    const int rc = ekv::attend_check(ENTMAXKV_OP_SPARSE_ATTEND, pool, q, H_q, page_table, max_pages, seq_lens, B,
                                     sel, sel_count, k_max, alpha, scale, out, status);
    if (rc || B == 0) return rc;
    const size_t need = entmaxkv_workspace_size(ENTMAXKV_OP_SPARSE_ATTEND, B, H_q, pool->H_kv, max_pages, k_max,
                                                pool->ps, pool->d);
    if (need == 0) return ENTMAXKV_INVALID_ARG;
    if (need > ekv::kStaticScratchBytes) return ENTMAXKV_STATIC_LIMIT;
    void* scratch = ekv::static_scratch_address();
    if (!scratch) return ENTMAXKV_CUDA_ERROR;
    return entmaxkv_sparse_attend(pool, q, H_q, page_table, max_pages, seq_lens, B, sel, sel_count, k_max, alpha,
                                  scale, out, tau_out, v_pages, scratch, ekv::kStaticScratchBytes, status, stream);
}

}  // extern "C"
