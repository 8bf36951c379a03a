// Device helpers shared by the EntmaxKV kernels (sm_100a).
//
// - status reporting (first error sticks),
// - shared-memory barriers with a bounded wait (globaltimer based),
// - TMA tile loads into 128-byte-swizzled shared memory,
// - ldmatrix + mma.sync m16n8k16 (bf16 in, fp32 accumulate) wrappers,
// - bf16 helpers and block reductions.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "entmaxkv.h"

#define EKV_DEV __device__ __forceinline__

namespace ekv {

constexpr int kThreads = 128;            // CTA size of the pipelined kernels
constexpr int kStageTok = 64;            // tokens per pipeline stage
constexpr uint64_t kWaitLimitNs = 1000000000ull;   // 1 s bounded wait

EKV_DEV void report(int32_t* status, int code)
{
    if (status) atomicCAS(status, 0, code);
}

// ---------------------------------------------------------------- bf16
EKV_DEV float bf16_bits_to_f32(uint32_t u16) { return __uint_as_float(u16 << 16); }

// round-to-nearest-even fp32 -> bf16 bits (finite inputs)
EKV_DEV uint32_t f32_to_bf16_bits(float f)
{
    uint32_t u = __float_as_uint(f);
    u += 0x7FFFu + ((u >> 16) & 1u);
    return u >> 16;
}

// split f into hi + lo, both bf16, packed helpers return the bits
EKV_DEV void split_bf16(float f, uint32_t& hi, uint32_t& lo)
{
    hi = f32_to_bf16_bits(f);
    lo = f32_to_bf16_bits(f - bf16_bits_to_f32(hi));
}

EKV_DEV uint32_t pack2(uint32_t lo16, uint32_t hi16) { return (lo16 & 0xFFFFu) | (hi16 << 16); }

// ---------------------------------------------------------------- shared memory
EKV_DEV uint32_t smem_addr(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

EKV_DEV void mbar_init(uint64_t* bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

EKV_DEV void fence_mbar_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

EKV_DEV void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
                 : "memory");
}

EKV_DEV void mbar_arrive(uint64_t* bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

EKV_DEV bool mbar_try_wait(uint64_t* bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n"
        " .reg .pred p;\n"
        " mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n"
        "}\n"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

EKV_DEV uint64_t global_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// try_wait that lets the hardware suspend the thread until the phase
// completes or about hint_ns elapse, so that waiting warps do not spin on the
// issue slots the working warps of the SM need.
EKV_DEV bool mbar_try_wait_for(uint64_t* bar, uint32_t parity, uint32_t hint_ns)
{
    uint32_t ok;
    asm volatile(
        "{\n"
        " .reg .pred p;\n"
        " mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n"
        " selp.u32 %0, 1, 0, p;\n"
        "}\n"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity), "r"(hint_ns)
        : "memory");
    return ok != 0;
}

// Bounded wait for the phase with the given parity to complete.  Returns false
// when limit_ns elapsed first (the caller reports ENTMAXKV_TIMEOUT).
EKV_DEV bool mbar_wait(uint64_t* bar, uint32_t parity, uint64_t limit_ns)
{
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    while (true) {
        if (mbar_try_wait_for(bar, parity, 100000u)) return true;
        if (global_ns() - t0 > limit_ns) return false;
    }
}

// 2-D TMA tile load global -> shared, completion counted on `bar` in bytes.
// x (innermost coordinate, elements) must be a multiple of 8 for bf16.
EKV_DEV void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        ::"r"(smem_addr(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_addr(bar))
        : "memory");
}

// 1-D bulk copy global -> shared (both 16-byte aligned, bytes a multiple of 16),
// completion counted on `bar` in bytes.
EKV_DEV void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(smem_addr(dst)), "l"(src), "r"(bytes), "r"(smem_addr(bar))
                 : "memory");
}

// Order this thread's generic-proxy shared-memory writes before later
// async-proxy (TMA) accesses of the same memory.
EKV_DEV void fence_proxy_async()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

EKV_DEV void prefetch_tmap(const CUtensorMap* map)
{
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// Address of the 16-byte chunk `chunk` (0..D/8-1) of stage row `row` (0..63)
// in a stage written by TMA with 128-byte swizzle: the stage holds D/64
// column halves of 64 rows x 128 bytes each.
EKV_DEV uint32_t swz_addr(uint32_t base, int row, int chunk)
{
    const int half = chunk >> 3;
    const int c = chunk & 7;
    return base + half * (kStageTok * 128) + row * 128 + ((c ^ (row & 7)) << 4);
}

// Round a dynamic shared-memory base up to `align` bytes by offsetting from
// the shared array itself (keeps the pointer in the shared address space, so
// the compiler emits shared loads/stores instead of generic ones).
template <int ALIGN>
EKV_DEV uint8_t* smem_align(uint8_t* base)
{
    const uint32_t a = smem_addr(base);
    return base + ((ALIGN - (a & (ALIGN - 1))) & (ALIGN - 1));
}

EKV_DEV uint4 lds128(uint32_t addr)
{
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
    return v;
}

EKV_DEV float4 lds128f(uint32_t addr)
{
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr));
    return v;
}

// ---------------------------------------------------------------- tensor cores
EKV_DEV void ldsm_x4(uint32_t addr, uint32_t (&r)[4])
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

EKV_DEV void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4])
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

// D[16x8] += A[16x16] * B[16x8], bf16 inputs, fp32 accumulators.
EKV_DEV void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// ---------------------------------------------------------------- reductions
template <typename T>
EKV_DEV T warp_sum(T v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

EKV_DEV float warp_max(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

EKV_DEV double warp_max_d(double v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmax(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

EKV_DEV double warp_min_d(double v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmin(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

EKV_DEV float warp_min(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fminf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// Block-wide reductions; `red` is shared scratch of >= blockDim/32 elements.
// All threads get the result.  Two __syncthreads inside.
template <typename T>
EKV_DEV T block_sum(T v, T* red)
{
    v = warp_sum(v);
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31, nw = blockDim.x >> 5;
    __syncthreads();
    if (l == 0) red[w] = v;
    __syncthreads();
    T t = 0;
    for (int i = 0; i < nw; ++i) t += red[i];
    return t;
}

EKV_DEV float block_max(float v, float* red)
{
    v = warp_max(v);
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31, nw = blockDim.x >> 5;
    __syncthreads();
    if (l == 0) red[w] = v;
    __syncthreads();
    float t = -INFINITY;
    for (int i = 0; i < nw; ++i) t = fmaxf(t, red[i]);
    return t;
}

EKV_DEV float block_min(float v, float* red)
{
    v = warp_min(v);
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31, nw = blockDim.x >> 5;
    __syncthreads();
    if (l == 0) red[w] = v;
    __syncthreads();
    float t = INFINITY;
    for (int i = 0; i < nw; ++i) t = fminf(t, red[i]);
    return t;
}

// ---------------------------------------------------------------- cp.async
// Per-thread asynchronous 16-byte global -> shared copies (L1 bypassed); a
// thread waits only for its own groups, so a thread that reads back nothing
// but what it copied itself needs no block barrier.
EKV_DEV void cp_async16(uint32_t dst, const void* src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
EKV_DEV void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
EKV_DEV void cp_async_wait()
{
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// ---------------------------------------------------------------- clusters
// Thread-block clusters: the CTAs of a cluster are co-scheduled on one GPC and
// read each other's shared memory (distributed shared memory).  A CTA may
// touch another CTA's shared memory only after a cluster barrier that both
// have passed, and must not exit while another CTA may still read its own.
EKV_DEV uint32_t cluster_rank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
EKV_DEV void cluster_arrive() { asm volatile("barrier.cluster.arrive.release;" ::: "memory"); }
EKV_DEV void cluster_wait() { asm volatile("barrier.cluster.wait.acquire;" ::: "memory"); }
EKV_DEV void cluster_sync()
{
    cluster_arrive();
    cluster_wait();
}
// Address, in the cluster's shared window, of this CTA's shared variable `p`
// as held by the CTA of rank `rank`.
EKV_DEV uint32_t dsmem(const void* p, uint32_t rank)
{
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr(p)), "r"(rank));
    return r;
}
EKV_DEV void st_dsmem_f32(uint32_t a, float v)
{
    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(a), "f"(v) : "memory");
}
EKV_DEV void st_dsmem_s32(uint32_t a, int v)
{
    asm volatile("st.shared::cluster.s32 [%0], %1;" ::"r"(a), "r"(v) : "memory");
}
EKV_DEV float ld_dsmem_f32(uint32_t a)
{
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(a) : "memory");
    return v;
}
EKV_DEV int ld_dsmem_s32(uint32_t a)
{
    int v;
    asm volatile("ld.shared::cluster.s32 %0, [%1];" : "=r"(v) : "r"(a) : "memory");
    return v;
}
EKV_DEV uint4 ld_dsmem_v4(uint32_t a)
{
    uint4 v;
    asm volatile("ld.shared::cluster.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(a)
                 : "memory");
    return v;
}
EKV_DEV unsigned long long ld_dsmem_u64(uint32_t a)
{
    unsigned long long v;
    asm volatile("ld.shared::cluster.u64 %0, [%1];" : "=l"(v) : "r"(a) : "memory");
    return v;
}

// Ordered integer key of a float: larger float -> larger key; -0 maps like +0.
EKV_DEV uint32_t ordered_key(float f)
{
    if (f == 0.0f) f = 0.0f;
    uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

EKV_DEV int ceil_div(int a, int b) { return (a + b - 1) / b; }

// Programmatic dependent launch: every kernel of the library starts with
// pdl_enter(), which lets the next kernel in the stream begin launching and
// then waits until the previous grid has completed and its writes are
// visible.  Every CTA calls it before anything else, so completion stays
// transitive along the stream.
EKV_DEV void pdl_enter()
{
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

// Pages of a sequence of L tokens, clipped to the page-table row length; a
// longer sequence is reported as ENTMAXKV_DEVICE_BOUNDS.
EKV_DEV int pages_of(int L, int ps, int max_pages, int32_t* status)
{
    const int P = L > 0 ? (L + ps - 1) / ps : 0;
    if (P > max_pages) {
        report(status, ENTMAXKV_DEVICE_BOUNDS);
        return max_pages;
    }
    return P;
}

}  // namespace ekv
