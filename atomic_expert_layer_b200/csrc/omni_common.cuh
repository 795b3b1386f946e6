// omni_common.cuh -- device helpers shared by the sm_100a kernels of libomni:
// the workspace status word, bounded mbarrier waits, order-preserving float
// keys, warp reductions and the launch helper (programmatic dependent
// launch).  Nothing here is method arithmetic.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "omni.h"

namespace omni {

// ---------------------------------------------------------------- status word
// The first 256 bytes of every workspace are a header: word 0 is the device
// status (OMNI_DEV_*), the rest are counters used by individual kernels.
struct WsHeader {
    int status;
    int pad[63];
};
static_assert(sizeof(WsHeader) == 256, "header must stay 256 bytes");

__device__ __forceinline__ void set_status(int *status, int code) {
    atomicCAS(status, 0, code);   // first error wins
}

// --------------------------------------------------------------- float keys
// Monotone map fp32 -> uint32: a < b (as floats, -0 == +0) <=> key(a) < key(b)
// except that -0 maps just below +0; callers that need -0 == +0 canonicalise.
__device__ __forceinline__ uint32_t f2key(float f) {
    uint32_t u = __float_as_uint(f);
    if (u == 0x80000000u) u = 0u;                    // -0 -> +0
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key2f(uint32_t k) {
    uint32_t u = (k & 0x80000000u) ? (k & 0x7fffffffu) : ~k;
    return __uint_as_float(u);
}

__device__ __forceinline__ unsigned lane_id() { return threadIdx.x & 31u; }
__device__ __forceinline__ unsigned lanemask_lt() {
    unsigned m;
    asm volatile("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

// ------------------------------------------------------------------ mbarrier
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}"
                 ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}"
                 ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Bounded wait for the phase with the given parity to complete.  Gives up
// after kWaitLimitNs of wall time (or kWaitSpinLimit polls), records
// OMNI_DEV_WAIT_TIMEOUT and returns false; the caller then unwinds.
constexpr uint64_t kWaitLimitNs = 4000000000ull;   // 4 s
constexpr uint32_t kWaitSpinLimit = 1u << 30;

__device__ __forceinline__ bool mbar_wait_limit(uint64_t *bar, uint32_t parity, int *status,
                                                uint64_t limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t it = 0; it < kWaitSpinLimit; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 63u) == 63u) {
            const uint64_t dt = global_timer_ns() - t0;
            if (dt > limit_ns) break;
            // another thread already gave up: poll a little longer only
            if (*(volatile int *)status != 0 && dt > limit_ns / 64) break;
        }
    }
    set_status(status, OMNI_DEV_WAIT_TIMEOUT);
    return false;
}

__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, int *status) {
    return mbar_wait_limit(bar, parity, status, kWaitLimitNs);
}

// ------------------------------------------------------------ warp helpers
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ __forceinline__ int warp_isum(int v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
// inclusive prefix sum over the warp
__device__ __forceinline__ int warp_iscan(int v) {
    const unsigned l = lane_id();
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int n = __shfl_up_sync(0xffffffffu, v, o);
        if (l >= (unsigned)o) v += n;
    }
    return v;
}

// ------------------------------------------- programmatic dependent launch
// Kernels of the library are launched with programmatic stream serialisation
// (launch() below): their CTAs may be scheduled while the previous kernel in
// the stream is still finishing.  Each kernel therefore
// calls grid_dependency_wait() in every thread, before its first access to
// global memory that earlier work in the stream writes or reads; since every
// kernel waits, a kernel's completion implies that of all earlier ones.
// grid_dependents_launch() lets the next kernel's CTAs start their prologue
// as this kernel's CTAs leave the SMs (it carries no memory ordering).
__device__ __forceinline__ void grid_dependency_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void grid_dependents_launch() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

//
// griddepcontrol.wait orders a kernel only after earlier KERNELS; a copy or a
// memset that precedes it in the stream is not covered.  So only launches
// whose predecessor is one of this library's kernels use the attribute: every
// entry point calls first_launch_in_call() after its workspace memset, and
// the next launch() then goes out with ordinary stream ordering.
inline thread_local bool t_plain_next_launch = false;

inline void first_launch_in_call() { t_plain_next_launch = true; }

template <typename... KArgs, typename... Args>
inline cudaError_t launch(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                          cudaStream_t st, Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = t_plain_next_launch ? 0 : 1;
    t_plain_next_launch = false;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

}  // namespace omni
