// noalloc.cu -- the grouped expert computation for callers that cannot
// allocate device memory at call time.
//
// Some callers of this library must not call cudaMalloc (or any allocating
// routine) when they run the layer: a serving runtime whose device memory is
// planned once at start-up, or code running where allocation is not allowed.
// They cannot hand the library a workspace either.  This entry point takes
// the same inputs and outputs as omni_grouped_expert_fwd and keeps its
// scratch in a fixed array that is part of the library image on every device
// that loads it (about 2 MB, held until the process exits).
//
// Host code must not use the array's name as a device address: in host code
// it names a host-side stand-in.  The device address is looked up with
// cudaGetSymbolAddress, with the device current, on the first call made in
// each CUDA context, and cached under that context's unique id: after a
// cudaDeviceReset, or in a driver-API context other than the device's primary
// one, the library image is loaded again at another address, and the new
// context's id forces a fresh lookup.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstring>
#include <mutex>

#include "omni_common.cuh"
#include "omni_internal.h"

namespace omni {
namespace {

constexpr int kNoAllocMaxL = 16384;               // tokens
constexpr int64_t kNoAllocMaxM = 262144;          // tasks (L * K)
constexpr size_t kOffCount = 256;                 // after the 256-byte header
constexpr size_t kOffSlots = kOffCount + 4 * (size_t)kNoAllocMaxL;
constexpr size_t kNoAllocBytes = kOffSlots + 8 * (size_t)kNoAllocMaxM;

// Scratch shared by every call on a device: header (status word), per-token
// slot counters, per-task (expert, p) slots.
__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocBytes];

constexpr int kMaxDevices = 64;
struct ScratchEntry {
    unsigned long long ctx_id;   // unique id of the context the address belongs to
    void *addr;                  // nullptr: nothing cached
};
ScratchEntry g_scratch[kMaxDevices] = {};
std::mutex g_scratch_mutex;

typedef CUresult (*CtxGetCurrentFn)(CUcontext *);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long *);

// Unique id of the calling thread's current context; false when no context
// is current yet or the driver lacks the query.
bool current_context_id(unsigned long long *id) {
    static const CtxGetCurrentFn get_current = []() -> CtxGetCurrentFn {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        return reinterpret_cast<CtxGetCurrentFn>(p);
    }();
    static const CtxGetIdFn get_id = []() -> CtxGetIdFn {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        return reinterpret_cast<CtxGetIdFn>(p);
    }();
    if (!get_current || !get_id) return false;
    CUcontext ctx = nullptr;
    if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
    return get_id(ctx, id) == CUDA_SUCCESS;
}

// Device address of the scratch array in the current context.
cudaError_t scratch_address(void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    unsigned long long id = 0;
    bool have_id = current_context_id(&id);
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    ScratchEntry &c = g_scratch[dev];
    if (have_id && c.addr && c.ctx_id == id) {
        *out = c.addr;
        return cudaSuccess;
    }
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    // the lookup makes the device's primary context current if none was
    if (!have_id) have_id = current_context_id(&id);
    c.ctx_id = have_id ? id : 0;
    c.addr = have_id ? p : nullptr;           // without an id nothing is cached
    *out = p;
    return cudaSuccess;
}

}  // namespace
}  // namespace omni

using namespace omni;

extern "C" int omni_grouped_expert_fwd_noalloc(
    const omni_bf16 *x, const omni_bf16 *W, const omni_bf16 *V, int L, int d, int K, int N,
    int B, const int32_t *task_token, const int32_t *task_expert, const float *task_gate,
    const int32_t *group_offsets, const int32_t *active_groups, const int32_t *num_active,
    float *y, unsigned flags, omni_stream_t stream) {
    Sizes sz;
    if (N <= 0 || !make_sizes(L, d, N, 1, K, B, &sz)) return OMNI_ERR_INVALID_ARG;
    if ((int64_t)K > sz.N) return OMNI_ERR_INVALID_ARG;
    if (!x || !W || !V || !task_token || !task_expert || !task_gate || !group_offsets ||
        !active_groups || !num_active || !y)
        return OMNI_ERR_INVALID_ARG;
    if (L > kNoAllocMaxL || sz.M > kNoAllocMaxM) return OMNI_ERR_UNSUPPORTED;
    if (K > OMNI_MAX_K || B > OMNI_MAX_B || sz.N > INT32_MAX) return OMNI_ERR_UNSUPPORTED;
    if (d % 256 != 0 || d > OMNI_MAX_D) return OMNI_ERR_UNSUPPORTED;
    const uintptr_t a = reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(W) |
                        reinterpret_cast<uintptr_t>(V) | reinterpret_cast<uintptr_t>(y);
    if (a & 15u) return OMNI_ERR_INVALID_ARG;

    void *scratch = nullptr;
    if (scratch_address(&scratch) != cudaSuccess) return OMNI_ERR_CUDA;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    // the same launches as omni_grouped_expert_fwd, on a layout inside the array
    WsLayout lay;
    std::memset(&lay, 0, sizeof lay);
    lay.hdr = 0;
    lay.tok_count = kOffCount;
    lay.tok_slots = kOffSlots;
    lay.zero_end = kOffCount + 4 * (size_t)L;
    lay.total = kNoAllocBytes;
    // status word and this call's slot counters
    first_launch_in_call();
    if (cudaMemsetAsync(scratch, 0, lay.zero_end, st) != cudaSuccess) return OMNI_ERR_CUDA;
    const cudaError_t e = launch_grouped_expert(x, W, V, sz, task_token, task_expert, task_gate,
                                                y, (flags & OMNI_Y_ACCUMULATE) != 0, scratch, lay,
                                                st);
    return e == cudaSuccess ? OMNI_OK : OMNI_ERR_CUDA;
}

extern "C" int omni_noalloc_get_device_status(omni_stream_t stream, int *status_out) {
    if (!status_out) return OMNI_ERR_INVALID_ARG;
    void *scratch = nullptr;
    if (scratch_address(&scratch) != cudaSuccess) return OMNI_ERR_CUDA;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    int host = 0;
    if (cudaMemcpyAsync(&host, scratch, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess)
        return OMNI_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return OMNI_ERR_CUDA;
    if (cudaMemsetAsync(scratch, 0, sizeof(int), st) != cudaSuccess) return OMNI_ERR_CUDA;
    *status_out = host;
    return host == 0 ? OMNI_OK : OMNI_ERR_DEVICE;
}
