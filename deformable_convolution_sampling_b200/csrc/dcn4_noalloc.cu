// dcn4_noalloc.cu — dcn4_backward without a caller-provided workspace.
//
// Some callers cannot hand the library device memory at the point of the
// call: a plugin embedded in a host runtime that owns every device buffer and
// exposes no allocator to it, or a service that fixes its device-memory budget
// at start-up and must not allocate afterwards.  For them the backward's
// scratch (per-image reach words, per-pixel cell boxes and per-sample cell
// codes) lives in the file-scope array below, which the CUDA driver places on
// every device that loads this library and keeps there until the process
// exits.  Nothing here calls cudaMalloc, cudaFree or an allocating library
// routine.
#include <cuda.h>  // CUcontext and CUresult only: the two driver calls below come from cudaGetDriverEntryPoint

#include <cstdio>
#include <mutex>

#include "dcn4.h"
#include "dcn4_common.cuh"

namespace {

constexpr size_t kScratchBytes = static_cast<size_t>(DCN4_NOALLOC_SCRATCH_BYTES);

// The shared scratch.  In host code this name is only a stand-in for the
// device symbol: its device address comes from cudaGetSymbolAddress.
__device__ __align__(256) unsigned char g_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;

// The area's address is looked up once per device and context: a device reset
// (cudaDeviceReset, or the primary context released and made again) unloads
// the module, so the array may come back elsewhere.  Contexts are told apart by
// the driver's context id, which is never reused within a process.
struct ScratchSlot {
    unsigned long long ctx_id;  // 0: not set up
    void* ptr;
};
ScratchSlot g_slot[kMaxDevices];
std::mutex g_setup_mutex;

thread_local char g_error[256] = "";

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// Id of the calling thread's current context, or 0 when there is none yet.
cudaError_t current_context_id(unsigned long long* id) {
    static CtxGetCurrentFn get_current = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static std::once_flag once;
    static cudaError_t resolved = cudaSuccess;
    std::call_once(once, [] {
        void* a = nullptr;
        void* b = nullptr;
        cudaError_t e = cudaGetDriverEntryPoint("cuCtxGetCurrent", &a, cudaEnableDefault, nullptr);
        if (e == cudaSuccess) e = cudaGetDriverEntryPoint("cuCtxGetId", &b, cudaEnableDefault, nullptr);
        if (e == cudaSuccess && (a == nullptr || b == nullptr)) e = cudaErrorSymbolNotFound;
        resolved = e;
        get_current = reinterpret_cast<CtxGetCurrentFn>(a);
        get_id = reinterpret_cast<CtxGetIdFn>(b);
    });
    if (resolved != cudaSuccess) return resolved;
    CUcontext ctx = nullptr;
    if (get_current(&ctx) != CUDA_SUCCESS) return cudaErrorContextIsDestroyed;
    *id = 0;
    if (ctx != nullptr && get_id(ctx, id) != CUDA_SUCCESS) return cudaErrorContextIsDestroyed;
    return cudaSuccess;
}

}  // namespace

extern "C" const char* dcn4_noalloc_last_error(void) { return g_error; }

extern "C" int dcn4_backward_noalloc(const dcn4_params* p, const void* value, const void* offset_mask,
                                     const void* grad_out, void* grad_value, void* grad_offset_mask, void* stream) {
    const int st = dcn4_check_params(p);
    if (st != DCN4_OK) return st;
    const size_t need = dcn4_backward_workspace_size(p);
    if (need > kScratchBytes) {
        snprintf(g_error, sizeof g_error,
                 "dcn4_backward_noalloc: this problem needs %zu bytes of scratch, the built-in area holds %zu",
                 need, kScratchBytes);
        return DCN4_ERR_WORKSPACE;
    }
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        snprintf(g_error, sizeof g_error, "dcn4_backward_noalloc: no usable current device (%s)",
                 cudaGetErrorString(e));
        return DCN4_ERR_LAUNCH;
    }
    void* scratch = nullptr;
    {
        // Set-up, once per device (and again after a device reset), with that
        // device current: look the area's device address up.
        std::lock_guard<std::mutex> lock(g_setup_mutex);
        unsigned long long ctx = 0;
        e = current_context_id(&ctx);
        if (e == cudaSuccess && (ctx == 0 || g_slot[dev].ctx_id != ctx)) {
            e = cudaGetSymbolAddress(&scratch, g_scratch);  // makes the device's context current if none is
            if (e == cudaSuccess) e = current_context_id(&ctx);
            if (e == cudaSuccess && (scratch == nullptr || ctx == 0)) e = cudaErrorContextIsDestroyed;
            if (e == cudaSuccess) g_slot[dev] = ScratchSlot{ctx, scratch};
        }
        if (e != cudaSuccess) {
            g_slot[dev] = ScratchSlot{0, nullptr};
            snprintf(g_error, sizeof g_error, "dcn4_backward_noalloc: scratch look-up on device %d failed (%s)",
                     dev, cudaGetErrorString(e));
            return DCN4_ERR_LAUNCH;
        }
        scratch = g_slot[dev].ptr;
    }
    g_error[0] = '\0';
    return dcn4_backward(p, value, offset_mask, grad_out, grad_value, grad_offset_mask, scratch, kScratchBytes,
                         stream);
}

extern "C" size_t dcn4_backward_noalloc_capacity(void) { return kScratchBytes; }
