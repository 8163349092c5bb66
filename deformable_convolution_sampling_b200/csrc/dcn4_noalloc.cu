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
#include <atomic>
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
std::atomic<void*> g_scratch_ptr[kMaxDevices];
std::mutex g_setup_mutex;

thread_local char g_error[256] = "";

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
    void* scratch = g_scratch_ptr[dev].load(std::memory_order_acquire);
    if (scratch == nullptr) {
        // Set-up, once per device, with that device current.
        std::lock_guard<std::mutex> lock(g_setup_mutex);
        scratch = g_scratch_ptr[dev].load(std::memory_order_acquire);
        if (scratch == nullptr) {
            e = cudaGetSymbolAddress(&scratch, g_scratch);
            if (e != cudaSuccess || scratch == nullptr) {
                snprintf(g_error, sizeof g_error, "dcn4_backward_noalloc: cudaGetSymbolAddress failed (%s)",
                         cudaGetErrorString(e));
                return DCN4_ERR_LAUNCH;
            }
            g_scratch_ptr[dev].store(scratch, std::memory_order_release);
        }
    }
    g_error[0] = '\0';
    return dcn4_backward(p, value, offset_mask, grad_out, grad_value, grad_offset_mask, scratch, kScratchBytes,
                         stream);
}

extern "C" size_t dcn4_backward_noalloc_capacity(void) { return kScratchBytes; }
