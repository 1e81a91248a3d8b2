// logo_global_attn_sparse_noalloc: the selected-query global branch (and the
// gated merge) for callers that cannot allocate device memory.
//
// Who cannot allocate: a caller that only receives the op's own tensors from a
// framework whose allocator owns the device memory (a plugin or FFI layer with
// no way to ask that allocator for a workspace), or a latency-critical serving
// loop where cudaMalloc / cudaFree would synchronise the device and stall work
// on other streams.  They still pass every input and output; only the
// library's scratch (the device status word the kernel reports through) is
// replaced by a fixed array compiled into the library.
//
// The array is a file-scope __device__ variable of kNoAllocScratchBytes bytes.
// Every GPU that loads the library holds it until the process exits.  Host
// code cannot use the array's name as a device address, so the first call on
// each device (with that device current) looks the address up once with
// cudaGetSymbolAddress and caches it with the context it belongs to (a device
// reset makes the next call look it up again); make that first call, and the
// first call after a reset, before any stream capture.  Every call on a device shares the one array and finds the previous
// call's contents in it: each call clears the status word first, and two
// calls that overlap on the GPU (different streams, no ordering) race on it.
// Device-side errors of a call land in that shared status word, which this
// entry point does not read back: callers that need the report use
// logo_global_attn_sparse with their own workspace and logo_check.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "kernels.cuh"
#include "logo.h"

namespace {

constexpr size_t kNoAllocScratchBytes = 256 * 1024;
constexpr size_t kStatusBytes = 256;  // the workspace header the kernels report through
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};
CUcontext g_scratch_ctx[kMaxDevices] = {};

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);

// The calling thread's current context (nullptr when none is current or the
// driver entry point is unavailable).
CUcontext current_context()
{
    static std::once_flag once;
    static CtxGetCurrentFn fn = nullptr;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<CtxGetCurrentFn>(p);
    });
    CUcontext c = nullptr;
    if (fn && fn(&c) != CUDA_SUCCESS) c = nullptr;
    return c;
}

// Device address of the static scratch on the current device, looked up once
// per device and context: after a cudaDeviceReset the runtime creates a new
// primary context on the next call, the array lives at a new address there,
// and the changed context handle makes this look it up again.
logo_status scratch_address(void** out)
{
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        logo::set_last_error("no-alloc scratch: cudaGetDevice failed: %s", cudaGetErrorString(e));
        return LOGO_ERR_CUDA;
    }
    if (dev < 0 || dev >= kMaxDevices) {
        logo::set_last_error("no-alloc scratch: device %d beyond the %d devices supported", dev, kMaxDevices);
        return LOGO_ERR_UNSUPPORTED;
    }
    std::lock_guard<std::mutex> lock(g_mu);
    const CUcontext ctx = current_context();
    if (!g_scratch_addr[dev] || !ctx || ctx != g_scratch_ctx[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);  // also makes the primary context current
        if (e != cudaSuccess || !p) {
            logo::set_last_error("no-alloc scratch: cudaGetSymbolAddress failed on device %d: %s", dev,
                                 cudaGetErrorString(e));
            return LOGO_ERR_CUDA;
        }
        g_scratch_addr[dev] = p;
        g_scratch_ctx[dev] = current_context();
    }
    *out = g_scratch_addr[dev];
    return LOGO_OK;
}

}  // namespace

extern "C" LOGO_API logo_status logo_global_attn_sparse_noalloc(
    const logo_bf16* q, const logo_bf16* k, const logo_bf16* v, const float* gate, const int32_t* sel_idx,
    const int32_t* cu_sel, const logo_shape* shape, int max_selected, float scale, int merge, logo_bf16* out,
    logo_stream_t stream)
{
    // Scratch this shape needs (ratio 1 is the largest case); refuse what the fixed array cannot hold.
    const size_t need = logo_workspace_size(shape, 1.0);
    if (need == 0) {
        logo::set_last_error("no-alloc global attention: invalid shape");
        return LOGO_ERR_INVALID_ARG;
    }
    if (need > kNoAllocScratchBytes) {
        logo::set_last_error("no-alloc global attention: this shape needs %zu bytes of scratch, the fixed array "
                             "holds %zu; use logo_global_attn_sparse with a workspace",
                             need, kNoAllocScratchBytes);
        return LOGO_ERR_WORKSPACE;
    }
    void* ws = nullptr;
    logo_status st = scratch_address(&ws);
    if (st != LOGO_OK) return st;
    cudaError_t e = cudaMemsetAsync(ws, 0, kStatusBytes, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) {
        logo::set_last_error("no-alloc global attention: clearing the status word failed: %s", cudaGetErrorString(e));
        return LOGO_ERR_CUDA;
    }
    return logo_global_attn_sparse(q, k, v, gate, sel_idx, cu_sel, shape, max_selected, scale, merge, out, ws,
                                   kNoAllocScratchBytes, stream);
}
