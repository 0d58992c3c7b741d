// pa_noalloc.cu — pa_decode_noalloc: pa_decode for callers that cannot
// allocate device memory.
//
// Some callers cannot call cudaMalloc (or any allocating routine) where they
// decode: code that runs inside a memory arena sized up front, plug-ins of a
// host engine that owns every device allocation, or loops that must never
// enter an allocator. pa_decode needs a workspace for the partial results of a
// split context and, for grouped-query heads, for the tensor-core kernel's
// work-item counter; this entry point takes that workspace from a buffer inside
// the library instead: a file-scope device array of PA_NOALLOC_SCRATCH_BYTES,
// which every GPU that loads the library holds until the process exits.
// Nothing here allocates.
//
// On the host, `s_scratch` names a host-side stand-in, not device memory, so
// its device address is looked up with cudaGetSymbolAddress, with the device
// current, and cached per device together with the CUDA context it was looked
// up in. A call that finds another context current on the device (after a
// cudaDeviceReset, the runtime creates a new primary context and loads the
// library's device code again, so the buffer may move) looks it up again; that
// call, like the first one on a device, should come before any stream capture.
// Every call shares the one buffer per device: calls whose kernels overlap on
// the GPU (different streams, no ordering between them) race on it. The buffer
// needs no clearing: each call writes every partial result before its merge
// reads it, and zeroes the counter before its kernel.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "pa.h"
#include "pa_internal.h"

static __device__ __align__(256) unsigned char s_scratch[PA_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
struct ScratchEntry {
    CUcontext ctx;  // context current when the address was looked up
    void* addr;
};
ScratchEntry g_scratch[kMaxDevices];
std::mutex g_scratch_mutex;

using CtxGetCurrentFn = CUresult (*)(CUcontext*);

// cuCtxGetCurrent from the driver (the library links only the runtime).
CtxGetCurrentFn ctx_get_current_fn() {
    static CtxGetCurrentFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &f, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<CtxGetCurrentFn>(f);
    });
    return fn;
}

// Device address of s_scratch on the current device: looked up on the first
// call on a device and again whenever the current context is not the one the
// cached address belongs to.
cudaError_t scratch_address(void** addr) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    const CtxGetCurrentFn get_ctx = ctx_get_current_fn();
    if (!get_ctx) return cudaErrorNotSupported;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    CUcontext ctx = nullptr;
    if (get_ctx(&ctx) != CUDA_SUCCESS) return cudaErrorDeviceUninitialized;
    ScratchEntry& ent = g_scratch[dev];
    if (!ent.addr || !ctx || ctx != ent.ctx) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, s_scratch);  // binds the device's primary context
        if (e != cudaSuccess) return e;
        if (!p) return cudaErrorInvalidSymbol;
        if (get_ctx(&ctx) != CUDA_SUCCESS || !ctx) return cudaErrorDeviceUninitialized;
        ent.ctx = ctx;
        ent.addr = p;
    }
    *addr = ent.addr;
    return cudaSuccess;
}

}  // namespace

extern "C" int pa_decode_noalloc(void* out, const void* q, const void* k_cache,
                                 const void* v_cache, const int32_t* block_tables,
                                 int32_t block_table_stride, const int32_t* context_lens,
                                 int32_t max_context_len, int32_t num_seqs, int32_t num_heads,
                                 float scale, const pa_cache_desc* cache,
                                 int32_t partition_size, void* stream) {
    // 0 means "no split" or invalid arguments; pa_decode reports the latter.
    const size_t need = pa_decode_workspace_size(num_seqs, num_heads, max_context_len, cache,
                                                 partition_size);
    if (need > (size_t)PA_NOALLOC_SCRATCH_BYTES)
        return pa::report_error(
            PA_ERR_WORKSPACE,
            "pa_decode_noalloc: this call needs %zu bytes of scratch, more than the library's "
            "fixed %zu (PA_NOALLOC_SCRATCH_BYTES); use pa_decode with a workspace of your own, "
            "or a larger partition_size",
            need, (size_t)PA_NOALLOC_SCRATCH_BYTES);
    void* scratch = nullptr;
    if (need > 0) {
        const cudaError_t e = scratch_address(&scratch);
        if (e != cudaSuccess)
            return pa::report_error(PA_ERR_CUDA,
                                    "pa_decode_noalloc: cudaGetSymbolAddress of the scratch "
                                    "buffer failed: %s", cudaGetErrorString(e));
    }
    return pa_decode(out, q, k_cache, v_cache, block_tables, block_table_stride, context_lens,
                     max_context_len, num_seqs, num_heads, scale, cache, partition_size, scratch,
                     need > 0 ? (size_t)PA_NOALLOC_SCRATCH_BYTES : 0, stream);
}
