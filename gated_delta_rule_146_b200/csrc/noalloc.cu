// noalloc.cu -- gdr_chunk_fwd_noalloc: the chunk-parallel forward with its scratch memory
// in a static device array instead of a caller-provided workspace.
//
// Some callers cannot allocate device memory for a workspace: a serving process whose GPU
// memory is reserved up front by its own pool (cudaMalloc there may fail, and it
// synchronises the device, stalling every other stream), code running inside a framework
// hook or callback where calling the CUDA allocator is not allowed, or a plain-C caller
// with no device allocator of its own.  This entry point needs nothing but the inputs and
// outputs: its scratch is one file-scope __device__ array of GDR_NOALLOC_SCRATCH_BYTES,
// which every GPU that loads this library holds until the process exits.
#include <cuda.h>

#include <mutex>

#include "common.cuh"

namespace gdr {
gdr_status chunk_args_status(const gdr_chunk_args* a);
}

namespace {

__device__ __align__(256) unsigned char g_noalloc_scratch[GDR_NOALLOC_SCRATCH_BYTES];

// Device address of the array, looked up with the device current and cached per device
// together with the CUDA context it was looked up in: a module's device symbols move when
// the device's primary context is destroyed and created again (cudaDeviceReset), so a new
// context means a new lookup.  In host code the name g_noalloc_scratch is only a host-side
// stand-in for the symbol, never a device address, so it is never passed to a kernel.
constexpr int kMaxDevices = 64;
struct Cached {
    CUcontext ctx;
    void* addr;
};
Cached g_scratch[kMaxDevices];
std::mutex g_scratch_mutex;

using CtxGetCurrentFn = CUresult (*)(CUcontext*);

// cuCtxGetCurrent through the runtime's driver entry point (no link against libcuda)
CUcontext current_context() {
    static CtxGetCurrentFn fn = nullptr;
    static bool looked = false;
    if (!looked) {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<CtxGetCurrentFn>(f);
        looked = true;
    }
    CUcontext c = nullptr;
    if (fn && fn(&c) != CUDA_SUCCESS) c = nullptr;
    return c;
}

gdr_status scratch_on_current_device(void** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return GDR_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return GDR_ERR_UNSUPPORTED;
    // (no context yet: the lookup below creates the device's primary context, and the
    // context is read again after it)
    const CUcontext ctx = current_context();
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    Cached& c = g_scratch[dev];
    if (!c.addr || !ctx || c.ctx != ctx) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return GDR_ERR_CUDA;
        c.addr = p;
        c.ctx = current_context();
    }
    *out = c.addr;
    return GDR_OK;
}

}  // namespace

extern "C" gdr_status gdr_chunk_fwd_noalloc(const gdr_chunk_args* args, const void* q,
                                            const void* k, const void* v, const void* g,
                                            const void* beta, const float* S0,
                                            const int32_t* cu_seqlens, void* o, float* S_final,
                                            void* stream) {
    // invalid arguments, or valid ones without a kernel path, are named as such
    const gdr_status ast = gdr::chunk_args_status(args);
    if (ast != GDR_OK) return ast;
    const size_t need = gdr_chunk_fwd_workspace_size(args);
    if (need > (size_t)GDR_NOALLOC_SCRATCH_BYTES) return GDR_ERR_WORKSPACE;
    void* scratch = nullptr;
    const gdr_status st = scratch_on_current_device(&scratch);
    if (st != GDR_OK) return st;
    // Every field of the scratch this call reads is written by the call itself first (the
    // chunk map and error word), so the previous call's contents need no clearing.
    return gdr_chunk_fwd(args, q, k, v, g, beta, S0, cu_seqlens, o, S_final, scratch,
                         (size_t)GDR_NOALLOC_SCRATCH_BYTES, stream);
}

extern "C" gdr_status gdr_noalloc_read_device_error(void* stream) {
    void* scratch = nullptr;
    const gdr_status st = scratch_on_current_device(&scratch);
    if (st != GDR_OK) return st;
    return gdr_read_device_error(nullptr, scratch, stream);
}
