// noalloc.cu -- ns_polar for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc at the point where they need the
// orthogonalisation: code running while a CUDA graph is being captured (an
// allocation there is not part of the graph), allocators or runtimes that
// forbid allocations outside their own pool, and plugins or callbacks that
// only receive pointers to existing buffers.  ns_polar asks those callers for
// a workspace they may be unable to provide; ns_polar_noalloc instead uses a
// fixed scratch array compiled into this library.
//
// The scratch is a file-scope device array of kScratchBytes (32 MiB).  Every
// GPU that loads the library holds it until the process exits.  All calls on
// a device share it and it keeps the previous call's contents: whatever the
// iteration needs to start at zero (the per-matrix sums of squares) is
// cleared by each call, and two calls that overlap on the GPU (different
// streams without ordering between them) race on the same memory.
#include <cuda.h>

#include <mutex>

#include "gemm.h"

namespace {

constexpr size_t kScratchBytes = size_t(32) << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

// Device address of g_scratch per device, valid for one CUDA context: in host
// code the array's name is only a stand-in, not an address the GPU can use,
// and a context that is destroyed and created again (cudaDeviceReset, or the
// primary context released and retained) reloads this module, so the array
// may move.  The address is therefore cached together with the unique id of
// the context it was taken in and looked up again when the current context's
// id differs.
struct ScratchSlot {
    unsigned long long ctx_id;
    void* ptr;
};
ScratchSlot g_slot[kMaxDevices] = {};
std::mutex g_scratch_mu;

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// Driver entry points (the library links no driver library directly).
template <typename Fn>
Fn driver_fn(const char* name) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion(name, &p, 12000, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
        return nullptr;
    return reinterpret_cast<Fn>(p);
}

muon_status current_context_id(unsigned long long* id) {
    static const CtxGetCurrentFn get_current = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
    static const CtxGetIdFn get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
    if (!get_current || !get_id) return MUON_ERR_CUDA;
    CUcontext ctx = nullptr;
    if (get_current(&ctx) != CUDA_SUCCESS || !ctx) return MUON_ERR_CUDA;
    return get_id(ctx, id) == CUDA_SUCCESS ? MUON_OK : MUON_ERR_CUDA;
}

muon_status scratch_for_current_device(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MUON_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return MUON_ERR_UNSUPPORTED;
    unsigned long long id = 0;
    const bool have_id = current_context_id(&id) == MUON_OK;   // false before the context exists
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    ScratchSlot& slot = g_slot[dev];
    if (!have_id || !slot.ptr || slot.ctx_id != id) {
        // the lookup also creates the device's context if there is none yet
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || !p) return MUON_ERR_CUDA;
        muon_status st = current_context_id(&id);
        if (st != MUON_OK) return st;
        slot.ptr = p;
        slot.ctx_id = id;
    }
    *out = slot.ptr;
    return MUON_OK;
}

}  // namespace

extern "C" {

muon_status ns_polar_noalloc(const void* X_in, void* X_out, int batch, int rows, int cols,
                             long long batch_stride, muon_dtype dtype, const muon_schedule* sched,
                             int* d_status, muon_stream_t stream) {
    size_t need = 0;
    muon_status st = ns_polar_workspace_size(batch, rows, cols, dtype, &need);
    if (st != MUON_OK) return st;
    if (need > kScratchBytes) return MUON_ERR_WORKSPACE;   // larger than the fixed scratch
    void* scratch = nullptr;
    st = scratch_for_current_device(&scratch);
    if (st != MUON_OK) return st;
    return ns_polar(X_in, X_out, batch, rows, cols, batch_stride, dtype, sched, scratch, kScratchBytes,
                    d_status, stream);
}

size_t ns_polar_noalloc_capacity(void) { return kScratchBytes; }

}  // extern "C"
