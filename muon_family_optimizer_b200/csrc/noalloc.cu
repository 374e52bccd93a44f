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
#include <mutex>

#include "gemm.h"

namespace {

constexpr size_t kScratchBytes = size_t(32) << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

// Device address of g_scratch per device (in host code the array's name is
// only a stand-in, not an address the GPU can use).
void* g_scratch_ptr[kMaxDevices] = {};
std::mutex g_scratch_mu;

muon_status scratch_for_current_device(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MUON_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return MUON_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || !p) return MUON_ERR_CUDA;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
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
