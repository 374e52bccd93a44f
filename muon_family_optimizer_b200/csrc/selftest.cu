// selftest.cu -- exercise the library's bounded waits without a GPU fault.
//
// Every spin in the kernels (an mbarrier wait for a copy, an accumulator or a
// tile) gives up after a limit, records MUON_FLAG_TIMEOUT in the caller's
// status word and lets the kernel wind down.  This entry point runs that same
// wait (mbar_wait) on a barrier nothing will ever complete, with a short
// limit, so the failure path can be tested: the kernel returns normally and
// the context stays usable.
#include "gemm.h"

namespace muon {
namespace {

__global__ void wait_selftest_kernel(unsigned long long limit_ns, int* d_status) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        // no thread arrives on `bar`: the wait for its first phase runs out
        (void)mbar_wait(&bar, 0, reinterpret_cast<volatile int*>(&abort_flag), d_status, limit_ns);
    }
    __syncthreads();
}

}  // namespace
}  // namespace muon

extern "C" muon_status muon_wait_selftest(int wait_ms, int* d_status, muon_stream_t stream) {
    if (!d_status || wait_ms < 1 || wait_ms > 4000) return MUON_ERR_INVALID_ARG;
    muon::wait_selftest_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        (unsigned long long)wait_ms * 1000000ull, d_status);
    return cudaGetLastError() == cudaSuccess ? MUON_OK : MUON_ERR_CUDA;
}
