// adamw.cu -- AdamW for vector-valued parameters (embeddings, biases).
//
// [MONA] section 2, "Ontwerprichtlijnen": vector-valued parameters keep the
// standard AdamW of Muon's convention.  Read as Adam with bias correction and
// decoupled weight decay, per element in fp32:
//     m <- b1 m + (1 - b1) g,   v <- b2 v + (1 - b2) g^2
//     W <- W - lr ( (m / (1 - b1^t)) / (sqrt(v / (1 - b2^t)) + eps) + wd W )
//
// A streaming pass: 22 bytes per element for bf16 W/G (read W 2, G 2, m 4,
// v 4; write W 2, m 4, v 4).  The parameters of one launch (up to 128) form
// one element space cut into runs of 2048 consecutive elements; 256 threads
// each take 8 consecutive elements of a run (16-byte accesses of 16-bit data,
// two of fp32), every load of a run issued before any use.  Blocks own
// contiguous ranges of runs (one wave of resident blocks).
#include <algorithm>
#include <cmath>
#include <cstring>
#include <mutex>

#include "adamw_elem.cuh"
#include "gemm.h"

namespace muon {

namespace {

constexpr int kRun = 2048;
constexpr int kMaxVec = 128;

struct VecEntry {
    void* W;
    const void* G;
    float* m;
    float* v;
    long long n, run_begin, runs;
    int vec_ok;
};

struct AdamWParams {
    VecEntry e[kMaxVec];
    int n;
    long long total_runs;
    AdamWCoeffs c;
    int* d_status;
};

template <int W_DT>
__global__ void __launch_bounds__(256, 4) adamw_kernel(const __grid_constant__ AdamWParams p) {
    const long long per = (p.total_runs + gridDim.x - 1) / gridDim.x;
    const long long r_begin = (long long)blockIdx.x * per;
    const long long r_end = min(p.total_runs, r_begin + per);
    int ei = 0;
    bool bad = false;
    for (long long r = r_begin; r < r_end; ++r) {
        while (ei + 1 < p.n && r >= p.e[ei + 1].run_begin) ++ei;
        const VecEntry& E = p.e[ei];
        const long long idx = (r - E.run_begin) * kRun + (long long)threadIdx.x * 8;
        const int nvalid = (int)max(0LL, min(8LL, E.n - idx));
        if (nvalid == 0) continue;
        const bool vec = E.vec_ok && nvalid == 8;
        float w[8], g[8], m[8], v[8];
        load8_dt(E.W, idx, W_DT, vec, nvalid, w);
        load8_dt(E.G, idx, W_DT, vec, nvalid, g);
        load8_dt(E.m, idx, DT_FP32, vec, nvalid, m);
        load8_dt(E.v, idx, DT_FP32, vec, nvalid, v);
        bad |= adamw8(p.c, w, g, m, v, nvalid);
        store8_dt(E.W, idx, W_DT, vec, nvalid, w);
        store8_dt(E.m, idx, DT_FP32, vec, nvalid, m);
        store8_dt(E.v, idx, DT_FP32, vec, nvalid, v);
    }
    if (__syncthreads_or(bad) && threadIdx.x == 0 && p.d_status) atomicOr(p.d_status, MUON_FLAG_NONFINITE);
}

muon_status launch_adamw(AdamWParams& prm, int w_dtype, cudaStream_t stream) {
    long long runs = 0;
    double elems = 0.0;
    for (int i = 0; i < prm.n; ++i) {
        prm.e[i].run_begin = runs;
        prm.e[i].runs = (prm.e[i].n + kRun - 1) / kRun;
        runs += prm.e[i].runs;
        elems += (double)prm.e[i].n;
    }
    prm.total_runs = runs;
    int dev = 0, nsm = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    static int occ = 0;
    if (occ <= 0 && (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, adamw_kernel<DT_BF16>, 256, 0) !=
                         cudaSuccess || occ <= 0))
        occ = 1;
    const long long want = (long long)nsm * occ;
    const int grid = (int)(runs < want ? runs : want);
    const double wsz = dt_size(w_dtype);
    trace_begin(MUON_KERNEL_ADAMW, elems * (3.0 * wsz + 16.0), stream);
    if (w_dtype == DT_BF16) adamw_kernel<DT_BF16><<<grid, 256, 0, stream>>>(prm);
    else if (w_dtype == DT_FP16) adamw_kernel<DT_FP16><<<grid, 256, 0, stream>>>(prm);
    else adamw_kernel<DT_FP32><<<grid, 256, 0, stream>>>(prm);
    trace_end(stream);
    return cudaGetLastError() == cudaSuccess ? MUON_OK : MUON_ERR_CUDA;
}

}  // namespace
}  // namespace muon

using namespace muon;

namespace muon {

muon_status adamw_check(const muon_vec_param* params, int n, const muon_adamw_hparams* hp, int step) {
    if (!params || n < 1 || !hp || step < 1) return MUON_ERR_INVALID_ARG;
    const float hv[5] = {hp->lr, hp->beta1, hp->beta2, hp->eps, hp->weight_decay};
    for (float x : hv)
        if (!std::isfinite(x)) return MUON_ERR_INVALID_ARG;
    if (hp->beta1 < 0.f || hp->beta1 >= 1.f || hp->beta2 < 0.f || hp->beta2 >= 1.f || hp->eps < 0.f)
        return MUON_ERR_INVALID_ARG;
    for (int i = 0; i < n; ++i) {
        const muon_vec_param& q = params[i];
        if (q.n < 1 || !q.W || !q.G || !q.m || !q.v) return MUON_ERR_INVALID_ARG;
        if (q.n > (1LL << 40)) return MUON_ERR_UNSUPPORTED;
    }
    return MUON_OK;
}

AdamWCoeffs adamw_coeffs(const muon_adamw_hparams* hp, int step) {
    AdamWCoeffs c;
    c.lr = hp->lr; c.b1 = hp->beta1; c.b2 = hp->beta2; c.eps = hp->eps; c.wd = hp->weight_decay;
    c.ic1 = (float)(1.0 / (1.0 - std::pow((double)hp->beta1, (double)step)));
    c.ic2 = (float)(1.0 / (1.0 - std::pow((double)hp->beta2, (double)step)));
    return c;
}

}  // namespace muon

extern "C" {

muon_status adamw_step_batched(const muon_vec_param* params, int n, muon_dtype w_dtype, const muon_adamw_hparams* hp,
                               int step, int* d_status, muon_stream_t stream) {
    if (w_dtype != MUON_BF16 && w_dtype != MUON_FP16 && w_dtype != MUON_FP32) return MUON_ERR_INVALID_ARG;
    muon_status chk = adamw_check(params, n, hp, step);
    if (chk != MUON_OK) return chk;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    static AdamWParams prm;            // large: kept off the stack, filled and consumed per launch
    static std::mutex mu;
    std::lock_guard<std::mutex> lock(mu);
    for (int b = 0; b < n; b += kMaxVec) {
        memset(&prm, 0, sizeof(prm));
        prm.n = std::min(kMaxVec, n - b);
        prm.c = adamw_coeffs(hp, step);
        prm.d_status = d_status;
        for (int i = 0; i < prm.n; ++i) {
            const muon_vec_param& q = params[b + i];
            VecEntry& E = prm.e[i];
            E.W = q.W; E.G = q.G; E.m = q.m; E.v = q.v; E.n = q.n;
            const uintptr_t al = reinterpret_cast<uintptr_t>(q.W) | reinterpret_cast<uintptr_t>(q.G) |
                                 reinterpret_cast<uintptr_t>(q.m) | reinterpret_cast<uintptr_t>(q.v);
            E.vec_ok = (al & 15) == 0;
        }
        muon_status st = launch_adamw(prm, w_dtype, s);
        if (st != MUON_OK) return st;
    }
    return MUON_OK;
}

}  // extern "C"
