// gemm_simt.cu -- fp32 CUDA-core GEMMs for the fp32 Newton-Schulz path.
//
// The tensor cores have no plain-fp32 multiply (tf32 keeps 10 mantissa bits),
// so the fp32 iteration runs on the CUDA cores: 64 x 64 output tiles, 256
// threads each computing 4 x 4 outputs from 16-deep shared-memory slices.
// Same problem shapes and epilogues as the tensor-core path (see gemm.h):
// symmetric products compute the upper tiles only and mirror them.
#include "epilogue.cuh"
#include "gemm.h"

namespace muon {
namespace simt {

constexpr int TB = 64;
constexpr int TK = 16;

struct SimtParams {
    GemmOp op;
    int tiles_m, tiles_n;
    FinalCtx fc;
    FinalEntry fin[kMaxFinal];
};

__global__ void __launch_bounds__(256) simt_gemm_kernel(const __grid_constant__ SimtParams p) {
    __shared__ float As[TK][TB + 4];
    __shared__ float Bs[TK][TB + 4];
    const GemmOp& o = p.op;
    const int m = blockIdx.y;
    int r = blockIdx.x, ti, tj;
    if (o.sym) {
        int nt = p.tiles_m, i = 0;
        while (r >= nt - i) { r -= nt - i; ++i; }
        ti = i;
        tj = i + r;
    } else {
        ti = r % p.tiles_m;
        tj = r / p.tiles_m;
    }
    const float* A = static_cast<const float*>(o.A) + (size_t)m * o.strideA;
    const float* B = static_cast<const float*>(o.B) + (size_t)m * o.strideB;
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    float acc[4][4] = {};
    for (int k0 = 0; k0 < o.K; k0 += TK) {
        for (int e = threadIdx.x; e < TB * TK; e += 256) {
            int rr = e / TK, kk = e % TK;
            int gr = ti * TB + rr, gk = k0 + kk;
            As[kk][rr] = (gr < o.M && gk < o.K) ? A[(size_t)gr * o.lda + gk] : 0.f;
            if (o.sym) {
                int gn = tj * TB + rr;
                Bs[kk][rr] = (gn < o.N && gk < o.K) ? B[(size_t)gn * o.ldb + gk] : 0.f;
            } else {
                int kk2 = e / TB, nn = e % TB;
                int gk2 = k0 + kk2, gn = tj * TB + nn;
                Bs[kk2][nn] = (gn < o.N && gk2 < o.K) ? B[(size_t)gk2 * o.ldb + gn] : 0.f;
            }
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < TK; ++kk) {
            float a[4], b[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = As[kk][ty + 16 * i];
#pragma unroll
            for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx + 16 * j];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        }
        __syncthreads();
    }

    const Epilogue& E = o.epi;
    const float sc = epi_scale(E, m);
    if (E.fin != FIN_STORE && !epi_finite(E, m, sc)) {
        if (threadIdx.x == 0 && ti == 0 && tj == 0 && p.fc.d_status)
            atomicOr(p.fc.d_status, MUON_FLAG_NONFINITE);
        if (E.fin == FIN_WUPD) return;
    }
    FinalCtx fc = p.fc;
    fc.fin = p.fin;
    const float* Cin = static_cast<const float*>(E.Cin) + (size_t)m * E.strideC;
    float* D = static_cast<float*>(E.D) + (size_t)m * E.strideD;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int gi = ti * TB + ty + 16 * i;
        if (gi >= o.M) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int gj = tj * TB + tx + 16 * j;
            if (gj >= o.N) continue;
            float v = E.alpha * acc[i][j];
            if (E.beta != 0.f) v += E.beta * Cin[(size_t)gi * E.ldc + gj];
            v *= sc;
            if (gi == gj) v += E.diag;
            if (E.fin == FIN_STORE) {
                if (!o.sym) {
                    D[(size_t)gi * E.ldd + gj] = v;
                } else if (gj >= gi) {
                    D[(size_t)gi * E.ldd + gj] = v;
                    if (gj > gi) D[(size_t)gj * E.ldd + gi] = v;
                }
            } else {
                epi_final_elem(E, fc, m, o.M, o.N, gi, gj, v);
            }
        }
    }
}

muon_status simt_run(const GemmOp* ops, int nops, const FinalCtx& fc, const FinalEntry* fin, int nfin,
                     cudaStream_t stream) {
    if (nfin > kMaxFinal) return MUON_ERR_UNSUPPORTED;
    for (int i = 0; i < nops; ++i) {
        SimtParams prm;
        memset(&prm, 0, sizeof(prm));
        prm.op = ops[i];
        prm.tiles_m = (ops[i].M + TB - 1) / TB;
        prm.tiles_n = (ops[i].N + TB - 1) / TB;
        prm.fc = fc;
        prm.fc.fin = nullptr;
        for (int f = 0; f < nfin; ++f) prm.fin[f] = fin[f];
        const int tiles = ops[i].sym ? prm.tiles_m * (prm.tiles_m + 1) / 2 : prm.tiles_m * prm.tiles_n;
        if (ops[i].count > 65535) return MUON_ERR_UNSUPPORTED;
        dim3 grid(tiles, ops[i].count);
        const GemmOp& o = ops[i];
        trace_begin(MUON_KERNEL_SIMT,
                    o.sym ? (double)o.count * o.N * o.N * o.K : 2.0 * o.count * o.M * o.N * o.K, stream);
        simt_gemm_kernel<<<grid, 256, 0, stream>>>(prm);
        trace_end(stream);
        if (cudaGetLastError() != cudaSuccess) return MUON_ERR_CUDA;
    }
    return MUON_OK;
}

}  // namespace simt
}  // namespace muon
