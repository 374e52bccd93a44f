// epilogue.cuh -- per-element epilogue shared by the tensor-core and the
// CUDA-core GEMM kernels (see the Epilogue descriptor in muon_internal.cuh).
#pragma once

#include "muon_internal.cuh"

namespace muon {

// Launch-wide data the final epilogues need.
struct FinalCtx {
    int w_dt;            // FIN_WUPD: element type of W
    int out_dt;          // FIN_OUT: element type of the output
    void* out;           // FIN_OUT: base of the output batch
    long long out_stride;
    int out_transposed;  // FIN_OUT: 1 when the user matrix is the transpose of the wide view
    int out_vec;         // FIN_OUT: 16-byte accesses allowed (aligned, cols % 8 == 0)
    float eta, lambda;
    int* d_status;
    const FinalEntry* fin;   // FIN_WUPD table (device-visible: kernel parameter space)
};

// Scale of matrix m: sc_mul * (sqrt(sumsq[m]) + eps)^(-sc_pow).
__device__ __forceinline__ float epi_scale(const Epilogue& E, int m) {
    float sc = E.sc_mul;
    if (E.sumsq != nullptr && E.sc_pow > 0) {
        double n = sqrt(E.sumsq[m]);
        double r = 1.0 / (n + (double)E.eps);
        sc = (float)((double)sc * (E.sc_pow == 1 ? r : r * r));
    }
    return sc;
}

// False when matrix m's norm is not finite (final steps only).
__device__ __forceinline__ bool epi_finite(const Epilogue& E, int m, float sc) {
    return isfinite(sc) && (E.check == nullptr || isfinite(E.check[m]));
}

// Index of wide-view element (i, j) (0 <= i < s, 0 <= j < l) in a user
// matrix that is either the wide view itself (s x l) or its transpose (l x s).
__device__ __forceinline__ long long user_index(int i, int j, int s, int l, int transposed) {
    return transposed ? (long long)j * s + i : (long long)i * l + j;
}

// Final epilogue for one element (FIN_OUT or FIN_WUPD); `v` is the output of
// the last iteration step at wide-view position (i, j) of matrix m.
__device__ __forceinline__ void epi_final_elem(const Epilogue& E, const FinalCtx& F, int m,
                                               int s, int l, int i, int j, float v) {
    if (E.fin == FIN_OUT) {
        void* base = static_cast<char*>(F.out) + (size_t)m * F.out_stride * dt_size(F.out_dt);
        st_elem(base, user_index(i, j, s, l, F.out_transposed), F.out_dt, v);
    } else {
        const FinalEntry& fe = F.fin[E.fin_base + m];
        long long idx = user_index(i, j, s, l, fe.transposed);
        float w = ld_elem(fe.W, idx, F.w_dt);
        w = w - F.eta * (fe.gamma * v + F.lambda * w);
        st_elem(fe.W, idx, F.w_dt, w);
        if (fe.O_out) fe.O_out[idx] = v;
    }
}

}  // namespace muon
