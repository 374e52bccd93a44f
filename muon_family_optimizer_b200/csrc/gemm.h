// gemm.h -- host-side description of one batched GEMM problem of the
// Newton-Schulz iteration and the two back ends that run it.
#pragma once

#include "adamw_elem.cuh"
#include "epilogue.cuh"

namespace muon {

// D = A B^T (sym = 1: B given as N x K rows, result symmetric, upper tiles
// computed and mirrored) or D = A B (sym = 0: B given as K x N row-major),
// for `count` matrices; strides and leading dimensions in elements.
struct GemmOp {
    int sym;
    // Operand stored as a symmetric matrix of which only the tiles on or above
    // the diagonal (128 x 128) are valid (tensor-core path): blocks left of the
    // diagonal tile are read transposed from the stored upper tile.
    int a_sym, b_sym;
    // Symmetric result that an update product will read on CTA pairs: also
    // store the first tile below the diagonal (exact mirror of the one above).
    int band;
    // Operand stored transposed in full (tensor-core path; a matrix copied in
    // its parameter's orientation, K x M instead of M x K): SYM A (a_tr) / B
    // (b_tr) are read as MN-major tiles; UPD B (b_tr: N x K, K contiguous) as
    // K-major tiles.
    int a_tr, b_tr;
    int count, M, N, K;
    const void* A; long long lda, strideA;
    const void* B; long long ldb, strideB;
    Epilogue epi;
};

namespace tc {
// tcgen05 back end for 16-bit operands (dt = DT_BF16 or DT_FP16); all ops of
// one call must have the same `sym` and are run by one launch.
muon_status tc_run(const GemmOp* ops, int nops, int dt, const FinalCtx& fc, const FinalEntry* fin,
                   int nfin, cudaStream_t stream);
}
namespace simt {
// CUDA-core fp32 back end (dt = DT_FP32): one launch per op.
muon_status simt_run(const GemmOp* ops, int nops, const FinalCtx& fc, const FinalEntry* fin, int nfin,
                     cudaStream_t stream);
}

// Fused elementwise passes ahead of the iteration (prepass.cu).
constexpr int kMaxPrep = 192;

struct PrepEntry {
    const void* G; void* Gp; float* A; float* M;   // MONA mode: this parameter's state
                                                   // (AdamW item: G the gradient, Gp the weights W,
                                                   //  A the first moment m, M the second moment v)
    const void* X; long long x_stride;             // COPY mode: batch input
    void* X0; long long x0_stride, ld;             // wide-view destination
    int rows, cols, count, transposed, vec_ok;
    int sumsq_index;
    int tiles_c;
    int flat;          // set by prep_run: processed as one contiguous array
    int kind;          // 0: a matrix of the launch's mode; 1: an AdamW vector item of nel elements
    long long nel;
    long long tiles_per_mat, tile_begin;
};

struct PrepParams {
    PrepEntry e[kMaxPrep];
    int n;
    long long total_tiles;
    int in_dt, x0_dt, mode;   // mode 0 = MONA pre-pass, 1 = copy (normalisation input of ns/gram_polar),
                              // 2 = MONA-Lite (Gp holds the bfloat16 buffer B, A unused),
                              // 3 = norm only (sums of squares of the batch input, nothing stored)
    int prescale;             // copy mode after a norm pass: store X / (||X|| + eps), sums left as they are
    float eps;
    float beta_a, alpha, mu;
    double* sumsq;
    // AdamW items (kind 1), after every matrix entry of the launch
    AdamWCoeffs adam;
    int* d_status;
};

muon_status prep_run(PrepParams& prm, cudaStream_t stream);

// AdamW host helpers (adamw.cu): argument checks and the launch's coefficients.
muon_status adamw_check(const muon_vec_param* params, int n, const muon_adamw_hparams* hp, int step);
AdamWCoeffs adamw_coeffs(const muon_adamw_hparams* hp, int step);

// Launch tracing (trace.cu): no-ops unless muon_trace_enable(1) was called.
void trace_begin(int kind, double work, cudaStream_t stream);
void trace_end(cudaStream_t stream);

// Small helpers (prepass.cu)
muon_status fill_identity(void* D, int dt, int count, int s, long long ld, long long stride,
                          cudaStream_t stream);

}  // namespace muon
