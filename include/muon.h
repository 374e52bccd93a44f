/*
 * muon.h -- C ABI of the B200 (sm_100a) Muon / MONA optimizer step.
 *
 * The method (sources):
 *   [MONA]  "MONA - Muon-optimizer met Nesterov-versnelling" (gist.science,
 *           paper 2605.26842), section 2 "Methodologie: MONA", Kernalgoritme
 *           steps 1-4:
 *             D = G - G_prev;  A = beta_a A + (1 - beta_a) D;  Gt = G + alpha A;
 *             M = mu M + Gt;   O = Newton-Schulz(M);
 *             W = W - eta (gamma O + lambda W).
 *           "Ontwerprichtlijnen": the acceleration term is applied before the
 *           orthogonalisation, never after.
 *   [POLAR] quant_prune_distill post 677 (tgviewer.app): the Muon step
 *           substitutes the polar factor polar(X) = U V^T (X = U S V^T) of the
 *           momentum; it is found by Newton-Schulz.  Gram route:
 *           polar(X) = X (X^T X)^{-1/2} with the inverse square root also found
 *           by Newton-Schulz on the small Gram matrix, half of every symmetric
 *           product computed and mirrored, restarts, and a division by
 *           1.02-1.05 so that the eigenvalues stay inside [0, 1].
 *   [LiMuon] "LiMuon: Light and Fast Muon Optimizer for Large Models"
 *           (arxiv.sitesynth.xyz digest 2509.14562v1), section "Метод":
 *           Muon's momentum with the update taken from a randomized SVD
 *           (limuon_step_batched below).
 *
 * Iteration used by every entry point (readings of the pages, which name
 * Newton-Schulz but print no coefficients): on the wide view X (s x l,
 * s = min(rows, cols); a matrix with rows > cols is iterated transposed,
 * polar(X^T) = polar(X)^T) start from X0 = M / ((||M||_F + eps) f) and, for
 * k = 0 .. n_steps-1 with (a, b, c) = coeffs[k]:
 *     A = X X^T;   B = b A + c A A;   X = a X + B X
 * At every step k > 0 listed in `restarts` X is divided by f once more before
 * the step.  The Gram route evaluates the same polynomial through
 * R = X X^T:  h = a I + b R + c R^2,  Q <- h Q,  R <- h R h, and at a restart
 * k > 0: Xb <- Q Xb / f, R <- Xb Xb^T, Q <- I;  finally X = Q Xb.
 *
 * Conventions common to all entry points:
 *   - Every pointer named d_* or documented as "device" is CUDA device memory
 *     of the current device, owned by the caller.  Host arrays (schedule
 *     coefficients, restarts, parameter descriptors) are read during the call
 *     only and may be freed as soon as it returns.
 *   - The library allocates no memory.  Scratch space is the caller-provided
 *     `workspace` (device, >= the size returned by the matching *_size query,
 *     256-byte aligned).  Its contents need no initialisation and are
 *     clobbered.
 *   - Matrices are dense, row-major and contiguous (row stride = cols).
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and the call returns without synchronising.  Argument errors
 *     are returned before anything is enqueued.  Faults seen on the device
 *     (non-finite norm, a wait that ran out) are OR-ed into *d_status
 *     (MUON_FLAG_* bits) when d_status is not NULL; the caller reads it after
 *     synchronising.  d_status is never cleared by the library.
 *   - Calls that share a workspace must be ordered on the GPU (same stream,
 *     or events); concurrent calls on one workspace race.
 */
#ifndef MUON_B200_H
#define MUON_B200_H

#include <stddef.h>

#if defined(__GNUC__)
#define MUON_API __attribute__((visibility("default")))
#else
#define MUON_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same handle type as cudaStream_t / CUstream. */
typedef struct CUstream_st* muon_stream_t;

typedef enum {
    MUON_OK = 0,
    MUON_ERR_INVALID_ARG = 1,   /* NULL pointer, bad size, bad enum, bad schedule */
    MUON_ERR_UNSUPPORTED = 2,   /* valid request the library cannot run (no sm_100 device, shape limits) */
    MUON_ERR_WORKSPACE = 3,     /* workspace NULL, misaligned or smaller than the size query */
    MUON_ERR_NONFINITE = 4,     /* host-side name for MUON_FLAG_NONFINITE */
    MUON_ERR_CUDA = 5,          /* a CUDA runtime/driver call failed (see cudaGetLastError) */
    MUON_ERR_TIMEOUT = 6        /* host-side name for MUON_FLAG_TIMEOUT */
} muon_status;

/* Bits OR-ed into *d_status by the device. */
#define MUON_FLAG_NONFINITE 1   /* a matrix had a non-finite Frobenius norm; its W was left unchanged */
#define MUON_FLAG_TIMEOUT   2   /* a kernel's internal wait ran out (about 4 s); its output is invalid */

typedef enum {
    MUON_BF16 = 0,
    MUON_FP16 = 1,
    MUON_FP32 = 2
} muon_dtype;

/* One Newton-Schulz step X <- a X + (b A + c A^2) X. */
typedef struct {
    float a, b, c;
} muon_ns_coeff;

typedef struct {
    int n_steps;                 /* >= 1, <= 64 */
    const muon_ns_coeff* coeffs; /* host array of n_steps entries */
    float eps;                   /* added to ||M||_F before dividing; >= 0 (1e-7 is the usual choice) */
    const int* restarts;         /* host array of step indices (0 allowed, ignored); may be NULL if n_restarts == 0 */
    int n_restarts;              /* >= 0, <= 64 */
    float scale_f;               /* >= 1: extra divisor at the start and at every restart (1.02-1.05 on the Gram route) */
    float gram_aspect;           /* optimizer steps only: a shape group whose long side is at least gram_aspect
                                    times its short side runs the Gram route (with restarts and scale_f);
                                    0 keeps every group on the direct iteration.  >= 0.  ns_polar and
                                    gram_polar ignore it. */
} muon_schedule;

/* Hyper-parameters of [MONA] section 2. */
typedef struct {
    float mu;       /* momentum */
    float eta;      /* learning rate */
    float lambda;   /* decoupled weight decay */
    float gamma;    /* scale of the orthogonalised update */
    float beta_a;   /* EMA factor of the acceleration buffer */
    float alpha;    /* weight of the acceleration term */
} muon_hparams;

/* One matrix parameter and its optimizer state (all device memory). */
typedef struct {
    int rows, cols;    /* >= 1 */
    void* W;           /* rows x cols, w_dtype, updated in place */
    const void* G;     /* rows x cols, w_dtype, this step's gradient (read only) */
    void* G_prev;      /* rows x cols, w_dtype, previous gradient; receives G */
    float* A;          /* rows x cols, fp32 acceleration buffer, updated in place */
    float* M;          /* rows x cols, fp32 momentum, updated in place */
    float gamma;       /* per-matrix gamma; NaN means "use hparams.gamma" */
    float* O_out;      /* optional rows x cols fp32: receives O (the orthogonalised momentum); NULL to skip */
} muon_param;

/*
 * Bytes of workspace muon_step_batched needs for these parameters under this
 * schedule.  params: host array of n descriptors (only rows/cols are read).
 * sched: the schedule the step will use (its gram_aspect decides which shape
 * groups need the Gram route's larger workspace); NULL sizes every group for
 * the direct iteration.
 * Returns MUON_ERR_INVALID_ARG for n < 1, NULL pointers, non-positive sizes or
 * an invalid schedule.
 */
MUON_API muon_status muon_workspace_size(const muon_param* params, int n, muon_dtype ns_dtype,
                                const muon_schedule* sched, size_t* bytes);

/*
 * One optimizer step ([MONA] section 2, steps 1-4) for n matrix parameters.
 *   1. One fused pass over every element: A, M, G_prev updated in place as in
 *      steps 1-4, the Frobenius norm of the new M accumulated per matrix, and
 *      M written in ns_dtype (wide view) to the workspace.
 *   2. The iteration above on every matrix (matrices with the same
 *      (short side, long side) are batched together): the direct iteration,
 *      or the Gram route for the shape groups sched->gram_aspect selects
 *      ([POLAR]: elongated matrices iterate on their small s x s Gram
 *      matrix; in exact arithmetic both routes give the same O).  A matrix
 *      whose short side is below 16 is iterated in fp32 on CUDA cores
 *      whatever ns_dtype says (its 16-bit intermediates would cost accuracy
 *      for no measurable time).
 *   3. W <- W - eta (gamma O + lambda W), fused into the last iteration step;
 *      O never reaches memory unless O_out is given.
 * w_dtype: element type of W, G and G_prev (MUON_BF16, MUON_FP16 or MUON_FP32).
 * ns_dtype: arithmetic of the iteration: MUON_BF16 / MUON_FP16 (tensor cores,
 *   fp32 accumulation, 16-bit operands) or MUON_FP32 (CUDA-core fp32).
 * hp: host struct.  sched: host struct (restarts divide by scale_f as above).
 * A matrix whose norm is not finite keeps its W and sets MUON_FLAG_NONFINITE.
 * W, G, G_prev, A, M of one parameter may not overlap another parameter's.
 */
MUON_API muon_status muon_step_batched(const muon_param* params, int n, muon_dtype w_dtype,
                              muon_dtype ns_dtype, const muon_hparams* hp,
                              const muon_schedule* sched, void* workspace, size_t ws_bytes,
                              int* d_status, muon_stream_t stream);

/*
 * MONA-Lite ([MONA] section "Efficientie en Implementatie"): the auxiliary
 * state kept in bfloat16 and the gradient difference formed in place, without
 * a stored previous gradient.  One buffer per parameter replaces G_prev and A:
 *     B = beta_a A - (1 - beta_a) G      (of the previous step; 0 at the start)
 * so that step 2 reads A_k = B + (1 - beta_a) G_k, and after step 4
 *     B <- beta_a A_k - (1 - beta_a) G_k   (rounded to bfloat16, RNE).
 * Unrounded this is exactly steps 1-4; the state shrinks from G_prev + A to
 * one bfloat16 matrix and the fused pass from 24 to 16 bytes per element
 * (bf16 W/G, fp32 M, 16-bit copy).
 */
typedef struct {
    int rows, cols;    /* >= 1 */
    void* W;           /* rows x cols, w_dtype, updated in place */
    const void* G;     /* rows x cols, w_dtype, this step's gradient (read only) */
    void* B;           /* rows x cols, bfloat16 auxiliary buffer, updated in place (zero initially) */
    float* M;          /* rows x cols, fp32 momentum, updated in place */
    float gamma;       /* per-matrix gamma; NaN means "use hparams.gamma" */
    float* O_out;      /* optional rows x cols fp32: receives O; NULL to skip */
} muon_lite_param;

/* Bytes of workspace muon_lite_step_batched needs (only rows/cols are read;
 * sched as for muon_workspace_size). */
MUON_API muon_status muon_lite_workspace_size(const muon_lite_param* params, int n, muon_dtype ns_dtype,
                                     const muon_schedule* sched, size_t* bytes);

/*
 * One MONA-Lite optimizer step for n matrix parameters: the fused pass above
 * (B and M updated in place, the norm of the new M, its 16-bit wide view),
 * then the same iteration and fused weight update as muon_step_batched, with
 * the same arguments, errors and ownership rules (B takes the place of G_prev
 * and A).
 */
MUON_API muon_status muon_lite_step_batched(const muon_lite_param* params, int n, muon_dtype w_dtype,
                                   muon_dtype ns_dtype, const muon_hparams* hp,
                                   const muon_schedule* sched, void* workspace, size_t ws_bytes,
                                   int* d_status, muon_stream_t stream);

/*
 * AdamW for vector-valued parameters ([MONA] section 2, "Ontwerprichtlijnen":
 * embeddings and biases keep standard AdamW, as in Muon; the page gives no
 * formulas, read as Adam with bias correction and decoupled weight decay):
 *     m <- beta1 m + (1 - beta1) g          v <- beta2 v + (1 - beta2) g^2
 *     W <- W - lr ( (m / (1 - beta1^t)) / (sqrt(v / (1 - beta2^t)) + eps) + weight_decay W )
 * evaluated in fp32 per element.  One streaming launch per 128 parameters.
 */
typedef struct {
    long long n;       /* elements (>= 1); any shape, contiguous */
    void* W;           /* n elements, w_dtype, updated in place */
    const void* G;     /* n elements, w_dtype (read only) */
    float* m;          /* n fp32 first moments, updated in place (zero initially) */
    float* v;          /* n fp32 second moments, updated in place (zero initially) */
} muon_vec_param;

typedef struct {
    float lr, beta1, beta2, eps, weight_decay;   /* 0 <= beta < 1, eps >= 0 */
} muon_adamw_hparams;

/*
 * One AdamW step (t = step >= 1, the bias-correction count) on n vector
 * parameters, asynchronous on `stream`.  Argument errors return before any
 * launch (MUON_ERR_INVALID_ARG: NULL pointers, n < 1, step < 1, non-finite or
 * out-of-range hyper-parameters).  An element whose gradient is not finite
 * keeps its W, m and v, and MUON_FLAG_NONFINITE is OR-ed into *d_status
 * (when given).  No workspace.
 */
MUON_API muon_status adamw_step_batched(const muon_vec_param* params, int n, muon_dtype w_dtype,
                               const muon_adamw_hparams* hp, int step, int* d_status,
                               muon_stream_t stream);

/*
 * One optimizer step for a whole model: the n matrix parameters exactly as
 * muon_step_batched, and the nvec vector-valued parameters (embeddings,
 * biases, norm weights: [MONA] section 2, "Ontwerprichtlijnen") with AdamW
 * exactly as adamw_step_batched -- their elements are further work items of
 * the step's fused pre-pass launch, so the model needs no separate AdamW pass.
 * vecs: host array of nvec descriptors (NULL when nvec == 0); every W and G
 * of them in w_dtype, m and v fp32.  adamw, step: as adamw_step_batched
 * (ignored when nvec == 0).  workspace: muon_workspace_size of the matrix
 * parameters under `sched` (the vectors need none).  Errors, ownership and
 * asynchrony as muon_step_batched and adamw_step_batched; a vector element
 * with a non-finite gradient keeps its state and sets MUON_FLAG_NONFINITE.
 */
MUON_API muon_status muon_model_step(const muon_param* params, int n, const muon_vec_param* vecs, int nvec,
                                     muon_dtype w_dtype, muon_dtype ns_dtype, const muon_hparams* hp,
                                     const muon_adamw_hparams* adamw, int step, const muon_schedule* sched,
                                     void* workspace, size_t ws_bytes, int* d_status, muon_stream_t stream);

/*
 * LiMuon ([LiMuon] section "Метод": Muon's momentum, with the update taken
 * from a randomized SVD of the momentum).  The page gives no formulas; read
 * as the basic randomized SVD of Halko, Martinsson and Tropp ("Finding
 * structure with randomness", 2011) in place of the Newton-Schulz iteration:
 *     M <- mu M + G
 *     Y = M Omega,  Q = orth(Y),  B = Q^T M = U~ S V^T,  U = Q U~
 *     O = U_r V_r^T over the r = rank largest singular values
 *     W <- W - eta (gamma O + lambda W)
 * Omega (cols x k, k = rank + oversample <= 64) is the caller's test matrix:
 * the method draws it (Gaussian, fresh or fixed) and passes it in.  Singular
 * values at or below 1e-5 of the largest count as zero and are left out, so a
 * rank-deficient M gives a partial isometry and M = 0 gives O = 0.  Y, Q and
 * the products run in fp32; the k x k Gram, Cholesky and eigen steps in fp64.
 */
typedef struct {
    int rows, cols;       /* >= 1 */
    void* W;              /* rows x cols, w_dtype, updated in place */
    const void* G;        /* rows x cols, w_dtype, this step's gradient (read only) */
    float* M;             /* rows x cols, fp32 momentum, updated in place (zero initially) */
    const float* Omega;   /* cols x k fp32 test matrix, row-major, read only; parameters with the
                             same cols may share one */
    float gamma;          /* per-matrix gamma; NaN means "use hparams.gamma" */
    float* O_out;         /* optional rows x cols fp32: receives O; NULL to skip */
} muon_rsvd_param;

typedef struct {
    float mu, eta, lambda, gamma;
    int rank;             /* r >= 1 */
    int oversample;       /* p >= 0; k = r + p <= 64 (else MUON_ERR_UNSUPPORTED) */
} muon_rsvd_hparams;

/* Bytes of workspace limuon_step_batched needs (only rows/cols are read). */
MUON_API muon_status limuon_workspace_size(const muon_rsvd_param* params, int n, const muon_rsvd_hparams* hp,
                                           size_t* bytes);

/*
 * One LiMuon step for n matrix parameters, asynchronous on `stream`: five
 * launches per 128 parameters (fused momentum pass and sketch; per-matrix
 * QR; projection; per-matrix eigen-decomposition; O fused with the weight
 * update, O never stored unless O_out is given).  workspace: device,
 * 256-byte aligned, at least limuon_workspace_size bytes; no state is kept
 * in it between calls.  Argument errors return before any launch.  A matrix
 * whose new momentum holds a non-finite value keeps its W, and
 * MUON_FLAG_NONFINITE is OR-ed into *d_status (when given).  Parameters may
 * not overlap one another (Omega excepted, which is only read).
 */
MUON_API muon_status limuon_step_batched(const muon_rsvd_param* params, int n, muon_dtype w_dtype,
                                         const muon_rsvd_hparams* hp, void* workspace, size_t ws_bytes,
                                         int* d_status, muon_stream_t stream);

/*
 * Bytes of workspace ns_polar / gram_polar need for a batch of rows x cols
 * matrices in `dtype`.
 */
MUON_API muon_status ns_polar_workspace_size(int batch, int rows, int cols, muon_dtype dtype,
                                    size_t* bytes);
MUON_API muon_status gram_polar_workspace_size(int batch, int rows, int cols, muon_dtype dtype,
                                      size_t* bytes);

/*
 * Orthogonalise a batch of matrices with the direct iteration ([POLAR]
 * Newton-Schulz).  X_in: device, batch matrices of rows x cols in `dtype`,
 * matrix i at X_in + i * batch_stride elements (batch_stride >= rows*cols).
 * X_out: device, same layout and dtype; may equal X_in.
 * dtype MUON_BF16 / MUON_FP16 run on tensor cores, MUON_FP32 on CUDA cores.
 * A MUON_BF16 batch is iterated in fp16 ([POLAR]: fp16 is the recommended
 * type; bfloat16's 8 significant bits lose the small singular directions at
 * condition numbers near 1e3): one extra read of the input sums its squares,
 * and the copy the iteration starts from is X / (||X||_F + eps), which fp16
 * holds without overflow.  Input and output stay bfloat16.
 */
MUON_API muon_status ns_polar(const void* X_in, void* X_out, int batch, int rows, int cols,
                     long long batch_stride, muon_dtype dtype, const muon_schedule* sched,
                     void* workspace, size_t ws_bytes, int* d_status, muon_stream_t stream);

/*
 * The same result through the Gram route ([POLAR] X (X^T X)^{-1/2}): all
 * iteration steps work on s x s symmetric matrices (upper tiles computed and
 * mirrored); the s x l operand is touched only at the start, at restarts and
 * at the end.  Arguments as ns_polar; sched->restarts and sched->scale_f
 * select the restart steps and the divisor f.
 */
MUON_API muon_status gram_polar(const void* X_in, void* X_out, int batch, int rows, int cols,
                       long long batch_stride, muon_dtype dtype, const muon_schedule* sched,
                       void* workspace, size_t ws_bytes, int* d_status, muon_stream_t stream);

/*
 * ns_polar without a workspace argument, for callers that cannot allocate
 * device memory when they need the orthogonalisation: code running during CUDA
 * graph capture, runtimes whose allocators forbid outside allocations, and
 * plugins that only receive pointers to existing buffers.  The pages describe
 * no such entry point; it exists for this library's users.
 *
 * It runs exactly the ns_polar iteration with a fixed scratch array compiled
 * into the library: ns_polar_noalloc_capacity() bytes (32 MiB) of device
 * memory that every GPU loading the library keeps until the process exits.
 * A request whose ns_polar_workspace_size exceeds that capacity returns
 * MUON_ERR_WORKSPACE without launching anything.  Nothing is allocated: no
 * cudaMalloc, cudaFree or allocating library routine is called.
 *   - The first call on each device looks up the scratch array's device
 *     address (cudaGetSymbolAddress, with that device current); make that
 *     first call before any stream capture.  The address is remembered with
 *     the id of the CUDA context it was taken in and looked up again when a
 *     call finds a different context current (after cudaDeviceReset, say);
 *     such a call, too, should come before any capture.
 *   - All calls on a device share the scratch, which keeps the previous
 *     call's contents (each call clears what must start at zero).  Calls that
 *     overlap on the GPU (unordered streams) race: order them.
 * Arguments and results are those of ns_polar.
 */
MUON_API muon_status ns_polar_noalloc(const void* X_in, void* X_out, int batch, int rows, int cols,
                                      long long batch_stride, muon_dtype dtype,
                                      const muon_schedule* sched, int* d_status, muon_stream_t stream);
/* Bytes of the fixed scratch behind ns_polar_noalloc. */
MUON_API size_t ns_polar_noalloc_capacity(void);

/*
 * Tracing aid (optional).  While enabled, every kernel the library launches
 * is bracketed by two CUDA events recorded on the launch stream, and the
 * launch's algorithmic work is noted: floating-point operations for the
 * Newton-Schulz products (a symmetric product counts the half it needs,
 * n*n*k; a full product 2*m*n*k) or bytes moved for the elementwise pass.
 * Events come from a fixed host-side pool created on first use (up to
 * MUON_TRACE_CAPACITY launches; later launches are not recorded).
 * muon_trace_read synchronises on the recorded events, copies up to `max`
 * records (oldest first) to `out` (host array), clears the log and returns
 * the number of records copied (or -1 on a CUDA error).
 */
#define MUON_TRACE_CAPACITY 8192
typedef enum {
    MUON_KERNEL_PREPASS = 0,   /* fused MONA pre-pass / input copy + norms (work = bytes) */
    MUON_KERNEL_SYM = 1,       /* tcgen05 symmetric product X X^T, A A, ... (work = flops) */
    MUON_KERNEL_UPD = 2,       /* tcgen05 update product X <- aX + BX, Q Xb (work = flops) */
    MUON_KERNEL_SIMT = 3,      /* fp32 CUDA-core product (work = flops) */
    MUON_KERNEL_OTHER = 4,     /* identity fill (work = bytes) */
    MUON_KERNEL_ADAMW = 5,     /* AdamW streaming pass over vector parameters (work = bytes) */
    MUON_KERNEL_RSVD = 6,      /* LiMuon streaming passes: momentum + sketch, projection, update (work = bytes) */
    MUON_KERNEL_RSVD_SMALL = 7 /* LiMuon per-matrix factorisations: QR, eigen-decomposition (work = bytes) */
} muon_kernel_kind;

typedef struct {
    int kind;        /* muon_kernel_kind */
    double work;     /* algorithmic flops or bytes of this launch */
    float ms;        /* device time between the bracketing events */
} muon_trace_record;

MUON_API muon_status muon_trace_enable(int enable);
MUON_API int muon_trace_read(muon_trace_record* out, int max);

/*
 * Self-test of the failure path: one block runs the library's bounded wait
 * on a barrier that nothing completes, with a limit of wait_ms milliseconds
 * (1..4000); the wait gives up, ORs MUON_FLAG_TIMEOUT into *d_status (device,
 * required) and the kernel returns normally.  No pages' counterpart: it lets a
 * caller check that a stuck wait ends in a status word, not a hung GPU.
 */
MUON_API muon_status muon_wait_selftest(int wait_ms, int* d_status, muon_stream_t stream);

/* Static, NUL-terminated description of a status code. */
MUON_API const char* muon_status_string(muon_status status);

#ifdef __cplusplus
}
#endif

#endif /* MUON_B200_H */
