// limuon.cu -- LiMuon step: momentum, then a randomized truncated SVD of the
// momentum in place of the Newton-Schulz orthogonalisation.
//
// [LiMuon] section "Метод": LiMuon keeps Muon's momentum and computes its
// update from a randomized SVD.  Read as the basic randomized SVD of Halko,
// Martinsson and Tropp ("Finding structure with randomness", 2011):
//     M <- mu M + G
//     Y = M Omega (Omega: cols x k Gaussian test matrix, given), Q = orth(Y)
//     B = Q^T M = U~ S V^T,  O = (Q U~)_r V_r^T over the r largest S
//     W <- W - eta (gamma O + lambda W)
// Singular values at or below 1e-5 of the largest count as zero.
//
// With C = B B^T = E L E^T (so U~ = E, S^2 = L) and V_r^T = L_r^{-1/2} E_r^T B:
//     O = Q P B,   P = E_r L_r^{-1/2} E_r^T      (k x k)
// and Q = Y R^-1 with Y^T Y = R^T R (Cholesky QR).  Every pass over an l x s
// array streams; everything per matrix touches only k x k data:
//   1 lim_sketch   M <- mu M + G and Y = M Omega, 64-row blocks over 64-column
//                  chunks double-buffered in shared memory (cp.async), the
//                  product on tensor cores (tf32 x 3, fp32 accuracy); each
//                  block adds its rows' share of the Gram Y^T Y (fp64) to the
//                  matrix's k x k sum.  Reads G and M, writes M.
//   2 lim_chol     per matrix (k x k): Cholesky of Y^T Y in fp64 (a column whose
//                  pivot falls to 1e-10 of its squared norm lies in the span of
//                  the previous ones and is dropped: its Q column is zero), R^-1.
//   3 lim_rowmul   Q = Y R^-1, row by row in place (fp64 sums), all matrices'
//                  rows in one grid.
//   4 lim_project  B^T = M^T Q, 128-column blocks over 32-row chunks (three
//                  cp.async stages), tensor cores as in 1; each block adds its
//                  columns' share of B B^T (fp64) to the matrix's k x k sum.
//                  Reads M.
//   5 lim_eig      per matrix (k x k): cyclic Jacobi on B B^T in fp64,
//                  round-robin order (k/2 disjoint rotations per round), a
//                  rotation only while |C_pq| > 1e-15 sqrt(C_pp C_qq) (and
//                  above 1e-16 of the trace: fp64 noise), stop after a sweep
//                  without one; P from the r largest eigenpairs.
//   6 lim_rowmul   Z = Q P in place.
//   7 lim_update   O = Z B on 128 x 128 tiles (tensor cores as in 1), fused
//                  with the weight update (reads and writes W; O never stored
//                  unless O_out is given).
// The sketch and the projection order their blocks longest first.
// A non-finite momentum element or k x k factor marks its matrix: its W is
// kept and MUON_FLAG_NONFINITE raised.
#include <algorithm>
#include <cmath>
#include <cstring>
#include <mutex>
#include <type_traits>

#include "gemm.h"

namespace muon {

namespace {

constexpr int kLimMax = 128;      // matrices per launch
constexpr int kThreads = 256;
constexpr int kSmallThreads = 64; // per-matrix k x k kernels
constexpr int kSkRows = 64;       // lim_sketch: rows per block
constexpr int kSkCols = 64;       // lim_sketch: columns per chunk (two stages)
constexpr int kSkLd = kSkCols + 4;   // padded row of a staged M chunk
constexpr int kPjCols = 128;      // lim_project: columns per block
constexpr int kPjRows = 32;       // lim_project: rows per chunk
constexpr int kPjStages = 3;
constexpr int kUpRows = 128;      // lim_update: tile rows
constexpr int kUpCols = 128;      // lim_update: tile columns
constexpr double kDrop = 1e-10;   // Cholesky pivot / squared column norm below which a column is dropped
constexpr double kTau2 = 1e-10;   // (singular value / largest)^2 at or below which it counts as zero
constexpr double kRotTol = 1e-15; // Jacobi: rotate while |C_pq| > kRotTol sqrt(C_pp C_qq)
constexpr int kMaxSweeps = 30;
constexpr int kMaxDevices = 64;    // devices whose kernel attributes are tracked

struct LimEntry {
    void* W; const void* G; float* M; const float* Omega; float* O_out;
    float* Y;        // rows x KT workspace: Y, then Q, then Z (in place)
    float* Bt;       // cols x KT workspace: B^T
    double* Gy;      // KT x KT: Y^T Y, upper triangle summed by lim_sketch (zeroed per call)
    double* Cg;      // KT x KT: B B^T, upper triangle summed by lim_project (zeroed per call)
    double* K;       // KT x KT: R^-1 (lim_chol), then P (lim_eig)
    int* bad;        // this matrix's non-finite flag (workspace, zeroed per call)
    int rows, cols;
    float gamma;
    int vec_ok;      // W, G, M, O_out 16-byte aligned and cols % 8 == 0
    int t_sketch, t_rows, t_proj, t_upd;   // first block of this matrix in each launch's grid
};

struct LimParams {
    LimEntry e[kLimMax];
    // order of the matrices in each launch's grid (which: 0 sketch, 1 row
    // transforms, 2 projection, 3 update): the sketch and the projection give
    // the matrices with the longest blocks (most columns, most rows) the first
    // blocks, so no long block starts in the last wave
    unsigned char ord[4][kLimMax];
    int n, k, r;
    float mu, eta, lambda;
    int* d_status;
};

__device__ __forceinline__ int first_block(const LimEntry& e, int which) {
    return which == 0 ? e.t_sketch : which == 1 ? e.t_rows : which == 2 ? e.t_proj : e.t_upd;
}

// The matrix that block b of a launch works on: in the launch's order, the
// last matrix whose first block is <= b.
__device__ __forceinline__ int find_entry(const LimParams& p, int b, int which) {
    int lo = 0, hi = p.n - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (first_block(p.e[p.ord[which][mid]], which) <= b) lo = mid; else hi = mid - 1;
    }
    return p.ord[which][lo];
}

__device__ __forceinline__ void mark_bad(const LimParams& p, const LimEntry& E) {
    atomicOr(E.bad, 1);
    if (p.d_status) atomicOr(p.d_status, MUON_FLAG_NONFINITE);
}

// Entry e of the upper triangle (row-major, a <= b) of a KT x KT matrix.
template <int KT>
__device__ __forceinline__ void upper_entry(int e, int& a, int& b) {
    a = 0;
    while (e >= KT - a) { e -= KT - a; ++a; }
    b = a + e;
}

// Add this block's share S = X^T X of a k x k Gram matrix (X: `n` rows of KT
// floats in shared memory, columns >= k ignored) to the upper triangle of the
// fp64 sum `dst`.
template <int KT>
__device__ __forceinline__ void add_gram(const float* X, int n, int k, double* dst) {
    constexpr int NE = KT * (KT + 1) / 2;
    for (int e = threadIdx.x; e < NE; e += blockDim.x) {
        int a, b;
        upper_entry<KT>(e, a, b);
        if (b >= k) continue;
        double s = 0.0;
        for (int rr = 0; rr < n; ++rr) s = fma((double)X[rr * KT + a], (double)X[rr * KT + b], s);
        if (s != 0.0) atomicAdd(&dst[a * KT + b], s);
    }
}

// ---------------------------------------------------------------------------
// Tensor-core products with fp32 accuracy.  The three products with k columns
// (Y = M Omega, B^T = M^T Q, O = Z B) run on mma.sync m16n8k8 in tf32 with
// each operand split as x = hi + lo (hi = x rounded to tf32, lo = the
// remainder rounded to tf32) and the product summed as hi*lo + lo*hi + hi*hi
// into fp32 accumulators ("3xTF32"): the dropped lo*lo term and the rounding
// of lo are below 2^-21 of |a b| per product, under the fp32 accumulation's
// own rounding for sums of a few hundred terms or more.  At 2 k flops per
// element these products are below the HBM ridge once on tensor cores; the
// legacy warp-level MMA gives that rate with the fragments in registers,
// next to the fused momentum, Gram and weight-update code.
// Fragments of m16n8k8 (g = lane / 4, q = lane % 4): A (16 x 8) a0 = (g, q),
// a1 = (g + 8, q), a2 = (g, q + 4), a3 = (g + 8, q + 4); B (8 x 8) b0 = (q, g),
// b1 = (q + 4, g); C (16 x 8) c0, c1 = (g, 2q), (g, 2q + 1); c2, c3 = the same
// columns of row g + 8.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t to_tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}

__device__ __forceinline__ void split_tf32(float x, uint32_t& hi, uint32_t& lo) {
    hi = to_tf32(x);
    lo = to_tf32(x - __uint_as_float(hi));
}

__device__ __forceinline__ void mma_tf32(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// d += a b with a = ah + al, b = (bh0, bh1) + (bl0, bl1): small terms first.
__device__ __forceinline__ void mma3_tf32(float (&d)[4], const uint32_t (&ah)[4], const uint32_t (&al)[4],
                                          uint32_t bh0, uint32_t bh1, uint32_t bl0, uint32_t bl1) {
    mma_tf32(d, ah, bl0, bl1);
    mma_tf32(d, al, bh0, bh1);
    mma_tf32(d, ah, bh0, bh1);
}

// ---------------------------------------------------------------------------
// 1. momentum + sketch (+ share of Y^T Y)
// ---------------------------------------------------------------------------
template <int G_DT>
__host__ __device__ constexpr int g_size() { return G_DT == DT_FP32 ? 4 : 2; }

// Shared memory of the sketch.  Two stages of raw chunks: G [kSkRows][kSkCols]
// in its own type, M [kSkRows][kSkLd] fp32 (its tf32 high part after the
// momentum phase, in place), Omega [kSkCols][KT] fp32.  One buffer each of the
// chunk's M low part [kSkRows][kSkLd] and Omega's high and low parts
// [kSkCols][KT + 8].  Row pitches 4 (M) and 8 (Omega) words past a multiple
// of 32 make the fragment loads conflict-free.
template <int KT, int G_DT>
struct SketchSmem {
    static constexpr int kOmLd = KT + 8;
    static constexpr int kG = kSkRows * kSkCols * g_size<G_DT>();
    static constexpr int kM = kSkRows * kSkLd * 4;
    static constexpr int kOm = kSkCols * KT * 4;
    static constexpr int kStage = kG + kM + kOm;
    static constexpr int kMlo = 2 * kStage;
    static constexpr int kOmHi = kMlo + kSkRows * kSkLd * 4;
    static constexpr int kOmLo = kOmHi + kSkCols * kOmLd * 4;
    static constexpr int kBytes = kOmLo + kSkCols * kOmLd * 4;
};

template <int KT, int G_DT>
__global__ void __launch_bounds__(kThreads, 2) lim_sketch(const __grid_constant__ LimParams p) {
    using S = SketchSmem<KT, G_DT>;
    constexpr int GSZ = g_size<G_DT>();
    constexpr int NT = KT / 16;                // 8-column MMA tiles per warp (a warp takes half of Y's columns)
    static_assert(kSkRows == 64 && kThreads == 256, "four 16-row MMA tiles x two column halves");
    extern __shared__ __align__(16) unsigned char sm[];
    const LimEntry& E = p.e[find_entry(p, blockIdx.x, 0)];
    const int row0 = (blockIdx.x - E.t_sketch) * kSkRows;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, q4 = lane & 3;
    const int mt = warp & 3, n0 = (warp >> 2) * (KT / 2);   // rows 16 mt.., columns n0.. of Y
    const int nchunks = (E.cols + kSkCols - 1) / kSkCols;
    const bool om_vec = (p.k & 3) == 0;       // Omega rows 16-byte aligned
    uint32_t* mlo = reinterpret_cast<uint32_t*>(sm + S::kMlo);
    uint32_t* omh = reinterpret_cast<uint32_t*>(sm + S::kOmHi);
    uint32_t* oml = reinterpret_cast<uint32_t*>(sm + S::kOmLo);
    float acc[NT][4];
#pragma unroll
    for (int t = 0; t < NT; ++t)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[t][c] = 0.f;
    bool bad = false;

    // Chunk c (columns c*kSkCols..) of G, M and Omega into stage s; zeros outside.
    auto issue = [&](int c, int s) {
        const int c0 = c * kSkCols;
        unsigned char* gs = sm + s * S::kStage;
        float* ms = reinterpret_cast<float*>(gs + S::kG);
        float* os = reinterpret_cast<float*>(gs + S::kG + S::kM);
        if (E.vec_ok) {
            constexpr int GP = kSkCols * GSZ / 16, GE = 16 / GSZ;    // 16-byte pieces per row, elements per piece
            for (int q = threadIdx.x; q < kSkRows * GP; q += kThreads) {
                const int rr = q / GP, pc = q % GP, i = row0 + rr, j = c0 + pc * GE;
                const bool in = i < E.rows && j < E.cols;
                const char* src = static_cast<const char*>(E.G) + (in ? ((long long)i * E.cols + j) * GSZ : 0);
                cp_async16(gs + (rr * kSkCols + pc * GE) * GSZ, src, in ? 16u : 0u);
            }
            constexpr int MP = kSkCols / 4;
            for (int q = threadIdx.x; q < kSkRows * MP; q += kThreads) {
                const int rr = q / MP, pc = q % MP, i = row0 + rr, j = c0 + pc * 4;
                const bool in = i < E.rows && j < E.cols;
                cp_async16(ms + rr * kSkLd + pc * 4, E.M + (in ? (long long)i * E.cols + j : 0), in ? 16u : 0u);
            }
        } else {
            for (int q = threadIdx.x; q < kSkRows * kSkCols; q += kThreads) {
                const int rr = q / kSkCols, cc = q % kSkCols, i = row0 + rr, j = c0 + cc;
                const bool in = i < E.rows && j < E.cols;
                const long long idx = (long long)i * E.cols + j;
                st_elem(gs, rr * kSkCols + cc, G_DT, in ? ld_elem(E.G, idx, G_DT) : 0.f);
                ms[rr * kSkLd + cc] = in ? E.M[idx] : 0.f;
            }
        }
        if (om_vec) {
            constexpr int OP = KT / 4;
            for (int q = threadIdx.x; q < kSkCols * OP; q += kThreads) {
                const int jj = q / OP, pc = q % OP, j = c0 + jj;
                const bool in = j < E.cols && pc * 4 < p.k;
                cp_async16(os + jj * KT + pc * 4, E.Omega + (in ? (long long)j * p.k + pc * 4 : 0), in ? 16u : 0u);
            }
        } else {
            for (int q = threadIdx.x; q < kSkCols * KT; q += kThreads) {
                const int jj = q / KT, t = q % KT, j = c0 + jj;
                os[q] = (j < E.cols && t < p.k) ? E.Omega[(long long)j * p.k + t] : 0.f;
            }
        }
        cp_async_commit();
    };

    issue(0, 0);
    for (int c = 0; c < nchunks; ++c) {
        const int s = c & 1;
        if (c + 1 < nchunks) {
            issue(c + 1, s ^ 1);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();                       // chunk c complete for every thread
        const int c0 = c * kSkCols;
        unsigned char* gs = sm + s * S::kStage;
        float* ms = reinterpret_cast<float*>(gs + S::kG);
        const float* os = reinterpret_cast<const float*>(gs + S::kG + S::kM);
        // momentum: M <- mu M + G, back to global memory; its tf32 high part
        // replaces it in shared memory and the low part goes to mlo.  4
        // consecutive elements per thread, so a warp's 16-byte accesses are
        // consecutive in shared memory
#pragma unroll
        for (int it = 0; it < kSkRows * kSkCols / (4 * kThreads); ++it) {
            const int q = threadIdx.x + kThreads * it;
            const int rr = q / (kSkCols / 4), cc = (q % (kSkCols / 4)) * 4;
            const int i = row0 + rr, j = c0 + cc;
            float g4[4];
            if (GSZ == 2) {
                const uint2 u = *reinterpret_cast<const uint2*>(gs + (rr * kSkCols + cc) * 2);
                using T = typename std::conditional<G_DT == DT_BF16, __nv_bfloat16, __half>::type;
                g4[0] = unpack_lo<T>(u.x); g4[1] = unpack_hi<T>(u.x); g4[2] = unpack_lo<T>(u.y); g4[3] = unpack_hi<T>(u.y);
            } else {
                const float4 u = *reinterpret_cast<const float4*>(gs + (rr * kSkCols + cc) * 4);
                g4[0] = u.x; g4[1] = u.y; g4[2] = u.z; g4[3] = u.w;
            }
            float4* mp = reinterpret_cast<float4*>(ms + rr * kSkLd + cc);
            float4 m = *mp;
            m.x = fmaf(p.mu, m.x, g4[0]);      // zero outside the matrix
            m.y = fmaf(p.mu, m.y, g4[1]);
            m.z = fmaf(p.mu, m.z, g4[2]);
            m.w = fmaf(p.mu, m.w, g4[3]);
            bad |= !isfinite(m.x) || !isfinite(m.y) || !isfinite(m.z) || !isfinite(m.w);
            if (i < E.rows && j < E.cols) {
                float* dst = E.M + (long long)i * E.cols + j;
                if (E.vec_ok) {
                    *reinterpret_cast<float4*>(dst) = m;
                } else {
                    const float mv[4] = {m.x, m.y, m.z, m.w};
                    for (int e = 0; e < 4 && j + e < E.cols; ++e) dst[e] = mv[e];
                }
            }
            uint4 h, l;
            split_tf32(m.x, h.x, l.x);
            split_tf32(m.y, h.y, l.y);
            split_tf32(m.z, h.z, l.z);
            split_tf32(m.w, h.w, l.w);
            *reinterpret_cast<uint4*>(mp) = h;
            *reinterpret_cast<uint4*>(mlo + rr * kSkLd + cc) = l;
        }
        for (int q = threadIdx.x; q < kSkCols * KT; q += kThreads) {
            const int jj = q / KT, t = q % KT;
            split_tf32(os[q], omh[jj * S::kOmLd + t], oml[jj * S::kOmLd + t]);
        }
        __syncthreads();
        // Y[16 mt + .., n0 + ..] += M[rows, chunk] Omega[chunk, columns]
        const uint32_t* mh = reinterpret_cast<const uint32_t*>(ms);
#pragma unroll
        for (int kk = 0; kk < kSkCols; kk += 8) {
            const int a0 = (16 * mt + g) * kSkLd + kk + q4;
            const uint32_t ah[4] = {mh[a0], mh[a0 + 8 * kSkLd], mh[a0 + 4], mh[a0 + 8 * kSkLd + 4]};
            const uint32_t al[4] = {mlo[a0], mlo[a0 + 8 * kSkLd], mlo[a0 + 4], mlo[a0 + 8 * kSkLd + 4]};
#pragma unroll
            for (int t = 0; t < NT; ++t) {
                const int b0 = (kk + q4) * S::kOmLd + n0 + 8 * t + g;
                mma3_tf32(acc[t], ah, al, omh[b0], omh[b0 + 4 * S::kOmLd], oml[b0], oml[b0 + 4 * S::kOmLd]);
            }
        }
        __syncthreads();                       // stage s and the split buffers free for the next chunks
    }
    // Y to the workspace, and this block's rows' share of Y^T Y
    float* ys = reinterpret_cast<float*>(sm);  // [kSkRows][KT]
#pragma unroll
    for (int t = 0; t < NT; ++t) {
        const int col = n0 + 8 * t + 2 * q4;
        *reinterpret_cast<float2*>(ys + (16 * mt + g) * KT + col) = make_float2(acc[t][0], acc[t][1]);
        *reinterpret_cast<float2*>(ys + (16 * mt + g + 8) * KT + col) = make_float2(acc[t][2], acc[t][3]);
    }
    __syncthreads();
    for (int q = threadIdx.x; q < kSkRows * (KT / 4); q += kThreads) {
        const int rr = q / (KT / 4), pc = q % (KT / 4), i = row0 + rr;   // zero for rows past the matrix
        if (i < E.rows)
            *reinterpret_cast<float4*>(E.Y + (long long)i * KT + 4 * pc) =
                *reinterpret_cast<const float4*>(ys + rr * KT + 4 * pc);
    }
    add_gram<KT>(ys, min(kSkRows, E.rows - row0), p.k, E.Gy);
    if (__syncthreads_or(bad) && threadIdx.x == 0) mark_bad(p, E);
}

// ---------------------------------------------------------------------------
// 2. Cholesky of Y^T Y and R^-1 (one small block per matrix, k x k only)
// ---------------------------------------------------------------------------
template <int KT>
__global__ void __launch_bounds__(kSmallThreads) lim_chol(const __grid_constant__ LimParams p) {
    extern __shared__ __align__(16) double dsm[];
    double* Gm = dsm;                   // [KT][KT]: the Gram matrix, updated in place
    double* R = dsm + KT * KT;          // [KT][KT]: R (upper), then R^-1
    double* d0 = R + KT * KT;           // [KT]: squared column norms
    int* ok = reinterpret_cast<int*>(d0 + KT);   // [KT]
    __shared__ int nonfinite;
    const LimEntry& E = p.e[blockIdx.x];
    const int k = p.k;
    if (threadIdx.x == 0) nonfinite = 0;
    __syncthreads();
    for (int idx = threadIdx.x; idx < KT * KT; idx += blockDim.x) {
        const int a = idx / KT, b = idx % KT;
        const double v = (a < k && b < k) ? (a <= b ? E.Gy[a * KT + b] : E.Gy[b * KT + a]) : 0.0;
        if (!isfinite(v)) nonfinite = 1;
        Gm[idx] = v;
        R[idx] = 0.0;
    }
    __syncthreads();
    if (nonfinite) {                    // an overflow in the sketch: keep W, no factor
        for (int idx = threadIdx.x; idx < KT * KT; idx += blockDim.x) E.K[idx] = 0.0;
        if (threadIdx.x == 0) mark_bad(p, E);
        return;
    }
    if (threadIdx.x < KT) d0[threadIdx.x] = Gm[threadIdx.x * KT + threadIdx.x];
    __syncthreads();
    // right-looking Cholesky of the upper triangle: G = R^T R
    for (int j = 0; j < k; ++j) {
        const double d = Gm[j * KT + j];
        const bool keep = d > kDrop * d0[j] && d > 0.0;
        const double rj = keep ? sqrt(d) : 0.0;
        for (int b = j + threadIdx.x; b < k; b += blockDim.x) R[j * KT + b] = keep ? (b == j ? rj : Gm[j * KT + b] / rj) : 0.0;
        if (threadIdx.x == 0) ok[j] = keep;
        __syncthreads();
        const int m = k - j - 1;
        for (int idx = threadIdx.x; idx < m * m; idx += blockDim.x) {
            const int a = j + 1 + idx / m, b = j + 1 + idx % m;
            if (b >= a) Gm[a * KT + b] -= R[j * KT + a] * R[j * KT + b];
        }
        __syncthreads();
    }
    // R^-1 (upper) column by column into Gm; dropped rows stay zero
    for (int idx = threadIdx.x; idx < KT * KT; idx += blockDim.x) Gm[idx] = 0.0;
    __syncthreads();
    for (int b = threadIdx.x; b < k; b += blockDim.x) {
        for (int a = b; a >= 0; --a) {
            if (!ok[a]) continue;
            double s = a == b ? 1.0 : 0.0;
            for (int c = a + 1; c <= b; ++c) s -= R[a * KT + c] * Gm[c * KT + b];
            Gm[a * KT + b] = s / R[a * KT + a];
        }
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < KT * KT; idx += blockDim.x) E.K[idx] = Gm[idx];
}

// ---------------------------------------------------------------------------
// 3 / 6. rows of Y times the matrix's k x k factor K, in place (fp64 sums)
// ---------------------------------------------------------------------------
template <int KT>
__global__ void __launch_bounds__(kThreads) lim_rowmul(const __grid_constant__ LimParams p) {
    __shared__ double Ks[KT * KT];
    const LimEntry& E = p.e[find_entry(p, blockIdx.x, 1)];
    for (int idx = threadIdx.x; idx < KT * KT; idx += kThreads) Ks[idx] = E.K[idx];
    __syncthreads();
    const int i = (blockIdx.x - E.t_rows) * kThreads + threadIdx.x;
    if (i >= E.rows) return;
    float* row = E.Y + (long long)i * KT;
    float y[KT];
#pragma unroll
    for (int t = 0; t < KT; t += 4) {
        const float4 v = *reinterpret_cast<const float4*>(row + t);
        y[t] = v.x; y[t + 1] = v.y; y[t + 2] = v.z; y[t + 3] = v.w;
    }
    // four output columns at a time, stored as they are formed (the row was read whole)
#pragma unroll 1
    for (int j = 0; j < KT; j += 4) {
        double s0 = 0.0, s1 = 0.0, s2 = 0.0, s3 = 0.0;
#pragma unroll
        for (int a = 0; a < KT; ++a) {
            const double ya = (double)y[a];
            s0 = fma(ya, Ks[a * KT + j], s0);
            s1 = fma(ya, Ks[a * KT + j + 1], s1);
            s2 = fma(ya, Ks[a * KT + j + 2], s2);
            s3 = fma(ya, Ks[a * KT + j + 3], s3);
        }
        *reinterpret_cast<float4*>(row + j) = make_float4((float)s0, (float)s1, (float)s2, (float)s3);
    }
}

// ---------------------------------------------------------------------------
// 4. B^T = M^T Q (+ share of B B^T)
// ---------------------------------------------------------------------------
// Shared memory of the projection: kPjStages stages of M rows [kPjRows][kPjLd]
// (the block's columns) and Q rows [kPjRows][KT], then one buffer each of the
// chunk's Q high and low tf32 parts [kPjRows][KT + 8].  The pitches (8 words
// past a multiple of 32) make the fragment loads conflict-free.
constexpr int kPjLd = kPjCols + 8;

template <int KT>
struct ProjSmem {
    static constexpr int kQLd = KT + 8;
    static constexpr int kM = kPjRows * kPjLd * 4;
    static constexpr int kStage = kM + kPjRows * KT * 4;
    static constexpr int kQHi = kPjStages * kStage;
    static constexpr int kQLo = kQHi + kPjRows * kQLd * 4;
    static constexpr int kBytes = kQLo + kPjRows * kQLd * 4;
};

template <int KT>
__global__ void __launch_bounds__(kThreads, KT == 32 ? 3 : 2) lim_project(const __grid_constant__ LimParams p) {
    using S = ProjSmem<KT>;
    constexpr int NT = KT / 8;                 // 8-column MMA tiles: a warp takes every column of Q
    static_assert(kPjCols == 16 * (kThreads / 32), "one 16-column MMA tile of M per warp");
    extern __shared__ __align__(16) unsigned char sm[];
    const LimEntry& E = p.e[find_entry(p, blockIdx.x, 2)];
    const int c0 = (blockIdx.x - E.t_proj) * kPjCols;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, q4 = lane & 3;
    const int nchunks = (E.rows + kPjRows - 1) / kPjRows;
    uint32_t* qh = reinterpret_cast<uint32_t*>(sm + S::kQHi);
    uint32_t* ql = reinterpret_cast<uint32_t*>(sm + S::kQLo);
    float acc[NT][4];
#pragma unroll
    for (int t = 0; t < NT; ++t)
#pragma unroll
        for (int h = 0; h < 4; ++h) acc[t][h] = 0.f;

    // rows i0.. of M (this block's columns) and of Q into stage s
    auto issue = [&](int ch, int s) {
        const int i0 = ch * kPjRows;
        float* ms = reinterpret_cast<float*>(sm + s * S::kStage);
        float* qs = reinterpret_cast<float*>(sm + s * S::kStage + S::kM);
        if (E.vec_ok) {
            constexpr int MP = kPjCols / 4;
            for (int q = threadIdx.x; q < kPjRows * MP; q += kThreads) {
                const int rr = q / MP, pc = q % MP, i = i0 + rr, j = c0 + pc * 4;
                const bool in = i < E.rows && j < E.cols;
                cp_async16(ms + rr * kPjLd + pc * 4, E.M + (in ? (long long)i * E.cols + j : 0), in ? 16u : 0u);
            }
        } else {
            for (int q = threadIdx.x; q < kPjRows * kPjCols; q += kThreads) {
                const int rr = q / kPjCols, cc = q % kPjCols, i = i0 + rr, j = c0 + cc;
                ms[rr * kPjLd + cc] = (i < E.rows && j < E.cols) ? E.M[(long long)i * E.cols + j] : 0.f;
            }
        }
        constexpr int QP = KT / 4;
        for (int q = threadIdx.x; q < kPjRows * QP; q += kThreads) {
            const int rr = q / QP, pc = q % QP, i = i0 + rr;
            const bool in = i < E.rows;
            cp_async16(qs + rr * KT + pc * 4, E.Y + (in ? (long long)i * KT + pc * 4 : 0), in ? 16u : 0u);
        }
        cp_async_commit();
    };

    for (int ch = 0; ch < kPjStages - 1; ++ch)
        if (ch < nchunks) issue(ch, ch); else cp_async_commit();   // empty groups keep the count uniform
    for (int ch = 0; ch < nchunks; ++ch) {
        if (ch + kPjStages - 1 < nchunks) issue(ch + kPjStages - 1, (ch + kPjStages - 1) % kPjStages);
        else cp_async_commit();
        cp_async_wait<kPjStages - 1>();
        __syncthreads();
        const float* ms = reinterpret_cast<const float*>(sm + (ch % kPjStages) * S::kStage);
        const float* qs = reinterpret_cast<const float*>(sm + (ch % kPjStages) * S::kStage + S::kM);
        for (int q = threadIdx.x; q < kPjRows * KT; q += kThreads) {
            const int rr = q / KT, t = q % KT;
            split_tf32(qs[q], qh[rr * S::kQLd + t], ql[rr * S::kQLd + t]);
        }
        __syncthreads();
        // B^T[16 warp + .., :] += M[chunk, columns]^T Q[chunk, :]
#pragma unroll
        for (int kk = 0; kk < kPjRows; kk += 8) {
            const float* mr = ms + (kk + q4) * kPjLd + 16 * warp + g;
            uint32_t ah[4], al[4];
            split_tf32(mr[0], ah[0], al[0]);
            split_tf32(mr[8], ah[1], al[1]);
            split_tf32(mr[4 * kPjLd], ah[2], al[2]);
            split_tf32(mr[4 * kPjLd + 8], ah[3], al[3]);
#pragma unroll
            for (int t = 0; t < NT; ++t) {
                const int b0 = (kk + q4) * S::kQLd + 8 * t + g;
                mma3_tf32(acc[t], ah, al, qh[b0], qh[b0 + 4 * S::kQLd], ql[b0], ql[b0 + 4 * S::kQLd]);
            }
        }
        __syncthreads();                       // this stage and the split buffers are refilled next
    }
    cp_async_wait<0>();
    // B^T to the workspace, and this block's columns' share of B B^T
    float* bs = reinterpret_cast<float*>(sm);  // [kPjCols][KT]
#pragma unroll
    for (int t = 0; t < NT; ++t) {
        const int col = 8 * t + 2 * q4;
        *reinterpret_cast<float2*>(bs + (16 * warp + g) * KT + col) = make_float2(acc[t][0], acc[t][1]);
        *reinterpret_cast<float2*>(bs + (16 * warp + g + 8) * KT + col) = make_float2(acc[t][2], acc[t][3]);
    }
    __syncthreads();
    for (int q = threadIdx.x; q < kPjCols * (KT / 4); q += kThreads) {
        const int cc = q / (KT / 4), pc = q % (KT / 4), j = c0 + cc;
        if (j < E.cols)
            *reinterpret_cast<float4*>(E.Bt + (long long)j * KT + 4 * pc) =
                *reinterpret_cast<const float4*>(bs + cc * KT + 4 * pc);
    }
    add_gram<KT>(bs, min(kPjCols, E.cols - c0), p.k, E.Cg);
}

// ---------------------------------------------------------------------------
// 5. eigen-decomposition of B B^T and P = E_r L_r^{-1/2} E_r^T (one block per
//    matrix, k x k only).  A round applies k/2 disjoint rotations J at once:
//    C <- J^T C J touches the 2 x 2 blocks (rows of pair i, columns of pair j),
//    each updated by one thread from its own four entries, so a round is one
//    pass over C (and E <- E J) after the rotations are chosen.
// ---------------------------------------------------------------------------
template <int KT>
__global__ void __launch_bounds__(kThreads) lim_eig(const __grid_constant__ LimParams p) {
    constexpr int LD = KT + 1;          // padded rows: a column of C spreads over the banks
    extern __shared__ __align__(16) double dsm[];
    double* C = dsm;                    // [KT][LD]
    double* Ev = dsm + KT * LD;         // [KT][LD] eigenvectors (columns)
    double* cs = Ev + KT * LD;          // [KT/2] cosines
    double* sn = cs + KT / 2;           // [KT/2] sines
    double* lam = sn + KT / 2;          // [KT] eigenvalues
    int* pp = reinterpret_cast<int*>(lam + KT);   // [KT/2]
    int* pq = pp + KT / 2;                         // [KT/2]
    __shared__ int rotated, nonfinite;
    const LimEntry& E = p.e[blockIdx.x];
    const int k = p.k, ke = k + (k & 1), n = ke - 1, np = ke / 2;
    if (threadIdx.x == 0) nonfinite = 0;
    __syncthreads();
    for (int idx = threadIdx.x; idx < KT * KT; idx += blockDim.x) {
        const int a = idx / KT, b = idx % KT;
        const double v = (a < k && b < k) ? (a <= b ? E.Cg[a * KT + b] : E.Cg[b * KT + a]) : 0.0;
        if (!isfinite(v)) nonfinite = 1;
        C[a * LD + b] = v;
        Ev[a * LD + b] = a == b ? 1.0 : 0.0;
    }
    __syncthreads();
    if (nonfinite || *E.bad) {          // no factor for a marked matrix: its W is kept
        for (int idx = threadIdx.x; idx < KT * KT; idx += blockDim.x) E.K[idx] = 0.0;
        if (nonfinite && threadIdx.x == 0) mark_bad(p, E);
        return;
    }
    // Off-diagonal entries at the fp64 rounding level of the whole matrix are
    // noise, not coupling: below 0.1 kRotTol * trace no rotation is made, so a
    // pair of negligible eigenvalues cannot keep the sweeps going.
    double tr = 0.0;
    for (int a = 0; a < k; ++a) tr += fabs(C[a * LD + a]);
    const double floor_abs = kRotTol * 0.1 * tr;
    for (int sweep = 0; sweep < kMaxSweeps && n > 0; ++sweep) {
        if (threadIdx.x == 0) rotated = 0;
        __syncthreads();
        for (int rd = 0; rd < n; ++rd) {
            if (threadIdx.x < np) {
                const int i = threadIdx.x;
                int a = i == 0 ? n : (rd + i) % n, b = i == 0 ? rd : (rd - i + n) % n;
                if (a > b) { const int t = a; a = b; b = t; }
                const double apq = C[a * LD + b], app = C[a * LD + a], aqq = C[b * LD + b];
                double c = 1.0, s = 0.0;
                if (fabs(apq) > kRotTol * sqrt(fabs(app * aqq)) && fabs(apq) > floor_abs) {
                    const double tau = (aqq - app) / (2.0 * apq);
                    const double t = (tau >= 0.0 ? 1.0 : -1.0) / (fabs(tau) + sqrt(1.0 + tau * tau));
                    c = 1.0 / sqrt(1.0 + t * t);
                    s = t * c;
                    rotated = 1;
                }
                pp[i] = a; pq[i] = b; cs[i] = c; sn[i] = s;
            }
            __syncthreads();
            for (int idx = threadIdx.x; idx < np * np; idx += blockDim.x) {   // C <- J^T C J, block by block
                const int i = idx / np, j = idx % np;
                const double c1 = cs[i], s1 = sn[i], c2 = cs[j], s2 = sn[j];
                if (s1 == 0.0 && s2 == 0.0) continue;
                const int a1 = pp[i], b1 = pq[i], a2 = pp[j], b2 = pq[j];
                const double x = C[a1 * LD + a2], y = C[a1 * LD + b2], z = C[b1 * LD + a2], w = C[b1 * LD + b2];
                const double r0 = c1 * x - s1 * z, r1 = c1 * y - s1 * w;   // rows a1, b1 rotated
                const double r2 = s1 * x + c1 * z, r3 = s1 * y + c1 * w;
                C[a1 * LD + a2] = c2 * r0 - s2 * r1;                      // then columns a2, b2
                C[a1 * LD + b2] = s2 * r0 + c2 * r1;
                C[b1 * LD + a2] = c2 * r2 - s2 * r3;
                C[b1 * LD + b2] = s2 * r2 + c2 * r3;
            }
            for (int idx = threadIdx.x; idx < ke * np; idx += blockDim.x) {   // E <- E J
                const int row = idx / np, i = idx % np;
                const double c = cs[i], s = sn[i];
                if (s == 0.0) continue;
                const double u = Ev[row * LD + pp[i]], v = Ev[row * LD + pq[i]];
                Ev[row * LD + pp[i]] = c * u - s * v;
                Ev[row * LD + pq[i]] = s * u + c * v;
            }
            __syncthreads();
        }
        const bool again = rotated != 0;       // read by every thread before the next reset
        __syncthreads();
        if (!again) break;                     // a sweep without a rotation: converged
    }
    // the r largest eigenvalues above kTau2 * largest: weights 1 / sqrt(lambda)
    if (threadIdx.x < k) lam[threadIdx.x] = C[threadIdx.x * LD + threadIdx.x];
    __syncthreads();
    double lmax = 0.0;
    for (int a = 0; a < k; ++a) lmax = fmax(lmax, lam[a]);
    double* wgt = cs;                   // reuse: [KT] weights (cs and sn are contiguous)
    __syncthreads();
    for (int a = threadIdx.x; a < k; a += blockDim.x) {
        int rank = 0;
        for (int b = 0; b < k; ++b) rank += (lam[b] > lam[a]) || (lam[b] == lam[a] && b < a);
        const bool sel = lmax > 0.0 && rank < p.r && lam[a] > kTau2 * lmax;
        wgt[a] = sel ? 1.0 / sqrt(lam[a]) : 0.0;
    }
    __syncthreads();
    // P = E diag(w) E^T
    for (int idx = threadIdx.x; idx < KT * KT; idx += blockDim.x) {
        const int a = idx / KT, b = idx % KT;
        double s = 0.0;
        if (a < k && b < k)
            for (int e = 0; e < k; ++e) s += Ev[a * LD + e] * wgt[e] * Ev[b * LD + e];
        E.K[idx] = s;
    }
}

// ---------------------------------------------------------------------------
// 7. O = Z B and the weight update
// ---------------------------------------------------------------------------
// Shared memory of lim_update: Z rows [kUpRows][KT + 4] and the B^T rows of
// the tile's columns [kUpCols][KT + 4] as loaded, each then replaced by its
// tf32 high part with the low parts in two more such arrays, and the tile of W
// [kUpRows][kUpCols + 8] in W's type.  The pitches make the fragment loads
// and the epilogue's accesses to W conflict-free.
template <int KT, int W_DT>
struct UpdSmem {
    static constexpr int kLd = KT + 4;
    static constexpr int kWLd = kUpCols + 8;
    static constexpr int kArr = kUpRows * kLd * 4;
    static constexpr int kZ = 0, kZlo = kArr, kBt = 2 * kArr, kBtlo = 3 * kArr, kW = 4 * kArr;
    static constexpr int kBytes = kW + kUpRows * kWLd * g_size<W_DT>();
    static_assert(kUpRows == kUpCols, "Z and B^T tiles share a shape");
};

template <int KT, int W_DT>
__global__ void __launch_bounds__(kThreads, 2) lim_update(const __grid_constant__ LimParams p) {
    using S = UpdSmem<KT, W_DT>;
    constexpr int WSZ = g_size<W_DT>();
    constexpr int NT = kUpCols / 8;            // 8-column MMA tiles: a warp takes 16 rows x every column
    static_assert(kUpRows == 16 * (kThreads / 32), "one 16-row MMA tile per warp");
    extern __shared__ __align__(16) unsigned char sm[];
    float* Zs = reinterpret_cast<float*>(sm + S::kZ);
    float* Bts = reinterpret_cast<float*>(sm + S::kBt);
    uint32_t* Zlo = reinterpret_cast<uint32_t*>(sm + S::kZlo);
    uint32_t* Btlo = reinterpret_cast<uint32_t*>(sm + S::kBtlo);
    unsigned char* Ws = sm + S::kW;
    const LimEntry& E = p.e[find_entry(p, blockIdx.x, 3)];
    const int tile = blockIdx.x - E.t_upd;
    const int tiles_c = (E.cols + kUpCols - 1) / kUpCols;
    const int row0 = (tile / tiles_c) * kUpRows, c0 = (tile % tiles_c) * kUpCols;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, q4 = lane & 3;
    const bool skip = *E.bad != 0;
    const bool wtile = E.vec_ok && !skip;      // W through shared memory (16-byte pieces)
    // every global read of the tile in one asynchronous group: Z rows, the
    // B^T rows of the tile's columns, and (aligned rows) the tile of W
    constexpr int ZP = KT / 4;
    for (int q = threadIdx.x; q < kUpRows * ZP; q += kThreads) {
        const int rr = q / ZP, pc = q % ZP, i = row0 + rr;
        const bool in = i < E.rows;
        cp_async16(Zs + rr * S::kLd + pc * 4, E.Y + (in ? (long long)i * KT + pc * 4 : 0), in ? 16u : 0u);
    }
    for (int q = threadIdx.x; q < kUpCols * ZP; q += kThreads) {
        const int jj = q / ZP, pc = q % ZP, j = c0 + jj;
        const bool in = j < E.cols;
        cp_async16(Bts + jj * S::kLd + pc * 4, E.Bt + (in ? (long long)j * KT + pc * 4 : 0), in ? 16u : 0u);
    }
    if (wtile) {
        constexpr int WP = kUpCols * WSZ / 16, WE = 16 / WSZ;   // 16-byte pieces per row, elements per piece
        for (int q = threadIdx.x; q < kUpRows * WP; q += kThreads) {
            const int rr = q / WP, pc = q % WP, i = row0 + rr, j = c0 + pc * WE;
            const bool in = i < E.rows && j < E.cols;
            const char* src = static_cast<const char*>(E.W) + (in ? ((long long)i * E.cols + j) * WSZ : 0);
            cp_async16(Ws + (rr * S::kWLd + pc * WE) * WSZ, src, in ? 16u : 0u);
        }
    }
    cp_async_commit();
    cp_async_wait<0>();
    __syncthreads();
    const int kk8 = (p.k + 7) & ~7;            // columns of Z (and of B^T) past k are zero
    for (int q = threadIdx.x; q < kUpRows * KT; q += kThreads) {
        const int rr = q / KT, t = q % KT, o = rr * S::kLd + t;
        if (t >= kk8) continue;
        uint32_t h;
        split_tf32(Zs[o], h, Zlo[o]);
        Zs[o] = __uint_as_float(h);
        split_tf32(Bts[o], h, Btlo[o]);
        Bts[o] = __uint_as_float(h);
    }
    __syncthreads();
    const uint32_t* Zh = reinterpret_cast<const uint32_t*>(Zs);
    const uint32_t* Bth = reinterpret_cast<const uint32_t*>(Bts);
    float o[NT][4];
#pragma unroll
    for (int t = 0; t < NT; ++t)
#pragma unroll
        for (int c = 0; c < 4; ++c) o[t][c] = 0.f;
#pragma unroll 1
    for (int kk = 0; kk < kk8; kk += 8) {
        const int a0 = (16 * warp + g) * S::kLd + kk + q4;
        const uint32_t ah[4] = {Zh[a0], Zh[a0 + 8 * S::kLd], Zh[a0 + 4], Zh[a0 + 8 * S::kLd + 4]};
        const uint32_t al[4] = {Zlo[a0], Zlo[a0 + 8 * S::kLd], Zlo[a0 + 4], Zlo[a0 + 8 * S::kLd + 4]};
#pragma unroll
        for (int t = 0; t < NT; ++t) {
            // B (k x columns) = (B^T)^T: b0 = B^T[8 t + g][kk + q4]
            const int b0 = (8 * t + g) * S::kLd + kk + q4;
            mma3_tf32(o[t], ah, al, Bth[b0], Bth[b0 + 4], Btlo[b0], Btlo[b0 + 4]);
        }
    }
    // epilogue: O (optional) and W <- W - eta (gamma O + lambda W); this
    // thread holds rows 16 warp + g (+ 8), columns 8 t + 2 q4 (+ 1)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int rr = 16 * warp + g + 8 * h, i = row0 + rr;
#pragma unroll
        for (int t = 0; t < NT; ++t) {
            const int cc = 8 * t + 2 * q4, j = c0 + cc;
            const float v0 = o[t][2 * h], v1 = o[t][2 * h + 1];
            const bool in0 = i < E.rows && j < E.cols, in1 = i < E.rows && j + 1 < E.cols;
            if (E.O_out) {
                const long long idx = (long long)i * E.cols + j;
                if (E.vec_ok && in0) *reinterpret_cast<float2*>(E.O_out + idx) = make_float2(v0, v1);
                else {
                    if (in0) E.O_out[idx] = v0;
                    if (in1) E.O_out[idx + 1] = v1;
                }
            }
            if (skip) continue;
            if (wtile) {                       // in shared memory, stored below
                unsigned char* wp = Ws + (rr * S::kWLd + cc) * WSZ;
                if (W_DT == DT_FP32) {
                    float2 w = *reinterpret_cast<float2*>(wp);
                    w.x = w.x - p.eta * (E.gamma * v0 + p.lambda * w.x);
                    w.y = w.y - p.eta * (E.gamma * v1 + p.lambda * w.y);
                    *reinterpret_cast<float2*>(wp) = w;
                } else {
                    using T = typename std::conditional<W_DT == DT_BF16, __nv_bfloat16, __half>::type;
                    const uint32_t u = *reinterpret_cast<const uint32_t*>(wp);
                    float w0 = unpack_lo<T>(u), w1 = unpack_hi<T>(u);
                    w0 = w0 - p.eta * (E.gamma * v0 + p.lambda * w0);
                    w1 = w1 - p.eta * (E.gamma * v1 + p.lambda * w1);
                    *reinterpret_cast<uint32_t*>(wp) = pack2<T>(w0, w1);
                }
            } else {
                const long long idx = (long long)i * E.cols + j;
                if (in0) {
                    const float w0 = ld_elem(E.W, idx, W_DT);
                    st_elem(E.W, idx, W_DT, w0 - p.eta * (E.gamma * v0 + p.lambda * w0));
                }
                if (in1) {
                    const float w1 = ld_elem(E.W, idx + 1, W_DT);
                    st_elem(E.W, idx + 1, W_DT, w1 - p.eta * (E.gamma * v1 + p.lambda * w1));
                }
            }
        }
    }
    if (wtile) {                               // uniform over the block
        __syncthreads();
        constexpr int WP = kUpCols * WSZ / 16, WE = 16 / WSZ;
        for (int q = threadIdx.x; q < kUpRows * WP; q += kThreads) {
            const int rr = q / WP, pc = q % WP, i = row0 + rr, j = c0 + pc * WE;
            if (i < E.rows && j < E.cols)       // cols % 8 == 0: a piece is wholly in or out
                *reinterpret_cast<uint4*>(static_cast<char*>(E.W) + ((long long)i * E.cols + j) * WSZ) =
                    *reinterpret_cast<const uint4*>(Ws + (rr * S::kWLd + pc * WE) * WSZ);
        }
    }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

template <int KT, int G_DT>
constexpr size_t sketch_smem() { return (size_t)SketchSmem<KT, G_DT>::kBytes; }
template <int KT>
constexpr size_t project_smem() { return (size_t)ProjSmem<KT>::kBytes; }
template <int KT, int W_DT>
constexpr size_t update_smem() { return (size_t)UpdSmem<KT, W_DT>::kBytes; }
template <int KT>
constexpr size_t chol_smem() { return sizeof(double) * (2 * KT * KT + KT) + sizeof(int) * KT; }
template <int KT>
constexpr size_t eig_smem() { return sizeof(double) * (2 * KT * (KT + 1) + KT / 2 * 2 + KT) + sizeof(int) * KT; }

static_assert(sketch_smem<64, DT_FP32>() >= sizeof(float) * kSkRows * 64, "sketch Y staging fits a stage");
static_assert(project_smem<64>() >= sizeof(float) * kPjCols * 64, "projection B^T staging fits the stages");

template <typename K>
cudaError_t allow_smem(K kernel, size_t bytes) {
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

struct LaunchShape {
    int sketch, rows, proj, upd;       // blocks of the grid-wide launches
    double elems, rows_k, cols_k, rows_total;
};

template <int KT, int W_DT>
muon_status launch_all(LimParams& prm, cudaStream_t s, const LaunchShape& L) {
    // The shared-memory limit is a per-device attribute of each kernel: set it
    // once on every device this instantiation is launched on.
    static std::mutex mu;
    static bool configured[kMaxDevices] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MUON_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return MUON_ERR_UNSUPPORTED;
    {
        std::lock_guard<std::mutex> lock(mu);
        if (!configured[dev]) {
            cudaError_t e[5] = {allow_smem(lim_sketch<KT, W_DT>, sketch_smem<KT, W_DT>()),
                                allow_smem(lim_chol<KT>, chol_smem<KT>()),
                                allow_smem(lim_project<KT>, project_smem<KT>()),
                                allow_smem(lim_eig<KT>, eig_smem<KT>()),
                                allow_smem(lim_update<KT, W_DT>, update_smem<KT, W_DT>())};
            for (cudaError_t x : e)
                if (x != cudaSuccess) return MUON_ERR_CUDA;
            configured[dev] = true;
        }
    }
    const double wsz = dt_size(W_DT), k = prm.k, kk = (double)KT * KT * 8.0 * prm.n;
    // algorithmic bytes (MUON_KERNEL_RSVD: the passes over the matrices; _SMALL: the k x k work)
    trace_begin(MUON_KERNEL_RSVD, L.elems * (wsz + 8.0) + 4.0 * L.rows_k, s);       // G, M read; M, Y written
    lim_sketch<KT, W_DT><<<L.sketch, kThreads, sketch_smem<KT, W_DT>(), s>>>(prm);
    trace_end(s);
    trace_begin(MUON_KERNEL_RSVD_SMALL, 2.0 * kk, s);                                // Gram read, R^-1 written
    lim_chol<KT><<<prm.n, kSmallThreads, chol_smem<KT>(), s>>>(prm);
    trace_end(s);
    trace_begin(MUON_KERNEL_RSVD_SMALL, 8.0 * L.rows_total * KT + kk, s);           // Y read and written
    lim_rowmul<KT><<<L.rows, kThreads, 0, s>>>(prm);
    trace_end(s);
    trace_begin(MUON_KERNEL_RSVD, L.elems * 4.0 + 4.0 * (L.rows_k + L.cols_k), s);  // M, Q read; B^T written
    lim_project<KT><<<L.proj, kThreads, project_smem<KT>(), s>>>(prm);
    trace_end(s);
    trace_begin(MUON_KERNEL_RSVD_SMALL, 2.0 * kk, s);                                // Gram read, P written
    lim_eig<KT><<<prm.n, kThreads, eig_smem<KT>(), s>>>(prm);
    trace_end(s);
    trace_begin(MUON_KERNEL_RSVD_SMALL, 8.0 * L.rows_total * KT + kk, s);           // Q read, Z written
    lim_rowmul<KT><<<L.rows, kThreads, 0, s>>>(prm);
    trace_end(s);
    trace_begin(MUON_KERNEL_RSVD, L.elems * 2.0 * wsz + 4.0 * (L.rows_k + L.cols_k), s);   // W read and written
    lim_update<KT, W_DT><<<L.upd, kThreads, update_smem<KT, W_DT>(), s>>>(prm);
    trace_end(s);
    (void)k;
    return cudaGetLastError() == cudaSuccess ? MUON_OK : MUON_ERR_CUDA;
}

size_t matrix_ws(int rows, int cols, int KT) {
    return align256(sizeof(float) * (size_t)rows * KT) + align256(sizeof(float) * (size_t)cols * KT);
}

int kt_for(int k) { return k <= 32 ? 32 : 64; }

muon_status check_hp(const muon_rsvd_hparams* hp) {
    if (!hp) return MUON_ERR_INVALID_ARG;
    const float v[4] = {hp->mu, hp->eta, hp->lambda, hp->gamma};
    for (float x : v)
        if (!std::isfinite(x)) return MUON_ERR_INVALID_ARG;
    if (hp->rank < 1 || hp->oversample < 0) return MUON_ERR_INVALID_ARG;
    if (hp->rank + hp->oversample > 64) return MUON_ERR_UNSUPPORTED;
    return MUON_OK;
}

muon_status check_shapes(const muon_rsvd_param* params, int n) {
    if (!params || n < 1) return MUON_ERR_INVALID_ARG;
    for (int i = 0; i < n; ++i) {
        if (params[i].rows < 1 || params[i].cols < 1) return MUON_ERR_INVALID_ARG;
        if (params[i].rows > (1 << 24) || params[i].cols > (1 << 24)) return MUON_ERR_UNSUPPORTED;
    }
    return MUON_OK;
}

// Workspace: the per-matrix flags, then the k x k sums that start at zero
// (Y^T Y, B B^T), then the k x k factors, then per matrix Y and B^T.
struct WsLayout {
    size_t flags, zero_bytes, gy, cg, kf, mats, total;
};

WsLayout ws_layout(const muon_rsvd_param* params, int n, int KT) {
    WsLayout L;
    const size_t kk = sizeof(double) * (size_t)KT * KT * n;
    L.flags = 0;
    L.gy = align256(sizeof(int) * (size_t)n);
    L.cg = L.gy + align256(kk);
    L.zero_bytes = L.cg + align256(kk);
    L.kf = L.zero_bytes;
    L.mats = L.kf + align256(kk);
    L.total = L.mats;
    for (int i = 0; i < n; ++i) L.total += matrix_ws(params[i].rows, params[i].cols, KT);
    return L;
}

}  // namespace
}  // namespace muon

using namespace muon;

extern "C" {

muon_status limuon_workspace_size(const muon_rsvd_param* params, int n, const muon_rsvd_hparams* hp,
                                  size_t* bytes) {
    muon_status st = check_shapes(params, n);
    if (st != MUON_OK) return st;
    if ((st = check_hp(hp)) != MUON_OK) return st;
    if (!bytes) return MUON_ERR_INVALID_ARG;
    *bytes = ws_layout(params, n, kt_for(hp->rank + hp->oversample)).total;
    return MUON_OK;
}

muon_status limuon_step_batched(const muon_rsvd_param* params, int n, muon_dtype w_dtype,
                                const muon_rsvd_hparams* hp, void* workspace, size_t ws_bytes, int* d_status,
                                muon_stream_t stream) {
    size_t need = 0;
    muon_status st = limuon_workspace_size(params, n, hp, &need);
    if (st != MUON_OK) return st;
    if (w_dtype != MUON_BF16 && w_dtype != MUON_FP16 && w_dtype != MUON_FP32) return MUON_ERR_INVALID_ARG;
    for (int i = 0; i < n; ++i) {
        const muon_rsvd_param& q = params[i];
        if (!q.W || !q.G || !q.M || !q.Omega) return MUON_ERR_INVALID_ARG;
    }
    if (!workspace || ws_bytes < need) return MUON_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) & 255) return MUON_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int k = hp->rank + hp->oversample, KT = kt_for(k);
    const WsLayout W = ws_layout(params, n, KT);
    char* ws = static_cast<char*>(workspace);
    // flags and the two Gram sums start at zero
    if (cudaMemsetAsync(ws, 0, W.zero_bytes, s) != cudaSuccess) return MUON_ERR_CUDA;
    int* bad = reinterpret_cast<int*>(ws + W.flags);
    double* gy = reinterpret_cast<double*>(ws + W.gy);
    double* cg = reinterpret_cast<double*>(ws + W.cg);
    double* kf = reinterpret_cast<double*>(ws + W.kf);
    char* cur = ws + W.mats;
    static LimParams prm;              // large: kept off the stack, filled and consumed per launch
    static std::mutex mu;
    std::lock_guard<std::mutex> lock(mu);
    for (int b = 0; b < n; b += kLimMax) {
        memset(&prm, 0, sizeof(prm));
        prm.n = std::min(kLimMax, n - b);
        prm.k = k; prm.r = hp->rank;
        prm.mu = hp->mu; prm.eta = hp->eta; prm.lambda = hp->lambda;
        prm.d_status = d_status;
        LaunchShape L = {};
        for (int i = 0; i < prm.n; ++i) {
            const muon_rsvd_param& q = params[b + i];
            LimEntry& E = prm.e[i];
            E.W = q.W; E.G = q.G; E.M = q.M; E.Omega = q.Omega; E.O_out = q.O_out;
            E.rows = q.rows; E.cols = q.cols;
            E.gamma = std::isnan(q.gamma) ? hp->gamma : q.gamma;
            E.bad = bad + b + i;
            const size_t kk = (size_t)KT * KT * (b + i);
            E.Gy = gy + kk; E.Cg = cg + kk; E.K = kf + kk;
            E.Y = reinterpret_cast<float*>(cur);
            E.Bt = reinterpret_cast<float*>(cur + align256(sizeof(float) * (size_t)q.rows * KT));
            cur += matrix_ws(q.rows, q.cols, KT);
            const uintptr_t al = reinterpret_cast<uintptr_t>(q.W) | reinterpret_cast<uintptr_t>(q.G) |
                                 reinterpret_cast<uintptr_t>(q.M) | reinterpret_cast<uintptr_t>(q.O_out);
            E.vec_ok = (al & 15) == 0 && q.cols % 8 == 0;
            L.elems += (double)q.rows * q.cols;
            L.rows_k += (double)q.rows * k;
            L.cols_k += (double)q.cols * k;
            L.rows_total += q.rows;
        }
        // Each launch's grid in its own order of the matrices: a sketch block
        // runs over its matrix's columns and a projection block over its rows,
        // so those two put the longest first (stable: ties keep their order).
        long long tot[4] = {0, 0, 0, 0};
        for (int w = 0; w < 4; ++w) {
            int idx[kLimMax];
            for (int i = 0; i < prm.n; ++i) idx[i] = i;
            if (w == 0 || w == 2)
                std::stable_sort(idx, idx + prm.n, [&](int a, int b) {
                    return w == 0 ? prm.e[a].cols > prm.e[b].cols : prm.e[a].rows > prm.e[b].rows;
                });
            for (int pos = 0; pos < prm.n; ++pos) {
                LimEntry& E = prm.e[idx[pos]];
                prm.ord[w][pos] = (unsigned char)idx[pos];
                const long long first = tot[w];
                if (w == 0) { E.t_sketch = (int)first; tot[w] += (E.rows + kSkRows - 1) / kSkRows; }
                else if (w == 1) { E.t_rows = (int)first; tot[w] += (E.rows + kThreads - 1) / kThreads; }
                else if (w == 2) { E.t_proj = (int)first; tot[w] += (E.cols + kPjCols - 1) / kPjCols; }
                else {
                    E.t_upd = (int)first;
                    tot[w] += (long long)((E.rows + kUpRows - 1) / kUpRows) * ((E.cols + kUpCols - 1) / kUpCols);
                }
                if (tot[w] > INT32_MAX) return MUON_ERR_UNSUPPORTED;
            }
        }
        L.sketch = (int)tot[0]; L.rows = (int)tot[1]; L.proj = (int)tot[2]; L.upd = (int)tot[3];
        if (KT == 32) {
            if (w_dtype == MUON_BF16) st = launch_all<32, DT_BF16>(prm, s, L);
            else if (w_dtype == MUON_FP16) st = launch_all<32, DT_FP16>(prm, s, L);
            else st = launch_all<32, DT_FP32>(prm, s, L);
        } else {
            if (w_dtype == MUON_BF16) st = launch_all<64, DT_BF16>(prm, s, L);
            else if (w_dtype == MUON_FP16) st = launch_all<64, DT_FP16>(prm, s, L);
            else st = launch_all<64, DT_FP32>(prm, s, L);
        }
        if (st != MUON_OK) return st;
    }
    return MUON_OK;
}

}  // extern "C"
