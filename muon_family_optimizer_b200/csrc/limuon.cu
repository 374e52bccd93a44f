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
//   1 lim_sketch   M <- mu M + G and Y = M Omega, 128-row blocks over
//                  32-column chunks double-buffered in shared memory
//                  (cp.async), the product on tensor cores (warp-level MMA,
//                  tf32 x 3, fp32 accuracy); each block adds its rows' share
//                  of the Gram Y^T Y (fp64) to the matrix's k x k sum.  Reads
//                  G and M, writes M.
//   2 lim_chol     per matrix (k x k): Cholesky of Y^T Y in fp64 (a column whose
//                  pivot falls to 1e-10 of its squared norm lies in the span of
//                  the previous ones and is dropped: its Q column is zero), R^-1.
//   3 lim_rowmul   Q = Y R^-1, row by row in place (fp64 sums), all matrices'
//                  rows in one grid.
//   4 lim_project  B^T = M^T Q, 128-column blocks over 32-row chunks (three
//                  cp.async stages), tensor cores as in 1; each block adds its
//                  columns' share of B B^T (fp64) to the matrix's k x k sum.
//                  Reads M.
//   5 lim_eig      per matrix (k x k): cyclic Jacobi on B B^T in fp64, padded
//                  with zeros to KT = 32 or 64 indices, round-robin order
//                  from a table (KT/2 disjoint rotations per round), a
//                  rotation only while |C_pq| > 1e-15 sqrt(C_pp C_qq) (and
//                  above 1e-16 of the trace: fp64 noise), stop after a sweep
//                  without one; P from the r largest eigenpairs.
//   6 lim_rowmul   Z = Q P in place.  Q and Z are stored as tf32 high and low
//                  parts (the operands of 4 and 7).
//   7 lim_update   O = Z B on 128 x 128 tiles with tcgen05 (kind::tf32,
//                  accumulator in tensor memory, tf32 x 3), fused with the
//                  weight update (reads and writes W, staged in shared memory
//                  while the MMAs run; O never stored unless O_out is given).
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
constexpr int kSkRows = 128;      // lim_sketch: rows per block (one 16-row MMA tile per warp)
constexpr int kSkCols = 32;       // lim_sketch: columns per chunk (two stages)
constexpr int kPjCols = 128;      // lim_project: columns per block (one 16-column MMA tile per warp)
constexpr int kPjRows = 32;       // lim_project: rows per chunk
constexpr int kPjStages = 3;
constexpr int kPjSegRows = 1024;  // lim_project: rows per block; taller matrices split into segments
constexpr int kUpRows = 128;      // lim_update: tile rows (the MMA's M)
constexpr int kUpCols = 128;      // lim_update: tile columns (the MMA's N)
constexpr double kDrop = 1e-10;   // Cholesky pivot / squared column norm below which a column is dropped
constexpr double kTau2 = 1e-10;   // (singular value / largest)^2 at or below which it counts as zero
constexpr double kRotTol = 1e-15; // Jacobi: rotate while |C_pq| > kRotTol sqrt(C_pp C_qq)
constexpr int kMaxSweeps = 30;
constexpr int kMaxDevices = 64;    // devices whose kernel attributes are tracked

struct LimEntry {
    void* W; const void* G; float* M; const float* Omega; float* O_out;
    float* Y;        // rows x KT workspace: Y, then the tf32 high parts of Q, then of Z (in place)
    float* Ylo;      // rows x KT workspace: the tf32 low parts of Q, then of Z
    float* Bt;       // cols x KT workspace: the tf32 high parts of B^T
    float* Btlo;     // cols x KT workspace: the tf32 low parts of B^T
    float* Bpart;    // nseg x cols x KT workspace: the projection's per-segment partial B^T (nseg > 1)
    int* pj_count;   // per 128-column block: segments finished (workspace, zeroed per call; nseg > 1)
    int nseg;        // row segments of the projection
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
// (Y = M Omega, B^T = M^T Q, O = Z B) run in tf32 with each operand split as
// x = hi + lo (hi = x rounded to tf32, lo = the remainder rounded to tf32) and
// the product summed as hi*lo + lo*hi + hi*hi into fp32 accumulators
// ("3xTF32"): the dropped lo*lo term and the rounding of lo are below 2^-21 of
// |a b| per product, under the fp32 accumulation's own rounding for sums of a
// few hundred terms or more.  At 2 k flops per element these products are
// below the HBM ridge once on tensor cores.  The update, a 128 x 128 x k
// product per tile, runs on tcgen05 (kind::tf32) with the accumulator in
// tensor memory; the sketch and the projection, whose contraction runs over a
// whole row or column of the matrix next to per-element momentum work, use
// the warp-level MMA with the fragments in registers.
// Fragments of m16n8k8 (g = lane / 4, q = lane % 4): A (16 x 8) a0 = (g, q),
// a1 = (g + 8, q), a2 = (g, q + 4), a3 = (g + 8, q + 4); B (8 x 8) b0 = (q, g),
// b1 = (q + 4, g); C (16 x 8) c0, c1 = (g, 2q), (g, 2q + 1); c2, c3 = the same
// columns of row g + 8.
// ---------------------------------------------------------------------------
// x rounded to the nearest tf32 value (ties away from zero): add half of the
// dropped 13 bits' weight to the magnitude bits and clear them (integer ops,
// full-rate pipes).  Finite values that round past the largest float become
// infinite; infinities and NaN (whose bits could wrap) are only truncated.
__device__ __forceinline__ uint32_t to_tf32(float x) {
    const uint32_t u = __float_as_uint(x);
    return ((u & 0x7f800000u) == 0x7f800000u ? u : u + 0x1000u) & 0xffffe000u;
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

// tcgen05 in tf32 (kind::tf32, fp32 accumulators in tensor memory), one CTA.
// Instruction descriptor: fp32 accumulate, A and B tf32, K-major unless the
// operand is MN-major, N >> 3 at bit 17, M >> 4 at bit 24.
__host__ __device__ constexpr uint32_t idesc_tf32(int a_mn, int b_mn, int M, int N) {
    return (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)a_mn << 15) | ((uint32_t)b_mn << 16) |
           ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void tc_mma_tf32(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Byte offset of the 16-byte piece `pc` (4 words) of row r in a K-major
// 128-byte-swizzled operand of `rows` rows and KT words per row: KT / 32
// atoms of [rows][128 bytes], piece (pc % 8) of a row at (pc % 8) ^ (r % 8).
__device__ __forceinline__ int sw128_piece(int r, int pc, int rows) {
    return (pc >> 3) * rows * 128 + r * 128 + (((pc & 7) ^ (r & 7)) << 4);
}

// ---------------------------------------------------------------------------
// 1. momentum + sketch (+ share of Y^T Y)
// ---------------------------------------------------------------------------
template <int G_DT>
__host__ __device__ constexpr int g_size() { return G_DT == DT_FP32 ? 4 : 2; }

// Swizzled rows of 32-bit words (a multiple of 32 per row): word c of row r
// sits at c ^ 16 (r & 1), so a quarter-warp's 16-byte loads of two adjacent
// rows at the same columns fall in different banks.  16-byte pieces stay whole.
__device__ __forceinline__ int swz(int r, int c) { return c ^ ((r & 1) << 4); }

// Tensor-core operand loads with the k index permuted inside each 16-wide
// group: in k-step s (0, 1) of the group, the MMA's k = q and q + 4 take the
// group's columns 4 q + 2 s and 4 q + 2 s + 1, the same for A and B, so one
// 16-byte load gives a thread its A (or B) words for both k-steps.  (The
// contraction runs over every column of the group either way.)
struct Frag16 {
    uint32_t h[4], l[4];   // the four words at columns 4 q .. 4 q + 3: high and low parts
};

__device__ __forceinline__ void ld_frag16(Frag16& f, const uint32_t* hi, const uint32_t* lo, int off) {
    const uint4 a = *reinterpret_cast<const uint4*>(hi + off);
    const uint4 b = *reinterpret_cast<const uint4*>(lo + off);
    f.h[0] = a.x; f.h[1] = a.y; f.h[2] = a.z; f.h[3] = a.w;
    f.l[0] = b.x; f.l[1] = b.y; f.l[2] = b.z; f.l[3] = b.w;
}

// d0 += A B over k-step 0 and d1 += A B over k-step 1 of one 16-wide k group
// (two accumulators: independent MMA chains): ra / rb = the A rows g and
// g + 8, fb = the B column g (all loaded by ld_frag16 at the group's columns 4 q ..).
__device__ __forceinline__ void mma16(float (&d0)[4], float (&d1)[4], const Frag16& ra, const Frag16& rb,
                                      const Frag16& fb) {
#pragma unroll
    for (int st = 0; st < 2; ++st) {
        const uint32_t ah[4] = {ra.h[2 * st], rb.h[2 * st], ra.h[2 * st + 1], rb.h[2 * st + 1]};
        const uint32_t al[4] = {ra.l[2 * st], rb.l[2 * st], ra.l[2 * st + 1], rb.l[2 * st + 1]};
        mma3_tf32(st ? d1 : d0, ah, al, fb.h[2 * st], fb.h[2 * st + 1], fb.l[2 * st], fb.l[2 * st + 1]);
    }
}

// Shared memory of the sketch.  Two stages of raw chunks: G [kSkRows][kSkCols]
// in its own type, M [kSkRows][kSkCols] fp32 swizzled (its tf32 high part after
// the momentum phase, in place), Omega [kSkCols][KT + 4] fp32 (the pitch makes
// the transposing reads conflict-free).  One buffer each of the chunk's M low
// part (as M) and of Omega^T's high and low parts [KT][kSkCols] swizzled.
template <int KT, int G_DT>
struct SketchSmem {
    static constexpr int kOmLd = KT + 4;
    static constexpr int kG = kSkRows * kSkCols * g_size<G_DT>();
    static constexpr int kM = kSkRows * kSkCols * 4;
    static constexpr int kOm = kSkCols * kOmLd * 4;
    static constexpr int kStage = kG + kM + kOm;
    static constexpr int kMlo = 2 * kStage;
    static constexpr int kOtHi = kMlo + kSkRows * kSkCols * 4;
    static constexpr int kOtLo = kOtHi + KT * kSkCols * 4;
    static constexpr int kBytes = kOtLo + KT * kSkCols * 4;
    static_assert(kStage % 16 == 0 && kSkCols == 32, "16-byte aligned stages; one swizzled 32-word row per chunk row");
};

template <int KT, int G_DT>
__global__ void __launch_bounds__(kThreads, KT == 32 ? 2 : 1) lim_sketch(const __grid_constant__ LimParams p) {
    using S = SketchSmem<KT, G_DT>;
    constexpr int GSZ = g_size<G_DT>();
    constexpr int NT = KT / 8;                 // 8-column MMA tiles: a warp takes 16 rows x every column of Y
    static_assert(kSkRows == 16 * (kThreads / 32), "one 16-row MMA tile per warp");
    extern __shared__ __align__(16) unsigned char sm[];
    const LimEntry& E = p.e[find_entry(p, blockIdx.x, 0)];
    const int row0 = (blockIdx.x - E.t_sketch) * kSkRows;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, q4 = lane & 3;
    const int nchunks = (E.cols + kSkCols - 1) / kSkCols;
    const bool om_vec = (p.k & 3) == 0;       // Omega rows 16-byte aligned
    uint32_t* mlo = reinterpret_cast<uint32_t*>(sm + S::kMlo);
    uint32_t* oth = reinterpret_cast<uint32_t*>(sm + S::kOtHi);
    uint32_t* otl = reinterpret_cast<uint32_t*>(sm + S::kOtLo);
    float acc[2][NT][4];                      // the two k-steps of a group: independent chains
#pragma unroll
    for (int e = 0; e < 2; ++e)
#pragma unroll
        for (int t = 0; t < NT; ++t)
#pragma unroll
            for (int c = 0; c < 4; ++c) acc[e][t][c] = 0.f;
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
                cp_async16(ms + rr * kSkCols + swz(rr, pc * 4), E.M + (in ? (long long)i * E.cols + j : 0),
                           in ? 16u : 0u);
            }
        } else {
            for (int q = threadIdx.x; q < kSkRows * kSkCols; q += kThreads) {
                const int rr = q / kSkCols, cc = q % kSkCols, i = row0 + rr, j = c0 + cc;
                const bool in = i < E.rows && j < E.cols;
                const long long idx = (long long)i * E.cols + j;
                st_elem(gs, rr * kSkCols + cc, G_DT, in ? ld_elem(E.G, idx, G_DT) : 0.f);
                ms[rr * kSkCols + swz(rr, cc)] = in ? E.M[idx] : 0.f;
            }
        }
        if (om_vec) {
            constexpr int OP = KT / 4;
            for (int q = threadIdx.x; q < kSkCols * OP; q += kThreads) {
                const int jj = q / OP, pc = q % OP, j = c0 + jj;
                const bool in = j < E.cols && pc * 4 < p.k;
                cp_async16(os + jj * S::kOmLd + pc * 4, E.Omega + (in ? (long long)j * p.k + pc * 4 : 0),
                           in ? 16u : 0u);
            }
        } else {
            for (int q = threadIdx.x; q < kSkCols * KT; q += kThreads) {
                const int jj = q / KT, t = q % KT, j = c0 + jj;
                os[jj * S::kOmLd + t] = (j < E.cols && t < p.k) ? E.Omega[(long long)j * p.k + t] : 0.f;
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
            const int o = rr * kSkCols + swz(rr, cc);
            float4* mp = reinterpret_cast<float4*>(ms + o);
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
            *reinterpret_cast<uint4*>(mlo + o) = l;
        }
        // Omega^T high and low parts: a thread takes 4 consecutive columns t of one row jj
        for (int q = threadIdx.x; q < kSkCols * (KT / 4); q += kThreads) {
            const int jj = q % kSkCols, t0 = (q / kSkCols) * 4;
            const float4 v = *reinterpret_cast<const float4*>(os + jj * S::kOmLd + t0);
            const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int t = t0 + e, o = t * kSkCols + swz(t, jj);
                split_tf32(vv[e], oth[o], otl[o]);
            }
        }
        __syncthreads();
        // Y[16 warp + .., :] += M[rows, chunk] Omega[chunk, :]
        const uint32_t* mh = reinterpret_cast<const uint32_t*>(ms);
        const int ra = 16 * warp + g;          // rows ra and ra + 8 share a swizzle
#pragma unroll
        for (int kk = 0; kk < kSkCols; kk += 16) {
            const int co = swz(ra, kk + 4 * q4);
            Frag16 fa, fb;
            ld_frag16(fa, mh, mlo, ra * kSkCols + co);
            ld_frag16(fb, mh, mlo, (ra + 8) * kSkCols + co);
#pragma unroll
            for (int t = 0; t < NT; ++t) {
                const int n = 8 * t + g;
                Frag16 fo;
                ld_frag16(fo, oth, otl, n * kSkCols + swz(n, kk + 4 * q4));
                mma16(acc[0][t], acc[1][t], fa, fb, fo);
            }
        }
        __syncthreads();                       // stage s and the split buffers free for the next chunks
    }
    // Y to the workspace, and this block's rows' share of Y^T Y
    float* ys = reinterpret_cast<float*>(sm);  // [kSkRows][KT]
#pragma unroll
    for (int t = 0; t < NT; ++t) {
        const int col = 8 * t + 2 * q4;
        *reinterpret_cast<float2*>(ys + (16 * warp + g) * KT + col) =
            make_float2(acc[0][t][0] + acc[1][t][0], acc[0][t][1] + acc[1][t][1]);
        *reinterpret_cast<float2*>(ys + (16 * warp + g + 8) * KT + col) =
            make_float2(acc[0][t][2] + acc[1][t][2], acc[0][t][3] + acc[1][t][3]);
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
// 3 / 6. rows times the matrix's k x k factor K, in place (fp64 sums): step 3
//    reads Y and forms Q = Y R^-1, step 6 reads Q (high + low parts) and forms
//    Z = Q P.  The result is stored as its tf32 high and low parts, the
//    operands of the tensor-core products that read it.
// ---------------------------------------------------------------------------
template <int KT, bool FROM_SPLIT>
__global__ void __launch_bounds__(kThreads) lim_rowmul(const __grid_constant__ LimParams p) {
    __shared__ double Ks[KT * KT];
    const LimEntry& E = p.e[find_entry(p, blockIdx.x, 1)];
    for (int idx = threadIdx.x; idx < KT * KT; idx += kThreads) Ks[idx] = E.K[idx];
    __syncthreads();
    const int i = (blockIdx.x - E.t_rows) * kThreads + threadIdx.x;
    if (i >= E.rows) return;
    float* row = E.Y + (long long)i * KT;
    float* rlo = E.Ylo + (long long)i * KT;
    float y[KT];
#pragma unroll
    for (int t = 0; t < KT; t += 4) {
        const float4 v = *reinterpret_cast<const float4*>(row + t);
        y[t] = v.x; y[t + 1] = v.y; y[t + 2] = v.z; y[t + 3] = v.w;
        if (FROM_SPLIT) {
            const float4 w = *reinterpret_cast<const float4*>(rlo + t);
            y[t] += w.x; y[t + 1] += w.y; y[t + 2] += w.z; y[t + 3] += w.w;
        }
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
        uint4 h, l;
        split_tf32((float)s0, h.x, l.x);
        split_tf32((float)s1, h.y, l.y);
        split_tf32((float)s2, h.z, l.z);
        split_tf32((float)s3, h.w, l.w);
        *reinterpret_cast<uint4*>(row + j) = h;
        *reinterpret_cast<uint4*>(rlo + j) = l;
    }
}

// ---------------------------------------------------------------------------
// 4. B^T = M^T Q (+ share of B B^T)
// ---------------------------------------------------------------------------
// Shared memory of the projection: kPjStages stages of M rows [kPjRows][kPjLd]
// (the block's columns) and of Q's high and low parts [kPjRows][KT + 8].  The
// pitches (8 words past a multiple of 32) make the fragment loads
// conflict-free.
constexpr int kPjLd = kPjCols + 8;

template <int KT>
struct ProjSmem {
    static constexpr int kQLd = KT + 8;
    static constexpr int kM = kPjRows * kPjLd * 4;
    static constexpr int kQ = kPjRows * kQLd * 4;
    static constexpr int kStage = kM + 2 * kQ;
    static constexpr int kBytes = kPjStages * kStage;
    static_assert(kStage % 16 == 0, "16-byte aligned stages");
};

// Block b of the projection: column block cb of its matrix and row segment
// seg (rows seg * kPjSegRows ..).  A matrix with more rows than one segment
// has each segment's partial B^T written to Bpart; the segment that finishes
// a column block last (counted in pj_count) adds the partials in segment
// order and finishes the block: the same sums in the same order on every run.
template <int KT>
__global__ void __launch_bounds__(kThreads, 2) lim_project(const __grid_constant__ LimParams p) {
    using S = ProjSmem<KT>;
    constexpr int NT = KT / 8;                 // 8-column MMA tiles: a warp takes every column of Q
    static_assert(kPjCols == 16 * (kThreads / 32), "one 16-column MMA tile of M per warp");
    extern __shared__ __align__(16) unsigned char sm[];
    __shared__ int last;
    const LimEntry& E = p.e[find_entry(p, blockIdx.x, 2)];
    const int local = blockIdx.x - E.t_proj, cb = local / E.nseg, seg = local % E.nseg;
    const int c0 = cb * kPjCols;
    const int r_begin = seg * kPjSegRows, r_end = min(E.rows, r_begin + kPjSegRows);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, q4 = lane & 3;
    const int nchunks = (r_end - r_begin + kPjRows - 1) / kPjRows;
    // two accumulator sets, for the even and the odd k-steps: twice as many
    // independent MMA chains (each k-step is three dependent MMAs per tile)
    float acc[2][NT][4];
#pragma unroll
    for (int e = 0; e < 2; ++e)
#pragma unroll
        for (int t = 0; t < NT; ++t)
#pragma unroll
            for (int h = 0; h < 4; ++h) acc[e][t][h] = 0.f;

    // rows i0.. of M (this block's columns) and of Q's two parts into stage s
    auto issue = [&](int ch, int s) {
        const int i0 = r_begin + ch * kPjRows;
        float* ms = reinterpret_cast<float*>(sm + s * S::kStage);
        float* qh = reinterpret_cast<float*>(sm + s * S::kStage + S::kM);
        float* ql = reinterpret_cast<float*>(sm + s * S::kStage + S::kM + S::kQ);
        if (E.vec_ok) {
            constexpr int MP = kPjCols / 4;
            for (int q = threadIdx.x; q < kPjRows * MP; q += kThreads) {
                const int rr = q / MP, pc = q % MP, i = i0 + rr, j = c0 + pc * 4;
                const bool in = i < r_end && j < E.cols;
                cp_async16(ms + rr * kPjLd + pc * 4, E.M + (in ? (long long)i * E.cols + j : 0), in ? 16u : 0u);
            }
        } else {
            for (int q = threadIdx.x; q < kPjRows * kPjCols; q += kThreads) {
                const int rr = q / kPjCols, cc = q % kPjCols, i = i0 + rr, j = c0 + cc;
                ms[rr * kPjLd + cc] = (i < r_end && j < E.cols) ? E.M[(long long)i * E.cols + j] : 0.f;
            }
        }
        constexpr int QP = KT / 4;
        for (int q = threadIdx.x; q < 2 * kPjRows * QP; q += kThreads) {
            const int part = q / (kPjRows * QP), r = q % (kPjRows * QP), rr = r / QP, pc = r % QP, i = i0 + rr;
            const bool in = i < r_end;
            const float* src = (part ? E.Ylo : E.Y) + (in ? (long long)i * KT + pc * 4 : 0);
            cp_async16((part ? ql : qh) + rr * S::kQLd + pc * 4, src, in ? 16u : 0u);
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
        const uint32_t* qh = reinterpret_cast<const uint32_t*>(sm + (ch % kPjStages) * S::kStage + S::kM);
        const uint32_t* ql = reinterpret_cast<const uint32_t*>(sm + (ch % kPjStages) * S::kStage + S::kM + S::kQ);
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
                mma3_tf32(acc[(kk >> 3) & 1][t], ah, al, qh[b0], qh[b0 + 4 * S::kQLd], ql[b0], ql[b0 + 4 * S::kQLd]);
            }
        }
        __syncthreads();                       // this stage is refilled next
    }
    cp_async_wait<0>();
    float* bs = reinterpret_cast<float*>(sm);  // [kPjCols][KT]
#pragma unroll
    for (int t = 0; t < NT; ++t) {
        const int col = 8 * t + 2 * q4;
        *reinterpret_cast<float2*>(bs + (16 * warp + g) * KT + col) =
            make_float2(acc[0][t][0] + acc[1][t][0], acc[0][t][1] + acc[1][t][1]);
        *reinterpret_cast<float2*>(bs + (16 * warp + g + 8) * KT + col) =
            make_float2(acc[0][t][2] + acc[1][t][2], acc[0][t][3] + acc[1][t][3]);
    }
    __syncthreads();
    if (E.nseg > 1) {                          // uniform over the block
        float* part = E.Bpart + ((long long)seg * E.cols + c0) * KT;
        for (int q = threadIdx.x; q < kPjCols * (KT / 4); q += kThreads) {
            const int cc = q / (KT / 4), pc = q % (KT / 4);
            if (c0 + cc < E.cols)
                *reinterpret_cast<float4*>(part + cc * KT + 4 * pc) = *reinterpret_cast<const float4*>(bs + cc * KT + 4 * pc);
        }
        __threadfence();                       // this segment's partial visible before it is counted
        __syncthreads();
        if (threadIdx.x == 0) last = atomicAdd(E.pj_count + cb, 1) == E.nseg - 1;
        __syncthreads();
        if (!last) return;
        __threadfence();                       // the other segments' partials, counted before ours
        for (int q = threadIdx.x; q < kPjCols * (KT / 4); q += kThreads) {
            const int cc = q / (KT / 4), pc = q % (KT / 4);
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            if (c0 + cc < E.cols)
                for (int sg = 0; sg < E.nseg; ++sg) {
                    const float4 w = __ldcg(reinterpret_cast<const float4*>(
                        E.Bpart + ((long long)sg * E.cols + c0 + cc) * KT + 4 * pc));
                    v.x += w.x; v.y += w.y; v.z += w.z; v.w += w.w;
                }
            *reinterpret_cast<float4*>(bs + cc * KT + 4 * pc) = v;
        }
        __syncthreads();
    }
    // B^T (high and low parts) to the workspace, and this block's columns' share of B B^T
    for (int q = threadIdx.x; q < kPjCols * (KT / 4); q += kThreads) {
        const int cc = q / (KT / 4), pc = q % (KT / 4), j = c0 + cc;
        if (j < E.cols) {
            const float4 v = *reinterpret_cast<const float4*>(bs + cc * KT + 4 * pc);
            uint4 h, l;
            split_tf32(v.x, h.x, l.x);
            split_tf32(v.y, h.y, l.y);
            split_tf32(v.z, h.z, l.z);
            split_tf32(v.w, h.w, l.w);
            *reinterpret_cast<uint4*>(E.Bt + (long long)j * KT + 4 * pc) = h;
            *reinterpret_cast<uint4*>(E.Btlo + (long long)j * KT + 4 * pc) = l;
        }
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
    constexpr int NP = KT / 2, NR = KT - 1;   // pairs per round, rounds per sweep (on all KT indices)
    extern __shared__ __align__(16) double dsm[];
    double* C = dsm;                    // [KT][LD]
    double* Ev = dsm + KT * LD;         // [KT][LD] eigenvectors (columns)
    double* cs = Ev + KT * LD;          // [NP] cosines
    double* sn = cs + NP;               // [NP] sines
    double* lam = sn + NP;              // [KT] eigenvalues
    unsigned char* pa = reinterpret_cast<unsigned char*>(lam + KT);   // [NR][NP] pair tables
    unsigned char* pb = pa + NR * NP;
    __shared__ int rotated, nonfinite;
    const LimEntry& E = p.e[blockIdx.x];
    const int k = p.k;
    if (threadIdx.x == 0) nonfinite = 0;
    __syncthreads();
    // C padded to KT x KT with zeros: indices >= k never rotate (their couplings are 0)
    for (int idx = threadIdx.x; idx < KT * KT; idx += blockDim.x) {
        const int a = idx / KT, b = idx % KT;
        const double v = (a < k && b < k) ? (a <= b ? E.Cg[a * KT + b] : E.Cg[b * KT + a]) : 0.0;
        if (!isfinite(v)) nonfinite = 1;
        C[a * LD + b] = v;
        Ev[a * LD + b] = a == b ? 1.0 : 0.0;
    }
    // round-robin schedule: in round rd, pair 0 is (NR, rd) and pair i is
    // ((rd + i) mod NR, (rd - i) mod NR); every index pair meets once a sweep
    for (int idx = threadIdx.x; idx < NR * NP; idx += blockDim.x) {
        const int rd = idx / NP, i = idx % NP;
        int a = i == 0 ? NR : (rd + i) % NR, b = i == 0 ? rd : (rd - i + NR) % NR;
        if (a > b) { const int t = a; a = b; b = t; }
        pa[idx] = (unsigned char)a;
        pb[idx] = (unsigned char)b;
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
    for (int sweep = 0; sweep < kMaxSweeps; ++sweep) {
        if (threadIdx.x == 0) rotated = 0;
        __syncthreads();
        for (int rd = 0; rd < NR; ++rd) {
            const unsigned char* ra = pa + rd * NP;
            const unsigned char* rb = pb + rd * NP;
            if (threadIdx.x < NP) {
                const int i = threadIdx.x, a = ra[i], b = rb[i];
                const double apq = C[a * LD + b], app = C[a * LD + a], aqq = C[b * LD + b];
                double c = 1.0, s = 0.0;
                if (apq * apq > kRotTol * kRotTol * fabs(app * aqq) && fabs(apq) > floor_abs) {
                    // the textbook rotation t = sign(tau) / (|tau| + sqrt(1 + tau^2)),
                    // tau = d / (2 apq), d = aqq - app, multiplied through by 2 |apq|:
                    // one square root, one division and one reciprocal square root
                    const double d = aqq - app;
                    const double t = (d >= 0.0 ? 2.0 : -2.0) * apq / (fabs(d) + sqrt(d * d + 4.0 * apq * apq));
                    c = rsqrt(1.0 + t * t);
                    s = t * c;
                    rotated = 1;
                }
                cs[i] = c; sn[i] = s;
            }
            __syncthreads();
#pragma unroll
            for (int it = 0; it < (NP * NP + kThreads - 1) / kThreads; ++it) {   // C <- J^T C J, block by block
                const int idx = threadIdx.x + it * kThreads;
                if (idx >= NP * NP) break;
                const int i = idx / NP, j = idx % NP;
                const double c1 = cs[i], s1 = sn[i], c2 = cs[j], s2 = sn[j];
                if (s1 == 0.0 && s2 == 0.0) continue;
                const int a1 = ra[i], b1 = rb[i], a2 = ra[j], b2 = rb[j];
                const double x = C[a1 * LD + a2], y = C[a1 * LD + b2], z = C[b1 * LD + a2], w = C[b1 * LD + b2];
                const double r0 = c1 * x - s1 * z, r1 = c1 * y - s1 * w;   // rows a1, b1 rotated
                const double r2 = s1 * x + c1 * z, r3 = s1 * y + c1 * w;
                C[a1 * LD + a2] = c2 * r0 - s2 * r1;                      // then columns a2, b2
                C[a1 * LD + b2] = s2 * r0 + c2 * r1;
                C[b1 * LD + a2] = c2 * r2 - s2 * r3;
                C[b1 * LD + b2] = s2 * r2 + c2 * r3;
            }
#pragma unroll
            for (int it = 0; it < (KT * NP + kThreads - 1) / kThreads; ++it) {   // E <- E J
                const int idx = threadIdx.x + it * kThreads;
                if (idx >= KT * NP) break;
                const int row = idx / NP, i = idx % NP;
                const double c = cs[i], s = sn[i];
                if (s == 0.0) continue;
                const int a = ra[i], b = rb[i];
                const double u = Ev[row * LD + a], v = Ev[row * LD + b];
                Ev[row * LD + a] = c * u - s * v;
                Ev[row * LD + b] = s * u + c * v;
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
// Shared memory of lim_update (1024-byte aligned): the high and low parts of
// Z's rows [kUpRows] and of the B^T rows of the tile's columns [kUpCols], each
// K-major with KT words per row in 128-byte swizzled atoms; then the tile of W
// [kUpRows] rows of kUpCols elements plus 16 bytes (rows 16 bytes apart in the
// banks: the epilogue's row-per-lane accesses are conflict-free).
template <int KT, int W_DT>
struct UpdSmem {
    static constexpr int kA = kUpRows * KT * 4, kB = kUpCols * KT * 4;
    static constexpr int kAh = 0, kAl = kA, kBh = 2 * kA, kBl = 2 * kA + kB, kW = 2 * kA + 2 * kB;
    static constexpr int kWRow = kUpCols * g_size<W_DT>() + 16;
    static constexpr int kBytes = kW + kUpRows * kWRow + 1024;   // + the alignment slack
    static_assert(KT % 32 == 0, "whole 128-byte atoms");
};

// 7. O = Z B on a 128 x 128 tile: one thread issues the tf32 MMAs (K = 8
// each, three per k-step for the split parts) while the tile of W streams into
// shared memory; eight warps read the fp32 accumulator from tensor memory (a
// lane quadrant and half of the columns each) and write W row-wise, 16-byte
// pieces where aligned.
template <int KT, int W_DT>
__global__ void __launch_bounds__(kThreads, 2) lim_update(const __grid_constant__ LimParams p) {
    using S = UpdSmem<KT, W_DT>;
    constexpr int WSZ = g_size<W_DT>();
    constexpr int ZP = KT / 4;                 // 16-byte pieces per row of Z / B^T
    constexpr uint32_t kTmemCols = kUpCols;
    extern __shared__ uint8_t sm_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(sm_raw) + 1023) & ~uintptr_t(1023));
    __shared__ __align__(8) uint64_t done_bar;
    __shared__ uint32_t tmem_slot;
    __shared__ int abort_flag;
    const LimEntry& E = p.e[find_entry(p, blockIdx.x, 3)];
    const int tile = blockIdx.x - E.t_upd;
    const int tiles_c = (E.cols + kUpCols - 1) / kUpCols;
    const int row0 = (tile / tiles_c) * kUpRows, c0 = (tile % tiles_c) * kUpCols;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const bool skip = *E.bad != 0;
    const bool wtile = E.vec_ok && !skip;      // W through shared memory (16-byte pieces)
    if (threadIdx.x == 0) {
        mbar_init(&done_bar, 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(&tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    // the two parts of Z's rows and of the tile's B^T rows, swizzled for the MMA
    for (int q = threadIdx.x; q < 2 * (kUpRows + kUpCols) * ZP; q += kThreads) {
        const int part = q / ((kUpRows + kUpCols) * ZP), r0 = q % ((kUpRows + kUpCols) * ZP);
        const bool is_a = r0 < kUpRows * ZP;
        const int r = (is_a ? r0 : r0 - kUpRows * ZP) / ZP, pc = (is_a ? r0 : r0 - kUpRows * ZP) % ZP;
        const int idx = is_a ? row0 + r : c0 + r;
        const bool in = idx < (is_a ? E.rows : E.cols);
        const float* base = is_a ? (part ? E.Ylo : E.Y) : (part ? E.Btlo : E.Bt);
        const int off = (is_a ? (part ? S::kAl : S::kAh) : (part ? S::kBl : S::kBh)) +
                        sw128_piece(r, pc, is_a ? kUpRows : kUpCols);
        cp_async16(sm + off, base + (in ? (long long)idx * KT + pc * 4 : 0), in ? 16u : 0u);
    }
    cp_async_commit();
    if (wtile) {                               // its own group: waited for after the MMAs are issued
        constexpr int WP = kUpCols * WSZ / 16, WE = 16 / WSZ;   // 16-byte pieces per row, elements per piece
        for (int q = threadIdx.x; q < kUpRows * WP; q += kThreads) {
            const int rr = q / WP, pc = q % WP, i = row0 + rr, j = c0 + pc * WE;
            const bool in = i < E.rows && j < E.cols;
            const char* src = static_cast<const char*>(E.W) + (in ? ((long long)i * E.cols + j) * WSZ : 0);
            cp_async16(sm + S::kW + rr * S::kWRow + pc * 16, src, in ? 16u : 0u);
        }
    }
    cp_async_commit();
    cp_async_wait<1>();                        // the operands (the W tile may still be in flight)
    fence_proxy_async_smem();                  // the copies, visible to the tensor cores
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_slot;
    if (threadIdx.x == 0) {
        constexpr uint32_t idesc = idesc_tf32(0, 0, kUpRows, kUpCols);
        const uint32_t base = smem_u32(sm);
        const int nks = (p.k + 7) / 8;         // columns of Z (and of B^T) past k are zero
        for (int ks = 0; ks < nks; ++ks) {
            const uint32_t ao = (ks >> 2) * (kUpRows * 128) + (ks & 3) * 32;
            const uint32_t bo = (ks >> 2) * (kUpCols * 128) + (ks & 3) * 32;
            const uint64_t ah = smem_desc_sw128(base + S::kAh + ao, 16, 1024);
            const uint64_t al = smem_desc_sw128(base + S::kAl + ao, 16, 1024);
            const uint64_t bh = smem_desc_sw128(base + S::kBh + bo, 16, 1024);
            const uint64_t bl = smem_desc_sw128(base + S::kBl + bo, 16, 1024);
            tc_mma_tf32(tmem, ah, bl, idesc, ks > 0 ? 1u : 0u);   // small terms first
            tc_mma_tf32(tmem, al, bh, idesc, 1u);
            tc_mma_tf32(tmem, ah, bh, idesc, 1u);
        }
        tc_commit(&done_bar);
    }
    __syncwarp();
    cp_async_wait<0>();                        // this thread's pieces of the W tile
    __syncthreads();                           // everyone's
    if (mbar_wait(&done_bar, 0, &abort_flag, p.d_status)) {
        tc_fence_after();
        // epilogue: warp w reads lanes 32 (w % 4).. (rows) and columns 64 (w / 4)..
        const int q = warp & 3, h = warp >> 2, rr = 32 * q + lane, i = row0 + rr;
#pragma unroll 1
        for (int ch = 0; ch < 2; ++ch) {
            const int cc = 64 * h + 32 * ch, j0 = c0 + cc;
            float v[32];
            tmem_ld_32x32b_x32(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)cc, v);   // whole warp
            if (i >= E.rows || j0 >= E.cols) continue;
            const long long idx = (long long)i * E.cols + j0;
            const int nv = min(32, E.cols - j0);
            if (E.O_out) {
                if (E.vec_ok) {                // cols % 8 == 0: 8-column pieces are whole
#pragma unroll
                    for (int e = 0; e < 32; e += 4)
                        if (e < nv)
                            *reinterpret_cast<float4*>(E.O_out + idx + e) = make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        if (e < nv) E.O_out[idx + e] = v[e];
                }
            }
            if (skip) continue;
            const uint8_t* ws = sm + S::kW + rr * S::kWRow + cc * WSZ;    // this row's staged W
            if (E.vec_ok && W_DT != DT_FP32) {
                using T = typename std::conditional<W_DT == DT_BF16, __nv_bfloat16, __half>::type;
                uint4* wp = reinterpret_cast<uint4*>(static_cast<uint16_t*>(E.W) + idx);
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    if (8 * u >= nv) continue;
                    const uint4 x = reinterpret_cast<const uint4*>(ws)[u];
                    const uint32_t xw[4] = {x.x, x.y, x.z, x.w};
                    uint32_t r[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        float w0 = unpack_lo<T>(xw[e]), w1 = unpack_hi<T>(xw[e]);
                        w0 = w0 - p.eta * (E.gamma * v[8 * u + 2 * e] + p.lambda * w0);
                        w1 = w1 - p.eta * (E.gamma * v[8 * u + 2 * e + 1] + p.lambda * w1);
                        r[e] = pack2<T>(w0, w1);
                    }
                    wp[u] = make_uint4(r[0], r[1], r[2], r[3]);
                }
            } else if (E.vec_ok) {
                float4* wp = reinterpret_cast<float4*>(static_cast<float*>(E.W) + idx);
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    if (4 * u >= nv) continue;
                    float4 w = reinterpret_cast<const float4*>(ws)[u];
                    w.x = w.x - p.eta * (E.gamma * v[4 * u] + p.lambda * w.x);
                    w.y = w.y - p.eta * (E.gamma * v[4 * u + 1] + p.lambda * w.y);
                    w.z = w.z - p.eta * (E.gamma * v[4 * u + 2] + p.lambda * w.z);
                    w.w = w.w - p.eta * (E.gamma * v[4 * u + 3] + p.lambda * w.w);
                    wp[u] = w;
                }
            } else {
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    if (e >= nv) continue;
                    const float w = ld_elem(E.W, idx + e, W_DT);
                    st_elem(E.W, idx + e, W_DT, w - p.eta * (E.gamma * v[e] + p.lambda * w));
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
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
constexpr size_t eig_smem() { return sizeof(double) * (2 * KT * (KT + 1) + KT / 2 * 2 + KT) + 2 * (KT - 1) * (KT / 2); }

static_assert(sketch_smem<64, DT_FP32>() >= sizeof(float) * kSkRows * 64, "sketch Y staging fits");
static_assert(project_smem<64>() >= sizeof(float) * kPjCols * 64, "projection B^T staging fits the stages");
static_assert(sketch_smem<64, DT_FP32>() <= 227 * 1024 && update_smem<64, DT_FP32>() <= 227 * 1024,
              "shared memory per block");

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
    trace_begin(MUON_KERNEL_RSVD_SMALL, 12.0 * L.rows_total * KT + kk, s);          // Y read, Q's parts written
    lim_rowmul<KT, false><<<L.rows, kThreads, 0, s>>>(prm);
    trace_end(s);
    trace_begin(MUON_KERNEL_RSVD, L.elems * 4.0 + 8.0 * (L.rows_k + L.cols_k), s);  // M, Q read; B^T written
    lim_project<KT><<<L.proj, kThreads, project_smem<KT>(), s>>>(prm);
    trace_end(s);
    trace_begin(MUON_KERNEL_RSVD_SMALL, 2.0 * kk, s);                                // Gram read, P written
    lim_eig<KT><<<prm.n, kThreads, eig_smem<KT>(), s>>>(prm);
    trace_end(s);
    trace_begin(MUON_KERNEL_RSVD_SMALL, 16.0 * L.rows_total * KT + kk, s);          // Q's parts read, Z's written
    lim_rowmul<KT, true><<<L.rows, kThreads, 0, s>>>(prm);
    trace_end(s);
    trace_begin(MUON_KERNEL_RSVD, L.elems * 2.0 * wsz + 8.0 * (L.rows_k + L.cols_k), s);   // W read and written
    lim_update<KT, W_DT><<<L.upd, kThreads, update_smem<KT, W_DT>(), s>>>(prm);
    trace_end(s);
    (void)k;
    return cudaGetLastError() == cudaSuccess ? MUON_OK : MUON_ERR_CUDA;
}

int proj_segments(int rows) { return (rows + kPjSegRows - 1) / kPjSegRows; }
int proj_col_blocks(int cols) { return (cols + kPjCols - 1) / kPjCols; }

// Per matrix: Y and its low parts (rows x KT each), B^T and its low parts
// (cols x KT each), and with more than one projection segment the partial B^T
// of every segment (nseg x cols x KT).
size_t matrix_ws(int rows, int cols, int KT) {
    const int nseg = proj_segments(rows);
    return 2 * align256(sizeof(float) * (size_t)rows * KT) + 2 * align256(sizeof(float) * (size_t)cols * KT) +
           (nseg > 1 ? align256(sizeof(float) * (size_t)nseg * cols * KT) : 0);
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

// Workspace: the per-matrix flags, the projection's per-column-block segment
// counters, then the k x k sums (all these start at zero: Y^T Y, B B^T), then
// the k x k factors, then the per-matrix arrays.
struct WsLayout {
    size_t flags, counts, zero_bytes, gy, cg, kf, mats, total;
};

WsLayout ws_layout(const muon_rsvd_param* params, int n, int KT) {
    WsLayout L;
    const size_t kk = sizeof(double) * (size_t)KT * KT * n;
    size_t ncount = 0;
    for (int i = 0; i < n; ++i)
        if (proj_segments(params[i].rows) > 1) ncount += proj_col_blocks(params[i].cols);
    L.flags = 0;
    L.counts = align256(sizeof(int) * (size_t)n);
    L.gy = L.counts + (ncount ? align256(sizeof(int) * ncount) : 0);
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
    int* counts = reinterpret_cast<int*>(ws + W.counts);
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
            const size_t yb = align256(sizeof(float) * (size_t)q.rows * KT);
            const size_t bb = align256(sizeof(float) * (size_t)q.cols * KT);
            E.Y = reinterpret_cast<float*>(cur);
            E.Ylo = reinterpret_cast<float*>(cur + yb);
            E.Bt = reinterpret_cast<float*>(cur + 2 * yb);
            E.Btlo = reinterpret_cast<float*>(cur + 2 * yb + bb);
            E.nseg = proj_segments(q.rows);
            E.Bpart = E.nseg > 1 ? reinterpret_cast<float*>(cur + 2 * yb + 2 * bb) : nullptr;
            E.pj_count = nullptr;
            if (E.nseg > 1) {
                E.pj_count = counts;
                counts += proj_col_blocks(q.cols);
            }
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
                else if (w == 2) { E.t_proj = (int)first; tot[w] += (long long)proj_col_blocks(E.cols) * E.nseg; }
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
