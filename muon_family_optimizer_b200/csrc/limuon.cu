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
// Five launches per batch of up to 128 matrices (k = r + p <= 64, templated
// on KT = 32 or 64 columns):
//   1 lim_sketch   fused momentum pass and Y = M Omega: reads G and M, writes
//                  M (10 bytes per element for 16-bit G), k FMAs per element.
//   2 lim_qr       per matrix, one block: Q = Y R^-1 by Cholesky QR in fp64
//                  (Gram Y^T Y, Cholesky; a column whose pivot falls to 1e-10
//                  of its squared norm lies in the span of the previous ones
//                  and is dropped: its Q column is zero).
//   3 lim_project  B^T = M^T Q: reads M once more (4 bytes per element).
//   4 lim_factor   per matrix, one block, fp64: C = B B^T = E L E^T by cyclic
//                  Jacobi in parallel (round-robin) order; with the r largest
//                  eigenvalues, O = Q E_r L_r^{-1/2} E_r^T B, so the kernel
//                  forms Z = Q P, P = E_r L_r^{-1/2} E_r^T, in Q's place.
//   5 lim_update   O = Z B row tile by row tile, fused with the weight update
//                  (reads and writes W: 4 bytes per element for 16-bit W).
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
constexpr int kSketchRows = 64;   // lim_sketch: rows per block
constexpr int kChunk = 128;       // columns per smem chunk (sketch, project, update)
constexpr int kMsLd = kChunk + 4; // padded row of a staged M tile
constexpr int kProjRows = 32;     // lim_project: rows per chunk
constexpr int kUpdRows = 32;      // lim_update: rows per tile
constexpr int kGramRows = 64;     // rows of Y / B^T staged per Gram chunk
constexpr double kDrop = 1e-10;   // Cholesky pivot / squared column norm below which a column is dropped
constexpr double kTau2 = 1e-10;   // (singular value / largest)^2 at or below which it counts as zero
constexpr int kMaxSweeps = 30;
constexpr int kMaxDevices = 64;    // devices whose kernel attributes are tracked

struct LimEntry {
    void* W; const void* G; float* M; const float* Omega; float* O_out;
    float* Y;        // rows x KT workspace: Y, then Q, then Z
    float* Bt;       // cols x KT workspace: B^T
    int* bad;        // this matrix's non-finite flag (workspace)
    int rows, cols;
    float gamma;
    int vec_ok;      // W, G, M 16-byte aligned and cols % 8 == 0
    int t_sketch, t_proj, t_upd;   // first block of this matrix in each launch's grid
};

struct LimParams {
    LimEntry e[kLimMax];
    int n, k, r;
    float mu, eta, lambda;
    int* d_status;
};

__device__ __forceinline__ int find_entry(const LimParams& p, int b, int which) {
    int lo = 0, hi = p.n - 1;        // last entry whose first block is <= b
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        const int t = which == 0 ? p.e[mid].t_sketch : which == 1 ? p.e[mid].t_proj : p.e[mid].t_upd;
        if (t <= b) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// ---------------------------------------------------------------------------
// 1. momentum + sketch
// ---------------------------------------------------------------------------
template <int KT, int G_DT>
__global__ void __launch_bounds__(kThreads) lim_sketch(const __grid_constant__ LimParams p) {
    constexpr int H = KT / 32;
    extern __shared__ __align__(16) float smem[];
    float* Ms = smem;                              // [kSketchRows][kMsLd]
    float* Os = smem + kSketchRows * kMsLd;        // [kChunk][KT]
    const LimEntry& E = p.e[find_entry(p, blockIdx.x, 0)];
    const int row0 = (blockIdx.x - E.t_sketch) * kSketchRows;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float acc[8][H];
#pragma unroll
    for (int r = 0; r < 8; ++r)
#pragma unroll
        for (int h = 0; h < H; ++h) acc[r][h] = 0.f;
    bool bad = false;
    for (int c0 = 0; c0 < E.cols; c0 += kChunk) {
#pragma unroll 1
        for (int pass = 0; pass < kSketchRows * kChunk / (8 * kThreads); ++pass) {
            const int g = threadIdx.x + kThreads * pass;
            const int rr = g >> 4, cc = (g & 15) * 8;
            const int i = row0 + rr, j = c0 + cc;
            float m[8];
            if (i < E.rows && j < E.cols) {
                const long long idx = (long long)i * E.cols + j;
                const int nvalid = min(8, E.cols - j);
                const bool vec = E.vec_ok && nvalid == 8;
                float g8[8];
                load8_dt(E.G, idx, G_DT, vec, nvalid, g8);
                load8_dt(E.M, idx, DT_FP32, vec, nvalid, m);
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    m[q] = q < nvalid ? fmaf(p.mu, m[q], g8[q]) : 0.f;
                    bad |= !isfinite(m[q]);
                }
                store8_dt(E.M, idx, DT_FP32, vec, nvalid, m);
            } else {
#pragma unroll
                for (int q = 0; q < 8; ++q) m[q] = 0.f;
            }
            float4* dst = reinterpret_cast<float4*>(Ms + rr * kMsLd + cc);
            dst[0] = make_float4(m[0], m[1], m[2], m[3]);
            dst[1] = make_float4(m[4], m[5], m[6], m[7]);
        }
        for (int idx = threadIdx.x; idx < kChunk * KT; idx += kThreads) {
            const int jj = idx / KT, t = idx % KT;
            Os[idx] = (t < p.k && c0 + jj < E.cols) ? E.Omega[(long long)(c0 + jj) * p.k + t] : 0.f;
        }
        __syncthreads();
#pragma unroll 2
        for (int jj = 0; jj < kChunk; jj += 4) {
            float om[4][H];
#pragma unroll
            for (int q = 0; q < 4; ++q)
#pragma unroll
                for (int h = 0; h < H; ++h) om[q][h] = Os[(jj + q) * KT + lane + 32 * h];
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                const float4 mv = *reinterpret_cast<const float4*>(Ms + (8 * warp + r) * kMsLd + jj);
#pragma unroll
                for (int h = 0; h < H; ++h) {
                    acc[r][h] = fmaf(mv.x, om[0][h], acc[r][h]);
                    acc[r][h] = fmaf(mv.y, om[1][h], acc[r][h]);
                    acc[r][h] = fmaf(mv.z, om[2][h], acc[r][h]);
                    acc[r][h] = fmaf(mv.w, om[3][h], acc[r][h]);
                }
            }
        }
        __syncthreads();
    }
#pragma unroll
    for (int r = 0; r < 8; ++r) {
        const int i = row0 + 8 * warp + r;
        if (i >= E.rows) continue;
#pragma unroll
        for (int h = 0; h < H; ++h) E.Y[(long long)i * KT + lane + 32 * h] = acc[r][h];
    }
    if (__syncthreads_or(bad) && threadIdx.x == 0) {
        atomicOr(E.bad, 1);
        if (p.d_status) atomicOr(p.d_status, MUON_FLAG_NONFINITE);
    }
}

// ---------------------------------------------------------------------------
// Gram matrix G = X^T X (k x k, fp64) of an n x KT fp32 array (columns >= k
// ignored), into Gm[KT * KT] (shared); stage: kGramRows x KT floats (shared).
// ---------------------------------------------------------------------------
template <int KT>
__device__ void gram_fp64(const float* X, int n, int k, double* Gm, float* stage) {
    constexpr int NE = KT * (KT + 1) / 2;
    constexpr int PER = (NE + kThreads - 1) / kThreads;
    int ea[PER], eb[PER];
    double acc[PER];
#pragma unroll
    for (int q = 0; q < PER; ++q) {
        // entry e -> (a, b), a <= b, row-major over the upper triangle
        int e = threadIdx.x + kThreads * q, a = 0;
        if (e < NE) {
            while (e >= KT - a) { e -= KT - a; ++a; }
            ea[q] = a; eb[q] = a + e;
        } else {
            ea[q] = eb[q] = -1;
        }
        acc[q] = 0.0;
    }
    for (int r0 = 0; r0 < n; r0 += kGramRows) {
        __syncthreads();
        for (int idx = threadIdx.x; idx < kGramRows * KT; idx += kThreads) {
            const int rr = idx / KT, t = idx % KT;
            stage[idx] = (r0 + rr < n && t < k) ? X[(long long)(r0 + rr) * KT + t] : 0.f;
        }
        __syncthreads();
        const int nr = min(kGramRows, n - r0);
#pragma unroll
        for (int q = 0; q < PER; ++q) {
            if (ea[q] < 0) continue;
            double s = 0.0;
            for (int rr = 0; rr < nr; ++rr)
                s = fma((double)stage[rr * KT + ea[q]], (double)stage[rr * KT + eb[q]], s);
            acc[q] += s;
        }
    }
#pragma unroll
    for (int q = 0; q < PER; ++q)
        if (ea[q] >= 0) {
            Gm[ea[q] * KT + eb[q]] = acc[q];
            Gm[eb[q] * KT + ea[q]] = acc[q];
        }
    __syncthreads();
}

// ---------------------------------------------------------------------------
// 2. Cholesky QR (one block per matrix)
// ---------------------------------------------------------------------------
template <int KT>
__global__ void __launch_bounds__(kThreads) lim_qr(const __grid_constant__ LimParams p) {
    extern __shared__ __align__(16) double dsm[];
    double* Gm = dsm;                   // [KT][KT]: Gram, then R^-1
    double* R = dsm + KT * KT;          // [KT][KT]: R (upper)
    double* d0 = R + KT * KT;           // [KT]: squared column norms
    int* ok = reinterpret_cast<int*>(d0 + KT);                  // [KT]
    float* stage = reinterpret_cast<float*>(ok + KT);          // [kGramRows][KT]
    const LimEntry& E = p.e[blockIdx.x];
    const int k = p.k;
    gram_fp64<KT>(E.Y, E.rows, k, Gm, stage);
    for (int idx = threadIdx.x; idx < KT * KT; idx += kThreads) R[idx] = 0.0;
    if (threadIdx.x < KT) d0[threadIdx.x] = Gm[threadIdx.x * KT + threadIdx.x];
    __syncthreads();
    // right-looking Cholesky of the upper triangle: G = R^T R
    for (int j = 0; j < k; ++j) {
        const double d = Gm[j * KT + j];
        const bool keep = d > kDrop * d0[j] && d > 0.0;
        const double rj = keep ? sqrt(d) : 0.0;
        for (int b = j + threadIdx.x; b < k; b += kThreads) R[j * KT + b] = keep ? (b == j ? rj : Gm[j * KT + b] / rj) : 0.0;
        if (threadIdx.x == 0) ok[j] = keep;
        __syncthreads();
        const int m = k - j - 1;
        for (int idx = threadIdx.x; idx < m * m; idx += kThreads) {
            const int a = j + 1 + idx / m, b = j + 1 + idx % m;
            if (b >= a) Gm[a * KT + b] -= R[j * KT + a] * R[j * KT + b];
        }
        __syncthreads();
    }
    // R^-1 (upper) column by column into Gm; dropped rows stay zero
    for (int idx = threadIdx.x; idx < KT * KT; idx += kThreads) Gm[idx] = 0.0;
    __syncthreads();
    if (threadIdx.x < k) {
        const int b = threadIdx.x;
        for (int a = b; a >= 0; --a) {
            if (!ok[a]) continue;
            double s = a == b ? 1.0 : 0.0;
            for (int c = a + 1; c <= b; ++c) s -= R[a * KT + c] * Gm[c * KT + b];
            Gm[a * KT + b] = s / R[a * KT + a];
        }
    }
    __syncthreads();
    // Q = Y R^-1, row by row in place
    for (int i = threadIdx.x; i < E.rows; i += kThreads) {
        float y[KT];
        float* row = E.Y + (long long)i * KT;
#pragma unroll
        for (int t = 0; t < KT; ++t) y[t] = t < k ? row[t] : 0.f;
#pragma unroll 4
        for (int j = 0; j < KT; ++j) {
            if (j >= k) break;
            double s = 0.0;
#pragma unroll
            for (int a = 0; a < KT; ++a)
                if (a <= j) s = fma((double)y[a], Gm[a * KT + j], s);
            row[j] = (float)s;
        }
    }
}

// ---------------------------------------------------------------------------
// 3. B^T = M^T Q
// ---------------------------------------------------------------------------
template <int KT>
__global__ void __launch_bounds__(kThreads) lim_project(const __grid_constant__ LimParams p) {
    constexpr int H = KT / 32;
    extern __shared__ __align__(16) float smem[];
    float* Ms = smem;                          // [kProjRows][kMsLd]
    float* Qs = smem + kProjRows * kMsLd;      // [kProjRows][KT]
    const LimEntry& E = p.e[find_entry(p, blockIdx.x, 1)];
    const int c0 = (blockIdx.x - E.t_proj) * kChunk;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float acc[16][H];
#pragma unroll
    for (int c = 0; c < 16; ++c)
#pragma unroll
        for (int h = 0; h < H; ++h) acc[c][h] = 0.f;
    for (int i0 = 0; i0 < E.rows; i0 += kProjRows) {
#pragma unroll
        for (int pass = 0; pass < kProjRows * kChunk / (8 * kThreads); ++pass) {
            const int g = threadIdx.x + kThreads * pass;
            const int rr = g >> 4, cc = (g & 15) * 8;
            const int i = i0 + rr, j = c0 + cc;
            float m[8];
            if (i < E.rows && j < E.cols) {
                const long long idx = (long long)i * E.cols + j;
                const int nvalid = min(8, E.cols - j);
                load8_dt(E.M, idx, DT_FP32, E.vec_ok && nvalid == 8, nvalid, m);
#pragma unroll
                for (int q = 0; q < 8; ++q) m[q] = q < nvalid ? m[q] : 0.f;
            } else {
#pragma unroll
                for (int q = 0; q < 8; ++q) m[q] = 0.f;
            }
            float4* dst = reinterpret_cast<float4*>(Ms + rr * kMsLd + cc);
            dst[0] = make_float4(m[0], m[1], m[2], m[3]);
            dst[1] = make_float4(m[4], m[5], m[6], m[7]);
        }
        for (int idx = threadIdx.x; idx < kProjRows * KT; idx += kThreads) {
            const int rr = idx / KT, t = idx % KT;
            Qs[idx] = (i0 + rr < E.rows && t < p.k) ? E.Y[(long long)(i0 + rr) * KT + t] : 0.f;
        }
        __syncthreads();
#pragma unroll 2
        for (int rr = 0; rr < kProjRows; ++rr) {
            float qv[H];
#pragma unroll
            for (int h = 0; h < H; ++h) qv[h] = Qs[rr * KT + lane + 32 * h];
            const float4* mrow = reinterpret_cast<const float4*>(Ms + rr * kMsLd + 16 * warp);
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4) {
                const float4 mv = mrow[c4];
#pragma unroll
                for (int h = 0; h < H; ++h) {
                    acc[4 * c4 + 0][h] = fmaf(mv.x, qv[h], acc[4 * c4 + 0][h]);
                    acc[4 * c4 + 1][h] = fmaf(mv.y, qv[h], acc[4 * c4 + 1][h]);
                    acc[4 * c4 + 2][h] = fmaf(mv.z, qv[h], acc[4 * c4 + 2][h]);
                    acc[4 * c4 + 3][h] = fmaf(mv.w, qv[h], acc[4 * c4 + 3][h]);
                }
            }
        }
        __syncthreads();
    }
#pragma unroll
    for (int c = 0; c < 16; ++c) {
        const int j = c0 + 16 * warp + c;
        if (j >= E.cols) continue;
#pragma unroll
        for (int h = 0; h < H; ++h) E.Bt[(long long)j * KT + lane + 32 * h] = acc[c][h];
    }
}

// ---------------------------------------------------------------------------
// 4. eigen-decomposition of B B^T and Z = Q P (one block per matrix)
// ---------------------------------------------------------------------------
template <int KT>
__global__ void __launch_bounds__(kThreads) lim_factor(const __grid_constant__ LimParams p) {
    extern __shared__ __align__(16) double dsm[];
    double* C = dsm;                    // [KT][KT]
    double* Ev = dsm + KT * KT;         // [KT][KT] eigenvectors (columns)
    double* cs = Ev + KT * KT;          // [KT/2] cosines
    double* sn = cs + KT / 2;           // [KT/2] sines
    double* lam = sn + KT / 2;          // [KT] eigenvalues
    double* red = lam + KT;             // [2 * 8] reduction scratch
    int* pp = reinterpret_cast<int*>(red + 16);   // [KT/2]
    int* pq = pp + KT / 2;                         // [KT/2]
    float* stage = reinterpret_cast<float*>(pq + KT / 2);   // [kGramRows][KT]
    const LimEntry& E = p.e[blockIdx.x];
    const int k = p.k, ke = k + (k & 1), n = ke - 1;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    gram_fp64<KT>(E.Bt, E.cols, k, C, stage);
    for (int idx = threadIdx.x; idx < KT * KT; idx += kThreads) Ev[idx] = (idx / KT == idx % KT) ? 1.0 : 0.0;
    __syncthreads();
    for (int sweep = 0; sweep < kMaxSweeps; ++sweep) {
        double off = 0.0, tot = 0.0;
        for (int idx = threadIdx.x; idx < ke * ke; idx += kThreads) {
            const int a = idx / ke, b = idx % ke;
            const double v = C[a * KT + b] * C[a * KT + b];
            tot += v;
            if (a != b) off += v;
        }
        for (int o = 16; o > 0; o >>= 1) {
            off += __shfl_xor_sync(0xffffffffu, off, o);
            tot += __shfl_xor_sync(0xffffffffu, tot, o);
        }
        if (lane == 0) { red[warp] = off; red[8 + warp] = tot; }
        __syncthreads();
        off = 0.0; tot = 0.0;
        for (int w = 0; w < kThreads / 32; ++w) { off += red[w]; tot += red[8 + w]; }
        __syncthreads();
        if (!(off > 1e-30 * tot)) break;          // also leaves on tot == 0
        for (int rd = 0; rd < n; ++rd) {
            if (threadIdx.x < ke / 2) {
                const int i = threadIdx.x;
                int a = i == 0 ? n : (rd + i) % n, b = i == 0 ? rd : (rd - i + n) % n;
                if (a > b) { const int t = a; a = b; b = t; }
                const double apq = C[a * KT + b];
                double c = 1.0, s = 0.0;
                if (apq != 0.0) {
                    const double tau = (C[b * KT + b] - C[a * KT + a]) / (2.0 * apq);
                    const double t = (tau >= 0.0 ? 1.0 : -1.0) / (fabs(tau) + sqrt(1.0 + tau * tau));
                    c = 1.0 / sqrt(1.0 + t * t);
                    s = t * c;
                }
                pp[i] = a; pq[i] = b; cs[i] = c; sn[i] = s;
            }
            __syncthreads();
            for (int idx = threadIdx.x; idx < (ke / 2) * ke; idx += kThreads) {   // rows p, q <- J^T C
                const int i = idx / ke, col = idx % ke;
                const double c = cs[i], s = sn[i];
                const double x = C[pp[i] * KT + col], y = C[pq[i] * KT + col];
                C[pp[i] * KT + col] = c * x - s * y;
                C[pq[i] * KT + col] = s * x + c * y;
            }
            __syncthreads();
            for (int idx = threadIdx.x; idx < (ke / 2) * ke; idx += kThreads) {   // columns p, q <- C J, E J
                const int i = idx / ke, row = idx % ke;
                const double c = cs[i], s = sn[i];
                const double x = C[row * KT + pp[i]], y = C[row * KT + pq[i]];
                C[row * KT + pp[i]] = c * x - s * y;
                C[row * KT + pq[i]] = s * x + c * y;
                const double u = Ev[row * KT + pp[i]], v = Ev[row * KT + pq[i]];
                Ev[row * KT + pp[i]] = c * u - s * v;
                Ev[row * KT + pq[i]] = s * u + c * v;
            }
            __syncthreads();
        }
    }
    // the r largest eigenvalues above kTau2 * largest: weights 1 / sqrt(lambda)
    if (threadIdx.x < k) lam[threadIdx.x] = C[threadIdx.x * KT + threadIdx.x];
    __syncthreads();
    double lmax = 0.0;
    for (int a = 0; a < k; ++a) lmax = fmax(lmax, lam[a]);
    double* wgt = cs;                   // reuse: [KT] weights (cs and sn are contiguous)
    __syncthreads();
    if (threadIdx.x < k) {
        const int a = threadIdx.x;
        int rank = 0;
        for (int b = 0; b < k; ++b) rank += (lam[b] > lam[a]) || (lam[b] == lam[a] && b < a);
        const bool sel = lmax > 0.0 && rank < p.r && lam[a] > kTau2 * lmax;
        wgt[a] = sel ? 1.0 / sqrt(lam[a]) : 0.0;
    }
    __syncthreads();
    // P = E diag(w) E^T into C
    for (int idx = threadIdx.x; idx < KT * KT; idx += kThreads) {
        const int a = idx / KT, b = idx % KT;
        double s = 0.0;
        if (a < k && b < k)
            for (int e = 0; e < k; ++e) s += Ev[a * KT + e] * wgt[e] * Ev[b * KT + e];
        C[idx] = s;
    }
    __syncthreads();
    // Z = Q P, row by row in place
    for (int i = threadIdx.x; i < E.rows; i += kThreads) {
        float q[KT];
        float* row = E.Y + (long long)i * KT;
#pragma unroll
        for (int t = 0; t < KT; ++t) q[t] = t < k ? row[t] : 0.f;
        for (int j = 0; j < KT; ++j) {
            double s = 0.0;
#pragma unroll
            for (int a = 0; a < KT; ++a) s = fma((double)q[a], C[a * KT + j], s);
            row[j] = (float)s;
        }
    }
}

// ---------------------------------------------------------------------------
// 5. O = Z B and the weight update
// ---------------------------------------------------------------------------
template <int W_DT>
__device__ __forceinline__ void load4_w(const void* base, long long idx, bool vec, int nvalid, float* v) {
    if (vec) {
        if (W_DT == DT_FP32) {
            const float4 x = *reinterpret_cast<const float4*>(static_cast<const float*>(base) + idx);
            v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
        } else {
            const uint2 x = *reinterpret_cast<const uint2*>(static_cast<const uint16_t*>(base) + idx);
            using T = typename std::conditional<W_DT == DT_BF16, __nv_bfloat16, __half>::type;
            v[0] = unpack_lo<T>(x.x); v[1] = unpack_hi<T>(x.x);
            v[2] = unpack_lo<T>(x.y); v[3] = unpack_hi<T>(x.y);
        }
        return;
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) v[c] = c < nvalid ? ld_elem(base, idx + c, W_DT) : 0.f;
}

template <int W_DT>
__device__ __forceinline__ void store4_w(void* base, long long idx, bool vec, int nvalid, const float* v) {
    if (vec) {
        if (W_DT == DT_FP32) {
            *reinterpret_cast<float4*>(static_cast<float*>(base) + idx) = make_float4(v[0], v[1], v[2], v[3]);
        } else {
            using T = typename std::conditional<W_DT == DT_BF16, __nv_bfloat16, __half>::type;
            *reinterpret_cast<uint2*>(static_cast<uint16_t*>(base) + idx) =
                make_uint2(pack2<T>(v[0], v[1]), pack2<T>(v[2], v[3]));
        }
        return;
    }
#pragma unroll
    for (int c = 0; c < 4; ++c)
        if (c < nvalid) st_elem(base, idx + c, W_DT, v[c]);
}

template <int KT, int W_DT>
__global__ void __launch_bounds__(kThreads) lim_update(const __grid_constant__ LimParams p) {
    extern __shared__ __align__(16) float smem[];
    float* Zs = smem;                          // [kUpdRows][KT]
    float* Bs = smem + kUpdRows * KT;          // [KT][kMsLd]: B = (B^T)^T, this tile's columns
    const LimEntry& E = p.e[find_entry(p, blockIdx.x, 2)];
    const int tile = blockIdx.x - E.t_upd;
    const int tiles_c = (E.cols + kChunk - 1) / kChunk;
    const int row0 = (tile / tiles_c) * kUpdRows, c0 = (tile % tiles_c) * kChunk;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int idx = threadIdx.x; idx < kUpdRows * KT; idx += kThreads) {
        const int rr = idx / KT;
        Zs[idx] = row0 + rr < E.rows ? E.Y[(long long)(row0 + rr) * KT + idx % KT] : 0.f;
    }
    for (int idx = threadIdx.x; idx < kChunk * KT; idx += kThreads) {
        const int jj = idx / KT, t = idx % KT;
        Bs[t * kMsLd + jj] = c0 + jj < E.cols ? E.Bt[(long long)(c0 + jj) * KT + t] : 0.f;
    }
    __syncthreads();
    float o[4][4];
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < 4; ++c) o[r][c] = 0.f;
#pragma unroll 2
    for (int t = 0; t < KT; t += 4) {
        float4 z[4], b[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) z[r] = *reinterpret_cast<const float4*>(Zs + (4 * warp + r) * KT + t);
#pragma unroll
        for (int q = 0; q < 4; ++q) b[q] = *reinterpret_cast<const float4*>(Bs + (t + q) * kMsLd + 4 * lane);
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const float zz[4] = {z[r].x, z[r].y, z[r].z, z[r].w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                o[r][0] = fmaf(zz[q], b[q].x, o[r][0]);
                o[r][1] = fmaf(zz[q], b[q].y, o[r][1]);
                o[r][2] = fmaf(zz[q], b[q].z, o[r][2]);
                o[r][3] = fmaf(zz[q], b[q].w, o[r][3]);
            }
        }
    }
    const bool skip = *E.bad != 0;
    const int j = c0 + 4 * lane;
    if (j >= E.cols) return;
    const int nvalid = min(4, E.cols - j);
    const bool vec = E.vec_ok && nvalid == 4;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const int i = row0 + 4 * warp + r;
        if (i >= E.rows) break;
        const long long idx = (long long)i * E.cols + j;
        if (E.O_out) {
            if (vec) *reinterpret_cast<float4*>(E.O_out + idx) = make_float4(o[r][0], o[r][1], o[r][2], o[r][3]);
            else
                for (int c = 0; c < nvalid; ++c) E.O_out[idx + c] = o[r][c];
        }
        if (skip) continue;
        float w[4];
        load4_w<W_DT>(E.W, idx, vec, nvalid, w);
#pragma unroll
        for (int c = 0; c < 4; ++c) w[c] = w[c] - p.eta * (E.gamma * o[r][c] + p.lambda * w[c]);
        store4_w<W_DT>(E.W, idx, vec, nvalid, w);
    }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

constexpr size_t sketch_smem(int KT) { return sizeof(float) * (kSketchRows * kMsLd + kChunk * KT); }
constexpr size_t project_smem(int KT) { return sizeof(float) * (kProjRows * kMsLd + kProjRows * KT); }
constexpr size_t update_smem(int KT) { return sizeof(float) * (kUpdRows * KT + KT * kMsLd); }
constexpr size_t qr_smem(int KT) {
    return sizeof(double) * (2 * KT * KT + KT) + sizeof(int) * KT + sizeof(float) * kGramRows * KT;
}
constexpr size_t factor_smem(int KT) {
    return sizeof(double) * (2 * KT * KT + KT / 2 * 2 + KT + 16) + sizeof(int) * KT + sizeof(float) * kGramRows * KT;
}

template <typename K>
cudaError_t allow_smem(K kernel, size_t bytes) {
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

template <int KT, int W_DT>
muon_status launch_all(LimParams& prm, cudaStream_t s, int sketch_blocks, int proj_blocks, int upd_blocks,
                       double elems, double rows_k, double cols_k) {
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
            cudaError_t e[5] = {allow_smem(lim_sketch<KT, W_DT>, sketch_smem(KT)), allow_smem(lim_qr<KT>, qr_smem(KT)),
                                allow_smem(lim_project<KT>, project_smem(KT)),
                                allow_smem(lim_factor<KT>, factor_smem(KT)),
                                allow_smem(lim_update<KT, W_DT>, update_smem(KT))};
            for (cudaError_t x : e)
                if (x != cudaSuccess) return MUON_ERR_CUDA;
            configured[dev] = true;
        }
    }
    const double wsz = dt_size(W_DT), k = prm.k;
    // algorithmic bytes: per element G, M read + M written; the sketch Y written (rows x k)
    trace_begin(MUON_KERNEL_RSVD, elems * (wsz + 8.0) + 4.0 * rows_k, s);
    lim_sketch<KT, W_DT><<<sketch_blocks, kThreads, sketch_smem(KT), s>>>(prm);
    trace_end(s);
    trace_begin(MUON_KERNEL_RSVD_SMALL, 2.0 * rows_k * k, s);     // Y read, Q written
    lim_qr<KT><<<prm.n, kThreads, qr_smem(KT), s>>>(prm);
    trace_end(s);
    trace_begin(MUON_KERNEL_RSVD, elems * 4.0 + 4.0 * (rows_k + cols_k), s);   // M, Q read; B^T written
    lim_project<KT><<<proj_blocks, kThreads, project_smem(KT), s>>>(prm);
    trace_end(s);
    trace_begin(MUON_KERNEL_RSVD_SMALL, 4.0 * (cols_k + 2.0 * rows_k), s);     // B^T, Q read; Z written
    lim_factor<KT><<<prm.n, kThreads, factor_smem(KT), s>>>(prm);
    trace_end(s);
    trace_begin(MUON_KERNEL_RSVD, elems * 2.0 * wsz + 4.0 * (rows_k + cols_k), s);   // W read and written
    lim_update<KT, W_DT><<<upd_blocks, kThreads, update_smem(KT), s>>>(prm);
    trace_end(s);
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
    const int KT = kt_for(hp->rank + hp->oversample);
    size_t total = align256(sizeof(int) * (size_t)n);
    for (int i = 0; i < n; ++i) total += matrix_ws(params[i].rows, params[i].cols, KT);
    *bytes = total;
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
    char* ws = static_cast<char*>(workspace);
    int* bad = reinterpret_cast<int*>(ws);
    if (cudaMemsetAsync(bad, 0, sizeof(int) * (size_t)n, s) != cudaSuccess) return MUON_ERR_CUDA;
    char* cur = ws + align256(sizeof(int) * (size_t)n);
    static LimParams prm;              // large: kept off the stack, filled and consumed per launch
    static std::mutex mu;
    std::lock_guard<std::mutex> lock(mu);
    for (int b = 0; b < n; b += kLimMax) {
        memset(&prm, 0, sizeof(prm));
        prm.n = std::min(kLimMax, n - b);
        prm.k = k; prm.r = hp->rank;
        prm.mu = hp->mu; prm.eta = hp->eta; prm.lambda = hp->lambda;
        prm.d_status = d_status;
        long long ts = 0, tp = 0, tu = 0;
        double elems = 0.0, rows_k = 0.0, cols_k = 0.0;
        for (int i = 0; i < prm.n; ++i) {
            const muon_rsvd_param& q = params[b + i];
            LimEntry& E = prm.e[i];
            E.W = q.W; E.G = q.G; E.M = q.M; E.Omega = q.Omega; E.O_out = q.O_out;
            E.rows = q.rows; E.cols = q.cols;
            E.gamma = std::isnan(q.gamma) ? hp->gamma : q.gamma;
            E.bad = bad + b + i;
            E.Y = reinterpret_cast<float*>(cur);
            E.Bt = reinterpret_cast<float*>(cur + align256(sizeof(float) * (size_t)q.rows * KT));
            cur += matrix_ws(q.rows, q.cols, KT);
            const uintptr_t al = reinterpret_cast<uintptr_t>(q.W) | reinterpret_cast<uintptr_t>(q.G) |
                                 reinterpret_cast<uintptr_t>(q.M) | reinterpret_cast<uintptr_t>(q.O_out);
            E.vec_ok = (al & 15) == 0 && q.cols % 8 == 0;
            E.t_sketch = (int)ts; E.t_proj = (int)tp; E.t_upd = (int)tu;
            ts += (q.rows + kSketchRows - 1) / kSketchRows;
            tp += (q.cols + kChunk - 1) / kChunk;
            tu += (long long)((q.rows + kUpdRows - 1) / kUpdRows) * ((q.cols + kChunk - 1) / kChunk);
            elems += (double)q.rows * q.cols;
            rows_k += (double)q.rows * k;
            cols_k += (double)q.cols * k;
        }
        if (ts > INT32_MAX || tp > INT32_MAX || tu > INT32_MAX) return MUON_ERR_UNSUPPORTED;
        const int a = (int)ts, pj = (int)tp, u = (int)tu;
        if (KT == 32) {
            if (w_dtype == MUON_BF16) st = launch_all<32, DT_BF16>(prm, s, a, pj, u, elems, rows_k, cols_k);
            else if (w_dtype == MUON_FP16) st = launch_all<32, DT_FP16>(prm, s, a, pj, u, elems, rows_k, cols_k);
            else st = launch_all<32, DT_FP32>(prm, s, a, pj, u, elems, rows_k, cols_k);
        } else {
            if (w_dtype == MUON_BF16) st = launch_all<64, DT_BF16>(prm, s, a, pj, u, elems, rows_k, cols_k);
            else if (w_dtype == MUON_FP16) st = launch_all<64, DT_FP16>(prm, s, a, pj, u, elems, rows_k, cols_k);
            else st = launch_all<64, DT_FP32>(prm, s, a, pj, u, elems, rows_k, cols_k);
        }
        if (st != MUON_OK) return st;
    }
    return MUON_OK;
}

}  // extern "C"
