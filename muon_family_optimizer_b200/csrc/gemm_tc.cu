// gemm_tc.cu -- batched, grouped tcgen05 GEMMs for the Newton-Schulz steps.
//
// [POLAR] (quant_prune_distill post 677): the Muon step replaces the momentum
// by its polar factor, computed by Newton-Schulz; products of symmetric
// matrices need only half of their elements.  Every product of one iteration
// step is one of two shapes:
//   SYM:  D = A B^T with a symmetric result: X X^T, A A (A symmetric), and on
//         the Gram route R R, h Q, h R, (h R) h (polynomials in one symmetric
//         matrix commute, so each product is symmetric).  Only the 128 x 128
//         tiles on or above the diagonal are computed and stored; nothing is
//         mirrored.  A consumer that needs a block left of the diagonal tile
//         reads the stored block above the diagonal transposed (MN-major
//         operand layout), chosen per 64-deep k-block.
//   UPD:  D = A X with A (s x s) symmetric and X (s x l) row-major, i.e. the
//         B operand is MN-major: X <- (a I + b A + c A^2) X, Xb <- Q Xb.
//
// Kernel shape (one CTA per SM, persistent over a flattened tile list that
// spans every matrix of up to four shape groups):
//   warp 0      TMA producer: 128-byte-swizzled boxes of A and B into a ring
//               of shared-memory stages (no multicast: every CTA loads its own
//               tiles);
//   warp 1      allocates tensor memory; one thread issues tcgen05.mma
//               (kind::f16, fp32 accumulate, 128 x BN x 16) and commits stage
//               releases and accumulator hand-offs to mbarriers;
//   warps 2-9   epilogue, two warps per tensor-memory lane quadrant (each takes
//               half of the columns): tcgen05.ld of the fp32 accumulator,
//               scale / combine, round to 16 bits into a per-warp 128B-swizzled
//               staging box (32 rows x 64 columns) and a TMA bulk store of the
//               box; the final step writes the caller's layout directly.
// Two accumulator buffers in tensor memory let the epilogue of tile t overlap
// the main loop of tile t+1.
#include <cudaTypedefs.h>

#include <stdlib.h>
#include <string.h>

#include <mutex>

#include "epilogue.cuh"
#include "gemm.h"

namespace muon {
namespace tc {

constexpr int BM = 128;
constexpr int kWideMinK = 1024;   // 256 x 512 tiles from this depth (update) or size (symmetric)
constexpr int BK = 64;    // 64 16-bit elements = one 128-byte swizzle row
constexpr int kEpiWarps = 8;    // two per tensor-memory lane quadrant, each takes half the columns
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr int kEpiThreads = 32 * kEpiWarps;

// Per-CTA configuration.  PAIR: two CTAs share each MMA (cta_group::2): the
// pair computes a 256 x BN tile, each CTA loads its 128 rows of A and BN/2 of B.
// S1: a symmetric product on CTA pairs whose diagonal tiles need no
// cross-warp symmetrisation (every problem a product of one operand with
// itself): each epilogue warp stages its two boxes one after the other in one
// box, and the 64 KB this frees hold a sixth pipeline stage.  The operand
// stream is latency-bound per SM, so the k-loop runs in proportion to the
// stages in flight.
template <int BN, bool PAIR, bool B_MN, bool FIN, bool S1 = false>
struct Cfg {
    // symmetric products on CTA pairs stage a whole 128 x 256 output (16 boxes,
    // or 8 with S1); the final step keeps two 32 x 32 blocks of the target per
    // epilogue warp
    static constexpr bool kSymPair = PAIR && !B_MN;
    // BN = 512 (update products, and symmetric products of one operand with
    // itself, on pairs): two N = 256 MMAs per k-slice into all
    // 512 tensor-memory columns, one accumulator buffer
    static constexpr bool kWide = BN == 512;
    static constexpr int kStages = FIN ? (PAIR ? 4 : 3) : kWide ? 4 : kSymPair ? (S1 ? 6 : 5) : ((PAIR || BN == 128) ? 6 : 4);
    static constexpr int kABytes = BM * BK * 2;
    static constexpr int kBBytes = (PAIR ? BN / 2 : BN) * BK * 2;
    static constexpr int kStageBytes = kABytes + kBBytes;
    static constexpr int kNumBuf = kWide ? 1 : 2;            // accumulator buffers
    static constexpr int kTmemCols = kNumBuf * BN;
    static constexpr int kStgBytes = 32 * 64 * 2;              // one 32 x 64 16-bit box
    static constexpr int kBoxes = (kSymPair && !S1) ? 16 : kEpiWarps;   // staging boxes
    static constexpr int kFinBlock = 32 * 32 * 4;               // one 32 x 32 block of the target (up to fp32)
    static constexpr int kStgRegion = FIN ? kEpiWarps * 2 * kFinBlock : kBoxes * kStgBytes;
    static constexpr int kStgOffset = kStages * kStageBytes;
    static constexpr int kBarOffset = kStgOffset + kStgRegion;
    static constexpr int kBarBytes = 256;
    static constexpr int kSmemBytes = 1024 + kBarOffset + kBarBytes;
    static constexpr int kRows = PAIR ? 2 * BM : BM;           // output rows per tile
};

struct TcProblem {
    CUtensorMap mapA;    // A rows, K-major boxes 64 (K) x 128 (M)
    CUtensorMap mapAt;   // A symmetric: transposed reads, boxes 64 (M) x 64 (K)
    CUtensorMap mapB;    // SYM: B rows, boxes 64 (K) x 128 (N); UPD: X panel, boxes 64 (N) x 64 (K),
                         // or (b_tr) X stored N x K, boxes 64 (K) x BN/2 (N)
    CUtensorMap mapBt;   // B symmetric: transposed reads, boxes 64 (N) x 64 (K)
    CUtensorMap mapD;    // output stores, boxes 64 (N) x 32 (M)
    CUtensorMap mapDt;   // band: transposed stores, boxes 32 (M) x 64 (N), no swizzle
    int count, M, N, K;
    int tiles_m, tiles_n, tiles_per_mat, sym, a_sym, b_sym, band;
    int a_tr, b_tr;      // operands stored transposed in full (see GemmOp)
    int same_ab;         // A and B are one operand: a diagonal tile loads one panel for both
    int wide;            // symmetric on 256 x 512 tiles: row tile ti spans 512-column tiles ti / 2 ..
    long long tile_begin;
    Epilogue epi;
};

struct TcParams {
    TcProblem prob[kMaxProblems];
    int nprob;
    long long total_tiles;
    FinalCtx fc;
    FinalEntry fin[kMaxFinal];
};

__device__ __forceinline__ void decode_tile(const TcParams& p, long long t, int& pi, int& m,
                                            int& ti, int& tj) {
    pi = 0;
    while (pi + 1 < p.nprob && t >= p.prob[pi + 1].tile_begin) ++pi;
    const TcProblem& P = p.prob[pi];
    long long local = t - P.tile_begin;
    m = (int)(local / P.tiles_per_mat);
    int r = (int)(local - (long long)m * P.tiles_per_mat);
    if (P.sym && P.wide) {
        int i = 0;
        while (r >= P.tiles_n - (i >> 1)) { r -= P.tiles_n - (i >> 1); ++i; }
        ti = i;
        tj = (i >> 1) + r;
    } else if (P.sym) {
        int nt = P.tiles_m, i = 0;
        while (r >= nt - i) { r -= nt - i; ++i; }
        ti = i;
        tj = i + r;
    } else {
        ti = r % P.tiles_m;
        tj = r / P.tiles_m;
    }
}

// Previous-operand values of one chunk (row gi, columns gj0..gj0+31) as raw
// 16-bit data in four 16-byte words; issued ahead of use to hide its latency.
template <typename T>
__device__ __forceinline__ void cin_fetch(const Epilogue& E, int m, int gi, int gj0, int M, int N,
                                          uint4 (&c)[4]) {
    if (gi >= M || gj0 >= N) return;
    const T* src = static_cast<const T*>(E.Cin) + (size_t)m * E.strideC + (size_t)gi * E.ldc + gj0;
    if (gj0 + 32 <= N) {
#pragma unroll
        for (int q = 0; q < 4; ++q) c[q] = reinterpret_cast<const uint4*>(src)[q];
    } else {
        T* e = reinterpret_cast<T*>(c);
        for (int q = 0; q < 32; ++q) e[q] = gj0 + q < N ? src[q] : from_float<T>(0.f);
    }
}

// ---------------------------------------------------------------------------
// Final step (FIN_WUPD: W <- W - eta (gamma O + lambda W); FIN_OUT: the
// caller's output), one warp at a time: wide rows gi0..gi0+31 (one per lane)
// and 32-column blocks of wide columns.  Each block of the target matrix is
// moved between global and shared memory in its own orientation with
// coalesced 16-byte accesses (W prefetched with cp.async one block ahead),
// updated in shared memory by the lane that owns the row of O, and written
// back.  Block layout in shared memory (param rows of 32 * sizeof(TW) bytes):
//   wide view (!tr): row = wide row, 16-byte chunks XOR-swizzled by row;
//   transposed (tr): row = wide column, unswizzled (lanes then touch
//   consecutive elements of one row).
// ---------------------------------------------------------------------------
struct FinalTarget {
    void* W;
    float* O_out;
    float g;
    int tr, vec, dt;
    bool wupd;
};

__device__ __forceinline__ FinalTarget final_target(const Epilogue& E, const FinalCtx& fc, int m) {
    FinalTarget F;
    F.wupd = E.fin == FIN_WUPD;
    if (!F.wupd) {
        F.W = static_cast<char*>(fc.out) + (size_t)m * fc.out_stride * dt_size(fc.out_dt);
        F.O_out = nullptr; F.g = 0.f; F.tr = fc.out_transposed; F.vec = fc.out_vec; F.dt = fc.out_dt;
    } else {
        const FinalEntry& fe = fc.fin[E.fin_base + m];
        F.W = fe.W; F.O_out = fe.O_out; F.g = fe.gamma; F.tr = fe.transposed; F.vec = fe.vec_ok; F.dt = fc.w_dt;
    }
    return F;
}

template <typename TW>
__device__ __forceinline__ int wb_off(int prow, int chunk, bool swz) {
    constexpr int kRowBytes = 32 * (int)sizeof(TW);
    const int c = !swz ? chunk : (sizeof(TW) == 2 ? chunk ^ ((prow >> 1) & 3) : chunk ^ (prow & 7));
    return prow * kRowBytes + c * 16;
}

// Copy the target's block (wide rows gi0.., wide columns gj0..) into `buf`
// (to_smem) or back from it; chunks outside the matrix are zero-filled on the
// way in and skipped on the way out.
template <typename TW, bool kIn>
__device__ __forceinline__ void final_move(const FinalTarget& F, int M, int N, int gi0, int gj0, uint8_t* buf,
                                           int lane) {
    constexpr int kEpc = 16 / (int)sizeof(TW);       // elements per 16-byte chunk
    constexpr int kChunks = 32 / kEpc;               // chunks per block row
    const int prow_n = F.tr ? N : M, pcol_n = F.tr ? M : N;
    const int prow0 = F.tr ? gj0 : gi0, pcol0 = F.tr ? gi0 : gj0;
    TW* W = static_cast<TW*>(F.W);
#pragma unroll
    for (int k = 0; k < kChunks; ++k) {
        const int id = lane + 32 * k;
        const int pr = id / kChunks, ch = id % kChunks;
        const int prow = prow0 + pr, pcol = pcol0 + ch * kEpc;
        const bool in = prow < prow_n && pcol < pcol_n;
        uint8_t* sp = buf + wb_off<TW>(pr, ch, !F.tr);
        if (kIn) {
            cp_async16(sp, in ? W + (size_t)prow * pcol_n + pcol : W, in ? 16u : 0u);
        } else if (in) {
            *reinterpret_cast<uint4*>(W + (size_t)prow * pcol_n + pcol) = *reinterpret_cast<const uint4*>(sp);
        }
    }
}

// Apply the final step to this lane's row of the staged block.
template <typename TW>
__device__ __forceinline__ void final_apply(const FinalTarget& F, const FinalCtx& fc, uint8_t* buf,
                                            const float (&v)[32], int lane) {
    constexpr int kEpc = 16 / (int)sizeof(TW);
    if (!F.tr) {
#pragma unroll
        for (int ch = 0; ch < 32 / kEpc; ++ch) {
            uint4* p = reinterpret_cast<uint4*>(buf + wb_off<TW>(lane, ch, true));
            uint4 u = *p;
            uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                if constexpr (sizeof(TW) == 4) {
                    const float o = v[ch * 4 + h];
                    const float w = __uint_as_float(w4[h]);
                    w4[h] = __float_as_uint(F.wupd ? w - fc.eta * (F.g * o + fc.lambda * w) : o);
                } else {
                    const float o0 = v[ch * 8 + 2 * h], o1 = v[ch * 8 + 2 * h + 1];
                    float a = o0, b = o1;
                    if (F.wupd) {
                        const float w0 = unpack_lo<TW>(w4[h]), w1 = unpack_hi<TW>(w4[h]);
                        a = w0 - fc.eta * (F.g * o0 + fc.lambda * w0);
                        b = w1 - fc.eta * (F.g * o1 + fc.lambda * w1);
                    }
                    w4[h] = pack2<TW>(a, b);
                }
            }
            u.x = w4[0]; u.y = w4[1]; u.z = w4[2]; u.w = w4[3];
            *p = u;
        }
    } else {
#pragma unroll
        for (int q = 0; q < 32; ++q) {
            TW* p = reinterpret_cast<TW*>(buf + (q * 32 + lane) * (int)sizeof(TW));
            if (F.wupd) {
                const float w = to_float(*p);
                *p = from_float<TW>(w - fc.eta * (F.g * v[q] + fc.lambda * w));
            } else {
                *p = from_float<TW>(v[q]);
            }
        }
    }
}

// Unaligned or ragged target: element by element from and to global memory.
template <typename TW>
__device__ __forceinline__ void final_scalar(const FinalTarget& F, const FinalCtx& fc, int M, int N, int gi,
                                             int gj0, const float (&v)[32]) {
    if (gi >= M) return;
    TW* W = static_cast<TW*>(F.W);
    float w[32];
#pragma unroll
    for (int q = 0; q < 32; ++q) {
        const int j = gj0 + q;
        const size_t idx = F.tr ? (size_t)j * M + gi : (size_t)gi * N + j;
        w[q] = (F.wupd && j < N) ? to_float(W[idx]) : 0.f;
    }
#pragma unroll
    for (int q = 0; q < 32; ++q) {
        const int j = gj0 + q;
        if (j >= N) continue;
        const size_t idx = F.tr ? (size_t)j * M + gi : (size_t)gi * N + j;
        W[idx] = from_float<TW>(F.wupd ? w[q] - fc.eta * (F.g * v[q] + fc.lambda * w[q]) : v[q]);
    }
}

// Optional fp32 copy of O in the parameter's orientation.
__device__ __forceinline__ void final_o_out(const FinalTarget& F, int M, int N, int gi, int gj0,
                                            const float (&v)[32]) {
    if (!F.O_out || gi >= M) return;
#pragma unroll
    for (int q = 0; q < 32; ++q) {
        const int j = gj0 + q;
        if (j < N) F.O_out[F.tr ? (size_t)j * M + gi : (size_t)gi * N + j] = v[q];
    }
}

template <typename T>
__device__ __forceinline__ void epi_combine(const Epilogue& E, int gi, int gj0, float sc, float (&v)[32],
                                            const uint4 (&c)[4]);

// Start the copies of the target's blocks for the warp's wide rows gi0.. and
// BN/2 wide columns from col0.  16-bit targets: all four 2 KB blocks (one
// cp.async group each, empty groups past the matrix edge); 32-bit: block 0.
template <typename TW, int BN>
__device__ __forceinline__ void final_prefetch(const FinalTarget& F, int M, int N, int gi0, int col0, uint8_t* wbuf,
                                               int lane) {
    constexpr int kBlocks = BN / 64;
    if constexpr (sizeof(TW) == 2) {
#pragma unroll 1
        for (int b = 0; b < kBlocks; ++b) {
            if (col0 + 32 * b < N) final_move<TW, true>(F, M, N, gi0, col0 + 32 * b, wbuf + b * 2048, lane);
            cp_async_commit();
        }
    } else {
        final_move<TW, true>(F, M, N, gi0, col0, wbuf, lane);
        cp_async_commit();
    }
}

__device__ __forceinline__ void cp_async_wait_upto(int n) {   // at most n groups still pending
    if (n <= 0) cp_async_wait<0>();
    else if (n == 1) cp_async_wait<1>();
    else if (n == 2) cp_async_wait<2>();
    else cp_async_wait<3>();
}

// The final step for the warp's wide rows gi0.. and its BN/2 wide columns
// from col0: four 32-column blocks.  16-bit targets: block b's data in
// wbuf + 2 KB * b, all copies started by final_prefetch (pf_issued);
// 32-bit: wbuf[b % 2], block b + 1's copy started while block b is applied
// (block 0's possibly by final_prefetch).
template <typename T, typename TW, int BN>
__device__ __forceinline__ void final_tile(const FinalTarget& F, const Epilogue& E, const FinalCtx& fc, int m,
                                           const TcProblem& P, int gi0, int col0, int gi, float sc, uint32_t tcol0,
                                           uint8_t* wbuf, int lane, bool pf_issued) {
    constexpr int kBlocks = BN / 64;                 // 32-column blocks per warp
    constexpr bool kAll = sizeof(TW) == 2;          // every block's copy started up front
    constexpr int kBlockBytes = kAll ? 32 * 32 * 2 : 32 * 32 * 4;
    const bool staged = F.vec;                      // aligned target: go through shared memory
    const uint4 none[4] = {};
    if (kAll && staged && F.wupd && !pf_issued) final_prefetch<TW, BN>(F, P.M, P.N, gi0, col0, wbuf, lane);
#pragma unroll 1
    for (int b = 0; b < kBlocks; ++b) {
        const int gj0 = col0 + 32 * b;
        if (gj0 >= P.N) break;                       // warp-uniform
        uint8_t* cur = wbuf + (kAll ? b : (b & 1)) * kBlockBytes;
        if (!kAll && staged && F.wupd) {
            if (b == 0 && !pf_issued) {
                final_move<TW, true>(F, P.M, P.N, gi0, gj0, cur, lane);
                cp_async_commit();
            }
            if (b + 1 < kBlocks && gj0 + 32 < P.N) {  // next block's copy in flight during this one
                final_move<TW, true>(F, P.M, P.N, gi0, gj0 + 32, wbuf + ((b + 1) & 1) * kBlockBytes, lane);
                cp_async_commit();
            }
        }
        float v[32];
        tmem_ld_32x32b_x32(tcol0 + 32 * b, v);
        epi_combine<T>(E, gi, gj0, sc, v, none);
        final_o_out(F, P.M, P.N, gi, gj0, v);
        if (!staged) {
            final_scalar<TW>(F, fc, P.M, P.N, gi, gj0, v);
            continue;
        }
        if (F.wupd) {
            if (kAll) cp_async_wait_upto(kBlocks - 1 - b);
            else if (b + 1 < kBlocks && gj0 + 32 < P.N) cp_async_wait<1>();
            else cp_async_wait<0>();
        }
        __syncwarp();                                // this block's copy visible to every lane
        final_apply<TW>(F, fc, cur, v, lane);
        __syncwarp();
        final_move<TW, false>(F, P.M, P.N, gi0, gj0, cur, lane);
        __syncwarp();                                // cur free for the block after next
    }
}

// Combine one 32-column chunk of the accumulator (row gi, columns
// gj0..gj0+31) with the scale, the previous operand (`c`, when beta != 0) and
// the diagonal shift.
template <typename T>
__device__ __forceinline__ void epi_combine(const Epilogue& E, int gi, int gj0, float sc, float (&v)[32],
                                            const uint4 (&c)[4]) {
    if (E.beta != 0.f) {
        const float a = sc * E.alpha, b = sc * E.beta;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint32_t w[4] = {c[q].x, c[q].y, c[q].z, c[q].w};
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                v[8 * q + 2 * h] = a * v[8 * q + 2 * h] + b * unpack_lo<T>(w[h]);
                v[8 * q + 2 * h + 1] = a * v[8 * q + 2 * h + 1] + b * unpack_hi<T>(w[h]);
            }
        }
    } else {
        const float s = sc * E.alpha;
        if (s != 1.f) {   // uniform: most products have no scale after the first step
#pragma unroll
            for (int q = 0; q < 32; ++q) v[q] *= s;
        }
    }
    if (E.diag != 0.f && (unsigned)(gi - gj0) < 32u) {   // only a chunk crossing the diagonal
#pragma unroll
        for (int q = 0; q < 32; ++q)   // static indices only: keeps v in registers
            if (gi == gj0 + q) v[q] += E.diag;
    }
}

// Write 32 values (row `r` of the warp's 32 x 64 staging box, 16-byte chunks
// c16 .. c16+3) in the 128-byte swizzle the store's tensor map expects:
// chunk c of row r lives at r * 128 + ((c ^ (r % 8)) * 16).
template <typename T>
__device__ __forceinline__ void stage32(uint8_t* stg, int r, int c16, const float (&v)[32]) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        uint4 u;
        u.x = pack2<T>(v[8 * q + 0], v[8 * q + 1]);
        u.y = pack2<T>(v[8 * q + 2], v[8 * q + 3]);
        u.z = pack2<T>(v[8 * q + 4], v[8 * q + 5]);
        u.w = pack2<T>(v[8 * q + 6], v[8 * q + 7]);
        *reinterpret_cast<uint4*>(stg + r * 128 + (((c16 + q) ^ (r & 7)) * 16)) = u;
    }
}

// Transpose of 32 columns (c0..c0+31) of the warp's 32 x 64 block into the
// staging box taken as a dense 64 x 32 box (row c = block column c, 64 bytes
// per row, no swizzle): lane r writes column r, so the warp's 32 lanes fill
// one 64-byte row per element.
template <typename T>
__device__ __forceinline__ void stage_transposed(uint8_t* stg, int lane, int c0, const float (&v)[32]) {
    T* box = reinterpret_cast<T*>(stg);
#pragma unroll
    for (int c = 0; c < 32; ++c) box[(c0 + c) * 32 + lane] = from_float<T>(v[c]);
}

// One 32-column chunk of a symmetric result's box: accumulator -> epilogue ->
// staging box (16-byte chunks c16..c16+3).
template <typename T>
__device__ __forceinline__ void sym_chunk(const Epilogue& E, int gi, int gj0, float sc, uint32_t tcol, uint8_t* box,
                                          int lane, int c16, const uint4 (&c)[4]) {
    float v[32];
    tmem_ld_32x32b_x32(tcol, v);
    epi_combine<T>(E, gi, gj0, sc, v, c);
    stage32<T>(box, lane, c16, v);
}

// Barrier over the epilogue warps only (named barrier 1).
__device__ __forceinline__ void epi_bar() {
    asm volatile("bar.sync 1, %0;" ::"n"(kEpiThreads) : "memory");
}

// Byte offset of element (r, c) (r < 32, c < 64) in a 32 x 64 16-bit staging box.
__device__ __forceinline__ int stg_off(int r, int c) {
    return r * 128 + (((c >> 3) ^ (r & 7)) << 4) + ((c & 7) << 1);
}

// The mirror of a staged 32 x 64 box of a symmetric result (rows gi0.., columns
// gj0..): element (gi0 + i, gj0 + c) is written to (gj0 + c, gi0 + i).  Lane l
// takes box columns l and l + 32; a column's 32 elements are read from shared
// memory (for one i the warp reads 64 bytes of one 128-byte row: no bank
// conflict) and written as 64 contiguous bytes of the destination row.
template <typename T>
__device__ __forceinline__ void mirror_box(const Epilogue& E, int m, int gi0, int gj0, int M, int N,
                                           const uint8_t* box, int lane) {
    T* base = static_cast<T*>(E.D) + (size_t)m * E.strideD;
    const bool full_rows = gi0 + 32 <= M;
#pragma unroll 1
    for (int h = 0; h < 2; ++h) {
        const int c = lane + 32 * h;
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const uint32_t lo = *reinterpret_cast<const uint16_t*>(box + stg_off(2 * i, c));
            const uint32_t hi = *reinterpret_cast<const uint16_t*>(box + stg_off(2 * i + 1, c));
            w[i] = lo | (hi << 16);
        }
        if (gj0 + c >= N) continue;
        T* dst = base + (size_t)(gj0 + c) * E.ldd + gi0;
        if (full_rows && (reinterpret_cast<uintptr_t>(dst) & 15) == 0) {
#pragma unroll
            for (int q = 0; q < 4; ++q)
                reinterpret_cast<uint4*>(dst)[q] = make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
        } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                if (gi0 + i < M) {
                    const uint16_t e = (uint16_t)(i & 1 ? w[i >> 1] >> 16 : w[i >> 1] & 0xFFFFu);
                    reinterpret_cast<uint16_t*>(dst)[i] = e;
                }
            }
        }
    }
}

// Diagonal 128 x 128 block of a symmetric result, held in staging boxes
// (box (q, c): rows 32q.., columns 64c.. of the CTA's tile; the block is box
// columns cb0, cb0 + 1).  Overwrite this thread's elements of its box
// (q = quad, c = cown) that lie below the diagonal (block row i, column j < i)
// with element (j, i) above it, so the stored block is exactly symmetric.
// Reads touch only positions above the diagonal, writes only positions below.
template <typename T>
__device__ __forceinline__ void fix_lower(uint8_t* stg_base, int quad, int cb0, int cown, int lane) {
    const int i = quad * 32 + lane;
    uint8_t* mine = stg_base + (quad + 4 * cown) * (32 * 64 * 2);
    const int jbase = (cown - cb0) * 64;
    for (int q = 0; q < 64; ++q) {
        const int j = jbase + q;
        if (j >= i) break;
        const uint8_t* ob = stg_base + ((j >> 5) + 4 * (cb0 + (i >> 6))) * (32 * 64 * 2);
        const T x = *reinterpret_cast<const T*>(ob + stg_off(j & 31, i & 63));
        *reinterpret_cast<T*>(mine + stg_off(lane, q)) = x;
    }
}

// TRX: the launch may hold operands stored transposed in full (the first step
// of an optimizer step); without it the operand layouts of every k-block are
// compile-time or per-problem symmetric-storage decisions only, which keeps
// the single MMA-issuing thread's work per instruction minimal.
template <int BN, bool B_MN, bool PAIR, bool FIN, bool TRX, typename T, bool S1 = false>
__global__ void __launch_bounds__(kThreads, 1) tc_gemm_kernel(const __grid_constant__ TcParams p) {
    static_assert(!PAIR || BN == 256 || (BN == 512 && !FIN && (B_MN || S1)),
                  "CTA pairs compute 256 x 256 tiles, or 256 x 512 update / one-operand symmetric tiles");
    static_assert(PAIR || BN <= 256, "one CTA computes 128 x 128 or 128 x 256 tiles");
    static_assert(!FIN || B_MN, "the final step is an update product");
    static_assert(!S1 || (PAIR && !B_MN), "one staging box per warp: symmetric products on pairs");
    using C = Cfg<BN, PAIR, B_MN, FIN, S1>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + C::kBarOffset);
    uint64_t* empty_bar = full_bar + C::kStages;
    uint64_t* tfull_bar = empty_bar + C::kStages;
    uint64_t* tempty_bar = tfull_bar + 2;
    uint64_t* drain_bar = tempty_bar + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain_bar + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    int* d_status = p.fc.d_status;
    // CTA pairs: rank 0 (leader) issues the MMAs for both CTAs of the cluster
    const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
    const long long unit = PAIR ? (blockIdx.x >> 1) : blockIdx.x;
    const long long nunits = PAIR ? (gridDim.x >> 1) : gridDim.x;
    constexpr uint32_t kTemptyCount = kEpiWarps * (PAIR ? 2 : 1);   // one arrival per epilogue warp

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull_bar[b], 1);
            mbar_init(&tempty_bar[b], kTemptyCount);
        }
        mbar_init(drain_bar, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        for (int i = 0; i < p.nprob; ++i) {
            prefetch_tensormap(TRX && p.prob[i].a_tr ? &p.prob[i].mapAt : &p.prob[i].mapA);
            prefetch_tensormap(TRX && p.prob[i].sym && p.prob[i].b_tr ? &p.prob[i].mapBt : &p.prob[i].mapB);
        }
    }
    if (warp == 1) {
        if (PAIR) {
            tmem_alloc_pair(tmem_slot, C::kTmemCols);
            tmem_relinquish_pair();
        } else {
            tmem_alloc(tmem_slot, C::kTmemCols);
            tmem_relinquish();
        }
    }
    tc_fence_before();
    __syncwarp();
    if (PAIR) cluster_sync(); else __syncthreads();   // barriers of both CTAs initialised
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------ TMA producer
            int stage = 0;
            uint32_t phase = 0;
            uint32_t armed = 0;          // bit s: stage s has been armed at least once
            uint32_t armed_parity = 0;   // bit s: parity of the phase stage s was last armed in
            constexpr int kBCols = PAIR ? BN / 2 : BN;
            auto chunks_of = [&](int N, int c0) { return max(0, min(kBCols / 64, (N - c0 + 63) / 64)); };
            for (long long t = unit; t < p.total_tiles && !*abort_flag; t += nunits) {
                int pi, m, ti, tj;
                decode_tile(p, t, pi, m, ti, tj);
                const TcProblem& P = p.prob[pi];
                const int nkb = (P.K + BK - 1) / BK;
                const int rows0 = ti * C::kRows + (int)rank * BM;   // this CTA's rows of A
                // this CTA's columns of the result (rows of a K-major B, columns of an
                // MN-major B panel) and, for a panel, the 64-wide boxes they span
                const int bcol0 = tj * BN + (int)rank * kBCols;
                auto chunks = [&](int c0) { return chunks_of(P.N, c0); };
                const int nchunk = B_MN ? chunks(bcol0) : kBCols / 64;
                // wide update tiles: MMA h (0, 1) covers the tile's columns 256 h..; this
                // CTA supplies 128 of them (256 h + 128 rank..), as two 64-column chunks
                auto wide_col = [&](int r, int c) { return tj * BN + 256 * (c >> 1) + 128 * r + 64 * (c & 1); };
                // A diagonal tile of a product whose operands are one matrix (X X^T,
                // S S) needs the same rows as A and as B: one panel serves both.
                const bool one_panel = !C::kWide && !B_MN && P.same_ab && ti == tj;
                // an update product whose X is stored transposed loads whole K-major boxes
                const bool b_kmaj = B_MN && TRX && P.b_tr;
                uint32_t bytes = C::kABytes + (B_MN ? (b_kmaj ? C::kBBytes : nchunk * 64 * BK * 2)
                                                    : (one_panel ? 0 : C::kBBytes));
                if (PAIR) {   // the leader's barrier counts both CTAs' boxes
                    bytes = B_MN ? (b_kmaj ? 2 * (C::kABytes + C::kBBytes)
                                           : 2 * C::kABytes + (chunks(tj * BN) + chunks(tj * BN + kBCols)) * 64 * BK * 2)
                                 : 2 * (C::kABytes + (one_panel ? 0 : C::kBBytes));
                    if constexpr (C::kWide) {
                        // 64-column panel chunks, or 128-row units (K-major boxes of X stored
                        // transposed; symmetric products: B rows, or two transposed chunks)
                        const bool rows128 = b_kmaj || !B_MN;
                        int n = 0;
                        for (int r = 0; r < 2; ++r)
                            for (int c = 0; c < 4; ++c)
                                n += (rows128 ? (c & 1) == 0 : true) && wide_col(r, c) < P.N ? 1 : 0;
                        bytes = 2 * C::kABytes + n * (rows128 ? 128 : 64) * BK * 2;
                    }
                }
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!mbar_wait(&empty_bar[stage], phase ^ 1, abort_flag, d_status)) break;
                    uint8_t* sa = smem + stage * C::kStageBytes;
                    uint8_t* sb = sa + C::kABytes;
                    // Blocks left of the diagonal of a stored symmetric operand are read
                    // transposed from the block above the diagonal.  On a pair the
                    // decision is taken on the pair's first 128-row (128-column) block,
                    // so both halves agree (such operands also store the first tile
                    // below the diagonal).
                    const bool at = (TRX && P.a_tr) || (P.a_sym && (kb >> 1) < (PAIR ? 2 * ti : ti));
                    const bool bt = !B_MN && ((TRX && P.b_tr) || (P.b_sym && (kb >> 1) < (PAIR ? 2 * tj : tj)));
                    const uint32_t fb = PAIR ? mapa_shared(smem_u32(&full_bar[stage]), 0) : 0u;
                    auto load = [&](const CUtensorMap* map, void* dst, int x, int y) {
                        if (PAIR) tma_load_3d_pair(map, fb, dst, x, y, m);
                        else tma_load_3d(map, &full_bar[stage], dst, x, y, m);
                    };
                    if (!PAIR || rank == 0) mbar_arrive_expect_tx(&full_bar[stage], bytes);
                    if (at) {
                        load(&P.mapAt, sa, rows0, kb * BK);
                        load(&P.mapAt, sa + 64 * BK * 2, rows0 + 64, kb * BK);
                    } else {
                        load(&P.mapA, sa, kb * BK, rows0);
                    }
                    if (b_kmaj && C::kWide) {
                        // this CTA's 128 rows of X for each half of the tile, K-major
                        for (int h = 0; h < 2; ++h) {
                            const int row = wide_col((int)rank, 2 * h);
                            if (row < P.N) load(&P.mapB, sb + h * (128 * BK * 2), kb * BK, row);
                        }
                    } else if (b_kmaj) {
                        load(&P.mapB, sb, kb * BK, bcol0);
                    } else if (B_MN && C::kWide) {
                        for (int c = 0; c < 4; ++c) {
                            const int col = wide_col((int)rank, c);
                            if (col < P.N) load(&P.mapB, sb + c * (64 * BK * 2), col, kb * BK);
                        }
                    } else if (B_MN) {
                        for (int c = 0; c < nchunk; ++c) load(&P.mapB, sb + c * (64 * BK * 2), bcol0 + c * 64, kb * BK);
                    } else if (C::kWide) {
                        // symmetric, 256 x 512: for each half of the tile this CTA's 128 B rows
                        // (the half's own transposed-read rule for a stored symmetric operand)
                        for (int h = 0; h < 2; ++h) {
                            const int row = wide_col((int)rank, 2 * h);
                            if (row >= P.N) continue;
                            const bool bth = (TRX && P.b_tr) || (P.b_sym && (kb >> 1) < 2 * (2 * tj + h));
                            if (bth) {
                                load(&P.mapBt, sb + h * 16384, row, kb * BK);
                                load(&P.mapBt, sb + h * 16384 + 64 * BK * 2, row + 64, kb * BK);
                            } else {
                                load(&P.mapB, sb + h * 16384, kb * BK, row);
                            }
                        }
                    } else if (one_panel) {
                        // B is the A panel just loaded
                    } else if (bt) {
                        for (int c = 0; c < kBCols / 64; ++c)
                            load(&P.mapBt, sb + c * (64 * BK * 2), bcol0 + c * 64, kb * BK);
                    } else {
                        load(&P.mapB, sb, kb * BK, bcol0);
                    }
                    armed |= 1u << stage;
                    armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
                    if (++stage == C::kStages) { stage = 0; phase ^= 1; }
                }
            }
            if (*abort_flag) {
                // wind down: every copy this CTA started must land before it exits
                const unsigned long long t0 = global_ns();
                if (!PAIR || rank == 0) {
                    for (int s = 0; s < C::kStages; ++s) {
                        if (!(armed >> s & 1u)) continue;
                        const uint32_t par = armed_parity >> s & 1u;
                        while (!mbar_try_wait(&full_bar[s], par) && global_ns() - t0 < kWaitLimitNs) {
                        }
                    }
                } else {
                    // the second CTA of a pair counts its copies on the leader's
                    // barriers: give them a fixed time to land
                    while (global_ns() - t0 < 200000ull) {
                    }
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && rank == 0) {
            // ------------------------------------------------ MMA issuer
            constexpr uint32_t idesc0 = make_idesc_f16(IsBf16<T>::value ? 1 : 0, 0, C::kRows, C::kWide ? 256 : BN);
            int stage = 0;
            uint32_t phase = 0;
            int it = 0;
            bool ok = true;
            for (long long t = unit; ok && t < p.total_tiles; t += nunits, ++it) {
                int pi, m, ti, tj;
                decode_tile(p, t, pi, m, ti, tj);
                const TcProblem& P = p.prob[pi];
                const int nkb = (P.K + BK - 1) / BK;
                const int buf = it % C::kNumBuf;
                const uint32_t tphase = (it / C::kNumBuf) & 1;
                if (!mbar_wait(&tempty_bar[buf], tphase ^ 1, abort_flag, d_status)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(buf * BN);
                const bool one_panel = !C::kWide && !B_MN && P.same_ab && ti == tj;   // B read from the A panel
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!mbar_wait(&full_bar[stage], phase, abort_flag, d_status)) { ok = false; break; }
                    tc_fence_after();
                    // A block read transposed; B block MN-major (an update product's X panel
                    // always, unless stored transposed in full)
                    const bool at = (TRX && P.a_tr) || (P.a_sym && (kb >> 1) < (PAIR ? 2 * ti : ti));
                    const int tjb = C::kWide && !B_MN ? 2 * tj : tj;   // 256-column tile of the (first) MMA
                    const bool bm = B_MN ? !(TRX && P.b_tr)
                                         : ((TRX && P.b_tr) || (P.b_sym && (kb >> 1) < (PAIR ? 2 * tjb : tjb)));
                    const bool bm1 = B_MN ? bm : ((TRX && P.b_tr) || (P.b_sym && (kb >> 1) < 2 * (tjb + 1)));
                    const uint32_t idesc = idesc0 | (at ? 1u << 15 : 0u) | (bm ? 1u << 16 : 0u);
                    const uint32_t idesc1 = idesc0 | (at ? 1u << 15 : 0u) | (bm1 ? 1u << 16 : 0u);
                    (void)idesc1;
                    const uint32_t sa = smem_u32(smem + stage * C::kStageBytes);
                    const uint32_t sb = one_panel ? sa : sa + C::kABytes;
#pragma unroll
                    for (int k = 0; k < BK / 16; ++k) {
                        // K-major: the k-th 16-element slice sits 32 bytes further in each
                        // swizzled 128-byte row; MN-major: 16 rows of 128 bytes further,
                        // 64-element MN chunks 64 x BK x 2 bytes apart.
                        const uint64_t ad = at ? smem_desc_sw128(sa + k * 2048, 64 * BK * 2, 1024)
                                               : smem_desc_sw128(sa + k * 32, 16, 1024);
                        const uint64_t bd = bm ? smem_desc_sw128(sb + k * 2048, 64 * BK * 2, 1024)
                                               : smem_desc_sw128(sb + k * 32, 16, 1024);
                        if (PAIR) tc_mma_f16_pair(d_tmem, ad, bd, idesc, (kb | k) != 0 ? 1u : 0u);
                        else tc_mma_f16(d_tmem, ad, bd, idesc, (kb | k) != 0 ? 1u : 0u);
                        if constexpr (C::kWide) {   // the tile's columns 256..511: the second 16 KB of B
                            const uint64_t bd1 = bm1 ? smem_desc_sw128(sb + 16384 + k * 2048, 64 * BK * 2, 1024)
                                                     : smem_desc_sw128(sb + 16384 + k * 32, 16, 1024);
                            tc_mma_f16_pair(d_tmem + 256, ad, bd1, idesc1, (kb | k) != 0 ? 1u : 0u);
                        }
                    }
                    if (PAIR) {   // release the stage in both CTAs
                        tc_commit_pair(smem_u32(&empty_bar[stage]));
                        tc_commit_pair(mapa_shared(smem_u32(&empty_bar[stage]), 1));
                    } else {
                        tc_commit(&empty_bar[stage]);
                    }
                    if (++stage == C::kStages) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
                if (PAIR) {       // accumulators ready in both CTAs
                    tc_commit_pair(smem_u32(&tfull_bar[buf]));
                    tc_commit_pair(mapa_shared(smem_u32(&tfull_bar[buf]), 1));
                } else {
                    tc_commit(&tfull_bar[buf]);
                }
            }
            // make sure no MMA is still writing tensor memory before it is freed
            if (PAIR) tc_commit_pair(smem_u32(drain_bar)); else tc_commit(drain_bar);
            const unsigned long long t0 = global_ns();
            while (!mbar_try_wait(drain_bar, 0) && global_ns() - t0 < kWaitLimitNs) {
            }
        }
    } else {
        // ---------------------------------------------------- epilogue
        // No warp leaves this loop early: diagonal tiles of symmetric results
        // synchronise the eight epilogue warps, so every warp walks every tile
        // and attends those barriers; a warp whose wait failed (abort) only
        // skips the work.
        const int ew = warp - 2;              // 0..7
        const int quad = warp & 3;            // TMEM lanes 32*quad .. 32*quad+31
        const int half = ew >> 2;             // which half of the tile's columns
        const int row = quad * 32 + lane;
        constexpr int kPairs = BN / 128;      // 64-column boxes per half
        uint8_t* stg_base = smem + C::kStgOffset;
        uint8_t* stg = stg_base + (quad + 4 * half) * C::kStgBytes;   // box of rows 32*quad.., columns 64*half..
        uint8_t* wbuf = stg_base + (quad + 4 * half) * 2 * C::kFinBlock;   // final step: two target blocks
        bool stg_busy = false;                // a bulk store may still be reading stg
        bool dead = false;
        FinalCtx fc = p.fc;
        fc.fin = p.fin;
        int it = 0;
        for (long long t = unit; t < p.total_tiles; t += nunits, ++it) {
            int pi, m, ti, tj;
            decode_tile(p, t, pi, m, ti, tj);
            const TcProblem& P = p.prob[pi];
            const Epilogue& E = P.epi;
            const int buf = it % C::kNumBuf;
            const uint32_t tphase = (it / C::kNumBuf) & 1;
            const int row0 = ti * C::kRows + (int)rank * BM;   // first output row of this CTA
            const int gi = row0 + row;
            const int col0 = tj * BN + half * (BN / 2);
            const bool has_cin = E.beta != 0.f;
            const bool diag_sym = P.sym && !P.same_ab && ti == tj && E.fin == FIN_STORE;   // uniform over the CTA
            uint4 c0[4] = {}, c1[4] = {};
            uint4 c2[4] = {}, c3[4] = {};   // symmetric pair tiles: the second box's columns
            bool released = false;          // accumulator buffer handed back early
            bool pf_issued = false;
            if constexpr (FIN) {
                // the target's first block is independent of the accumulator: prefetch it
                if (!dead && row0 + quad * 32 < P.M) {
                    const FinalTarget F = final_target(E, fc, m);
                    if (F.wupd && F.vec && col0 < P.N) {
                        if (F.dt == DT_BF16) final_prefetch<__nv_bfloat16, BN>(F, P.M, P.N, row0 + quad * 32, col0, wbuf, lane);
                        else if (F.dt == DT_FP16) final_prefetch<__half, BN>(F, P.M, P.N, row0 + quad * 32, col0, wbuf, lane);
                        else final_prefetch<float, BN>(F, P.M, P.N, row0 + quad * 32, col0, wbuf, lane);
                        pf_issued = true;
                    }
                }
            }
            if (!dead) {
                if (has_cin) {   // independent of the accumulator: fetch before waiting for it
                    cin_fetch<T>(E, m, gi, col0, P.M, P.N, c0);
                    cin_fetch<T>(E, m, gi, col0 + 32, P.M, P.N, c1);
                    if constexpr (C::kSymPair) {
                        cin_fetch<T>(E, m, gi, col0 + 64, P.M, P.N, c2);
                        cin_fetch<T>(E, m, gi, col0 + 96, P.M, P.N, c3);
                    }
                }
                // warp-uniform outcome: tcgen05.ld below is warp-collective
                const bool ok = mbar_wait(&tfull_bar[buf], tphase, abort_flag, d_status);
                dead = !__all_sync(0xffffffffu, ok);
                if (!dead) tc_fence_after();
            }
            const float sc = epi_scale(E, m);
            bool skip = false;
            if (!dead && E.fin != FIN_STORE && !epi_finite(E, m, sc)) {
                skip = E.fin == FIN_WUPD;   // keep W; a FIN_OUT result carries the NaN
                if (row == 0 && half == 0 && tj == 0 && ti == 0 && rank == 0 && d_status)
                    atomicOr(d_status, MUON_FLAG_NONFINITE);
            }
            if constexpr (FIN) {
                // final step: W update (or the caller's output) block by block,
                // the target's next block prefetched while this one is applied
                if (!dead && !skip && row0 + quad * 32 < P.M) {
                    const FinalTarget F = final_target(E, fc, m);
                    if (F.dt == DT_BF16) final_tile<T, __nv_bfloat16, BN>(F, E, fc, m, P, row0 + quad * 32, col0, gi, sc,
                                                                        tmem_base + ((uint32_t)(quad * 32) << 16) +
                                                                            (uint32_t)(buf * BN + half * (BN / 2)),
                                                                        wbuf, lane, pf_issued);
                    else if (F.dt == DT_FP16) final_tile<T, __half, BN>(F, E, fc, m, P, row0 + quad * 32, col0, gi, sc,
                                                                      tmem_base + ((uint32_t)(quad * 32) << 16) +
                                                                          (uint32_t)(buf * BN + half * (BN / 2)),
                                                                      wbuf, lane, pf_issued);
                    else final_tile<T, float, BN>(F, E, fc, m, P, row0 + quad * 32, col0, gi, sc,
                                                  tmem_base + ((uint32_t)(quad * 32) << 16) +
                                                      (uint32_t)(buf * BN + half * (BN / 2)),
                                                  wbuf, lane, pf_issued);
                }
                cp_async_wait<0>();   // nothing of this tile stays in flight
                __syncwarp();
            } else if constexpr (C::kSymPair) {
                // Symmetric result on a CTA pair: this CTA holds rows row0.. of a
                // 256-column tile; box (q, c) = rows 32q.., columns 64c..; this warp
                // owns box columns 2*half and 2*half + 1, i.e. the 128-block
                // (bi, bj) below.  Both boxes are staged before anything is stored,
                // so a diagonal block (tile on the diagonal: this CTA's block column
                // `rank`) can be made exactly symmetric across the warps first.  In a
                // diagonal tile the second CTA's first block column lies below the
                // diagonal and is not stored: its exact mirror is written by the
                // warps holding the first block right of the diagonal (bj = bi + 1),
                // straight from the registers that fill their staging boxes.  The
                // accumulator buffer is handed back as soon as it has been read.
                if constexpr (C::kWide) {
                    // 256 x 512 tile of a product of one operand with itself: this warp's
                    // half of the columns is the 256 x 256 tile (ti, tjh); its four 64-column
                    // boxes in turn through one staging box.  A 128-block (bi, bj) is stored
                    // when bj >= bi (on or above the diagonal; the part of the tile left of
                    // the diagonal is computed and dropped), and mirrored below the
                    // diagonal when it is the first block right of it (band).
                    const int tjh = 2 * tj + half;
                    const int bi = 2 * ti + (int)rank;
                    const bool rows_ok = row0 + quad * 32 < P.M;
                    uint8_t* box = stg_base + (quad + 4 * half) * C::kStgBytes;
#pragma unroll 1
                    for (int b = 0; b < 4; ++b) {
                        const int bj = 2 * tjh + (b >> 1), gj = 256 * tjh + 64 * b;
                        if (dead || bj < bi || gj >= P.N) continue;   // warp-uniform
                        if (stg_busy) {
                            if (lane == 0) bulk_wait_read0();
                            __syncwarp();
                        }
                        uint4 ca[4] = {}, cb[4] = {};
                        if (has_cin) {
                            if (b == 0) {
                                for (int q = 0; q < 4; ++q) { ca[q] = c0[q]; cb[q] = c1[q]; }
                            } else if (b == 1) {
                                for (int q = 0; q < 4; ++q) { ca[q] = c2[q]; cb[q] = c3[q]; }
                            } else {
                                cin_fetch<T>(E, m, gi, gj, P.M, P.N, ca);
                                cin_fetch<T>(E, m, gi, gj + 32, P.M, P.N, cb);
                            }
                        }
                        const uint32_t tc = tmem_base + ((uint32_t)(quad * 32) << 16) +
                                            (uint32_t)(buf * BN + half * 256 + 64 * b);
                        sym_chunk<T>(E, gi, gj, sc, tc, box, lane, 0, ca);
                        sym_chunk<T>(E, gi, gj + 32, sc, tc + 32, box, lane, 4, cb);
                        if (rows_ok) {
                            fence_proxy_async_smem();
                            __syncwarp();
                            if (lane == 0) {
                                tma_store_3d(&P.mapD, box, gj, row0 + quad * 32, m);
                                bulk_commit();
                            }
                            stg_busy = true;
                            if (P.band && bj == bi + 1) {
                                __syncwarp();
                                mirror_box<T>(E, m, row0 + quad * 32, gj, P.M, P.N, box, lane);
                            }
                        }
                    }
                    if (!dead) {               // every column this warp needs has been read
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&tempty_bar[buf]), 0));
                        released = true;
                    }
                } else {
                const bool diag_pair = ti == tj;
                const int bi = 2 * ti + (int)rank, bj = 2 * tj + half;
                const bool mirror = P.band && bj == bi + 1;
                const int gjb = tj * BN + 2 * half * 64;   // first column of box 2*half
                const bool have0 = !dead && gjb < P.N;
                const bool have1 = !dead && gjb + 64 < P.N;
                if (!dead && stg_busy) {
                    if (lane == 0) bulk_wait_read0();
                    __syncwarp();
                }
                const uint32_t tcol = tmem_base + ((uint32_t)(quad * 32) << 16) + (uint32_t)(buf * BN + 2 * half * 64);
                if constexpr (S1) {
                    // one box per warp, the two 64-column boxes in turn (the product's
                    // diagonal blocks are exactly symmetric as formed: nothing to fix)
                    uint8_t* box = stg_base + (quad + 4 * half) * C::kStgBytes;
                    const bool rows_ok = row0 + quad * 32 < P.M;
                    const bool lower = diag_pair && rank == 1 && half == 0;   // below the diagonal
                    const bool store = rows_ok && !lower;
                    if (have0) {
                        sym_chunk<T>(E, gi, gjb, sc, tcol, box, lane, 0, c0);
                        sym_chunk<T>(E, gi, gjb + 32, sc, tcol + 32, box, lane, 4, c1);
                        if (!have1) {          // the accumulator has been read
                            tc_fence_before();
                            __syncwarp();
                            if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&tempty_bar[buf]), 0));
                            released = true;
                        }
                        if (store) {
                            fence_proxy_async_smem();
                            __syncwarp();
                            if (lane == 0) {
                                tma_store_3d(&P.mapD, box, gjb, row0 + quad * 32, m);
                                bulk_commit();
                            }
                            stg_busy = true;
                        }
                        if (mirror && rows_ok) {
                            __syncwarp();
                            mirror_box<T>(E, m, row0 + quad * 32, gjb, P.M, P.N, box, lane);
                        }
                    }
                    if (have1) {
                        if (stg_busy) {        // the box is reused: the first store has read it
                            if (lane == 0) bulk_wait_read0();
                        }
                        __syncwarp();
                        sym_chunk<T>(E, gi, gjb + 64, sc, tcol + 64, box, lane, 0, c2);
                        sym_chunk<T>(E, gi, gjb + 96, sc, tcol + 96, box, lane, 4, c3);
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&tempty_bar[buf]), 0));
                        released = true;
                        if (store) {
                            fence_proxy_async_smem();
                            __syncwarp();
                            if (lane == 0) {
                                tma_store_3d(&P.mapD, box, gjb + 64, row0 + quad * 32, m);
                                bulk_commit();
                            }
                            stg_busy = true;
                        }
                        if (mirror && rows_ok) {
                            __syncwarp();
                            mirror_box<T>(E, m, row0 + quad * 32, gjb + 64, P.M, P.N, box, lane);
                        }
                    }
                    if (!dead && !released) {  // no column of this warp's half inside the matrix
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&tempty_bar[buf]), 0));
                        released = true;
                    }
                } else {
                uint8_t* box0 = stg_base + (quad + 4 * (2 * half)) * C::kStgBytes;
                uint8_t* box1 = stg_base + (quad + 4 * (2 * half + 1)) * C::kStgBytes;
                if (have0) {
                    sym_chunk<T>(E, gi, gjb, sc, tcol, box0, lane, 0, c0);
                    sym_chunk<T>(E, gi, gjb + 32, sc, tcol + 32, box0, lane, 4, c1);
                }
                if (have1) {
                    sym_chunk<T>(E, gi, gjb + 64, sc, tcol + 64, box1, lane, 0, c2);
                    sym_chunk<T>(E, gi, gjb + 96, sc, tcol + 96, box1, lane, 4, c3);
                }
                if (!dead) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&tempty_bar[buf]), 0));
                    released = true;
                }
                // A product of one operand with itself (X X^T, S S with S stored exactly
                // symmetric) is formed at (i, j) and (j, i) from the same products in the
                // same order, so its diagonal block is already exactly symmetric; a
                // product of two matrices (h Q, (h R) h) is symmetrised here.
                if (diag_pair && !P.same_ab) {     // uniform over the CTA: every epilogue warp attends
                    epi_bar();
                    if (half == (int)rank) {
                        if (have0) fix_lower<T>(stg_base, quad, 2 * (int)rank, 2 * half, lane);
                        if (have1) fix_lower<T>(stg_base, quad, 2 * (int)rank, 2 * half + 1, lane);
                    }
                    epi_bar();
                }
                const bool rows_ok = row0 + quad * 32 < P.M;
                const bool lower = diag_pair && rank == 1 && half == 0;   // below the diagonal
                if (rows_ok && !lower && (have0 || have1)) {
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        if (have0) tma_store_3d(&P.mapD, box0, gjb, row0 + quad * 32, m);
                        if (have1) tma_store_3d(&P.mapD, box1, gjb + 64, row0 + quad * 32, m);
                        bulk_commit();
                    }
                    stg_busy = true;
                }
                if (mirror && rows_ok) {   // off-diagonal block: the staged boxes are final
                    __syncwarp();
                    if (have0) mirror_box<T>(E, m, row0 + quad * 32, gjb, P.M, P.N, box0, lane);
                    if (have1) mirror_box<T>(E, m, row0 + quad * 32, gjb + 64, P.M, P.N, box1, lane);
                }
                }   // S1
                }   // kWide
            } else {
#pragma unroll 1
            for (int pr = 0; pr < kPairs; ++pr) {
                const int gj0 = col0 + pr * 64;
                const bool work = !dead && gj0 < P.N;       // warp-uniform
                const uint32_t tcol = tmem_base + ((uint32_t)(quad * 32) << 16) +
                                      (uint32_t)(buf * BN + half * (BN / 2) + pr * 64);
                if (work && has_cin && pr > 0) {
                    cin_fetch<T>(E, m, gi, gj0, P.M, P.N, c0);
                    cin_fetch<T>(E, m, gi, gj0 + 32, P.M, P.N, c1);
                }
                if (E.fin == FIN_STORE) {
                    // 32 rows x 64 columns -> staging box -> one bulk tensor store;
                    // one 32-column chunk in registers at a time
                    if (work) {
                        if (stg_busy) {
                            if (lane == 0) bulk_wait_read0();
                            __syncwarp();
                        }
                        float v[32];
                        tmem_ld_32x32b_x32(tcol, v);
                        epi_combine<T>(E, gi, gj0, sc, v, c0);
                        stage32<T>(stg, lane, 0, v);
                        tmem_ld_32x32b_x32(tcol + 32, v);
                        epi_combine<T>(E, gi, gj0 + 32, sc, v, c1);
                        stage32<T>(stg, lane, 4, v);
                    }
                    if (diag_sym) {          // BN == 128 here: the eight boxes cover the tile
                        epi_bar();
                        if (work) fix_lower<T>(stg_base, quad, 0, half, lane);
                        epi_bar();
                    }
                    if (work && row0 + quad * 32 < P.M) {
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) {
                            tma_store_3d(&P.mapD, stg, gj0, row0 + quad * 32, m);
                            bulk_commit();
                        }
                        stg_busy = true;
                        if (P.band && tj == ti + 1) {
                            // first tile right of the diagonal: also store its transpose
                            // (the tile below the diagonal), exactly mirrored; the values
                            // are formed again from the accumulator, still in TMEM
                            if (lane == 0) bulk_wait_read0();
                            __syncwarp();
                            float v[32];
                            tmem_ld_32x32b_x32(tcol, v);
                            epi_combine<T>(E, gi, gj0, sc, v, c0);
                            stage_transposed<T>(stg, lane, 0, v);
                            tmem_ld_32x32b_x32(tcol + 32, v);
                            epi_combine<T>(E, gi, gj0 + 32, sc, v, c1);
                            stage_transposed<T>(stg, lane, 32, v);
                            fence_proxy_async_smem();
                            __syncwarp();
                            if (lane == 0) {
                                tma_store_3d(&P.mapDt, stg, row0 + quad * 32, gj0, m);
                                bulk_commit();
                            }
                        }
                    }
                }
            }
            }   // kSymPair
            if (!dead && !released) {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    if (PAIR) mbar_arrive_cluster(mapa_shared(smem_u32(&tempty_bar[buf]), 0));
                    else mbar_arrive(&tempty_bar[buf]);
                }
            }
        }
        if (lane == 0) bulk_wait0();   // stores complete before the CTA's shared memory goes away
        __syncwarp();
    }

    tc_fence_before();
    __syncwarp();
    if (PAIR) cluster_sync(); else __syncthreads();   // neither CTA of a pair leaves while the other works
    if (warp == 1) {
        tc_fence_after();
        if (PAIR) tmem_dealloc_pair(tmem_base, C::kTmemCols);
        else tmem_dealloc(tmem_base, C::kTmemCols);
    }
}

// ----------------------------------------------------------------------------
// Host side
// ----------------------------------------------------------------------------
static PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

// 3-D map over `count` matrices of `rows` x `inner` 16-bit elements with row
// stride `ld` and matrix stride `mstride` (elements); box = box_inner x box_rows x 1.
static bool encode_map(CUtensorMap* map, int dt, const void* base, long long inner, long long rows,
                       long long count, long long ld, long long mstride, int box_inner, int box_rows,
                       bool swizzle = true) {
    auto enc = get_encode();
    if (!enc) return false;
    cuuint64_t dims[3] = {(cuuint64_t)inner, (cuuint64_t)rows, (cuuint64_t)count};
    cuuint64_t strides[2] = {(cuuint64_t)ld * 2, (cuuint64_t)mstride * 2};
    cuuint32_t box[3] = {(cuuint32_t)box_inner, (cuuint32_t)box_rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(map, dt == DT_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3,
                     const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <int BN, bool B_MN, bool PAIR, bool FIN, bool TRX, typename T, bool S1 = false>
static cudaError_t launch_one(const TcParams& prm, int grid, cudaStream_t stream) {
    using C = Cfg<BN, PAIR, B_MN, FIN, S1>;
    auto kern = tc_gemm_kernel<BN, B_MN, PAIR, FIN, TRX, T, S1>;
    static thread_local int configured_dev = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (configured_dev != dev) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
        if (e != cudaSuccess) return e;
        configured_dev = dev;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = C::kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    if (PAIR) {
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
    }
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, prm);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

muon_status tc_run(const GemmOp* ops, int nops, int dt, const FinalCtx& fc, const FinalEntry* fin,
                   int nfin, cudaStream_t stream) {
    if (nops <= 0) return MUON_OK;
    if (nops > kMaxProblems || nfin > kMaxFinal) return MUON_ERR_UNSUPPORTED;
    const int sym = ops[0].sym;
    // Products run on CTA pairs (cta_group::2, 256 x 256 tiles) unless
    // MUON_CTA_PAIRS=0 selects one CTA per tile (128 x 128 symmetric, 128 x 256
    // update).  On pairs every symmetric result also stores its first tile below
    // the diagonal, which pair consumers need.
    static const bool pair = [] {
        const char* v = getenv("MUON_CTA_PAIRS");
        return !(v && strcmp(v, "0") == 0);
    }();
    // Update products on pairs with K >= kWideMinK in every problem run on
    // 256 x 512 tiles: 25% fewer operand bytes per flop
    // (the operand stream per SM bounds these products) for an epilogue that no
    // longer overlaps the next tile's MMAs (one accumulator in all 512 columns).
    // MUON_WIDE_UPDATES=0 keeps 256 x 256 tiles.
    static const bool wide_ok = [] {
        const char* v = getenv("MUON_WIDE_UPDATES");
        return !(v && strcmp(v, "0") == 0);
    }();
    bool wide = wide_ok && pair && !sym && ops[0].epi.fin == FIN_STORE;
    for (int i = 0; i < nops; ++i) wide = wide && ops[i].K >= kWideMinK;
    // Symmetric products of one operand with itself (X X^T, S S) with s >= kWideMinK
    // in every problem run on 256 x 512 tiles too: row tile ti spans the 512-column
    // tiles from ti / 2, the blocks left of the diagonal computed and dropped.
    // MUON_WIDE_SYMMETRIC=0 keeps them on 256 x 256 tiles.
    static const bool wide_sym_ok = [] {
        const char* v = getenv("MUON_WIDE_SYMMETRIC");
        return !(v && strcmp(v, "0") == 0);
    }();
    bool wide_sym = wide_sym_ok && pair && sym != 0;
    for (int i = 0; i < nops; ++i) {
        const GemmOp& o = ops[i];
        wide_sym = wide_sym && o.N >= kWideMinK && o.A == o.B && o.lda == o.ldb && o.strideA == o.strideB &&
                   o.a_sym == o.b_sym && o.a_tr == o.b_tr;
    }
    const int BN = (sym && !pair) ? 128 : (wide || wide_sym) ? 512 : 256;
    const int rows_per_tile = pair ? 2 * BM : BM;
    // the final-step staging boxes overlap the store boxes: one kind per launch
    for (int i = 1; i < nops; ++i)
        if ((ops[i].epi.fin == FIN_STORE) != (ops[0].epi.fin == FIN_STORE)) return MUON_ERR_INVALID_ARG;
    static TcParams prm_storage;   // large: keep off the stack; filled and consumed within this call
    static std::mutex mu;
    std::lock_guard<std::mutex> lock(mu);
    TcParams& prm = prm_storage;
    memset(&prm, 0, sizeof(prm));
    long long tiles = 0;
    for (int i = 0; i < nops; ++i) {
        const GemmOp& o = ops[i];
        if (o.sym != sym) return MUON_ERR_INVALID_ARG;
        TcProblem& P = prm.prob[i];
        P.count = o.count; P.M = o.M; P.N = o.N; P.K = o.K; P.sym = sym;
        P.tiles_m = (o.M + rows_per_tile - 1) / rows_per_tile;
        P.tiles_n = (o.N + BN - 1) / BN;
        P.wide = wide_sym ? 1 : 0;
        if (wide_sym) {
            P.tiles_per_mat = 0;
            for (int ti = 0; ti < P.tiles_m; ++ti) P.tiles_per_mat += P.tiles_n - ti / 2;
        } else {
            P.tiles_per_mat = sym ? P.tiles_m * (P.tiles_m + 1) / 2 : P.tiles_m * P.tiles_n;
        }
        P.tile_begin = tiles;
        tiles += (long long)P.tiles_per_mat * o.count;
        P.epi = o.epi;
        P.a_sym = o.a_sym;
        P.b_sym = sym ? o.b_sym : 0;
        P.band = sym ? (pair ? 1 : o.band) : 0;
        P.a_tr = o.a_tr;
        P.b_tr = o.b_tr;
        P.same_ab = sym && o.A == o.B && o.lda == o.ldb && o.strideA == o.strideB && o.a_sym == o.b_sym &&
                    o.a_tr == o.b_tr;
        // A operand: M rows x K (K contiguous); a symmetric A is also read transposed;
        // a transposed A (K rows x M) only transposed
        if (!o.a_tr && !encode_map(&P.mapA, dt, o.A, o.K, o.M, o.count, o.lda, o.strideA, BK, BM))
            return MUON_ERR_CUDA;
        if ((o.a_sym || o.a_tr) && !encode_map(&P.mapAt, dt, o.A, o.a_tr ? o.M : o.K, o.a_tr ? o.K : o.M, o.count,
                                               o.lda, o.strideA, 64, BK))
            return MUON_ERR_CUDA;
        if (sym) {
            // each CTA of a pair loads half of the tile's B rows (128 of them for each
            // 256-column half of a 256 x 512 tile)
            if (!o.b_tr && !encode_map(&P.mapB, dt, o.B, o.K, o.N, o.count, o.ldb, o.strideB, BK,
                                       pair ? (BN == 512 ? 128 : BN / 2) : BN))
                return MUON_ERR_CUDA;
            if ((o.b_sym || o.b_tr) && !encode_map(&P.mapBt, dt, o.B, o.b_tr ? o.N : o.K, o.b_tr ? o.K : o.N,
                                                   o.count, o.ldb, o.strideB, 64, BK))
                return MUON_ERR_CUDA;
        } else if (o.b_tr) {
            // X stored N x K (K contiguous); boxes of BK (K) x the CTA's N columns (128 of
            // them per half of a 256 x 512 tile)
            if (!encode_map(&P.mapB, dt, o.B, o.K, o.N, o.count, o.ldb, o.strideB, BK,
                            BN == 512 ? 128 : (pair ? BN / 2 : BN)))
                return MUON_ERR_CUDA;
        } else {
            // X panel: K rows x N (N contiguous); boxes of 64 (N) x BK (K)
            if (!encode_map(&P.mapB, dt, o.B, o.N, o.K, o.count, o.ldb, o.strideB, 64, BK)) return MUON_ERR_CUDA;
        }
        if (o.epi.fin == FIN_STORE &&
            !encode_map(&P.mapD, dt, o.epi.D, o.N, o.M, o.count, o.epi.ldd, o.epi.strideD, 64, 32))
            return MUON_ERR_CUDA;
        if (P.band && (o.epi.fin != FIN_STORE ||
                       !encode_map(&P.mapDt, dt, o.epi.D, o.N, o.M, o.count, o.epi.ldd, o.epi.strideD, 32, 64,
                                   false)))
            return MUON_ERR_CUDA;
    }
    prm.nprob = nops;
    prm.total_tiles = tiles;
    prm.fc = fc;
    for (int i = 0; i < nfin; ++i) prm.fin[i] = fin[i];
    prm.fc.fin = nullptr;   // the kernel points it at its own copy of the table
    int dev = 0, nsm = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    const long long units = pair ? nsm / 2 : nsm;   // persistent CTAs (pairs)
    const int grid = (int)((tiles < units ? tiles : units) * (pair ? 2 : 1));
    if (grid <= 0) return MUON_OK;
    double work = 0.0;   // algorithmic flops: half of a symmetric product, all of a full one
    for (int i = 0; i < nops; ++i)
        work += sym ? (double)ops[i].count * ops[i].N * ops[i].N * ops[i].K
                    : 2.0 * ops[i].count * ops[i].M * ops[i].N * ops[i].K;
    trace_begin(sym ? MUON_KERNEL_SYM : MUON_KERNEL_UPD, work, stream);
    cudaError_t e;
    const bool final_step = ops[0].epi.fin != FIN_STORE;
    bool any_tr = false, one_operand = sym != 0;
    for (int i = 0; i < nops; ++i) {
        any_tr |= ops[i].a_tr || ops[i].b_tr;
        one_operand &= prm.prob[i].same_ab != 0;   // diagonal tiles exactly symmetric as formed
    }
    // one instantiation per product kind, CTA-pair mode, operand layouts and element type
#define MUON_TC_LAUNCH(TRX, T)                                                                         \
    do {                                                                                               \
        if (sym && wide_sym) e = launch_one<512, false, true, false, TRX, T, true>(prm, grid, stream); \
        else if (sym) e = pair ? (one_operand ? launch_one<256, false, true, false, TRX, T, true>(prm, grid, stream) \
                                         : launch_one<256, false, true, false, TRX, T>(prm, grid, stream))     \
                          : launch_one<128, false, false, false, TRX, T>(prm, grid, stream);           \
        else if (final_step) e = pair ? launch_one<256, true, true, true, TRX, T>(prm, grid, stream)   \
                               : launch_one<256, true, false, true, TRX, T>(prm, grid, stream);        \
        else if (wide) e = launch_one<512, true, true, false, TRX, T>(prm, grid, stream);              \
        else e = pair ? launch_one<256, true, true, false, TRX, T>(prm, grid, stream)                  \
                      : launch_one<256, true, false, false, TRX, T>(prm, grid, stream);                \
    } while (0)
    if (dt == DT_BF16) {
        if (any_tr) MUON_TC_LAUNCH(true, __nv_bfloat16);
        else MUON_TC_LAUNCH(false, __nv_bfloat16);
    } else {
        if (any_tr) MUON_TC_LAUNCH(true, __half);
        else MUON_TC_LAUNCH(false, __half);
    }
#undef MUON_TC_LAUNCH
    trace_end(stream);
    return e == cudaSuccess ? MUON_OK : MUON_ERR_CUDA;
}

}  // namespace tc
}  // namespace muon
