// prepass.cu -- the fused elementwise pass ahead of the iteration.
//
// MONA mode ([MONA] section 2, steps 1-4, one read and one write of every
// state element):
//     D = G - G_prev;  A = beta_a A + (1 - beta_a) D;  Gt = G + alpha A;
//     M = mu M + Gt;   G_prev = G
// plus, for the orthogonalisation that follows, the sum of squares of the
// new M per matrix (Frobenius norm) and M rounded to the iteration's element
// type, written in the wide view (transposed when rows > cols) into the
// workspace.  COPY mode does the last two for a batch of input matrices
// (ns_polar / gram_polar); NORM mode only sums the squares, so that a
// following COPY pass can write the copy already divided by (||X|| + eps)
// (prescale) -- the iteration of a bfloat16 input runs in fp16, whose range
// needs the normalised values.
//
// Traffic per element (bf16 G/G_prev, fp32 A/M, bf16 copy): 12 bytes read,
// 12 bytes written; the norm costs no extra bytes.  Tiles of 32 rows x 64
// columns; 256 threads, each 8 consecutive elements of one row (16-byte loads
// of 16-bit data, 2 x 16-byte loads of fp32), all loads of a tile issued
// before any use; at most 64 registers so that four blocks share an SM.  The
// gradient is read once (streaming loads).  Transposed copies go through a
// shared-memory tile so both the reads and the writes stay coalesced.  Blocks own contiguous runs
// of tiles and flush the per-matrix sum once per run (warp shuffles, then one
// double atomic per block and matrix).
#include "gemm.h"

namespace muon {

namespace {

constexpr int TR = 32, TC = 64;

__device__ __forceinline__ double block_sum(double x, double* red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    const int w = threadIdx.x >> 5;
    if ((threadIdx.x & 31) == 0) red[w] = x;
    __syncthreads();
    double t = 0.0;
    if (threadIdx.x == 0)
        for (int i = 0; i < (int)(blockDim.x >> 5); ++i) t += red[i];
    __syncthreads();
    return t;
}

// 8 consecutive 16-bit elements, read once: no L1 allocation.
__device__ __forceinline__ uint4 ld_stream16(const void* p) {
    uint4 u;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(u.x), "=r"(u.y), "=r"(u.z), "=r"(u.w) : "l"(p));
    return u;
}

template <int dt>
__device__ __forceinline__ void load8_in(const void* base, long long idx, bool vec, int nvalid, float* out) {
    if (vec && dt != DT_FP32) {
        const uint4 u = ld_stream16(static_cast<const char*>(base) + idx * 2);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int h = 0; h < 4; ++h) {
            out[2 * h] = dt == DT_BF16 ? unpack_lo<__nv_bfloat16>(w[h]) : unpack_lo<__half>(w[h]);
            out[2 * h + 1] = dt == DT_BF16 ? unpack_hi<__nv_bfloat16>(w[h]) : unpack_hi<__half>(w[h]);
        }
    } else {
        load8_dt(base, idx, dt, vec, nvalid, out);
    }
}

template <int IN_DT, int X0_DT>
__global__ void __launch_bounds__(256, 4) prep_kernel(const __grid_constant__ PrepParams p) {
    __shared__ float stile[TC][TR + 1];
    __shared__ double red[8];
    const long long T = p.total_tiles;
    const long long per = (T + gridDim.x - 1) / gridDim.x;
    const long long t_begin = (long long)blockIdx.x * per;
    const long long t_end = min(T, t_begin + per);
    const int r = threadIdx.x >> 3;          // row r of the tile
    const int c8 = (threadIdx.x & 7) * 8;    // first of 8 columns inside the tile
    int cur = -1;
    double acc = 0.0;
    int ei = 0;
    bool bad = false;                        // an AdamW item saw a non-finite gradient
    for (long long t = t_begin; t < t_end; ++t) {
        while (ei + 1 < p.n && t >= p.e[ei + 1].tile_begin) ++ei;
        const PrepEntry& E = p.e[ei];
        const long long local = t - E.tile_begin;
        if (E.kind == 1) {
            // AdamW item (uniform over the block): TR*TC consecutive elements,
            // 8 per thread; nothing of the iteration follows
            const long long e0 = local * (TR * TC) + (long long)threadIdx.x * 8;
            const int nv = (int)max(0LL, min(8LL, E.nel - e0));
            if (nv > 0) {
                const bool vec = E.vec_ok && nv == 8;
                float w[8], g[8], m[8], v[8];
                load8_in<IN_DT>(E.G, e0, vec, nv, g);
                load8_dt(E.Gp, e0, IN_DT, vec, nv, w);
                load8_dt(E.A, e0, DT_FP32, vec, nv, m);
                load8_dt(E.M, e0, DT_FP32, vec, nv, v);
                bad |= adamw8(p.adam, w, g, m, v, nv);
                store8_dt(E.Gp, e0, IN_DT, vec, nv, w);
                store8_dt(E.A, e0, DT_FP32, vec, nv, m);
                store8_dt(E.M, e0, DT_FP32, vec, nv, v);
            }
            continue;
        }
        const int b = (int)(local / E.tiles_per_mat);
        const long long tt = local - (long long)b * E.tiles_per_mat;
        const int tr = E.flat ? 0 : (int)(tt / E.tiles_c), tc = E.flat ? 0 : (int)(tt % E.tiles_c);
        const int key = E.sumsq_index + b;
        if (key != cur) {   // uniform over the block
            if (cur >= 0 && !p.prescale) {
                double s = block_sum(acc, red);
                if (threadIdx.x == 0) atomicAdd(&p.sumsq[cur], s);
            }
            cur = key;
            acc = 0.0;
        }
        const int gc0 = tc * TC + c8;
        constexpr int H = TR / 32;           // rows per thread
        int gr[H], nvalid[H];
        bool vec[H];
        long long idx[H];
        static_assert(H == 1, "the contiguous layout below gives each thread one group of 8");
        if (E.flat) {
            // contiguous run of TR*TC elements: thread i takes elements 8i..8i+7
            const long long e0 = tt * (TR * TC) + (long long)threadIdx.x * 8;
            const long long n = (long long)E.rows * E.cols;
            gr[0] = 0;
            nvalid[0] = (int)max(0LL, min(8LL, n - e0));
            vec[0] = E.vec_ok && nvalid[0] == 8;
            idx[0] = e0;
        } else {
#pragma unroll
            for (int h = 0; h < H; ++h) {
                gr[h] = tr * TR + r + 32 * h;
                nvalid[h] = gr[h] < E.rows ? max(0, min(8, E.cols - gc0)) : 0;
                vec[h] = E.vec_ok && nvalid[h] == 8;
                idx[h] = (long long)gr[h] * E.cols + gc0;
            }
        }
        float x[H][8];
        if (p.mode == 0) {
            float g[H][8], gp[H][8], a[H][8], mm[H][8];
#pragma unroll
            for (int h = 0; h < H; ++h) {        // every load of the tile first
                load8_in<IN_DT>(E.G, idx[h], vec[h], nvalid[h], g[h]);
                load8_in<IN_DT>(E.Gp, idx[h], vec[h], nvalid[h], gp[h]);
                load8_dt(E.A, idx[h], DT_FP32, vec[h], nvalid[h], a[h]);
                load8_dt(E.M, idx[h], DT_FP32, vec[h], nvalid[h], mm[h]);
            }
#pragma unroll
            for (int h = 0; h < H; ++h) {
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float d = g[h][i] - gp[h][i];                            // step 1
                    const float an = p.beta_a * a[h][i] + (1.f - p.beta_a) * d;    // step 2
                    const float gt = g[h][i] + p.alpha * an;                        // step 3
                    const float mn = p.mu * mm[h][i] + gt;                          // step 4
                    a[h][i] = an;
                    x[h][i] = mn;
                }
                store8_dt(E.A, idx[h], DT_FP32, vec[h], nvalid[h], a[h]);
                store8_dt(E.M, idx[h], DT_FP32, vec[h], nvalid[h], x[h]);
                store8_dt(E.Gp, idx[h], IN_DT, vec[h], nvalid[h], g[h]);
            }
        } else if (p.mode == 2) {
            // MONA-Lite: B = beta_a A - (1 - beta_a) G of the previous step, bfloat16
            float g[H][8], bb[H][8], mm[H][8];
#pragma unroll
            for (int h = 0; h < H; ++h) {
                load8_in<IN_DT>(E.G, idx[h], vec[h], nvalid[h], g[h]);
                load8_in<DT_BF16>(E.Gp, idx[h], vec[h], nvalid[h], bb[h]);
                load8_dt(E.M, idx[h], DT_FP32, vec[h], nvalid[h], mm[h]);
            }
#pragma unroll
            for (int h = 0; h < H; ++h) {
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float an = bb[h][i] + (1.f - p.beta_a) * g[h][i];       // step 2 (= A_k)
                    const float gt = g[h][i] + p.alpha * an;                         // step 3
                    x[h][i] = p.mu * mm[h][i] + gt;                                  // step 4
                    bb[h][i] = p.beta_a * an - (1.f - p.beta_a) * g[h][i];           // next step's B
                }
                store8_dt(E.M, idx[h], DT_FP32, vec[h], nvalid[h], x[h]);
                store8_dt(E.Gp, idx[h], DT_BF16, vec[h], nvalid[h], bb[h]);
            }
        } else {   // COPY or NORM
            const void* X = static_cast<const char*>(E.X) + (size_t)b * E.x_stride * dt_size(IN_DT);
#pragma unroll
            for (int h = 0; h < H; ++h) load8_in<IN_DT>(X, idx[h], vec[h], nvalid[h], x[h]);
            if (p.prescale) {   // the norm is complete: store X / (||X|| + eps)
                const float sc = (float)(1.0 / (sqrt(p.sumsq[key]) + (double)p.eps));
#pragma unroll
                for (int h = 0; h < H; ++h)
#pragma unroll
                    for (int i = 0; i < 8; ++i) x[h][i] *= sc;
            }
        }
        float part = 0.f;
#pragma unroll
        for (int h = 0; h < H; ++h)
#pragma unroll
            for (int i = 0; i < 8; ++i) part += x[h][i] * x[h][i];
        acc += (double)part;
        if (p.mode == 3) continue;   // NORM: nothing to store (uniform over the block)

        void* X0 = static_cast<char*>(E.X0) + (size_t)b * E.x0_stride * dt_size(X0_DT);
        if (!E.transposed) {
            // wide view = the matrix itself; X0 rows are 16-byte aligned (ld % 8 == 0)
#pragma unroll
            for (int h = 0; h < H; ++h)
                store8_dt(X0, E.flat ? idx[h] : (long long)gr[h] * E.ld + gc0, X0_DT, nvalid[h] == 8, nvalid[h], x[h]);
        } else {
            // wide view = transpose: X0[c][r] = M[r][c], written as TR-row column segments
#pragma unroll
            for (int h = 0; h < H; ++h)
#pragma unroll
                for (int i = 0; i < 8; ++i) stile[c8 + i][r + 32 * h] = x[h][i];
            __syncthreads();
            const int cc = threadIdx.x >> 2;          // tile column -> X0 row
            const int rr0 = (threadIdx.x & 3) * (TR / 4);   // TR/4 tile rows -> X0 columns
            const int xrow = tc * TC + cc;
            if (xrow < E.cols) {
#pragma unroll
                for (int h = 0; h < H; ++h) {
                    const int xcol0 = tr * TR + rr0 + 8 * h;
                    float y[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) y[i] = stile[cc][rr0 + 8 * h + i];
                    const int nv = max(0, min(8, E.rows - xcol0));
                    store8_dt(X0, (long long)xrow * E.ld + xcol0, X0_DT, nv == 8, nv, y);
                }
            }
            __syncthreads();
        }
    }
    if (cur >= 0 && !p.prescale) {
        double s = block_sum(acc, red);
        if (threadIdx.x == 0) atomicAdd(&p.sumsq[cur], s);
    }
    if (__syncthreads_or(bad) && threadIdx.x == 0 && p.d_status) atomicOr(p.d_status, MUON_FLAG_NONFINITE);
}

__global__ void identity_kernel(void* D, int dt, int count, int s, long long ld, long long stride) {
    const long long total = (long long)count * s * s;
    for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < total;
         e += (long long)gridDim.x * blockDim.x) {
        const int m = (int)(e / ((long long)s * s));
        const long long rem = e - (long long)m * s * s;
        const int i = (int)(rem / s), j = (int)(rem % s);
        st_elem(D, (long long)m * stride + (long long)i * ld + j, dt, i == j ? 1.f : 0.f);
    }
}

}  // namespace

muon_status prep_run(PrepParams& prm, cudaStream_t stream) {
    long long tiles = 0;
    for (int i = 0; i < prm.n; ++i) {
        PrepEntry& E = prm.e[i];
        const int tiles_r = (E.rows + TR - 1) / TR;
        E.tiles_c = (E.cols + TC - 1) / TC;
        E.tiles_per_mat = (long long)tiles_r * E.tiles_c;
        // not transposed and X0 rows unpadded: every buffer of the matrix is one
        // contiguous array, processed in runs of TR*TC elements (long coalesced
        // streams per array instead of TR separate row segments)
        E.flat = !E.transposed && E.ld == E.cols;
        if (E.flat) E.tiles_per_mat = ((long long)E.rows * E.cols + TR * TC - 1) / (TR * TC);
        if (E.kind == 1) E.tiles_per_mat = (E.nel + TR * TC - 1) / (TR * TC);
        E.tile_begin = tiles;
        tiles += E.tiles_per_mat * E.count;
    }
    prm.total_tiles = tiles;
    if (tiles == 0) return MUON_OK;
    int dev = 0, nsm = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    // one wave of resident blocks: each block owns a contiguous run of tiles
    static int occ = 0;
    if (occ <= 0 && cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, prep_kernel<DT_BF16, DT_BF16>, 256, 0) !=
                        cudaSuccess)
        occ = 1;
    const long long want = (long long)nsm * (occ > 0 ? occ : 1);
    const int grid = (int)(tiles < want ? tiles : want);
    double elems = 0.0, vec_elems = 0.0;
    for (int i = 0; i < prm.n; ++i) {
        if (prm.e[i].kind == 1) vec_elems += (double)prm.e[i].nel;
        else elems += (double)prm.e[i].rows * prm.e[i].cols * prm.e[i].count;
    }
    const int isz = dt_size(prm.in_dt), xsz = dt_size(prm.x0_dt);
    // MONA: read G, G_prev, A, M; write A, M, G_prev, X0.  COPY: read X, write X0.
    // MONA-Lite: read G, B, M; write B, M, X0.  NORM: read X.
    // AdamW item: read G, W, m, v; write W, m, v.
    const double per = prm.mode == 0 ? 3.0 * isz + 16.0 + xsz
                     : prm.mode == 2 ? isz + 12.0 + xsz : prm.mode == 3 ? (double)isz : (double)(isz + xsz);
    trace_begin(MUON_KERNEL_PREPASS, elems * per + vec_elems * (3.0 * isz + 16.0), stream);
    // element types are compile-time in the kernel: loads and stores stay in registers
#define MUON_PREP(I, X)                                                   \
    if (prm.in_dt == I && prm.x0_dt == X) prep_kernel<I, X><<<grid, 256, 0, stream>>>(prm);
    MUON_PREP(DT_BF16, DT_BF16) else MUON_PREP(DT_BF16, DT_FP16) else MUON_PREP(DT_BF16, DT_FP32)
    else MUON_PREP(DT_FP16, DT_BF16) else MUON_PREP(DT_FP16, DT_FP16) else MUON_PREP(DT_FP16, DT_FP32)
    else MUON_PREP(DT_FP32, DT_BF16) else MUON_PREP(DT_FP32, DT_FP16) else MUON_PREP(DT_FP32, DT_FP32)
#undef MUON_PREP
    trace_end(stream);
    return cudaGetLastError() == cudaSuccess ? MUON_OK : MUON_ERR_CUDA;
}

muon_status fill_identity(void* D, int dt, int count, int s, long long ld, long long stride,
                          cudaStream_t stream) {
    trace_begin(MUON_KERNEL_OTHER, (double)count * s * s * dt_size(dt), stream);
    identity_kernel<<<256, 256, 0, stream>>>(D, dt, count, s, ld, stride);
    trace_end(stream);
    return cudaGetLastError() == cudaSuccess ? MUON_OK : MUON_ERR_CUDA;
}

}  // namespace muon
