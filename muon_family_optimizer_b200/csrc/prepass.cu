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
// (ns_polar / gram_polar).
//
// Traffic per element (bf16 G/G_prev, fp32 A/M, bf16 copy): 12 bytes read,
// 12 bytes written; the norm costs no extra bytes.  Tiles of 32 rows x 64
// columns; 256 threads, 8 consecutive elements each (16-byte loads of
// 16-bit data, 2 x 16-byte loads of fp32).  Transposed copies go through a
// shared-memory tile so both the reads and the writes stay coalesced.
// Blocks own contiguous runs of tiles and flush the per-matrix sum once per
// run (warp shuffles, then one double atomic per block and matrix).
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

__global__ void __launch_bounds__(256) prep_kernel(const __grid_constant__ PrepParams p) {
    __shared__ float stile[TC][TR + 1];
    __shared__ double red[8];
    const long long T = p.total_tiles;
    const long long per = (T + gridDim.x - 1) / gridDim.x;
    const long long t_begin = (long long)blockIdx.x * per;
    const long long t_end = min(T, t_begin + per);
    const int r = threadIdx.x >> 3;          // row inside the tile
    const int c8 = (threadIdx.x & 7) * 8;    // first of 8 columns inside the tile
    int cur = -1;
    double acc = 0.0;
    int ei = 0;
    for (long long t = t_begin; t < t_end; ++t) {
        while (ei + 1 < p.n && t >= p.e[ei + 1].tile_begin) ++ei;
        const PrepEntry& E = p.e[ei];
        const long long local = t - E.tile_begin;
        const int b = (int)(local / E.tiles_per_mat);
        const long long tt = local - (long long)b * E.tiles_per_mat;
        const int tr = (int)(tt / E.tiles_c), tc = (int)(tt % E.tiles_c);
        const int key = E.sumsq_index + b;
        if (key != cur) {   // uniform over the block
            if (cur >= 0) {
                double s = block_sum(acc, red);
                if (threadIdx.x == 0) atomicAdd(&p.sumsq[cur], s);
            }
            cur = key;
            acc = 0.0;
        }
        const int gr = tr * TR + r;
        const int gc0 = tc * TC + c8;
        const int nvalid = gr < E.rows ? max(0, min(8, E.cols - gc0)) : 0;
        const bool vec = E.vec_ok && nvalid == 8;
        const long long idx = (long long)gr * E.cols + gc0;
        float x[8];
        if (p.mode == 0) {
            float g[8], gp[8], a[8], mm[8];
            load8_dt(E.G, idx, p.in_dt, vec, nvalid, g);
            load8_dt(E.Gp, idx, p.in_dt, vec, nvalid, gp);
            load8_dt(E.A, idx, DT_FP32, vec, nvalid, a);
            load8_dt(E.M, idx, DT_FP32, vec, nvalid, mm);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float d = g[i] - gp[i];                                   // step 1
                const float an = p.beta_a * a[i] + (1.f - p.beta_a) * d;        // step 2
                const float gt = g[i] + p.alpha * an;                            // step 3
                const float mn = p.mu * mm[i] + gt;                              // step 4
                a[i] = an;
                x[i] = mn;
            }
            store8_dt(E.A, idx, DT_FP32, vec, nvalid, a);
            store8_dt(E.M, idx, DT_FP32, vec, nvalid, x);
            store8_dt(E.Gp, idx, p.in_dt, vec, nvalid, g);
        } else {
            const void* X = static_cast<const char*>(E.X) + (size_t)b * E.x_stride * dt_size(p.in_dt);
            load8_dt(X, idx, p.in_dt, vec, nvalid, x);
        }
        float part = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) part += x[i] * x[i];
        acc += (double)part;

        void* X0 = static_cast<char*>(E.X0) + (size_t)b * E.x0_stride * dt_size(p.x0_dt);
        if (!E.transposed) {
            // wide view = the matrix itself; X0 rows are 16-byte aligned (ld % 8 == 0)
            store8_dt(X0, (long long)gr * E.ld + gc0, p.x0_dt, nvalid == 8, nvalid, x);
        } else {
            // wide view = transpose: X0[c][r] = M[r][c]
#pragma unroll
            for (int i = 0; i < 8; ++i) stile[c8 + i][r] = x[i];
            __syncthreads();
            const int cc = threadIdx.x >> 2;          // tile column -> X0 row
            const int rr0 = (threadIdx.x & 3) * 8;    // 8 tile rows -> X0 columns
            const int xrow = tc * TC + cc;
            const int xcol0 = tr * TR + rr0;
            if (xrow < E.cols) {
                float y[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) y[i] = stile[cc][rr0 + i];
                const int nv = max(0, min(8, E.rows - xcol0));
                store8_dt(X0, (long long)xrow * E.ld + xcol0, p.x0_dt, nv == 8, nv, y);
            }
            __syncthreads();
        }
    }
    if (cur >= 0) {
        double s = block_sum(acc, red);
        if (threadIdx.x == 0) atomicAdd(&p.sumsq[cur], s);
    }
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
        E.tile_begin = tiles;
        tiles += E.tiles_per_mat * E.count;
    }
    prm.total_tiles = tiles;
    if (tiles == 0) return MUON_OK;
    int dev = 0, nsm = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    const long long want = (long long)nsm * 8;
    const int grid = (int)(tiles < want ? tiles : want);
    double elems = 0.0;
    for (int i = 0; i < prm.n; ++i) elems += (double)prm.e[i].rows * prm.e[i].cols * prm.e[i].count;
    const int isz = dt_size(prm.in_dt), xsz = dt_size(prm.x0_dt);
    // MONA: read G, G_prev, A, M; write A, M, G_prev, X0.  COPY: read X, write X0.
    const double per = prm.mode == 0 ? 3.0 * isz + 16.0 + xsz : (double)(isz + xsz);
    trace_begin(MUON_KERNEL_PREPASS, elems * per, stream);
    prep_kernel<<<grid, 256, 0, stream>>>(prm);
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
