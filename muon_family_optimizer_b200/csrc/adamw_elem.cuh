// adamw_elem.cuh -- the per-element AdamW update shared by the standalone
// AdamW pass (adamw.cu) and the fused pre-pass of a whole-model step
// (prepass.cu), so that both compute the same bits.
//
// [MONA] section 2, "Ontwerprichtlijnen": vector-valued parameters keep the
// standard AdamW of Muon's convention, read as Adam with bias correction and
// decoupled weight decay, per element in fp32:
//     m <- b1 m + (1 - b1) g,   v <- b2 v + (1 - b2) g^2
//     W <- W - lr ( (m / (1 - b1^t)) / (sqrt(v / (1 - b2^t)) + eps) + wd W )
#pragma once

#include <cuda_runtime.h>

namespace muon {

struct AdamWCoeffs {
    float lr, b1, b2, eps, wd;
    float ic1, ic2;   // 1 / (1 - b1^t), 1 / (1 - b2^t)
};

// Update the first nvalid of 8 consecutive elements in registers.  An element
// with a non-finite gradient keeps its state; returns whether one was seen.
__device__ __forceinline__ bool adamw8(const AdamWCoeffs& c, float (&w)[8], const float (&g)[8], float (&m)[8],
                                       float (&v)[8], int nvalid) {
    bool bad = false;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        if (!isfinite(g[i])) {
            bad |= i < nvalid;
            continue;
        }
        const float mn = c.b1 * m[i] + (1.f - c.b1) * g[i];
        const float vn = c.b2 * v[i] + (1.f - c.b2) * g[i] * g[i];
        const float upd = (mn * c.ic1) / (sqrtf(vn * c.ic2) + c.eps);
        w[i] = w[i] - c.lr * (upd + c.wd * w[i]);
        m[i] = mn;
        v[i] = vn;
    }
    return bad;
}

}  // namespace muon
