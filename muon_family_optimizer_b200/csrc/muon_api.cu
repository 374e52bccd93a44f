// muon_api.cu -- the C ABI declared in include/muon.h.
//
// Host-side orchestration only: argument checks, workspace layout, grouping
// of parameters by (short side, long side), and the sequence of kernel
// launches of one step.  All arithmetic runs in the kernels of prepass.cu,
// gemm_tc.cu (16-bit, tensor cores) and gemm_simt.cu (fp32, CUDA cores).
#include <math.h>
#include <string.h>

#include <algorithm>
#include <map>
#include <vector>

#include "gemm.h"

namespace muon {
namespace {

constexpr size_t kAlign = 1024;
constexpr int kMaxSteps = 64;
constexpr int kMaxRestarts = 64;
constexpr int kMaxGroupMembers = kMaxFinal;   // one final launch table per group

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
inline long long pad8(long long x) { return (x + 7) / 8 * 8; }

bool valid_dtype(int d) { return d == DT_BF16 || d == DT_FP16 || d == DT_FP32; }

muon_status check_schedule(const muon_schedule* s) {
    if (!s || s->n_steps < 1 || s->n_steps > kMaxSteps || !s->coeffs) return MUON_ERR_INVALID_ARG;
    if (!(s->eps >= 0.f) || !isfinite(s->eps)) return MUON_ERR_INVALID_ARG;
    if (!(s->scale_f >= 1.f) || !isfinite(s->scale_f)) return MUON_ERR_INVALID_ARG;
    if (s->n_restarts < 0 || s->n_restarts > kMaxRestarts) return MUON_ERR_INVALID_ARG;
    if (s->n_restarts > 0 && !s->restarts) return MUON_ERR_INVALID_ARG;
    for (int i = 0; i < s->n_restarts; ++i)
        if (s->restarts[i] < 0 || s->restarts[i] >= s->n_steps) return MUON_ERR_INVALID_ARG;
    for (int k = 0; k < s->n_steps; ++k) {
        const muon_ns_coeff& c = s->coeffs[k];
        if (!isfinite(c.a) || !isfinite(c.b) || !isfinite(c.c)) return MUON_ERR_INVALID_ARG;
    }
    return MUON_OK;
}

bool is_restart(const muon_schedule* s, int k) {
    if (k == 0) return false;
    for (int i = 0; i < s->n_restarts; ++i)
        if (s->restarts[i] == k) return true;
    return false;
}

muon_status check_device() {
    int dev = 0, major = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MUON_ERR_CUDA;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
        return MUON_ERR_CUDA;
    return major == 10 ? MUON_OK : MUON_ERR_UNSUPPORTED;
}

// ---------------------------------------------------------------- layouts

// A batch of same-shape matrices in the wide view (s <= l).
struct Group {
    int s = 0, l = 0;
    std::vector<int> members;        // indices into the caller's parameter array
    long long ldl = 0, lds = 0;      // padded row strides of s x l and s x s buffers
    size_t x[2] = {0, 0};            // s x l ping-pong
    size_t sq[6] = {0, 0, 0, 0, 0, 0};   // s x s buffers (direct route uses 2, Gram route 6)
    int sumsq0 = 0;                  // first sumsq slot of this group
};

struct Layout {
    size_t status = 0, sumsq = 0, total = 0;
    std::vector<Group> groups;
};

void place_group(Group& g, size_t& off, int esz, int nsq) {
    const long long cnt = (long long)g.members.size();
    g.ldl = pad8(g.l);
    g.lds = pad8(g.s);
    for (int i = 0; i < 2; ++i) {
        g.x[i] = off;
        off = align_up(off + (size_t)cnt * g.s * g.ldl * esz, kAlign);
    }
    for (int i = 0; i < nsq; ++i) {
        g.sq[i] = off;
        off = align_up(off + (size_t)cnt * g.s * g.lds * esz, kAlign);
    }
}

// Parameters grouped by (s, l); a group holds at most kMaxGroupMembers.
Layout step_layout(const muon_param* params, int n, int ns_dt) {
    Layout L;
    std::map<std::pair<int, int>, std::vector<int>> by_shape;
    for (int i = 0; i < n; ++i) {
        const int s = std::min(params[i].rows, params[i].cols);
        const int l = std::max(params[i].rows, params[i].cols);
        by_shape[{s, l}].push_back(i);
    }
    std::vector<Group> groups;
    for (auto& kv : by_shape) {
        const std::vector<int>& all = kv.second;
        for (size_t b = 0; b < all.size(); b += kMaxGroupMembers) {
            Group g;
            g.s = kv.first.first;
            g.l = kv.first.second;
            g.members.assign(all.begin() + b, all.begin() + std::min(all.size(), b + kMaxGroupMembers));
            groups.push_back(g);
        }
    }
    // heaviest groups first: their tiles are scheduled first in each launch
    std::stable_sort(groups.begin(), groups.end(), [](const Group& a, const Group& b) {
        return (double)a.s * a.s * a.l * a.members.size() > (double)b.s * b.s * b.l * b.members.size();
    });
    size_t off = 0;
    L.status = off;
    off = align_up(off + 256, kAlign);
    L.sumsq = off;
    off = align_up(off + sizeof(double) * (size_t)n, kAlign);
    const int esz = dt_size(ns_dt);
    int slot = 0;
    for (Group& g : groups) {
        g.sumsq0 = slot;
        slot += (int)g.members.size();
        place_group(g, off, esz, 2);
    }
    L.groups = groups;
    L.total = off;
    return L;
}

Layout batch_layout(int batch, int rows, int cols, int dt, int nsq) {
    Layout L;
    Group g;
    g.s = std::min(rows, cols);
    g.l = std::max(rows, cols);
    g.members.resize(batch);
    size_t off = 0;
    L.status = off;
    off = align_up(off + 256, kAlign);
    L.sumsq = off;
    off = align_up(off + sizeof(double) * (size_t)batch, kAlign);
    place_group(g, off, dt_size(dt), nsq);
    L.groups.push_back(g);
    L.total = off;
    return L;
}

inline void* at(void* ws, size_t off) { return static_cast<char*>(ws) + off; }

// ---------------------------------------------------------------- launching

struct Runner {
    int dt;                 // element type of the iteration
    FinalCtx fc;
    cudaStream_t stream;

    // Run ops that share `sym`; the tensor-core path packs up to four per launch.
    muon_status run(const std::vector<GemmOp>& ops, const std::vector<FinalEntry>& fin) {
        if (ops.empty()) return MUON_OK;
        if (dt == DT_FP32) return simt::simt_run(ops.data(), (int)ops.size(), fc, fin.data(), (int)fin.size(), stream);
        for (size_t b = 0; b < ops.size(); b += kMaxProblems) {
            const int n = (int)std::min(ops.size() - b, (size_t)kMaxProblems);
            muon_status st = tc::tc_run(ops.data() + b, n, dt, fc, fin.data(), (int)fin.size(), stream);
            if (st != MUON_OK) return st;
        }
        return MUON_OK;
    }
};

Epilogue epi_store(void* D, long long ldd, long long strideD) {
    Epilogue e;
    memset(&e, 0, sizeof(e));
    e.D = D; e.ldd = ldd; e.strideD = strideD;
    e.alpha = 1.f; e.beta = 0.f; e.diag = 0.f; e.sc_mul = 1.f;
    e.fin = FIN_STORE;
    return e;
}

// D = A B^T, symmetric result; a_sym / b_sym: the operand itself is a stored
// symmetric matrix (only its upper tiles are valid on the tensor-core path).
GemmOp sym_op(int count, int n, int k, const void* A, long long lda, long long sA, const void* B,
              long long ldb, long long sB, const Epilogue& e, int a_sym = 0, int b_sym = 0, int band = 0) {
    GemmOp o;
    o.sym = 1; o.a_sym = a_sym; o.b_sym = b_sym; o.band = band; o.count = count; o.M = n; o.N = n; o.K = k;
    o.A = A; o.lda = lda; o.strideA = sA;
    o.B = B; o.ldb = ldb; o.strideB = sB;
    o.epi = e;
    return o;
}

// D = A X with A a stored symmetric s x s matrix and X s x l.
GemmOp upd_op(int count, int s, int l, const void* A, long long lda, long long sA, const void* X,
              long long ldx, long long sX, const Epilogue& e) {
    GemmOp o;
    o.sym = 0; o.a_sym = 1; o.b_sym = 0; o.band = 0; o.count = count; o.M = s; o.N = l; o.K = s;
    o.A = A; o.lda = lda; o.strideA = sA;
    o.B = X; o.ldb = ldx; o.strideB = sX;
    o.epi = e;
    return o;
}

// The direct quintic iteration on every group of `L`, starting from the
// unnormalised wide views in x[0] (norms in sumsq).  The last step's
// epilogue is `final_epi` (FIN_OUT or FIN_WUPD) with the given table.
muon_status run_direct(Runner& R, const Layout& L, void* ws, const muon_schedule* sch,
                       const std::vector<std::vector<FinalEntry>>& fin_per_group, int final_kind) {
    const int esz = dt_size(R.dt);
    const double* sumsq = static_cast<const double*>(at(ws, L.sumsq));
    const float f = sch->scale_f;
    int cur = 0;
    for (int k = 0; k < sch->n_steps; ++k) {
        const muon_ns_coeff c = sch->coeffs[k];
        const bool first = k == 0;
        const float pre = first ? 1.f / f : (is_restart(sch, k) ? 1.f / f : 1.f);
        const bool last = k == sch->n_steps - 1;
        // A = X X^T (scaled by pre^2, and by 1/(|M|+eps)^2 at the first step)
        std::vector<GemmOp> ops;
        for (const Group& g : L.groups) {
            const int cnt = (int)g.members.size();
            const long long sx = (long long)g.s * g.ldl, ss = (long long)g.s * g.lds;
            Epilogue e = epi_store(at(ws, g.sq[0]), g.lds, ss);
            e.sc_mul = pre * pre;
            if (first) { e.sumsq = sumsq + g.sumsq0; e.eps = sch->eps; e.sc_pow = 2; }
            ops.push_back(sym_op(cnt, g.s, g.l, at(ws, g.x[cur]), g.ldl, sx, at(ws, g.x[cur]), g.ldl, sx, e));
        }
        muon_status st = R.run(ops, {});
        if (st != MUON_OK) return st;
        // B' = a I + b A + c A A   (the a X term of the step rides on the diagonal)
        ops.clear();
        for (const Group& g : L.groups) {
            const int cnt = (int)g.members.size();
            const long long ss = (long long)g.s * g.lds;
            Epilogue e = epi_store(at(ws, g.sq[1]), g.lds, ss);
            e.alpha = c.c; e.beta = c.b; e.diag = c.a;
            e.Cin = at(ws, g.sq[0]); e.ldc = g.lds; e.strideC = ss;
            ops.push_back(sym_op(cnt, g.s, g.s, at(ws, g.sq[0]), g.lds, ss, at(ws, g.sq[0]), g.lds, ss, e, 1, 1, 1));
        }
        st = R.run(ops, {});
        if (st != MUON_OK) return st;
        // X' = pre B' X   (and 1/(|M|+eps) at the first step); on the last
        // step the result goes to the caller (FIN_OUT) or into W (FIN_WUPD).
        // A launch carries at most kMaxProblems groups and kMaxFinal table rows.
        ops.clear();
        std::vector<FinalEntry> fin;
        for (size_t gi = 0; gi < L.groups.size(); ++gi) {
            const Group& g = L.groups[gi];
            const int cnt = (int)g.members.size();
            const long long sx = (long long)g.s * g.ldl, ss = (long long)g.s * g.lds;
            Epilogue e = epi_store(at(ws, g.x[cur ^ 1]), g.ldl, sx);
            e.sc_mul = pre;
            if (first) { e.sumsq = sumsq + g.sumsq0; e.eps = sch->eps; e.sc_pow = 1; }
            const int rows_needed = (last && final_kind == FIN_WUPD) ? cnt : 0;
            if (!ops.empty() && (ops.size() == (size_t)kMaxProblems || (int)fin.size() + rows_needed > kMaxFinal)) {
                st = R.run(ops, fin);
                if (st != MUON_OK) return st;
                ops.clear();
                fin.clear();
            }
            if (last) {
                e.fin = final_kind;
                e.check = sumsq + g.sumsq0;
                if (rows_needed) {
                    e.fin_base = (int)fin.size();
                    fin.insert(fin.end(), fin_per_group[gi].begin(), fin_per_group[gi].end());
                }
            }
            ops.push_back(upd_op(cnt, g.s, g.l, at(ws, g.sq[1]), g.lds, ss, at(ws, g.x[cur]), g.ldl, sx, e));
        }
        st = R.run(ops, fin);
        if (st != MUON_OK) return st;
        cur ^= 1;
    }
    return MUON_OK;
}

// The Gram route for one batch group (see include/muon.h).
muon_status run_gram(Runner& R, const Layout& L, void* ws, const muon_schedule* sch) {
    const Group& g = L.groups[0];
    const int cnt = (int)g.members.size();
    const long long sx = (long long)g.s * g.ldl, ss = (long long)g.s * g.lds;
    const double* sumsq = static_cast<const double*>(at(ws, L.sumsq)) + g.sumsq0;
    const float f = sch->scale_f;
    // buffer roles: indices into g.sq
    int iR = 0, iRn = 1, iH = 2, iQ = 3, iQn = 4, iT = 5;
    int xb = 0;                 // current Xb buffer
    bool xb_raw = true;         // Xb still holds the unnormalised input (scale pending)
    bool q_identity = true;
    auto sq = [&](int i) { return at(ws, g.sq[i]); };
    auto xbuf = [&](int i) { return at(ws, g.x[i]); };

    // R = Xb Xb^T / ((|X|+eps) f)^2
    {
        Epilogue e = epi_store(sq(iR), g.lds, ss);
        e.sc_mul = 1.f / (f * f); e.sumsq = sumsq; e.eps = sch->eps; e.sc_pow = 2;
        muon_status st = R.run({sym_op(cnt, g.s, g.l, xbuf(xb), g.ldl, sx, xbuf(xb), g.ldl, sx, e)}, {});
        if (st != MUON_OK) return st;
    }
    auto apply_q = [&](Epilogue e) -> muon_status {
        // Xb' = scale * Q Xb  (the pending normalisation folded in)
        if (xb_raw) { e.sc_mul *= 1.f / f; e.sumsq = sumsq; e.eps = sch->eps; e.sc_pow = 1; }
        if (q_identity) {
            muon_status st = fill_identity(sq(iQ), R.dt, cnt, g.s, g.lds, ss, R.stream);
            if (st != MUON_OK) return st;
        }
        return R.run({upd_op(cnt, g.s, g.l, sq(iQ), g.lds, ss, xbuf(xb), g.ldl, sx, e)}, {});
    };
    for (int k = 0; k < sch->n_steps; ++k) {
        const muon_ns_coeff c = sch->coeffs[k];
        muon_status st;
        if (is_restart(sch, k)) {
            // Xb <- Q Xb / f;  R <- Xb Xb^T;  Q <- I
            Epilogue e = epi_store(xbuf(xb ^ 1), g.ldl, sx);
            e.sc_mul = 1.f / f;
            st = apply_q(e);
            if (st != MUON_OK) return st;
            xb ^= 1;
            xb_raw = false;
            q_identity = true;
            Epilogue e2 = epi_store(sq(iR), g.lds, ss);
            st = R.run({sym_op(cnt, g.s, g.l, xbuf(xb), g.ldl, sx, xbuf(xb), g.ldl, sx, e2)}, {});
            if (st != MUON_OK) return st;
        }
        // h = a I + b R + c R R
        {
            Epilogue e = epi_store(sq(iH), g.lds, ss);
            e.alpha = c.c; e.beta = c.b; e.diag = c.a;
            e.Cin = sq(iR); e.ldc = g.lds; e.strideC = ss;
            st = R.run({sym_op(cnt, g.s, g.s, sq(iR), g.lds, ss, sq(iR), g.lds, ss, e, 1, 1, 1)}, {});
            if (st != MUON_OK) return st;
        }
        const bool need_r = k + 1 < sch->n_steps && !is_restart(sch, k + 1);
        // Q <- h Q  and  T = h R  (one launch)
        std::vector<GemmOp> ops;
        if (!q_identity)
            ops.push_back(sym_op(cnt, g.s, g.s, sq(iH), g.lds, ss, sq(iQ), g.lds, ss, epi_store(sq(iQn), g.lds, ss),
                                 1, 1, 1));
        if (need_r)
            ops.push_back(sym_op(cnt, g.s, g.s, sq(iH), g.lds, ss, sq(iR), g.lds, ss, epi_store(sq(iT), g.lds, ss),
                                 1, 1));
        st = R.run(ops, {});
        if (st != MUON_OK) return st;
        const int h_buf = iH;     // h stays in this buffer until the end of the step
        if (q_identity) {
            std::swap(iQ, iH);    // Q = h: Q takes over h's buffer, the old Q buffer is free
            q_identity = false;
        } else {
            std::swap(iQ, iQn);
        }
        // R <- (h R) h
        if (need_r) {
            st = R.run({sym_op(cnt, g.s, g.s, sq(iT), g.lds, ss, sq(h_buf), g.lds, ss,
                               epi_store(sq(iRn), g.lds, ss), 1, 1)}, {});
            if (st != MUON_OK) return st;
            std::swap(iR, iRn);
        }
    }
    // X = Q Xb  -> caller's output
    Epilogue e = epi_store(nullptr, 0, 0);
    e.fin = FIN_OUT;
    e.check = sumsq;
    return apply_q(e);
}

}  // namespace
}  // namespace muon

using namespace muon;

extern "C" {

const char* muon_status_string(muon_status s) {
    switch (s) {
        case MUON_OK: return "ok";
        case MUON_ERR_INVALID_ARG: return "invalid argument";
        case MUON_ERR_UNSUPPORTED: return "unsupported (needs an sm_100 GPU, or a shape limit was exceeded)";
        case MUON_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
        case MUON_ERR_NONFINITE: return "non-finite norm: the matrix was left unchanged";
        case MUON_ERR_CUDA: return "CUDA runtime or driver error";
        case MUON_ERR_TIMEOUT: return "a device-side wait ran out";
    }
    return "unknown status";
}

static muon_status check_params(const muon_param* params, int n) {
    if (!params || n < 1) return MUON_ERR_INVALID_ARG;
    for (int i = 0; i < n; ++i) {
        const muon_param& p = params[i];
        if (p.rows < 1 || p.cols < 1) return MUON_ERR_INVALID_ARG;
        if ((long long)p.rows * p.cols > (1LL << 40)) return MUON_ERR_UNSUPPORTED;
    }
    return MUON_OK;
}

muon_status muon_workspace_size(const muon_param* params, int n, muon_dtype ns_dtype, size_t* bytes) {
    if (!bytes || !valid_dtype(ns_dtype)) return MUON_ERR_INVALID_ARG;
    muon_status st = check_params(params, n);
    if (st != MUON_OK) return st;
    *bytes = step_layout(params, n, ns_dtype).total;
    return MUON_OK;
}

// lite: MONA-Lite state (G_prev holds the bfloat16 buffer B, A is unused).
static muon_status step_common(const muon_param* params, int n, muon_dtype w_dtype, muon_dtype ns_dtype,
                               const muon_hparams* hp, const muon_schedule* sched, void* workspace,
                               size_t ws_bytes, int* d_status, muon_stream_t stream, bool lite) {
    if (!valid_dtype(w_dtype) || !valid_dtype(ns_dtype) || !hp) return MUON_ERR_INVALID_ARG;
    muon_status st = check_params(params, n);
    if (st != MUON_OK) return st;
    for (int i = 0; i < n; ++i)
        if (!params[i].W || !params[i].G || !params[i].G_prev || (!lite && !params[i].A) || !params[i].M)
            return MUON_ERR_INVALID_ARG;
    st = check_schedule(sched);
    if (st != MUON_OK) return st;
    const float hv[6] = {hp->mu, hp->eta, hp->lambda, hp->gamma, hp->beta_a, hp->alpha};
    for (float v : hv)
        if (!isfinite(v)) return MUON_ERR_INVALID_ARG;
    Layout L = step_layout(params, n, ns_dtype);
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255) || ws_bytes < L.total)
        return MUON_ERR_WORKSPACE;
    st = check_device();
    if (st != MUON_OK) return st;
    cudaStream_t stream_ = reinterpret_cast<cudaStream_t>(stream);
    int* status = d_status ? d_status : static_cast<int*>(at(workspace, L.status));
    double* sumsq = static_cast<double*>(at(workspace, L.sumsq));
    if (cudaMemsetAsync(sumsq, 0, sizeof(double) * n, stream_) != cudaSuccess) return MUON_ERR_CUDA;

    // 1. fused MONA pre-pass + norms + wide-view copies
    PrepParams pp;
    memset(&pp, 0, sizeof(pp));
    pp.in_dt = w_dtype; pp.x0_dt = ns_dtype; pp.mode = lite ? 2 : 0;
    pp.beta_a = hp->beta_a; pp.alpha = hp->alpha; pp.mu = hp->mu;
    pp.sumsq = sumsq;
    const size_t in_sz = dt_size(w_dtype);
    for (const Group& g : L.groups) {
        for (size_t j = 0; j < g.members.size(); ++j) {
            const muon_param& p = params[g.members[j]];
            PrepEntry& E = pp.e[pp.n++];
            E.G = p.G; E.Gp = p.G_prev; E.A = p.A; E.M = p.M;
            E.rows = p.rows; E.cols = p.cols; E.count = 1;
            E.transposed = p.rows > p.cols;
            E.X0 = static_cast<char*>(at(workspace, g.x[0])) + j * (size_t)g.s * g.ldl * dt_size(ns_dtype);
            E.ld = g.ldl;
            E.sumsq_index = g.sumsq0 + (int)j;
            const uintptr_t al = reinterpret_cast<uintptr_t>(p.G) | reinterpret_cast<uintptr_t>(p.G_prev) |
                                 reinterpret_cast<uintptr_t>(p.A) | reinterpret_cast<uintptr_t>(p.M);
            E.vec_ok = (p.cols % 8 == 0) && (al & 15) == 0 && in_sz >= 2;
            if (pp.n == kMaxPrep) {
                st = prep_run(pp, stream_);
                if (st != MUON_OK) return st;
                pp.n = 0;
            }
        }
    }
    if (pp.n > 0) {
        st = prep_run(pp, stream_);
        if (st != MUON_OK) return st;
    }

    // 2-3. iteration with the weight update fused into its last step
    Runner R;
    R.dt = ns_dtype;
    R.stream = stream_;
    memset(&R.fc, 0, sizeof(R.fc));
    R.fc.w_dt = w_dtype;
    R.fc.eta = hp->eta;
    R.fc.lambda = hp->lambda;
    R.fc.d_status = status;
    std::vector<std::vector<FinalEntry>> fins;
    for (const Group& g : L.groups) {
        std::vector<FinalEntry> f;
        for (int idx : g.members) {
            const muon_param& p = params[idx];
            FinalEntry fe;
            fe.W = p.W;
            fe.O_out = p.O_out;
            fe.gamma = isnan(p.gamma) ? hp->gamma : p.gamma;
            fe.transposed = p.rows > p.cols;
            const uintptr_t al = reinterpret_cast<uintptr_t>(p.W) | reinterpret_cast<uintptr_t>(p.O_out);
            fe.vec_ok = (p.cols % 8 == 0) && (al & 15) == 0;
            f.push_back(fe);
        }
        fins.push_back(f);
    }
    return run_direct(R, L, workspace, sched, fins, FIN_WUPD);
}

muon_status muon_step_batched(const muon_param* params, int n, muon_dtype w_dtype, muon_dtype ns_dtype,
                              const muon_hparams* hp, const muon_schedule* sched, void* workspace,
                              size_t ws_bytes, int* d_status, muon_stream_t stream) {
    return step_common(params, n, w_dtype, ns_dtype, hp, sched, workspace, ws_bytes, d_status, stream, false);
}

// MONA-Lite descriptors as the common path's (B in the G_prev slot, no A).
static std::vector<muon_param> lite_as_params(const muon_lite_param* lp, int n) {
    std::vector<muon_param> out(n > 0 ? n : 0);
    for (int i = 0; i < n; ++i) {
        muon_param& p = out[i];
        p.rows = lp[i].rows; p.cols = lp[i].cols;
        p.W = lp[i].W; p.G = lp[i].G; p.G_prev = lp[i].B; p.A = nullptr; p.M = lp[i].M;
        p.gamma = lp[i].gamma; p.O_out = lp[i].O_out;
    }
    return out;
}

muon_status muon_lite_workspace_size(const muon_lite_param* params, int n, muon_dtype ns_dtype, size_t* bytes) {
    if (!params || n < 1) return MUON_ERR_INVALID_ARG;
    std::vector<muon_param> p = lite_as_params(params, n);
    return muon_workspace_size(p.data(), n, ns_dtype, bytes);
}

muon_status muon_lite_step_batched(const muon_lite_param* params, int n, muon_dtype w_dtype, muon_dtype ns_dtype,
                                   const muon_hparams* hp, const muon_schedule* sched, void* workspace,
                                   size_t ws_bytes, int* d_status, muon_stream_t stream) {
    if (!params || n < 1) return MUON_ERR_INVALID_ARG;
    std::vector<muon_param> p = lite_as_params(params, n);
    return step_common(p.data(), n, w_dtype, ns_dtype, hp, sched, workspace, ws_bytes, d_status, stream, true);
}

static muon_status check_batch(const void* X_in, void* X_out, int batch, int rows, int cols,
                               long long batch_stride, muon_dtype dtype) {
    if (!X_in || !X_out || batch < 1 || rows < 1 || cols < 1 || !valid_dtype(dtype))
        return MUON_ERR_INVALID_ARG;
    if (batch_stride < (long long)rows * cols && batch > 1) return MUON_ERR_INVALID_ARG;
    if (batch > 65535) return MUON_ERR_UNSUPPORTED;
    return MUON_OK;
}

muon_status ns_polar_workspace_size(int batch, int rows, int cols, muon_dtype dtype, size_t* bytes) {
    if (!bytes || batch < 1 || rows < 1 || cols < 1 || !valid_dtype(dtype)) return MUON_ERR_INVALID_ARG;
    *bytes = batch_layout(batch, rows, cols, dtype, 2).total;
    return MUON_OK;
}

muon_status gram_polar_workspace_size(int batch, int rows, int cols, muon_dtype dtype, size_t* bytes) {
    if (!bytes || batch < 1 || rows < 1 || cols < 1 || !valid_dtype(dtype)) return MUON_ERR_INVALID_ARG;
    *bytes = batch_layout(batch, rows, cols, dtype, 6).total;
    return MUON_OK;
}

static muon_status polar_common(int route, const void* X_in, void* X_out, int batch, int rows, int cols,
                                long long batch_stride, muon_dtype dtype, const muon_schedule* sched,
                                void* workspace, size_t ws_bytes, int* d_status, muon_stream_t stream) {
    muon_status st = check_batch(X_in, X_out, batch, rows, cols, batch_stride, dtype);
    if (st != MUON_OK) return st;
    st = check_schedule(sched);
    if (st != MUON_OK) return st;
    if (batch == 1) batch_stride = (long long)rows * cols;
    Layout L = batch_layout(batch, rows, cols, dtype, route == 0 ? 2 : 6);
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255) || ws_bytes < L.total)
        return MUON_ERR_WORKSPACE;
    st = check_device();
    if (st != MUON_OK) return st;
    cudaStream_t stream_ = reinterpret_cast<cudaStream_t>(stream);
    int* status = d_status ? d_status : static_cast<int*>(at(workspace, L.status));
    double* sumsq = static_cast<double*>(at(workspace, L.sumsq));
    if (cudaMemsetAsync(sumsq, 0, sizeof(double) * batch, stream_) != cudaSuccess) return MUON_ERR_CUDA;
    const Group& g = L.groups[0];

    PrepParams pp;
    memset(&pp, 0, sizeof(pp));
    pp.in_dt = dtype; pp.x0_dt = dtype; pp.mode = 1; pp.sumsq = sumsq; pp.n = 1;
    PrepEntry& E = pp.e[0];
    E.X = X_in; E.x_stride = batch_stride;
    E.X0 = at(workspace, g.x[0]); E.x0_stride = (long long)g.s * g.ldl; E.ld = g.ldl;
    E.rows = rows; E.cols = cols; E.count = batch; E.transposed = rows > cols;
    E.sumsq_index = 0;
    E.vec_ok = (cols % 8 == 0) && (batch_stride % 8 == 0) && (reinterpret_cast<uintptr_t>(X_in) & 15) == 0;
    st = prep_run(pp, stream_);
    if (st != MUON_OK) return st;

    Runner R;
    R.dt = dtype;
    R.stream = stream_;
    memset(&R.fc, 0, sizeof(R.fc));
    R.fc.out_dt = dtype;
    R.fc.out = X_out;
    R.fc.out_stride = batch_stride;
    R.fc.out_transposed = rows > cols;
    R.fc.out_vec = (cols % 8 == 0) && (batch_stride % 8 == 0) && (reinterpret_cast<uintptr_t>(X_out) & 15) == 0;
    R.fc.d_status = status;
    if (route == 0) return run_direct(R, L, workspace, sched, {}, FIN_OUT);
    return run_gram(R, L, workspace, sched);
}

muon_status ns_polar(const void* X_in, void* X_out, int batch, int rows, int cols, long long batch_stride,
                     muon_dtype dtype, const muon_schedule* sched, void* workspace, size_t ws_bytes,
                     int* d_status, muon_stream_t stream) {
    return polar_common(0, X_in, X_out, batch, rows, cols, batch_stride, dtype, sched, workspace, ws_bytes,
                        d_status, stream);
}

muon_status gram_polar(const void* X_in, void* X_out, int batch, int rows, int cols, long long batch_stride,
                       muon_dtype dtype, const muon_schedule* sched, void* workspace, size_t ws_bytes,
                       int* d_status, muon_stream_t stream) {
    return polar_common(1, X_in, X_out, batch, rows, cols, batch_stride, dtype, sched, workspace, ws_bytes,
                        d_status, stream);
}

}  // extern "C"
