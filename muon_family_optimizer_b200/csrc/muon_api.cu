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
    if (!(s->gram_aspect >= 0.f) || !isfinite(s->gram_aspect)) return MUON_ERR_INVALID_ARG;
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

// Smallest short side the tensor-core path takes inside an optimizer step:
// narrower matrices (at most 15 rows in the wide view) are iterated in fp32 on
// CUDA cores, where their 16-bit intermediates would cost more accuracy than
// their negligible work saves.
constexpr int kMinTcSide = 16;

// A batch of same-shape matrices in the wide view (s <= l).
struct Group {
    int s = 0, l = 0;
    std::vector<int> members;        // indices into the caller's parameter array
    int dt = DT_BF16;                // element type of this group's iteration
    int x0_dt = DT_BF16;             // element type of the pre-pass copy of M (x[0])
    int gram = 0;                    // 1: the Gram route, 0: the direct iteration
    // Members with rows <= cols come first (n_wide of them).  When param_tr is
    // set, the pre-pass copies a taller member in its own orientation (l x s,
    // row stride lds) and the first step's products read it transposed.
    int n_wide = 0, param_tr = 0;
    long long ldl = 0, lds = 0;      // padded row strides of s x l and s x s buffers
    long long xs = 0;                // elements per member in the s x l buffers
    size_t x[2] = {0, 0};            // s x l ping-pong
    size_t sq[6] = {0, 0, 0, 0, 0, 0};   // s x s buffers (direct route uses 2, Gram route 6)
    int sumsq0 = 0;                  // first sumsq slot of this group
};

struct Layout {
    size_t status = 0, sumsq = 0, total = 0;
    std::vector<Group> groups;
};

void place_group(Group& g, size_t& off) {
    const long long cnt = (long long)g.members.size();
    const int esz = dt_size(g.dt);
    g.ldl = pad8(g.l);
    g.lds = pad8(g.s);
    g.xs = (long long)g.s * g.ldl;
    if (g.param_tr && g.n_wide < cnt) g.xs = std::max(g.xs, (long long)g.l * g.lds);
    for (int i = 0; i < 2; ++i) {
        g.x[i] = off;
        off = align_up(off + (size_t)cnt * g.xs * esz, kAlign);
    }
    for (int i = 0; i < (g.gram ? 6 : 2); ++i) {
        g.sq[i] = off;
        off = align_up(off + (size_t)cnt * g.s * g.lds * esz, kAlign);
    }
}

// Whether a shape group of an optimizer step runs the Gram route.
bool gram_group(const muon_schedule* sch, int s, int l, int dt) {
    return sch && dt != DT_FP32 && sch->gram_aspect > 0.f && (double)l >= (double)sch->gram_aspect * s;
}

// Parameters grouped by (s, l); a group holds at most kMaxGroupMembers.  The
// schedule (may be NULL: every group direct) selects the Gram route per group.
Layout step_layout(const muon_param* params, int n, int ns_dt, const muon_schedule* sch) {
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
            g.dt = (ns_dt != DT_FP32 && g.s < kMinTcSide) ? DT_FP32 : ns_dt;
            g.gram = gram_group(sch, g.s, g.l, g.dt) ? 1 : 0;
            g.x0_dt = g.dt;
            if (g.gram) {
                // The Gram route iterates in fp16 whatever the 16-bit type ([POLAR]:
                // fp16 is recommended; with bfloat16's 8 bits rounding turns small
                // eigenvalues of R negative and the polynomial h R h multiplies them
                // about 12 times a step): the pre-pass copy of M is bfloat16 (any
                // range), then divided by its norm into fp16 (x[1]).
                g.x0_dt = DT_BF16;
                g.dt = DT_FP16;
            }
            g.members.assign(all.begin() + b, all.begin() + std::min(all.size(), b + kMaxGroupMembers));
            std::stable_partition(g.members.begin(), g.members.end(),
                                  [&](int i) { return params[i].rows <= params[i].cols; });
            g.n_wide = 0;
            for (int i : g.members) g.n_wide += params[i].rows <= params[i].cols;
            // the tensor-core direct groups read a taller member in its own orientation
            g.param_tr = (!g.gram && g.dt != DT_FP32) ? 1 : 0;
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
    int slot = 0;
    for (Group& g : groups) {
        g.sumsq0 = slot;
        slot += (int)g.members.size();
        place_group(g, off);
    }
    L.groups = groups;
    L.total = off;
    return L;
}

Layout batch_layout(int batch, int rows, int cols, int dt, int gram) {
    Layout L;
    Group g;
    g.s = std::min(rows, cols);
    g.l = std::max(rows, cols);
    g.dt = dt;
    g.gram = gram;
    g.members.resize(batch);
    size_t off = 0;
    L.status = off;
    off = align_up(off + 256, kAlign);
    L.sumsq = off;
    off = align_up(off + sizeof(double) * (size_t)batch, kAlign);
    place_group(g, off);
    L.groups.push_back(g);
    L.total = off;
    return L;
}

inline void* at(void* ws, size_t off) { return static_cast<char*>(ws) + off; }

// ---------------------------------------------------------------- launching

struct Runner {
    int dt;                 // element type of the iteration
    bool prenorm = false;   // the wide views already hold X / (||X|| + eps): no norm scale in the products
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
    o.a_tr = 0; o.b_tr = 0;
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
    o.a_tr = 0; o.b_tr = 0;
    o.A = A; o.lda = lda; o.strideA = sA;
    o.B = X; o.ldb = ldx; o.strideB = sX;
    o.epi = e;
    return o;
}

using GroupList = std::vector<const Group*>;
using FinalTables = std::vector<std::vector<FinalEntry>>;   // per group of a GroupList: its W-update rows

// The last product of the iteration, one op per group (ops[i] belongs to
// group i): FIN_OUT writes the caller's output; FIN_WUPD updates W through
// each group's rows of the final table.  A launch carries at most
// kMaxProblems ops and kMaxFinal table rows.
muon_status run_final(Runner& R, const std::vector<GemmOp>& ops, const FinalTables& fins, int final_kind) {
    std::vector<GemmOp> batch;
    std::vector<FinalEntry> fin;
    for (size_t i = 0; i < ops.size(); ++i) {
        GemmOp o = ops[i];
        const int rows_needed = final_kind == FIN_WUPD ? o.count : 0;
        if (!batch.empty() && (batch.size() == (size_t)kMaxProblems || (int)fin.size() + rows_needed > kMaxFinal)) {
            muon_status st = R.run(batch, fin);
            if (st != MUON_OK) return st;
            batch.clear();
            fin.clear();
        }
        o.epi.fin = final_kind;
        if (rows_needed) {
            o.epi.fin_base = (int)fin.size();
            fin.insert(fin.end(), fins[i].begin(), fins[i].end());
        }
        batch.push_back(o);
    }
    return R.run(batch, fin);
}

// The members of a group as the first products see them: the wide members
// (rows <= cols), then -- read transposed when the group copies them in their
// own orientation -- the taller ones.  {first member, count, transposed}.
struct Part {
    int first, count, tr;
};

std::vector<Part> first_parts(const Group& g) {
    const int cnt = (int)g.members.size();
    if (!g.param_tr || g.n_wide == cnt) return {{0, cnt, 0}};
    if (g.n_wide == 0) return {{0, cnt, 1}};
    return {{0, g.n_wide, 0}, {g.n_wide, cnt - g.n_wide, 1}};
}

// The direct quintic iteration on the groups `gs` (all of R.dt), starting
// from the unnormalised copies in x[0] (norms in sumsq).  The last step's
// epilogue is `final_kind` (FIN_OUT or FIN_WUPD with the groups' tables).
muon_status run_direct(Runner& R, const GroupList& gs, void* ws, const double* sumsq, const muon_schedule* sch,
                       const FinalTables& fins, int final_kind) {
    if (gs.empty()) return MUON_OK;
    const float f = sch->scale_f;
    const int esz = dt_size(R.dt);
    int cur = 0;
    for (int k = 0; k < sch->n_steps; ++k) {
        const muon_ns_coeff c = sch->coeffs[k];
        const bool first = k == 0;
        const float pre = first ? 1.f / f : (is_restart(sch, k) ? 1.f / f : 1.f);
        const bool last = k == sch->n_steps - 1;
        // member ranges of each product: the first step reads transposed copies
        // of the taller members separately, later steps the wide views only
        auto parts = [&](const Group& g) {
            return first ? first_parts(g) : std::vector<Part>{{0, (int)g.members.size(), 0}};
        };
        // A = X X^T (scaled by pre^2, and by 1/(|M|+eps)^2 at the first step)
        std::vector<GemmOp> ops;
        for (const Group* gp : gs) {
            const Group& g = *gp;
            const long long ss = (long long)g.s * g.lds;
            for (const Part& q : parts(g)) {
                Epilogue e = epi_store(static_cast<char*>(at(ws, g.sq[0])) + (size_t)q.first * ss * esz, g.lds, ss);
                e.sc_mul = pre * pre;
                if (first && !R.prenorm) { e.sumsq = sumsq + g.sumsq0 + q.first; e.eps = sch->eps; e.sc_pow = 2; }
                const void* X = static_cast<char*>(at(ws, g.x[cur])) + (size_t)q.first * g.xs * esz;
                const long long ldx = q.tr ? g.lds : g.ldl;
                GemmOp o = sym_op(q.count, g.s, g.l, X, ldx, g.xs, X, ldx, g.xs, e);
                o.a_tr = o.b_tr = q.tr;
                ops.push_back(o);
            }
        }
        muon_status st = R.run(ops, {});
        if (st != MUON_OK) return st;
        // B' = a I + b A + c A A   (the a X term of the step rides on the diagonal)
        ops.clear();
        for (const Group* gp : gs) {
            const Group& g = *gp;
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
        ops.clear();
        FinalTables op_fins;
        for (size_t gi = 0; gi < gs.size(); ++gi) {
            const Group& g = *gs[gi];
            const long long ss = (long long)g.s * g.lds;
            for (const Part& q : parts(g)) {
                Epilogue e = epi_store(static_cast<char*>(at(ws, g.x[cur ^ 1])) + (size_t)q.first * g.xs * esz,
                                       g.ldl, g.xs);
                e.sc_mul = pre;
                if (first && !R.prenorm) { e.sumsq = sumsq + g.sumsq0 + q.first; e.eps = sch->eps; e.sc_pow = 1; }
                if (last) e.check = sumsq + g.sumsq0 + q.first;
                const void* B = static_cast<char*>(at(ws, g.sq[1])) + (size_t)q.first * ss * esz;
                const void* X = static_cast<char*>(at(ws, g.x[cur])) + (size_t)q.first * g.xs * esz;
                GemmOp o = upd_op(q.count, g.s, g.l, B, g.lds, ss, X, q.tr ? g.lds : g.ldl, g.xs, e);
                o.b_tr = q.tr;
                ops.push_back(o);
                if (last && final_kind == FIN_WUPD)
                    op_fins.emplace_back(fins[gi].begin() + q.first, fins[gi].begin() + q.first + q.count);
                else
                    op_fins.emplace_back();
            }
        }
        st = last ? run_final(R, ops, op_fins, final_kind) : R.run(ops, {});
        if (st != MUON_OK) return st;
        cur ^= 1;
    }
    return MUON_OK;
}

// The Gram route (see include/muon.h) on the groups `gs` (all of R.dt, each
// with six s x s buffers), starting from the wide views in x[xb0] (normalised
// already when R.prenorm);
// the last product's epilogue is `final_kind` as for run_direct.  Every launch
// carries the same product for all groups.
muon_status run_gram(Runner& R, const GroupList& gs, void* ws, const double* sumsq, const muon_schedule* sch,
                     const FinalTables& fins, int final_kind, int xb0 = 0) {
    if (gs.empty()) return MUON_OK;
    const float f = sch->scale_f;
    // buffer roles: indices into each group's sq[]
    int iR = 0, iRn = 1, iH = 2, iQ = 3, iQn = 4, iT = 5;
    int xb = xb0;               // current Xb buffer
    bool xb_raw = true;         // Xb still holds the unnormalised input (scale pending)
    bool q_identity = true;
    auto sq = [&](const Group& g, int i) { return at(ws, g.sq[i]); };
    auto xbuf = [&](const Group& g, int i) { return at(ws, g.x[i]); };
    auto strides = [](const Group& g, long long& sx, long long& ss) {
        sx = g.xs;
        ss = (long long)g.s * g.lds;
    };
    // one symmetric s x s product per group: D = A B^T (A, B, D given as buffer roles)
    auto sym_all = [&](int ia, int ib, int id, bool with_band, const muon_ns_coeff* poly) -> muon_status {
        std::vector<GemmOp> ops;
        for (const Group* gp : gs) {
            const Group& g = *gp;
            long long sx, ss;
            strides(g, sx, ss);
            Epilogue e = epi_store(sq(g, id), g.lds, ss);
            if (poly) {   // h = a I + b R + c R R
                e.alpha = poly->c; e.beta = poly->b; e.diag = poly->a;
                e.Cin = sq(g, ia); e.ldc = g.lds; e.strideC = ss;
            }
            ops.push_back(sym_op((int)g.members.size(), g.s, g.s, sq(g, ia), g.lds, ss, sq(g, ib), g.lds, ss, e, 1, 1,
                                 with_band ? 1 : 0));
        }
        return R.run(ops, {});
    };
    // R = Xb Xb^T (normalised when Xb is still the raw input)
    auto gram_all = [&](float sc_mul, bool normalise) -> muon_status {
        std::vector<GemmOp> ops;
        for (const Group* gp : gs) {
            const Group& g = *gp;
            long long sx, ss;
            strides(g, sx, ss);
            Epilogue e = epi_store(sq(g, iR), g.lds, ss);
            e.sc_mul = sc_mul;
            if (normalise && !R.prenorm) { e.sumsq = sumsq + g.sumsq0; e.eps = sch->eps; e.sc_pow = 2; }
            ops.push_back(sym_op((int)g.members.size(), g.s, g.l, xbuf(g, xb), g.ldl, sx, xbuf(g, xb), g.ldl, sx, e));
        }
        return R.run(ops, {});
    };
    // Xb' = scale Q Xb (the pending normalisation folded in): into the other
    // Xb buffer, or (final) to the caller / W
    auto apply_q = [&](bool final) -> muon_status {
        std::vector<GemmOp> ops;
        for (const Group* gp : gs) {
            const Group& g = *gp;
            long long sx, ss;
            strides(g, sx, ss);
            if (q_identity) {
                muon_status st = fill_identity(sq(g, iQ), R.dt, (int)g.members.size(), g.s, g.lds, ss, R.stream);
                if (st != MUON_OK) return st;
            }
            Epilogue e = final ? epi_store(nullptr, 0, 0) : epi_store(xbuf(g, xb ^ 1), g.ldl, sx);
            e.sc_mul = final ? 1.f : 1.f / f;
            if (xb_raw) {
                e.sc_mul *= 1.f / f;
                if (!R.prenorm) { e.sumsq = sumsq + g.sumsq0; e.eps = sch->eps; e.sc_pow = 1; }
            }
            if (final) e.check = sumsq + g.sumsq0;
            ops.push_back(upd_op((int)g.members.size(), g.s, g.l, sq(g, iQ), g.lds, ss, xbuf(g, xb), g.ldl, sx, e));
        }
        return final ? run_final(R, ops, fins, final_kind) : R.run(ops, {});
    };

    // R = Xb Xb^T / ((|X|+eps) f)^2
    muon_status st = gram_all(1.f / (f * f), true);
    if (st != MUON_OK) return st;
    for (int k = 0; k < sch->n_steps; ++k) {
        const muon_ns_coeff c = sch->coeffs[k];
        if (is_restart(sch, k)) {
            // Xb <- Q Xb / f;  R <- Xb Xb^T;  Q <- I
            st = apply_q(false);
            if (st != MUON_OK) return st;
            xb ^= 1;
            xb_raw = false;
            q_identity = true;
            st = gram_all(1.f, false);
            if (st != MUON_OK) return st;
        }
        // h = a I + b R + c R R
        st = sym_all(iR, iR, iH, true, &c);
        if (st != MUON_OK) return st;
        const bool need_r = k + 1 < sch->n_steps && !is_restart(sch, k + 1);
        // Q <- h Q  and  T = h R  (one launch)
        std::vector<GemmOp> ops;
        for (const Group* gp : gs) {
            const Group& g = *gp;
            long long sx, ss;
            strides(g, sx, ss);
            const int cnt = (int)g.members.size();
            if (!q_identity)
                ops.push_back(sym_op(cnt, g.s, g.s, sq(g, iH), g.lds, ss, sq(g, iQ), g.lds, ss,
                                     epi_store(sq(g, iQn), g.lds, ss), 1, 1, 1));
            if (need_r)
                ops.push_back(sym_op(cnt, g.s, g.s, sq(g, iH), g.lds, ss, sq(g, iR), g.lds, ss,
                                     epi_store(sq(g, iT), g.lds, ss), 1, 1));
        }
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
            st = sym_all(iT, h_buf, iRn, false, nullptr);
            if (st != MUON_OK) return st;
            std::swap(iR, iRn);
        }
    }
    // X = Q Xb  -> the caller's output or W
    return apply_q(true);
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

muon_status muon_workspace_size(const muon_param* params, int n, muon_dtype ns_dtype, const muon_schedule* sched,
                                size_t* bytes) {
    if (!bytes || !valid_dtype(ns_dtype)) return MUON_ERR_INVALID_ARG;
    muon_status st = check_params(params, n);
    if (st != MUON_OK) return st;
    if (sched) {
        st = check_schedule(sched);
        if (st != MUON_OK) return st;
    }
    *bytes = step_layout(params, n, ns_dtype, sched).total;
    return MUON_OK;
}

// Optional vector-valued parameters of a whole-model step (AdamW items of the
// pre-pass launch).
struct VecItems {
    const muon_vec_param* vecs = nullptr;
    int n = 0;
    AdamWCoeffs c = {};
};

// lite: MONA-Lite state (G_prev holds the bfloat16 buffer B, A is unused).
static muon_status step_common(const muon_param* params, int n, muon_dtype w_dtype, muon_dtype ns_dtype,
                               const muon_hparams* hp, const muon_schedule* sched, void* workspace,
                               size_t ws_bytes, int* d_status, muon_stream_t stream, bool lite,
                               const VecItems& vec = VecItems()) {
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
    Layout L = step_layout(params, n, ns_dtype, sched);
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255) || ws_bytes < L.total)
        return MUON_ERR_WORKSPACE;
    st = check_device();
    if (st != MUON_OK) return st;
    cudaStream_t stream_ = reinterpret_cast<cudaStream_t>(stream);
    int* status = d_status ? d_status : static_cast<int*>(at(workspace, L.status));
    double* sumsq = static_cast<double*>(at(workspace, L.sumsq));
    if (cudaMemsetAsync(sumsq, 0, sizeof(double) * n, stream_) != cudaSuccess) return MUON_ERR_CUDA;

    // 1. fused MONA pre-pass + norms + wide-view copies: one launch per
    //    element type of the copies (the iteration's, and fp32 for narrow groups)
    const size_t in_sz = dt_size(w_dtype);
    int x0_types[3], n_x0 = 0;
    x0_types[n_x0++] = (int)ns_dtype;
    for (const Group& g : L.groups) {
        bool seen = false;
        for (int t = 0; t < n_x0; ++t) seen |= x0_types[t] == g.x0_dt;
        if (!seen) x0_types[n_x0++] = g.x0_dt;
    }
    for (int t = 0; t < n_x0; ++t) {
        const int x0_dt = x0_types[t];
        PrepParams pp;
        memset(&pp, 0, sizeof(pp));
        pp.in_dt = w_dtype; pp.x0_dt = x0_dt; pp.mode = lite ? 2 : 0;
        pp.beta_a = hp->beta_a; pp.alpha = hp->alpha; pp.mu = hp->mu;
        pp.sumsq = sumsq;
        for (const Group& g : L.groups) {
            if (g.x0_dt != x0_dt) continue;
            for (size_t j = 0; j < g.members.size(); ++j) {
                const muon_param& p = params[g.members[j]];
                PrepEntry& E = pp.e[pp.n++];
                E.G = p.G; E.Gp = p.G_prev; E.A = p.A; E.M = p.M;
                E.rows = p.rows; E.cols = p.cols; E.count = 1;
                // wide copy (a taller member transposed), or the member's own orientation
                const bool own = g.param_tr && p.rows > p.cols;
                E.transposed = p.rows > p.cols && !own;
                E.X0 = static_cast<char*>(at(workspace, g.x[0])) + j * (size_t)g.xs * dt_size(g.x0_dt);
                E.ld = own ? g.lds : g.ldl;
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
        if (t == 0) {
            // the vector-valued parameters' AdamW as further items of the same launch
            pp.adam = vec.c;
            pp.d_status = status;
            for (int i = 0; i < vec.n; ++i) {
                const muon_vec_param& q = vec.vecs[i];
                PrepEntry& E = pp.e[pp.n++];
                E.kind = 1;
                E.nel = q.n;
                E.G = q.G; E.Gp = q.W; E.A = q.m; E.M = q.v;
                E.rows = E.cols = 1; E.ld = 1; E.count = 1;
                const uintptr_t al = reinterpret_cast<uintptr_t>(q.W) | reinterpret_cast<uintptr_t>(q.G) |
                                     reinterpret_cast<uintptr_t>(q.m) | reinterpret_cast<uintptr_t>(q.v);
                E.vec_ok = (al & 15) == 0 && in_sz >= 2;
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
    }

    // 1b. Gram-route groups: x[1] = x[0] / (||M|| + eps) in fp16 (norms complete)
    {
        PrepParams pp;
        memset(&pp, 0, sizeof(pp));
        pp.in_dt = DT_BF16; pp.x0_dt = DT_FP16; pp.mode = 1; pp.prescale = 1; pp.eps = sched->eps;
        pp.sumsq = sumsq;
        for (const Group& g : L.groups) {
            if (!g.gram) continue;
            PrepEntry& E = pp.e[pp.n++];
            E.X = at(workspace, g.x[0]); E.x_stride = g.xs;
            E.X0 = at(workspace, g.x[1]); E.x0_stride = g.xs; E.ld = g.ldl;
            E.rows = g.s; E.cols = (int)g.ldl; E.count = (int)g.members.size(); E.transposed = 0;
            E.sumsq_index = g.sumsq0;
            E.vec_ok = 1;             // rows of ldl elements (a multiple of 8), 1024-byte aligned buffers
            if (pp.n == kMaxPrep) {
                st = prep_run(pp, stream_);
                if (st != MUON_OK) return st;
                pp.n = 0;
            }
        }
        if (pp.n > 0) {
            st = prep_run(pp, stream_);
            if (st != MUON_OK) return st;
        }
    }

    // 2-3. iteration with the weight update fused into its last step: the
    //      direct groups of the iteration's type, the Gram-route groups, and
    //      the narrow groups in fp32
    Runner R;
    R.stream = stream_;
    memset(&R.fc, 0, sizeof(R.fc));
    R.fc.w_dt = w_dtype;
    R.fc.eta = hp->eta;
    R.fc.lambda = hp->lambda;
    R.fc.d_status = status;
    GroupList direct16, gram16, direct32;
    FinalTables fin_d16, fin_g16, fin_d32;
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
        if (g.gram) { gram16.push_back(&g); fin_g16.push_back(f); }
        else if (g.dt != (int)ns_dtype) { direct32.push_back(&g); fin_d32.push_back(f); }
        else { direct16.push_back(&g); fin_d16.push_back(f); }
    }
    R.dt = ns_dtype;
    st = run_direct(R, direct16, workspace, sumsq, sched, fin_d16, FIN_WUPD);
    if (st != MUON_OK) return st;
    R.dt = DT_FP16;
    R.prenorm = true;          // the Gram groups start from their normalised fp16 copies in x[1]
    st = run_gram(R, gram16, workspace, sumsq, sched, fin_g16, FIN_WUPD, 1);
    if (st != MUON_OK) return st;
    R.prenorm = false;
    R.dt = DT_FP32;
    return run_direct(R, direct32, workspace, sumsq, sched, fin_d32, FIN_WUPD);
}

muon_status muon_step_batched(const muon_param* params, int n, muon_dtype w_dtype, muon_dtype ns_dtype,
                              const muon_hparams* hp, const muon_schedule* sched, void* workspace,
                              size_t ws_bytes, int* d_status, muon_stream_t stream) {
    return step_common(params, n, w_dtype, ns_dtype, hp, sched, workspace, ws_bytes, d_status, stream, false);
}

muon_status muon_model_step(const muon_param* params, int n, const muon_vec_param* vecs, int nvec,
                            muon_dtype w_dtype, muon_dtype ns_dtype, const muon_hparams* hp,
                            const muon_adamw_hparams* adamw, int step, const muon_schedule* sched,
                            void* workspace, size_t ws_bytes, int* d_status, muon_stream_t stream) {
    if (nvec < 0) return MUON_ERR_INVALID_ARG;
    VecItems v;
    if (nvec > 0) {
        muon_status st = adamw_check(vecs, nvec, adamw, step);
        if (st != MUON_OK) return st;
        v.vecs = vecs;
        v.n = nvec;
        v.c = adamw_coeffs(adamw, step);
    }
    return step_common(params, n, w_dtype, ns_dtype, hp, sched, workspace, ws_bytes, d_status, stream, false, v);
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

muon_status muon_lite_workspace_size(const muon_lite_param* params, int n, muon_dtype ns_dtype,
                                     const muon_schedule* sched, size_t* bytes) {
    if (!params || n < 1) return MUON_ERR_INVALID_ARG;
    std::vector<muon_param> p = lite_as_params(params, n);
    return muon_workspace_size(p.data(), n, ns_dtype, sched, bytes);
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
    *bytes = batch_layout(batch, rows, cols, dtype, 0).total;
    return MUON_OK;
}

muon_status gram_polar_workspace_size(int batch, int rows, int cols, muon_dtype dtype, size_t* bytes) {
    if (!bytes || batch < 1 || rows < 1 || cols < 1 || !valid_dtype(dtype)) return MUON_ERR_INVALID_ARG;
    *bytes = batch_layout(batch, rows, cols, dtype, 1).total;
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
    // A bfloat16 input is iterated in fp16 ([POLAR]: fp16 is the recommended
    // type; its three extra significand bits carry the small singular
    // directions at condition numbers near 1e3): the copy of the input is
    // divided by its norm first, which puts it in fp16's range.  Storage in and
    // out stays bfloat16; both types take the same workspace.
    const int it_dt = (int)dtype == DT_BF16 ? (int)DT_FP16 : (int)dtype;
    Layout L = batch_layout(batch, rows, cols, it_dt, route);
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
    pp.in_dt = dtype; pp.x0_dt = it_dt; pp.mode = 1; pp.sumsq = sumsq; pp.n = 1; pp.eps = sched->eps;
    PrepEntry& E = pp.e[0];
    E.X = X_in; E.x_stride = batch_stride;
    E.X0 = at(workspace, g.x[0]); E.x0_stride = g.xs; E.ld = g.ldl;
    E.rows = rows; E.cols = cols; E.count = batch; E.transposed = rows > cols;
    E.sumsq_index = 0;
    E.vec_ok = (cols % 8 == 0) && (batch_stride % 8 == 0) && (reinterpret_cast<uintptr_t>(X_in) & 15) == 0;
    const bool prenorm = it_dt != (int)dtype;
    if (prenorm) {
        pp.mode = 3;                  // norms first
        st = prep_run(pp, stream_);
        if (st != MUON_OK) return st;
        pp.mode = 1;
        pp.prescale = 1;              // then the normalised copy
    }
    st = prep_run(pp, stream_);
    if (st != MUON_OK) return st;

    Runner R;
    R.dt = it_dt;
    R.prenorm = prenorm;
    R.stream = stream_;
    memset(&R.fc, 0, sizeof(R.fc));
    R.fc.out_dt = dtype;
    R.fc.out = X_out;
    R.fc.out_stride = batch_stride;
    R.fc.out_transposed = rows > cols;
    R.fc.out_vec = (cols % 8 == 0) && (batch_stride % 8 == 0) && (reinterpret_cast<uintptr_t>(X_out) & 15) == 0;
    R.fc.d_status = status;
    const GroupList gs = {&L.groups[0]};
    const FinalTables none(1);
    if (route == 0) return run_direct(R, gs, workspace, sumsq, sched, none, FIN_OUT);
    return run_gram(R, gs, workspace, sumsq, sched, none, FIN_OUT);
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
