// trace.cu -- optional per-launch CUDA-event tracing (see muon_trace_* in muon.h).
#include <mutex>
#include <vector>

#include "gemm.h"

namespace muon {

namespace {
struct TraceState {
    std::mutex mu;
    bool enabled = false;
    std::vector<cudaEvent_t> pool;   // 2 per record, created on first use
    std::vector<muon_trace_record> recs;
    int open = -1;                   // index of the record whose end event is pending
};
TraceState& state() {
    static TraceState s;
    return s;
}
}  // namespace

void trace_begin(int kind, double work, cudaStream_t stream) {
    TraceState& s = state();
    std::lock_guard<std::mutex> lock(s.mu);
    s.open = -1;
    if (!s.enabled || (int)s.recs.size() >= MUON_TRACE_CAPACITY) return;
    const size_t i = s.recs.size();
    while (s.pool.size() < 2 * (i + 1)) {
        cudaEvent_t e;
        if (cudaEventCreate(&e) != cudaSuccess) return;
        s.pool.push_back(e);
    }
    if (cudaEventRecord(s.pool[2 * i], stream) != cudaSuccess) return;
    muon_trace_record r;
    r.kind = kind;
    r.work = work;
    r.ms = 0.f;
    s.recs.push_back(r);
    s.open = (int)i;
}

void trace_end(cudaStream_t stream) {
    TraceState& s = state();
    std::lock_guard<std::mutex> lock(s.mu);
    if (s.open < 0) return;
    cudaEventRecord(s.pool[2 * s.open + 1], stream);
    s.open = -1;
}

}  // namespace muon

extern "C" {

muon_status muon_trace_enable(int enable) {
    muon::TraceState& s = muon::state();
    std::lock_guard<std::mutex> lock(s.mu);
    s.enabled = enable != 0;
    return MUON_OK;
}

int muon_trace_read(muon_trace_record* out, int max) {
    muon::TraceState& s = muon::state();
    std::lock_guard<std::mutex> lock(s.mu);
    int n = 0;
    for (size_t i = 0; i < s.recs.size(); ++i) {
        if (cudaEventSynchronize(s.pool[2 * i + 1]) != cudaSuccess) return -1;
        float ms = 0.f;
        if (cudaEventElapsedTime(&ms, s.pool[2 * i], s.pool[2 * i + 1]) != cudaSuccess) return -1;
        s.recs[i].ms = ms;
        if (out && n < max) out[n++] = s.recs[i];
    }
    s.recs.clear();
    s.open = -1;
    return n;
}

}  // extern "C"
