// Kernel timing by class, and the latency of the sweep's dependent chain.
//
// Diagnostics for benchmarks (the pages have no counterpart): when enabled, the
// library records a pair of CUDA events around each launch of the timed kernel
// classes, on the stream that launch uses, and sums their elapsed times on request.
// Nothing is recorded while a stream is being captured into a CUDA graph.
#include <mutex>
#include <vector>

#include "common.cuh"

namespace gptq {

namespace {
struct ProfRecord {
    int kind, lane;
    cudaEvent_t a, b;
};
std::mutex g_prof_mu;
bool g_prof_on = false;
std::vector<ProfRecord> g_prof;          // records of this profiling window
std::vector<cudaEvent_t> g_prof_pool;    // events to reuse
size_t g_prof_used = 0;
std::vector<cudaStream_t> g_prof_lanes;  // streams of this window, in order of first use

int lane_of(cudaStream_t st) {
    for (size_t i = 0; i < g_prof_lanes.size(); ++i)
        if (g_prof_lanes[i] == st) return (int)i;
    g_prof_lanes.push_back(st);
    return (int)g_prof_lanes.size() - 1;
}

cudaEvent_t pool_event() {
    if (g_prof_used < g_prof_pool.size()) return g_prof_pool[g_prof_used++];
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) {
        cudaGetLastError();
        return nullptr;
    }
    g_prof_pool.push_back(e);
    ++g_prof_used;
    return e;
}
}  // namespace

int prof_begin(int kind, cudaStream_t st) {
    std::lock_guard<std::mutex> lock(g_prof_mu);
    if (!g_prof_on || kind < 0 || kind >= GPTQ_PROF_KINDS) return -1;
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(st, &cs) != cudaSuccess || cs != cudaStreamCaptureStatusNone) {
        cudaGetLastError();
        return -1;
    }
    cudaEvent_t a = pool_event(), b = pool_event();
    if (!a || !b || cudaEventRecord(a, st) != cudaSuccess) {
        cudaGetLastError();
        return -1;
    }
    g_prof.push_back({kind, lane_of(st), a, b});
    return (int)g_prof.size() - 1;
}

void prof_end(int rec, cudaStream_t st) {
    if (rec < 0) return;
    std::lock_guard<std::mutex> lock(g_prof_mu);
    if (rec >= (int)g_prof.size()) return;
    if (cudaEventRecord(g_prof[rec].b, st) != cudaSuccess) {
        cudaGetLastError();
        g_prof[rec].kind = -1;
    }
}

// The sweep's dependent chain for one coordinate per step: the previous step's error
// reaches this coordinate (FMA), which is scaled, rounded to the grid and clamped, and
// its normalised error formed (FMA, multiply); one thread, `steps` steps, timed with
// the SM clock and the global timer.
__global__ void k_chain_latency(float *out, int steps, float u, float rs, float s, float rp,
                                float cmin, float cmax, float w0) {
    float w = w0, e = 0.f;
    const long long c0 = clock64();
    unsigned long long g0;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(g0));
#pragma unroll 8
    for (int i = 0; i < steps; ++i) {
        w = fmaf(-e, u, w);
        const float cf = fminf(fmaxf(rintf(w * rs), cmin), cmax);
        e = fmaf(-s, cf, w) * rp;
    }
    const long long c1 = clock64();
    unsigned long long g1;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(g1));
    out[0] = (float)(c1 - c0) / steps;
    out[1] = (float)(g1 - g0) / steps;
    out[2] = w + e;
}

}  // namespace gptq

using namespace gptq;

extern "C" {

gptq_status gptq_profile_enable(int on) {
    std::lock_guard<std::mutex> lock(g_prof_mu);
    g_prof_on = on != 0;
    if (g_prof_on) {          // a new window: earlier records are dropped
        g_prof.clear();
        g_prof_lanes.clear();
        g_prof_used = 0;
    }
    return GPTQ_OK;
}

gptq_status gptq_profile_read(int kind, double *ms, int *launches) {
    if (kind < 0 || kind >= GPTQ_PROF_KINDS || !ms || !launches) return GPTQ_ERR_ARG;
    std::lock_guard<std::mutex> lock(g_prof_mu);
    double total = 0.0;
    int count = 0;
    for (const ProfRecord &r : g_prof) {
        if (r.kind != kind) continue;
        float t = 0.f;
        if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&t, r.a, r.b) != cudaSuccess) {
            cudaGetLastError();
            return GPTQ_ERR_CUDA;
        }
        total += t;
        ++count;
    }
    *ms = total;
    *launches = count;
    return GPTQ_OK;
}

gptq_status gptq_profile_timeline(int max, int *kind, int *lane, double *begin_ms, double *end_ms,
                                  int *count) {
    if (max < 0 || !kind || !lane || !begin_ms || !end_ms || !count) return GPTQ_ERR_ARG;
    std::lock_guard<std::mutex> lock(g_prof_mu);
    *count = (int)g_prof.size();
    for (int i = 0; i < (int)g_prof.size() && i < max; ++i) {
        const ProfRecord &r = g_prof[i];
        float t0 = 0.f, t1 = 0.f;
        if (r.kind >= 0 && (cudaEventSynchronize(r.b) != cudaSuccess ||
            cudaEventElapsedTime(&t0, g_prof[0].a, r.a) != cudaSuccess ||
            cudaEventElapsedTime(&t1, g_prof[0].a, r.b) != cudaSuccess)) {
            cudaGetLastError();
            return GPTQ_ERR_CUDA;
        }
        kind[i] = r.kind;
        lane[i] = r.lane;
        begin_ms[i] = t0;
        end_ms[i] = t1;
    }
    return GPTQ_OK;
}

gptq_status gptq_chain_latency(float *out, int steps, void *stream) {
    if (!out || steps < 8 || steps % 8 != 0) return GPTQ_ERR_ARG;
    // values in the ranges a 3-bit sweep sees (the timing does not depend on them)
    k_chain_latency<<<1, 1, 0, static_cast<cudaStream_t>(stream)>>>(
        out, steps, 1e-3f, 1.f / 0.0123f, 0.0123f, 37.f, -4.f, 3.f, 0.02f);
    return launch_status();
}

}  // extern "C"
