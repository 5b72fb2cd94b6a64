// C ABI of the library: argument validation, plan choice, workspace accounting and
// error mapping. Every numerical step runs in the plans' CUDA kernels.
#include <stdio.h>
#include <string.h>

#include <mutex>
#include <string>
#include <vector>

#include "gla_common.cuh"
#include "gla_plans.h"

using namespace gla;

// ------------------------------------------------------------ launch accounting
namespace {
thread_local char g_last_detail[256] = "no error";
struct ProfRecord {
    std::string name;
    cudaEvent_t start, stop;
};
std::mutex g_prof_mu;
bool g_prof_on = false;
unsigned long long g_launches = 0;
std::vector<ProfRecord> g_prof_open;  // recorded, not yet read
std::vector<cudaEvent_t> g_event_pool;

cudaEvent_t take_event() {
    if (!g_event_pool.empty()) {
        cudaEvent_t e = g_event_pool.back();
        g_event_pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
}
}  // namespace

namespace gla {
gla_status record_cuda(cudaError_t e, const char* where) {
    if (e == cudaSuccess) return GLA_OK;
    snprintf(g_last_detail, sizeof(g_last_detail), "%s: %s (%s)", where, cudaGetErrorName(e), cudaGetErrorString(e));
    return GLA_ERR_CUDA;
}
void prof_begin(const char* name, cudaStream_t st) {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    ++g_launches;
    if (!g_prof_on) return;
    ProfRecord r{name, take_event(), take_event()};
    cudaEventRecord(r.start, st);
    g_prof_open.push_back(r);
}
bool prof_enabled() {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    return g_prof_on;
}
void prof_end(cudaStream_t st) {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    if (!g_prof_on || g_prof_open.empty()) return;
    cudaEventRecord(g_prof_open.back().stop, st);
}
}  // namespace gla

namespace {

bool aligned16(const void* p) { return p == nullptr || (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool dim_ok(int d) { return d == 64 || d == 128 || d == 256; }

// Validates the problem; fills Dims and the resolved plan.
gla_status check_problem(const gla_problem* p, Dims* P, int* plan) {
    if (!p) return GLA_ERR_INVALID_ARG;
    if (p->B < 0 || p->H < 0 || p->L < 0) return GLA_ERR_INVALID_ARG;
    if (p->io != GLA_F32 && p->io != GLA_BF16) return GLA_ERR_INVALID_ARG;
    if (p->gate != GLA_GATE_NONE && p->gate != GLA_GATE_PER_KEY && p->gate != GLA_GATE_PER_HEAD)
        return GLA_ERR_INVALID_ARG;
    if (p->plan < GLA_PLAN_AUTO || p->plan > GLA_PLAN_TC) return GLA_ERR_INVALID_ARG;
    if (p->chunk < 16 || p->chunk > 1024 || p->chunk % 16 != 0) return GLA_ERR_UNSUPPORTED;
    if (!dim_ok(p->Dk) || !dim_ok(p->Dv)) return GLA_ERR_UNSUPPORTED;
    if ((long long)p->B * p->H > 65535LL) return GLA_ERR_UNSUPPORTED;  // grid z extent
    P->B = p->B; P->H = p->H; P->L = p->L; P->Dk = p->Dk; P->Dv = p->Dv; P->C = p->chunk;
    P->N = cdiv(p->L, p->chunk);
    P->gate = p->gate;
    P->scale = p->scale;
    *plan = p->plan;
    return GLA_OK;
}

// The tensor-core plan runs bf16 I/O with chunks that are whole 64-token tiles; its
// backward holds the Dk x Dv state gradient in tensor memory (Dk <= 128).
bool tc_ok(const gla_problem* p, const Dims& P, bool bwd) {
    return p->io == GLA_BF16 && (bwd ? tc::bwd_supports(P) : tc::supports(P));
}

// Plan of the forward / backward: AUTO prefers the tensor-core plan where it applies.
gla_status resolve(const gla_problem* p, const Dims& P, bool bwd, int* plan) {
    int pl = p->plan;
    if (pl == GLA_PLAN_AUTO) pl = tc_ok(p, P, bwd) ? GLA_PLAN_TC : GLA_PLAN_SIMT;
    if (pl == GLA_PLAN_TC && !tc_ok(p, P, bwd)) return GLA_ERR_UNSUPPORTED;
    *plan = pl;
    return GLA_OK;
}

gla_status map_cuda(cudaError_t e, const char* where = "launch") { return gla::record_cuda(e, where); }

size_t ws_bytes(const Dims& P, int plan, bool bwd) {
    if (plan == GLA_PLAN_TC) return bwd ? tc::bwd_workspace_bytes(P) : tc::fwd_workspace_bytes(P);
    return simt::workspace_bytes(P, bwd);
}

}  // namespace

extern "C" {

size_t gla_workspace_bytes(const gla_problem* p, int for_backward) {
    Dims P;
    int plan;
    if (check_problem(p, &P, &plan) != GLA_OK) return 0;
    if (resolve(p, P, for_backward != 0, &plan) != GLA_OK) return 0;
    return ws_bytes(P, plan, for_backward != 0);
}

size_t gla_saved_states_bytes(const gla_problem* p) {
    Dims P;
    int plan;
    if (check_problem(p, &P, &plan) != GLA_OK) return 0;
    if (resolve(p, P, true, &plan) != GLA_OK || plan != GLA_PLAN_TC) return 0;
    int nseg = 1, tps = 0;
    tc::bwd_plan_info(P, &nseg, &tps);
    return nseg > 1 ? 4 * (size_t)P.B * P.H * nseg * P.Dk * P.Dv : 0;
}

gla_status gla_fwd(const gla_problem* p, const void* q, const void* k, const void* v, const float* g,
                   const float* igate, const float* h0, void* o, float* hT, void* ws, size_t ws_bytes_given,
                   void* stream) {
    return gla_fwd_save(p, q, k, v, g, igate, h0, o, hT, nullptr, ws, ws_bytes_given, stream);
}

gla_status gla_fwd_save(const gla_problem* p, const void* q, const void* k, const void* v, const float* g,
                        const float* igate, const float* h0, void* o, float* hT, float* saved, void* ws,
                        size_t ws_bytes_given, void* stream) {
    Dims P;
    int plan;
    gla_status s = check_problem(p, &P, &plan);
    if (s != GLA_OK) return s;
    s = resolve(p, P, false, &plan);
    if (s != GLA_OK) return s;
    const bool empty = (size_t)P.B * P.H * P.L == 0;
    if (!empty && (!q || !k || !v || !o)) return GLA_ERR_INVALID_ARG;
    if ((p->gate == GLA_GATE_NONE) != (g == nullptr) && !empty) return GLA_ERR_INVALID_ARG;
    if (!ws) return GLA_ERR_INVALID_ARG;
    const void* ptrs[] = {q, k, v, g, igate, h0, o, hT, saved, ws};
    for (const void* x : ptrs)
        if (!aligned16(x)) return GLA_ERR_INVALID_ARG;
    if (ws_bytes_given < ws_bytes(P, plan, false)) return GLA_ERR_WORKSPACE;
    // saved states are only needed (and written) when the backward runs on tensor cores in
    // more than one segment; they are written by the tensor-core forward
    if (saved && gla_saved_states_bytes(p) == 0) saved = nullptr;
    if (saved && plan != GLA_PLAN_TC) return GLA_ERR_UNSUPPORTED;
    cudaStream_t st = (cudaStream_t)stream;
    cudaError_t e = cudaMemsetAsync(ws, 0, kStatusBytes, st);
    if (e != cudaSuccess) return map_cuda(e, "status word reset");
    if ((size_t)P.B * P.H == 0) return GLA_OK;
    if (plan == GLA_PLAN_TC && P.L > 0)
        e = tc::fwd(P, q, k, v, g, igate, h0, o, hT, saved, ws, st);
    else
        e = simt::fwd(P, p->io, q, k, v, g, igate, h0, o, hT, ws, st);
    return map_cuda(e);
}

gla_status gla_bwd(const gla_problem* p, const void* q, const void* k, const void* v, const float* g,
                   const float* igate, const float* h0, const void* dO, const float* dhT, void* dq, void* dk,
                   void* dv, float* dg, float* di, float* dh0, void* ws, size_t ws_bytes_given, void* stream) {
    return gla_bwd_saved(p, q, k, v, g, igate, h0, dO, dhT, nullptr, dq, dk, dv, dg, di, dh0, ws, ws_bytes_given,
                         stream);
}

gla_status gla_bwd_saved(const gla_problem* p, const void* q, const void* k, const void* v, const float* g,
                         const float* igate, const float* h0, const void* dO, const float* dhT, const float* saved,
                         void* dq, void* dk, void* dv, float* dg, float* di, float* dh0, void* ws,
                         size_t ws_bytes_given, void* stream) {
    Dims P;
    int plan;
    gla_status s = check_problem(p, &P, &plan);
    if (s != GLA_OK) return s;
    s = resolve(p, P, true, &plan);
    if (s != GLA_OK) return s;
    const bool empty = (size_t)P.B * P.H * P.L == 0;
    if (!empty && (!q || !k || !v || !dO || !dq || !dk || !dv)) return GLA_ERR_INVALID_ARG;
    if (!empty && (p->gate == GLA_GATE_NONE) != (g == nullptr)) return GLA_ERR_INVALID_ARG;
    if (!empty && (p->gate == GLA_GATE_NONE) != (dg == nullptr)) return GLA_ERR_INVALID_ARG;
    if (di && !igate) return GLA_ERR_INVALID_ARG;
    if (!ws) return GLA_ERR_INVALID_ARG;
    const void* ptrs[] = {q, k, v, g, igate, h0, dO, dhT, saved, dq, dk, dv, dg, di, dh0, ws};
    for (const void* x : ptrs)
        if (!aligned16(x)) return GLA_ERR_INVALID_ARG;
    if (ws_bytes_given < ws_bytes(P, plan, true)) return GLA_ERR_WORKSPACE;
    cudaStream_t st = (cudaStream_t)stream;
    cudaError_t e = cudaMemsetAsync(ws, 0, kStatusBytes, st);
    if (e != cudaSuccess) return map_cuda(e, "status word reset");
    if ((size_t)P.B * P.H == 0) return GLA_OK;
    if (plan == GLA_PLAN_TC && P.L > 0)
        e = tc::bwd(P, q, k, v, g, igate, h0, dO, dhT, dq, dk, dv, dg, di, dh0,
                    gla_saved_states_bytes(p) ? saved : nullptr, ws, st);
    else
        e = simt::bwd(P, p->io, q, k, v, g, igate, h0, dO, dhT, dq, dk, dv, dg, di, dh0, ws, st);
    return map_cuda(e);
}

const char* gla_status_string(gla_status status) {
    const int s = static_cast<int>(status);  // any int may arrive through the ABI
    switch (s) {
        case GLA_OK: return "ok";
        case GLA_ERR_INVALID_ARG: return "invalid argument (null or misaligned pointer, bad size or enum)";
        case GLA_ERR_UNSUPPORTED: return "unsupported problem (head dims, chunk size or plan)";
        case GLA_ERR_WORKSPACE: return "workspace too small";
        case GLA_ERR_CUDA: return "CUDA runtime error";
        case GLA_ERR_TIMEOUT: return "bounded device-side wait timed out";
        case GLA_ERR_RANGE: return "log-gate decay within a 64-token tile beyond the tensor-core plan's range";
    }
    return "unknown status";
}

gla_status gla_check_device_status(void* ws, void* stream) {
    if (!ws) return GLA_ERR_INVALID_ARG;
    int word = 0;
    cudaStream_t st = (cudaStream_t)stream;
    cudaError_t e = cudaMemcpyAsync(&word, ws, sizeof(int), cudaMemcpyDeviceToHost, st);
    if (e != cudaSuccess) return map_cuda(e, "status word read");
    e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return map_cuda(e, "stream synchronisation");
    if (word & kDevStatusTimeout) return GLA_ERR_TIMEOUT;
    if (word & kDevStatusRange) return GLA_ERR_RANGE;
    return word == kDevStatusOk ? GLA_OK : GLA_ERR_TIMEOUT;
}

int gla_version(void) { return 100; }

gla_status gla_plan_info(const gla_problem* p, int for_backward, int* plan_out, int* nseg_out, int* tiles_out) {
    Dims P;
    int plan;
    gla_status s = check_problem(p, &P, &plan);
    if (s != GLA_OK) return s;
    s = resolve(p, P, for_backward != 0, &plan);
    if (s != GLA_OK) return s;
    int nseg = 1, tiles = P.N;
    if (plan == GLA_PLAN_TC) {
        if (for_backward) {
            tc::bwd_plan_info(P, &nseg, &tiles);
        } else {
            const tc::FwdPlan pl = tc::plan_fwd(P);
            nseg = pl.nseg;
            tiles = pl.tiles_per_seg;
        }
    }
    if (plan_out) *plan_out = plan;
    if (nseg_out) *nseg_out = nseg;
    if (tiles_out) *tiles_out = tiles;
    return GLA_OK;
}

const char* gla_last_error_detail(void) { return g_last_detail; }

unsigned long long gla_launch_count(void) {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    return g_launches;
}

gla_status gla_profiler_enable(int enable) {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    g_prof_on = enable != 0;
    return GLA_OK;
}

int gla_profiler_read(char* names, int name_stride, int* launches, double* total_ms, int max_kernels) {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    std::vector<std::string> keys;
    std::vector<int> cnt;
    std::vector<double> ms;
    for (ProfRecord& r : g_prof_open) {
        float t = 0.f;
        if (cudaEventSynchronize(r.stop) != cudaSuccess || cudaEventElapsedTime(&t, r.start, r.stop) != cudaSuccess)
            return -1;
        size_t i = 0;
        while (i < keys.size() && keys[i] != r.name) ++i;
        if (i == keys.size()) {
            keys.push_back(r.name);
            cnt.push_back(0);
            ms.push_back(0.0);
        }
        cnt[i] += 1;
        ms[i] += t;
        g_event_pool.push_back(r.start);
        g_event_pool.push_back(r.stop);
    }
    g_prof_open.clear();
    const int n = (int)keys.size();
    for (int i = 0; i < n && i < max_kernels; ++i) {
        if (names && name_stride > 0) {
            strncpy(names + (size_t)i * name_stride, keys[i].c_str(), name_stride - 1);
            names[(size_t)i * name_stride + name_stride - 1] = 0;
        }
        if (launches) launches[i] = cnt[i];
        if (total_ms) total_ms[i] = ms[i];
    }
    return n;
}

}  // extern "C"
