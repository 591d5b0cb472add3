// C ABI of libgla: argument checks, defaults, workspace sizing, dispatch,
// status strings and the measurement hooks (launch counter, per-kernel event
// timing). The arithmetic lives in the kernel files.

#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <vector>

#include "gla_internal.h"
#include "tc_prims.cuh"

namespace gla {
namespace {

std::atomic<uint64_t> g_launches{0};

// ---- per-kernel event timing ----------------------------------------------
struct ProfRec {
    int id;
    cudaEvent_t a, b;
};
std::mutex g_mu;
bool g_prof = false;
std::vector<ProfRec> g_pending;
std::vector<cudaEvent_t> g_pool;
std::vector<const char*> g_names;
std::vector<uint64_t> g_counts;
std::vector<double> g_ms;
thread_local cudaEvent_t t_begin = nullptr;

int name_id(const char* name) {
    for (size_t i = 0; i < g_names.size(); ++i)
        if (g_names[i] == name || std::strcmp(g_names[i], name) == 0) return int(i);
    g_names.push_back(name);
    g_counts.push_back(0);
    g_ms.push_back(0.0);
    return int(g_names.size() - 1);
}

cudaEvent_t get_event() {
    if (!g_pool.empty()) {
        cudaEvent_t e = g_pool.back();
        g_pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
}

void drain_locked() {
    for (auto& r : g_pending) {
        float ms = 0.f;
        if (cudaEventSynchronize(r.b) == cudaSuccess && cudaEventElapsedTime(&ms, r.a, r.b) == cudaSuccess) {
            g_counts[r.id] += 1;
            g_ms[r.id] += ms;
        }
        g_pool.push_back(r.a);
        g_pool.push_back(r.b);
    }
    g_pending.clear();
}

// ---- device error word ------------------------------------------------------
__device__ int g_device_error;

}  // namespace

void launch_begin(const char* name, cudaStream_t s) {
    (void)name;
    g_launches.fetch_add(1, std::memory_order_relaxed);
    t_begin = nullptr;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_prof) return;
    cudaEvent_t a = get_event();
    if (a && cudaEventRecord(a, s) == cudaSuccess) t_begin = a;
    else if (a) g_pool.push_back(a);
}

gla_status launch_end(const char* name, cudaStream_t s) {
    const cudaError_t err = cudaGetLastError();
    if (t_begin) {
        std::lock_guard<std::mutex> lk(g_mu);
        cudaEvent_t b = get_event();
        if (b && cudaEventRecord(b, s) == cudaSuccess) {
            g_pending.push_back(ProfRec{name_id(name), t_begin, b});
        } else {
            g_pool.push_back(t_begin);
            if (b) g_pool.push_back(b);
        }
        t_begin = nullptr;
        if (g_pending.size() > 4096) drain_locked();
    }
    return err == cudaSuccess ? GLA_OK : GLA_ERR_CUDA;
}

int* device_error_word() {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return nullptr;
    return static_cast<int*>(p);
}

}  // namespace gla

using gla::Problem;

namespace {

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// Gate kind and temperature (include/gla.h, gla_gate).
bool gate_ok(const gla_desc* d, Problem& p) {
    if (d->gate < GLA_GATE_CHANNEL || d->gate > GLA_GATE_PREACT) return false;
    p.gate = d->gate;
    p.inv_tau = 0.f;
    if (d->gate == GLA_GATE_PREACT) {
        if (!(d->gate_tau > 0.f) || !(d->gate_tau < 3.0e38f)) return false;
        p.inv_tau = 1.f / d->gate_tau;
    }
    return true;
}

// Fill `p` from `d` (defaults applied). Returns GLA_OK or an error status.
gla_status resolve(const gla_desc* d, Problem& p) {
    if (!d) return GLA_ERR_INVALID_ARG;
    if (d->B < 1 || d->H < 1 || d->L < 1 || d->Dk < 1 || d->Dv < 1) return GLA_ERR_INVALID_ARG;
    if (d->dtype != GLA_DTYPE_F32 && d->dtype != GLA_DTYPE_BF16) return GLA_ERR_INVALID_ARG;
    if (d->chunk != 0 && d->chunk != 16 && d->chunk != 32 && d->chunk != 64 && d->chunk != 128)
        return GLA_ERR_INVALID_ARG;
    if (d->subchunk < 0) return GLA_ERR_INVALID_ARG;
    if (d->state_mode < GLA_STATE_AUTO || d->state_mode > GLA_STATE_NONMATERIALIZED) return GLA_ERR_INVALID_ARG;
    if (d->impl < GLA_IMPL_AUTO || d->impl > GLA_IMPL_TC) return GLA_ERR_INVALID_ARG;
    if (d->flags & ~int32_t(GLA_FLAG_WS_FROM_FWD | GLA_FLAG_CHECKS)) return GLA_ERR_INVALID_ARG;
    if (!gate_ok(d, p)) return GLA_ERR_INVALID_ARG;
    p.B = d->B;
    p.H = d->H;
    p.L = d->L;
    p.K = d->Dk;
    p.V = d->Dv;
    p.BH = d->B * d->H;
    p.bf16 = d->dtype == GLA_DTYPE_BF16;
    p.flags = d->flags;
    if (p.BH > 65535) return GLA_ERR_UNSUPPORTED;
    int impl = d->impl;
    if (impl == GLA_IMPL_AUTO) {
        Problem probe = p;
        probe.C = d->chunk ? d->chunk : 128;
        probe.c = d->subchunk ? d->subchunk : 128;
        probe.N = (p.L + probe.C - 1) / probe.C;
        probe.impl = GLA_IMPL_TC;
        probe.state_mode = d->state_mode;
        impl = (p.bf16 && gla::tc_supported(probe)) ? GLA_IMPL_TC : GLA_IMPL_SIMT;
    }
    p.impl = impl;
    if (impl == GLA_IMPL_SIMT) {
        p.C = d->chunk ? d->chunk : 64;
        p.c = d->subchunk ? d->subchunk : (p.C < 16 ? p.C : 16);  // secondary chunks of 16 rows
        if (d->state_mode == GLA_STATE_NONMATERIALIZED) return GLA_ERR_UNSUPPORTED;
        p.state_mode = GLA_STATE_MATERIALIZED;
    } else {
        if (!p.bf16) return GLA_ERR_UNSUPPORTED;
        p.C = d->chunk ? d->chunk : 128;
        p.c = d->subchunk ? d->subchunk : 128;  // one GEMM per chunk; 16 selects two-level chunking
        // materialised states are the faster mode on this path (the backward needs the stored states in
        // either mode); non-materialised keeps the forward's footprint free of them
        p.state_mode = d->state_mode == GLA_STATE_AUTO ? GLA_STATE_MATERIALIZED : d->state_mode;
    }
    if (p.c > p.C || p.C % p.c != 0) return GLA_ERR_INVALID_ARG;
    p.N = (p.L + p.C - 1) / p.C;
    if (p.N > 65535) return GLA_ERR_UNSUPPORTED;
    if (impl == GLA_IMPL_TC && !gla::tc_supported(p)) return GLA_ERR_UNSUPPORTED;
    return GLA_OK;
}

// Workspace layout of a pass: [per-channel log alpha when the gate kind is not per channel] [the
// path's own slices] [backward of a scalar or head gate: the per-channel gate gradient]. The
// forward's part is a prefix of the backward's, so a backward can reuse a forward's workspace.
struct Layout {
    float* la_pc = nullptr;   // expanded per-channel log alpha (null: the caller's log_a is per channel)
    float* dla_pc = nullptr;  // per-channel gate gradient (backward, scalar and head kinds)
};

// The tensor-core path reads every gate kind natively; the CUDA-core path works on the expansion.
Layout carve_all(const Problem& p, gla::Arena& a, bool bwd, bool path_too) {
    Layout l;
    if (p.gate != GLA_GATE_CHANNEL && p.impl == GLA_IMPL_SIMT) l.la_pc = a.take<float>(size_t(p.BH * p.L * p.K));
    if (path_too) {
        if (bwd) (p.impl == GLA_IMPL_TC ? gla::tc_layout : gla::simt_layout)(p, a, true);
        else (p.impl == GLA_IMPL_TC ? gla::tc_layout : gla::simt_layout)(p, a, false);
    }
    return l;
}

float* carve_dla_pc(const Problem& p, gla::Arena& a) {
    return (p.impl == GLA_IMPL_SIMT && (p.gate == GLA_GATE_SCALAR || p.gate == GLA_GATE_HEAD))
               ? a.take<float>(size_t(p.BH * p.L * p.K))
               : nullptr;
}

size_t ws_size(const Problem& p, bool bwd) {
    gla::Arena a = gla::make_arena(p, nullptr, 0);
    carve_all(p, a, bwd, true);
    if (bwd) carve_dla_pc(p, a);
    return a.used;
}

size_t fwd_ws(const Problem& p) { return ws_size(p, false); }
size_t bwd_ws(const Problem& p) { return ws_size(p, true); }

int64_t gate_elems(const Problem& p, int64_t steps) {
    switch (p.gate) {
        case GLA_GATE_SCALAR: return p.BH * steps;
        case GLA_GATE_HEAD: return p.H;
        default: return p.BH * steps * p.K;
    }
}

gla_status check_ws(void* ws, size_t bytes, size_t need) {
    if (need == 0) return GLA_OK;
    if (!ws || !aligned(ws, 256) || bytes < need) return GLA_ERR_WORKSPACE;
    return GLA_OK;
}

// The two GLA passes of gated slot attention (include/gla.h): layer one has GLA key width `slots` and
// value width Dk, layer two key width `slots` and value width Dv. bf16 with 128 slots takes the
// tensor-core route when both passes resolve to the tensor-core path; everything else runs both passes
// on the CUDA-core path in fp32.
gla_status resolve_gsa(const gla_desc* d, int32_t slots, gla::GsaProblem& g) {
    if (!d || slots < 1) return GLA_ERR_INVALID_ARG;
    if (d->flags & ~int32_t(GLA_FLAG_WS_FROM_FWD | GLA_FLAG_CHECKS)) return GLA_ERR_INVALID_ARG;
    Problem gp{};
    if (!gate_ok(d, gp)) return GLA_ERR_INVALID_ARG;
    if (d->gate != GLA_GATE_CHANNEL && d->gate != GLA_GATE_PREACT) return GLA_ERR_UNSUPPORTED;
    if (d->dtype != GLA_DTYPE_F32 && d->dtype != GLA_DTYPE_BF16) return GLA_ERR_INVALID_ARG;
    g.preact = d->gate == GLA_GATE_PREACT;
    g.inv_tau = gp.inv_tau;
    gla_desc da = *d, db = *d;
    // the passes take the expanded per-slot log a
    da.gate = db.gate = GLA_GATE_CHANNEL;
    da.gate_tau = db.gate_tau = 0.f;
    da.Dk = slots;
    da.Dv = d->Dk;
    da.flags = 0;
    db.Dk = slots;
    db.Dv = d->Dv;
    db.flags = 0;
    g.m = slots;
    g.io_bf16 = d->dtype == GLA_DTYPE_BF16;
    g.tc = false;
    if (g.io_bf16 && d->impl != GLA_IMPL_SIMT && (d->subchunk == 0 || d->subchunk == 128) &&
        d->state_mode != GLA_STATE_NONMATERIALIZED) {
        gla_desc ta = da, tb = db;
        ta.state_mode = tb.state_mode = GLA_STATE_MATERIALIZED;
        gla::GsaProblem t{};
        if (resolve(&ta, t.A) == GLA_OK && resolve(&tb, t.B) == GLA_OK && gla::gsa_tc_route(t.A, t.B, slots)) {
            g.A = t.A;
            g.B = t.B;
            g.tc = true;
            return GLA_OK;
        }
    }
    if (d->impl == GLA_IMPL_TC) return GLA_ERR_UNSUPPORTED;
    da.dtype = db.dtype = GLA_DTYPE_F32;
    da.impl = db.impl = GLA_IMPL_SIMT;
    gla_status st = resolve(&da, g.A);
    if (st == GLA_OK) st = resolve(&db, g.B);
    return st;
}

#define GLA_REQUIRE_PTR(ptr) \
    do {                     \
        if (!(ptr) || !aligned((ptr), 16)) return GLA_ERR_INVALID_ARG; \
    } while (0)
#define GLA_OPTIONAL_PTR(ptr) \
    do {                      \
        if ((ptr) && !aligned((ptr), 16)) return GLA_ERR_INVALID_ARG; \
    } while (0)

}  // namespace

extern "C" {

int gla_abi_version(void) { return GLA_ABI_VERSION; }

const char* gla_status_string(gla_status s) {
    switch (s) {
        case GLA_OK: return "ok";
        case GLA_ERR_INVALID_ARG: return "invalid argument (null or misaligned pointer, bad size or enum)";
        case GLA_ERR_UNSUPPORTED: return "unsupported shape or option for the selected kernel path";
        case GLA_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
        case GLA_ERR_CUDA: return "CUDA runtime error or failed kernel launch";
        case GLA_ERR_TIMEOUT: return "a device-side bounded wait ran out";
    }
    return "unknown status";
}

gla_status gla_resolve(const gla_desc* d, int32_t* chunk, int32_t* subchunk, int32_t* impl, int32_t* state_mode) {
    Problem p{};
    gla_status st = resolve(d, p);
    if (st != GLA_OK) return st;
    if (chunk) *chunk = p.C;
    if (subchunk) *subchunk = p.c;
    if (impl) *impl = p.impl;
    if (state_mode) *state_mode = p.state_mode;
    return GLA_OK;
}

size_t gla_fwd_workspace_size(const gla_desc* d) {
    Problem p{};
    if (resolve(d, p) != GLA_OK) return 0;
    return fwd_ws(p);
}

size_t gla_bwd_workspace_size(const gla_desc* d) {
    Problem p{};
    if (resolve(d, p) != GLA_OK) return 0;
    const size_t a = fwd_ws(p), b = bwd_ws(p);
    return a > b ? a : b;
}

gla_status gla_fwd(const gla_desc* d, const void* q, const void* k, const void* v, const float* log_a,
                   const float* h0, void* o, float* hT, void* workspace, size_t workspace_bytes, void* stream) {
    Problem p{};
    gla_status st = resolve(d, p);
    if (st != GLA_OK) return st;
    GLA_REQUIRE_PTR(q);
    GLA_REQUIRE_PTR(k);
    GLA_REQUIRE_PTR(v);
    GLA_REQUIRE_PTR(log_a);
    GLA_REQUIRE_PTR(o);
    GLA_OPTIONAL_PTR(h0);
    GLA_OPTIONAL_PTR(hT);
    const size_t need = fwd_ws(p);
    st = check_ws(workspace, workspace_bytes, need);
    if (st != GLA_OK) return st;
    gla::Arena a = gla::make_arena(p, workspace, workspace_bytes);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const bool chk = gla::checks_on(p);
    const Layout l = carve_all(p, a, false, false);  // gate slices; the path carves the rest itself
    const float* la = log_a;
    if (l.la_pc) {
        st = gla::gate_expand(p, log_a, l.la_pc, s);
        if (st != GLA_OK) return st;
        la = l.la_pc;
    }
    gla::Arena layout = gla::make_arena(p, workspace, workspace_bytes);
    if (chk) {
        carve_all(p, layout, false, true);
        st = p.gate == GLA_GATE_PREACT ? GLA_OK : gla::check_gates(log_a, gate_elems(p, p.L), s);
        if (st == GLA_OK) st = gla::guards_fill(layout, s);
        if (st != GLA_OK) return st;
    }
    st = p.impl == GLA_IMPL_TC ? gla::tc_fwd(p, q, k, v, la, h0, o, hT, a, s)
                               : gla::simt_fwd(p, q, k, v, la, h0, o, hT, a, s);
    if (st != GLA_OK || !chk) return st;
    st = gla::check_finite(o, p.BH * p.L * p.V, p.bf16, s);
    if (st == GLA_OK) st = gla::check_finite(hT, p.BH * p.K * p.V, false, s);
    if (st == GLA_OK) st = gla::guards_check(layout, s);
    return st;
}

gla_status gla_bwd(const gla_desc* d, const void* q, const void* k, const void* v, const float* log_a,
                   const float* h0, const void* dO, const float* dhT, void* dq, void* dk, void* dv, float* dlog_a,
                   float* dh0, void* workspace, size_t workspace_bytes, void* stream) {
    Problem p{};
    gla_status st = resolve(d, p);
    if (st != GLA_OK) return st;
    GLA_REQUIRE_PTR(q);
    GLA_REQUIRE_PTR(k);
    GLA_REQUIRE_PTR(v);
    GLA_REQUIRE_PTR(log_a);
    GLA_REQUIRE_PTR(dO);
    GLA_REQUIRE_PTR(dq);
    GLA_REQUIRE_PTR(dk);
    GLA_REQUIRE_PTR(dv);
    GLA_REQUIRE_PTR(dlog_a);
    GLA_OPTIONAL_PTR(h0);
    GLA_OPTIONAL_PTR(dhT);
    GLA_OPTIONAL_PTR(dh0);
    const size_t need = bwd_ws(p);
    st = check_ws(workspace, workspace_bytes, need);
    if (st != GLA_OK) return st;
    gla::Arena a = gla::make_arena(p, workspace, workspace_bytes);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const bool chk = gla::checks_on(p);
    const Layout l = carve_all(p, a, true, false);
    const float* la = log_a;
    if (l.la_pc) {
        // a forward's workspace holds the expansion already, unless the caller says nothing of it
        if (!(p.flags & GLA_FLAG_WS_FROM_FWD)) {
            st = gla::gate_expand(p, log_a, l.la_pc, s);
            if (st != GLA_OK) return st;
        }
        la = l.la_pc;
    }
    gla::Arena layout = gla::make_arena(p, workspace, workspace_bytes);
    if (chk) {
        carve_all(p, layout, true, true);
        carve_dla_pc(p, layout);
        st = p.gate == GLA_GATE_PREACT ? GLA_OK : gla::check_gates(log_a, gate_elems(p, p.L), s);
        if (st == GLA_OK) st = gla::guards_fill(layout, s);
        if (st != GLA_OK) return st;
    }
    // the per-channel gate gradient goes to the workspace (scalar, head) or to dlog_a itself (channel,
    // preact: scaled in place afterwards)
    float* dla_pc = dlog_a;
    {
        gla::Arena tail = gla::make_arena(p, workspace, workspace_bytes);
        carve_all(p, tail, true, true);
        float* w = carve_dla_pc(p, tail);
        if (tail.used > tail.cap) return GLA_ERR_WORKSPACE;
        if (w) dla_pc = w;
    }
    st = p.impl == GLA_IMPL_TC ? gla::tc_bwd(p, q, k, v, la, h0, dO, dhT, dq, dk, dv, dla_pc, dh0, a, s)
                               : gla::simt_bwd(p, q, k, v, la, h0, dO, dhT, dq, dk, dv, dla_pc, dh0, a, s);
    if (st == GLA_OK && p.gate != GLA_GATE_CHANNEL && p.impl == GLA_IMPL_SIMT)
        st = gla::gate_grad(p, log_a, dla_pc, dlog_a, s);
    if (st != GLA_OK || !chk) return st;
    const int64_t nk = p.BH * p.L * p.K, nv = p.BH * p.L * p.V;
    st = gla::check_finite(dq, nk, p.bf16, s);
    if (st == GLA_OK) st = gla::check_finite(dk, nk, p.bf16, s);
    if (st == GLA_OK) st = gla::check_finite(dv, nv, p.bf16, s);
    if (st == GLA_OK) st = gla::check_finite(dlog_a, gate_elems(p, p.L), false, s);
    if (st == GLA_OK) st = gla::check_finite(dh0, p.BH * p.K * p.V, false, s);
    if (st == GLA_OK) st = gla::guards_check(layout, s);
    return st;
}

gla_status gla_step(const gla_desc* d, const void* q, const void* k, const void* v, const float* log_a, float* S,
                    void* o, void* stream) {
    if (!d) return GLA_ERR_INVALID_ARG;
    if (d->B < 1 || d->H < 1 || d->Dk < 1 || d->Dv < 1) return GLA_ERR_INVALID_ARG;
    if (d->dtype != GLA_DTYPE_F32 && d->dtype != GLA_DTYPE_BF16) return GLA_ERR_INVALID_ARG;
    GLA_REQUIRE_PTR(q);
    GLA_REQUIRE_PTR(k);
    GLA_REQUIRE_PTR(v);
    GLA_REQUIRE_PTR(log_a);
    GLA_REQUIRE_PTR(S);
    GLA_REQUIRE_PTR(o);
    if (d->B * d->H > 65535 || d->Dk > 8192) return GLA_ERR_UNSUPPORTED;
    if (d->flags & ~int32_t(GLA_FLAG_WS_FROM_FWD | GLA_FLAG_CHECKS)) return GLA_ERR_INVALID_ARG;
    Problem p{};
    if (!gate_ok(d, p)) return GLA_ERR_INVALID_ARG;
    p.B = d->B;
    p.H = d->H;
    p.L = 1;
    p.K = d->Dk;
    p.V = d->Dv;
    p.BH = d->B * d->H;
    p.bf16 = d->dtype == GLA_DTYPE_BF16;
    p.flags = d->flags;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const bool chk = gla::checks_on(p);
    gla_status st = chk && p.gate != GLA_GATE_PREACT ? gla::check_gates(log_a, gate_elems(p, 1), s) : GLA_OK;
    if (st == GLA_OK) st = gla::step_launch(p, q, k, v, log_a, S, o, s);
    if (st != GLA_OK || !chk) return st;
    st = gla::check_finite(o, p.BH * p.V, p.bf16, s);
    if (st == GLA_OK) st = gla::check_finite(S, p.BH * p.K * p.V, false, s);
    return st;
}

gla_status gla_chunk_cumsum(const gla_desc* d, const float* log_a, float* Bcum, void* stream) {
    if (!d) return GLA_ERR_INVALID_ARG;
    if (d->B < 1 || d->H < 1 || d->L < 1 || d->Dk < 1) return GLA_ERR_INVALID_ARG;
    const int C = d->chunk ? d->chunk : 64;
    if (C != 16 && C != 32 && C != 64 && C != 128) return GLA_ERR_INVALID_ARG;
    if (d->gate != GLA_GATE_CHANNEL) return GLA_ERR_UNSUPPORTED;
    GLA_REQUIRE_PTR(log_a);
    GLA_REQUIRE_PTR(Bcum);
    Problem p{};
    p.B = d->B;
    p.H = d->H;
    p.L = d->L;
    p.K = d->Dk;
    p.V = d->Dv;
    p.BH = d->B * d->H;
    p.C = C;
    p.N = (p.L + C - 1) / C;
    if (p.BH > 65535 || p.N > 65535) return GLA_ERR_UNSUPPORTED;
    return gla::simt_chunk_cumsum(p, log_a, Bcum, static_cast<cudaStream_t>(stream));
}

gla_status gla_fwd_final_state(const gla_desc* d, const void* q, const void* k, const void* v, const float* log_a,
                               const float* h0, float* hT, void* workspace, size_t workspace_bytes, void* stream) {
    Problem p{};
    gla_status st = resolve(d, p);
    if (st != GLA_OK) return st;
    if (p.impl != GLA_IMPL_TC || p.state_mode != GLA_STATE_MATERIALIZED) return GLA_ERR_UNSUPPORTED;
    GLA_REQUIRE_PTR(q);
    GLA_REQUIRE_PTR(k);
    GLA_REQUIRE_PTR(v);
    GLA_REQUIRE_PTR(log_a);
    GLA_REQUIRE_PTR(hT);
    GLA_OPTIONAL_PTR(h0);
    st = check_ws(workspace, workspace_bytes, fwd_ws(p));
    if (st != GLA_OK) return st;
    gla::Arena a = gla::make_arena(p, workspace, workspace_bytes);
    return gla::tc_fwd_final_state(p, q, k, v, log_a, h0, hT, a, static_cast<cudaStream_t>(stream));
}

gla_status gla_bwd_initial_grad(const gla_desc* d, const void* q, const void* k, const float* log_a, const void* dO,
                                const float* dhT, float* dh0, void* workspace, size_t workspace_bytes, void* stream) {
    Problem p{};
    gla_status st = resolve(d, p);
    if (st != GLA_OK) return st;
    if (p.impl != GLA_IMPL_TC || p.state_mode != GLA_STATE_MATERIALIZED) return GLA_ERR_UNSUPPORTED;
    GLA_REQUIRE_PTR(q);
    GLA_REQUIRE_PTR(k);
    GLA_REQUIRE_PTR(log_a);
    GLA_REQUIRE_PTR(dO);
    GLA_REQUIRE_PTR(dh0);
    GLA_OPTIONAL_PTR(dhT);
    st = check_ws(workspace, workspace_bytes, bwd_ws(p));
    if (st != GLA_OK) return st;
    gla::Arena a = gla::make_arena(p, workspace, workspace_bytes);
    return gla::tc_bwd_initial_grad(p, q, k, log_a, dO, dhT, dh0, a, static_cast<cudaStream_t>(stream));
}

gla_status gla_segment_decay(const gla_desc* d, const float* log_a, float* a, void* stream) {
    Problem p{};
    gla_status st = resolve(d, p);
    if (st != GLA_OK) return st;
    GLA_REQUIRE_PTR(log_a);
    GLA_REQUIRE_PTR(a);
    return gla::segment_decay(p, log_a, a, static_cast<cudaStream_t>(stream));
}

gla_status gla_state_combine(int64_t G, int64_t BH, int64_t Dk, int64_t Dv, const float* a, const float* U,
                             const float* init, int32_t r, int32_t reverse, float* out, void* stream) {
    if (G < 1 || BH < 1 || Dk < 1 || Dv < 1 || Dv % 4 != 0 || r < 0 || r >= G) return GLA_ERR_INVALID_ARG;
    if (reverse != 0 && reverse != 1) return GLA_ERR_INVALID_ARG;
    if (BH * Dk * (Dv / 4) > (int64_t(1) << 31) - 1) return GLA_ERR_UNSUPPORTED;
    GLA_REQUIRE_PTR(a);
    GLA_REQUIRE_PTR(U);
    GLA_OPTIONAL_PTR(init);
    GLA_REQUIRE_PTR(out);
    return gla::state_combine(G, BH, Dk, Dv, a, U, init, r, reverse, out, static_cast<cudaStream_t>(stream));
}

gla_status gla_gsa_resolve(const gla_desc* d, int32_t slots, int32_t* impl) {
    gla::GsaProblem g{};
    const gla_status st = resolve_gsa(d, slots, g);
    if (st == GLA_OK && impl) *impl = g.tc ? GLA_IMPL_TC : GLA_IMPL_SIMT;
    return st;
}

size_t gla_gsa_fwd_workspace_size(const gla_desc* d, int32_t slots) {
    gla::GsaProblem g{};
    if (resolve_gsa(d, slots, g) != GLA_OK) return 0;
    return gla::gsa_workspace(g, false);
}

size_t gla_gsa_bwd_workspace_size(const gla_desc* d, int32_t slots) {
    gla::GsaProblem g{};
    if (resolve_gsa(d, slots, g) != GLA_OK) return 0;
    return gla::gsa_workspace(g, true);
}

gla_status gla_gsa_fwd(const gla_desc* d, int32_t slots, const void* q, const void* k, const void* v,
                       const float* log_a, const float* hk0, const float* hv0, void* o, float* hkT, float* hvT,
                       void* workspace, size_t workspace_bytes, void* stream) {
    gla::GsaProblem g{};
    gla_status st = resolve_gsa(d, slots, g);
    if (st != GLA_OK) return st;
    if (d->flags & GLA_FLAG_WS_FROM_FWD) return GLA_ERR_INVALID_ARG;
    GLA_REQUIRE_PTR(q);
    GLA_REQUIRE_PTR(k);
    GLA_REQUIRE_PTR(v);
    GLA_REQUIRE_PTR(log_a);
    GLA_REQUIRE_PTR(o);
    GLA_OPTIONAL_PTR(hk0);
    GLA_OPTIONAL_PTR(hv0);
    GLA_OPTIONAL_PTR(hkT);
    GLA_OPTIONAL_PTR(hvT);
    st = check_ws(workspace, workspace_bytes, gla::gsa_workspace(g, false));
    if (st != GLA_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    Problem pc = g.B;
    pc.flags = d->flags;
    const bool chk = gla::checks_on(pc);
    const int64_t nm = g.B.BH * g.B.L * g.m;
    if (chk && !g.preact && (st = gla::check_gates(log_a, nm, s)) != GLA_OK) return st;
    st = gla::gsa_fwd(g, q, k, v, log_a, hk0, hv0, o, hkT, hvT, workspace, workspace_bytes, s);
    if (st != GLA_OK || !chk) return st;
    st = gla::check_finite(o, g.B.BH * g.B.L * g.B.V, g.io_bf16, s);
    if (st == GLA_OK) st = gla::check_finite(hkT, g.A.BH * g.m * g.A.V, false, s);
    if (st == GLA_OK) st = gla::check_finite(hvT, g.B.BH * g.m * g.B.V, false, s);
    return st;
}

gla_status gla_gsa_step(const gla_desc* d, int32_t slots, const void* q, const void* k, const void* v,
                        const float* log_a, float* Kmem, float* Vmem, void* o, void* stream) {
    if (!d || slots < 1) return GLA_ERR_INVALID_ARG;
    if (d->B < 1 || d->H < 1 || d->Dk < 1 || d->Dv < 1) return GLA_ERR_INVALID_ARG;
    if (d->dtype != GLA_DTYPE_F32 && d->dtype != GLA_DTYPE_BF16) return GLA_ERR_INVALID_ARG;
    if (d->flags & ~int32_t(GLA_FLAG_WS_FROM_FWD | GLA_FLAG_CHECKS)) return GLA_ERR_INVALID_ARG;
    Problem gp{};
    if (!gate_ok(d, gp)) return GLA_ERR_INVALID_ARG;
    if (d->gate != GLA_GATE_CHANNEL && d->gate != GLA_GATE_PREACT) return GLA_ERR_UNSUPPORTED;
    GLA_REQUIRE_PTR(q);
    GLA_REQUIRE_PTR(k);
    GLA_REQUIRE_PTR(v);
    GLA_REQUIRE_PTR(log_a);
    GLA_REQUIRE_PTR(Kmem);
    GLA_REQUIRE_PTR(Vmem);
    GLA_REQUIRE_PTR(o);
    if (!gla::gsa_step_supported(slots, d->Dk, d->Dv)) return GLA_ERR_UNSUPPORTED;
    Problem p{};
    p.B = d->B;
    p.H = d->H;
    p.L = 1;
    p.K = d->Dk;
    p.V = d->Dv;
    p.BH = d->B * d->H;
    p.flags = d->flags;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const bool chk = gla::checks_on(p);
    const bool bf16 = d->dtype == GLA_DTYPE_BF16;
    gla_status st = chk && d->gate == GLA_GATE_CHANNEL ? gla::check_gates(log_a, p.BH * slots, s) : GLA_OK;
    if (st == GLA_OK)
        st = gla::gsa_step(p.BH, slots, d->Dk, d->Dv, bf16, q, k, v, log_a, gp.inv_tau, Kmem, Vmem, o, s);
    if (st != GLA_OK || !chk) return st;
    st = gla::check_finite(o, p.BH * d->Dv, bf16, s);
    if (st == GLA_OK) st = gla::check_finite(Kmem, p.BH * slots * d->Dk, false, s);
    if (st == GLA_OK) st = gla::check_finite(Vmem, p.BH * slots * d->Dv, false, s);
    return st;
}

gla_status gla_gsa_bwd(const gla_desc* d, int32_t slots, const void* q, const void* k, const void* v,
                       const float* log_a, const float* hk0, const float* hv0, const void* dO, const float* dhkT,
                       const float* dhvT, void* dq, void* dk, void* dv, float* dlog_a, float* dhk0, float* dhv0,
                       void* workspace, size_t workspace_bytes, void* stream) {
    gla::GsaProblem g{};
    gla_status st = resolve_gsa(d, slots, g);
    if (st != GLA_OK) return st;
    GLA_REQUIRE_PTR(q);
    GLA_REQUIRE_PTR(k);
    GLA_REQUIRE_PTR(v);
    GLA_REQUIRE_PTR(log_a);
    GLA_REQUIRE_PTR(dO);
    GLA_REQUIRE_PTR(dq);
    GLA_REQUIRE_PTR(dk);
    GLA_REQUIRE_PTR(dv);
    GLA_REQUIRE_PTR(dlog_a);
    GLA_OPTIONAL_PTR(hk0);
    GLA_OPTIONAL_PTR(hv0);
    GLA_OPTIONAL_PTR(dhkT);
    GLA_OPTIONAL_PTR(dhvT);
    GLA_OPTIONAL_PTR(dhk0);
    GLA_OPTIONAL_PTR(dhv0);
    st = check_ws(workspace, workspace_bytes, gla::gsa_workspace(g, true));
    if (st != GLA_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    Problem pc = g.B;
    pc.flags = d->flags;
    const bool chk = gla::checks_on(pc);
    const int64_t nm = g.B.BH * g.B.L * g.m;
    if (chk && !g.preact && (st = gla::check_gates(log_a, nm, s)) != GLA_OK) return st;
    st = gla::gsa_bwd(g, q, k, v, log_a, hk0, hv0, dO, dhkT, dhvT, dq, dk, dv, dlog_a, dhk0, dhv0,
                      (d->flags & GLA_FLAG_WS_FROM_FWD) != 0, workspace, workspace_bytes, s);
    if (st != GLA_OK || !chk) return st;
    const int64_t nk = g.B.BH * g.B.L * g.A.V, nv = g.B.BH * g.B.L * g.B.V;
    st = gla::check_finite(dq, nk, g.io_bf16, s);
    if (st == GLA_OK) st = gla::check_finite(dk, nk, g.io_bf16, s);
    if (st == GLA_OK) st = gla::check_finite(dv, nv, g.io_bf16, s);
    if (st == GLA_OK) st = gla::check_finite(dlog_a, nm, false, s);
    if (st == GLA_OK) st = gla::check_finite(dhk0, g.A.BH * g.m * g.A.V, false, s);
    if (st == GLA_OK) st = gla::check_finite(dhv0, g.B.BH * g.m * g.B.V, false, s);
    return st;
}

namespace {
// One thread waits on an mbarrier nothing arrives on: the bounded wait must give up, record the
// timeout and let the kernel finish.
__global__ void k_selftest_wait_timeout(int* err, long long limit_cycles) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        gla::tc::mbar_init(&bar, 1);
        abort_flag = 0;
        gla::tc::fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) (void)gla::tc::mbar_wait(&bar, 0, err, &abort_flag, limit_cycles);
}
}  // namespace

gla_status gla_selftest_wait_timeout(long long limit_cycles, void* stream) {
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    GLA_LAUNCH("selftest_wait_timeout", k_selftest_wait_timeout, 1, 32, 0, s, gla::device_error_word(),
               limit_cycles > 0 ? limit_cycles : 2000000LL);
    return GLA_OK;
}

gla_status gla_check_device_error(void* stream) {
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return GLA_ERR_CUDA;
    int* w = gla::device_error_word();
    if (!w) return GLA_ERR_CUDA;
    int h = 0;
    if (cudaMemcpy(&h, w, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return GLA_ERR_CUDA;
    if (h != 0) {
        const int zero = 0;
        if (cudaMemcpy(w, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return GLA_ERR_CUDA;
        if (h & gla::tc::kErrWaitTimeout) return GLA_ERR_TIMEOUT;
        if (h & (gla::kErrBadGate | gla::kErrNonFinite)) return GLA_ERR_INVALID_ARG;
        if (h & gla::kErrGuard) return GLA_ERR_WORKSPACE;
        return GLA_ERR_CUDA;
    }
    return GLA_OK;
}

gla_status gla_last_device_error(void* stream) { return gla_check_device_error(stream); }

size_t gla_fwd_workspace_bytes(const gla_desc* d) { return gla_fwd_workspace_size(d); }
size_t gla_bwd_workspace_bytes(const gla_desc* d) { return gla_bwd_workspace_size(d); }

uint64_t gla_launch_count(void) { return gla::g_launches.load(); }
void gla_launch_count_reset(void) { gla::g_launches.store(0); }

void gla_profile_enable(int on) {
    std::lock_guard<std::mutex> lk(gla::g_mu);
    gla::g_prof = on != 0;
}

int gla_profile_read(const char** names, uint64_t* launches, double* total_ms, int cap) {
    std::lock_guard<std::mutex> lk(gla::g_mu);
    gla::drain_locked();
    const int n = int(gla::g_names.size());
    for (int i = 0; i < n && i < cap; ++i) {
        if (names) names[i] = gla::g_names[i];
        if (launches) launches[i] = gla::g_counts[i];
        if (total_ms) total_ms[i] = gla::g_ms[i];
    }
    return n;
}

void gla_profile_reset(void) {
    std::lock_guard<std::mutex> lk(gla::g_mu);
    gla::drain_locked();
    for (cudaEvent_t e : gla::g_pool) cudaEventDestroy(e);
    gla::g_pool.clear();
    gla::g_names.clear();
    gla::g_counts.clear();
    gla::g_ms.clear();
}

}  // extern "C"
