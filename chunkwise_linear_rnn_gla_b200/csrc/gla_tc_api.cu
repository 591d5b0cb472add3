// Tensor-core path: support check, workspace layout and the kernel sequence
// of the forward (and, for now, the backward).
//
// Forward, non-materialised states (default):
//   tc_prep  (chunk-parallel)  cumsum, Q~, K~, e^Gamma, intra-chunk P
//   tc_walk  (fused)           per (head, 64-column tile): state walk on chip
//                               and o = Q~ S + P v
// Forward, materialised states:
//   tc_prep, tc_walk (states only: writes S_[i] in bf16 to the workspace),
//   tc_output (chunk-parallel: o = Q~ S_[i] + P v from the stored states)

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "gla_internal.h"
#include "gla_tc.h"

namespace gla {

namespace {

struct TcBuffers {
    __nv_bfloat16 *Qt, *Kt, *P;
    float* gam;
    __nv_bfloat16* states;
};

TcBuffers carve_fwd(const Problem& p, Arena& a) {
    TcBuffers b{};
    b.Qt = a.take<__nv_bfloat16>(size_t(p.BH * p.L * p.K));
    b.Kt = a.take<__nv_bfloat16>(size_t(p.BH * p.L * p.K));
    b.P = a.take<__nv_bfloat16>(size_t(p.BH * p.N * kTcChunk * kTcChunk));
    b.gam = a.take<float>(size_t(p.BH * p.N * p.K));
    if (p.state_mode == GLA_STATE_MATERIALIZED) b.states = a.take<__nv_bfloat16>(size_t(p.BH * p.N * p.K * p.V));
    return b;
}

}  // namespace

bool tc_supported(const Problem& p) {
    if (!p.bf16) return false;
    if (p.C != kTcChunk || p.c != kTcSub) return false;
    if (p.K != 128 && p.K != 256) return false;
    if (p.V < 64 || p.V % 64 != 0 || p.V / 64 > 65535) return false;
    if (p.BH > 65535 || p.N > 65535) return false;
    if (p.BH * p.N > (int64_t(1) << 31) - 1) return false;
    return true;
}

size_t tc_fwd_workspace(const Problem& p) {
    Arena a{nullptr, 0, 0};
    carve_fwd(p, a);
    return a.used;
}

size_t tc_bwd_workspace(const Problem& p) {
    // interim: the backward runs the CUDA-core kernels after the forward's buffers
    Arena a{nullptr, 0, 0};
    carve_fwd(p, a);
    Problem ps = p;
    ps.C = 64;
    ps.c = 64;
    ps.N = (p.L + 63) / 64;
    return a.used + 256 + simt_bwd_workspace(ps);
}

gla_status tc_fwd(const Problem& p, const void* q, const void* k, const void* v, const float* la, const float* h0,
                  void* o, float* hT, Arena& ws, cudaStream_t s) {
    TcBuffers b = carve_fwd(p, ws);
    if (ws.used > ws.cap) return GLA_ERR_WORKSPACE;
    gla_status st = tc_prep_launch(p, q, k, la, b.Qt, b.Kt, b.P, b.gam, nullptr, s);
    if (st != GLA_OK) return st;
    WalkArgs a{};
    a.A1 = b.Kt;
    a.B1 = static_cast<const __nv_bfloat16*>(v);
    a.A2 = b.Qt;
    a.Pm = b.P;
    a.gam = b.gam;
    a.init = h0;
    a.fin = hT;
    a.Y = static_cast<__nv_bfloat16*>(o);
    a.reverse = false;
    a.p_transposed = false;
    if (p.state_mode == GLA_STATE_NONMATERIALIZED) {
        a.mode = kWalkFused;
        return tc_walk_launch(p, a, s, "tc_walk_fwd");
    }
    a.states = b.states;
    a.mode = kWalkStatesOnly;
    st = tc_walk_launch(p, a, s, "tc_walk_states");
    if (st != GLA_OK) return st;
    a.mode = kWalkOutputOnly;
    a.fin = nullptr;
    return tc_walk_launch(p, a, s, "tc_output");
}

gla_status tc_bwd(const Problem& p, const void* q, const void* k, const void* v, const float* la, const float* h0,
                  const void* dO, const float* dhT, void* dq, void* dk, void* dv, float* dla, float* dh0, Arena& ws,
                  cudaStream_t s) {
    // interim: CUDA-core backward (recomputes its own intermediates)
    Arena a{nullptr, 0, 0};
    carve_fwd(p, a);
    Problem ps = p;
    ps.impl = GLA_IMPL_SIMT;
    ps.C = 64;
    ps.c = 64;
    ps.N = (p.L + 63) / 64;
    ps.state_mode = GLA_STATE_MATERIALIZED;
    ps.flags = 0;
    const size_t off = (a.used + 255) & ~size_t(255);
    Arena rest{ws.base + off, ws.cap > off ? ws.cap - off : 0, 0};
    return simt_bwd(ps, q, k, v, la, h0, dO, dhT, dq, dk, dv, dla, dh0, rest, s);
}

}  // namespace gla
