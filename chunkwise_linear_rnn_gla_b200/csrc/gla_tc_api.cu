// Tensor-core path: support check, workspace layout and kernel sequences.
//
// Forward, non-materialised states (default):
//   tc_prep      (chunk-parallel)  cumsum, Q~, K~, e^Gamma, intra-chunk P
//   tc_walk_fwd  (per head and 64 value columns) state walk kept on chip,
//                o = Q~ S + P v
// Forward, materialised states:
//   tc_prep, tc_walk_states (writes S_[i] in bf16), tc_output (chunk-parallel
//   o = Q~ S_[i] + P v from the stored states)
// Backward:
//   [tc_prep]          unless the forward's workspace is reused
//   [tc_walk_states]   unless the reused forward materialised its states
//   tc_walk_dv         reverse walk: D_i chain, dv = K~ D_i + P^T dO, writes D_i
//                      (materialised mode: tc_walk_dstates writes D_i, then the
//                      chunk-parallel tc_output_dv computes dv)
//   tc_bwd_chunk       dP = dO v^T, dQ~ = dO S_[i]^T, dK~ = v D_i^T and the
//                      intra-chunk terms on tcgen05, dq, dk, closed-form dlog a
//   [gate_grad_partials] scalar gate kinds: the gate gradient summed over channels
// Every kernel reads the caller's gate argument natively (gla_gate.cuh).

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "gla_internal.h"
#include "gla_tc.h"

namespace gla {

// The backward layout extends the forward's, so a forward workspace can be
// handed to the backward unchanged.
TcBuffers tc_carve(const Problem& p, Arena& a, bool bwd) {
    TcBuffers b{};
    b.Qt = a.take<__nv_bfloat16>(size_t(p.BH * p.L * p.K));
    b.Kt = a.take<__nv_bfloat16>(size_t(p.BH * p.L * p.K));
    b.P = a.take<__nv_bfloat16>(size_t(p.BH * p.N * kTcChunk * kTcChunk));
    b.gam = a.take<float>(size_t(p.BH * p.N * p.K));
    b.hT = a.take<float>(size_t(p.BH * p.K * p.V));
    if (bwd || p.state_mode == GLA_STATE_MATERIALIZED) b.states = a.take<__nv_bfloat16>(size_t(p.BH * p.N * p.K * p.V));
    const size_t nseg = tc_walk_seg_floats(p);
    if (nseg) b.segbuf = a.take<float>(nseg);
    if (bwd) b.Dbuf = a.take<__nv_bfloat16>(size_t(p.BH * p.N * p.K * p.V));
    if (bwd && (p.gate == GLA_GATE_SCALAR || p.gate == GLA_GATE_HEAD))
        b.gpart = a.take<float>(size_t(p.BH * p.N * (p.K / 128) * kTcChunk));
    return b;
}

namespace {

TcBuffers carve(const Problem& p, Arena& a, bool bwd) { return tc_carve(p, a, bwd); }

// Sub-chunk length 16 with a per-channel gate: the intra-chunk scores by two-level chunking (the
// scalar kinds' scores are exact decay-weighted products already).
bool two_level(const Problem& p) {
    return p.c == 16 && (p.gate == GLA_GATE_CHANNEL || p.gate == GLA_GATE_PREACT);
}

}  // namespace

bool tc_supported(const Problem& p) {
    if (!p.bf16) return false;
    if (p.C != kTcChunk || (p.c != kTcSub && p.c != 16)) return false;
    if (p.K != 128 && p.K != 256) return false;
    if (p.V < 64 || p.V % 64 != 0 || p.V / 64 > 65535) return false;
    if (p.BH > 65535 || p.N > 65535) return false;
    if (p.BH * p.N > (int64_t(1) << 31) - 1) return false;
    return true;
}

size_t tc_fwd_workspace(const Problem& p) {
    Arena a = make_arena(p, nullptr, 0);
    carve(p, a, false);
    return a.used;
}

size_t tc_bwd_workspace(const Problem& p) {
    Arena a = make_arena(p, nullptr, 0);
    carve(p, a, true);
    return a.used;
}

void tc_layout(const Problem& p, Arena& a, bool bwd) { carve(p, a, bwd); }

gla_status tc_fwd(const Problem& p, const void* q, const void* k, const void* v, const float* la, const float* h0,
                  void* o, float* hT, Arena& ws, cudaStream_t s) {
    TcBuffers b = carve(p, ws, false);
    if (ws.used > ws.cap) return GLA_ERR_WORKSPACE;
    gla_status st = tc_prep_launch(p, q, k, la, b.Qt, b.Kt, b.P, b.gam, p.gate, s);
    if (st == GLA_OK && two_level(p)) st = tc_intra_twolevel_launch(p, q, k, la, b.P, s);
    if (st != GLA_OK) return st;
    WalkArgs a{};
    a.A1 = b.Kt;
    a.B1 = static_cast<const __nv_bfloat16*>(v);
    a.A2 = b.Qt;
    a.Pm = b.P;
    a.gam = b.gam;
    a.init = h0;
    a.fin = hT;
    a.fin2 = b.hT;
    a.Y = static_cast<__nv_bfloat16*>(o);
    if (p.state_mode == GLA_STATE_NONMATERIALIZED) {
        a.mode = kWalkFused;
        // few heads, many chunks: the walk runs as parallel segments from the entering states that a
        // zero-start pass and a scan provide (the scan writes hT)
        a.seg_count = tc_walk_seg_prepare(p, b.Kt, a.B1, b.gam, h0, hT, b.hT, b.segbuf, false, s, &a.seg_len,
                                          &a.seg_init, &a.seg_stride, &st);
        if (st != GLA_OK) return st;
        return tc_walk_launch(p, a, s, "tc_walk_fwd");
    }
    a.states = b.states;
    a.mode = kWalkStatesOnly;
    st = tc_states_walk_supported(p)
             ? tc_states_walk_launch(p, b.Kt, a.B1, b.gam, h0, hT, b.hT, b.states, b.segbuf, false, s, "tc_walk_states")
             : tc_walk_launch(p, a, s, "tc_walk_states");
    if (st != GLA_OK) return st;
    return tc_chunk_out_launch(p, b.Qt, b.states, b.P, static_cast<const __nv_bfloat16*>(v), false,
                               static_cast<__nv_bfloat16*>(o), false, s, "tc_output");
}

gla_status tc_fwd_final_state(const Problem& p, const void* q, const void* k, const void* v, const float* la,
                              const float* h0, float* hT, Arena& ws, cudaStream_t s) {
    TcBuffers b = carve(p, ws, false);
    if (ws.used > ws.cap) return GLA_ERR_WORKSPACE;
    gla_status st = tc_prep_launch(p, q, k, la, b.Qt, b.Kt, b.P, b.gam, p.gate, s);
    if (st != GLA_OK) return st;
    return tc_states_walk_final(p, b.Kt, static_cast<const __nv_bfloat16*>(v), b.gam, h0, hT, b.segbuf, false, s,
                                "tc_walk_final");
}

gla_status tc_bwd_initial_grad(const Problem& p, const void* q, const void* k, const float* la, const void* dO,
                               const float* dhT, float* dh0, Arena& ws, cudaStream_t s) {
    TcBuffers b = carve(p, ws, true);
    if (ws.used > ws.cap) return GLA_ERR_WORKSPACE;
    gla_status st = tc_prep_launch(p, q, k, la, b.Qt, b.Kt, b.P, b.gam, p.gate, s);
    if (st != GLA_OK) return st;
    return tc_states_walk_final(p, b.Qt, static_cast<const __nv_bfloat16*>(dO), b.gam, dhT, dh0, b.segbuf, true, s,
                                "tc_walk_dfinal");
}

gla_status tc_bwd(const Problem& p, const void* q, const void* k, const void* v, const float* la, const float* h0,
                  const void* dO, const float* dhT, void* dq, void* dk, void* dv, float* dla, float* dh0, Arena& ws,
                  cudaStream_t s) {
    TcBuffers b = carve(p, ws, true);
    if (ws.used > ws.cap) return GLA_ERR_WORKSPACE;
    const bool reuse = (p.flags & GLA_FLAG_WS_FROM_FWD) != 0;
    gla_status st;
    if (!reuse) {
        st = tc_prep_launch(p, q, k, la, b.Qt, b.Kt, b.P, b.gam, p.gate, s);
        if (st == GLA_OK && two_level(p)) st = tc_intra_twolevel_launch(p, q, k, la, b.P, s);
        if (st != GLA_OK) return st;
    }
    if (!(reuse && p.state_mode == GLA_STATE_MATERIALIZED)) {
        WalkArgs a{};
        a.A1 = b.Kt;
        a.B1 = static_cast<const __nv_bfloat16*>(v);
        a.gam = b.gam;
        a.init = h0;
        a.fin = b.hT;
        a.states = b.states;
        a.mode = kWalkStatesOnly;
        st = tc_states_walk_supported(p)
                 ? tc_states_walk_launch(p, b.Kt, a.B1, b.gam, h0, b.hT, nullptr, b.states, b.segbuf, false, s, "tc_walk_states")
                 : tc_walk_launch(p, a, s, "tc_walk_states");
        if (st != GLA_OK) return st;
    }
    {
        // D_i chain (reverse) and dv = K~ D_i + P^T dO
        WalkArgs a{};
        a.A1 = b.Qt;
        a.B1 = static_cast<const __nv_bfloat16*>(dO);
        a.A2 = b.Kt;
        a.Pm = b.P;
        a.gam = b.gam;
        a.init = dhT;
        a.fin = dh0;
        a.Y = static_cast<__nv_bfloat16*>(dv);
        a.states = b.Dbuf;
        a.reverse = true;
        if (p.state_mode == GLA_STATE_NONMATERIALIZED) {
            a.mode = kWalkFused;
            a.p_transposed = true;
            a.seg_count = tc_walk_seg_prepare(p, b.Qt, a.B1, b.gam, dhT, dh0, nullptr, b.segbuf, true, s,
                                              &a.seg_len, &a.seg_init, &a.seg_stride, &st);
            if (st != GLA_OK) return st;
            st = tc_walk_launch(p, a, s, "tc_walk_dv");
            if (st != GLA_OK) return st;
        } else {
            a.mode = kWalkStatesOnly;
            st = tc_states_walk_supported(p) ? tc_states_walk_launch(p, b.Qt, a.B1, b.gam, dhT, dh0, nullptr, b.Dbuf,
                                                                     b.segbuf, true, s, "tc_walk_dstates")
                                             : tc_walk_launch(p, a, s, "tc_walk_dstates");
            if (st != GLA_OK) return st;
            // dv does not depend on the chunk backward, which triggers its dependents only after its
            // own wait: launched after it, the dv GEMM starts on the SMs that the backward's last
            // wave leaves idle and waits for the backward only before it exits
            st = tc_bwd_chunk_launch(p, q, k, la, dO, v, b.Qt, b.gam, b.states, b.Dbuf, dq, dk, dla, b.gpart, s);
            if (st != GLA_OK) return st;
            st = tc_chunk_out_launch(p, b.Kt, b.Dbuf, b.P, static_cast<const __nv_bfloat16*>(dO), true,
                                     static_cast<__nv_bfloat16*>(dv), true, s, "tc_output_dv");
            // the dv GEMM waits for the chunk backward before it exits: the partials are complete
            if (st == GLA_OK && b.gpart) st = tc_gate_grad_partials(p, b.gpart, dla, s);
            return st;
        }
    }
    st = tc_bwd_chunk_launch(p, q, k, la, dO, v, b.Qt, b.gam, b.states, b.Dbuf, dq, dk, dla, b.gpart, s);
    if (st == GLA_OK && b.gpart) st = tc_gate_grad_partials(p, b.gpart, dla, s);
    return st;
}

}  // namespace gla
