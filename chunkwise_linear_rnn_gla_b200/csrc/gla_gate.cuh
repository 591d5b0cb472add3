// Gate kinds (gla_gate in include/gla.h): how the `log_a` argument maps to the
// per-key-channel log decay log alpha_t[c] that every kernel of the layer uses.
//   channel: log_a[b,h,t,c]           scalar: log_a[b,h,t] for every c
//   head:    log_a[h] for every b,t,c preact: logsigmoid(z[b,h,t,c]) / tau
// The coarser kinds are the decays the pages' ablations compare with the
// per-channel gate ("Gated Linear Attention Transformers with Hardware-
// Efficient Training", atlas.scime.ai summary, "Measured effects"); preact is
// the data-dependent gate applied to its argument inside the kernels
// ("Approach").
#pragma once

#include <cuda_runtime.h>
#include <cstdint>

namespace gla {

enum GateKind : int { kGateChannel = 0, kGateScalar = 1, kGateHead = 2, kGatePreact = 3 };

// log(sigmoid(z)) = min(z, 0) - log(1 + e^{-|z|}): both terms are bounded, so nothing overflows.
__device__ __forceinline__ float logsigmoid_f(float z) { return fminf(z, 0.f) - log1pf(__expf(-fabsf(z))); }

// sigmoid(-z) = 1 / (1 + e^z); e^z may overflow to +inf for large z, giving exactly 0.
__device__ __forceinline__ float sigmoid_neg_f(float z) { return 1.f / (1.f + __expf(z)); }

struct GateArgs {
    const float* g;  // the log_a argument as the caller passed it
    int kind;        // GateKind
    float inv_tau;   // preact: 1 / tau
    int64_t H;       // heads (head kind: g is indexed by bh % H)
};

// log alpha of head bh, step t, key channel c (L steps, K channels per head)
__device__ __forceinline__ float gate_log_alpha(const GateArgs& ga, int64_t bh, int64_t t, int64_t c, int64_t L,
                                                int64_t K) {
    switch (ga.kind) {
        case kGateScalar: return ga.g[bh * L + t];
        case kGateHead: return ga.g[bh % ga.H];
        case kGatePreact: return logsigmoid_f(ga.g[(bh * L + t) * K + c]) * ga.inv_tau;
        default: return ga.g[(bh * L + t) * K + c];
    }
}

}  // namespace gla
