// Sequence-sharded evaluation: the per-segment summary and the combine that
// joins segments evaluated on different devices.
//
// The state recurrence S_t = diag(alpha_t) S_{t-1} + k_t^T v_t is affine in
// S_{t-1}, so a segment of steps maps an entering state X to
//     X_out = diag(a) X + U,     a = prod_t alpha_t = exp(sum_t log alpha_t),
// with U the segment's end state from a zero start. Composing segments is the
// affine combine (a2, U2) o (a1, U1) = (a2 a1, diag(a2) U1 + U2), so the state
// entering segment r follows from the summaries of segments 0 .. r-1; the
// backward mirrors it with W_g, the gradient a segment sends to its entering
// state when nothing arrives at its end state: the gradient arriving at the end
// of segment r-1 is diag(a_r) (gradient arriving at the end of r) + W_r. The
// pages train with the recurrent state carried across 2K segments ("Gated Linear
// Attention Transformers with Hardware-Efficient Training", atlas.scime.ai
// summary, "Measured effects" / "Findings": truncated BPTT and length
// extrapolation); these kernels let the segments of one sequence live on
// different devices.

#include <cuda_runtime.h>

#include "gla_common.cuh"
#include "gla_gate.cuh"
#include "gla_internal.h"

namespace gla {
namespace {

constexpr int kThreads = 256;

// a[bh][c] = exp(sum over the L steps of log alpha[bh][t][c]). A block covers 32 channels of one head
// (a warp reads 32 adjacent channels of a step) and splits the steps into 8 slices, one per warp; the
// slices are added in a fixed order.
__global__ void __launch_bounds__(kThreads) k_segment_decay(GateArgs ga, float* __restrict__ a, int64_t BH,
                                                            int64_t L, int64_t K) {
    __shared__ float part[8][32];
    const int64_t bh = blockIdx.y;
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int64_t c = int64_t(blockIdx.x) * 32 + lane;
    const int64_t per = (L + 7) / 8, t_lo = w * per, t_hi = t_lo + per < L ? t_lo + per : L;
    float s = 0.f;
    if (c < K)
        for (int64_t t = t_lo; t < t_hi; ++t) s += la_floor(gate_log_alpha(ga, bh, t, c, L, K));
    part[w][lane] = s;
    __syncthreads();
    if (w == 0 && c < K) {
        float tot = 0.f;
#pragma unroll
        for (int j = 0; j < 8; ++j) tot += part[j][lane];
        a[bh * K + c] = __expf(tot);
    }
}

// out = the state entering segment r (forward) or the gradient arriving at its end (reverse);
// one thread per 4 value columns of a state row (bh, c)
__global__ void __launch_bounds__(kThreads) k_state_combine(const float* __restrict__ a, const float* __restrict__ U,
                                                            const float* __restrict__ init, float* __restrict__ out,
                                                            int64_t G, int64_t BH, int64_t K, int64_t V, int r,
                                                            int reverse) {
    const int64_t nrow4 = V / 4;
    const int64_t e = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
    if (e >= BH * K * nrow4) return;
    const int64_t row = e / nrow4;  // bh * K + c
    const int64_t stateN = BH * K * V;
    float4 x = init ? reinterpret_cast<const float4*>(init)[e] : make_float4(0.f, 0.f, 0.f, 0.f);
    if (!reverse) {
        for (int g = 0; g < r; ++g) {  // X_{g+1} = diag(a_g) X_g + U_g
            const float d = a[g * BH * K + row];
            const float4 u = reinterpret_cast<const float4*>(U + g * stateN)[e];
            x = make_float4(fmaf(d, x.x, u.x), fmaf(d, x.y, u.y), fmaf(d, x.z, u.z), fmaf(d, x.w, u.w));
        }
    } else {
        for (int g = int(G) - 1; g > r; --g) {  // Y_{g-1} = diag(a_g) Y_g + W_g
            const float d = a[g * BH * K + row];
            const float4 u = reinterpret_cast<const float4*>(U + g * stateN)[e];
            x = make_float4(fmaf(d, x.x, u.x), fmaf(d, x.y, u.y), fmaf(d, x.z, u.z), fmaf(d, x.w, u.w));
        }
    }
    reinterpret_cast<float4*>(out)[e] = x;
}

}  // namespace

gla_status segment_decay(const Problem& p, const float* log_a, float* a, cudaStream_t s) {
    const GateArgs ga{log_a, p.gate, p.inv_tau, p.H};
    GLA_LAUNCH("segment_decay", k_segment_decay, dim3(unsigned((p.K + 31) / 32), unsigned(p.BH)), kThreads, 0, s, ga, a,
               p.BH, p.L, p.K);
    return GLA_OK;
}

gla_status state_combine(int64_t G, int64_t BH, int64_t K, int64_t V, const float* a, const float* U,
                         const float* init, int r, int reverse, float* out, cudaStream_t s) {
    const int64_t n = BH * K * (V / 4);
    GLA_LAUNCH("state_combine", k_state_combine, unsigned((n + kThreads - 1) / kThreads), kThreads, 0, s, a, U, init,
               out, G, BH, K, V, r, reverse);
    return GLA_OK;
}

}  // namespace gla
