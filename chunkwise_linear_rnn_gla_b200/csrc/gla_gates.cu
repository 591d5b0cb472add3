// Gate kinds on the paths that work on a per-channel log alpha: the caller's
// gate argument is expanded into a per-channel log alpha [B,H,L,Dk] in the
// workspace before the pass, and the per-channel gate gradient the backward
// produces is mapped back to the caller's kind after it:
//   scalar : dL/dlog_a[b,h,t] = sum_c dL/dlog alpha[b,h,t,c]
//   head   : dL/dlog_a[h]     = sum_{b,t,c} dL/dlog alpha[b,h,t,c]
//   preact : dL/dz            = dL/dlog alpha * sigmoid(-z) / tau
// (the chain rule through log alpha[b,h,t,c] = log_a[...] broadcast, or =
// logsigmoid(z)/tau, whose derivative is sigmoid(-z)/tau).

#include <cuda_runtime.h>

#include "gla_gate.cuh"
#include "gla_internal.h"
#include "gla_tc.h"

namespace gla {
namespace {

constexpr int kThreads = 256;

unsigned grid_for(int64_t n) {
    int64_t b = (n + kThreads - 1) / kThreads;
    return unsigned(b < 1 ? 1 : b > 148 * 32 ? 148 * 32 : b);
}

__global__ void __launch_bounds__(kThreads) k_expand_gate(GateArgs ga, float* __restrict__ out, int64_t BH, int64_t L,
                                                          int64_t K) {
    const int64_t n = BH * L * K;
    for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += int64_t(gridDim.x) * blockDim.x) {
        const int64_t c = i % K, row = i / K;
        out[i] = gate_log_alpha(ga, row / L, row % L, c, L, K);
    }
}

// one warp per (head, step) row: sum over the K channels
__global__ void __launch_bounds__(kThreads) k_reduce_scalar(const float* __restrict__ dpc, float* __restrict__ dla,
                                                            int64_t rows, int64_t K) {
    const int lane = threadIdx.x & 31;
    const int64_t nwarps = int64_t(gridDim.x) * (blockDim.x / 32);
    for (int64_t row = int64_t(blockIdx.x) * (blockDim.x / 32) + threadIdx.x / 32; row < rows; row += nwarps) {
        float s = 0.f;
        for (int64_t c = lane; c < K; c += 32) s += dpc[row * K + c];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (lane == 0) dla[row] = s;
    }
}

// one block per head h: sum over every (b, t, c) of that head, in a fixed order (deterministic)
__global__ void __launch_bounds__(1024) k_reduce_head(const float* __restrict__ dpc, float* __restrict__ dla,
                                                      int64_t B, int64_t H, int64_t LK) {
    __shared__ float part[32];
    const int64_t h = blockIdx.x;
    float s = 0.f;
    for (int64_t b = 0; b < B; ++b) {
        const float* base = dpc + (b * H + h) * LK;
        for (int64_t i = threadIdx.x; i < LK; i += blockDim.x) s += base[i];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if ((threadIdx.x & 31) == 0) part[threadIdx.x / 32] = s;
    __syncthreads();
    if (threadIdx.x < 32) {
        s = threadIdx.x < blockDim.x / 32 ? part[threadIdx.x] : 0.f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (threadIdx.x == 0) dla[h] = s;
    }
}

// dL/dz = dL/dlog alpha * sigmoid(-z) / tau, in place
__global__ void __launch_bounds__(kThreads) k_preact_grad(const float* __restrict__ z, float* __restrict__ d, int64_t n,
                                                          float inv_tau) {
    for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += int64_t(gridDim.x) * blockDim.x)
        d[i] = d[i] * sigmoid_neg_f(z[i]) * inv_tau;
}

// scalar gate: dla[bh, t] = sum over the K/128 channel blocks of the backward's partials
__global__ void __launch_bounds__(kThreads) k_partials_scalar(const float* __restrict__ gp, float* __restrict__ dla,
                                                              int64_t BH, int64_t L, int64_t N, int KH) {
    const int64_t n = BH * L;
    for (int64_t e = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; e < n; e += int64_t(gridDim.x) * blockDim.x) {
        const int64_t bh = e / L, t = e % L;
        const float* g = gp + ((bh * N + t / 128) * KH) * 128 + t % 128;
        float s = 0.f;
        for (int kh = 0; kh < KH; ++kh) s += g[kh * 128];
        dla[e] = s;
    }
}

// head gate: dla[h] = sum of every partial of the heads bh with bh % H == h, in a fixed order
__global__ void __launch_bounds__(1024) k_partials_head(const float* __restrict__ gp, float* __restrict__ dla,
                                                        int64_t B, int64_t H, int64_t per_head) {
    __shared__ float part[32];
    const int64_t h = blockIdx.x;
    float s = 0.f;
    for (int64_t b = 0; b < B; ++b) {
        const float* g = gp + (b * H + h) * per_head;
        for (int64_t i = threadIdx.x; i < per_head; i += blockDim.x) s += g[i];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if ((threadIdx.x & 31) == 0) part[threadIdx.x / 32] = s;
    __syncthreads();
    if (threadIdx.x < 32) {
        s = threadIdx.x < blockDim.x / 32 ? part[threadIdx.x] : 0.f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (threadIdx.x == 0) dla[h] = s;
    }
}

}  // namespace

gla_status tc_gate_grad_partials(const Problem& p, const float* gpart, float* dla, cudaStream_t s) {
    const int KH = int(p.K / 128);
    if (p.gate == kGateScalar) {
        const int64_t n = p.BH * p.L;
        GLA_LAUNCH("gate_grad_partials", k_partials_scalar, grid_for(n), kThreads, 0, s, gpart, dla, p.BH, p.L, p.N, KH);
    } else if (p.gate == kGateHead) {
        GLA_LAUNCH("gate_grad_partials", k_partials_head, unsigned(p.H), 1024, 0, s, gpart, dla, p.B, p.H,
                   p.N * KH * int64_t(128));
    }
    return GLA_OK;
}

GateArgs gate_args(const Problem& p, const float* g) { return GateArgs{g, p.gate, p.inv_tau, p.H}; }

gla_status gate_expand(const Problem& p, const float* g, float* out, cudaStream_t s) {
    const int64_t n = p.BH * p.L * p.K;
    GLA_LAUNCH("gate_expand", k_expand_gate, grid_for(n), kThreads, 0, s, gate_args(p, g), out, p.BH, p.L, p.K);
    return GLA_OK;
}

gla_status gate_grad(const Problem& p, const float* g, const float* dpc, float* dla, cudaStream_t s) {
    if (p.gate == kGateScalar) {
        const int64_t rows = p.BH * p.L;
        const unsigned grid = unsigned((rows + 7) / 8 < 148 * 32 ? (rows + 7) / 8 : 148 * 32);
        GLA_LAUNCH("gate_grad_scalar", k_reduce_scalar, grid, kThreads, 0, s, dpc, dla, rows, p.K);
    } else if (p.gate == kGateHead) {
        GLA_LAUNCH("gate_grad_head", k_reduce_head, unsigned(p.H), 1024, 0, s, dpc, dla, p.B, p.H, p.L * p.K);
    } else if (p.gate == kGatePreact) {
        const int64_t n = p.BH * p.L * p.K;
        GLA_LAUNCH("gate_grad_preact", k_preact_grad, grid_for(n), kThreads, 0, s, g, dla, n, p.inv_tau);
    }
    return GLA_OK;
}

}  // namespace gla
