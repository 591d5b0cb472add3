// Single-token recurrent decode step:
//   S <- diag(exp(log_a)) S + k^T v   (fp32, in place),   o = q S.
// The recurrent form of the layer (podcast.app episode page "Gated Linear
// Attention for Efficient Long Sequences": a gated, recurrent-style memory
// update; the gate is G = alpha^T 1, "Gated Linear Attention Transformers with
// Hardware-Efficient Training", atlas.scime.ai summary, "Approach").
//
// The step is a pure stream over the fp32 state (read + write 8*Dk*Dv bytes
// per head), so the kernel is laid out for HBM: each thread owns four
// adjacent state columns (16-byte loads/stores, a warp covers 512 contiguous
// bytes of one state row), a block covers up to 256 columns of one head, and
// the Dk rows are split over KS row-slices whose partial q.S sums are reduced
// in shared memory.

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "gla_common.cuh"
#include "gla_internal.h"

namespace gla {
namespace {

constexpr int kStepThreads = 256;

template <typename T, int VEC>
__global__ void __launch_bounds__(kStepThreads) k_step(const T* __restrict__ q, const T* __restrict__ k,
                                                       const T* __restrict__ v, const float* __restrict__ la,
                                                       float* __restrict__ S, T* __restrict__ o, int K, int V,
                                                       int CG) {
    extern __shared__ float sm[];
    float* sq = sm;
    float* sk = sm + K;
    float* sa = sm + 2 * K;
    float* red = sm + 3 * K;  // [KS][CG*VEC]
    const int KS = kStepThreads / CG;
    const int64_t bh = blockIdx.y;
    const int tid = threadIdx.x;
    for (int c = tid; c < K; c += kStepThreads) {
        sq[c] = ldf(q + bh * K + c);
        sk[c] = ldf(k + bh * K + c);
        sa[c] = expf(la[bh * K + c]);
    }
    __syncthreads();
    const int cg = tid % CG, ks = tid / CG;
    const int col0 = (blockIdx.x * CG + cg) * VEC;
    float acc[VEC];
#pragma unroll
    for (int e = 0; e < VEC; ++e) acc[e] = 0.f;
    if (ks < KS && col0 < V) {
        float vv[VEC];
#pragma unroll
        for (int e = 0; e < VEC; ++e) vv[e] = ldf(v + bh * V + col0 + e);
        float* base = S + bh * int64_t(K) * V + col0;
        if (VEC == 4) {
#pragma unroll 4
            for (int c = ks; c < K; c += KS) {
                float4 s4 = *reinterpret_cast<const float4*>(base + int64_t(c) * V);
                const float a = sa[c], kc = sk[c], qc = sq[c];
                s4.x = a * s4.x + kc * vv[0];
                s4.y = a * s4.y + kc * vv[VEC > 1 ? 1 : 0];
                s4.z = a * s4.z + kc * vv[VEC > 2 ? 2 : 0];
                s4.w = a * s4.w + kc * vv[VEC > 3 ? 3 : 0];
                *reinterpret_cast<float4*>(base + int64_t(c) * V) = s4;
                acc[0] += qc * s4.x;
                acc[VEC > 1 ? 1 : 0] += qc * s4.y;
                acc[VEC > 2 ? 2 : 0] += qc * s4.z;
                acc[VEC > 3 ? 3 : 0] += qc * s4.w;
            }
        } else {
            for (int c = ks; c < K; c += KS) {
                float s1 = base[int64_t(c) * V];
                s1 = sa[c] * s1 + sk[c] * vv[0];
                base[int64_t(c) * V] = s1;
                acc[0] += sq[c] * s1;
            }
        }
    }
#pragma unroll
    for (int e = 0; e < VEC; ++e) red[ks * CG * VEC + cg * VEC + e] = acc[e];
    __syncthreads();
    if (ks == 0 && col0 < V) {
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
            float t = 0.f;
            for (int r = 0; r < KS; ++r) t += red[r * CG * VEC + cg * VEC + e];
            stf(o + bh * V + col0 + e, t);
        }
    }
}

template <typename T>
gla_status step_typed(const Problem& p, const T* q, const T* k, const T* v, const float* la, float* S, T* o,
                      cudaStream_t s) {
    const int K = int(p.K), V = int(p.V);
    const bool vec = (V % 4) == 0;
    const int VEC = vec ? 4 : 1;
    const int ncols = V / VEC + (vec ? 0 : 0);
    int CG = ncols < 64 ? ncols : 64;
    // a power of two that divides the block so that every row-slice is full
    int cg2 = 1;
    while (cg2 * 2 <= CG) cg2 *= 2;
    CG = cg2;
    const int KS = kStepThreads / CG;
    const size_t smem = sizeof(float) * (3 * size_t(K) + size_t(KS) * CG * VEC);
    const dim3 grid(unsigned(cdiv(ncols, CG)), unsigned(p.BH));
    if (vec) {
        if (smem > 48 * 1024 &&
            cudaFuncSetAttribute(k_step<T, 4>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) != cudaSuccess)
            return GLA_ERR_CUDA;
        GLA_LAUNCH("step", (k_step<T, 4>), grid, kStepThreads, smem, s, q, k, v, la, S, o, K, V, CG);
    } else {
        if (smem > 48 * 1024 &&
            cudaFuncSetAttribute(k_step<T, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) != cudaSuccess)
            return GLA_ERR_CUDA;
        GLA_LAUNCH("step", (k_step<T, 1>), grid, kStepThreads, smem, s, q, k, v, la, S, o, K, V, CG);
    }
    return GLA_OK;
}

}  // namespace

gla_status step_launch(const Problem& p, const void* q, const void* k, const void* v, const float* la, float* S,
                       void* o, cudaStream_t s) {
    if (p.bf16)
        return step_typed<__nv_bfloat16>(p, static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
                                         static_cast<const __nv_bfloat16*>(v), la, S, static_cast<__nv_bfloat16*>(o),
                                         s);
    return step_typed<float>(p, static_cast<const float*>(q), static_cast<const float*>(k),
                             static_cast<const float*>(v), la, S, static_cast<float*>(o), s);
}

}  // namespace gla
