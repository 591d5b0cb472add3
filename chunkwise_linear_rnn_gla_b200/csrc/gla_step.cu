// Single-token recurrent decode step:
//   S <- diag(exp(log_a)) S + k^T v   (fp32, in place),   o = q S.
// The recurrent form of the layer (podcast.app episode page "Gated Linear
// Attention for Efficient Long Sequences", summary: a gated memory updated
// once per token; the gate is G = alpha^T 1, "Gated Linear Attention Transformers with
// Hardware-Efficient Training", atlas.scime.ai summary, "Approach").
//
// The step is a pure stream over the fp32 state (read + write 8*Dk*Dv bytes
// per head), so the kernels are laid out for HBM. The default kernel gives
// each head one block of 16 warps; a warp streams whole state rows, four at a
// time with their 16-byte loads in flight together, and o is reduced over the
// warps in shared memory. The fallback (unaligned or very wide states) gives
// each thread four adjacent state columns of a batch of rows: a block covers
// up to 128 columns of one head, and the Dk rows are split over KS row-slices
// whose partial q.S sums are reduced in shared memory.

#include <cstdint>

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "gla_common.cuh"
#include "gla_gate.cuh"
#include "gla_internal.h"

namespace gla {
namespace {

constexpr int kStepThreads = 256;
constexpr int kStepBatch = 8;  // state rows a thread has in flight

template <int VEC>
struct StepVec;
template <>
struct StepVec<4> {
    using type = float4;
    static __device__ __forceinline__ float get(const float4& x, int e) {
        return e == 0 ? x.x : e == 1 ? x.y : e == 2 ? x.z : x.w;
    }
    static __device__ __forceinline__ void set(float4& x, int e, float y) {
        if (e == 0) x.x = y;
        else if (e == 1) x.y = y;
        else if (e == 2) x.z = y;
        else x.w = y;
    }
};
template <>
struct StepVec<1> {
    using type = float;
    static __device__ __forceinline__ float get(const float& x, int) { return x; }
    static __device__ __forceinline__ void set(float& x, int, float y) { x = y; }
};

template <typename T, int VEC>
__global__ void __launch_bounds__(kStepThreads) k_step(const T* __restrict__ q, const T* __restrict__ k,
                                                       const T* __restrict__ v, GateArgs la,
                                                       float* __restrict__ S, T* __restrict__ o, int K, int V,
                                                       int CG) {
    using SV = StepVec<VEC>;
    using vec_t = typename SV::type;
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
        sa[c] = expf(gate_log_alpha(la, bh, 0, c, 1, K));
    }
    __syncthreads();
    const int cg = tid % CG, ks = tid / CG;
    const int col0 = (blockIdx.x * CG + cg) * VEC;
    float acc[VEC];
#pragma unroll
    for (int e = 0; e < VEC; ++e) acc[e] = 0.f;
    if (col0 < V) {
        float vv[VEC];
#pragma unroll
        for (int e = 0; e < VEC; ++e) vv[e] = ldf(v + bh * V + col0 + e);
        float* base = S + bh * int64_t(K) * V + col0;
        // rows ks, ks+KS, ...: a batch of kStepBatch rows is loaded before any of them is stored, so
        // that every thread keeps that many independent loads in flight
        for (int c0 = ks; c0 < K; c0 += KS * kStepBatch) {
            vec_t sv[kStepBatch];
#pragma unroll
            for (int u = 0; u < kStepBatch; ++u) {
                const int c = c0 + u * KS;
                if (c < K) sv[u] = *reinterpret_cast<const vec_t*>(base + int64_t(c) * V);
            }
#pragma unroll
            for (int u = 0; u < kStepBatch; ++u) {
                const int c = c0 + u * KS;
                if (c < K) {
                    const float a = sa[c], kc = sk[c], qc = sq[c];
#pragma unroll
                    for (int e = 0; e < VEC; ++e) {
                        const float x = a * SV::get(sv[u], e) + kc * vv[e];
                        SV::set(sv[u], e, x);
                        acc[e] += qc * x;
                    }
                    *reinterpret_cast<vec_t*>(base + int64_t(c) * V) = sv[u];
                }
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

// Row-major kernel (the default): one block of 512 threads per head; a warp takes four state rows at a
// time, their 16-byte loads issued together with the lanes spread over the columns, so that every warp
// streams whole 1 KB rows; o sums the warps' partial rows through shared memory in a fixed order.
constexpr int kRowThreads = 512;  // two blocks per SM (at most 64 registers a thread)
constexpr int kRowBatch = 4;

template <typename T>
__global__ void __launch_bounds__(kRowThreads, 2) k_step_rows(const T* __restrict__ q, const T* __restrict__ k,
                                                           const T* __restrict__ v, GateArgs la,
                                                           float* __restrict__ S, T* __restrict__ o, int K, int V) {
    extern __shared__ float sm[];
    // the arrays read as float4 first (V is a multiple of 4, so every one starts on 16 bytes), then the
    // per-row scalars
    const int nw = blockDim.x >> 5;
    float* op = sm;            // [warps][V]
    float* vs = op + nw * V;   // [V]
    float* sq = vs + V;
    float* sk = sq + K;
    float* sa = sk + K;
    const int64_t bh = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, wp = tid >> 5;
    for (int c = tid; c < K; c += blockDim.x) {
        sq[c] = ldf(q + bh * K + c);
        sk[c] = ldf(k + bh * K + c);
        sa[c] = expf(gate_log_alpha(la, bh, 0, c, 1, K));
    }
    for (int x = tid; x < V; x += blockDim.x) vs[x] = ldf(v + bh * V + x);
    for (int i = tid; i < nw * V; i += blockDim.x) op[i] = 0.f;
    __syncthreads();
    const int v4n = V / 4;
    float4* S4 = reinterpret_cast<float4*>(S + bh * int64_t(K) * V);
    const float4* v4 = reinterpret_cast<const float4*>(vs);
    float4* o4 = reinterpret_cast<float4*>(op + wp * V);
    for (int c0 = wp * kRowBatch; c0 < K; c0 += nw * kRowBatch) {
        for (int x4 = lane; x4 < v4n; x4 += 32) {
            float4 r[kRowBatch];
#pragma unroll
            for (int u = 0; u < kRowBatch; ++u)
                if (c0 + u < K) r[u] = S4[int64_t(c0 + u) * v4n + x4];
            const float4 vv = v4[x4];
            float4 acc = o4[x4];
#pragma unroll
            for (int u = 0; u < kRowBatch; ++u) {
                if (c0 + u >= K) continue;
                const float a = sa[c0 + u], kc = sk[c0 + u], qc = sq[c0 + u];
                float4 y = r[u];
                y.x = fmaf(a, y.x, kc * vv.x);
                y.y = fmaf(a, y.y, kc * vv.y);
                y.z = fmaf(a, y.z, kc * vv.z);
                y.w = fmaf(a, y.w, kc * vv.w);
                S4[int64_t(c0 + u) * v4n + x4] = y;
                acc.x = fmaf(qc, y.x, acc.x);
                acc.y = fmaf(qc, y.y, acc.y);
                acc.z = fmaf(qc, y.z, acc.z);
                acc.w = fmaf(qc, y.w, acc.w);
            }
            o4[x4] = acc;
        }
    }
    __syncthreads();
    for (int x = tid; x < V; x += blockDim.x) {
        float acc = 0.f;
        for (int w2 = 0; w2 < nw; ++w2) acc += op[w2 * V + x];
        stf(o + bh * V + x, acc);
    }
}

template <typename T>
gla_status step_typed(const Problem& p, const T* q, const T* k, const T* v, const float* g, float* S, T* o,
                      cudaStream_t s) {
    const GateArgs la{g, p.gate, p.inv_tau, p.H};
    const int K = int(p.K), V = int(p.V);
    // 16-byte state accesses need a 16-byte aligned state and rows of a multiple of 4 floats
    const bool vec = (V % 4) == 0 && (reinterpret_cast<uintptr_t>(S) & 15) == 0;
    {
        // the row-major kernel, while its per-warp partial rows fit the default shared memory
        const size_t smem = sizeof(float) * (3 * size_t(K) + size_t(V) + size_t(kRowThreads / 32) * V);
        if (vec && smem <= 48 * 1024) {
            GLA_LAUNCH("step", k_step_rows<T>, unsigned(p.BH), kRowThreads, smem, s, q, k, v, la, S, o, K, V);
            return GLA_OK;
        }
    }
    // otherwise (unaligned or very wide states) the column-sliced kernel below
    const int VEC = vec ? 4 : 1;
    const int ncols = V / VEC;
    // 32 column groups (512 bytes of a state row per warp) and 8 row-slices per block: several
    // blocks per head, so that even a small batch fills the SMs
    int CG = ncols < 32 ? ncols : 32;
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
