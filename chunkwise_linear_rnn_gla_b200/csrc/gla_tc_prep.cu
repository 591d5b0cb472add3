// Chunk-parallel preparation for the tensor-core path (bf16 inputs, C = 128,
// secondary chunk c = 16, so 8 sub-chunks per chunk).
//
// For every chunk i of every head this kernel computes, once:
//   B_j   = sum_{r<=j} log a_r          per-chunk inclusive gate cumsum (fp32)
//   Q~_j  = q_j * e^{B_j}               (bf16, operand of the inter-chunk output GEMM)
//   K~_j  = k_j * e^{Gamma - B_j}       (bf16, operand of the state-update GEMM)
//   e^Gamma                             (fp32 per key channel)
//   P_js  = sum_c q_jc k_sc e^{B_jc - B_sc} for s <= j (bf16 [128 x 128])
// P is built with two-level (secondary) chunking ("Gated Linear Attention
// Transformers with Hardware-Efficient Training", atlas.scime.ai summary,
// section "Approach": "two-level (secondary) chunking so most intra-chunk
// matmuls use half-precision tensor cores"):
//  * off-diagonal sub-chunk blocks (query sub-chunk I > key sub-chunk J) are
//    bf16 tensor-core GEMMs of gate-rescaled operands
//        P_IJ = (q_I * e^{B_I - rho_I}) (k_J * e^{last_J - B_J} * e^{rho_I - last_J})^T
//    with rho_I = B at the first row of I and last_J = B at the last row of
//    J; every factor is <= 1, so nothing overflows whatever the gates;
//  * diagonal blocks are fp32 sums on the CUDA cores,
//        P_js = sum_c (q_jc e^{B_jc - rho_I}) (k_sc e^{last_I - B_sc} e^{rho_I - last_I}),
//    and for a channel whose within-sub-chunk decay span rho_I - last_I
//    exceeds 80 (where e^{span} would leave the fp32 range) the terms are
//    computed one by one as q_jc k_sc exp(B_jc - B_sc) (log space).
// The exponentials are shared: every per-row factor is one exp of a
// non-positive log-space difference, and Q~, K~ reuse them through
// per-sub-chunk factors (e^{rho_I}, e^{Gamma - last_I}).

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "gla_common.cuh"
#include "gla_internal.h"
#include "gla_tc.h"

namespace gla {
namespace {

constexpr int C = 128;   // chunk
constexpr int SC = 16;   // sub-chunk
constexpr int NS = 8;    // sub-chunks per chunk
constexpr int KT = 32;   // key channels per tile
constexpr int QS = KT + 8;  // bf16 row stride of the mma operands (conflict-free ldmatrix)
constexpr float kUnsafeSpan = 80.f;

__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

__device__ __forceinline__ void mma_16816(float* d, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                          uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t scale_bf16x2(uint32_t v, float s0, float s1) {
    __nv_bfloat162 h = *reinterpret_cast<__nv_bfloat162*>(&v);
    float2 f = __bfloat1622float2(h);
    __nv_bfloat162 r = __floats2bfloat162_rn(f.x * s0, f.y * s1);
    return *reinterpret_cast<uint32_t*>(&r);
}

// Pair index of (I, J), J < I, in [0, 28).
__host__ __device__ constexpr int pair_index(int I, int J) { return I * (I - 1) / 2 + J; }

// cp.async 16-byte copy with zero fill when `valid` is false
__device__ __forceinline__ void cp_async16(void* dst, const void* src, bool valid) {
    const uint32_t n = valid ? 16u : 0u;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(tc_smem_u32(dst)), "l"(src), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_1() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_0() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

struct Stage {  // raw inputs of one channel tile, filled by cp.async
    float la[C][KT];
    __nv_bfloat16 q[C][KT];
    __nv_bfloat16 k[C][KT];
};

constexpr int TS = C + 4;  // row stride of the transposed fp32 operands (16-byte aligned rows)

struct PrepSmem {
    Stage st;
    float qfT[KT][TS];  // q_jc e^{B_jc - rho_I}, channel-major for vector loads
    float kfT[KT][TS];  // k_sc e^{rho_I - B_sc} (0 for channels that need the exact path)
    __nv_bfloat16 qh[C][QS];
    __nv_bfloat16 kh[C][QS];
    float tot[NS][KT];
    float d[28][KT];
    unsigned unsafe_mask[NS];
};

// One CTA per (chunk, head), 8 warps; warp I owns query sub-chunk I. Two CTAs
// fit per SM so one CTA's loads overlap the other's arithmetic.
__global__ void __launch_bounds__(256, 2) k_tc_prep(const __nv_bfloat16* __restrict__ q,
                                                    const __nv_bfloat16* __restrict__ k,
                                                    const float* __restrict__ la, __nv_bfloat16* __restrict__ Qt,
                                                    __nv_bfloat16* __restrict__ Kt, __nv_bfloat16* __restrict__ P,
                                                    float* __restrict__ gam, float* __restrict__ Bout, int64_t L,
                                                    int64_t K, int64_t N) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    PrepSmem& sm = *reinterpret_cast<PrepSmem*>(smem_raw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t i = blockIdx.x, bh = blockIdx.y;
    const int64_t t0 = i * C;
    const int nvalid = int(L - t0 < C ? L - t0 : C);

    // off-diagonal accumulators: warp I owns query sub-chunk I, key blocks J < I
    float acc[NS - 1][2][4];
#pragma unroll
    for (int J = 0; J < NS - 1; ++J)
#pragma unroll
        for (int nb = 0; nb < 2; ++nb)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[J][nb][e] = 0.f;
    // diagonal accumulators: rows jr0, jr0+1; cols s0..s0+3 of block (I,I)
    float dg[2][4];
#pragma unroll
    for (int a = 0; a < 2; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) dg[a][b] = 0.f;
    const int I = warp;
    const int jr0 = 2 * (lane >> 2), s0 = 4 * (lane & 3);

    for (int64_t c0 = 0; c0 < K; c0 += KT) {
        // ---- stage the raw tile [128 rows x 32 channels]
        {
            Stage& S = sm.st;
            for (int e = tid; e < C * (KT / 4); e += 256) {  // log a: 8 x 16 B per row
                const int row = e / (KT / 4), cc = (e % (KT / 4)) * 4;
                const bool ok = row < nvalid;
                cp_async16(&S.la[row][cc], la + (bh * L + t0 + (ok ? row : 0)) * K + c0 + cc, ok);
            }
            for (int e = tid; e < C * (KT / 8); e += 256) {  // q, k: 4 x 16 B per row
                const int row = e / (KT / 8), cc = (e % (KT / 8)) * 8;
                const bool ok = row < nvalid;
                const int64_t off = (bh * L + t0 + (ok ? row : 0)) * K + c0 + cc;
                cp_async16(&S.q[row][cc], q + off, ok);
                cp_async16(&S.k[row][cc], k + off, ok);
            }
            cp_async_commit();
            cp_async_wait_0();
        }
        __syncthreads();
        const Stage& S = sm.st;
        // ---- phase 1: thread (channel cl, sub-chunk I) cumsum, factors, operands
        const int cl = lane;
        const int64_t ch = c0 + cl;
        float b[SC];
        float run = 0.f;
#pragma unroll
        for (int r = 0; r < SC; ++r) {
            run += S.la[I * SC + r][cl];
            b[r] = run;
        }
        sm.tot[I][cl] = run;
        if (tid < NS) sm.unsafe_mask[tid] = 0u;
        __syncthreads();
        float pre = 0.f, gamma = 0.f;
#pragma unroll
        for (int J = 0; J < NS; ++J) {
            const float t = sm.tot[J][cl];
            if (J < I) pre += t;
            gamma += t;
        }
        const float rho = pre + b[0];
        const float last = pre + b[SC - 1];
        // exponents are <= 0 in exact arithmetic; the clamps absorb cumsum rounding
        const float eRho = __expf(fminf(rho, 0.f));           // <= 1
        const float eGl = __expf(fminf(gamma - last, 0.f));    // <= 1
        const float span = fmaxf(rho - last, 0.f);             // >= 0
        const bool unsafe = span > kUnsafeSpan;
        const float eSpan = unsafe ? 0.f : __expf(span);
        if (unsafe) atomicOr(&sm.unsafe_mask[I], 1u << cl);
        // pair factors e^{rho_I - last_J} for J < I (last_J = cumsum through sub-chunk J)
        {
            float lastJ = 0.f;
#pragma unroll
            for (int J = 0; J < NS - 1; ++J) {
                lastJ += sm.tot[J][cl];
                if (J < I) sm.d[pair_index(I, J)][cl] = __expf(fminf(rho - lastJ, 0.f));
            }
        }
        if (I == 0 && gam) gam[(bh * N + i) * K + ch] = __expf(fminf(gamma, 0.f));
#pragma unroll
        for (int r = 0; r < SC; ++r) {
            const int row = I * SC + r;
            const float B = pre + b[r];
            const float qv = __bfloat162float(S.q[row][cl]);
            const float kv = __bfloat162float(S.k[row][cl]);
            const float a = __expf(fminf(B - rho, 0.f));     // e^{B_j - rho_I} <= 1
            const float kfac = __expf(fminf(last - B, 0.f)); // e^{last_I - B_j} <= 1
            const float qhat = qv * a;
            const float khat = kv * kfac;
            sm.qh[row][cl] = __float2bfloat16_rn(qhat);
            sm.kh[row][cl] = __float2bfloat16_rn(khat);
            sm.qfT[cl][row] = qhat;
            sm.kfT[cl][row] = unsafe ? 0.f : khat * eSpan;
            if (row < nvalid) {
                const int64_t off = (bh * L + t0 + row) * K + ch;
                Qt[off] = __float2bfloat16_rn(qhat * eRho);
                Kt[off] = __float2bfloat16_rn(khat * eGl);
                if (Bout) Bout[off] = B;
            }
        }
        __syncthreads();

        // ---- phase 2a: off-diagonal blocks on the tensor cores
#pragma unroll
        for (int ks = 0; ks < KT / 16; ++ks) {
            uint32_t a0, a1, a2, a3;
            {
                const int row = I * SC + (lane & 15);
                const int col = ks * 16 + (lane >> 4) * 8;
                ldmatrix_x4(tc_smem_u32(&sm.qh[row][col]), a0, a1, a2, a3);
            }
            const int t = lane & 3;
            const int ca = ks * 16 + 2 * t, cb = ks * 16 + 8 + 2 * t;
#pragma unroll
            for (int J = 0; J < NS - 1; ++J) {
                if (J < I) {
                    uint32_t b0, b1, b2, b3;
                    const int row = J * SC + (lane & 7) + ((lane >> 4) << 3);
                    const int col = ks * 16 + ((lane >> 3) & 1) * 8;
                    ldmatrix_x4(tc_smem_u32(&sm.kh[row][col]), b0, b1, b2, b3);
                    const float* dd = sm.d[pair_index(I, J)];
                    const float dA = dd[ca], dB = dd[ca + 1], dC = dd[cb], dD = dd[cb + 1];
                    b0 = scale_bf16x2(b0, dA, dB);
                    b1 = scale_bf16x2(b1, dC, dD);
                    b2 = scale_bf16x2(b2, dA, dB);
                    b3 = scale_bf16x2(b3, dC, dD);
                    mma_16816(acc[J][0], a0, a1, a2, a3, b0, b1);
                    mma_16816(acc[J][1], a0, a1, a2, a3, b2, b3);
                }
            }
        }
        // ---- phase 2b: diagonal block (I,I) in fp32 on the CUDA cores
#pragma unroll 8
        for (int c = 0; c < KT; ++c) {
            const float2 qa = *reinterpret_cast<const float2*>(&sm.qfT[c][I * SC + jr0]);
            const float4 kb = *reinterpret_cast<const float4*>(&sm.kfT[c][I * SC + s0]);
            dg[0][0] = fmaf(qa.x, kb.x, dg[0][0]);
            dg[0][1] = fmaf(qa.x, kb.y, dg[0][1]);
            dg[0][2] = fmaf(qa.x, kb.z, dg[0][2]);
            dg[0][3] = fmaf(qa.x, kb.w, dg[0][3]);
            dg[1][0] = fmaf(qa.y, kb.x, dg[1][0]);
            dg[1][1] = fmaf(qa.y, kb.y, dg[1][1]);
            dg[1][2] = fmaf(qa.y, kb.z, dg[1][2]);
            dg[1][3] = fmaf(qa.y, kb.w, dg[1][3]);
        }
        const unsigned um = sm.unsafe_mask[I];
        if (um) {  // rare: channels whose decay span inside the sub-chunk leaves the fp32 range
            for (int c = 0; c < KT; ++c) {
                if (!((um >> c) & 1u)) continue;
                // per-chunk cumsum of this channel, recomputed from the staged gates
                float Bj[SC];
                float run2 = 0.f;
                for (int r = 0; r < I * SC; ++r) run2 += S.la[r][c];
                for (int r = 0; r < SC; ++r) {
                    run2 += S.la[I * SC + r][c];
                    Bj[r] = run2;
                }
#pragma unroll
                for (int a = 0; a < 2; ++a) {
                    const int jr = jr0 + a;
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int sr = s0 + e;
                        if (sr > jr) continue;
                        const float qv = __bfloat162float(S.q[I * SC + jr][c]);
                        const float kv = __bfloat162float(S.k[I * SC + sr][c]);
                        dg[a][e] += qv * kv * expf(fminf(Bj[jr] - Bj[sr], 0.f));
                    }
                }
            }
        }
        __syncthreads();
    }
    // ---- write P (bf16, [128 x 128], zero above the diagonal)
    __nv_bfloat16* Pc = P + (bh * N + i) * C * C;
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int J = 0; J < NS - 1; ++J) {
        if (J < I) {
#pragma unroll
            for (int nb = 0; nb < 2; ++nb) {
                const int col = J * SC + nb * 8 + 2 * t;
                const int r0 = I * SC + g;
                *reinterpret_cast<uint32_t*>(&Pc[r0 * C + col]) = tc::pack_bf16x2(acc[J][nb][0], acc[J][nb][1]);
                *reinterpret_cast<uint32_t*>(&Pc[(r0 + 8) * C + col]) =
                    tc::pack_bf16x2(acc[J][nb][2], acc[J][nb][3]);
            }
        }
    }
#pragma unroll
    for (int a = 0; a < 2; ++a) {
        const int jrel = jr0 + a;
        float v[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) v[e] = (s0 + e <= jrel) ? dg[a][e] : 0.f;
        const int row = I * SC + jrel;
        *reinterpret_cast<uint32_t*>(&Pc[row * C + I * SC + s0]) = tc::pack_bf16x2(v[0], v[1]);
        *reinterpret_cast<uint32_t*>(&Pc[row * C + I * SC + s0 + 2]) = tc::pack_bf16x2(v[2], v[3]);
    }
    // zero blocks right of the diagonal: row block I, columns (I+1)*16 .. 127
    const int zc0 = (I + 1) * SC;
    for (int e = lane; e < SC * (C - zc0) / 2; e += 32) {
        const int r = e / ((C - zc0) / 2), cc = zc0 + 2 * (e % ((C - zc0) / 2));
        *reinterpret_cast<uint32_t*>(&Pc[(I * SC + r) * C + cc]) = 0u;
    }
}

}  // namespace

size_t tc_prep_smem_bytes() { return sizeof(PrepSmem); }

gla_status tc_prep_launch(const Problem& p, const void* q, const void* k, const float* la, __nv_bfloat16* Qt,
                          __nv_bfloat16* Kt, __nv_bfloat16* P, float* gam, float* Bout, cudaStream_t s) {
    const size_t sm = sizeof(PrepSmem);
    if (cudaFuncSetAttribute(k_tc_prep, cudaFuncAttributeMaxDynamicSharedMemorySize, int(sm)) != cudaSuccess)
        return GLA_ERR_CUDA;
    GLA_LAUNCH("tc_prep", k_tc_prep, dim3(unsigned(p.N), unsigned(p.BH)), 256, sm, s,
               static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k), la, Qt, Kt, P, gam, Bout,
               p.L, p.K, p.N);
    return GLA_OK;
}

}  // namespace gla
