// Tensor-core backward, chunk-parallel part.
//
// With D_i = dL/dS_[i+1] (written in bf16 by the reverse state walk that also
// produces dv) and the forward states S_[i], the backward of chunk i is
// ("Gated Linear Attention Transformers with Hardware-Efficient Training",
// atlas.scime.ai summary, "Approach": chunkwise form and the closed-form
// gate gradient):
//   dP_js  = dO_j . v_s  (s <= j)
//   dq_j   = e^{B_j} * (dO_j S_[i]^T) + sum_{s<=j} dP_js k_s e^{B_j - B_s}
//   dk_s   = e^{Gamma - B_s} * (v_s D_i^T) + sum_{j>=s} dP_js q_j e^{B_j - B_s}
//   dlog a_t = sum_{s>=t} (q_s dq_s - k_s dk_s) + sum_v dhT * hT
// k_bwd_gemm computes the three value-dimension contractions dP, dQ~ = dO S^T
// and dK~ = V D^T on tcgen05 (one CTA per chunk and 128 key channels);
// k_bwd_intra adds the intra-chunk terms with the same two-level chunking as
// the forward (off-diagonal 16x16 blocks on bf16 tensor cores with
// gate-rescaled operands, diagonal blocks in fp32), combines, and evaluates
// the gate gradient. Its reverse cumsum needs, for every chunk, the sum over
// all later chunks; that carry is exact and local:
//   sum_{s >= (i+1)C} r_s + sum_v dhT*hT = sum_v D_i[c,v] S_[i+1][c,v]
// (the gate gradient at the first row of chunk i+1 is the future-only
// gradient of the boundary state times the state), with S_[N] = hT and
// D_{N-1} = dhT for the last chunk.

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstring>

#include "gla_common.cuh"
#include "gla_internal.h"
#include "gla_tc.h"
#include "tc_host.h"

namespace gla {
namespace {

using namespace tc;

constexpr int C = kTcChunk;
constexpr uint32_t PIECE = 16384;
constexpr int NSTAGE = 3;  // each stage: dO, v, S, D pieces for 64 value columns

struct GemmBars {
    uint64_t full[NSTAGE], empty[NSTAGE], done;
    uint32_t tmem_slot;
    int abort_flag;
};

__global__ void __launch_bounds__(192, 1)
    k_bwd_gemm(const __grid_constant__ CUtensorMap tmDO, const __grid_constant__ CUtensorMap tmV,
               const __grid_constant__ CUtensorMap tmS, const __grid_constant__ CUtensorMap tmD,
               __nv_bfloat16* __restrict__ dP, __nv_bfloat16* __restrict__ dQt, __nv_bfloat16* __restrict__ dKt,
               int64_t L, int64_t N, int64_t K, int64_t V, int* err) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    GemmBars& bar = *reinterpret_cast<GemmBars*>(base + NSTAGE * 4 * PIECE);
    volatile int* abort_flag = &bar.abort_flag;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int i = blockIdx.x, kh = blockIdx.y;
    const int64_t bh = blockIdx.z;
    const int nvb = int(V / 64);
    if (threadIdx.x == 0) {
        for (int s = 0; s < NSTAGE; ++s) {
            mbar_init(&bar.full[s], 1);
            mbar_init(&bar.empty[s], 1);
        }
        mbar_init(&bar.done, 1);
        bar.abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(&bar.tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bar.tmem_slot;  // cols: dP [0,128), dQ~ [128,256), dK~ [256,384)
    if (warp == 0) {
        if (lane == 0) {
            bool ok = true;
            int vb = 0;
            for (; vb < nvb && ok; ++vb) {
                const int s = vb % NSTAGE;
                const uint32_t u = uint32_t(vb / NSTAGE);
                if (!mbar_wait(&bar.empty[s], (u & 1u) ^ 1u, err, abort_flag)) {
                    ok = false;
                    break;
                }
                uint8_t* st = base + s * 4 * PIECE;
                mbar_arrive_expect_tx(&bar.full[s], 4 * PIECE);
                tma_load_3d(st, &tmDO, 64 * vb, i * C, int(bh), &bar.full[s]);
                tma_load_3d(st + PIECE, &tmV, 64 * vb, i * C, int(bh), &bar.full[s]);
                tma_load_3d(st + 2 * PIECE, &tmS, 64 * vb, 128 * kh, int(bh * N + i), &bar.full[s]);
                tma_load_3d(st + 3 * PIECE, &tmD, 64 * vb, 128 * kh, int(bh * N + i), &bar.full[s]);
            }
            if (!ok)  // drain the loads already issued
                for (int w = vb - NSTAGE; w < vb; ++w)
                    if (w >= 0) mbar_wait(&bar.full[w % NSTAGE], uint32_t((w / NSTAGE) & 1), nullptr, abort_flag);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t id = idesc_bf16_f32(128, 128, false, false);
            bool ok = true;
            for (int vb = 0; vb < nvb && ok; ++vb) {
                const int s = vb % NSTAGE;
                ok = mbar_wait(&bar.full[s], uint32_t((vb / NSTAGE) & 1), err, abort_flag);
                if (!ok) break;
                tc_fence_after();
                const uint32_t st = smem_u32(base + s * 4 * PIECE);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const uint32_t acc = (vb > 0 || kk > 0) ? 1u : 0u;
                    const uint64_t aO = sdesc_sw128(st + kk * 32, 16, 1024);
                    const uint64_t aV = sdesc_sw128(st + PIECE + kk * 32, 16, 1024);
                    const uint64_t bS = sdesc_sw128(st + 2 * PIECE + kk * 32, 16, 1024);
                    const uint64_t bD = sdesc_sw128(st + 3 * PIECE + kk * 32, 16, 1024);
                    mma_bf16(tmem + 0, aO, aV, id, acc);    // dP  = dO v^T
                    mma_bf16(tmem + 128, aO, bS, id, acc);  // dQ~ = dO S^T
                    mma_bf16(tmem + 256, aV, bD, id, acc);  // dK~ = v D^T
                }
                mma_commit(&bar.empty[s]);
            }
            mma_commit(&bar.done);
            if (!ok) mbar_wait(&bar.done, 0, nullptr, abort_flag, 4000000000LL);
        }
    } else {
        const int q = warp & 3;
        const int r = 32 * q + lane;
        const uint32_t lane_off = uint32_t(32 * q) << 16;
        if (mbar_wait(&bar.done, 0, err, abort_flag)) {
            tc_fence_after();
            const int64_t t = int64_t(i) * C + r;
            for (int part = 0; part < 3; ++part) {
                if (part == 0 && kh != 0) continue;  // dP is written once per chunk
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    float y[64];
#pragma unroll
                    for (int c16 = 0; c16 < 4; ++c16)
                        tmem_ld16(tmem + lane_off + uint32_t(128 * part + 64 * half + 16 * c16), y + 16 * c16);
                    tmem_wait_ld();
                    uint4* dst;
                    if (part == 0) {
                        dst = reinterpret_cast<uint4*>(dP + ((bh * N + i) * C + r) * C + 64 * half);
                    } else {
                        if (t >= L) continue;
                        __nv_bfloat16* basep = part == 1 ? dQt : dKt;
                        dst = reinterpret_cast<uint4*>(basep + (bh * L + t) * K + 128 * kh + 64 * half);
                    }
#pragma unroll
                    for (int ch = 0; ch < 8; ++ch)
                        dst[ch] = make_uint4(pack_bf16x2(y[8 * ch], y[8 * ch + 1]), pack_bf16x2(y[8 * ch + 2], y[8 * ch + 3]),
                                             pack_bf16x2(y[8 * ch + 4], y[8 * ch + 5]),
                                             pack_bf16x2(y[8 * ch + 6], y[8 * ch + 7]));
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ---------------------------------------------------------------------------
// Intra-chunk gradients, combine and closed-form gate gradient.
constexpr int SC = kTcSub, NS = C / SC, KT = 32;
constexpr int DPS = C + 8;   // bf16 row stride of dP in smem
constexpr int QS = KT + 8;   // bf16 row stride of the rescaled operands
constexpr float kUnsafeSpan = 80.f;

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t* r) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t* r) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
__device__ __forceinline__ void mma16816(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t scale2(uint32_t v, float s) {
    __nv_bfloat162 h = *reinterpret_cast<__nv_bfloat162*>(&v);
    float2 f = __bfloat1622float2(h);
    __nv_bfloat162 o = __floats2bfloat162_rn(f.x * s, f.y * s);
    return *reinterpret_cast<uint32_t*>(&o);
}
__host__ __device__ constexpr int pidx(int I, int J) { return I * (I - 1) / 2 + J; }

struct IntraSmem {
    __nv_bfloat16 dP[C][DPS];
    float la[C][KT];
    __nv_bfloat16 q[C][KT], k[C][KT], dQt[C][KT], dKt[C][KT];
    float B[C][KT];
    float a[C][KT + 1], kf[C][KT + 1];      // e^{B_j - rho_I}, e^{last_I - B_j}
    float qf[C][KT + 1], kfD[C][KT + 1];    // fp32 operands of the diagonal blocks
    __nv_bfloat16 qh[C][QS], kh[C][QS];     // bf16 operands of the off-diagonal blocks
    float iq[C][KT + 1], ik[C][KT + 1];     // intra results
    float d[28][KT];
    float tot[NS][KT];
    float EI[NS][KT], FI[NS][KT];
    float carry[KT];
    unsigned unsafe_mask[NS];
};

__global__ void __launch_bounds__(256, 1)
    k_bwd_intra(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                const float* __restrict__ la, const __nv_bfloat16* __restrict__ dPg,
                const __nv_bfloat16* __restrict__ dQt, const __nv_bfloat16* __restrict__ dKt,
                const __nv_bfloat16* __restrict__ Sbuf, const __nv_bfloat16* __restrict__ Dbuf,
                const float* __restrict__ hT, const float* __restrict__ dhT, __nv_bfloat16* __restrict__ dq,
                __nv_bfloat16* __restrict__ dk, float* __restrict__ dla, int64_t L, int64_t N, int64_t K, int64_t V) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    IntraSmem& sm = *reinterpret_cast<IntraSmem*>(smem_raw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t i = blockIdx.x, bh = blockIdx.y;
    const int64_t t0 = i * C;
    const int nvalid = int(L - t0 < C ? L - t0 : C);
    const int g = lane >> 2, tq = lane & 3;

    // dP of this chunk (bf16, zero above the diagonal) -> smem
    for (int e = tid; e < C * C / 8; e += 256) {
        const int row = e / (C / 8), cc = (e % (C / 8)) * 8;
        *reinterpret_cast<uint4*>(&sm.dP[row][cc]) =
            *reinterpret_cast<const uint4*>(dPg + ((bh * N + i) * C + row) * C + cc);
    }

    for (int64_t c0 = 0; c0 < K; c0 += KT) {
        __syncthreads();
        // ---- stage the raw tile
        for (int e = tid; e < C * KT; e += 256) {
            const int row = e / KT, cc = e % KT;
            const bool ok = row < nvalid;
            const int64_t off = (bh * L + t0 + row) * K + c0 + cc;
            sm.la[row][cc] = ok ? la[off] : 0.f;
            sm.q[row][cc] = ok ? q[off] : __float2bfloat16_rn(0.f);
            sm.k[row][cc] = ok ? k[off] : __float2bfloat16_rn(0.f);
            sm.dQt[row][cc] = ok ? dQt[off] : __float2bfloat16_rn(0.f);
            sm.dKt[row][cc] = ok ? dKt[off] : __float2bfloat16_rn(0.f);
        }
        // ---- carry into this chunk from all later chunks: sum_v D_i * S_[i+1]
        {
            const int cl = tid >> 3, part = tid & 7;  // 32 channels x 8 threads
            const int64_t ch = c0 + cl;
            float acc = 0.f;
            if (i + 1 < N) {
                const __nv_bfloat16* Dr = Dbuf + ((bh * N + i) * K + ch) * V;
                const __nv_bfloat16* Sr = Sbuf + ((bh * N + i + 1) * K + ch) * V;
                for (int64_t v = part * 8; v < V; v += 64) {
                    const uint4 dv4 = *reinterpret_cast<const uint4*>(Dr + v);
                    const uint4 sv4 = *reinterpret_cast<const uint4*>(Sr + v);
                    const __nv_bfloat162* d2 = reinterpret_cast<const __nv_bfloat162*>(&dv4);
                    const __nv_bfloat162* s2 = reinterpret_cast<const __nv_bfloat162*>(&sv4);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 a = __bfloat1622float2(d2[e]), b = __bfloat1622float2(s2[e]);
                        acc += a.x * b.x + a.y * b.y;
                    }
                }
            } else if (dhT) {
                const float* Dr = dhT + (bh * K + ch) * V;
                const float* Sr = hT + (bh * K + ch) * V;
                for (int64_t v = part; v < V; v += 8) acc += Dr[v] * Sr[v];
            }
            acc += __shfl_xor_sync(0xffffffffu, acc, 1);
            acc += __shfl_xor_sync(0xffffffffu, acc, 2);
            acc += __shfl_xor_sync(0xffffffffu, acc, 4);
            if (part == 0) sm.carry[cl] = acc;
        }
        __syncthreads();
        // ---- phase 1: thread (channel cl, sub-chunk I): cumsum, factors, operands
        const int cl = lane, I = warp;
        float b[SC];
        float run = 0.f;
#pragma unroll
        for (int r = 0; r < SC; ++r) {
            run += sm.la[I * SC + r][cl];
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
        const float rho = pre + b[0], last = pre + b[SC - 1];
        const float span = rho - last;
        const bool unsafe = span > kUnsafeSpan;
        const float eSpan = unsafe ? 0.f : __expf(span);
        if (unsafe) atomicOr(&sm.unsafe_mask[I], 1u << cl);
        sm.EI[I][cl] = __expf(rho);
        sm.FI[I][cl] = __expf(gamma - last);
        {
            float lastJ = 0.f;
#pragma unroll
            for (int J = 0; J < NS - 1; ++J) {
                lastJ += sm.tot[J][cl];
                if (J < I) sm.d[pidx(I, J)][cl] = __expf(rho - lastJ);
            }
        }
#pragma unroll
        for (int r = 0; r < SC; ++r) {
            const int row = I * SC + r;
            const float Bv = pre + b[r];
            sm.B[row][cl] = Bv;
            const float av = __expf(Bv - rho), kv = __expf(last - Bv);
            const float qhat = __bfloat162float(sm.q[row][cl]) * av;
            const float khat = __bfloat162float(sm.k[row][cl]) * kv;
            sm.a[row][cl] = av;
            sm.kf[row][cl] = kv;
            sm.qf[row][cl] = qhat;
            sm.kfD[row][cl] = unsafe ? 0.f : khat * eSpan;
            sm.qh[row][cl] = __float2bfloat16_rn(qhat);
            sm.kh[row][cl] = __float2bfloat16_rn(khat);
        }
        __syncthreads();
        // ---- phase 2a: off-diagonal blocks, warp I: dq rows of sub-chunk I, dk rows of sub-chunk I
        {
            float aq[4][4], ak[4][4];
#pragma unroll
            for (int n = 0; n < 4; ++n)
#pragma unroll
                for (int e = 0; e < 4; ++e) aq[n][e] = ak[n][e] = 0.f;
            // dq_I += sum_{J<I} dP_IJ (K^_J * d_IJ)     (K^_J = k e^{last_J - B})
            for (int J = 0; J < I; ++J) {
                uint32_t A[4];
                ldsm_x4(tc_smem_u32(&sm.dP[I * SC + (lane & 15)][J * SC + (lane >> 4) * 8]), A);
                const float* dd = sm.d[pidx(I, J)];
#pragma unroll
                for (int nb2 = 0; nb2 < 2; ++nb2) {  // pairs of 8-channel blocks
                    uint32_t Bf[4];
                    const int row = J * SC + (lane & 7) + ((lane >> 3) & 1) * 8;
                    const int col = nb2 * 16 + (lane >> 4) * 8;
                    ldsm_x4_t(tc_smem_u32(&sm.kh[row][col]), Bf);
                    const float f0 = dd[nb2 * 16 + g], f1 = dd[nb2 * 16 + 8 + g];
                    mma16816(aq[2 * nb2], A, scale2(Bf[0], f0), scale2(Bf[1], f0));
                    mma16816(aq[2 * nb2 + 1], A, scale2(Bf[2], f1), scale2(Bf[3], f1));
                }
            }
            // dk_J += sum_{I>J} dP_IJ^T (Q^_I * d_IJ), here J = warp
            const int J = warp;
            for (int I2 = J + 1; I2 < NS; ++I2) {
                uint32_t A[4];
                ldsm_x4_t(tc_smem_u32(&sm.dP[I2 * SC + (lane & 7) + (lane >> 4) * 8][J * SC + ((lane >> 3) & 1) * 8]), A);
                const float* dd = sm.d[pidx(I2, J)];
#pragma unroll
                for (int nb2 = 0; nb2 < 2; ++nb2) {
                    uint32_t Bf[4];
                    const int row = I2 * SC + (lane & 7) + ((lane >> 3) & 1) * 8;
                    const int col = nb2 * 16 + (lane >> 4) * 8;
                    ldsm_x4_t(tc_smem_u32(&sm.qh[row][col]), Bf);
                    const float f0 = dd[nb2 * 16 + g], f1 = dd[nb2 * 16 + 8 + g];
                    mma16816(ak[2 * nb2], A, scale2(Bf[0], f0), scale2(Bf[1], f0));
                    mma16816(ak[2 * nb2 + 1], A, scale2(Bf[2], f1), scale2(Bf[3], f1));
                }
            }
            // scale by the row factors and park in smem (fragment layout -> [row][channel])
#pragma unroll
            for (int n = 0; n < 4; ++n) {
                const int c = n * 8 + 2 * tq;
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int row = warp * SC + g + 8 * hh;
                    sm.iq[row][c] = aq[n][2 * hh] * sm.a[row][c];
                    sm.iq[row][c + 1] = aq[n][2 * hh + 1] * sm.a[row][c + 1];
                    sm.ik[row][c] = ak[n][2 * hh] * sm.kf[row][c];
                    sm.ik[row][c + 1] = ak[n][2 * hh + 1] * sm.kf[row][c + 1];
                }
            }
        }
        __syncwarp();
        // ---- phase 2b: diagonal block of sub-chunk I in fp32 (lane = channel)
        {
            const int c = lane, I2 = warp;
            const unsigned um = sm.unsafe_mask[I2];
            const bool exact = (um >> c) & 1u;
            for (int jr = 0; jr < SC; ++jr) {
                const int j = I2 * SC + jr;
                float sq_ = 0.f, sk_ = 0.f;
                for (int sr = 0; sr <= jr; ++sr) {  // dq_j += sum_{s<=j} dP_js k_s e^{B_j-B_s}
                    const int s = I2 * SC + sr;
                    const float w = __bfloat162float(sm.dP[j][s]);
                    if (!exact) sq_ += w * sm.kfD[s][c];
                    else sq_ += w * __bfloat162float(sm.k[s][c]) * expf(sm.B[j][c] - sm.B[s][c]);
                }
                for (int sr = jr; sr < SC; ++sr) {  // dk_j += sum_{s'>=j} dP_{s'j} q_s' e^{B_s'-B_j}
                    const int s = I2 * SC + sr;
                    const float w = __bfloat162float(sm.dP[s][j]);
                    if (!exact) sk_ += w * sm.qf[s][c];
                    else sk_ += w * __bfloat162float(sm.q[s][c]) * expf(sm.B[s][c] - sm.B[j][c]);
                }
                if (!exact) {
                    sq_ *= sm.a[j][c];
                    // e^{B_s' - B_j} = a_s' * D_I * kf_j
                    sk_ *= sm.kf[j][c] * eSpan;
                }
                sm.iq[j][c] += sq_;
                sm.ik[j][c] += sk_;
            }
        }
        __syncthreads();
        // ---- combine, gate gradient (thread: channel cl, rows of sub-chunk I)
        {
            const float E = sm.EI[I][cl], F = sm.FI[I][cl];
            float rr[SC];
            float rs = 0.f;
            const int64_t ch = c0 + cl;
#pragma unroll
            for (int r = 0; r < SC; ++r) {
                const int row = I * SC + r;
                const float dqv = sm.a[row][cl] * E * __bfloat162float(sm.dQt[row][cl]) + sm.iq[row][cl];
                const float dkv = sm.kf[row][cl] * F * __bfloat162float(sm.dKt[row][cl]) + sm.ik[row][cl];
                rr[r] = __bfloat162float(sm.q[row][cl]) * dqv - __bfloat162float(sm.k[row][cl]) * dkv;
                rs += rr[r];
                if (row < nvalid) {
                    const int64_t off = (bh * L + t0 + row) * K + ch;
                    dq[off] = __float2bfloat16_rn(dqv);
                    dk[off] = __float2bfloat16_rn(dkv);
                }
            }
            sm.tot[I][cl] = rs;
            __syncthreads();
            float suf = sm.carry[cl];
            for (int J = I + 1; J < NS; ++J) suf += sm.tot[J][cl];
#pragma unroll
            for (int r = SC - 1; r >= 0; --r) {
                suf += rr[r];
                const int row = I * SC + r;
                if (row < nvalid) dla[(bh * L + t0 + row) * K + ch] = suf;
            }
        }
    }
}

bool map3(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t outer) {
    const uint64_t dims[3] = {inner, rows, outer};
    const uint64_t strides[2] = {inner * 2, inner * rows * 2};
    const uint32_t box[3] = {64, 128, 1};
    return encode_tmap(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

}  // namespace

gla_status tc_bwd_gemm_launch(const Problem& p, const void* dO, const void* v, const __nv_bfloat16* Sbuf,
                              const __nv_bfloat16* Dbuf, __nv_bfloat16* dP, __nv_bfloat16* dQt, __nv_bfloat16* dKt,
                              cudaStream_t s) {
    CUtensorMap m[4];
    memset(m, 0, sizeof(m));
    const uint64_t L = uint64_t(p.L), K = uint64_t(p.K), V = uint64_t(p.V), BH = uint64_t(p.BH), N = uint64_t(p.N);
    bool ok = map3(&m[0], dO, V, L, BH) && map3(&m[1], v, V, L, BH) && map3(&m[2], Sbuf, V, K, BH * N) &&
              map3(&m[3], Dbuf, V, K, BH * N);
    if (!ok) return GLA_ERR_CUDA;
    const size_t smem = 1024 + size_t(NSTAGE) * 4 * PIECE + sizeof(GemmBars);
    if (cudaFuncSetAttribute(k_bwd_gemm, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) != cudaSuccess)
        return GLA_ERR_CUDA;
    const dim3 grid(unsigned(p.N), unsigned(p.K / 128), unsigned(p.BH));
    GLA_LAUNCH("tc_bwd_gemm", k_bwd_gemm, grid, 192, smem, s, m[0], m[1], m[2], m[3], dP, dQt, dKt, p.L, p.N, p.K,
               p.V, device_error_word());
    return GLA_OK;
}

gla_status tc_bwd_intra_launch(const Problem& p, const void* q, const void* k, const float* la,
                               const __nv_bfloat16* dP, const __nv_bfloat16* dQt, const __nv_bfloat16* dKt,
                               const __nv_bfloat16* Sbuf, const __nv_bfloat16* Dbuf, const float* hT,
                               const float* dhT, void* dq, void* dk, float* dla, cudaStream_t s) {
    const size_t smem = sizeof(IntraSmem);
    if (cudaFuncSetAttribute(k_bwd_intra, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) != cudaSuccess)
        return GLA_ERR_CUDA;
    GLA_LAUNCH("tc_bwd_intra", k_bwd_intra, dim3(unsigned(p.N), unsigned(p.BH)), 256, smem, s,
               static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k), la, dP, dQt, dKt, Sbuf,
               Dbuf, hT, dhT, static_cast<__nv_bfloat16*>(dq), static_cast<__nv_bfloat16*>(dk), dla, p.L, p.N, p.K,
               p.V);
    return GLA_OK;
}

}  // namespace gla
