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
               float* __restrict__ xdot, int64_t L, int64_t N, int64_t K, int64_t V, int* err) {
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
            mbar_init(&bar.empty[s], 1 + 128);  // MMA commit + the 128 row-dot threads
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
        // while the MMAs run: x[c] = sum_v D_i[c,v] S_[i][c,v] for this thread's key channel
        float x = 0.f;
        bool ok = true;
        for (int vb = 0; vb < nvb; ++vb) {
            const int s = vb % NSTAGE;
            if (!mbar_wait(&bar.full[s], uint32_t((vb / NSTAGE) & 1), err, abort_flag)) {
                ok = false;
                break;
            }
            const uint8_t* st = base + s * 4 * PIECE;
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) {
                const uint32_t off = uint32_t(r) * 128u + uint32_t((ch ^ (r & 7)) * 16);
                const uint4 sv = *reinterpret_cast<const uint4*>(st + 2 * PIECE + off);
                const uint4 dv = *reinterpret_cast<const uint4*>(st + 3 * PIECE + off);
                const __nv_bfloat162* s2 = reinterpret_cast<const __nv_bfloat162*>(&sv);
                const __nv_bfloat162* d2 = reinterpret_cast<const __nv_bfloat162*>(&dv);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 a = __bfloat1622float2(s2[e]), b = __bfloat1622float2(d2[e]);
                    x = fmaf(a.x, b.x, fmaf(a.y, b.y, x));
                }
            }
            mbar_arrive(&bar.empty[s]);
        }
        if (ok) xdot[(bh * N + i) * K + 128 * kh + r] = x;
        if (ok && mbar_wait(&bar.done, 0, err, abort_flag)) {
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

__device__ __forceinline__ void cpa16(void* dst, const void* src, bool valid) {
    const uint32_t n = valid ? 16u : 0u;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(tc_smem_u32(dst)), "l"(src), "r"(n) : "memory");
}
__device__ __forceinline__ void cpa_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cpa_wait1() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }
__device__ __forceinline__ void cpa_wait0() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

struct IntraStage {  // raw inputs of one 32-channel tile (cp.async)
    float la[C][KT];
    __nv_bfloat16 q[C][KT];
    __nv_bfloat16 k[C][KT];
};

struct IntraSmem {
    __nv_bfloat16 dP[C][DPS];
    float dg[NS][SC][SC];   // diagonal blocks of dP in fp32: dg[I][j][s] = dP[16I+j][16I+s]
    float dgT[NS][SC][SC];  // the same blocks transposed: dgT[I][s][j]
    IntraStage st[2];
    float a[C][KT + 1], kf[C][KT + 1];   // e^{B_j - rho_I}, e^{last_I - B_j}
    __nv_bfloat16 qh[C][QS], kh[C][QS];  // bf16 operands of the off-diagonal blocks
    float iq[C][KT + 1], ik[C][KT + 1];  // intra-chunk parts of dq, dk
    float d[28][KT];
    float h8[NS][2][KT];   // per half sub-chunk: gate sums, then r sums
    float k8[NS][2][KT];   // per half sub-chunk: sum_j K~_j dK~_j
    float first[NS][KT];   // B offset of each sub-chunk's first row within its half 0
    float EI[NS][KT], FI[NS][KT], DI[NS][KT];
    float eG[KT];
    unsigned unsafe_mask[NS];
};

// One CTA per (chunk, head), 16 warps. Elementwise phases: thread (channel =
// lane, sub-chunk I = warp % 8, half = warp / 8) owns rows 8*half .. 8*half+7
// of sub-chunk I. Off-diagonal and diagonal blocks: warps 0-7 form the dq
// side (query sub-chunk I = warp), warps 8-15 the dk side (key sub-chunk
// J = warp - 8). Key channels are processed in tiles of 32.
__global__ void __launch_bounds__(512, 1)
    k_bwd_intra(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                const float* __restrict__ la, const __nv_bfloat16* __restrict__ dPg,
                const __nv_bfloat16* __restrict__ dQt, const __nv_bfloat16* __restrict__ dKt,
                const float* __restrict__ xdot, __nv_bfloat16* __restrict__ dq, __nv_bfloat16* __restrict__ dk,
                float* __restrict__ dla, int64_t L, int64_t N, int64_t K) {
    constexpr int NT = 512;
    constexpr int HR = SC / 2;  // rows per half sub-chunk
    extern __shared__ __align__(16) unsigned char smem_raw[];
    IntraSmem& sm = *reinterpret_cast<IntraSmem*>(smem_raw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t i = blockIdx.x, bh = blockIdx.y;
    const int64_t t0 = i * C;
    const int nvalid = int(L - t0 < C ? L - t0 : C);
    const int g = lane >> 2, tq = lane & 3;
    const int cl = lane, I = warp & 7, half = warp >> 3;
    const int r0 = I * SC + half * HR;  // first row owned in the elementwise phases

    for (int e = tid; e < C * C / 8; e += NT) {
        const int row = e / (C / 8), cc = (e % (C / 8)) * 8;
        cpa16(&sm.dP[row][cc], dPg + ((bh * N + i) * C + row) * C + cc, true);
    }
    auto issue = [&](int64_t c0, int sb) {
        IntraStage& S = sm.st[sb];
        for (int e = tid; e < C * (KT / 4); e += NT) {
            const int row = e / (KT / 4), cc = (e % (KT / 4)) * 4;
            const bool ok = row < nvalid;
            cpa16(&S.la[row][cc], la + (bh * L + t0 + (ok ? row : 0)) * K + c0 + cc, ok);
        }
        for (int e = tid; e < C * (KT / 8); e += NT) {
            const int row = e / (KT / 8), cc = (e % (KT / 8)) * 8;
            const bool ok = row < nvalid;
            const int64_t off = (bh * L + t0 + (ok ? row : 0)) * K + c0 + cc;
            cpa16(&S.q[row][cc], q + off, ok);
            cpa16(&S.k[row][cc], k + off, ok);
        }
        cpa_commit();
    };
    issue(0, 0);
    int sb = 0;

    for (int64_t c0 = 0; c0 < K; c0 += KT, sb ^= 1) {
        if (c0 + KT < K) {
            issue(c0 + KT, sb ^ 1);
            cpa_wait1();
        } else {
            cpa_wait0();
        }
        __syncthreads();
        if (c0 == 0) {
            for (int e = tid; e < NS * SC * SC; e += NT) {
                const int I2 = e / (SC * SC), j = (e / SC) % SC, s_ = e % SC;
                const float v = __bfloat162float(sm.dP[I2 * SC + j][I2 * SC + s_]);
                sm.dg[I2][j][s_] = v;
                sm.dgT[I2][s_][j] = v;
            }
        }
        const IntraStage& S = sm.st[sb];
        const int64_t ch = c0 + cl;
        // inter-chunk parts of this thread's rows, used by the combine at the end
        unsigned short hq[HR], hk[HR];
#pragma unroll
        for (int r = 0; r < HR; ++r) {
            const int row = r0 + r;
            const bool ok = row < nvalid;
            const int64_t off = (bh * L + t0 + (ok ? row : 0)) * K + ch;
            hq[r] = ok ? reinterpret_cast<const unsigned short*>(dQt)[off] : 0;
            hk[r] = ok ? reinterpret_cast<const unsigned short*>(dKt)[off] : 0;
        }
        const float xd = xdot[(bh * N + i) * K + ch];
        // ---- phase 1: cumsum over the half sub-chunk, factors, operands
        float b[HR];
        float run = 0.f;
#pragma unroll
        for (int r = 0; r < HR; ++r) {
            run += S.la[r0 + r][cl];
            b[r] = run;  // cumsum within this half
        }
        sm.h8[I][half][cl] = run;
        if (half == 0) sm.first[I][cl] = b[0];
        if (tid < NS) sm.unsafe_mask[tid] = 0u;
        __syncthreads();
        float pre = 0.f, gamma = 0.f, lastJ[NS];
#pragma unroll
        for (int J = 0; J < NS; ++J) {
            const float t = sm.h8[J][0][cl] + sm.h8[J][1][cl];
            if (J < I) pre += t;
            gamma += t;
            lastJ[J] = gamma;  // B at the last row of sub-chunk J
        }
        const float rho = pre + sm.first[I][cl];        // B at the first row of sub-chunk I
        const float last = lastJ[I];
        const float hoff = pre + (half ? sm.h8[I][0][cl] : 0.f);  // B offset of this half
        const float span = fmaxf(rho - last, 0.f);
        const bool unsafe = span > kUnsafeSpan;
        const float eSpan = unsafe ? 0.f : __expf(span);
        if (half == 0) {
            if (unsafe) atomicOr(&sm.unsafe_mask[I], 1u << cl);
            // every exponent below is <= 0 in exact arithmetic; the clamps only absorb the
            // rounding of cumsums summed in different orders (|B| can reach ~1e32 for alpha = 0)
            sm.EI[I][cl] = __expf(fminf(rho, 0.f));
            sm.FI[I][cl] = __expf(fminf(gamma - last, 0.f));
            sm.DI[I][cl] = eSpan;
            if (I == 0) sm.eG[cl] = __expf(fminf(gamma, 0.f));
#pragma unroll
            for (int J = 0; J < NS - 1; ++J)
                if (J < I) sm.d[pidx(I, J)][cl] = __expf(fminf(rho - lastJ[J], 0.f));
        }
#pragma unroll
        for (int r = 0; r < HR; ++r) {
            const int row = r0 + r;
            const float Bv = hoff + b[r];
            const float av = __expf(fminf(Bv - rho, 0.f)), kv = __expf(fminf(last - Bv, 0.f));
            sm.a[row][cl] = av;
            sm.kf[row][cl] = kv;
            sm.qh[row][cl] = __float2bfloat16_rn(__bfloat162float(S.q[row][cl]) * av);
            sm.kh[row][cl] = __float2bfloat16_rn(__bfloat162float(S.k[row][cl]) * kv);
        }
        __syncthreads();
        // ---- phase 2: warps 0-7 dq side of sub-chunk I, warps 8-15 dk side of sub-chunk J = I
        if (half == 0) {
            // off-diagonal: dq_I += sum_{J<I} dP_IJ (K^_J * d_IJ)
            float aq[4][4];
#pragma unroll
            for (int n = 0; n < 4; ++n)
#pragma unroll
                for (int e = 0; e < 4; ++e) aq[n][e] = 0.f;
            for (int J = 0; J < I; ++J) {
                uint32_t A[4];
                ldsm_x4(tc_smem_u32(&sm.dP[I * SC + (lane & 15)][J * SC + (lane >> 4) * 8]), A);
                const float* dd = sm.d[pidx(I, J)];
#pragma unroll
                for (int nb2 = 0; nb2 < 2; ++nb2) {
                    uint32_t Bf[4];
                    const int row = J * SC + (lane & 7) + ((lane >> 3) & 1) * 8;
                    const int col = nb2 * 16 + (lane >> 4) * 8;
                    ldsm_x4_t(tc_smem_u32(&sm.kh[row][col]), Bf);
                    const float f0 = dd[nb2 * 16 + g], f1 = dd[nb2 * 16 + 8 + g];
                    mma16816(aq[2 * nb2], A, scale2(Bf[0], f0), scale2(Bf[1], f0));
                    mma16816(aq[2 * nb2 + 1], A, scale2(Bf[2], f1), scale2(Bf[3], f1));
                }
            }
#pragma unroll
            for (int n = 0; n < 4; ++n) {
                const int c = n * 8 + 2 * tq;
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int row = I * SC + g + 8 * hh;
                    sm.iq[row][c] = aq[n][2 * hh] * sm.a[row][c];
                    sm.iq[row][c + 1] = aq[n][2 * hh + 1] * sm.a[row][c + 1];
                }
            }
            __syncwarp();
            // diagonal block in fp32 (lane = channel)
            const int c = lane;
            const bool exact = (sm.unsafe_mask[I] >> c) & 1u;
            if (!exact) {
                float kv[SC];
#pragma unroll
                for (int r = 0; r < SC; ++r)
                    kv[r] = __bfloat162float(S.k[I * SC + r][c]) * sm.kf[I * SC + r][c] * eSpan;  // k_s e^{rho-B_s}
#pragma unroll
                for (int j = 0; j < SC; ++j) {
                    float acc = 0.f;
                    const float4* row4 = reinterpret_cast<const float4*>(sm.dg[I][j]);
#pragma unroll
                    for (int q4 = 0; q4 <= j / 4; ++q4) {  // broadcast 16-byte loads of the dP row
                        const float4 w = row4[q4];
                        if (4 * q4 + 0 <= j) acc = fmaf(w.x, kv[4 * q4 + 0], acc);
                        if (4 * q4 + 1 <= j) acc = fmaf(w.y, kv[4 * q4 + 1], acc);
                        if (4 * q4 + 2 <= j) acc = fmaf(w.z, kv[4 * q4 + 2], acc);
                        if (4 * q4 + 3 <= j) acc = fmaf(w.w, kv[4 * q4 + 3], acc);
                    }
                    sm.iq[I * SC + j][c] += sm.a[I * SC + j][c] * acc;
                }
            } else {  // rare: the decay span leaves the fp32 range; exact log-space terms
                float Bj[SC];
                float run2 = 0.f;
                for (int r = 0; r < I * SC; ++r) run2 += S.la[r][c];
                for (int r = 0; r < SC; ++r) {
                    run2 += S.la[I * SC + r][c];
                    Bj[r] = run2;
                }
                for (int j = 0; j < SC; ++j) {
                    float acc = 0.f;
                    for (int s_ = 0; s_ <= j; ++s_)
                        acc += sm.dg[I][j][s_] * __bfloat162float(S.k[I * SC + s_][c]) * expf(fminf(Bj[j] - Bj[s_], 0.f));
                    sm.iq[I * SC + j][c] += acc;
                }
            }
        } else {
            // off-diagonal: dk_J += sum_{I2>J} dP_{I2 J}^T (Q^_{I2} * d_{I2 J}), J = I
            const int J = I;
            float ak[4][4];
#pragma unroll
            for (int n = 0; n < 4; ++n)
#pragma unroll
                for (int e = 0; e < 4; ++e) ak[n][e] = 0.f;
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
#pragma unroll
            for (int n = 0; n < 4; ++n) {
                const int c = n * 8 + 2 * tq;
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int row = J * SC + g + 8 * hh;
                    sm.ik[row][c] = ak[n][2 * hh] * sm.kf[row][c];
                    sm.ik[row][c + 1] = ak[n][2 * hh + 1] * sm.kf[row][c + 1];
                }
            }
            __syncwarp();
            const int c = lane;
            const bool exact = (sm.unsafe_mask[J] >> c) & 1u;
            const float Dv = sm.DI[J][c];
            if (!exact) {
                float qv[SC];
#pragma unroll
                for (int r = 0; r < SC; ++r)
                    qv[r] = __bfloat162float(S.q[J * SC + r][c]) * sm.a[J * SC + r][c];  // q_j e^{B_j-rho}
#pragma unroll
                for (int s_ = 0; s_ < SC; ++s_) {
                    float acc = 0.f;
                    const float4* row4 = reinterpret_cast<const float4*>(sm.dgT[J][s_]);
#pragma unroll
                    for (int q4 = s_ / 4; q4 < SC / 4; ++q4) {
                        const float4 w = row4[q4];
                        if (4 * q4 + 0 >= s_) acc = fmaf(w.x, qv[4 * q4 + 0], acc);
                        if (4 * q4 + 1 >= s_) acc = fmaf(w.y, qv[4 * q4 + 1], acc);
                        if (4 * q4 + 2 >= s_) acc = fmaf(w.z, qv[4 * q4 + 2], acc);
                        if (4 * q4 + 3 >= s_) acc = fmaf(w.w, qv[4 * q4 + 3], acc);
                    }
                    sm.ik[J * SC + s_][c] += sm.kf[J * SC + s_][c] * Dv * acc;
                }
            } else {
                float Bj[SC];
                float run2 = 0.f;
                for (int r = 0; r < J * SC; ++r) run2 += S.la[r][c];
                for (int r = 0; r < SC; ++r) {
                    run2 += S.la[J * SC + r][c];
                    Bj[r] = run2;
                }
                for (int s_ = 0; s_ < SC; ++s_) {
                    float acc = 0.f;
                    for (int j = s_; j < SC; ++j)
                        acc += sm.dgT[J][s_][j] * __bfloat162float(S.q[J * SC + j][c]) * expf(fminf(Bj[j] - Bj[s_], 0.f));
                    sm.ik[J * SC + s_][c] += acc;
                }
            }
        }
        __syncthreads();
        // ---- combine and closed-form gate gradient (thread: channel cl, rows r0 .. r0+7)
        {
            const float E = sm.EI[I][cl], F = sm.FI[I][cl];
            float rr[HR];
            float rs = 0.f, ks = 0.f;
#pragma unroll
            for (int r = 0; r < HR; ++r) {
                const int row = r0 + r;
                const float qv = __bfloat162float(S.q[row][cl]), kv = __bfloat162float(S.k[row][cl]);
                const float dQi = __bfloat162float(__ushort_as_bfloat16(hq[r]));
                const float dKi = __bfloat162float(__ushort_as_bfloat16(hk[r]));
                const float eGB = sm.kf[row][cl] * F;  // e^{Gamma - B_j}
                const float dqv = sm.a[row][cl] * E * dQi + sm.iq[row][cl];
                const float dkv = eGB * dKi + sm.ik[row][cl];
                rr[r] = qv * dqv - kv * dkv;
                rs += rr[r];
                ks += kv * eGB * dKi;  // K~_j dK~_j
                if (row < nvalid) {
                    const int64_t off = (bh * L + t0 + row) * K + ch;
                    dq[off] = __float2bfloat16_rn(dqv);
                    dk[off] = __float2bfloat16_rn(dkv);
                }
            }
            __syncthreads();  // everyone is done reading the gate sums in h8
            sm.h8[I][half][cl] = rs;
            sm.k8[I][half][cl] = ks;
            __syncthreads();
            // carry from all later chunks: sum_v D_i S_[i+1] = e^Gamma sum_v D_i S_[i] + sum_j K~_j dK~_j
            float suf = sm.eG[cl] * xd;
#pragma unroll
            for (int J = 0; J < NS; ++J)
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    suf += sm.k8[J][hh][cl];
                    if (J > I || (J == I && hh > half)) suf += sm.h8[J][hh][cl];
                }
#pragma unroll
            for (int r = HR - 1; r >= 0; --r) {
                suf += rr[r];
                const int row = r0 + r;
                if (row < nvalid) dla[(bh * L + t0 + row) * K + ch] = suf;
            }
        }
        __syncthreads();
    }
}

}  // namespace

bool map3(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t outer) {
    const uint64_t dims[3] = {inner, rows, outer};
    const uint64_t strides[2] = {inner * 2, inner * rows * 2};
    const uint32_t box[3] = {64, 128, 1};
    return encode_tmap(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

gla_status tc_bwd_gemm_launch(const Problem& p, const void* dO, const void* v, const __nv_bfloat16* Sbuf,
                              const __nv_bfloat16* Dbuf, __nv_bfloat16* dP, __nv_bfloat16* dQt, __nv_bfloat16* dKt,
                              float* xdot, cudaStream_t s) {
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
    GLA_LAUNCH("tc_bwd_gemm", k_bwd_gemm, grid, 192, smem, s, m[0], m[1], m[2], m[3], dP, dQt, dKt, xdot, p.L, p.N,
               p.K, p.V, device_error_word());
    return GLA_OK;
}

gla_status tc_bwd_intra_launch(const Problem& p, const void* q, const void* k, const float* la,
                               const __nv_bfloat16* dP, const __nv_bfloat16* dQt, const __nv_bfloat16* dKt,
                               const float* xdot, void* dq, void* dk, float* dla, cudaStream_t s) {
    const size_t smem = sizeof(IntraSmem);
    if (cudaFuncSetAttribute(k_bwd_intra, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) != cudaSuccess)
        return GLA_ERR_CUDA;
    GLA_LAUNCH("tc_bwd_intra", k_bwd_intra, dim3(unsigned(p.N), unsigned(p.BH)), 512, smem, s,
               static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k), la, dP, dQt, dKt, xdot,
               static_cast<__nv_bfloat16*>(dq), static_cast<__nv_bfloat16*>(dk), dla, p.L, p.N, p.K);
    return GLA_OK;
}

}  // namespace gla
