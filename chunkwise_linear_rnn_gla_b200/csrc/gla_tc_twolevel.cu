// Intra-chunk scores by two-level (secondary) chunking, the form the pages
// describe ("Gated Linear Attention Transformers with Hardware-Efficient
// Training", atlas.scime.ai summary, "Approach": a second level of chunking
// inside each chunk so that most intra-chunk products run on half-precision
// tensor cores), selected on the tensor-core path by a sub-chunk length of 16.
//
// With B the per-chunk cumsum of log alpha, P_js = sum_c q_jc k_sc e^{B_jc - B_sc}
// for s <= j. The chunk's 128 rows form 8 sub-chunks of 16:
//  - off-diagonal blocks (query sub-chunk I > key sub-chunk J): with rho_J the
//    cumsum at the last row of J, P_js = sum_c (q_jc e^{B_jc - rho_Jc})
//    (k_sc e^{rho_Jc - B_sc}); both factors are <= 1 (B decreases along the
//    chunk), so they never leave the bf16 range. For every J the block column
//    P[16(J+1).., J] is one tcgen05 GEMM (M = 128 query rows, rows of J and
//    before zeroed, N = 16 keys, K = d_k) into TMEM columns 16J ..;
//  - diagonal blocks: every term in fp32 in log space on the CUDA cores,
//    q_jc k_sc exp(B_jc - B_sc).
// The kernel overwrites the P that the preparation kernel wrote (the rescaled
// operands Q~, K~ and e^Gamma stay as prepared). One CTA per chunk: warps 0-7
// build the operands and the diagonal blocks, warp 8 issues the MMAs.

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "gla_common.cuh"
#include "gla_gate.cuh"
#include "gla_internal.h"
#include "gla_tc.h"

namespace gla {
namespace {

using namespace tc;

constexpr int C = kTcChunk;
constexpr int SC = 16;             // sub-chunk rows
constexpr int NS = C / SC;         // sub-chunks per chunk
constexpr int KP = 64;             // key channels per piece
constexpr int RS = KP + 1;         // padded fp32 row stride of the staged tiles (conflict-free columns)
constexpr uint32_t PIECE = 16384;  // [128 x 64] bf16 operand (A of one key sub-chunk)
constexpr uint32_t BPIECE = 2048;  // [16 x 64] bf16 operand (B of one key sub-chunk)
constexpr int kThreads = 288;

// shared memory layout (offsets from the 1024-aligned base)
constexpr uint32_t A_OFF = 0;                        // 2 A operands
constexpr uint32_t B_OFF = 2 * PIECE;                // NS-1 B operands
constexpr uint32_t BS_OFF = B_OFF + (NS - 1) * BPIECE;  // fp32 cumsum [128][RS]
constexpr uint32_t QS_OFF = BS_OFF + C * RS * 4;     // fp32 q [128][RS]
constexpr uint32_t KS_OFF = QS_OFF + C * RS * 4;     // fp32 k [128][RS]
constexpr uint32_t PD_OFF = KS_OFF + C * RS * 4;     // fp32 diagonal blocks [NS][16][16]
constexpr uint32_t BAR_OFF = PD_OFF + NS * SC * SC * 4;

struct TlBars {
    float tot[8][KP];  // per-warp 16-row gate sums of the current piece
    uint64_t ops_ready[2], mma_done[2], p_done, drain;
    uint32_t tmem_slot;
    int abort_flag;
};

constexpr size_t kSmem = 1024 + BAR_OFF + sizeof(TlBars);

__device__ __forceinline__ uint32_t sw_off(int row, int c) {  // bf16 element (row, c) of a SW128 [rows x 64] tile
    return uint32_t(row) * 128u + uint32_t(((c >> 3) ^ (row & 7)) << 4) + uint32_t(c & 7) * 2u;
}

template <int K, int GK>
__global__ void __launch_bounds__(kThreads, 1)
    k_tc_intra_twolevel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k, GateArgs ga,
                        __nv_bfloat16* __restrict__ P, int64_t L, int64_t N, int* err) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    TlBars& bar = *reinterpret_cast<TlBars*>(base + BAR_OFF);
    float* Bs = reinterpret_cast<float*>(base + BS_OFF);
    float* Qs = reinterpret_cast<float*>(base + QS_OFF);
    float* Ks = reinterpret_cast<float*>(base + KS_OFF);
    float* Pd = reinterpret_cast<float*>(base + PD_OFF);
    volatile int* abort_flag = &bar.abort_flag;
    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    const int i = blockIdx.x;
    const int64_t bh = blockIdx.y;
    const int64_t t0 = int64_t(i) * C;
    const int nvalid = int(L - t0 < C ? L - t0 : C);
    constexpr int npiece = K / KP;

    if (tid == 0) {
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bar.ops_ready[b], 256);
            mbar_init(&bar.mma_done[b], 1);
        }
        mbar_init(&bar.p_done, 1);
        mbar_init(&bar.drain, 1);
        bar.abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 8) {
        tmem_alloc(&bar.tmem_slot, 128);
        tmem_relinquish();
    }
    for (int e = tid; e < NS * SC * SC; e += kThreads) Pd[e] = 0.f;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bar.tmem_slot;
    pdl_launch_dependents();
    pdl_wait();

    if (warp == 8) {
        if (lane == 0) {
            const uint32_t id = idesc_bf16_f32(128, SC, false, false);
            bool ok = true;
            for (int n = 0; n < npiece * (NS - 1) && ok; ++n) {
                const int t = n / (NS - 1), J = n % (NS - 1), b = n & 1;
                ok = mbar_wait(&bar.ops_ready[b], uint32_t((n >> 1) & 1), err, abort_flag);
                if (!ok) break;
                tc_fence_after();
                const uint32_t a0 = smem_u32(base + A_OFF + b * PIECE);
                const uint32_t b0 = smem_u32(base + B_OFF + J * BPIECE);
#pragma unroll
                for (int kk = 0; kk < KP / 16; ++kk)
                    mma_bf16(tmem + uint32_t(SC * J), sdesc_sw128(a0 + kk * 32, 16, 1024),
                             sdesc_sw128(b0 + kk * 32, 16, 1024), id, (t > 0 || kk > 0) ? 1u : 0u);
                mma_commit(&bar.mma_done[b]);
            }
            if (ok) mma_commit(&bar.p_done);
            mma_commit(&bar.drain);
            mbar_drain(&bar.drain, 0);
        }
    } else {
        const int I = warp;
        const int cg = lane & 7, rs = lane >> 3;
        const int row0 = 16 * I + 4 * rs;
        bool ok = true;
        int n = 0;  // operand builds so far (the MMA sequence number)
        for (int t = 0; t < npiece; ++t) {
            const int64_t ch0 = int64_t(KP) * t + 8 * cg;
            // ---- stage q, k and the per-chunk cumsum B of this piece (fp32, padded rows)
            float Bv[4][8], tot[8];
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const bool v = row0 + r < nvalid;
                const int64_t tr = t0 + (v ? row0 + r : nvalid - 1);
                const int64_t off = (bh * L + tr) * K + ch0;
                const uint4 qu = *reinterpret_cast<const uint4*>(q + off);
                const uint4 ku = *reinterpret_cast<const uint4*>(k + off);
                const __nv_bfloat162* q2 = reinterpret_cast<const __nv_bfloat162*>(&qu);
                const __nv_bfloat162* k2 = reinterpret_cast<const __nv_bfloat162*>(&ku);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 qf = __bfloat1622float2(q2[e]), kf = __bfloat1622float2(k2[e]);
                    Qs[(row0 + r) * RS + 8 * cg + 2 * e] = v ? qf.x : 0.f;
                    Qs[(row0 + r) * RS + 8 * cg + 2 * e + 1] = v ? qf.y : 0.f;
                    Ks[(row0 + r) * RS + 8 * cg + 2 * e] = v ? kf.x : 0.f;
                    Ks[(row0 + r) * RS + 8 * cg + 2 * e + 1] = v ? kf.y : 0.f;
                }
#pragma unroll
                for (int e = 0; e < 8; ++e) Bv[r][e] = v ? la_floor(gate_log_alpha(ga, bh, tr, ch0 + e, L, K)) : 0.f;
            }
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                float run = 0.f;
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    run += Bv[r][e];
                    Bv[r][e] = run;
                }
                tot[e] = run;
            }
            float excl[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                float incl = tot[e];
                float y = __shfl_up_sync(0xffffffffu, incl, 8);
                if (rs >= 1) incl += y;
                y = __shfl_up_sync(0xffffffffu, incl, 16);
                if (rs >= 2) incl += y;
                excl[e] = incl - tot[e];
                if (rs == 3) bar.tot[I][8 * cg + e] = incl;
            }
            named_sync(1, 256);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                float pre = 0.f;
                for (int J = 0; J < I; ++J) pre += bar.tot[J][8 * cg + e];
#pragma unroll
                for (int r = 0; r < 4; ++r) Bs[(row0 + r) * RS + 8 * cg + e] = Bv[r][e] + pre + excl[e];
            }
            named_sync(1, 256);  // the staged tiles are complete (and the totals read)
            // ---- off-diagonal block columns: for every key sub-chunk J the rescaled operands, then its GEMM
            for (int J = 0; J < NS - 1; ++J, ++n) {
                const int b = n & 1;
                // operand buffer b is free once the GEMM two builds back is done
                if (n >= 2) ok = ok && mbar_wait(&bar.mma_done[b], uint32_t(((n >> 1) - 1) & 1), err, abort_flag);
                uint8_t* A = base + A_OFF + b * PIECE;
                uint8_t* Bo = base + B_OFF + J * BPIECE;
                const int rho_row = SC * J + SC - 1;
                if (ok) {
                    // A: thread = (row, 32 channels): q e^{B - rho} for rows after J, zero before
                    const int row = tid & 127, half = tid >> 7;
#pragma unroll 4
                    for (int c8 = 0; c8 < 4; ++c8) {
                        float f[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const int c = 32 * half + 8 * c8 + e;
                            f[e] = row > rho_row ? Qs[row * RS + c] * __expf(fminf(Bs[row * RS + c] - Bs[rho_row * RS + c], 0.f))
                                                 : 0.f;
                        }
                        *reinterpret_cast<uint4*>(A + sw_off(row, 32 * half + 8 * c8)) =
                            make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                                       pack_bf16x2(f[6], f[7]));
                    }
                    // B (at the first piece's visit only the rows of J exist; every piece rebuilds it): k e^{rho - B}
                    if (tid < SC * 8) {
                        const int s = tid >> 3, c8 = tid & 7;
                        const int srow = SC * J + s;
                        float f[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const int c = 8 * c8 + e;
                            f[e] = Ks[srow * RS + c] * __expf(fminf(Bs[rho_row * RS + c] - Bs[srow * RS + c], 0.f));
                        }
                        *reinterpret_cast<uint4*>(Bo + sw_off(s, 8 * c8)) =
                            make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                                       pack_bf16x2(f[6], f[7]));
                    }
                }
                fence_proxy_async_smem();
                mbar_arrive(&bar.ops_ready[b]);
            }
            // ---- diagonal blocks in log space: warp I owns block I; lane = one of its 136 (j >= s) pairs per round
            for (int pr = lane; pr < SC * (SC + 1) / 2; pr += 32) {
                int jj = 0;
                while ((jj + 1) * (jj + 2) / 2 <= pr) ++jj;  // pr = jj (jj + 1) / 2 + ss
                const int ss = pr - jj * (jj + 1) / 2;
                const int j = SC * I + jj, s = SC * I + ss;
                float acc = 0.f;
#pragma unroll 8
                for (int c = 0; c < KP; ++c)
                    acc += Qs[j * RS + c] * Ks[s * RS + c] * __expf(fminf(Bs[j * RS + c] - Bs[s * RS + c], 0.f));
                Pd[(I * SC + jj) * SC + ss] += acc;
            }
            // the staged tiles are overwritten by the next piece: every operand build and diagonal term is done
            // (the MMAs read only the operand buffers)
            named_sync(1, 256);
        }
        // ---- P rows: off-diagonal columns from TMEM, diagonal blocks from shared memory, zero above
        const int q4 = warp & 3, h = warp >> 2;
        const int row = 32 * q4 + lane;
        const bool have = __all_sync(0xffffffffu, ok && mbar_wait(&bar.p_done, 0, err, abort_flag));
        if (have) {
            tc_fence_after();
            const int I = row / SC;
            uint4* dst = reinterpret_cast<uint4*>(P + ((bh * N + i) * C + row) * C + 64 * h);
#pragma unroll
            for (int c16 = 0; c16 < 4; ++c16) {
                float y[16];
                tmem_ld16(tmem + (uint32_t(32 * q4) << 16) + uint32_t(64 * h + 16 * c16), y);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const int col = 64 * h + 16 * c16 + e;
                    float v = 0.f;
                    if (col < SC * I) v = y[e];
                    else if (col <= row) v = Pd[(I * SC + (row - SC * I)) * SC + (col - SC * I)];
                    y[e] = row < nvalid ? v : 0.f;
                }
                dst[2 * c16] = make_uint4(pack_bf16x2(y[0], y[1]), pack_bf16x2(y[2], y[3]), pack_bf16x2(y[4], y[5]),
                                          pack_bf16x2(y[6], y[7]));
                dst[2 * c16 + 1] = make_uint4(pack_bf16x2(y[8], y[9]), pack_bf16x2(y[10], y[11]),
                                              pack_bf16x2(y[12], y[13]), pack_bf16x2(y[14], y[15]));
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 8) {
        tc_fence_after();
        tmem_dealloc(tmem, 128);
    }
}

template <int GK>
gla_status launch_gk(const Problem& p, const void* q, const void* k, const GateArgs& ga, __nv_bfloat16* P,
                     cudaStream_t s) {
    auto fn = p.K == 256 ? k_tc_intra_twolevel<256, GK> : k_tc_intra_twolevel<128, GK>;
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kSmem)) != cudaSuccess)
        return GLA_ERR_CUDA;
    GLA_LAUNCH_PDL("tc_intra_twolevel", fn, dim3(unsigned(p.N), unsigned(p.BH)), kThreads, kSmem, s,
                   static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k), ga, P, p.L, p.N,
                   device_error_word());
    return GLA_OK;
}

}  // namespace

gla_status tc_intra_twolevel_launch(const Problem& p, const void* q, const void* k, const float* la,
                                    __nv_bfloat16* P, cudaStream_t s) {
    const GateArgs ga{la, p.gate, p.inv_tau, p.H};
    if (p.gate == kGatePreact) return launch_gk<kGatePreact>(p, q, k, ga, P, s);
    return launch_gk<kGateChannel>(p, q, k, ga, P, s);
}

}  // namespace gla
