// Tensor-core backward, chunk-parallel part: one fused kernel per chunk and
// 128 key channels.
//
// With D_i = dL/dS_[i+1] (written in bf16 by the reverse state walk that also
// produces dv) and the forward states S_[i], the backward of chunk i is
// ("Gated Linear Attention Transformers with Hardware-Efficient Training",
// atlas.scime.ai summary, "Approach": chunkwise form and the closed-form
// gate gradient):
//   dP_js    = dO_j . v_s  (s <= j)
//   dq_j     = e^{B_j} * (dO_j S_[i]^T) + sum_{s<=j} dP_js k_s e^{B_j - B_s}
//   dk_s     = e^{Gamma - B_s} * (v_s D_i^T) + sum_{j>=s} dP_js q_j e^{B_j - B_s}
//   dlog a_t = sum_{s>=t} (q_s dq_s - k_s dk_s) + sum_v dhT * hT
// The reverse cumsum needs, for every chunk, the sum over all later chunks;
// that carry is exact and local:
//   sum_{s >= (i+1)C} r_s + sum_v dhT*hT = sum_v D_i[c,v] S_[i+1][c,v]
//                                        = e^Gamma sum_v D_i S_[i] + sum_s K~_s (v_s D_i^T)
// (the state update S_[i+1] = e^Gamma S_[i] + K~^T v), with S_[N] = hT and
// D_{N-1} = dhT for the last chunk.
//
// Every contraction runs on tcgen05 with fp32 accumulators in TMEM. The
// intra-chunk sums use the chunk form with the gate bounded per key channel
// (as in the forward preparation): for a channel with Gamma_c >= -64 every
// e^{+-B} is inside [e^-64, e^64], so
//   dq_j = e^{B_j} * [ (dO S^T)_j + sum_{s<=j} dP_js K^0_s ],   K^0 = k e^{-B}
//   dk_s = e^{Gamma - B_s} (v D^T)_s + e^{-B_s} sum_{j>=s} dP_js Q~_j
// and the dq bracket accumulates in ONE TMEM accumulator. Channels beyond the
// bound get a zero K^0 column and exact log-space intra terms on the CUDA
// cores.
//
// The accumulators are transposed (TMEM lane = key channel, column = token)
// so that the epilogue thread of a channel walks the tokens in order: the
// per-chunk gate cumsum, the gate factors and the reverse cumsum of the gate
// gradient all run along a thread, and every global store is coalesced over
// the channels.
//
// TMEM (512 columns): [0,128) dP (lane = row j), later the intra part of dK~^T;
// [128,256) dQ^T; [256,384) dK~^T inter part (v D^T); [384,512) per-token gate
// table (e^{-B}, or B itself for a channel beyond the bound).
//
// Roles (576 threads): warp 0 TMA producer; warp 1 TMEM owner and MMA issuer;
// warps 2-5 "row" warps (x_c = sum_v D S from the staged tiles, then the dP
// epilogue: mask, bf16, swizzled shared tile); warps 6-9 "gate" warps
// (thread = key channel: cumsum from the staged log-gate tile, gate table, K^0
// operand); at the end warps 2-17 in four groups of 32 tokens form dq, dk and
// the gate gradient: dq and dk staged in shared memory and written by one TMA
// store per group, dlog a written directly (128-byte rows per warp store).

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstring>
#include <type_traits>

#include "gla_common.cuh"
#include "gla_gate.cuh"
#include "gla_internal.h"
#include "gla_tc.h"
#include "tc_host.h"

namespace gla {
namespace {

using namespace tc;

constexpr int C = kTcChunk;
constexpr uint32_t PIECE = 16384;
constexpr int NSTAGE = 2;  // each stage: dO, v, S, D pieces for 64 value columns
constexpr uint32_t STAGE_BYTES = 4 * PIECE;
constexpr uint32_t LA_OFF = 8 * PIECE;             // log a tile, fp32 [128 tokens][128 channels], read by the prologue
constexpr uint32_t KH_OFF = 12 * PIECE;            // k tile, rescaled in place into the K^0 operand, 2 pieces
constexpr uint32_t DPM_OFF = 0;                    // after the value loop: masked dP (bf16), 2 pieces
constexpr uint32_t QT_OFF = LA_OFF;                // once the prologue is done: Q~ tile, 2 pieces
constexpr uint32_t RB_OFF = 4 * PIECE;             //                       r = q dq - k dk, fp32 [128][128]
constexpr uint32_t QS_OFF = LA_OFF + 2 * PIECE;    // once the prologue is done: q tile, 2 pieces
constexpr uint32_t KS_OFF = 2 * PIECE;             // after the value loop: k tile, 2 pieces
// after the intra MMAs: exact-path dk terms for tokens 0-63 over the Q~ tile and for tokens
// 64-127 over K^0; after the exact pass: per-channel sums exchanged between the warp groups
// over the masked dP tile
constexpr int kThreads = 576;
constexpr int kFinal = 512;  // threads of the final phase: warps 2-17
constexpr float kSafeDecay = 64.f;
constexpr float kSafeGam = 1.6038109e-28f;  // e^-64
constexpr uint32_t kStaggerNs = 10000;      // start offset of every other first-wave CTA

struct BwdBars {
    uint64_t full[NSTAGE], empty[NSTAGE];
    uint64_t pro_full, accA, qt_full, qk_full, dpm_ready, khat_ready, xd_ready, accB, drain;
    uint32_t tmem_slot;
    int abort_flag;
    int any_exact;  // some key channel of this CTA is beyond the bound
    float xd[128];  // sum_v D_i[c,v] S_[i][c,v]
    float btab[128];  // scalar gate kinds: the per-token cumsum b_t in base-2 units
};

constexpr bool scalar_kind(int GK) { return GK == kGateScalar || GK == kGateHead; }

// byte offset of element (row, col) in a [128 x 128] bf16 tile stored as two
// SW128 pieces of 64 columns
__device__ __forceinline__ uint32_t tile_off(int row, int col) {
    const int c64 = col & 63;
    return uint32_t(col >> 6) * PIECE + uint32_t(row) * 128u + uint32_t(((c64 >> 3) ^ (row & 7)) << 4) +
           uint32_t(c64 & 7) * 2u;
}

template <int GK>
__global__ void __launch_bounds__(kThreads, 1)
    k_bwd_chunk(const __grid_constant__ CUtensorMap tmDO, const __grid_constant__ CUtensorMap tmV,
                const __grid_constant__ CUtensorMap tmS, const __grid_constant__ CUtensorMap tmD,
                const __grid_constant__ CUtensorMap tmQt, const __grid_constant__ CUtensorMap tmQ,
                const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmDQ,
                const __grid_constant__ CUtensorMap tmDK,
                const __grid_constant__ CUtensorMap tmLA,
                const __nv_bfloat16* __restrict__ q,
                const __nv_bfloat16* __restrict__ k, GateArgs ga, const float* __restrict__ gam,
                __nv_bfloat16* __restrict__ dq, __nv_bfloat16* __restrict__ dk, float* __restrict__ dla,
                float* __restrict__ gpart, int64_t L,
                int64_t N, int64_t K, int64_t V, uint32_t stagger_ns, uint32_t n_first, int* err) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    BwdBars& bar = *reinterpret_cast<BwdBars*>(base + KH_OFF + 2 * PIECE);
    volatile int* abort_flag = &bar.abort_flag;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int i = blockIdx.x, kh = blockIdx.y;
    const int64_t bh = blockIdx.z;
    const int64_t t0 = int64_t(i) * C;
    const int nvalid = int(L - t0 < C ? L - t0 : C);
    const int nvb = int(V / 64);
    if (threadIdx.x == 0) {
        for (int s = 0; s < NSTAGE; ++s) {
            mbar_init(&bar.full[s], 1);
            mbar_init(&bar.empty[s], 1 + 128);  // MMA commit + the 128 row threads
        }
        mbar_init(&bar.pro_full, 1);
        mbar_init(&bar.accA, 1);
        mbar_init(&bar.qt_full, 1);
        mbar_init(&bar.qk_full, 1);
        mbar_init(&bar.dpm_ready, 128);
        mbar_init(&bar.khat_ready, 128);
        mbar_init(&bar.xd_ready, 128);
        mbar_init(&bar.accB, 1);
        mbar_init(&bar.drain, 1);
        bar.abort_flag = 0;
        bar.any_exact = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(&bar.tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bar.tmem_slot;
    // programmatic dependent launch: the prologue above overlapped the previous kernel's tail;
    // nothing below touches global memory before that kernel has completed
    if (threadIdx.x == 0) {  // tensor maps are kernel parameters: fetch them while the previous kernel drains
        tma_prefetch(&tmDO);
        tma_prefetch(&tmV);
        tma_prefetch(&tmS);
        tma_prefetch(&tmD);
        tma_prefetch(&tmQt);
        tma_prefetch(&tmQ);
        tma_prefetch(&tmK);
        tma_prefetch(&tmLA);
    }
    // dependents are triggered only after the wait, so that a dependent that reads the same inputs
    // without waiting for this kernel (the dv GEMM) finds them complete
    pdl_wait();
    pdl_launch_dependents();

    if (warp == 0) {
        if (lane == 0) {
            // The CTAs of the first wave are released together (by the dependency wait) and would stay
            // in lockstep: all streaming at once, then all in their epilogues with HBM idle. Every
            // other first-wave CTA starts a fraction of a CTA's lifetime later, so that the loads of
            // one half overlap the epilogues of the other, in this wave and in the ones that follow.
            const uint32_t lin = blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z);
            if (stagger_ns > 0 && lin < n_first && (lin & 1u)) {
                const uint64_t until = global_ns() + stagger_ns;  // bounded: the host caps stagger_ns
                while (global_ns() < until) __nanosleep(256);
            }
            // the gate prologue's inputs first: log a (dense fp32) and k (into the K^0 operand area)
            mbar_arrive_expect_tx(&bar.pro_full, (scalar_kind(GK) ? 0u : 4 * PIECE) + 2 * PIECE);
            if (!scalar_kind(GK)) tma_load_3d(base + LA_OFF, &tmLA, 128 * kh, i * C, int(bh), &bar.pro_full);
            tma_load_3d(base + KH_OFF, &tmK, 128 * kh, i * C, int(bh), &bar.pro_full);
            tma_load_3d(base + KH_OFF + PIECE, &tmK, 128 * kh + 64, i * C, int(bh), &bar.pro_full);
            bool ok = true;
            int vb = 0;
            for (; vb < nvb && ok; ++vb) {
                const int s = vb % NSTAGE;
                if (!mbar_wait(&bar.empty[s], uint32_t(((vb / NSTAGE) & 1) ^ 1), err, abort_flag)) {
                    ok = false;
                    break;
                }
                uint8_t* st = base + s * STAGE_BYTES;
                mbar_arrive_expect_tx(&bar.full[s], STAGE_BYTES);
                tma_load_3d(st, &tmDO, 64 * vb, i * C, int(bh), &bar.full[s]);
                tma_load_3d(st + PIECE, &tmV, 64 * vb, i * C, int(bh), &bar.full[s]);
                tma_load_3d(st + 2 * PIECE, &tmS, 64 * vb, 128 * kh, int(bh * N + i), &bar.full[s]);
                tma_load_3d(st + 3 * PIECE, &tmD, 64 * vb, 128 * kh, int(bh * N + i), &bar.full[s]);
            }
            // Q~ and q go where the prologue's log a tile was as soon as the prologue is done (usually
            // before the last value stage is consumed); k goes where stage 0 was once the value loop
            // (MMAs and the row warps' reads) is over
            if (ok && mbar_wait(&bar.khat_ready, 0, err, abort_flag)) {
                mbar_arrive_expect_tx(&bar.qt_full, 2 * PIECE);
                tma_load_3d(base + QT_OFF, &tmQt, 128 * kh, i * C, int(bh), &bar.qt_full);
                tma_load_3d(base + QT_OFF + PIECE, &tmQt, 128 * kh + 64, i * C, int(bh), &bar.qt_full);
                // raw q and k tiles for the elementwise epilogue (one barrier for both)
                mbar_arrive_expect_tx(&bar.qk_full, 4 * PIECE);
                for (int h = 0; h < 2; ++h)
                    tma_load_3d(base + QS_OFF + h * PIECE, &tmQ, 128 * kh + 64 * h, i * C, int(bh), &bar.qk_full);
                if (mbar_wait(&bar.accA, 0, err, abort_flag) && mbar_wait(&bar.xd_ready, 0, err, abort_flag))
                    for (int h = 0; h < 2; ++h)
                        tma_load_3d(base + KS_OFF + h * PIECE, &tmK, 128 * kh + 64 * h, i * C, int(bh), &bar.qk_full);
                mbar_drain(&bar.qt_full, 0);
                mbar_drain(&bar.qk_full, 0);
            } else if (!ok) {
                for (int w = vb - NSTAGE; w < vb; ++w)
                    if (w >= 0) mbar_drain(&bar.full[w % NSTAGE], uint32_t((w / NSTAGE) & 1));
            }
            mbar_drain(&bar.pro_full, 0);
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
                const uint32_t st = smem_u32(base + s * STAGE_BYTES);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const uint32_t acc = (vb > 0 || kk > 0) ? 1u : 0u;
                    const uint64_t dO_ = sdesc_sw128(st + kk * 32, 16, 1024);
                    const uint64_t v_ = sdesc_sw128(st + PIECE + kk * 32, 16, 1024);
                    const uint64_t S_ = sdesc_sw128(st + 2 * PIECE + kk * 32, 16, 1024);
                    const uint64_t D_ = sdesc_sw128(st + 3 * PIECE + kk * 32, 16, 1024);
                    mma_bf16(tmem + 0, dO_, v_, id, acc);    // dP[j][s]     = dO v^T
                    mma_bf16(tmem + 128, S_, dO_, id, acc);  // dQ^T[c][j]  = S dO^T
                    mma_bf16(tmem + 256, D_, v_, id, acc);   // dK~^T[c][s] = D v^T
                }
                mma_commit(&bar.empty[s]);
            }
            if (ok) mma_commit(&bar.accA);
            ok = ok && mbar_wait(&bar.dpm_ready, 0, err, abort_flag) &&
                 mbar_wait(&bar.khat_ready, 0, err, abort_flag) && mbar_wait(&bar.qt_full, 0, err, abort_flag);
            if (ok) {
                tc_fence_after();
                const uint32_t dpm = smem_u32(base + DPM_OFF), qt = smem_u32(base + QT_OFF);
                const uint32_t kh0 = smem_u32(base + KH_OFF);
                // The masked dP is lower triangular (s <= j), so a 16-token slice of the contraction only
                // reaches part of the output: token slice kk of s feeds the dq columns j >= 16 kk, token
                // slice kk of j feeds the dk columns s < 16 (kk + 1). The dk slices run from the last,
                // whose MMA spans (and so initialises) every column.
#pragma unroll
                for (int kk = 0; kk < C / 16; ++kk) {
                    // dQ^T[c][j] += sum_s K^0[s][c] dP[j][s] for j >= 16 kk: A = K^0 (MN-major), B = dP
                    // (K-major) from row j = 16 kk
                    // scalar gate kinds: A = the raw k tile and a decay-weighted dP, into its own accumulator
                    // (columns 384.., initialised by the first slice, which spans every column)
                    const int j0 = 16 * kk;
                    mma_bf16(tmem + (scalar_kind(GK) ? 384u : 128u) + uint32_t(j0), sdesc_sw128(kh0 + kk * 2048, PIECE, 1024),
                             sdesc_sw128(dpm + (kk / 4) * PIECE + (kk % 4) * 32 + j0 * 128, 16, 1024),
                             idesc_bf16_f32(128, C - j0, true, false), (scalar_kind(GK) && kk == 0) ? 0u : 1u);
                    // dKi^T[c][s] = sum_j Q~[j][c] dP[j][s] for s < 16 (k + 1), k = 7 - kk: A = Q~
                    // (MN-major), B = dP (MN-major)
                    const int k = C / 16 - 1 - kk;
                    mma_bf16(tmem + 0, sdesc_sw128(qt + k * 2048, PIECE, 1024),
                             sdesc_sw128(dpm + k * 2048, PIECE, 1024), idesc_bf16_f32(128, 16 * (k + 1), true, true),
                             kk > 0 ? 1u : 0u);
                }
                mma_commit(&bar.accB);
            }
            mma_commit(&bar.drain);
            mbar_drain(&bar.drain, 0);
        }
    } else {
        // ---- warps 2-17: thread = key channel c of this CTA's 128 (TMEM lane c); warps 2-5 are
        // the row warps, warps 6-9 the gate warps, warps 10-17 join for the final phase only; each
        // group of four warps covers the four lane quadrants
        const int q4 = warp & 3;
        const int c = 32 * q4 + lane;
        const bool row_warp = warp < 6;
        const bool gate_warp = warp >= 6 && warp < 10;
        const int fgrp = (warp - 2) >> 2;  // final-phase group: tokens 32 fgrp .. 32 fgrp + 31
        const uint32_t lane_off = uint32_t(32 * q4) << 16;
        const int64_t chg = int64_t(128) * kh + c;
        // scalar gate kinds have no range bound: their intra terms are weighted by the decay in fp32
        const bool safe = scalar_kind(GK) || gam[(bh * N + i) * K + chg] >= kSafeGam;
        const int64_t rb = (bh * L + t0) * K + chg;
        // log alpha of token t (< nvalid) of this thread's channel, for the exact path (per-channel kinds)
        const float* lap = ga.g + rb;
        auto gate_t = [&](int t) -> float {
            const float x = lap[int64_t(t) * K];
            return la_floor(GK == kGatePreact ? logsigmoid_f(x) * ga.inv_tau : x);
        };
        if (row_warp) {
            // x_c = sum_v D_i[c,v] S_[i][c,v] from the staged tiles
            float x = 0.f;
            bool ok = true;
            for (int vb = 0; vb < nvb; ++vb) {
                const int s = vb % NSTAGE;
                if (!mbar_wait(&bar.full[s], uint32_t((vb / NSTAGE) & 1), err, abort_flag)) {
                    ok = false;
                    break;
                }
                const uint8_t* st = base + s * STAGE_BYTES;
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) {
                    const uint32_t off = uint32_t(c) * 128u + uint32_t((ch ^ (c & 7)) * 16);
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
            bar.xd[c] = x;
            mbar_arrive(&bar.xd_ready);
            // dP epilogue: thread = token row r (= c), mask s > r, bf16, swizzled tile; scalar gate kinds
            // weight each term by its decay e^{b_r - b_s} (<= 1), so that the intra products take the raw
            // q and k
            const int r = c;
            // tcgen05.ld is warp-collective: the condition must be the same for the whole warp
            if (__all_sync(0xffffffffu, ok && mbar_wait(&bar.accA, 0, err, abort_flag) &&
                                            (!scalar_kind(GK) || mbar_wait(&bar.khat_ready, 0, err, abort_flag)))) {
                tc_fence_after();
                const float br = scalar_kind(GK) ? bar.btab[r] : 0.f;
#pragma unroll 1
                for (int c16 = 0; c16 < C / 16; ++c16) {
                    float y[16];
                    tmem_ld16(tmem + lane_off + uint32_t(16 * c16), y);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const int sc = 16 * c16 + e;
                        float w = y[e];
                        if (scalar_kind(GK)) w *= exp2_ftz(fminf(br - bar.btab[sc], 0.f));
                        y[e] = sc <= r ? w : 0.f;
                    }
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        const int c8 = 2 * (c16 & 3) + hh;  // 16-byte chunk within the 64-column piece
                        *reinterpret_cast<uint4*>(base + DPM_OFF + (c16 >> 2) * PIECE + uint32_t(r) * 128u +
                                                  uint32_t((c8 ^ (r & 7)) * 16)) =
                            make_uint4(pack_bf16x2(y[8 * hh], y[8 * hh + 1]), pack_bf16x2(y[8 * hh + 2], y[8 * hh + 3]),
                                       pack_bf16x2(y[8 * hh + 4], y[8 * hh + 5]),
                                       pack_bf16x2(y[8 * hh + 6], y[8 * hh + 7]));
                    }
                }
                fence_proxy_async_smem();
                tc_fence_before();
                mbar_arrive(&bar.dpm_ready);
            }
        } else if (gate_warp) {
            // per-chunk cumsum along the tokens from the staged tiles (rows past the end of the
            // sequence are zero-filled by TMA) in base-2 units, e^x = 2^(x log2 e); gate table into
            // TMEM; the k tile becomes the K^0 operand in place
            const bool pro = __all_sync(0xffffffffu, mbar_wait(&bar.pro_full, 0, err, abort_flag));
            const float* sLA = reinterpret_cast<const float*>(base + LA_OFF);
            float B = 0.f;
#pragma unroll 1
            for (int g = 0; g < C / 16 && pro; ++g) {
                float tb[16];
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    // the loads of 8 tokens first, so that none waits behind a store of the group
                    float lv[8], kv[8];
#pragma unroll
                    for (int r = 0; r < 8; ++r) {
                        const int t = 16 * g + 8 * h + r;
                        if (scalar_kind(GK)) {  // one decay per token (or per head) for every channel
                            lv[r] = t < nvalid ? la_floor(GK == kGateScalar ? ga.g[bh * L + t0 + t] : ga.g[bh % ga.H])
                                               : 0.f;
                        } else {
                            // zero past the end of the sequence (TMA fill): a zero log alpha, except that the
                            // pre-activation's zero must be masked explicitly
                            const float x = sLA[t * C + c];
                            if (GK == kGatePreact) lv[r] = t < nvalid ? la_floor(logsigmoid_f(x) * ga.inv_tau) : 0.f;
                            else lv[r] = la_floor(x);
                            kv[r] = __bfloat162float(
                                *reinterpret_cast<const __nv_bfloat16*>(base + KH_OFF + tile_off(t, c)));
                        }
                    }
#pragma unroll
                    for (int r = 0; r < 8; ++r) {
                        B += lv[r] * kLog2e;
                        if (scalar_kind(GK)) {
                            if (c == 0) bar.btab[16 * g + 8 * h + r] = B;
                        } else {
                            const float e = exp2_ftz(fminf(-B, (kSafeDecay + 1.f) * kLog2e));  // e^{-B}; used when safe
                            tb[8 * h + r] = safe ? e : B;
                            kv[r] = safe ? kv[r] * e : 0.f;
                        }
                    }
                    if (!scalar_kind(GK)) {
#pragma unroll
                        for (int r = 0; r < 8; ++r)  // K^0 in place of k
                            *reinterpret_cast<__nv_bfloat16*>(base + KH_OFF + tile_off(16 * g + 8 * h + r, c)) =
                                __float2bfloat16_rn(kv[r]);
                    }
                }
                if (!scalar_kind(GK)) tmem_st16(tmem + lane_off + 384u + uint32_t(16 * g), tb);
            }
            if (__any_sync(0xffffffffu, !safe) && lane == 0) atomicOr(&bar.any_exact, 1);
            tmem_wait_st();
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&bar.khat_ready);
        }
        // ---- final phase, warps 2-17: four groups of 32 tokens.
        float* rbuf = reinterpret_cast<float*>(base + RB_OFF);  // [t][c]: exact dq terms, then r
        auto xk = [&](int t) -> float* {                        // [t][c]: exact dk terms
            return reinterpret_cast<float*>(base + (t < C / 2 ? QT_OFF : KH_OFF)) + (t & (C / 2 - 1)) * C + c;
        };
        auto qs = [&](int t) -> float {
            return __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(base + QS_OFF + tile_off(t, c)));
        };
        auto ks = [&](int t) -> float {
            return __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(base + KS_OFF + tile_off(t, c)));
        };
        // dpm_ready is waited on directly so that the masked dP tile the exact path reads is
        // ordered before it by this thread's own acquire
        const bool ok = __all_sync(0xffffffffu, mbar_wait(&bar.accB, 0, err, abort_flag) &&
                                                    mbar_wait(&bar.xd_ready, 0, err, abort_flag) &&
                                                    mbar_wait(&bar.dpm_ready, 0, err, abort_flag) &&
                                                    mbar_wait(&bar.qk_full, 0, err, abort_flag));
        if (gate_warp && ok && __any_sync(0xffffffffu, !safe)) {
            // channels beyond the bound: intra terms one by one in log space, for the whole warp
            // (the results are used by those lanes only)
            auto dpm = [&](int row, int col) -> float {
                return __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(base + DPM_OFF + tile_off(row, col)));
            };
#pragma unroll 1
            for (int t = 0; t < C; ++t) {
                float eq = 0.f, ek = 0.f, d = 0.f;
#pragma unroll 1
                for (int j = t; j >= 0; --j) {
                    eq += dpm(t, j) * ks(j) * __expf(fminf(d, 0.f));
                    d += j < nvalid ? gate_t(j) : 0.f;
                }
                d = 0.f;
#pragma unroll 1
                for (int j = t; j < C; ++j) {
                    if (j > t) d += j < nvalid ? gate_t(j) : 0.f;
                    ek += dpm(j, t) * qs(j) * __expf(fminf(d, 0.f));
                }
                rbuf[t * C + c] = eq;
                *xk(t) = ek;
            }
        }
        named_sync(3, kFinal);
        float* xch = reinterpret_cast<float*>(base + DPM_OFF);  // free once the exact pass is done
        // dq and dk are staged (bf16, 128-byte swizzle) over the Q~ and K^0 tiles and written by TMA
        // stores, unless those areas hold exact-path terms
        const bool stage = bar.any_exact == 0;
        // one thread per group of 32 tokens issues that group's TMA stores (rows past the end of the
        // sequence are clipped by the TMA unit; a group entirely past it stores nothing)
        const bool issuer = ((warp - 2) & 3) == 0 && lane == 0;
        const bool grp_rows = 32 * fgrp < nvalid;
        const int tlo = 32 * fgrp;
        float kin = 0.f, rsum = 0.f;  // sum_s K~_s (v_s D_i^T) and sum_s r_s over this group
        float eGam = 0.f, Gam = 0.f;  // Gamma in base-2 units
        if (ok) {
            tc_fence_after();
            if (scalar_kind(GK)) {
                // Gamma = b at the chunk's last row (rows past the end of the sequence add nothing)
                Gam = bar.btab[C - 1];
                eGam = exp2_ftz(fminf(Gam, 0.f));
            } else {
                // Gamma from the last column of the gate table (e^{-Gamma}, or Gamma itself)
                float v8[8];
                tmem_ld8(tmem + lane_off + 504u, v8);
                tmem_wait_ld();
                Gam = safe ? 0.f : v8[7];
                eGam = safe ? __fdividef(1.f, v8[7]) : exp2_ftz(fminf(v8[7], 0.f));
            }
            // tokens of the group in reverse order: rbuf keeps the suffix sum of r within the group,
            // the carry from later groups and chunks is added once every group's sum is known
            auto run = [&](auto all_safe) {
#pragma unroll 1
                for (int g = tlo / 8 + 3; g >= tlo / 8; --g) {
                    float vQ[8], vJ[8], vI[8], vT[8];
                    tmem_ld8(tmem + lane_off + 128u + uint32_t(8 * g), vQ);
                    tmem_ld8(tmem + lane_off + 256u + uint32_t(8 * g), vJ);
                    tmem_ld8(tmem + lane_off + 0u + uint32_t(8 * g), vI);
                    tmem_ld8(tmem + lane_off + 384u + uint32_t(8 * g), vT);
                    tmem_wait_ld();
                    // loads of the 8 tokens first, so that none waits behind a store of the group
                    float qv[8], kv[8];
#pragma unroll
                    for (int r = 0; r < 8; ++r) {
                        qv[r] = qs(8 * g + r);
                        kv[r] = ks(8 * g + r);
                    }
#pragma unroll
                    for (int r = 7; r >= 0; --r) {
                        const int t = 8 * g + r;
                        float eGB, dqv, dkv;
                        if (scalar_kind(GK)) {
                            // inter parts carry the decay factors, the intra accumulators (raw q, k and a
                            // decay-weighted dP) none: vT holds the intra part of dq
                            const float b2 = bar.btab[t];
                            eGB = exp2_ftz(fminf(Gam - b2, 0.f));
                            dqv = fmaf(exp2_ftz(fminf(b2, 0.f)), vQ[r], vT[r]);
                            dkv = fmaf(eGB, vJ[r], vI[r]);
                        } else if (decltype(all_safe)::value || safe) {
                            const float e = vT[r];  // e^{-B_t}
                            eGB = eGam * e;
                            dqv = __fdividef(vQ[r], e);
                            dkv = fmaf(eGB, vJ[r], e * vI[r]);
                        } else {
                            const float Bt = vT[r];
                            eGB = exp2_ftz(fminf(Gam - Bt, 0.f));
                            dqv = exp2_ftz(fminf(Bt, 0.f)) * vQ[r] + rbuf[t * C + c];
                            dkv = eGB * vJ[r] + *xk(t);
                        }
                        kin = fmaf(kv[r] * eGB, vJ[r], kin);
                        rsum += fmaf(qv[r], dqv, -kv[r] * dkv);
                        rbuf[t * C + c] = rsum;
                        if (stage) {
                            *reinterpret_cast<__nv_bfloat16*>(base + QT_OFF + tile_off(t, c)) = __float2bfloat16_rn(dqv);
                            *reinterpret_cast<__nv_bfloat16*>(base + KH_OFF + tile_off(t, c)) = __float2bfloat16_rn(dkv);
                        } else if (t < nvalid) {
                            dq[rb + int64_t(t) * K] = __float2bfloat16_rn(dqv);
                            dk[rb + int64_t(t) * K] = __float2bfloat16_rn(dkv);
                        }
                    }
                }
            };
            if (__all_sync(0xffffffffu, safe))
                run(std::true_type{});
            else
                run(std::false_type{});
            xch[128 * fgrp + c] = kin;
            xch[512 + 128 * fgrp + c] = rsum;
        }
        fence_proxy_async_smem();
        named_sync(4 + fgrp, 128);
        if (issuer && ok && stage && grp_rows) {
            for (int h = 0; h < 2; ++h) {
                tma_store_3d(&tmDQ, 128 * kh + 64 * h, i * C + tlo, int(bh), base + QT_OFF + h * PIECE + tlo * 128);
                tma_store_3d(&tmDK, 128 * kh + 64 * h, i * C + tlo, int(bh), base + KH_OFF + h * PIECE + tlo * 128);
            }
            bulk_commit();
        }
        named_sync(3, kFinal);  // every group's sums are in xch
        if (ok) {
            // the carry from all later chunks is e^Gamma x_c + sum_s K~_s (v_s D_i^T); the later
            // groups of this chunk add their sums of r. dlog a goes straight to global memory: a
            // warp writes 32 consecutive channels (128 bytes) of one token per store
            float carry = eGam * bar.xd[c];
#pragma unroll
            for (int f = 0; f < 4; ++f) carry += xch[128 * f + c] + (f > fgrp ? xch[512 + 128 * f + c] : 0.f);
            float dv[32];
#pragma unroll
            for (int u = 0; u < 32; ++u) {
                dv[u] = rbuf[(tlo + u) * C + c] + carry;
                if (scalar_kind(GK) && tlo + u >= nvalid) dv[u] = 0.f;  // rows past the end add nothing
            }
            if (scalar_kind(GK)) {
                // sum over this CTA's 128 channels per token: across the warp's 32 lanes by a butterfly that
                // leaves token tlo + l's sum in lane l, then over the group's 4 warps in fixed order
#pragma unroll
                for (int kb = 16; kb >= 1; kb >>= 1) {
#pragma unroll
                    for (int j = 0; j < kb; ++j) {
                        const bool hi = (lane & kb) != 0;
                        const float give = hi ? dv[j] : dv[j + kb];
                        const float got = __shfl_xor_sync(0xffffffffu, give, kb);
                        dv[j] = (hi ? dv[j + kb] : dv[j]) + got;
                    }
                }
                xch[2048 + (4 * fgrp + q4) * 32 + lane] = dv[0];
            } else {
#pragma unroll
                for (int u = 0; u < 32; ++u)
                    if (tlo + u < nvalid) {
                        const int64_t o = rb + int64_t(tlo + u) * K;
                        // preact: dL/dz = dL/dlog alpha * sigmoid(-z) / tau
                        dla[o] = GK == kGatePreact ? dv[u] * sigmoid_neg_f(ga.g[o]) * ga.inv_tau : dv[u];
                    }
            }
        }
        if (scalar_kind(GK)) {
            named_sync(4 + fgrp, 128);
            if (ok && q4 == 0) {  // one warp per group: this CTA's partial of the gradient of tokens tlo ..
                const float* red = xch + 2048 + 4 * fgrp * 32;  // [quadrant][token] after the group sums
                const float v = red[lane] + red[32 + lane] + red[64 + lane] + red[96 + lane];
                gpart[((bh * N + i) * (K / 128) + kh) * C + tlo + lane] = v;
            }
        }
        if (issuer) bulk_wait_read_all();  // the stores finish on their own; the CTA may exit once they have read smem
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// [outer][rows][inner] bf16 tensor, box [128 rows x 64 inner], 128-byte swizzle
bool map_sw128(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t outer,
               uint32_t box_rows = 128) {
    const uint64_t dims[3] = {inner, rows, outer};
    const uint64_t strides[2] = {inner * 2, inner * rows * 2};
    const uint32_t box[3] = {64, box_rows, 1};
    return encode_tmap(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

// [outer][rows][inner] fp32 tensor, box [128 rows x 128 inner], no swizzle
bool map_f32_tile(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t outer) {
    const uint64_t dims[3] = {inner, rows, outer};
    const uint64_t strides[2] = {inner * 4, inner * rows * 4};
    const uint32_t box[3] = {128, 128, 1};
    return encode_tmap(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE);
}

constexpr size_t kSmem = 1024 + KH_OFF + 2 * PIECE + sizeof(BwdBars);
static_assert(kSmem <= 232448, "shared memory");

template <int GK>
gla_status launch_bwd_gk(const Problem& p, const CUtensorMap* m, const void* q, const void* k, const GateArgs& ga,
                         const float* gam, void* dq, void* dk, float* dla, float* gpart, cudaStream_t s) {
    auto fn = k_bwd_chunk<GK>;
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kSmem)) != cudaSuccess)
        return GLA_ERR_CUDA;
    const dim3 grid(unsigned(p.N), unsigned(p.K / 128), unsigned(p.BH));
    // one CTA per SM: stagger the first wave only when there are later waves for it to shape
    const int64_t sms = sm_count();
    const uint32_t stagger = int64_t(grid.x) * grid.y * grid.z > sms ? kStaggerNs : 0u;
    GLA_LAUNCH_PDL("tc_bwd_chunk", fn, grid, kThreads, kSmem, s, m[0], m[1], m[2], m[3], m[4], m[5], m[6], m[7], m[8],
                   m[9], static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k), ga, gam,
                   static_cast<__nv_bfloat16*>(dq), static_cast<__nv_bfloat16*>(dk), dla, gpart, p.L, p.N, p.K, p.V,
                   stagger, unsigned(sms), device_error_word());
    return GLA_OK;
}

}  // namespace

gla_status tc_bwd_chunk_launch(const Problem& p, const void* q, const void* k, const float* la, const void* dO,
                               const void* v, const __nv_bfloat16* Qt, const float* gam, const __nv_bfloat16* Sbuf,
                               const __nv_bfloat16* Dbuf, void* dq, void* dk, float* dla, float* gpart,
                               cudaStream_t s) {
    CUtensorMap m[10];
    memset(m, 0, sizeof(m));
    const uint64_t L = uint64_t(p.L), K = uint64_t(p.K), V = uint64_t(p.V), BH = uint64_t(p.BH), N = uint64_t(p.N);
    const bool sk = p.gate == kGateScalar || p.gate == kGateHead;
    // scalar gate kinds: the intra dK~ product takes the raw q tile (decay in the dP weights), and there
    // is no per-channel gate tile (its map is never used; any valid descriptor stands in)
    if (!(map_sw128(&m[0], dO, V, L, BH) && map_sw128(&m[1], v, V, L, BH) && map_sw128(&m[2], Sbuf, V, K, BH * N) &&
          map_sw128(&m[3], Dbuf, V, K, BH * N) && map_sw128(&m[4], sk ? q : static_cast<const void*>(Qt), K, L, BH) &&
          map_sw128(&m[5], q, K, L, BH) && map_sw128(&m[6], k, K, L, BH) && map_sw128(&m[7], dq, K, L, BH, 32) &&
          map_sw128(&m[8], dk, K, L, BH, 32) && (sk ? map_sw128(&m[9], k, K, L, BH) : map_f32_tile(&m[9], la, K, L, BH))))
        return GLA_ERR_CUDA;
    const GateArgs ga{la, p.gate, p.inv_tau, p.H};
    switch (p.gate) {
        case kGateScalar: return launch_bwd_gk<kGateScalar>(p, m, q, k, ga, gam, dq, dk, dla, gpart, s);
        case kGateHead: return launch_bwd_gk<kGateHead>(p, m, q, k, ga, gam, dq, dk, dla, gpart, s);
        case kGatePreact: return launch_bwd_gk<kGatePreact>(p, m, q, k, ga, gam, dq, dk, dla, gpart, s);
        default: return launch_bwd_gk<kGateChannel>(p, m, q, k, ga, gam, dq, dk, dla, gpart, s);
    }
}

}  // namespace gla
