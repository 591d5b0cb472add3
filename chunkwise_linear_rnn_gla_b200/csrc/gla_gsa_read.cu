// Gated slot attention: the read of a slot memory from its value side, on tcgen05.
//
// Both memories of gated slot attention are GLA states over the slots (mlsanity
// card for "Gated Slot Attention for Efficient Linear-Time Sequence Modeling",
// abstract: two GLA layers joined by a softmax over the slots). With the slot
// gate's per-chunk cumsum B (one column per slot), the write weights w and the
// memory M_[i] entering chunk i ([m slots x D], a stored bf16 chunk state of the
// GLA walk with key w), the memory seen by token j of the chunk, read with a
// D-vector x_j, is
//   r_j = e^{B_j} * ( M_[i] x_j^T + sum_{s<=j} (x_j . y_s) w_s e^{-B_s} )      [m]
// (y the memory's value rows). Layer one's logits are this read with x = q,
// y = k, M = the key memory; the softmax backward needs the same read of the
// value memory with x = dO, y = v (the gradient of the read weights). Both stay
// in fp32 up to the softmax (forward) or its backward (the kernel's epilogue).
//
// One CTA per (chunk, head); m = 128 slots. Over D in 64-wide pieces:
//   TMEM cols [0,128)   A1 = x y^T          (M=128 tokens, N=128 tokens; later the next layer's P)
//   TMEM cols [128,256) L  = x M_[i]^T      (N=128 slots)
// as ONE N=256 tcgen05.mma per 16-wide k step (the y piece and the M piece sit
// side by side in shared memory). The epilogue masks A1 (s <= j) into bf16 P1,
// and L += P1 Phi with Phi = w e^{-B} (token x slot, MN-major operand built by
// the CUDA cores from the gate while the loads run). A slot whose chunk decay
// passes the range bound (Gamma < -64) gets a zero Phi column and exact
// log-space intra terms. Roles (576 threads): warp 0 TMA, warp 1 TMEM owner and
// MMA issuer, 16 compute warps: the gate cumsum (4 threads per slot, 32 rows
// each), then the epilogue (4 threads per token row, 32 slot columns each; the
// softmax and <s, r> combine the four partial results through shared memory).
//
// The kernel's result x (the read weights s, or the logit gradient G) is the
// query of the next GLA layer, whose key is w under the same gate. So the
// epilogue also forms that layer's chunk-local operands, as the GLA preparation
// would: Q~ = x e^{B} (bf16, stored and staged as a K-major operand in the
// free part of the ring) and the masked score block P = Q~ Phi^T (s <= j), one
// more tcgen05.mma into TMEM cols [0,128) with Phi = w e^{-B} as the K-major B
// operand, plus exact log-space terms x_jc w_sc e^{B_jc - B_sc} for the slots
// beyond the range bound (their Phi columns are zero).

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

constexpr int C = kTcChunk;  // 128 tokens per chunk
constexpr int kSlots = 128;
constexpr uint32_t PIECE = 16384;  // [128 rows x 64 bf16] with the 128-byte swizzle
constexpr int kCW = 16;                    // compute warps
constexpr int kNT = 32 * kCW;              // compute threads
constexpr int kQ = kCW / 4;                // compute threads per slot (cumsum) and per token row (epilogue)
constexpr int kPart = C / kQ;              // rows per cumsum thread, columns per epilogue thread
constexpr int kThreadsSR = 64 + kNT;
constexpr uint32_t kTmemCols = 256;
constexpr float kBound2 = 64.f * kLog2e;  // range bound in base-2 units

struct SRBars {
    uint64_t full[2], empty[2];
    uint64_t a_full, p_ready, phi_ready, l_full, s_full, qt_ready, q_full, drain;
    uint32_t tmem_slot;
    int abort_flag;
    int any_beyond;            // some slot of the chunk is beyond the range bound
    uint32_t flag[kSlots];     // 1: the slot's chunk decay passes the range bound
    float tot[kQ][kSlots];     // cumsum: each thread's partial sum over its rows
    float red[2][kQ][C];       // epilogue: per-row partial reductions of the column groups
};

constexpr size_t kRing = size_t(2) * 3 * PIECE;          // x, y, M pieces, two stages
constexpr size_t kPhi = size_t(2) * PIECE;               // Phi [128 tokens x 128 slots] bf16
constexpr size_t kBs = size_t(C) * kSlots * sizeof(float);  // e^B, or B (base 2) beyond the bound [128 x 128] fp32
constexpr size_t kSmem = 1024 + kRing + kPhi + kBs + sizeof(SRBars);
static_assert(kSmem <= 232448, "shared memory of one block");
// the forward read's staged s rows fill the ring's first four pieces, its Q~ operand the last two
static_assert(size_t(C) * kSlots * sizeof(float) == 4 * PIECE && kRing == 6 * PIECE, "ring areas");

// The read gradient's s tile (fp32 [128 rows x 128 slots], four TMA boxes of 32 columns with the 128-byte
// swizzle) goes to the ring once the D loop is done, into the four 16 KB pieces that P1 does not use.
__device__ __forceinline__ uint32_t s_piece(int p) { return uint32_t(2 + p) * PIECE; }

// The next layer's query operand Q~ (two K-major pieces): the ring's last two pieces in the forward read
// (the staged s rows take the first four), the first two (P1's, free after the second GEMM and the exact
// terms) in the read gradient (the s tile takes the other four).
template <int MODE>
__device__ __forceinline__ uint32_t qt_piece() { return MODE == 0 ? 4u * PIECE : 0u; }

// The table entry of (t, c) lives at t * 128 + (c ^ (t & 31)): a warp reading one column over 32 rows
// (epilogue) or one row over 32 columns (cumsum) touches 32 different banks.
__device__ __forceinline__ int bs_idx(int t, int c) { return t * kSlots + (c ^ (t & 31)); }

// bf16 write weight, exactly as the elementwise kernel that feeds the GLA passes rounds it
__device__ __forceinline__ float write_weight(float la) { return __bfloat162float(__float2bfloat16_rn(1.f - __expf(la))); }

// Exact intra-chunk term of a slot beyond the range bound: sum_{s<=r} P1[r][s] w_s e^{B_r - B_s}
__device__ __noinline__ float exact_intra(const uint8_t* p1, const float* Bs, const float* la_c, int64_t m, int r,
                                          int c, float b2r) {
    float acc = 0.f;
    for (int s = 0; s <= r; ++s) {
        const uint32_t off = uint32_t(s >> 6) * PIECE + sw128_offset(uint32_t(r), uint32_t(s & 63));
        const float pv = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(p1 + off));
        const float w = write_weight(la_c[int64_t(s) * m]);
        acc = fmaf(pv * w, exp2_ftz(b2r - Bs[bs_idx(s, c)]), acc);
    }
    return acc;
}

// e^{min(B, 0)} of row r, slot c: the table holds e^B, or B itself for a slot beyond the range bound
__device__ __forceinline__ float e_b(const float* Bs, int r, int c, bool beyond) {
    const float b = Bs[bs_idx(r, c)];
    // exponents are <= 0 in exact arithmetic; the clamp absorbs cumsum rounding
    return beyond ? exp2_ftz(fminf(b, 0.f)) : fminf(b, 1.f);
}

// The next layer's query operand from this thread's 32 columns of row r: Q~ = x e^{B} (one rounding to bf16)
// into the K-major operand in shared memory (16-byte chunks) and, for a valid row, into global memory
// (qg: the row's first column of the thread). fmask: the columns' slots beyond the range bound.
__device__ __forceinline__ void put_qt(uint8_t* qop, const float* Bs, int r, int c0, uint32_t fmask, const float* x,
                                       __nv_bfloat16* qg) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        uint32_t qpk[8];
#pragma unroll
        for (int e2 = 0; e2 < 8; ++e2) {
            const int e = 16 * h + 2 * e2, c = c0 + e;
            qpk[e2] = pack_bf16x2(x[e] * e_b(Bs, r, c, (fmask >> e) & 1u),
                                  x[e + 1] * e_b(Bs, r, c + 1, (fmask >> (e + 1)) & 1u));
        }
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int c = c0 + 16 * h + 8 * j;
            *reinterpret_cast<uint4*>(qop + (c >> 6) * PIECE + sw128_offset(uint32_t(r), uint32_t(c & 63))) =
                make_uint4(qpk[4 * j], qpk[4 * j + 1], qpk[4 * j + 2], qpk[4 * j + 3]);
        }
        if (qg) st_global_v8(qg + 16 * h, qpk);
    }
}

// one TMEM column of the warp's 32 lanes
__device__ __forceinline__ float tmem_ld1(uint32_t taddr) {
    uint32_t r;
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=r"(r) : "r"(taddr));
    return __uint_as_float(r);
}
__device__ __forceinline__ void tmem_st1(uint32_t taddr, float v) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x1.b32 [%0], {%1};" ::"r"(taddr), "r"(__float_as_uint(v)) : "memory");
}

template <int MODE>
__global__ void __launch_bounds__(kThreadsSR, 1)
    k_gsa_slot_read(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmY,
                    const __grid_constant__ CUtensorMap tmM, const __grid_constant__ CUtensorMap tmS,
                    const float* __restrict__ la,
                    const float* __restrict__ s_in, __nv_bfloat16* __restrict__ s_b, float* __restrict__ s_f,
                    __nv_bfloat16* __restrict__ Qt, __nv_bfloat16* __restrict__ Pq, int64_t L, int64_t N, int64_t D,
                    int* err) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* phi = ring + kRing;
    float* Bs = reinterpret_cast<float*>(phi + kPhi);
    SRBars& bar = *reinterpret_cast<SRBars*>(reinterpret_cast<uint8_t*>(Bs) + kBs);
    volatile int* abort_flag = &bar.abort_flag;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int i = int(blockIdx.x);
    const int64_t bh = blockIdx.y;
    const int64_t t0 = int64_t(i) * C;
    const int np = int(D / 64);

    if (threadIdx.x == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bar.full[s], 1);
            mbar_init(&bar.empty[s], 1);
        }
        mbar_init(&bar.a_full, 1);
        mbar_init(&bar.p_ready, kNT);
        mbar_init(&bar.phi_ready, kNT);
        mbar_init(&bar.l_full, 1);
        mbar_init(&bar.s_full, 1);
        mbar_init(&bar.qt_ready, kNT);
        mbar_init(&bar.q_full, 1);
        mbar_init(&bar.drain, 1);
        bar.abort_flag = 0;
        bar.any_beyond = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(&bar.tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bar.tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            tma_prefetch(&tmX);
            tma_prefetch(&tmY);
            tma_prefetch(&tmM);
            int pc = 0;
            for (; pc < np; ++pc) {
                const int s = pc & 1;
                if (!mbar_wait(&bar.empty[s], uint32_t(((pc >> 1) & 1) ^ 1), err, abort_flag)) break;
                uint8_t* st = ring + s * 3 * PIECE;
                mbar_arrive_expect_tx(&bar.full[s], 3 * PIECE);
                tma_load_3d(st, &tmX, 64 * pc, int(t0), int(bh), &bar.full[s]);
                tma_load_3d(st + PIECE, &tmY, 64 * pc, int(t0), int(bh), &bar.full[s]);
                tma_load_3d(st + 2 * PIECE, &tmM, 64 * pc, 0, int(bh * N + i), &bar.full[s]);
            }
            if (pc < np) {  // gave up: let the copies already issued land before the block exits
                for (int w = pc - 2; w < pc; ++w)
                    if (w >= 0) mbar_drain(&bar.full[w & 1], uint32_t((w >> 1) & 1));
            } else if (MODE == 1 && mbar_wait(&bar.a_full, 0, err, abort_flag)) {
                // every MMA reading the ring is done: the fp32 s tile of the chunk into the pieces P1 leaves free
                tma_prefetch(&tmS);
                mbar_arrive_expect_tx(&bar.s_full, 4 * PIECE);
#pragma unroll
                for (int p2 = 0; p2 < 4; ++p2)
                    tma_load_3d(ring + s_piece(p2), &tmS, 32 * p2, int(t0), int(bh), &bar.s_full);
                if (!mbar_wait(&bar.s_full, 0, err, abort_flag)) mbar_drain(&bar.s_full, 0);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t id1 = idesc_bf16_f32(128, 256, false, false);
            const uint32_t id3 = idesc_bf16_f32(128, kSlots, false, true);
            bool ok = true;
            for (int pc = 0; pc < np && ok; ++pc) {
                const int s = pc & 1;
                ok = mbar_wait(&bar.full[s], uint32_t((pc >> 1) & 1), err, abort_flag);
                if (!ok) break;
                tc_fence_after();
                const uint32_t st = smem_u32(ring + s * 3 * PIECE);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_bf16(tmem, sdesc_sw128(st + kk * 32, 16, 1024), sdesc_sw128(st + PIECE + kk * 32, 16, 1024),
                             id1, (pc > 0 || kk > 0) ? 1u : 0u);
                mma_commit(&bar.empty[s]);
            }
            if (ok) mma_commit(&bar.a_full);
            ok = ok && mbar_wait(&bar.p_ready, 0, err, abort_flag) && mbar_wait(&bar.phi_ready, 0, err, abort_flag);
            if (ok) {
                tc_fence_after();
                const uint32_t p1 = smem_u32(ring), ph = smem_u32(phi);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_bf16(tmem + 128, sdesc_sw128(p1 + (kk / 4) * PIECE + (kk % 4) * 32, 16, 1024),
                             sdesc_sw128(ph + kk * 2048, PIECE, 1024), id3, 1u);
                mma_commit(&bar.l_full);
            }
            // the next layer's score block P = Q~ Phi^T over the slots (both operands K-major), into cols [0,128)
            ok = ok && mbar_wait(&bar.qt_ready, 0, err, abort_flag);
            if (ok) {
                tc_fence_after();
                const uint32_t qa = smem_u32(ring + qt_piece<MODE>()), ph = smem_u32(phi);
                const uint32_t id4 = idesc_bf16_f32(128, 128, false, false);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_bf16(tmem, sdesc_sw128(qa + (kk / 4) * PIECE + (kk % 4) * 32, 16, 1024),
                             sdesc_sw128(ph + (kk / 4) * PIECE + (kk % 4) * 32, 16, 1024), id4, kk > 0 ? 1u : 0u);
                mma_commit(&bar.q_full);
            }
            mma_commit(&bar.drain);
            mbar_drain(&bar.drain, 0);
        }
    } else {
        // compute warps: kQ threads per slot in the cumsum, kQ threads per token row (one column group
        // each) in the epilogue. Every named barrier below is reached by every compute thread, whatever
        // a bounded wait returned, so that no thread can wait at one for a thread that gave up.
        const int tid = threadIdx.x - 64;
        const int64_t nvalid = L - t0 < C ? L - t0 : C;
        // ---- gate cumsum: thread (slot c, part) over rows [kPart part, kPart (part + 1)); Phi = w e^{-B} ----
        {
            const int c = tid % kSlots, part = tid / kSlots;
            const int r0 = part * kPart;
            const float* lac = la + (bh * L + t0) * kSlots + c;
            float v[kPart];
#pragma unroll
            for (int e = 0; e < kPart; ++e) v[e] = (r0 + e < nvalid) ? lac[int64_t(r0 + e) * kSlots] : 0.f;
            float run = 0.f;
#pragma unroll
            for (int e = 0; e < kPart; ++e) run = fmaf(la_floor(v[e]), kLog2e, run);
            bar.tot[part][c] = run;
            named_sync(1, kNT);
            float off = 0.f, gamma = 0.f;
#pragma unroll
            for (int p2 = 0; p2 < kQ; ++p2) {
                const float x = bar.tot[p2][c];
                if (p2 < part) off += x;
                gamma += x;
            }
            const bool beyond = gamma < -kBound2;  // the same for the kQ threads of the slot
            if (part == 0) {
                bar.flag[c] = beyond ? 1u : 0u;
                if (beyond) atomicOr(&bar.any_beyond, 1);
            }
            uint8_t* pp = phi + (c >> 6) * PIECE;
            run = off;
#pragma unroll
            for (int e = 0; e < kPart; ++e) {
                const int t = r0 + e;
                run = fmaf(la_floor(v[e]), kLog2e, run);
                // e^B for a slot within the bound (the epilogue's factor, formed here under the loads); the
                // exponent itself (base 2) for a slot beyond it, whose exact terms take differences
                Bs[bs_idx(t, c)] = beyond ? run : exp2_ftz(run);
                const float f = (!beyond && t < nvalid) ? write_weight(v[e]) * exp2_ftz(-run) : 0.f;
                *reinterpret_cast<__nv_bfloat16*>(pp + sw128_offset(uint32_t(t), uint32_t(c & 63))) =
                    __float2bfloat16_rn(f);
            }
            fence_proxy_async_smem();
            mbar_arrive(&bar.phi_ready);
        }
        named_sync(1, kNT);  // B and the flags are complete for every slot
        // ---- epilogue: thread = token row r, column group cg ----
        const int q4 = warp & 3, cg = (warp - 2) / 4;
        const int r = 32 * q4 + lane;
        const int c0 = cg * kPart;
        const uint32_t lane_off = uint32_t(32 * q4) << 16;
        const int64_t t = t0 + r;
        const bool valid = r < nvalid;
        uint32_t fmask = 0;  // slots of the column group beyond the range bound (the same across the warp)
#pragma unroll
        for (int e = 0; e < kPart; ++e) fmask |= bar.flag[c0 + e] ? (1u << e) : 0u;
        const bool ok_a = __all_sync(0xffffffffu, mbar_wait(&bar.a_full, 0, err, abort_flag));
        if (ok_a) {
            tc_fence_after();
            // P1 = A1 masked to s <= r, bf16, into the ring's first stage (every MMA reading the ring is done)
#pragma unroll
            for (int cb = 0; cb < kPart / 16; ++cb) {
                float a[16];
                tmem_ld16(tmem + lane_off + uint32_t(c0 + 16 * cb), a);
                tmem_wait_ld();
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int s0 = c0 + 16 * cb + 8 * h;
                    uint32_t pk[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float lo = (s0 + 2 * e <= r) ? a[8 * h + 2 * e] : 0.f;
                        const float hi = (s0 + 2 * e + 1 <= r) ? a[8 * h + 2 * e + 1] : 0.f;
                        pk[e] = pack_bf16x2(lo, hi);
                    }
                    uint8_t* dst = ring + (s0 >> 6) * PIECE + sw128_offset(uint32_t(r), uint32_t(s0 & 63));
                    *reinterpret_cast<uint4*>(dst) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
        }
        mbar_arrive(&bar.p_ready);
        const bool ok = ok_a && __all_sync(0xffffffffu, mbar_wait(&bar.l_full, 0, err, abort_flag));
        float rr[kPart];
#pragma unroll
        for (int e = 0; e < kPart; ++e) rr[e] = 0.f;
        if (ok) {
            tc_fence_after();
            // slots beyond the range bound get their final value first (warp-uniform single-column accesses):
            // the inter part times e^{B_r} plus the exact intra-chunk sum
#pragma unroll 1
            for (uint32_t f = fmask; f; f &= f - 1) {
                const int c = c0 + __ffs(int(f)) - 1;
                const uint32_t col = tmem + lane_off + uint32_t(128 + c);
                float x = tmem_ld1(col);
                tmem_wait_ld();
                const float b2 = Bs[bs_idx(r, c)];
                x = valid ? fmaf(x, exp2_ftz(b2),
                                 exact_intra(ring, Bs, la + (bh * L + t0) * kSlots + c, kSlots, r, c, b2))
                          : 0.f;
                tmem_st1(col, x);
                tmem_wait_st();
            }
#pragma unroll
            for (int cb = 0; cb < kPart / 16; ++cb) {
                tmem_ld16(tmem + lane_off + uint32_t(128 + c0 + 16 * cb), rr + 16 * cb);
                tmem_wait_ld();
            }
#pragma unroll
            for (int e = 0; e < kPart; ++e)
                if (!((fmask >> e) & 1u)) rr[e] *= Bs[bs_idx(r, c0 + e)];
        }
        if (MODE == 0) {
            // softmax over the row's 128 slots, spread over kQ threads
            float mx = rr[0];
#pragma unroll
            for (int e = 1; e < kPart; ++e) mx = fmaxf(mx, rr[e]);
            bar.red[0][cg][r] = mx;
            named_sync(1, kNT);
#pragma unroll
            for (int g2 = 0; g2 < kQ; ++g2) mx = fmaxf(mx, bar.red[0][g2][r]);
            float sum = 0.f;
#pragma unroll
            for (int e = 0; e < kPart; ++e) {
                rr[e] = __expf(rr[e] - mx);
                sum += rr[e];
            }
            bar.red[1][cg][r] = sum;
            named_sync(1, kNT);
            sum = 0.f;
#pragma unroll
            for (int g2 = 0; g2 < kQ; ++g2) sum += bar.red[1][g2][r];
            const float inv = 1.f / sum;
#pragma unroll
            for (int e = 0; e < kPart; ++e) rr[e] = (ok && valid) ? rr[e] * inv : 0.f;
            // the next layer's query operand first, so that its MMA runs under the stores below
            put_qt(ring + qt_piece<MODE>(), Bs, r, c0, fmask, rr,
                   (ok && valid) ? Qt + (bh * L + t) * kSlots + c0 : nullptr);
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&bar.qt_ready);
            // s staged in the ring's first four pieces (free: the second GEMM has read P1; the exact terms above
            // are done, every thread having passed the first exchange) in 16-byte chunks, chunk j of row t at
            // t * 128 + 4 (j ^ (t % 8)) floats, so that a warp writing one chunk over 32 rows, and one reading a
            // row, touch every bank once per 8 lanes; then whole rows are stored, one 16-byte (fp32) and one
            // 8-byte (bf16) store per lane and row
            float* stg = reinterpret_cast<float*>(ring);
            if (ok) {
#pragma unroll
                for (int j = 0; j < kPart / 4; ++j)
                    *reinterpret_cast<float4*>(stg + r * kSlots + 4 * (((c0 >> 2) + j) ^ (r & 7))) =
                        make_float4(rr[4 * j], rr[4 * j + 1], rr[4 * j + 2], rr[4 * j + 3]);
            }
            named_sync(1, kNT);
            if (ok) {
                for (int rho = warp - 2; rho < nvalid; rho += kCW) {
                    const float4 x = *reinterpret_cast<const float4*>(stg + rho * kSlots + 4 * (lane ^ (rho & 7)));
                    *reinterpret_cast<float4*>(s_f + (bh * L + t0 + rho) * kSlots + 4 * lane) = x;
                    *reinterpret_cast<uint2*>(s_b + (bh * L + t0 + rho) * kSlots + 4 * lane) =
                        make_uint2(pack_bf16x2(x.x, x.y), pack_bf16x2(x.z, x.w));
                }
            }
        } else {
            // G = s * (r - <s, r>), s from the tile in shared memory (piece cg: this thread's 32 columns;
            // 16-byte chunk j of row r at (j ^ (r % 8)) * 16)
            const bool ok_s = ok && __all_sync(0xffffffffu, mbar_wait(&bar.s_full, 0, err, abort_flag));
            const uint8_t* sp = ring + s_piece(cg) + r * 128;
            float4 sv[kPart / 4];
#pragma unroll
            for (int e4 = 0; e4 < kPart / 4; ++e4)
                sv[e4] = ok_s ? *reinterpret_cast<const float4*>(sp + ((e4 ^ (r & 7)) << 4)) : make_float4(0.f, 0.f, 0.f, 0.f);
            float dot = 0.f;
#pragma unroll
            for (int e4 = 0; e4 < kPart / 4; ++e4) {
                dot = fmaf(sv[e4].x, rr[4 * e4], dot);
                dot = fmaf(sv[e4].y, rr[4 * e4 + 1], dot);
                dot = fmaf(sv[e4].z, rr[4 * e4 + 2], dot);
                dot = fmaf(sv[e4].w, rr[4 * e4 + 3], dot);
            }
            bar.red[0][cg][r] = dot;
            named_sync(1, kNT);
            dot = 0.f;
#pragma unroll
            for (int g2 = 0; g2 < kQ; ++g2) dot += bar.red[0][g2][r];
#pragma unroll
            for (int e4 = 0; e4 < kPart / 4; ++e4) {
                const float4 x = sv[e4];
                float* y = rr + 4 * e4;
                const bool on = ok_s && valid;
                y[0] = on ? x.x * (y[0] - dot) : 0.f;
                y[1] = on ? x.y * (y[1] - dot) : 0.f;
                y[2] = on ? x.z * (y[2] - dot) : 0.f;
                y[3] = on ? x.w * (y[3] - dot) : 0.f;
            }
            // the next layer's query operand goes where P1 was: every thread has passed the exact terms
            // (which read P1) before the exchange above
            put_qt(ring + qt_piece<MODE>(), Bs, r, c0, fmask, rr,
                   (ok && valid) ? Qt + (bh * L + t) * kSlots + c0 : nullptr);
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&bar.qt_ready);
            if (ok_s && valid) {
                __nv_bfloat16* db = s_b + (bh * L + t) * kSlots + c0;
#pragma unroll
                for (int c16 = 0; c16 < kPart / 16; ++c16) {
                    uint32_t wb[8];
#pragma unroll
                    for (int e2 = 0; e2 < 8; ++e2)
                        wb[e2] = pack_bf16x2(rr[16 * c16 + 2 * e2], rr[16 * c16 + 2 * e2 + 1]);
                    st_global_v8(db + 16 * c16, wb);
                }
            }
        }
        // ---- the next layer's score block P: thread = row r, P columns c0 .. c0 + 31 ----
        // every row of x is stored: the exact terms below read other threads' columns back
        __threadfence_block();
        named_sync(1, kNT);
        if (__all_sync(0xffffffffu, ok && mbar_wait(&bar.q_full, 0, err, abort_flag))) {
            tc_fence_after();
            float pv[kPart];
#pragma unroll
            for (int cb = 0; cb < kPart / 16; ++cb) tmem_ld16(tmem + lane_off + uint32_t(c0 + 16 * cb), pv + 16 * cb);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < kPart; ++e) pv[e] = (c0 + e <= r) ? pv[e] : 0.f;
            if (bar.any_beyond && valid) {
                // slots beyond the range bound: x_rc w_sc e^{B_rc - B_sc} for s <= r, in log space
                const float* lab = la + (bh * L + t0) * kSlots;
                const __nv_bfloat16* xrow = s_b + (bh * L + t) * kSlots;
#pragma unroll 1
                for (int c = 0; c < kSlots; ++c) {
                    if (!bar.flag[c]) continue;
                    const float xr = __bfloat162float(xrow[c]);
                    const float b2r = Bs[bs_idx(r, c)];
#pragma unroll
                    for (int e = 0; e < kPart; ++e) {
                        const int sj = c0 + e;
                        if (sj <= r)
                            pv[e] = fmaf(xr * write_weight(lab[int64_t(sj) * kSlots + c]),
                                         exp2_ftz(fminf(b2r - Bs[bs_idx(sj, c)], 0.f)), pv[e]);
                    }
                }
            }
            __nv_bfloat16* dp = Pq + ((bh * N + i) * C + r) * C + c0;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                uint32_t pk[8];
#pragma unroll
                for (int e2 = 0; e2 < 8; ++e2) pk[e2] = pack_bf16x2(pv[16 * h + 2 * e2], pv[16 * h + 2 * e2 + 1]);
                st_global_v8(dp + 16 * h, pk);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// Gate preparation of the slot memories' walks, per (chunk, head): the write weight
// w = bf16(1 - e^{log a}), the walk operand K~ = w e^{Gamma - B} (B the per-chunk cumsum of log a, Gamma
// its last row) and e^Gamma, as the GLA preparation kernel forms them for a GLA key w. Both GLA layers of
// the method have key w under this gate, so K~ and e^Gamma also go to the second layer's buffers when
// given (Kt2, gam2). kQ threads per slot (32 rows each): partial sums, a prefix over them through shared
// memory, then every row's values.
constexpr int kGateThreads = kSlots * kQ;

__global__ void __launch_bounds__(kGateThreads, 2) k_gsa_gate_prep(const float* __restrict__ la,
                                                                __nv_bfloat16* __restrict__ w,
                                                                __nv_bfloat16* __restrict__ Kt,
                                                                float* __restrict__ gam,
                                                                __nv_bfloat16* __restrict__ Kt2,
                                                                float* __restrict__ gam2, int64_t L, int64_t N) {
    __shared__ float tot[kQ][kSlots];
    const int c = threadIdx.x % kSlots, part = threadIdx.x / kSlots, i = blockIdx.x;
    const int r0 = part * kPart;
    const int64_t bh = blockIdx.y, t0 = int64_t(i) * C;
    const int64_t nvalid = L - t0 < C ? L - t0 : C;
    const int64_t base = (bh * L + t0) * kSlots + c;
    float v[kPart];
#pragma unroll
    for (int e = 0; e < kPart; ++e) v[e] = r0 + e < nvalid ? la[base + int64_t(r0 + e) * kSlots] : 0.f;
    float run = 0.f;
#pragma unroll
    for (int e = 0; e < kPart; ++e) run += la_floor(v[e]);
    tot[part][c] = run;
    __syncthreads();
    float off = 0.f, gamma = 0.f;
#pragma unroll
    for (int p2 = 0; p2 < kQ; ++p2) {
        const float x = tot[p2][c];
        if (p2 < part) off += x;
        gamma += x;
    }
    // exponents are <= 0 in exact arithmetic; the clamps absorb cumsum rounding
    if (part == 0) {
        const float eg = __expf(fminf(gamma, 0.f));
        gam[(bh * N + i) * kSlots + c] = eg;
        if (gam2) gam2[(bh * N + i) * kSlots + c] = eg;
    }
    run = off;
#pragma unroll
    for (int e = 0; e < kPart; ++e) {
        const int t = r0 + e;
        run += la_floor(v[e]);
        if (t < nvalid) {
            const __nv_bfloat16 wb = __float2bfloat16_rn(1.f - __expf(v[e]));
            const __nv_bfloat16 kt = __float2bfloat16_rn(__bfloat162float(wb) * __expf(fminf(gamma - run, 0.f)));
            w[base + int64_t(t) * kSlots] = wb;
            Kt[base + int64_t(t) * kSlots] = kt;
            if (Kt2) Kt2[base + int64_t(t) * kSlots] = kt;
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

bool tc_gsa_slot_read_supported(const Problem& p) {
    return p.bf16 && p.K == kSlots && p.V >= 64 && p.V % 64 == 0 && p.V <= 4096 && p.N <= 65535 && p.BH <= 65535;
}

gla_status tc_gsa_gate_prep_launch(const Problem& p, const float* la, __nv_bfloat16* w, __nv_bfloat16* Kt,
                                   float* gam, __nv_bfloat16* Kt2, float* gam2, cudaStream_t s) {
    if (p.K != kSlots || p.N > 65535 || p.BH > 65535) return GLA_ERR_UNSUPPORTED;
    GLA_LAUNCH("gsa_gate_prep", k_gsa_gate_prep, dim3(unsigned(p.N), unsigned(p.BH)), kGateThreads, 0, s, la, w, Kt,
               gam, Kt2, gam2, p.L, p.N);
    return GLA_OK;
}

gla_status tc_gsa_slot_read_launch(const Problem& p, const void* x, const void* y, const __nv_bfloat16* M,
                                   const float* la, const float* s_in, __nv_bfloat16* s_b, float* s_f,
                                   __nv_bfloat16* Qt, __nv_bfloat16* P, int mode, cudaStream_t s) {
    if (!tc_gsa_slot_read_supported(p)) return GLA_ERR_UNSUPPORTED;
    CUtensorMap m[4];
    memset(m, 0, sizeof(m));
    const uint64_t L = uint64_t(p.L), D = uint64_t(p.V), BH = uint64_t(p.BH), N = uint64_t(p.N);
    if (!(map3(&m[0], x, D, L, BH) && map3(&m[1], y, D, L, BH) && map3(&m[2], M, D, kSlots, BH * N)))
        return GLA_ERR_CUDA;
    if (mode == 1) {
        const uint64_t dims[3] = {uint64_t(kSlots), L, BH};
        const uint64_t strides[2] = {uint64_t(kSlots) * 4, uint64_t(kSlots) * L * 4};
        const uint32_t box[3] = {32, 128, 1};
        if (!encode_tmap(&m[3], CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, s_in, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
            return GLA_ERR_CUDA;
    } else {
        m[3] = m[0];  // unused: any valid descriptor
    }
    auto fn = mode == 0 ? k_gsa_slot_read<0> : k_gsa_slot_read<1>;
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kSmem)) != cudaSuccess)
        return GLA_ERR_CUDA;
    const dim3 grid(unsigned(p.N), unsigned(p.BH));
    GLA_LAUNCH(mode == 0 ? "gsa_slot_read" : "gsa_slot_read_bwd", fn, grid, kThreadsSR, kSmem, s, m[0], m[1], m[2],
               m[3], la, s_in, s_b, s_f, Qt, P, p.L, p.N, p.V, device_error_word());
    return GLA_OK;
}

}  // namespace gla
