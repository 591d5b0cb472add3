// Row-gated inter-chunk state walk on the 5th-generation tensor cores.
//
// One CTA owns a [K x 64] column tile of the state of one head and walks the
// chunks sequentially ("Gated Linear Attention Transformers with
// Hardware-Efficient Training", atlas.scime.ai summary, "Approach":
// chunkwise algorithm with materialised or non-materialised inter-chunk
// states). Per chunk i:
//   U_i = A1_i^T B1_i                  tcgen05, M = 128 key channels per half,
//                                       N = 64, K = 128 tokens, fp32 in TMEM
//   X  <- diag(gam_i) X + U_i          fp32 master state kept in TMEM
//   Y_i = A2_i X_bf16 + Pm_i B1_i      tcgen05, M = 128 tokens, N = 64
// Operands arrive by TMA (128-byte swizzle) into a ring of 16 KB pieces (the
// value tile, read by both GEMMs of a chunk, has its own double buffer); the
// bf16 copy of X that feeds the output GEMM is written to shared memory by
// the state epilogue. Warp roles: warp 0 issues TMA loads, warp 1 issues the
// MMAs (one thread) and owns the TMEM allocation, warps 2-5 update the state
// (TMEM lanes = key channels), warps 6-9 drain the output accumulator (TMEM
// lanes = tokens) to global memory. Every wait is bounded: a wait that runs
// out records an error in the device error word, every role drains to the
// exit, and TMEM is freed.

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
constexpr int BV = kTcBV;
constexpr uint32_t PIECE = 16384;  // 128 rows x 128 bytes
constexpr int RING = 8;  // short-lived operand pieces (released by the MMA that reads them)
constexpr int kWalkThreads = 320;

struct Bars {
    uint64_t full[RING];
    uint64_t empty[RING];
    uint64_t u_full[2], u_empty[2], o_full[2], o_empty[2];
    uint64_t v_full[2], v_empty[2];  // value tile, double-buffered outside the ring
    uint64_t s_ready[2], s_free[2];  // bf16 state copy, double-buffered: written / read
    uint64_t s_load, drain;
    uint32_t tmem_slot;
    int abort_flag;
};

// Deterministic ring cursor shared (by construction) by producer and MMA
// issuer: both walk the same schedule and therefore see the same slots.
template <int R>
struct Cursor {
    int pos = 0;
    __device__ int take() {
        const int s = pos;
        pos = (pos + 1) % R;
        return s;
    }
    __device__ int take_pair() {  // two adjacent slots (constant LBO)
        if (pos == R - 1) pos = 0;
        if (pos & 1) pos = (pos + 1) % R;
        const int s = pos;
        pos = (pos + 2) % R;
        return s;
    }
};

// Per-mode resources: ring pieces, bf16 state copies in smem, TMEM columns.
template <int NH, int MODE>
struct WalkCfg {
    static constexpr int ring = MODE == kWalkStatesOnly ? 4 : RING;
    static constexpr int s_bufs = MODE == kWalkStatesOnly ? 0 : 2;
    static constexpr uint32_t tmem_cols = MODE == kWalkStatesOnly ? (NH == 1 ? 256u : 512u) : 512u;
    // the states-only walk has no output epilogue (warps 6-9)
    static constexpr int threads = MODE == kWalkStatesOnly ? 192 : kWalkThreads;
    static constexpr int min_blocks = MODE == kWalkStatesOnly ? 2 : 1;
};

struct Sched {
    // Item sequence: U(0), [U(1), O(0)], [U(2), O(1)], ..., O(n-1). Returns
    // the number of items; item e -> (is_output, step).
    int n;
    int mode;
    __device__ int items() const {
        if (mode == kWalkStatesOnly || mode == kWalkOutputOnly) return n;
        return 2 * n;
    }
    __device__ void item(int e, bool& is_out, int& step) const {
        if (mode == kWalkStatesOnly) {
            is_out = false;
            step = e;
            return;
        }
        if (mode == kWalkOutputOnly) {
            is_out = true;
            step = e;
            return;
        }
        if (e == 0) {
            is_out = false;
            step = 0;
        } else if (e == 2 * n - 1) {
            is_out = true;
            step = n - 1;
        } else {
            const int k = (e - 1) / 2;  // pair k: U(k+1), O(k)
            if (((e - 1) & 1) == 0) {
                is_out = false;
                step = k + 1;
            } else {
                is_out = true;
                step = k;
            }
        }
    }
};

template <int NH>
__device__ __forceinline__ uint32_t col_S() { return 0; }
template <int NH>
__device__ __forceinline__ uint32_t col_U(int b, int h) { return uint32_t(NH * BV + b * NH * BV + h * BV); }
template <int NH>
__device__ __forceinline__ uint32_t col_O(int b) { return uint32_t(3 * NH * BV + b * BV); }

template <int NH, bool REVERSE, bool PT, int MODE>
__global__ void __launch_bounds__(WalkCfg<NH, MODE>::threads, WalkCfg<NH, MODE>::min_blocks)
    k_walk(const __grid_constant__ CUtensorMap tmA1, const __grid_constant__ CUtensorMap tmB1,
           const __grid_constant__ CUtensorMap tmA2, const __grid_constant__ CUtensorMap tmP,
           const __grid_constant__ CUtensorMap tmS, const float* __restrict__ gam, const float* __restrict__ init,
           float* __restrict__ fin, float* __restrict__ fin2, __nv_bfloat16* __restrict__ Y,
           __nv_bfloat16* __restrict__ states, int64_t L, int64_t N, int64_t V, int64_t K, int64_t BH, WalkSegs sg,
           int* err) {
    constexpr int KC = NH * 128;  // key channels owned by this CTA
    using Cfg = WalkCfg<NH, MODE>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* ring = base;
    uint8_t* vbuf = base + Cfg::ring * PIECE;  // 2 x PIECE
    uint8_t* sS = vbuf + 2 * PIECE;             // s_bufs x [KC x 64] bf16 copies of the state
    Bars& bar = *reinterpret_cast<Bars*>(sS + Cfg::s_bufs * KC * 128);
    volatile int* abort_flag = &bar.abort_flag;

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    // blockIdx.z = head + BH * (segment - sg.first); a segment is sg.len consecutive walk steps
    const int64_t bh = blockIdx.z % BH;
    const int seg = sg.first + int(blockIdx.z / BH);
    const int s0 = seg * sg.len;
    const int v0 = blockIdx.x * BV;
    const int nsteps = MODE == kWalkOutputOnly ? 1 : (int(N) - s0 < sg.len ? int(N) - s0 : sg.len);
    const int first_chunk = MODE == kWalkOutputOnly ? int(blockIdx.y) : 0;
    // states-only walks may split the key channels over blockIdx.y
    const int kbase = MODE == kWalkStatesOnly ? int(blockIdx.y) * KC : 0;
    auto chunk_of = [&](int step) -> int {
        if (MODE == kWalkOutputOnly) return first_chunk;
        return REVERSE ? int(N) - 1 - (s0 + step) : s0 + step;
    };
    const float* init_s = seg == 0 ? init : (sg.init_seg ? sg.init_seg + seg * sg.stride : nullptr);

    if (threadIdx.x == 0) {
        for (int s = 0; s < Cfg::ring; ++s) {
            mbar_init(&bar.full[s], 1);
            mbar_init(&bar.empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bar.u_full[b], 1);
            mbar_init(&bar.u_empty[b], 128);
            mbar_init(&bar.o_full[b], 1);
            mbar_init(&bar.o_empty[b], 128);
            mbar_init(&bar.v_full[b], 1);
            mbar_init(&bar.v_empty[b], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bar.s_ready[b], 128);
            mbar_init(&bar.s_free[b], 1);
        }
        mbar_init(&bar.s_load, 1);
        mbar_init(&bar.drain, 1);
        bar.abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(&bar.tmem_slot, Cfg::tmem_cols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bar.tmem_slot;
    // programmatic dependent launch: the prologue above overlapped the previous kernel's tail;
    // nothing below touches global memory before that kernel has completed
    if (threadIdx.x == 0) {  // tensor maps are kernel parameters: fetch them while the previous kernel drains
        tma_prefetch(&tmA1);
        tma_prefetch(&tmB1);
        tma_prefetch(&tmA2);
        tma_prefetch(&tmP);
    }
    pdl_launch_dependents();
    pdl_wait();
    const Sched sched{nsteps, MODE};

    if (warp == 0) {
        // ------------------------------------------------------ TMA producer
        if (lane == 0) {
            Cursor<Cfg::ring> cur;
            uint32_t par = 0;            // parity of the next use, one bit per slot
            uint32_t pending = 0;        // slots with a load whose completion nobody waited for yet
            uint32_t pending_par = 0;
            auto load = [&](int slot, const CUtensorMap* m, int x, int y, int z) -> bool {
                const uint32_t ph = (par >> slot) & 1u;
                if (!mbar_wait(&bar.empty[slot], ph ^ 1u, err, abort_flag)) return false;
                mbar_arrive_expect_tx(&bar.full[slot], PIECE);
                tma_load_3d(ring + slot * PIECE, m, x, y, z, &bar.full[slot]);
                pending |= 1u << slot;
                pending_par = (pending_par & ~(1u << slot)) | (ph << slot);
                par ^= 1u << slot;
                return true;
            };
            // value tile of `step` -> vbuf[step % 2] (its previous user released it)
            uint32_t vpend = 0;
            auto load_v = [&](int step, int row0) -> bool {
                const int vb = step & 1;
                const uint32_t ph = uint32_t((step >> 1) & 1);
                if (!mbar_wait(&bar.v_empty[vb], ph ^ 1u, err, abort_flag)) return false;
                mbar_arrive_expect_tx(&bar.v_full[vb], PIECE);
                tma_load_3d(vbuf + vb * PIECE, &tmB1, v0, row0, int(bh), &bar.v_full[vb]);
                vpend = (vpend & ~(3u << (2 * vb))) | ((1u | (ph << 1)) << (2 * vb));
                return true;
            };
            if (MODE == kWalkOutputOnly) {
                const int i = first_chunk;
                mbar_arrive_expect_tx(&bar.s_load, KC * 128);
                tma_load_3d(sS, &tmS, v0, 0, int(bh * N + i), &bar.s_load);
            }
            bool ok = true;
            for (int e = 0; e < sched.items() && ok; ++e) {
                bool is_out;
                int step;
                sched.item(e, is_out, step);
                const int i = chunk_of(step);
                const int row0 = i * C;
                if (!is_out) {
                    for (int h = 0; h < NH && ok; ++h) {
                        const int s = cur.take_pair();
                        ok = load(s, &tmA1, kbase + 128 * h, row0, int(bh)) &&
                             load(s + 1, &tmA1, kbase + 128 * h + 64, row0, int(bh));
                    }
                    if (ok) ok = load_v(step, row0);
                } else {
                    if (MODE == kWalkOutputOnly) ok = load_v(step, row0);
                    for (int pc = 0; pc < 2 * NH && ok; ++pc) ok = load(cur.take(), &tmA2, 64 * pc, row0, int(bh));
                    if (ok) {
                        const int s = cur.take_pair();
                        ok = load(s, &tmP, 0, 0, int(bh * N + i)) && load(s + 1, &tmP, 64, 0, int(bh * N + i));
                    }
                }
            }
            // on abort, wait (bounded) for loads still in flight before the block exits
            if (!ok) {
                for (int s = 0; s < Cfg::ring; ++s)
                    if ((pending >> s) & 1u) mbar_wait(&bar.full[s], (pending_par >> s) & 1u, nullptr, abort_flag);
                for (int vb = 0; vb < 2; ++vb)
                    if ((vpend >> (2 * vb)) & 1u)
                        mbar_wait(&bar.v_full[vb], (vpend >> (2 * vb + 1)) & 1u, nullptr, abort_flag);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idU = idesc_bf16_f32(128, BV, true, true);
            const uint32_t idQS = idesc_bf16_f32(128, BV, false, true);
            const uint32_t idPV = idesc_bf16_f32(128, BV, PT, true);
            Cursor<Cfg::ring> cur;
            uint32_t par = 0;
            bool ok = true;
            auto wait_full = [&](int slot) -> bool {
                const uint32_t ph = (par >> slot) & 1u;
                par ^= 1u << slot;
                return mbar_wait(&bar.full[slot], ph, err, abort_flag);
            };
            if (MODE == kWalkOutputOnly) ok = mbar_wait(&bar.s_load, 0, err, abort_flag);
            for (int e = 0; e < sched.items() && ok; ++e) {
                bool is_out;
                int step;
                sched.item(e, is_out, step);
                const int b = step & 1;
                const uint32_t use_par = uint32_t((step >> 1) & 1);
                if (!is_out) {
                    int sa[NH];
                    for (int h = 0; h < NH; ++h) sa[h] = cur.take_pair();
                    ok = mbar_wait(&bar.u_empty[b], use_par ^ 1u, err, abort_flag);
                    for (int h = 0; h < NH && ok; ++h) ok = wait_full(sa[h]) && wait_full(sa[h] + 1);
                    if (ok) ok = mbar_wait(&bar.v_full[b], use_par, err, abort_flag);
                    if (!ok) break;
                    tc_fence_after();
                    for (int h = 0; h < NH; ++h) {
                        const uint32_t a0 = smem_u32(ring + sa[h] * PIECE);
                        const uint32_t b0 = smem_u32(vbuf + b * PIECE);
#pragma unroll
                        for (int kk = 0; kk < C / 16; ++kk)
                            mma_bf16(tmem + col_U<NH>(b, h), sdesc_sw128(a0 + kk * 2048, PIECE, 1024),
                                     sdesc_sw128(b0 + kk * 2048, 16, 1024), idU, kk > 0 ? 1u : 0u);
                    }
                    mma_commit(&bar.u_full[b]);
                    for (int h = 0; h < NH; ++h) {
                        mma_commit(&bar.empty[sa[h]]);
                        mma_commit(&bar.empty[sa[h] + 1]);
                    }
                    if (MODE == kWalkStatesOnly) mma_commit(&bar.v_empty[b]);
                } else {
                    int sq[2 * NH];
                    for (int pc = 0; pc < 2 * NH; ++pc) sq[pc] = cur.take();
                    const int sp = cur.take_pair();
                    if (MODE == kWalkFused) ok = mbar_wait(&bar.s_ready[b], use_par, err, abort_flag);
                    if (ok) ok = mbar_wait(&bar.o_empty[b], use_par ^ 1u, err, abort_flag);
                    if (ok && MODE == kWalkOutputOnly) ok = mbar_wait(&bar.v_full[b], use_par, err, abort_flag);
                    for (int pc = 0; pc < 2 * NH && ok; ++pc) ok = wait_full(sq[pc]);
                    if (ok) ok = wait_full(sp) && wait_full(sp + 1);
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t dO_ = tmem + col_O<NH>(b);
                    const uint32_t s0 = smem_u32(sS + b * KC * 128);
#pragma unroll
                    for (int kk = 0; kk < KC / 16; ++kk)
                        mma_bf16(dO_, sdesc_sw128(smem_u32(ring + sq[kk / 4] * PIECE) + (kk % 4) * 32, 16, 1024),
                                 sdesc_sw128(s0 + kk * 2048, 16, 1024), idQS, kk > 0 ? 1u : 0u);
                    const uint32_t p0 = smem_u32(ring + sp * PIECE);
                    const uint32_t vb = smem_u32(vbuf + b * PIECE);
#pragma unroll
                    for (int kk = 0; kk < C / 16; ++kk) {
                        const uint64_t ad = PT ? sdesc_sw128(p0 + kk * 2048, PIECE, 1024)
                                               : sdesc_sw128(p0 + (kk / 4) * PIECE + (kk % 4) * 32, 16, 1024);
                        mma_bf16(dO_, ad, sdesc_sw128(vb + kk * 2048, 16, 1024), idPV, 1u);
                    }
                    mma_commit(&bar.o_full[b]);
                    if (MODE == kWalkFused) mma_commit(&bar.s_free[b]);
                    for (int pc = 0; pc < 2 * NH; ++pc) mma_commit(&bar.empty[sq[pc]]);
                    mma_commit(&bar.empty[sp]);
                    mma_commit(&bar.empty[sp + 1]);
                    mma_commit(&bar.v_empty[b]);
                }
            }
            // wait for every MMA issued so far before the block can free TMEM
            mma_commit(&bar.drain);
            mbar_wait(&bar.drain, 0, nullptr, abort_flag, 4000000000LL);
        }
    } else if (warp < 6) {
        // ------------------------------------------------------ state epilogue
        if (MODE != kWalkOutputOnly) {
            const int q = warp & 3;
            const int cq = kbase + 32 * q + lane;  // key channel (global index) in this CTA's first half
            const uint32_t lane_off = uint32_t(32 * q) << 16;
            // X0 = init tile (or zero) -> TMEM master and the bf16 copy in smem
            for (int h = 0; h < NH; ++h) {
                const int c = 128 * h + cq;
                for (int c16 = 0; c16 < BV / 16; ++c16) {
                    float x[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        x[e] = init_s ? init_s[(bh * K + c) * V + v0 + c16 * 16 + e] : 0.f;
                    tmem_st16(tmem + lane_off + col_S<NH>() + uint32_t(h * BV + c16 * 16), x);
                    if (MODE == kWalkFused) {  // only the fused walk keeps a bf16 copy in smem
                        uint8_t* row = sS + (c - kbase) * 128;
#pragma unroll
                        for (int half = 0; half < 2; ++half) {
                            const int chunk = c16 * 2 + half;
                            uint4 w;
                            w.x = pack_bf16x2(x[half * 8 + 0], x[half * 8 + 1]);
                            w.y = pack_bf16x2(x[half * 8 + 2], x[half * 8 + 3]);
                            w.z = pack_bf16x2(x[half * 8 + 4], x[half * 8 + 5]);
                            w.w = pack_bf16x2(x[half * 8 + 6], x[half * 8 + 7]);
                            *reinterpret_cast<uint4*>(row + ((chunk ^ ((c - kbase) & 7)) * 16)) = w;
                        }
                    }
                    if (MODE == kWalkStatesOnly || states) {
                        __nv_bfloat16* dst = states + ((bh * N + chunk_of(0)) * K + c) * V + v0 + c16 * 16;
                        uint4 w0, w1;
                        w0.x = pack_bf16x2(x[0], x[1]);
                        w0.y = pack_bf16x2(x[2], x[3]);
                        w0.z = pack_bf16x2(x[4], x[5]);
                        w0.w = pack_bf16x2(x[6], x[7]);
                        w1.x = pack_bf16x2(x[8], x[9]);
                        w1.y = pack_bf16x2(x[10], x[11]);
                        w1.z = pack_bf16x2(x[12], x[13]);
                        w1.w = pack_bf16x2(x[14], x[15]);
                        reinterpret_cast<uint4*>(dst)[0] = w0;
                        reinterpret_cast<uint4*>(dst)[1] = w1;
                    }
                }
            }
            tmem_wait_st();
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&bar.s_ready[0]);
            float g_next[NH];
            for (int h = 0; h < NH; ++h) g_next[h] = gam[(bh * N + chunk_of(0)) * K + 128 * h + cq];
            for (int step = 0; step < nsteps; ++step) {
                const int b = step & 1;
                const uint32_t use_par = uint32_t((step >> 1) & 1);
                float g[NH];
                for (int h = 0; h < NH; ++h) g[h] = g_next[h];
                if (step + 1 < nsteps)
                    for (int h = 0; h < NH; ++h) g_next[h] = gam[(bh * N + chunk_of(step + 1)) * K + 128 * h + cq];
                if (!mbar_wait(&bar.u_full[b], use_par, err, abort_flag)) break;
                tc_fence_after();
                // X <- diag(g) X + U in TMEM, 32 columns per batch; keep the new
                // state packed to bf16 in registers for the smem / global copy
                uint32_t pk[NH][BV / 2];
#pragma unroll
                for (int h = 0; h < NH; ++h) {
#pragma unroll
                    for (int c32 = 0; c32 < BV / 32; ++c32) {
                        float u[32], x[32];
                        const uint32_t cu = col_U<NH>(b, h) + uint32_t(c32 * 32);
                        const uint32_t cs = col_S<NH>() + uint32_t(h * BV + c32 * 32);
                        tmem_ld16(tmem + lane_off + cu, u);
                        tmem_ld16(tmem + lane_off + cu + 16, u + 16);
                        tmem_ld16(tmem + lane_off + cs, x);
                        tmem_ld16(tmem + lane_off + cs + 16, x + 16);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e) x[e] = fmaf(g[h], x[e], u[e]);
                        tmem_st16(tmem + lane_off + cs, x);
                        tmem_st16(tmem + lane_off + cs + 16, x + 16);
#pragma unroll
                        for (int e = 0; e < 16; ++e) pk[h][c32 * 16 + e] = pack_bf16x2(x[2 * e], x[2 * e + 1]);
                    }
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(&bar.u_empty[b]);
                if (step + 1 == nsteps) break;  // the final state is written below
                if (MODE == kWalkFused) {
                    // S_[i+1] -> bf16 copy in buffer (step+1)&1, last read by the output GEMM of step-1
                    const int nb = (step + 1) & 1;
                    if (step >= 1 &&
                        !mbar_wait(&bar.s_free[nb], uint32_t(((step - 1) >> 1) & 1), err, abort_flag))
                        break;
#pragma unroll
                    for (int h = 0; h < NH; ++h) {
                        const int c = 128 * h + cq;
                        uint8_t* row = sS + nb * KC * 128 + (c - kbase) * 128;
#pragma unroll
                        for (int ch = 0; ch < 8; ++ch)
                            *reinterpret_cast<uint4*>(row + ((ch ^ ((c - kbase) & 7)) * 16)) =
                                make_uint4(pk[h][4 * ch], pk[h][4 * ch + 1], pk[h][4 * ch + 2], pk[h][4 * ch + 3]);
                    }
                    fence_proxy_async_smem();
                    mbar_arrive(&bar.s_ready[nb]);
                }
                if (MODE == kWalkStatesOnly || states) {
#pragma unroll
                    for (int h = 0; h < NH; ++h) {
                        const int c = 128 * h + cq;
                        uint4* dst = reinterpret_cast<uint4*>(states + ((bh * N + chunk_of(step + 1)) * K + c) * V + v0);
#pragma unroll
                        for (int ch = 0; ch < 8; ++ch)
                            dst[ch] = make_uint4(pk[h][4 * ch], pk[h][4 * ch + 1], pk[h][4 * ch + 2], pk[h][4 * ch + 3]);
                    }
                }
            }
            if ((fin || fin2) && !*abort_flag) {
                for (int h = 0; h < NH; ++h) {
                    const int c = 128 * h + cq;
                    for (int c16 = 0; c16 < BV / 16; ++c16) {
                        float x[16];
                        tmem_ld16(tmem + lane_off + col_S<NH>() + uint32_t(h * BV + c16 * 16), x);
                        tmem_wait_ld();
                        for (int w = 0; w < 2; ++w) {
                            float* f = w ? fin2 : fin;
                            if (!f) continue;
                            float4* dst = reinterpret_cast<float4*>(f + (bh * K + c) * V + v0 + c16 * 16);
#pragma unroll
                            for (int e = 0; e < 4; ++e)
                                dst[e] = make_float4(x[4 * e], x[4 * e + 1], x[4 * e + 2], x[4 * e + 3]);
                        }
                    }
                }
            }
        }
    } else {
        // ------------------------------------------------------ output epilogue
        if (MODE != kWalkStatesOnly) {
            const int q = warp & 3;
            const int r = 32 * q + lane;  // token row within the chunk
            const uint32_t lane_off = uint32_t(32 * q) << 16;
            for (int step = 0; step < nsteps; ++step) {
                const int b = step & 1;
                const uint32_t use_par = uint32_t((step >> 1) & 1);
                if (!mbar_wait(&bar.o_full[b], use_par, err, abort_flag)) break;
                tc_fence_after();
                const int64_t t = int64_t(chunk_of(step)) * C + r;
                float y[BV];
#pragma unroll
                for (int c16 = 0; c16 < BV / 16; ++c16)
                    tmem_ld16(tmem + lane_off + col_O<NH>(b) + uint32_t(c16 * 16), y + 16 * c16);
                tmem_wait_ld();
                if (t < L) {
                    uint4* dst = reinterpret_cast<uint4*>(Y + (bh * L + t) * V + v0);
#pragma unroll
                    for (int ch = 0; ch < BV / 8; ++ch)
                        dst[ch] = make_uint4(pack_bf16x2(y[8 * ch], y[8 * ch + 1]), pack_bf16x2(y[8 * ch + 2], y[8 * ch + 3]),
                                             pack_bf16x2(y[8 * ch + 4], y[8 * ch + 5]),
                                             pack_bf16x2(y[8 * ch + 6], y[8 * ch + 7]));
                }
                tc_fence_before();
                mbar_arrive(&bar.o_empty[b]);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, Cfg::tmem_cols);
    }
}

bool map3(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t outer, uint32_t box_rows) {
    const uint64_t dims[3] = {inner, rows, outer};
    const uint64_t strides[2] = {inner * 2, inner * rows * 2};
    const uint32_t box[3] = {64, box_rows, 1};
    return encode_tmap(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

template <int NH, bool REVERSE, bool PT, int MODE>
gla_status launch_walk(const Problem& p, const WalkArgs& a, const CUtensorMap* maps, cudaStream_t s,
                       const char* name) {
    constexpr int KC = NH * 128;
    using Cfg = WalkCfg<NH, MODE>;
    auto fn = k_walk<NH, REVERSE, PT, MODE>;
    const size_t smem = 1024 + size_t(Cfg::ring + 2) * PIECE + size_t(Cfg::s_bufs) * KC * 128 + sizeof(Bars);
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) != cudaSuccess)
        return GLA_ERR_CUDA;
    const unsigned gy = MODE == kWalkOutputOnly ? unsigned(p.N)
                        : MODE == kWalkStatesOnly ? unsigned(p.K / KC) : 1u;
    const bool split = MODE == kWalkFused && a.seg_count > 1;
    const WalkSegs sg = split ? WalkSegs{0, a.seg_len, 1, a.seg_stride, a.seg_init} : WalkSegs{0, int(p.N), 1, 0, nullptr};
    const dim3 grid(unsigned(p.V / BV), gy, unsigned(p.BH * (split ? a.seg_count : 1)));
    // a split walk leaves the final state to the segment scan
    GLA_LAUNCH_PDL(name, fn, grid, Cfg::threads, smem, s, maps[0], maps[1], maps[2], maps[3], maps[4], a.gam, a.init,
                   split ? nullptr : a.fin, split ? nullptr : a.fin2, a.Y, a.states, p.L, p.N, p.V, p.K, p.BH, sg,
                   device_error_word());
    return GLA_OK;
}

}  // namespace



gla_status tc_walk_launch(const Problem& p, const WalkArgs& a, cudaStream_t s, const char* name) {
    CUtensorMap maps[5];
    memset(maps, 0, sizeof(maps));
    const uint64_t L = uint64_t(p.L), K = uint64_t(p.K), V = uint64_t(p.V), BH = uint64_t(p.BH), N = uint64_t(p.N);
    bool ok = true;
    if (a.mode != kWalkOutputOnly) ok = ok && map3(&maps[0], a.A1, K, L, BH, 128);
    ok = ok && map3(&maps[1], a.B1, V, L, BH, 128);
    if (a.mode != kWalkStatesOnly) {
        ok = ok && map3(&maps[2], a.A2, K, L, BH, 128);
        ok = ok && map3(&maps[3], a.Pm, 128, 128, BH * N, 128);
    }
    if (a.mode == kWalkOutputOnly) ok = ok && map3(&maps[4], a.states, V, K, BH * N, uint32_t(K));
    // unused maps must still be valid descriptors: reuse the value map
    for (int m = 0; m < 5; ++m)
        if (!ok) break;
        else if (maps[m].opaque[0] == 0 && maps[m].opaque[1] == 0) maps[m] = maps[1];
    if (!ok) return GLA_ERR_CUDA;
    const int NH = a.mode == kWalkStatesOnly ? 1 : int(p.K / 128);  // states-only: one half per CTA
#define GLA_WALK_CASE(nh_, rev_, pt_, mode_)                                                   \
    if (NH == nh_ && a.reverse == rev_ && a.p_transposed == pt_ && a.mode == mode_)            \
        return launch_walk<nh_, rev_, pt_, mode_>(p, a, maps, s, name);
    GLA_WALK_CASE(1, false, false, kWalkFused)
    GLA_WALK_CASE(2, false, false, kWalkFused)
    GLA_WALK_CASE(1, true, true, kWalkFused)
    GLA_WALK_CASE(2, true, true, kWalkFused)
    GLA_WALK_CASE(1, false, false, kWalkStatesOnly)
    GLA_WALK_CASE(1, true, false, kWalkStatesOnly)
    GLA_WALK_CASE(1, false, false, kWalkOutputOnly)
    GLA_WALK_CASE(2, false, false, kWalkOutputOnly)
    GLA_WALK_CASE(1, false, true, kWalkOutputOnly)
    GLA_WALK_CASE(2, false, true, kWalkOutputOnly)
#undef GLA_WALK_CASE
    return GLA_ERR_UNSUPPORTED;
}

}  // namespace gla
