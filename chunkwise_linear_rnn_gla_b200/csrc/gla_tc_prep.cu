// Chunk-parallel preparation for the tensor-core path (bf16 inputs, C = 128).
//
// For every chunk i of every head this kernel computes, once:
//   B_j   = sum_{r<=j} log a_r          per-chunk inclusive gate cumsum (fp32)
//   Q~_j  = q_j * e^{B_j}               (bf16, operand of the inter-chunk output GEMM)
//   K~_j  = k_j * e^{Gamma - B_j}       (bf16, operand of the state-update GEMM)
//   e^Gamma                             (fp32 per key channel, Gamma = B at the chunk's last row)
//   P_js  = sum_c q_jc k_sc e^{B_jc - B_sc} for s <= j, 0 above (bf16 [128 x 128])
//
// The intra-chunk scores follow the chunk form of the gated recurrence
// ("Gated Linear Attention Transformers with Hardware-Efficient Training",
// atlas.scime.ai summary, "Approach"): P = (q * e^B)(k * e^{-B})^T, masked.
// The pages split this into 16-row secondary chunks so that the factors never
// leave the half-precision range. Here the range is bounded per key channel
// instead: when Gamma_c >= -64, every e^{+-B_jc} lies in [e^-64, e^64], so the
// whole 128 x 128 block is ONE tcgen05 GEMM over the key channels,
//     P = Q~ K^0^T,   K^0_s = k_s * e^{-B_s} = K~_s * e^{-Gamma},
// with bf16 operands (the same relative rounding as the secondary-chunk
// products: each term of the sum is q k e^{B_j - B_s} up to two bf16
// roundings). A channel whose chunk decay exceeds the bound (Gamma_c < -64,
// e.g. a gate of exactly 0) gets a zero K^0 column, and its terms are added on
// the CUDA cores one by one as q_jc k_sc exp(B_jc - B_sc) (log space).
//
// Gate kinds (gla_gate.cuh): the per-channel kinds (channel, preact) take the
// form above. The scalar kinds (scalar, head) share one decay b_t across the
// key channels, so the intra block is ONE masked, decay-weighted GEMM of the raw
// bf16 q and k, P_js = (q_j . k_s) e^{b_j - b_s}, the decay applied per element
// in fp32 after the MMA (every factor <= 1, no range bound, no exact path).
//
// Roles (one CTA per chunk, 288 threads, two CTAs per SM). Warp 8 is the
// producer and MMA issuer: per 64-channel piece it loads the q and k tiles by
// TMA straight into the swizzled operand buffers (double-buffered), and the
// fp32 gate tile into a staging buffer one piece ahead, then issues the four
// MMAs of the piece once it is complete. Warps 0-7 are the element warps, warp
// I covering rows 16I .. 16I+15; lane l holds 8 adjacent channels (8 (l % 8) ..)
// of 4 rows (16I + 4 (l / 8) ..), i.e. one 16-byte chunk of each operand row.
// The per-chunk cumsum runs along a lane's 4 rows, across the warp's 4 row
// groups by shuffles and across the 8 warps through shared memory; the gate
// tile is then released for the next piece's load, and each operand chunk is
// rescaled in place (Q~ and K^0; the scalar kinds keep the raw q and k) while
// Q~ and K~ go to global memory. At the end the eight warps read P back from
// TMEM (warp w: lanes 32(w%4).., columns 64(w/4) ..) and store it.

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstring>

#include "gla_common.cuh"
#include "gla_gate.cuh"
#include "gla_internal.h"
#include "gla_tc.h"
#include "tc_host.h"

namespace gla {
namespace {

using namespace tc;

constexpr int C = kTcChunk;
constexpr int KP = 64;                      // key channels per piece
constexpr uint32_t PIECE = 16384;           // one [128 x 64] bf16 operand piece
constexpr uint32_t LA_BYTES = C * KP * 4;   // one [128 x 64] fp32 gate tile
constexpr uint32_t LA_OFF = 4 * PIECE;      // gate tile staging (also the exact-path tables at the end)
constexpr uint32_t BAR_OFF = LA_OFF + LA_BYTES;
constexpr int kThreads = 288;
constexpr float kSafeDecay = 64.f;          // |B| bound for the tensor-core form

struct PrepBars {
    float tot[2][8][KP];  // per-piece, per 16-row warp block gate sums
    float btab[C];        // scalar kinds: the per-token cumsum b_t
    uint64_t qk_full[2], ops_ready[2], mma_done[2], la_full, la_free, p_done, drain;
    uint32_t tmem_slot;
    int abort_flag;
    int nuns;
    unsigned short uns[256];  // key channels that take the exact path
};

constexpr bool scalar_kind(int GK) { return GK == kGateScalar || GK == kGateHead; }

// log alpha from the staged value (preact: logsigmoid(z) / tau), floored for the cumsum
template <int GK>
__device__ __forceinline__ float log_alpha_of(float x, float inv_tau) {
    return la_floor(GK == kGatePreact ? logsigmoid_f(x) * inv_tau : x);
}

// log alpha of one (row, channel) for the exact path
template <int K, int GK>
__device__ __forceinline__ float gate_at(const GateArgs& ga, int64_t bh, int64_t t, int64_t c, int64_t L) {
    return la_floor(gate_log_alpha(ga, bh, t, c, L, K));
}

__device__ __forceinline__ void unpack8(const uint4& u, float* f) {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const float2 v = __bfloat1622float2(h[e]);
        f[2 * e] = v.x;
        f[2 * e + 1] = v.y;
    }
}

__device__ __forceinline__ uint4 pack8(const float* f) {
    return make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                      pack_bf16x2(f[6], f[7]));
}

template <int K, int GK>
__global__ void __launch_bounds__(kThreads, 2)
    k_tc_prep(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
              const __grid_constant__ CUtensorMap tmG, const __nv_bfloat16* __restrict__ q,
              const __nv_bfloat16* __restrict__ k, GateArgs ga, __nv_bfloat16* __restrict__ Qt,
              __nv_bfloat16* __restrict__ Kt, __nv_bfloat16* __restrict__ P, float* __restrict__ gam, int64_t L,
              int64_t N, int* err) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    // [0, 4 PIECE): operand buffers [b][Q piece, K piece], b = piece parity
    PrepBars& bar = *reinterpret_cast<PrepBars*>(base + BAR_OFF);
    const float* sG = reinterpret_cast<const float*>(base + LA_OFF);
    volatile int* abort_flag = &bar.abort_flag;
    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    const int i = blockIdx.x;
    const int64_t bh = blockIdx.y;
    const int64_t t0 = int64_t(i) * C;
    const int nvalid = int(L - t0 < C ? L - t0 : C);
    constexpr int npiece = K / KP;
    constexpr bool SK = scalar_kind(GK);

    if (tid == 0) {
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bar.qk_full[b], 1);
            mbar_init(&bar.ops_ready[b], 256);
            mbar_init(&bar.mma_done[b], 1);
        }
        mbar_init(&bar.la_full, 1);
        mbar_init(&bar.la_free, 256);
        mbar_init(&bar.p_done, 1);
        mbar_init(&bar.drain, 1);
        bar.abort_flag = 0;
        bar.nuns = 0;
        fence_barrier_init();
    }
    if (warp == 8) {
        tmem_alloc(&bar.tmem_slot, 128);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bar.tmem_slot;
    if (tid == 256) {  // tensor maps are kernel parameters: fetch them while the previous kernel drains
        tma_prefetch(&tmQ);
        tma_prefetch(&tmK);
        if (!SK) tma_prefetch(&tmG);
    }
    // programmatic dependent launch: the prologue above overlapped the previous kernel's tail;
    // nothing below touches global memory before that kernel has completed
    pdl_launch_dependents();
    pdl_wait();

    if (warp == 8) {
        if (lane == 0) {
            const uint32_t id = idesc_bf16_f32(128, 128, false, false);
            bool ok = true;
            int n_qk = 0, n_la = 0;  // loads issued
            auto mma = [&](int t) {  // the four MMAs of piece t, once its operands are rescaled
                const int b = t & 1;
                ok = ok && mbar_wait(&bar.ops_ready[b], uint32_t((t >> 1) & 1), err, abort_flag);
                if (!ok) return;
                tc_fence_after();
                const uint32_t a0 = smem_u32(base + b * 2 * PIECE), b0 = a0 + PIECE;
#pragma unroll
                for (int kk = 0; kk < KP / 16; ++kk)
                    mma_bf16(tmem, sdesc_sw128(a0 + kk * 32, 16, 1024), sdesc_sw128(b0 + kk * 32, 16, 1024), id,
                             (t > 0 || kk > 0) ? 1u : 0u);
                mma_commit(&bar.mma_done[b]);
                if (t == npiece - 1) mma_commit(&bar.p_done);
            };
            for (int t = 0; t < npiece && ok; ++t) {
                const int b = t & 1;
                // q and k of piece t into operand buffer b, free once the MMAs of piece t-2 are done
                if (t >= 2) ok = mbar_wait(&bar.mma_done[b], uint32_t(((t >> 1) - 1) & 1), err, abort_flag);
                if (!ok) break;
                mbar_arrive_expect_tx(&bar.qk_full[b], 2 * PIECE);
                tma_load_3d(base + b * 2 * PIECE, &tmQ, KP * t, int(t0), int(bh), &bar.qk_full[b]);
                tma_load_3d(base + b * 2 * PIECE + PIECE, &tmK, KP * t, int(t0), int(bh), &bar.qk_full[b]);
                ++n_qk;
                if (!SK) {  // the gate tile of piece t, once every element thread has read piece t-1's
                    if (t >= 1) ok = mbar_wait(&bar.la_free, uint32_t((t - 1) & 1), err, abort_flag);
                    if (!ok) break;
                    mbar_arrive_expect_tx(&bar.la_full, LA_BYTES);
                    tma_load_3d(base + LA_OFF, &tmG, KP * t, int(t0), int(bh), &bar.la_full);
                    ++n_la;
                }
                if (t >= 1) mma(t - 1);
            }
            if (ok) mma(npiece - 1);
            if (!ok) {  // let the copies already issued land before the block exits
                for (int t = n_qk - 2; t < n_qk; ++t)
                    if (t >= 0) mbar_drain(&bar.qk_full[t & 1], uint32_t((t >> 1) & 1));
                if (n_la > 0) mbar_drain(&bar.la_full, uint32_t((n_la - 1) & 1));
            }
            mma_commit(&bar.drain);
            mbar_drain(&bar.drain, 0);
        }
    } else {
        const int I = warp;
        const int cg = lane & 7;   // channels 8 cg .. 8 cg + 7 of the piece
        const int rs = lane >> 3;  // rows 16 I + 4 rs .. + 3
        const int row0 = 16 * I + 4 * rs;
        // Every element thread passes every named barrier, also after a wait gave up (bar.sync has
        // no time limit); a failed wait only skips the work.
        bool ok = true;
        for (int t = 0; t < npiece; ++t) {
            const int b = t & 1;
            const int64_t ch0 = int64_t(KP) * t + 8 * cg;
            // ---- per-chunk cumsum: along the lane's 4 rows, across the warp's 4 row groups, across the
            // warps; B[r][e] becomes the inclusive cumsum at row row0 + r (zero gates past the end of the
            // sequence)
            float Bv[4][8], tot[8];
            if (SK) {
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    const float x = row0 + r < nvalid ? la_floor(GK == kGateScalar ? ga.g[bh * L + t0 + row0 + r]
                                                                                     : ga.g[bh % ga.H])
                                                      : 0.f;
#pragma unroll
                    for (int e = 0; e < 8; ++e) Bv[r][e] = x;
                }
            } else {
                ok = ok && mbar_wait(&bar.la_full, uint32_t(t & 1), err, abort_flag);
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    const float4 a = *reinterpret_cast<const float4*>(sG + (row0 + r) * KP + 8 * cg);
                    const float4 c4 = *reinterpret_cast<const float4*>(sG + (row0 + r) * KP + 8 * cg + 4);
                    const float x[8] = {a.x, a.y, a.z, a.w, c4.x, c4.y, c4.z, c4.w};
                    const bool v = row0 + r < nvalid;
#pragma unroll
                    for (int e = 0; e < 8; ++e) Bv[r][e] = v ? log_alpha_of<GK>(x[e], ga.inv_tau) : 0.f;
                }
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
                if (rs == 3) bar.tot[b][I][8 * cg + e] = incl;  // the warp's 16-row total
            }
            if (!SK) mbar_arrive(&bar.la_free);  // this thread's reads of the gate tile are done
            named_sync(1, 256);
            float pre[8], gamma[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) pre[e] = gamma[e] = 0.f;
#pragma unroll
            for (int J = 0; J < 8; ++J) {
                const float4 a = *reinterpret_cast<const float4*>(&bar.tot[b][J][8 * cg]);
                const float4 c4 = *reinterpret_cast<const float4*>(&bar.tot[b][J][8 * cg + 4]);
                const float v[8] = {a.x, a.y, a.z, a.w, c4.x, c4.y, c4.z, c4.w};
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    if (J < I) pre[e] += v[e];
                    gamma[e] += v[e];
                }
            }
            float eNG[8];
            bool any_unsafe = false;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
#pragma unroll
                for (int r = 0; r < 4; ++r) Bv[r][e] += pre[e] + excl[e];
                const bool unsafe = !SK && gamma[e] < -kSafeDecay;
                any_unsafe |= unsafe;
                eNG[e] = unsafe ? 0.f : __expf(fmaxf(-gamma[e], 0.f));  // e^{-Gamma} <= e^64
            }
            if (I == 0 && rs == 0) {
                float eg[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) eg[e] = __expf(fminf(gamma[e], 0.f));
                float4* gp = reinterpret_cast<float4*>(gam + (bh * N + i) * K + ch0);
                gp[0] = make_float4(eg[0], eg[1], eg[2], eg[3]);
                gp[1] = make_float4(eg[4], eg[5], eg[6], eg[7]);
                if (any_unsafe)
                    for (int e = 0; e < 8; ++e)
                        if (gamma[e] < -kSafeDecay) bar.uns[atomicAdd(&bar.nuns, 1)] = (unsigned short)(ch0 + e);
            }
            if (SK && t == 0 && cg == 0) {
#pragma unroll
                for (int r = 0; r < 4; ++r) bar.btab[row0 + r] = Bv[r][0];
            }
            // ---- the q and k rows of the piece (TMA, zero past the end of the sequence): Q~ and K~ to
            // global memory; the operand rows rescaled in place into Q~ and K^0 (scalar kinds: raw q, k)
            ok = ok && mbar_wait(&bar.qk_full[b], uint32_t((t >> 1) & 1), err, abort_flag);
            uint8_t* opQ = base + b * 2 * PIECE;
            uint8_t* opK = opQ + PIECE;
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const int row = row0 + r;
                const uint32_t o = uint32_t(row) * 128u + (uint32_t(cg ^ (row & 7)) << 4);
                const uint4 qraw = ok ? *reinterpret_cast<const uint4*>(opQ + o) : make_uint4(0, 0, 0, 0);
                const uint4 kraw = ok ? *reinterpret_cast<const uint4*>(opK + o) : make_uint4(0, 0, 0, 0);
                float qf[8], kf[8], qt[8], kt[8], k0[8];
                unpack8(qraw, qf);
                unpack8(kraw, kf);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    // exponents are <= 0 in exact arithmetic; the clamps absorb cumsum rounding
                    qt[e] = qf[e] * __expf(fminf(Bv[r][e], 0.f));
                    kt[e] = kf[e] * __expf(fminf(gamma[e] - Bv[r][e], 0.f));
                    k0[e] = kt[e] * eNG[e];
                }
                const uint4 qh = pack8(qt);
                if (ok && !SK) {
                    *reinterpret_cast<uint4*>(opQ + o) = qh;
                    *reinterpret_cast<uint4*>(opK + o) = pack8(k0);
                }
                if (row < nvalid) {
                    const int64_t off = (bh * L + t0 + row) * K + ch0;
                    *reinterpret_cast<uint4*>(Qt + off) = qh;
                    *reinterpret_cast<uint4*>(Kt + off) = pack8(kt);
                }
            }
            fence_proxy_async_smem();
            mbar_arrive(&bar.ops_ready[b]);
        }
        named_sync(1, 256);  // the list of exact-path channels and the scalar decay table are complete
        // ---- P from TMEM: thread = row, 64 columns
        const int q4 = warp & 3, h = warp >> 2;
        const int row = 32 * q4 + lane;
        // tcgen05.ld is warp-collective: the condition must be the same for the whole warp
        const bool have = __all_sync(0xffffffffu, ok && mbar_wait(&bar.p_done, 0, err, abort_flag));
        const int nuns = bar.nuns;  // the same for every element thread
        // exact terms of the channels beyond the bound, accumulated column-major in X[col][row] (fp32,
        // the operand memory, free once P is complete); 8 channels per round, warp w building the
        // cumsum / q / k columns of one of them in the gate staging area (free after the last piece)
        float* X = reinterpret_cast<float*>(base);
        float* tabB = reinterpret_cast<float*>(base + LA_OFF);
        float* tabQ = tabB + 8 * C;
        float* tabK = tabQ + 8 * C;
        if (nuns > 0) {
            if (have)
                for (int jj = 0; jj < 64; ++jj) X[(64 * h + jj) * C + row] = 0.f;
            for (int b0 = 0; b0 < nuns; b0 += 8) {
                named_sync(1, 256);
                const int u = b0 + warp;
                if (have && u < nuns) {
                    const int ch = bar.uns[u];
                    float a[4], qa[4], ka[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int tk = 4 * lane + e;
                        const bool v = tk < nvalid;
                        const int64_t tt = t0 + (v ? tk : 0);
                        const int64_t off = (bh * L + tt) * K + ch;
                        a[e] = v ? gate_at<K, GK>(ga, bh, tt, ch, L) : 0.f;
                        qa[e] = v ? __bfloat162float(q[off]) : 0.f;
                        ka[e] = v ? __bfloat162float(k[off]) : 0.f;
                    }
                    a[1] += a[0];
                    a[2] += a[1];
                    a[3] += a[2];
                    float incl = a[3];
#pragma unroll
                    for (int d = 1; d < 32; d <<= 1) {
                        const float o = __shfl_up_sync(0xffffffffu, incl, d);
                        if (lane >= d) incl += o;
                    }
                    const float excl = incl - a[3];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        tabB[warp * C + 4 * lane + e] = excl + a[e];
                        tabQ[warp * C + 4 * lane + e] = qa[e];
                        tabK[warp * C + 4 * lane + e] = ka[e];
                    }
                }
                named_sync(1, 256);
                const int nb = !have ? 0 : nuns - b0 < 8 ? nuns - b0 : 8;
                for (int w2 = 0; w2 < nb; ++w2) {
                    const float Bi = tabB[w2 * C + row], qi = tabQ[w2 * C + row];
                    const int jend = row < 64 * h + 63 ? row : 64 * h + 63;
                    for (int j = 64 * h; j <= jend; ++j)
                        X[j * C + row] += qi * tabK[w2 * C + j] * __expf(fminf(Bi - tabB[w2 * C + j], 0.f));
                }
            }
        }
        if (have) {
            tc_fence_after();
            const float brow = SK ? bar.btab[row] : 0.f;
            uint4* dst = reinterpret_cast<uint4*>(P + ((bh * N + i) * C + row) * C + 64 * h);
#pragma unroll
            for (int c16 = 0; c16 < 4; ++c16) {
                float y[16];
                tmem_ld16(tmem + (uint32_t(32 * q4) << 16) + uint32_t(64 * h + 16 * c16), y);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const int col = 64 * h + 16 * c16 + e;
                    float v = y[e];
                    if (SK) v *= __expf(fminf(brow - bar.btab[col], 0.f));  // decay e^{b_j - b_s}
                    else if (nuns > 0) v += X[col * C + row];
                    y[e] = col <= row ? v : 0.f;
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

constexpr size_t kSmem = 1024 + BAR_OFF + sizeof(PrepBars);
static_assert(3 * 8 * C * sizeof(float) <= LA_BYTES, "exact-path tables fit the gate staging area");

// [outer][rows][inner] tensor, box [128 rows x 64 inner]: bf16 with the 128-byte swizzle (operand
// layout) or fp32 unswizzled (gate tile)
bool map_piece(CUtensorMap* m, const void* p, uint64_t inner, uint64_t rows, uint64_t outer, bool f32) {
    const uint64_t es = f32 ? 4 : 2;
    const uint64_t dims[3] = {inner, rows, outer};
    const uint64_t strides[2] = {inner * es, inner * rows * es};
    const uint32_t box[3] = {uint32_t(KP), uint32_t(C), 1};
    return encode_tmap(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, p, dims,
                       strides, box, f32 ? CU_TENSOR_MAP_SWIZZLE_NONE : CU_TENSOR_MAP_SWIZZLE_128B);
}

template <int GK>
gla_status prep_launch_gk(const Problem& p, const void* q, const void* k, const GateArgs& ga, __nv_bfloat16* Qt,
                          __nv_bfloat16* Kt, __nv_bfloat16* P, float* gam, cudaStream_t s) {
    CUtensorMap m[3];
    memset(m, 0, sizeof(m));
    const uint64_t L = uint64_t(p.L), K = uint64_t(p.K), BH = uint64_t(p.BH);
    // scalar kinds read no gate tile: the q map stands in for the unused descriptor
    if (!(map_piece(&m[0], q, K, L, BH, false) && map_piece(&m[1], k, K, L, BH, false) &&
          (scalar_kind(GK) ? map_piece(&m[2], q, K, L, BH, false) : map_piece(&m[2], ga.g, K, L, BH, true))))
        return GLA_ERR_CUDA;
    auto fn = p.K == 256 ? k_tc_prep<256, GK> : k_tc_prep<128, GK>;
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kSmem)) != cudaSuccess)
        return GLA_ERR_CUDA;
    GLA_LAUNCH_PDL("tc_prep", fn, dim3(unsigned(p.N), unsigned(p.BH)), kThreads, kSmem, s, m[0], m[1], m[2],
                   static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k), ga, Qt, Kt, P, gam,
                   p.L, p.N, device_error_word());
    return GLA_OK;
}

}  // namespace

gla_status tc_prep_launch(const Problem& p, const void* q, const void* k, const float* la, __nv_bfloat16* Qt,
                          __nv_bfloat16* Kt, __nv_bfloat16* P, float* gam, int gate_kind, cudaStream_t s) {
    const GateArgs ga{la, gate_kind, p.inv_tau, p.H};
    switch (gate_kind) {
        case kGateScalar: return prep_launch_gk<kGateScalar>(p, q, k, ga, Qt, Kt, P, gam, s);
        case kGateHead: return prep_launch_gk<kGateHead>(p, q, k, ga, Qt, Kt, P, gam, s);
        case kGatePreact: return prep_launch_gk<kGatePreact>(p, q, k, ga, Qt, Kt, P, gam, s);
        default: return prep_launch_gk<kGateChannel>(p, q, k, ga, Qt, Kt, P, gam, s);
    }
}

}  // namespace gla
