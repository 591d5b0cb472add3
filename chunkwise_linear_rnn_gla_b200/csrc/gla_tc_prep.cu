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
// Roles (one CTA per chunk, 288 threads, two CTAs per SM): warps 0-7 (warp
// I = rows 16I .. 16I+15, lane = a pair of adjacent key channels) load log a,
// q and k of one 64-channel piece straight into registers (8-, 4- and 4-byte
// coalesced loads), do the cumsum and the elementwise work, write Q~/K~ to HBM
// and the swizzled operand piece to shared memory; warp 8 owns TMEM and issues
// the four MMAs of each piece as soon as it is complete (operand pieces are
// double-buffered); at the end warps 0-7 read P back from TMEM (warp w: lanes
// 32(w%4).., columns 64(w/4) ..) and store it.

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
constexpr int KP = 64;                      // key channels per piece
constexpr uint32_t PIECE = 16384;           // one [128 x 64] bf16 operand piece
constexpr int kThreads = 288;
constexpr float kSafeDecay = 64.f;          // |B| bound for the tensor-core form

struct PrepBars {
    float tot[2][8][KP];  // per-piece, per 16-row segment gate sums (first: 8-byte aligned)
    float btab[C];        // scalar kinds: the per-token cumsum b_t
    uint64_t ops_ready[2], mma_done[2], p_done, drain;
    uint32_t tmem_slot;
    int abort_flag;
    int nuns;
    unsigned short uns[256];  // key channels that take the exact path
};

constexpr uint32_t kTabOff = 4 * PIECE + (uint32_t(sizeof(PrepBars)) + 15u) / 16u * 16u;  // exact-path tables

// byte offset of (row, channel c64 of a piece) in a K-major SW128 piece
__device__ __forceinline__ uint32_t piece_off(int row, int c64) {
    return uint32_t(row) * 128u + uint32_t(((c64 >> 3) ^ (row & 7)) << 4) + uint32_t(c64 & 7) * 2u;
}

constexpr bool scalar_kind(int GK) { return GK == kGateScalar || GK == kGateHead; }

// Rows of one 64-channel piece: the log decays of a channel pair (fp32; preact: logsigmoid(z) / tau; the
// scalar kinds: the row's one decay for both) and q, k (bf16 pairs) of rows 16I .. 16I+15. Rows past the
// end of the sequence (last chunk only) read the last valid row and are zeroed.
template <int K, bool FULL, int GK>
__device__ __forceinline__ void load_rows(const GateArgs& ga, int64_t bh, int64_t t0, int64_t ch,
                                          const __nv_bfloat16* qp, const __nv_bfloat16* kp, int I, int nvalid,
                                          int64_t L, float2* bb, uint32_t* qv, uint32_t* kv) {
#pragma unroll
    for (int r = 0; r < 16; ++r) {
        const int row = 16 * I + r;
        const bool v = FULL || row < nvalid;
        const int rr = FULL ? row : (v ? row : nvalid - 1);
        const uint32_t o = uint32_t(rr) * uint32_t(K);
        float2 l2;
        if (GK == kGateScalar) l2.x = l2.y = ga.g[bh * L + t0 + rr];
        else if (GK == kGateHead) l2.x = l2.y = ga.g[bh % ga.H];
        else l2 = *reinterpret_cast<const float2*>(ga.g + (bh * L + t0 + rr) * K + ch);
        if (GK == kGatePreact) l2 = make_float2(logsigmoid_f(l2.x) * ga.inv_tau, logsigmoid_f(l2.y) * ga.inv_tau);
        const uint32_t qq = *reinterpret_cast<const uint32_t*>(qp + o);
        const uint32_t kk = *reinterpret_cast<const uint32_t*>(kp + o);
        bb[r] = v ? make_float2(la_floor(l2.x), la_floor(l2.y)) : make_float2(0.f, 0.f);
        qv[r] = v ? qq : 0u;
        kv[r] = v ? kk : 0u;
    }
}

template <int K, int GK>
__global__ void __launch_bounds__(kThreads, 2)
    k_tc_prep(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k, GateArgs ga,
              __nv_bfloat16* __restrict__ Qt, __nv_bfloat16* __restrict__ Kt, __nv_bfloat16* __restrict__ P,
              float* __restrict__ gam, int64_t L, int64_t N, int* err) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    // operand buffers: [b][Q~ piece, K^0 piece], b = piece parity
    PrepBars& bar = *reinterpret_cast<PrepBars*>(base + 4 * PIECE);
    volatile int* abort_flag = &bar.abort_flag;
    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    const int i = blockIdx.x;
    const int64_t bh = blockIdx.y;
    const int64_t t0 = int64_t(i) * C;
    const int nvalid = int(L - t0 < C ? L - t0 : C);
    const int npiece = int(K / KP);

    if (tid == 0) {
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bar.ops_ready[b], 256);
            mbar_init(&bar.mma_done[b], 1);
        }
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
    // programmatic dependent launch: the prologue above overlapped the previous kernel's tail;
    // nothing below touches global memory before that kernel has completed
    pdl_launch_dependents();
    pdl_wait();

    if (warp == 8) {
        if (lane == 0) {
            const uint32_t id = idesc_bf16_f32(128, 128, false, false);
            bool ok = true;
            for (int t = 0; t < npiece && ok; ++t) {
                const int b = t & 1;
                ok = mbar_wait(&bar.ops_ready[b], uint32_t((t >> 1) & 1), err, abort_flag);
                if (!ok) break;
                tc_fence_after();
                const uint32_t a0 = smem_u32(base + b * 2 * PIECE), b0 = a0 + PIECE;
#pragma unroll
                for (int kk = 0; kk < KP / 16; ++kk)
                    mma_bf16(tmem, sdesc_sw128(a0 + kk * 32, 16, 1024), sdesc_sw128(b0 + kk * 32, 16, 1024), id,
                             (t > 0 || kk > 0) ? 1u : 0u);
                mma_commit(&bar.mma_done[b]);
            }
            if (ok) mma_commit(&bar.p_done);
            mma_commit(&bar.drain);
            mbar_drain(&bar.drain, 0);
        }
    } else {
        const int I = warp;
        const int cp = 2 * lane;  // channel pair within the piece
        // Every compute thread passes every named barrier, also after a wait gave up (bar.sync
        // has no time limit); a failed wait only skips the work.
        bool ok = true;
        for (int t = 0; t < npiece; ++t) {
            const int b = t & 1;
            const int64_t ch = int64_t(KP) * t + cp;
            const int64_t rb = (bh * L + t0) * K + ch;
            float2 bb[16];
            uint32_t qv[16], kv[16];
            if (nvalid == C)
                load_rows<K, true, GK>(ga, bh, t0, ch, q + rb, k + rb, I, nvalid, L, bb, qv, kv);
            else
                load_rows<K, false, GK>(ga, bh, t0, ch, q + rb, k + rb, I, nvalid, L, bb, qv, kv);
            float2 run = make_float2(0.f, 0.f);
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                run.x += bb[r].x;
                run.y += bb[r].y;
                bb[r] = run;
            }
            *reinterpret_cast<float2*>(&bar.tot[b][I][cp]) = run;
            named_sync(1, 256);
            float2 pre = make_float2(0.f, 0.f), gamma = make_float2(0.f, 0.f);
#pragma unroll
            for (int J = 0; J < 8; ++J) {
                const float2 v = *reinterpret_cast<const float2*>(&bar.tot[b][J][cp]);
                if (J < I) {
                    pre.x += v.x;
                    pre.y += v.y;
                }
                gamma.x += v.x;
                gamma.y += v.y;
            }
            const bool unsafe0 = !scalar_kind(GK) && gamma.x < -kSafeDecay;
            const bool unsafe1 = !scalar_kind(GK) && gamma.y < -kSafeDecay;
            const float eNG0 = unsafe0 ? 0.f : __expf(fmaxf(-gamma.x, 0.f));  // e^{-Gamma} <= e^64
            const float eNG1 = unsafe1 ? 0.f : __expf(fmaxf(-gamma.y, 0.f));
            if (I == 0) {
                *reinterpret_cast<float2*>(gam + (bh * N + i) * K + ch) =
                    make_float2(__expf(fminf(gamma.x, 0.f)), __expf(fminf(gamma.y, 0.f)));
                if (unsafe0) bar.uns[atomicAdd(&bar.nuns, 1)] = (unsigned short)ch;
                if (unsafe1) bar.uns[atomicAdd(&bar.nuns, 1)] = (unsigned short)(ch + 1);
            }
            // the operand buffer of this parity is free once the MMAs of piece t-2 are done
            if (t >= 2) ok = ok && mbar_wait(&bar.mma_done[b], uint32_t(((t >> 1) - 1) & 1), err, abort_flag);
            uint8_t* opQ = base + b * 2 * PIECE;
            uint8_t* opK = opQ + PIECE;
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                const int row = 16 * I + r;
                const float Bx = pre.x + bb[r].x, By = pre.y + bb[r].y;
                const float2 qf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&qv[r]));
                const float2 kf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&kv[r]));
                // exponents are <= 0 in exact arithmetic; the clamps absorb cumsum rounding
                const float qt0 = qf.x * __expf(fminf(Bx, 0.f)), qt1 = qf.y * __expf(fminf(By, 0.f));
                const float kt0 = kf.x * __expf(fminf(gamma.x - Bx, 0.f));
                const float kt1 = kf.y * __expf(fminf(gamma.y - By, 0.f));
                const uint32_t qh = pack_bf16x2(qt0, qt1);
                const uint32_t o = piece_off(row, cp);
                if (ok) {  // scalar kinds: the raw q and k (the decay weights the product afterwards)
                    *reinterpret_cast<uint32_t*>(opQ + o) = scalar_kind(GK) ? qv[r] : qh;
                    *reinterpret_cast<uint32_t*>(opK + o) = scalar_kind(GK) ? kv[r] : pack_bf16x2(kt0 * eNG0, kt1 * eNG1);
                }
                if (scalar_kind(GK) && t == 0 && lane == 0) bar.btab[row] = Bx;
                if (row < nvalid) {
                    const int64_t off = (bh * L + t0 + row) * K + ch;
                    *reinterpret_cast<uint32_t*>(Qt + off) = qh;
                    *reinterpret_cast<uint32_t*>(Kt + off) = pack_bf16x2(kt0, kt1);
                }
            }
            fence_proxy_async_smem();
            mbar_arrive(&bar.ops_ready[b]);
        }
        named_sync(1, 256);  // the list of exact-path channels is complete
        // ---- P from TMEM: thread = row, 64 columns
        const int q4 = warp & 3, h = warp >> 2;
        const int row = 32 * q4 + lane;
        // tcgen05.ld is warp-collective: the condition must be the same for the whole warp
        const bool have = __all_sync(0xffffffffu, ok && mbar_wait(&bar.p_done, 0, err, abort_flag));
        const int nuns = bar.nuns;  // the same for every compute thread
        // exact terms of the channels beyond the bound, accumulated column-major in
        // X[col][row] (fp32, the operand memory, free once P is complete); 8 channels per
        // round, warp w building the cumsum / q / k columns of one of them
        float* X = reinterpret_cast<float*>(base);
        float* tabB = reinterpret_cast<float*>(base + kTabOff);
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
                        const int64_t off = (bh * L + t0 + (v ? tk : 0)) * K + ch;
                        // per-channel kinds only (the scalar kinds have no exact path)
                        const float x = ga.g[(bh * L + t0 + (v ? tk : 0)) * K + ch];
                        a[e] = v ? la_floor(GK == kGatePreact ? logsigmoid_f(x) * ga.inv_tau : x) : 0.f;
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
            const float brow = scalar_kind(GK) ? bar.btab[row] : 0.f;
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
                    if (scalar_kind(GK)) v *= __expf(fminf(brow - bar.btab[col], 0.f));  // decay e^{b_j - b_s}
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

constexpr size_t kSmem = 1024 + kTabOff + 3 * 8 * C * sizeof(float);

template <int GK>
gla_status prep_launch_gk(const Problem& p, const void* q, const void* k, const GateArgs& ga, __nv_bfloat16* Qt,
                          __nv_bfloat16* Kt, __nv_bfloat16* P, float* gam, cudaStream_t s) {
    auto fn = p.K == 256 ? k_tc_prep<256, GK> : k_tc_prep<128, GK>;
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kSmem)) != cudaSuccess)
        return GLA_ERR_CUDA;
    GLA_LAUNCH_PDL("tc_prep", fn, dim3(unsigned(p.N), unsigned(p.BH)), kThreads, kSmem, s,
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
