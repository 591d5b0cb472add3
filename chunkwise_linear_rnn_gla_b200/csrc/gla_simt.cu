// CUDA-core (SIMT) chunkwise GLA: every product and sum in fp32.
//
// This is the fp32-input path of the library and the fp32 cross-check of the
// tensor-core path. It follows the chunkwise form of the recurrence
// S_t = diag(alpha_t) S_{t-1} + k_t^T v_t, o_t = q_t S_t ("Gated Linear
// Attention Transformers with Hardware-Efficient Training", atlas.scime.ai
// summary, section "Approach": chunkwise algorithm with materialised
// inter-chunk states). With B the per-chunk inclusive cumsum of log alpha and
// Gamma = B at the chunk's last row:
//   o_j     = (q_j * e^{B_j}) S_[i] + sum_{s<=j} P_js v_s,
//   P_js    = sum_c q_jc k_sc e^{B_jc - B_sc}           (two-level: log space inside
//                                                        a sub-chunk, rescaled
//                                                        products across them)
//   S_[i+1] = diag(e^Gamma) S_[i] + sum_j (k_j * e^{Gamma - B_j})^T v_j
// and the backward in the same form with D_i = dL/dS_[i+1]; the gate gradient
// is the closed-form reverse cumsum of q*dq - k*dk plus sum_v dhT*hT.
//
// All exponents are <= 0 (B is non-increasing inside a chunk), so no step can
// overflow; rows past the end of the sequence are never read.

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "gla_common.cuh"
#include "gla_internal.h"

namespace gla {
namespace {

constexpr int kThreads = 256;

// ---------------------------------------------------------------------------
// Per-chunk inclusive cumsum of log alpha (one thread per key channel).
__global__ void __launch_bounds__(128) k_chunk_cumsum(const float* __restrict__ la, float* __restrict__ Bc,
                                                      int64_t L, int64_t K, int C) {
    const int64_t c = int64_t(blockIdx.x) * 128 + threadIdx.x;
    if (c >= K) return;
    const int64_t bh = blockIdx.z;
    const int64_t t0 = int64_t(blockIdx.y) * C;
    const int64_t t1 = t0 + C < L ? t0 + C : L;
    const float* src = la + (bh * L) * K + c;
    float* dst = Bc + (bh * L) * K + c;
    float acc = 0.f;
    for (int64_t t = t0; t < t1; ++t) {
        acc += la_floor(src[t * K]);
        dst[t * K] = acc;
    }
}

// ---------------------------------------------------------------------------
// Intra-chunk scores P_js = sum_c q_jc k_sc exp(B_jc - B_sc) for s <= j < nvalid
// (zero elsewhere), layout P[BH,N,C,C], with the two-level (secondary)
// chunking of the chunk form ("Gated Linear Attention Transformers with
// Hardware-Efficient Training", atlas.scime.ai summary, "Approach"): the rows
// split into sub-chunks of `csub`. For a key s in sub-chunk J below the query
// row's sub-chunk I, with rho_J = B at the last row of J,
//   q_j k_s e^{B_j - B_s} = (q_j e^{B_j - rho_J}) (k_s e^{rho_J - B_s}),
// both factors <= 1 (B is non-increasing), so the off-diagonal sub-blocks are
// plain products of rescaled operands: one exponential per (query row, key
// sub-chunk, channel) and one per key. Pairs inside a diagonal sub-block take
// one exponential per term (log space). Thread = one query row and SPT keys.
template <typename T, int C>
__global__ void __launch_bounds__(kThreads) k_intra_P(const T* __restrict__ q, const T* __restrict__ k,
                                                      const float* __restrict__ Bc, float* __restrict__ P,
                                                      int64_t L, int64_t K, int64_t N, int csub) {
    constexpr int CT = 16;                       // channel tile
    constexpr int SPT = C < 16 ? C : 16;         // keys per thread
    constexpr int TPR = C / SPT;                 // threads per query row
    constexpr int RPP = kThreads / TPR;          // query rows per pass
    constexpr int NPASS = (C + RPP - 1) / RPP;
    __shared__ float sq[C][CT + 1], sk[C][CT + 1], skr[C][CT + 1], sB[C][CT + 1];
    const int64_t i = blockIdx.x, bh = blockIdx.y;
    const int64_t t0 = i * C;
    const int nvalid = int(L - t0 < C ? L - t0 : C);
    const int tid = threadIdx.x;
    const int s0 = (tid % TPR) * SPT;
    float acc[NPASS][SPT];
#pragma unroll
    for (int ps = 0; ps < NPASS; ++ps)
#pragma unroll
        for (int e = 0; e < SPT; ++e) acc[ps][e] = 0.f;
    for (int64_t c0 = 0; c0 < K; c0 += CT) {
        for (int e = tid; e < C * CT; e += kThreads) {
            const int j = e / CT, cc = e % CT;
            const int64_t c = c0 + cc;
            float a = 0.f, b = 0.f, g = 0.f;
            if (j < nvalid && c < K) {
                const int64_t off = (bh * L + t0 + j) * K + c;
                a = ldf(q + off);
                b = ldf(k + off);
                g = Bc[off];
            }
            sq[j][cc] = a;
            sk[j][cc] = b;
            sB[j][cc] = g;
        }
        __syncthreads();
        // keys rescaled to the end of their sub-chunk (its last valid row): k_s e^{rho_J - B_s}
        for (int e = tid; e < C * CT; e += kThreads) {
            const int srow = e / CT, cc = e % CT;
            int last = (srow / csub + 1) * csub - 1;
            last = last < nvalid - 1 ? last : nvalid - 1;
            skr[srow][cc] = srow < nvalid ? sk[srow][cc] * expf(sB[last][cc] - sB[srow][cc]) : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int ps = 0; ps < NPASS; ++ps) {
            const int j = tid / TPR + ps * RPP;
            if (j >= C || j >= nvalid || s0 > j) continue;
            const int I = j / csub;
            for (int cc = 0; cc < CT; ++cc) {
                const float qj = sq[j][cc], bj = sB[j][cc];
                int Jc = -1;        // key sub-chunk whose factor is cached
                float qr = 0.f;     // q_j e^{B_j - rho_J}
#pragma unroll
                for (int e = 0; e < SPT; ++e) {
                    const int sk_ = s0 + e;
                    const int J = sk_ / csub;
                    float term = 0.f;
                    if (J == I) {
                        term = qj * sk[sk_][cc] * expf(bj - sB[sk_][cc]);
                    } else if (J < I) {
                        if (J != Jc) {
                            const int last = (J + 1) * csub - 1;  // J < I: its rows are all valid
                            qr = qj * expf(bj - sB[last][cc]);
                            Jc = J;
                        }
                        term = qr * skr[sk_][cc];
                    }
                    acc[ps][e] += sk_ <= j ? term : 0.f;
                }
            }
        }
        __syncthreads();
    }
    float* dst = P + (bh * N + i) * C * C;
#pragma unroll
    for (int ps = 0; ps < NPASS; ++ps) {
        const int j = tid / TPR + ps * RPP;
        if (j >= C) continue;
#pragma unroll
        for (int e = 0; e < SPT; ++e) dst[j * C + s0 + e] = (j < nvalid && s0 + e <= j) ? acc[ps][e] : 0.f;
    }
}

// ---------------------------------------------------------------------------
// Intra-chunk dP_js = dO_j . v_s for s <= j < nvalid (zero elsewhere).
template <typename T, int C>
__global__ void __launch_bounds__(kThreads) k_intra_dP(const T* __restrict__ dO, const T* __restrict__ v,
                                                       float* __restrict__ dP, int64_t L, int64_t V, int64_t N) {
    constexpr int VT = 16;
    constexpr int PP = (C * C + kThreads - 1) / kThreads;
    __shared__ float sd[C][VT + 1], sv[C][VT + 1];
    const int64_t i = blockIdx.x, bh = blockIdx.y;
    const int64_t t0 = i * C;
    const int nvalid = int(L - t0 < C ? L - t0 : C);
    const int tid = threadIdx.x;
    float acc[PP];
#pragma unroll
    for (int p = 0; p < PP; ++p) acc[p] = 0.f;
    for (int64_t x0 = 0; x0 < V; x0 += VT) {
        for (int e = tid; e < C * VT; e += kThreads) {
            const int j = e / VT, xx = e % VT;
            const int64_t x = x0 + xx;
            float a = 0.f, b = 0.f;
            if (j < nvalid && x < V) {
                const int64_t off = (bh * L + t0 + j) * V + x;
                a = ldf(dO + off);
                b = ldf(v + off);
            }
            sd[j][xx] = a;
            sv[j][xx] = b;
        }
        __syncthreads();
#pragma unroll
        for (int p = 0; p < PP; ++p) {
            const int pair = tid + p * kThreads;
            if (pair < C * C) {
                const int j = pair / C, s = pair % C;
                if (s <= j && j < nvalid) {
                    float a = acc[p];
#pragma unroll
                    for (int xx = 0; xx < VT; ++xx) a += sd[j][xx] * sv[s][xx];
                    acc[p] = a;
                }
            }
        }
        __syncthreads();
    }
    float* dst = dP + (bh * N + i) * C * C;
#pragma unroll
    for (int p = 0; p < PP; ++p) {
        const int pair = tid + p * kThreads;
        if (pair < C * C) dst[pair] = acc[p];
    }
}

// ---------------------------------------------------------------------------
// Sequential state walk over chunks for one [32 x 64] tile of the state.
// Forward (REVERSE = false): Sbuf[i] = S_[i] (state entering chunk i), then
//   S <- diag(e^Gamma) S + sum_j (x_j * e^{Gamma - B_j})^T y_j,  x = k, y = v.
// Backward (REVERSE = true), chunks in reverse: Sbuf[i] = D_i, then
//   D <- diag(e^Gamma) D + sum_j (x_j * e^{B_j})^T y_j,  x = q, y = dO.
// Sbuf has N+1 slots per (b,h) in the forward (slot N = final state) and N in
// the backward. `init` may be null (zero); `fin` (final state) may be null.
template <typename T, bool REVERSE>
__global__ void __launch_bounds__(kThreads) k_state_walk(const T* __restrict__ x, const T* __restrict__ y,
                                                         const float* __restrict__ Bc,
                                                         const float* __restrict__ init, float* __restrict__ Sbuf,
                                                         float* __restrict__ fin, int64_t L, int64_t K, int64_t V,
                                                         int C, int64_t N) {
    constexpr int BK = 32, BV = 64, RT = 32;  // RT: rows of the chunk per smem tile
    __shared__ float sx[RT][BK + 1];
    __shared__ float sy[RT][BV + 1];
    __shared__ float sG[BK];
    const int tid = threadIdx.x;
    const int vl = tid % BV, r0 = tid / BV;  // rows r0 + 4m
    const int64_t kb = int64_t(blockIdx.x) * BK, vb = int64_t(blockIdx.y) * BV, bh = blockIdx.z;
    const int64_t vcol = vb + vl;
    const int64_t nslots = REVERSE ? N : N + 1;
    float S[BK / 4];
#pragma unroll
    for (int m = 0; m < BK / 4; ++m) {
        const int64_t kr = kb + r0 + 4 * m;
        S[m] = (init && kr < K && vcol < V) ? init[(bh * K + kr) * V + vcol] : 0.f;
    }
    for (int64_t step = 0; step < N; ++step) {
        const int64_t i = REVERSE ? N - 1 - step : step;
        const int64_t t0 = i * C;
        const int nvalid = int(L - t0 < C ? L - t0 : C);
        float* slot = Sbuf + (bh * nslots + i) * K * V;
#pragma unroll
        for (int m = 0; m < BK / 4; ++m) {
            const int64_t kr = kb + r0 + 4 * m;
            if (kr < K && vcol < V) slot[kr * V + vcol] = S[m];
        }
        if (tid < BK) {
            const int64_t c = kb + tid;
            sG[tid] = c < K ? Bc[(bh * L + t0 + nvalid - 1) * K + c] : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int m = 0; m < BK / 4; ++m) S[m] *= expf(sG[r0 + 4 * m]);
        for (int j0 = 0; j0 < nvalid; j0 += RT) {
            for (int e = tid; e < RT * BK; e += kThreads) {
                const int jj = e / BK, cc = e % BK;
                const int64_t c = kb + cc;
                float val = 0.f;
                if (j0 + jj < nvalid && c < K) {
                    const int64_t off = (bh * L + t0 + j0 + jj) * K + c;
                    const float b = Bc[off];
                    val = ldf(x + off) * expf(REVERSE ? b : sG[cc] - b);
                }
                sx[jj][cc] = val;
            }
            for (int e = tid; e < RT * BV; e += kThreads) {
                const int jj = e / BV, xx = e % BV;
                const int64_t col = vb + xx;
                sy[jj][xx] = (j0 + jj < nvalid && col < V) ? ldf(y + (bh * L + t0 + j0 + jj) * V + col) : 0.f;
            }
            __syncthreads();
#pragma unroll 4
            for (int jj = 0; jj < RT; ++jj) {
                const float yv = sy[jj][vl];
#pragma unroll
                for (int m = 0; m < BK / 4; ++m) S[m] += sx[jj][r0 + 4 * m] * yv;
            }
            __syncthreads();
        }
    }
    if (!REVERSE) {
        float* slot = Sbuf + (bh * nslots + N) * K * V;
#pragma unroll
        for (int m = 0; m < BK / 4; ++m) {
            const int64_t kr = kb + r0 + 4 * m;
            if (kr < K && vcol < V) slot[kr * V + vcol] = S[m];
        }
    }
    if (fin) {
#pragma unroll
        for (int m = 0; m < BK / 4; ++m) {
            const int64_t kr = kb + r0 + 4 * m;
            if (kr < K && vcol < V) fin[(bh * K + kr) * V + vcol] = S[m];
        }
    }
}

// ---------------------------------------------------------------------------
// Output of chunk i for a 64-wide slice of v:
//   o_j = (q_j * e^{B_j}) S_[i] + sum_{s<=j} P_js v_s.
template <typename T, int C>
__global__ void __launch_bounds__(kThreads) k_output(const T* __restrict__ q, const T* __restrict__ v,
                                                     const float* __restrict__ Bc, const float* __restrict__ Sbuf,
                                                     const float* __restrict__ P, T* __restrict__ o, int64_t L,
                                                     int64_t K, int64_t V, int64_t N) {
    constexpr int BV = 64, KT = 32, RPT = C / 4;
    __shared__ float sa[C][KT + 1];
    __shared__ float sb[KT][BV + 1];
    const int tid = threadIdx.x;
    const int vl = tid % BV, g = tid / BV;
    const int64_t vb = int64_t(blockIdx.x) * BV, i = blockIdx.y, bh = blockIdx.z;
    const int64_t t0 = i * C;
    const int nvalid = int(L - t0 < C ? L - t0 : C);
    const float* S = Sbuf + (bh * (N + 1) + i) * K * V;
    float acc[RPT];
#pragma unroll
    for (int m = 0; m < RPT; ++m) acc[m] = 0.f;
    for (int64_t c0 = 0; c0 < K; c0 += KT) {
        for (int e = tid; e < C * KT; e += kThreads) {
            const int j = e / KT, cc = e % KT;
            const int64_t c = c0 + cc;
            float val = 0.f;
            if (j < nvalid && c < K) {
                const int64_t off = (bh * L + t0 + j) * K + c;
                val = ldf(q + off) * expf(Bc[off]);
            }
            sa[j][cc] = val;
        }
        for (int e = tid; e < KT * BV; e += kThreads) {
            const int cc = e / BV, xx = e % BV;
            const int64_t c = c0 + cc, col = vb + xx;
            sb[cc][xx] = (c < K && col < V) ? S[c * V + col] : 0.f;
        }
        __syncthreads();
#pragma unroll 4
        for (int cc = 0; cc < KT; ++cc) {
            const float sv = sb[cc][vl];
#pragma unroll
            for (int m = 0; m < RPT; ++m) acc[m] += sa[g + 4 * m][cc] * sv;
        }
        __syncthreads();
    }
    constexpr int ST = C < KT ? C : KT;
    const float* Pc = P + (bh * N + i) * C * C;
    for (int s0 = 0; s0 < C; s0 += ST) {
        for (int e = tid; e < C * ST; e += kThreads) {
            const int j = e / ST, ss = e % ST;
            sa[j][ss] = Pc[j * C + s0 + ss];
        }
        for (int e = tid; e < ST * BV; e += kThreads) {
            const int ss = e / BV, xx = e % BV;
            const int64_t col = vb + xx;
            sb[ss][xx] = (s0 + ss < nvalid && col < V) ? ldf(v + (bh * L + t0 + s0 + ss) * V + col) : 0.f;
        }
        __syncthreads();
#pragma unroll 4
        for (int ss = 0; ss < ST; ++ss) {
            const float vv = sb[ss][vl];
#pragma unroll
            for (int m = 0; m < RPT; ++m) acc[m] += sa[g + 4 * m][ss] * vv;
        }
        __syncthreads();
    }
    const int64_t col = vb + vl;
    if (col < V) {
#pragma unroll
        for (int m = 0; m < RPT; ++m) {
            const int j = g + 4 * m;
            if (j < nvalid) stf(o + (bh * L + t0 + j) * V + col, acc[m]);
        }
    }
}

// ---------------------------------------------------------------------------
// dq and dk of chunk i for a 32-wide slice of key channels, plus
// r = q*dq - k*dk (fp32) for the gate gradient.
//   dq_j = e^{B_j} * (dO_j S_[i]^T) + sum_{s<=j} dP_js k_s e^{B_j - B_s}
//   dk_s = e^{Gamma - B_s} * (v_s D_i^T) + sum_{j>=s} dP_js q_j e^{B_j - B_s}
template <typename T, int C>
__global__ void __launch_bounds__(kThreads) k_dqdk(const T* __restrict__ q, const T* __restrict__ k,
                                                   const T* __restrict__ v, const T* __restrict__ dO,
                                                   const float* __restrict__ Bc, const float* __restrict__ Sbuf,
                                                   const float* __restrict__ Dbuf, const float* __restrict__ dP,
                                                   T* __restrict__ dq, T* __restrict__ dk, float* __restrict__ r,
                                                   int64_t L, int64_t K, int64_t V, int64_t N, int csub) {
    constexpr int KT = 32, VT = 32, RPT = C / 8;
    extern __shared__ float smem[];
    float(*sq)[KT + 1] = reinterpret_cast<float(*)[KT + 1]>(smem);
    float(*sk)[KT + 1] = reinterpret_cast<float(*)[KT + 1]>(smem + C * (KT + 1));
    float(*sB)[KT + 1] = reinterpret_cast<float(*)[KT + 1]>(smem + 2 * C * (KT + 1));
    float(*sx)[VT + 1] = reinterpret_cast<float(*)[VT + 1]>(smem + 3 * C * (KT + 1));
    float(*sy)[VT + 1] = reinterpret_cast<float(*)[VT + 1]>(smem + 3 * C * (KT + 1) + C * (VT + 1));
    const int tid = threadIdx.x;
    const int cl = tid % KT, g = tid / KT;  // rows g + 8m
    const int64_t kb = int64_t(blockIdx.x) * KT, i = blockIdx.y, bh = blockIdx.z;
    const int64_t t0 = i * C;
    const int nvalid = int(L - t0 < C ? L - t0 : C);
    const int64_t c = kb + cl;
    for (int e = tid; e < C * KT; e += kThreads) {
        const int j = e / KT, cc = e % KT;
        const int64_t ch = kb + cc;
        float a = 0.f, b = 0.f, gg = 0.f;
        if (j < nvalid && ch < K) {
            const int64_t off = (bh * L + t0 + j) * K + ch;
            a = ldf(q + off);
            b = ldf(k + off);
            gg = Bc[off];
        } else if (ch < K) {
            gg = Bc[(bh * L + t0 + nvalid - 1) * K + ch];
        }
        sq[j][cc] = a;
        sk[j][cc] = b;
        sB[j][cc] = gg;
    }
    float aq[RPT], ak[RPT];
#pragma unroll
    for (int m = 0; m < RPT; ++m) aq[m] = ak[m] = 0.f;
    const float* S = Sbuf + (bh * (N + 1) + i) * K * V;
    const float* D = Dbuf + (bh * N + i) * K * V;
    // inter-chunk parts: dO S^T and v D^T over the value dimension
    for (int pass = 0; pass < 2; ++pass) {
        const T* X = pass == 0 ? dO : v;
        const float* Y = pass == 0 ? S : D;
        for (int64_t x0 = 0; x0 < V; x0 += VT) {
            __syncthreads();
            for (int e = tid; e < C * VT; e += kThreads) {
                const int j = e / VT, xx = e % VT;
                const int64_t col = x0 + xx;
                sx[j][xx] = (j < nvalid && col < V) ? ldf(X + (bh * L + t0 + j) * V + col) : 0.f;
            }
            for (int e = tid; e < KT * VT; e += kThreads) {
                const int cc = e / VT, xx = e % VT;
                const int64_t ch = kb + cc, col = x0 + xx;
                sy[cc][xx] = (ch < K && col < V) ? Y[ch * V + col] : 0.f;
            }
            __syncthreads();
#pragma unroll 4
            for (int xx = 0; xx < VT; ++xx) {
                const float yv = sy[cl][xx];
#pragma unroll
                for (int m = 0; m < RPT; ++m) {
                    if (pass == 0) aq[m] += sx[g + 8 * m][xx] * yv;
                    else ak[m] += sx[g + 8 * m][xx] * yv;
                }
            }
        }
    }
    __syncthreads();
    const float Gam = sB[C - 1][cl];  // rows past nvalid hold B of the last valid row
    const float* dPc = dP + (bh * N + i) * C * C;
    // two-level (secondary) chunking as in the forward scores: a pair in different sub-chunks is the
    // product of two factors <= 1 through rho = B at the last row of the earlier sub-chunk; a pair
    // in the same sub-chunk takes one exponential per term (log space)
    auto rho = [&](int J) { return sB[(J + 1) * csub - 1 < C ? (J + 1) * csub - 1 : C - 1][cl]; };
#pragma unroll
    for (int m = 0; m < RPT; ++m) {
        const int j = g + 8 * m;
        const float bj = sB[j][cl];
        float dqj = aq[m] * expf(bj);
        float dkj = ak[m] * expf(Gam - bj);
        if (j < nvalid) {
            const int I = j / csub;
            // dq_j: keys s <= j; sub-chunk J < I contributes e^{B_j - rho_J} sum_s dP_js k_s e^{rho_J - B_s}
            for (int J = 0; J < I; ++J) {
                const float rJ = rho(J);
                float part = 0.f;
                for (int s = J * csub; s < (J + 1) * csub; ++s) part += dPc[j * C + s] * sk[s][cl] * expf(rJ - sB[s][cl]);
                dqj += expf(bj - rJ) * part;
            }
            for (int s = I * csub; s <= j; ++s) dqj += dPc[j * C + s] * sk[s][cl] * expf(bj - sB[s][cl]);
            // dk_j: queries jj >= j; those past j's sub-chunk I contribute e^{rho_I - B_j} dP q e^{B_jj - rho_I}
            const int jend = (I + 1) * csub < nvalid ? (I + 1) * csub : nvalid;
            for (int jj = j; jj < jend; ++jj) dkj += dPc[jj * C + j] * sq[jj][cl] * expf(sB[jj][cl] - bj);
            if (jend < nvalid) {
                const float rI = rho(I);
                float part = 0.f;
                for (int jj = jend; jj < nvalid; ++jj) part += dPc[jj * C + j] * sq[jj][cl] * expf(sB[jj][cl] - rI);
                dkj += expf(rI - bj) * part;
            }
            if (c < K) {
                const int64_t off = (bh * L + t0 + j) * K + c;
                stf(dq + off, dqj);
                stf(dk + off, dkj);
                r[off] = sq[j][cl] * dqj - sk[j][cl] * dkj;
            }
        }
    }
}

// ---------------------------------------------------------------------------
// dv of chunk i for a 64-wide value slice:
//   dv_s = (k_s * e^{Gamma - B_s}) D_i + sum_{j>=s} P_js dO_j
template <typename T, int C>
__global__ void __launch_bounds__(kThreads) k_dv(const T* __restrict__ k, const T* __restrict__ dO,
                                                 const float* __restrict__ Bc, const float* __restrict__ Dbuf,
                                                 const float* __restrict__ P, T* __restrict__ dv, int64_t L,
                                                 int64_t K, int64_t V, int64_t N) {
    constexpr int BV = 64, KT = 32, RPT = C / 4;
    __shared__ float sa[KT > C ? KT : C][KT + 1];
    __shared__ float sb[KT][BV + 1];
    __shared__ float sG[KT];
    const int tid = threadIdx.x;
    const int vl = tid % BV, g = tid / BV;
    const int64_t vb = int64_t(blockIdx.x) * BV, i = blockIdx.y, bh = blockIdx.z;
    const int64_t t0 = i * C;
    const int nvalid = int(L - t0 < C ? L - t0 : C);
    const float* D = Dbuf + (bh * N + i) * K * V;
    float acc[RPT];
#pragma unroll
    for (int m = 0; m < RPT; ++m) acc[m] = 0.f;
    for (int64_t c0 = 0; c0 < K; c0 += KT) {
        if (tid < KT) {
            const int64_t ch = c0 + tid;
            sG[tid] = ch < K ? Bc[(bh * L + t0 + nvalid - 1) * K + ch] : 0.f;
        }
        __syncthreads();
        for (int e = tid; e < C * KT; e += kThreads) {
            const int s = e / KT, cc = e % KT;
            const int64_t ch = c0 + cc;
            float val = 0.f;
            if (s < nvalid && ch < K) {
                const int64_t off = (bh * L + t0 + s) * K + ch;
                val = ldf(k + off) * expf(sG[cc] - Bc[off]);
            }
            sa[s][cc] = val;
        }
        for (int e = tid; e < KT * BV; e += kThreads) {
            const int cc = e / BV, xx = e % BV;
            const int64_t ch = c0 + cc, col = vb + xx;
            sb[cc][xx] = (ch < K && col < V) ? D[ch * V + col] : 0.f;
        }
        __syncthreads();
#pragma unroll 4
        for (int cc = 0; cc < KT; ++cc) {
            const float dv_ = sb[cc][vl];
#pragma unroll
            for (int m = 0; m < RPT; ++m) acc[m] += sa[g + 4 * m][cc] * dv_;
        }
        __syncthreads();
    }
    // intra: sum_{j>=s} P_js dO_j, P^T staged in smem 32 query rows at a time
    constexpr int JT = C < KT ? C : KT;
    const float* Pc = P + (bh * N + i) * C * C;
    for (int j0 = 0; j0 < C; j0 += JT) {
        for (int e = tid; e < JT * C; e += kThreads) {
            const int jj = e / C, s = e % C;
            sa[s][jj] = Pc[(j0 + jj) * C + s];
        }
        for (int e = tid; e < JT * BV; e += kThreads) {
            const int jj = e / BV, xx = e % BV;
            const int64_t col = vb + xx;
            sb[jj][xx] = (j0 + jj < nvalid && col < V) ? ldf(dO + (bh * L + t0 + j0 + jj) * V + col) : 0.f;
        }
        __syncthreads();
#pragma unroll 4
        for (int jj = 0; jj < JT; ++jj) {
            const float d = sb[jj][vl];
#pragma unroll
            for (int m = 0; m < RPT; ++m) acc[m] += sa[g + 4 * m][jj] * d;
        }
        __syncthreads();
    }
    const int64_t col = vb + vl;
    if (col < V) {
#pragma unroll
        for (int m = 0; m < RPT; ++m) {
            const int s = g + 4 * m;
            if (s < nvalid) stf(dv + (bh * L + t0 + s) * V + col, acc[m]);
        }
    }
}

// ---------------------------------------------------------------------------
// Closed-form gate gradient: dlog_a_t = sum_{s>=t} r_s + sum_v dhT * hT.
__global__ void __launch_bounds__(128) k_dlog_a(const float* __restrict__ r, const float* __restrict__ hT,
                                                const float* __restrict__ dhT, float* __restrict__ dla,
                                                int64_t L, int64_t K, int64_t V, int64_t hT_stride) {
    const int64_t c = int64_t(blockIdx.x) * 128 + threadIdx.x;
    if (c >= K) return;
    const int64_t bh = blockIdx.y;
    float run = 0.f;
    if (dhT) {
        const float* a = dhT + (bh * K + c) * V;
        const float* b = hT + bh * hT_stride + c * V;
        for (int64_t x = 0; x < V; ++x) run += a[x] * b[x];
    }
    const float* src = r + bh * L * K + c;
    float* dst = dla + bh * L * K + c;
    for (int64_t t = L - 1; t >= 0; --t) {
        run += src[t * K];
        dst[t * K] = run;
    }
}

template <int C>
size_t dqdk_smem() {
    return sizeof(float) * (3 * C * 33 + C * 33 + 32 * 33);
}

template <typename T, int C>
gla_status fwd_impl(const Problem& p, const T* q, const T* k, const T* v, const float* la, const float* h0, T* o,
                    float* hT, float* Bc, float* P, float* Sbuf, cudaStream_t s) {
    const dim3 gc(unsigned(cdiv(p.K, 128)), unsigned(p.N), unsigned(p.BH));
    GLA_LAUNCH("simt_chunk_cumsum", k_chunk_cumsum, gc, 128, 0, s, la, Bc, p.L, p.K, p.C);
    GLA_LAUNCH("simt_intra_P", (k_intra_P<T, C>), dim3(unsigned(p.N), unsigned(p.BH)), kThreads, 0, s, q, k, Bc,
               P, p.L, p.K, p.N, int(p.c));
    const dim3 gw(unsigned(cdiv(p.K, 32)), unsigned(cdiv(p.V, 64)), unsigned(p.BH));
    GLA_LAUNCH("simt_state_walk", (k_state_walk<T, false>), gw, kThreads, 0, s, k, v, Bc, h0, Sbuf, hT, p.L, p.K,
               p.V, p.C, p.N);
    const dim3 go(unsigned(cdiv(p.V, 64)), unsigned(p.N), unsigned(p.BH));
    GLA_LAUNCH("simt_output", (k_output<T, C>), go, kThreads, 0, s, q, v, Bc, Sbuf, P, o, p.L, p.K, p.V, p.N);
    return GLA_OK;
}

template <typename T, int C>
gla_status bwd_impl(const Problem& p, const T* q, const T* k, const T* v, const float* la, const float* h0,
                    const T* dO, const float* dhT, T* dq, T* dk, T* dv, float* dla, float* dh0, float* Bc, float* P,
                    float* Sbuf, float* Dbuf, float* dP, float* r, bool reuse, cudaStream_t s) {
    if (!reuse) {
        const dim3 gc(unsigned(cdiv(p.K, 128)), unsigned(p.N), unsigned(p.BH));
        GLA_LAUNCH("simt_chunk_cumsum", k_chunk_cumsum, gc, 128, 0, s, la, Bc, p.L, p.K, p.C);
        GLA_LAUNCH("simt_intra_P", (k_intra_P<T, C>), dim3(unsigned(p.N), unsigned(p.BH)), kThreads, 0, s, q, k,
                   Bc, P, p.L, p.K, p.N, int(p.c));
        const dim3 gw(unsigned(cdiv(p.K, 32)), unsigned(cdiv(p.V, 64)), unsigned(p.BH));
        GLA_LAUNCH("simt_state_walk", (k_state_walk<T, false>), gw, kThreads, 0, s, k, v, Bc, h0, Sbuf,
                   (float*)nullptr, p.L, p.K, p.V, p.C, p.N);
    }
    const dim3 gw(unsigned(cdiv(p.K, 32)), unsigned(cdiv(p.V, 64)), unsigned(p.BH));
    GLA_LAUNCH("simt_dstate_walk", (k_state_walk<T, true>), gw, kThreads, 0, s, q, dO, Bc, dhT, Dbuf, dh0, p.L, p.K,
               p.V, p.C, p.N);
    GLA_LAUNCH("simt_intra_dP", (k_intra_dP<T, C>), dim3(unsigned(p.N), unsigned(p.BH)), kThreads, 0, s, dO, v, dP,
               p.L, p.V, p.N);
    const size_t sm = dqdk_smem<C>();
    if (cudaFuncSetAttribute(k_dqdk<T, C>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(sm)) != cudaSuccess)
        return GLA_ERR_CUDA;
    const dim3 gq(unsigned(cdiv(p.K, 32)), unsigned(p.N), unsigned(p.BH));
    GLA_LAUNCH("simt_dqdk", (k_dqdk<T, C>), gq, kThreads, sm, s, q, k, v, dO, Bc, Sbuf, Dbuf, dP, dq, dk, r, p.L, p.K,
               p.V, p.N, int(p.c));
    const dim3 gv(unsigned(cdiv(p.V, 64)), unsigned(p.N), unsigned(p.BH));
    GLA_LAUNCH("simt_dv", (k_dv<T, C>), gv, kThreads, 0, s, k, dO, Bc, Dbuf, P, dv, p.L, p.K, p.V, p.N);
    const float* hT = Sbuf + p.N * p.K * p.V;  // slot N of (b,h) = 0; stride below
    GLA_LAUNCH("simt_dlog_a", k_dlog_a, dim3(unsigned(cdiv(p.K, 128)), unsigned(p.BH)), 128, 0, s, r, hT, dhT, dla,
               p.L, p.K, p.V, (p.N + 1) * p.K * p.V);
    return GLA_OK;
}

struct SimtBuffers {
    float *Bc, *P, *Sbuf, *Dbuf, *dP, *r;
};

SimtBuffers carve(const Problem& p, Arena& a, bool bwd) {
    SimtBuffers b{};
    b.Bc = a.take<float>(size_t(p.BH * p.L * p.K));
    b.P = a.take<float>(size_t(p.BH * p.N * p.C * p.C));
    b.Sbuf = a.take<float>(size_t(p.BH * (p.N + 1) * p.K * p.V));
    if (bwd) {
        b.Dbuf = a.take<float>(size_t(p.BH * p.N * p.K * p.V));
        b.dP = a.take<float>(size_t(p.BH * p.N * p.C * p.C));
        b.r = a.take<float>(size_t(p.BH * p.L * p.K));
    }
    return b;
}

template <typename T>
gla_status fwd_dispatch(const Problem& p, const void* q, const void* k, const void* v, const float* la,
                        const float* h0, void* o, float* hT, const SimtBuffers& b, cudaStream_t s) {
    auto Q = static_cast<const T*>(q);
    auto Kp = static_cast<const T*>(k);
    auto Vp = static_cast<const T*>(v);
    auto O = static_cast<T*>(o);
    switch (p.C) {
        case 16: return fwd_impl<T, 16>(p, Q, Kp, Vp, la, h0, O, hT, b.Bc, b.P, b.Sbuf, s);
        case 32: return fwd_impl<T, 32>(p, Q, Kp, Vp, la, h0, O, hT, b.Bc, b.P, b.Sbuf, s);
        case 64: return fwd_impl<T, 64>(p, Q, Kp, Vp, la, h0, O, hT, b.Bc, b.P, b.Sbuf, s);
        case 128: return fwd_impl<T, 128>(p, Q, Kp, Vp, la, h0, O, hT, b.Bc, b.P, b.Sbuf, s);
    }
    return GLA_ERR_UNSUPPORTED;
}

template <typename T>
gla_status bwd_dispatch(const Problem& p, const void* q, const void* k, const void* v, const float* la,
                        const float* h0, const void* dO, const float* dhT, void* dq, void* dk, void* dv, float* dla,
                        float* dh0, const SimtBuffers& b, bool reuse, cudaStream_t s) {
    auto Q = static_cast<const T*>(q);
    auto Kp = static_cast<const T*>(k);
    auto Vp = static_cast<const T*>(v);
    auto G = static_cast<const T*>(dO);
    auto DQ = static_cast<T*>(dq);
    auto DK = static_cast<T*>(dk);
    auto DV = static_cast<T*>(dv);
#define GLA_BWD_CASE(CC)                                                                                       \
    case CC:                                                                                                   \
        return bwd_impl<T, CC>(p, Q, Kp, Vp, la, h0, G, dhT, DQ, DK, DV, dla, dh0, b.Bc, b.P, b.Sbuf, b.Dbuf, \
                               b.dP, b.r, reuse, s);
    switch (p.C) {
        GLA_BWD_CASE(16)
        GLA_BWD_CASE(32)
        GLA_BWD_CASE(64)
        GLA_BWD_CASE(128)
    }
#undef GLA_BWD_CASE
    return GLA_ERR_UNSUPPORTED;
}

}  // namespace

size_t simt_fwd_workspace(const Problem& p) {
    Arena a = make_arena(p, nullptr, 0);
    carve(p, a, false);
    return a.used;
}

size_t simt_bwd_workspace(const Problem& p) {
    Arena a = make_arena(p, nullptr, 0);
    carve(p, a, true);
    return a.used;
}

void simt_layout(const Problem& p, Arena& a, bool bwd) { carve(p, a, bwd); }

gla_status simt_chunk_cumsum(const Problem& p, const float* log_a, float* Bc, cudaStream_t s) {
    const dim3 gc(unsigned(cdiv(p.K, 128)), unsigned(p.N), unsigned(p.BH));
    GLA_LAUNCH("simt_chunk_cumsum", k_chunk_cumsum, gc, 128, 0, s, log_a, Bc, p.L, p.K, p.C);
    return GLA_OK;
}

gla_status simt_fwd(const Problem& p, const void* q, const void* k, const void* v, const float* la, const float* h0,
                    void* o, float* hT, Arena& ws, cudaStream_t s) {
    SimtBuffers b = carve(p, ws, false);
    if (ws.used > ws.cap) return GLA_ERR_WORKSPACE;
    if (p.bf16) return fwd_dispatch<__nv_bfloat16>(p, q, k, v, la, h0, o, hT, b, s);
    return fwd_dispatch<float>(p, q, k, v, la, h0, o, hT, b, s);
}

gla_status simt_bwd(const Problem& p, const void* q, const void* k, const void* v, const float* la,
                    const float* h0, const void* dO, const float* dhT, void* dq, void* dk, void* dv, float* dla,
                    float* dh0, Arena& ws, cudaStream_t s) {
    SimtBuffers b = carve(p, ws, true);
    if (ws.used > ws.cap) return GLA_ERR_WORKSPACE;
    const bool reuse = (p.flags & GLA_FLAG_WS_FROM_FWD) != 0;
    if (p.bf16) return bwd_dispatch<__nv_bfloat16>(p, q, k, v, la, h0, dO, dhT, dq, dk, dv, dla, dh0, b, reuse, s);
    return bwd_dispatch<float>(p, q, k, v, la, h0, dO, dhT, dq, dk, dv, dla, dh0, b, reuse, s);
}

}  // namespace gla
