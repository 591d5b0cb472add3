// Gated slot attention (GSA) on the GLA kernels.
//
// The method (mlsanity card for "Gated Slot Attention for Efficient Linear-Time
// Sequence Modeling", abstract): a memory of m slots, forgotten by a GLA-style
// data-dependent gate and read by two GLA layers joined by a softmax over the
// slots. Per batch b and head h, with a_t = exp(log_a_t) in (0,1]^m and the
// write weight w_t = 1 - a_t:
//     Kmem_t = diag(a_t) Kmem_{t-1} + w_t^T k_t          [m x Dk]
//     Vmem_t = diag(a_t) Vmem_{t-1} + w_t^T v_t          [m x Dv]
//     s_t    = softmax(Kmem_t q_t^T),   o_t = s_t Vmem_t
//
// Both memories are GLA states over the slot dimension (GLA key w, gate a):
//   layer one: GLA state Kmem (value k). Its read Kmem_t q_t^T is the gradient
//     of <q_t, o'_t> with respect to the GLA query, i.e. the dq of a GLA
//     backward with dO = q (the query itself drops out of dq);
//   layer two: a plain GLA with query s, key w, value v.
// The backward follows the same algebra:
//   layer two's GLA backward: ds, the gradient of w, dv, its gate gradient;
//   softmax backward:         G = s * (ds - <s, ds>) = dL/dlogits;
//   layer one: dq is the forward of the GLA with query G, key w, value k;
//     d(w), dk and the gate gradient are that GLA's backward with dO = q
//     (its dk, dv and dlog_a; its closed-form gate gradient holds as is);
//   the gate: dlog_a = dla_1 + dla_2 - a * (dw_1 + dw_2).
// Every step runs in the library's kernels. Two routes:
//  - tensor cores (bf16, m = 128): the GLA walk, output and backward kernels,
//    each memory walked once (the backward reuses the forward's chunk states),
//    plus two kernels of this method (gla_gsa_read.cu): the slot gate's
//    preparation (w and the walks' operands, for both layers) and the slot
//    read, which evaluates the logits and the read gradient in fp32 with the
//    softmax and its backward fused, and whose epilogue also forms the next
//    layer's query operands (Q~ and the masked scores), so no separate GLA
//    preparation runs;
//  - CUDA cores (every other shape): the GLA passes in fp32 (bf16 tensors are
//    converted at the boundary), the logits as the query gradient of layer
//    one, and the elementwise kernels below.

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "gla_common.cuh"
#include "gla_gate.cuh"
#include "gla_internal.h"
#include "gla_tc.h"

namespace gla {
namespace {

constexpr int kThreads = 256;

unsigned grid_for(int64_t n) {
    int64_t b = cdiv(n, kThreads);
    if (b > 148 * 32) b = 148 * 32;  // grid-stride beyond this
    if (b < 1) b = 1;
    return unsigned(b);
}

// w = 1 - exp(log a); four elements per thread (n4 = n / 4 groups), the tail one by one
template <typename T>
__global__ void __launch_bounds__(kThreads) k_write_weight(const float* __restrict__ la, T* __restrict__ w,
                                                           int64_t n) {
    const int64_t n4 = n / 4, stride = int64_t(gridDim.x) * blockDim.x;
    for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n4; i += stride) {
        const float4 x = reinterpret_cast<const float4*>(la)[i];
        stf(w + 4 * i, 1.f - __expf(x.x));
        stf(w + 4 * i + 1, 1.f - __expf(x.y));
        stf(w + 4 * i + 2, 1.f - __expf(x.z));
        stf(w + 4 * i + 3, 1.f - __expf(x.w));
    }
    for (int64_t i = 4 * n4 + int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += stride)
        stf(w + i, 1.f - __expf(la[i]));
}

// s = softmax over each row of m logits; one warp per row, rows grid-strided
template <typename T>
__global__ void __launch_bounds__(kThreads) k_softmax(const T* __restrict__ z, T* __restrict__ s, int64_t rows,
                                                      int m) {
    const int lane = threadIdx.x & 31;
    const int64_t warps = int64_t(gridDim.x) * (blockDim.x >> 5);
    for (int64_t r = int64_t(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows; r += warps) {
        const T* zr = z + r * m;
        float mx = -INFINITY;
        for (int c = lane; c < m; c += 32) mx = fmaxf(mx, ldf(zr + c));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        float sum = 0.f;
        for (int c = lane; c < m; c += 32) sum += __expf(ldf(zr + c) - mx);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        const float inv = 1.f / sum;
        for (int c = lane; c < m; c += 32) stf(s + r * m + c, __expf(ldf(zr + c) - mx) * inv);
    }
}

// G = s * (ds - <s, ds>) per row
template <typename T>
__global__ void __launch_bounds__(kThreads) k_softmax_bwd(const T* __restrict__ s, const T* __restrict__ ds,
                                                          T* __restrict__ G, int64_t rows, int m) {
    const int lane = threadIdx.x & 31;
    const int64_t warps = int64_t(gridDim.x) * (blockDim.x >> 5);
    for (int64_t r = int64_t(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows; r += warps) {
        const int64_t o0 = r * m;
        float dot = 0.f;
        for (int c = lane; c < m; c += 32) dot = fmaf(ldf(s + o0 + c), ldf(ds + o0 + c), dot);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
        for (int c = lane; c < m; c += 32) stf(G + o0 + c, ldf(s + o0 + c) * (ldf(ds + o0 + c) - dot));
    }
}

// dla += dla1 - a * (dw1 + dw2)   (dla holds layer two's gate gradient on entry); four elements per
// thread, the tail one by one
template <typename T>
__global__ void __launch_bounds__(kThreads) k_gate_grad(const float* __restrict__ la, const float* __restrict__ dla1,
                                                        const T* __restrict__ dw1, const T* __restrict__ dw2,
                                                        float* __restrict__ dla, int64_t n) {
    const int64_t n4 = n / 4, stride = int64_t(gridDim.x) * blockDim.x;
    for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n4; i += stride) {
        const float4 x = reinterpret_cast<const float4*>(la)[i];
        const float4 g1 = reinterpret_cast<const float4*>(dla1)[i];
        float4 g = reinterpret_cast<const float4*>(dla)[i];
        const int64_t e = 4 * i;
        g.x += g1.x - __expf(x.x) * (ldf(dw1 + e) + ldf(dw2 + e));
        g.y += g1.y - __expf(x.y) * (ldf(dw1 + e + 1) + ldf(dw2 + e + 1));
        g.z += g1.z - __expf(x.z) * (ldf(dw1 + e + 2) + ldf(dw2 + e + 2));
        g.w += g1.w - __expf(x.w) * (ldf(dw1 + e + 3) + ldf(dw2 + e + 3));
        reinterpret_cast<float4*>(dla)[i] = g;
    }
    for (int64_t i = 4 * n4 + int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += stride)
        dla[i] = dla[i] + dla1[i] - __expf(la[i]) * (ldf(dw1 + i) + ldf(dw2 + i));
}

template <typename Tin, typename Tout>
__global__ void __launch_bounds__(kThreads) k_convert(const Tin* __restrict__ x, Tout* __restrict__ y, int64_t n) {
    for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += int64_t(gridDim.x) * blockDim.x)
        stf(y + i, ldf(x + i));
}

template <typename T>
gla_status write_weight(int64_t n, const float* la, T* w, cudaStream_t s) {
    GLA_LAUNCH("gsa_write_weight", k_write_weight<T>, grid_for(cdiv(n, 4)), kThreads, 0, s, la, w, n);
    return GLA_OK;
}

template <typename T>
gla_status gate_grad_sum(int64_t n, const float* la, const float* dla1, const T* dw1, const T* dw2, float* dla,
                         cudaStream_t s) {
    GLA_LAUNCH("gsa_gate_grad", k_gate_grad<T>, grid_for(cdiv(n, 4)), kThreads, 0, s, la, dla1, dw1, dw2, dla, n);
    return GLA_OK;
}

template <typename Tin, typename Tout>
gla_status convert(const void* x, void* y, int64_t n, cudaStream_t s) {
    if (!x || !y || n == 0) return GLA_OK;
    GLA_LAUNCH("gsa_convert", (k_convert<Tin, Tout>), grid_for(n), kThreads, 0, s, static_cast<const Tin*>(x),
               static_cast<Tout*>(y), n);
    return GLA_OK;
}

size_t path_ws(const Problem& p) {
    Arena a = make_arena(p, nullptr, 0);
    (p.impl == GLA_IMPL_TC ? tc_layout : simt_layout)(p, a, true);
    return a.used;
}

// ================================================================ tensor-core route
// Workspace: [w][s bf16][s fp32][layer two's GLA workspace][layer one's GLA workspace], then for the
// backward [G][dw1][dw2][dla1][scratch dq]. The forward's part is a prefix of the backward's: the
// backward takes w, s, both memories' chunk states and layer two's preparation as they are.
struct TcRoute {
    __nv_bfloat16 *w, *s_b;
    float* s_f;
    char *wsB, *wsA;
    size_t capB, capA;
    __nv_bfloat16 *G, *dw1, *dw2, *junk;
    float* dla1;
};

TcRoute carve_tc(const GsaProblem& g, Arena& a, bool bwd) {
    const size_t nm = size_t(g.B.BH * g.B.L * g.m);
    TcRoute b{};
    b.w = a.take<__nv_bfloat16>(nm);
    b.s_b = a.take<__nv_bfloat16>(nm);
    b.s_f = a.take<float>(nm);
    b.capB = path_ws(g.B);
    b.wsB = a.take<char>(b.capB);
    b.capA = path_ws(g.A);
    b.wsA = a.take<char>(b.capA);
    if (bwd) {
        b.G = a.take<__nv_bfloat16>(nm);
        b.dw1 = a.take<__nv_bfloat16>(nm);
        b.dw2 = a.take<__nv_bfloat16>(nm);
        b.junk = a.take<__nv_bfloat16>(nm);
        b.dla1 = a.take<float>(nm);
    }
    return b;
}

// w, both memories' chunk states (walks with GLA key w over k and over v), the read weights s, and layer
// two's preparation (query s, key w): its K~ and e^Gamma from the gate preparation, its Q~ and scores P
// from the slot read's epilogue. hkT / hvT (nullable) receive the final memories.
gla_status tc_forward_state(const GsaProblem& g, const void* q, const void* k, const void* v, const float* la,
                            const float* hk0, const float* hv0, float* hkT, float* hvT, const TcRoute& r,
                            TcBuffers& A, TcBuffers& B, cudaStream_t s) {
    // w, and the walks' operands K~ = w e^{Gamma - B} and e^Gamma
    gla_status st = tc_gsa_gate_prep_launch(g.A, la, r.w, A.Kt, A.gam, B.Kt, B.gam, s);
    if (st == GLA_OK)
        st = tc_states_walk_launch(g.A, A.Kt, static_cast<const __nv_bfloat16*>(k), A.gam, hk0, hkT, A.hT, A.states,
                                   A.segbuf, false, s, "tc_walk_states");
    if (st == GLA_OK)
        st = tc_states_walk_launch(g.B, A.Kt, static_cast<const __nv_bfloat16*>(v), A.gam, hv0, hvT, B.hT, B.states,
                                   B.segbuf, false, s, "tc_walk_states");
    if (st == GLA_OK)
        st = tc_gsa_slot_read_launch(g.A, q, k, A.states, la, nullptr, r.s_b, r.s_f, B.Qt, B.P, 0, s);
    return st;
}

gla_status tc_route_fwd(const GsaProblem& g, const void* q, const void* k, const void* v, const float* la,
                        const float* hk0, const float* hv0, void* o, float* hkT, float* hvT, const TcRoute& r,
                        cudaStream_t s) {
    Arena aA = make_arena(g.A, r.wsA, r.capA), aB = make_arena(g.B, r.wsB, r.capB);
    TcBuffers A = tc_carve(g.A, aA, true), B = tc_carve(g.B, aB, true);
    gla_status st = tc_forward_state(g, q, k, v, la, hk0, hv0, hkT, hvT, r, A, B, s);
    if (st != GLA_OK) return st;
    return tc_chunk_out_launch(g.B, B.Qt, B.states, B.P, static_cast<const __nv_bfloat16*>(v), false,
                               static_cast<__nv_bfloat16*>(o), false, s, "tc_output");
}

gla_status tc_route_bwd(const GsaProblem& g, const void* q, const void* k, const void* v, const float* la,
                        const float* hk0, const float* hv0, const void* dO, const float* dhkT, const float* dhvT,
                        void* dq, void* dk, void* dv, float* dla, float* dhk0, float* dhv0, bool reuse,
                        const TcRoute& r, cudaStream_t s) {
    Arena aA = make_arena(g.A, r.wsA, r.capA), aB = make_arena(g.B, r.wsB, r.capB);
    TcBuffers A = tc_carve(g.A, aA, true), B = tc_carve(g.B, aB, true);
    gla_status st = GLA_OK;
    if (!reuse) st = tc_forward_state(g, q, k, v, la, hk0, hv0, nullptr, nullptr, r, A, B, s);
    if (st != GLA_OK) return st;
    // layer two (query s, key w, value v) from the stored value memory: dv, the gradient of w and its gate
    // gradient (into dla, completed at the end); its query gradient is recomputed in fp32 below
    Problem pB = g.B;
    pB.flags = GLA_FLAG_WS_FROM_FWD;
    Arena bB = make_arena(g.B, r.wsB, r.capB);
    st = tc_bwd(pB, r.s_b, r.w, v, la, hv0, dO, dhvT, r.junk, r.dw2, dv, dla, dhv0, bB, s);
    // G = dL/dlogits: the read of the value memory with dO, through the softmax backward
    // with layer one's chunk-local operands (query G; K~ and e^Gamma are the gate preparation's)
    if (st == GLA_OK)
        st = tc_gsa_slot_read_launch(g.B, dO, v, B.states, la, r.s_f, r.G, nullptr, A.Qt, A.P, 1, s);
    if (st != GLA_OK) return st;
    // layer one (query G, key w, value k) from the stored key memory: dq is its output, then its backward
    // with dO = q gives dk (its dv), the gradient of w (its dk) and its gate gradient
    st = tc_chunk_out_launch(g.A, A.Qt, A.states, A.P, static_cast<const __nv_bfloat16*>(k), false,
                             static_cast<__nv_bfloat16*>(dq), false, s, "tc_output");
    if (st != GLA_OK) return st;
    Problem pA = g.A;
    pA.flags = GLA_FLAG_WS_FROM_FWD;
    Arena bA = make_arena(g.A, r.wsA, r.capA);
    st = tc_bwd(pA, r.G, r.w, k, la, hk0, q, dhkT, r.junk, r.dw1, dk, r.dla1, dhk0, bA, s);
    if (st != GLA_OK) return st;
    return gate_grad_sum<__nv_bfloat16>(g.B.BH * g.B.L * g.m, la, r.dla1, r.dw1, r.dw2, dla, s);
}

// ================================================================ CUDA-core route
// The GLA passes in fp32. Workspace: [w][s][layer two's GLA workspace][layer one's][logits][scratch dk']
// [scratch dv'][scratch dla'] [fp32 copies of bf16 inputs and outputs], then for the backward
// [G][ds][dw2][dw1][dla1].
struct SimtRoute {
    float *w, *s, *logits, *junk_dk, *junk_dv, *junk_dla;
    char *wsB, *wsA;
    size_t capB, capA;
    float *q, *k, *v, *o;        // fp32 copies (bf16 tensors only)
    float *dO, *dq, *dk, *dv;    // backward, bf16 tensors only
    float *G, *ds, *dw2, *dw1, *dla1;
};

SimtRoute carve_simt(const GsaProblem& g, Arena& a, bool bwd) {
    const size_t nm = size_t(g.B.BH * g.B.L * g.m);
    const size_t nk = size_t(g.B.BH * g.B.L * g.A.V), nv = size_t(g.B.BH * g.B.L * g.B.V);
    SimtRoute b{};
    b.w = a.take<float>(nm);
    b.s = a.take<float>(nm);
    b.capB = path_ws(g.B);
    b.wsB = a.take<char>(b.capB);
    b.capA = path_ws(g.A);
    b.wsA = a.take<char>(b.capA);
    b.logits = a.take<float>(nm);
    b.junk_dk = a.take<float>(nm);
    b.junk_dv = a.take<float>(nk);
    b.junk_dla = a.take<float>(nm);
    if (g.io_bf16) {
        b.q = a.take<float>(nk);
        b.k = a.take<float>(nk);
        b.v = a.take<float>(nv);
        b.o = a.take<float>(nv);
    }
    if (bwd) {
        if (g.io_bf16) {
            b.dO = a.take<float>(nv);
            b.dq = a.take<float>(nk);
            b.dk = a.take<float>(nk);
            b.dv = a.take<float>(nv);
        }
        b.G = a.take<float>(nm);
        b.ds = a.take<float>(nm);
        b.dw2 = a.take<float>(nm);
        b.dw1 = a.take<float>(nm);
        b.dla1 = a.take<float>(nm);
    }
    return b;
}

gla_status simt_fwd_pass(const Problem& p, const void* q, const void* k, const void* v, const float* la,
                         const float* h0, void* o, float* hT, char* base, size_t cap, cudaStream_t s) {
    Arena a = make_arena(p, base, cap);
    return simt_fwd(p, q, k, v, la, h0, o, hT, a, s);
}

gla_status simt_bwd_pass(const Problem& p, const void* q, const void* k, const void* v, const float* la,
                         const float* h0, const void* dO, const float* dhT, void* dq, void* dk, void* dv, float* dla,
                         float* dh0, char* base, size_t cap, cudaStream_t s) {
    Arena a = make_arena(p, base, cap);
    return simt_bwd(p, q, k, v, la, h0, dO, dhT, dq, dk, dv, dla, dh0, a, s);
}

gla_status softmax_rows(const GsaProblem& g, const float* z, float* sm, cudaStream_t s) {
    const int64_t rows = g.B.BH * g.B.L;
    GLA_LAUNCH("gsa_softmax", k_softmax<float>, grid_for(rows * 32), kThreads, 0, s, z, sm, rows, int(g.m));
    return GLA_OK;
}

gla_status softmax_rows_bwd(const GsaProblem& g, const float* sm, const float* ds, float* G, cudaStream_t s) {
    const int64_t rows = g.B.BH * g.B.L;
    GLA_LAUNCH("gsa_softmax_bwd", k_softmax_bwd<float>, grid_for(rows * 32), kThreads, 0, s, sm, ds, G, rows,
               int(g.m));
    return GLA_OK;
}

// w, then the logits (layer one's read) as the dq of a GLA backward with dO = q, then s
gla_status simt_read_weights(const GsaProblem& g, const float* q, const float* k, const float* la, const float* hk0,
                             const SimtRoute& b, cudaStream_t s) {
    gla_status st = write_weight<float>(g.B.BH * g.B.L * g.m, la, b.w, s);
    if (st != GLA_OK) return st;
    // the GLA query does not enter its own dq; w stands in for it (any finite tensor of that shape)
    st = simt_bwd_pass(g.A, b.w, b.w, k, la, hk0, q, nullptr, b.logits, b.junk_dk, b.junk_dv, b.junk_dla, nullptr,
                       b.wsA, b.capA, s);
    if (st != GLA_OK) return st;
    return softmax_rows(g, b.logits, b.s, s);
}

gla_status simt_route_fwd(const GsaProblem& g, const void* q, const void* k, const void* v, const float* la,
                          const float* hk0, const float* hv0, void* o, float* hkT, float* hvT, const SimtRoute& b,
                          cudaStream_t s) {
    const int64_t nk = g.B.BH * g.B.L * g.A.V, nv = g.B.BH * g.B.L * g.B.V;
    const float *q32 = static_cast<const float*>(q), *k32 = static_cast<const float*>(k),
                *v32 = static_cast<const float*>(v);
    float* o32 = static_cast<float*>(o);
    gla_status st = GLA_OK;
    if (g.io_bf16) {
        st = convert<__nv_bfloat16, float>(q, b.q, nk, s);
        if (st == GLA_OK) st = convert<__nv_bfloat16, float>(k, b.k, nk, s);
        if (st == GLA_OK) st = convert<__nv_bfloat16, float>(v, b.v, nv, s);
        if (st != GLA_OK) return st;
        q32 = b.q, k32 = b.k, v32 = b.v, o32 = b.o;
    }
    st = simt_read_weights(g, q32, k32, la, hk0, b, s);
    if (st == GLA_OK) st = simt_fwd_pass(g.B, b.s, b.w, v32, la, hv0, o32, hvT, b.wsB, b.capB, s);
    // the final key memory: layer one's end state (a forward whose output goes to scratch)
    if (st == GLA_OK && hkT) st = simt_fwd_pass(g.A, b.w, b.w, k32, la, hk0, b.junk_dv, hkT, b.wsA, b.capA, s);
    if (st == GLA_OK && g.io_bf16) st = convert<float, __nv_bfloat16>(b.o, o, nv, s);
    return st;
}

gla_status simt_route_bwd(const GsaProblem& g, const void* q, const void* k, const void* v, const float* la,
                          const float* hk0, const float* hv0, const void* dO, const float* dhkT, const float* dhvT,
                          void* dq, void* dk, void* dv, float* dla, float* dhk0, float* dhv0, bool reuse,
                          const SimtRoute& b, cudaStream_t s) {
    const int64_t nk = g.B.BH * g.B.L * g.A.V, nv = g.B.BH * g.B.L * g.B.V;
    const float *q32 = static_cast<const float*>(q), *k32 = static_cast<const float*>(k),
                *v32 = static_cast<const float*>(v), *dO32 = static_cast<const float*>(dO);
    float *dq32 = static_cast<float*>(dq), *dk32 = static_cast<float*>(dk), *dv32 = static_cast<float*>(dv);
    gla_status st = GLA_OK;
    if (g.io_bf16) {
        st = convert<__nv_bfloat16, float>(q, b.q, nk, s);
        if (st == GLA_OK) st = convert<__nv_bfloat16, float>(k, b.k, nk, s);
        if (st == GLA_OK) st = convert<__nv_bfloat16, float>(v, b.v, nv, s);
        if (st == GLA_OK) st = convert<__nv_bfloat16, float>(dO, b.dO, nv, s);
        if (st != GLA_OK) return st;
        q32 = b.q, k32 = b.k, v32 = b.v, dO32 = b.dO, dq32 = b.dq, dk32 = b.dk, dv32 = b.dv;
    }
    if (!reuse) st = simt_read_weights(g, q32, k32, la, hk0, b, s);
    if (st != GLA_OK) return st;
    // layer two's backward (from the forward's workspace when it is intact); its gate gradient goes to dla
    Problem pB = g.B;
    pB.flags = reuse ? GLA_FLAG_WS_FROM_FWD : 0;
    st = simt_bwd_pass(pB, b.s, b.w, v32, la, hv0, dO32, dhvT, b.ds, b.dw2, dv32, dla, dhv0, b.wsB, b.capB, s);
    if (st == GLA_OK) st = softmax_rows_bwd(g, b.s, b.ds, b.G, s);
    if (st != GLA_OK) return st;
    // layer one: dq = the forward of the GLA with query G, key w, value k; its backward with dO = q from the
    // same workspace gives dk (its dv), the gradient of w (its dk) and its gate gradient
    Problem pA = g.A;
    pA.flags = 0;
    st = simt_fwd_pass(pA, b.G, b.w, k32, la, hk0, dq32, nullptr, b.wsA, b.capA, s);
    if (st != GLA_OK) return st;
    pA.flags = GLA_FLAG_WS_FROM_FWD;
    st = simt_bwd_pass(pA, b.G, b.w, k32, la, hk0, q32, dhkT, b.logits, b.dw1, dk32, b.dla1, dhk0, b.wsA, b.capA, s);
    if (st == GLA_OK) st = gate_grad_sum<float>(g.B.BH * g.B.L * g.m, la, b.dla1, b.dw1, b.dw2, dla, s);
    if (st == GLA_OK && g.io_bf16) {
        st = convert<float, __nv_bfloat16>(b.dq, dq, nk, s);
        if (st == GLA_OK) st = convert<float, __nv_bfloat16>(b.dk, dk, nk, s);
        if (st == GLA_OK) st = convert<float, __nv_bfloat16>(b.dv, dv, nv, s);
    }
    return st;
}

// ================================================================ decode step
// One token per head, both memories updated in place (fp32), one block per head:
//   keys:   Kmem[c] <- a_c Kmem[c] + w_c k,  z_c = Kmem[c] . q      (w = 1 - a, exact in fp32)
//   read:   s = softmax(z)
//   values: Vmem[c] <- a_c Vmem[c] + w_c v,  o = sum_c s_c Vmem[c]
// A warp takes four slot rows at a time (their loads issued together, 16 bytes per lane); the row dot
// products reduce by shuffles, the softmax runs in one warp, and o sums the warps' partial rows through
// shared memory in a fixed order.
constexpr int kStepThreads = 512;  // two blocks per SM (at most 64 registers a thread): 256 heads stay one wave
constexpr int kStepRows = 4;

template <typename T>
__global__ void __launch_bounds__(kStepThreads, 2) k_gsa_step(const T* __restrict__ q, const T* __restrict__ k,
                                                           const T* __restrict__ v, const float* __restrict__ la,
                                                           float inv_tau, float* __restrict__ Km,
                                                           float* __restrict__ Vm, T* __restrict__ o, int m, int Dk,
                                                           int Dv) {
    extern __shared__ float sh[];
    // the arrays read as float4 first (Dk and Dv are multiples of 4, so every one starts on 16 bytes),
    // then the per-slot scalars
    const int nw = blockDim.x >> 5;
    float* op = sh;            // [warps][Dv]
    float* qs = op + nw * Dv;  // [Dk]
    float* ks = qs + Dk;       // [Dk]
    float* vs = ks + Dk;       // [Dv]
    float* as = vs + Dv;
    float* ws = as + m;
    float* zs = ws + m;
    const int64_t bh = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, wp = tid >> 5;
    for (int i = tid; i < Dk; i += blockDim.x) {
        qs[i] = ldf(q + bh * Dk + i);
        ks[i] = ldf(k + bh * Dk + i);
    }
    for (int i = tid; i < Dv; i += blockDim.x) vs[i] = ldf(v + bh * Dv + i);
    for (int c = tid; c < m; c += blockDim.x) {
        const float g = la[bh * m + c];
        const float a = __expf(inv_tau > 0.f ? logsigmoid_f(g) * inv_tau : g);
        as[c] = a;
        ws[c] = 1.f - a;
    }
    for (int i = tid; i < nw * Dv; i += blockDim.x) op[i] = 0.f;
    __syncthreads();
    const int dk4 = Dk / 4, dv4 = Dv / 4;
    float4* K4 = reinterpret_cast<float4*>(Km + bh * int64_t(m) * Dk);
    float4* V4 = reinterpret_cast<float4*>(Vm + bh * int64_t(m) * Dv);
    const float4* q4 = reinterpret_cast<const float4*>(qs);
    const float4* k4 = reinterpret_cast<const float4*>(ks);
    const float4* v4 = reinterpret_cast<const float4*>(vs);
    // ---- keys and logits
    for (int c0 = wp * kStepRows; c0 < m; c0 += nw * kStepRows) {
        float dot[kStepRows];
#pragma unroll
        for (int u = 0; u < kStepRows; ++u) dot[u] = 0.f;
        for (int d4 = lane; d4 < dk4; d4 += 32) {
            float4 r[kStepRows];
#pragma unroll
            for (int u = 0; u < kStepRows; ++u)
                if (c0 + u < m) r[u] = K4[int64_t(c0 + u) * dk4 + d4];
            const float4 kk = k4[d4], qq = q4[d4];
#pragma unroll
            for (int u = 0; u < kStepRows; ++u) {
                if (c0 + u >= m) continue;
                const float a = as[c0 + u], w = ws[c0 + u];
                float4 x = r[u];
                x.x = fmaf(a, x.x, w * kk.x);
                x.y = fmaf(a, x.y, w * kk.y);
                x.z = fmaf(a, x.z, w * kk.z);
                x.w = fmaf(a, x.w, w * kk.w);
                K4[int64_t(c0 + u) * dk4 + d4] = x;
                dot[u] = fmaf(x.x, qq.x, fmaf(x.y, qq.y, fmaf(x.z, qq.z, fmaf(x.w, qq.w, dot[u]))));
            }
        }
#pragma unroll
        for (int u = 0; u < kStepRows; ++u) {
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) dot[u] += __shfl_xor_sync(0xffffffffu, dot[u], off);
            if (lane == 0 && c0 + u < m) zs[c0 + u] = dot[u];
        }
    }
    __syncthreads();
    // ---- softmax over the slots (warp 0)
    if (wp == 0) {
        float mx = -INFINITY;
        for (int c = lane; c < m; c += 32) mx = fmaxf(mx, zs[c]);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        float sum = 0.f;
        for (int c = lane; c < m; c += 32) {
            const float e = __expf(zs[c] - mx);
            zs[c] = e;
            sum += e;
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
        const float inv = 1.f / sum;
        __syncwarp();
        for (int c = lane; c < m; c += 32) zs[c] *= inv;
    }
    __syncthreads();
    // ---- values and the read
    float4* o4 = reinterpret_cast<float4*>(op + wp * Dv);
    for (int c0 = wp * kStepRows; c0 < m; c0 += nw * kStepRows) {
        for (int d4 = lane; d4 < dv4; d4 += 32) {
            float4 r[kStepRows];
#pragma unroll
            for (int u = 0; u < kStepRows; ++u)
                if (c0 + u < m) r[u] = V4[int64_t(c0 + u) * dv4 + d4];
            const float4 vv = v4[d4];
            float4 acc = o4[d4];
#pragma unroll
            for (int u = 0; u < kStepRows; ++u) {
                if (c0 + u >= m) continue;
                const float a = as[c0 + u], w = ws[c0 + u], sc = zs[c0 + u];
                float4 y = r[u];
                y.x = fmaf(a, y.x, w * vv.x);
                y.y = fmaf(a, y.y, w * vv.y);
                y.z = fmaf(a, y.z, w * vv.z);
                y.w = fmaf(a, y.w, w * vv.w);
                V4[int64_t(c0 + u) * dv4 + d4] = y;
                acc.x = fmaf(sc, y.x, acc.x);
                acc.y = fmaf(sc, y.y, acc.y);
                acc.z = fmaf(sc, y.z, acc.z);
                acc.w = fmaf(sc, y.w, acc.w);
            }
            o4[d4] = acc;
        }
    }
    __syncthreads();
    for (int x = tid; x < Dv; x += blockDim.x) {
        float acc = 0.f;
        for (int w2 = 0; w2 < nw; ++w2) acc += op[w2 * Dv + x];
        stf(o + bh * Dv + x, acc);
    }
}

size_t step_smem(int64_t m, int64_t Dk, int64_t Dv) {
    return sizeof(float) * size_t(2 * Dk + Dv + 3 * m + (kStepThreads / 32) * Dv);
}

}  // namespace

bool gsa_tc_route(const Problem& A, const Problem& B, int64_t m) {
    return m == 128 && A.impl == GLA_IMPL_TC && B.impl == GLA_IMPL_TC && A.state_mode == GLA_STATE_MATERIALIZED &&
           B.state_mode == GLA_STATE_MATERIALIZED && tc_gsa_slot_read_supported(A) && tc_gsa_slot_read_supported(B);
}

// The pre-activation gate's expansion, log a = logsigmoid(z) / tau, in front of either route's layout (the
// backward reuses the forward's with the rest of its workspace).
float* carve_gate(const GsaProblem& g, Arena& a) {
    return g.preact ? a.take<float>(size_t(g.B.BH * g.B.L * g.m)) : nullptr;
}

gla_status expand_gate(const GsaProblem& g, const float* z, float* la, cudaStream_t s) {
    Problem p = g.A;  // key width m: the gate's layout [BH][L][m]
    p.gate = GLA_GATE_PREACT;
    p.inv_tau = g.inv_tau;
    return gate_expand(p, z, la, s);
}

size_t gsa_workspace(const GsaProblem& g, bool bwd) {
    Arena a = make_arena(g.B, nullptr, 0);
    a.guard = false;
    carve_gate(g, a);
    if (g.tc) carve_tc(g, a, bwd);
    else carve_simt(g, a, bwd);
    return a.used;
}

gla_status gsa_fwd(const GsaProblem& g, const void* q, const void* k, const void* v, const float* la,
                   const float* hk0, const float* hv0, void* o, float* hkT, float* hvT, void* ws, size_t cap,
                   cudaStream_t s) {
    Arena a = make_arena(g.B, ws, cap);
    a.guard = false;
    float* la_x = carve_gate(g, a);
    if (g.tc) {
        const TcRoute r = carve_tc(g, a, false);
        if (a.used > a.cap) return GLA_ERR_WORKSPACE;
        if (la_x) {
            const gla_status st = expand_gate(g, la, la_x, s);
            if (st != GLA_OK) return st;
            la = la_x;
        }
        return tc_route_fwd(g, q, k, v, la, hk0, hv0, o, hkT, hvT, r, s);
    }
    const SimtRoute r = carve_simt(g, a, false);
    if (a.used > a.cap) return GLA_ERR_WORKSPACE;
    if (la_x) {
        const gla_status st = expand_gate(g, la, la_x, s);
        if (st != GLA_OK) return st;
        la = la_x;
    }
    return simt_route_fwd(g, q, k, v, la, hk0, hv0, o, hkT, hvT, r, s);
}

gla_status gsa_bwd(const GsaProblem& g, const void* q, const void* k, const void* v, const float* la,
                   const float* hk0, const float* hv0, const void* dO, const float* dhkT, const float* dhvT, void* dq,
                   void* dk, void* dv, float* dla, float* dhk0, float* dhv0, bool reuse, void* ws, size_t cap,
                   cudaStream_t s) {
    Arena a = make_arena(g.B, ws, cap);
    a.guard = false;
    float* la_x = carve_gate(g, a);
    const float* z = la;
    gla_status st = GLA_OK;
    if (g.tc) {
        const TcRoute r = carve_tc(g, a, true);
        if (a.used > a.cap) return GLA_ERR_WORKSPACE;
        if (la_x) {
            // a forward's workspace holds the expansion already
            if (!reuse) st = expand_gate(g, z, la_x, s);
            if (st != GLA_OK) return st;
            la = la_x;
        }
        st = tc_route_bwd(g, q, k, v, la, hk0, hv0, dO, dhkT, dhvT, dq, dk, dv, dla, dhk0, dhv0, reuse, r, s);
    } else {
        const SimtRoute r = carve_simt(g, a, true);
        if (a.used > a.cap) return GLA_ERR_WORKSPACE;
        if (la_x) {
            if (!reuse) st = expand_gate(g, z, la_x, s);
            if (st != GLA_OK) return st;
            la = la_x;
        }
        st = simt_route_bwd(g, q, k, v, la, hk0, hv0, dO, dhkT, dhvT, dq, dk, dv, dla, dhk0, dhv0, reuse, r, s);
    }
    if (st != GLA_OK || !g.preact) return st;
    // dL/dz = dL/dlog a * sigmoid(-z) / tau, in place
    Problem p = g.A;
    p.gate = GLA_GATE_PREACT;
    p.inv_tau = g.inv_tau;
    return gate_grad(p, z, dla, dla, s);
}

}  // namespace gla

namespace gla {

bool gsa_step_supported(int64_t m, int64_t Dk, int64_t Dv) {
    return m >= 1 && Dk >= 4 && Dv >= 4 && Dk % 4 == 0 && Dv % 4 == 0 && step_smem(m, Dk, Dv) <= 200 * 1024;
}

gla_status gsa_step(int64_t BH, int64_t m, int64_t Dk, int64_t Dv, bool bf16, const void* q, const void* k,
                    const void* v, const float* la, float inv_tau, float* Km, float* Vm, void* o, cudaStream_t s) {
    if (!gsa_step_supported(m, Dk, Dv) || BH > 2147483647) return GLA_ERR_UNSUPPORTED;
    const size_t smem = step_smem(m, Dk, Dv);
    if (bf16) {
        if (smem > 48 * 1024 && cudaFuncSetAttribute(k_gsa_step<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                     int(smem)) != cudaSuccess)
            return GLA_ERR_CUDA;
        GLA_LAUNCH("gsa_step", k_gsa_step<__nv_bfloat16>, unsigned(BH), kStepThreads, smem, s,
                   static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
                   static_cast<const __nv_bfloat16*>(v), la, inv_tau, Km, Vm, static_cast<__nv_bfloat16*>(o), int(m),
                   int(Dk), int(Dv));
    } else {
        if (smem > 48 * 1024 &&
            cudaFuncSetAttribute(k_gsa_step<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) != cudaSuccess)
            return GLA_ERR_CUDA;
        GLA_LAUNCH("gsa_step", k_gsa_step<float>, unsigned(BH), kStepThreads, smem, s, static_cast<const float*>(q),
                   static_cast<const float*>(k), static_cast<const float*>(v), la, inv_tau, Km, Vm,
                   static_cast<float*>(o), int(m), int(Dk), int(Dv));
    }
    return GLA_OK;
}

}  // namespace gla
