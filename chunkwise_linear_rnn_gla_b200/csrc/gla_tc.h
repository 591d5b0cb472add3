// Internal declarations of the tensor-core (tcgen05 / TMEM / TMA) path.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "gla_internal.h"
#include "tc_prims.cuh"

namespace gla {

__device__ __forceinline__ uint32_t tc_smem_u32(const void* p) { return tc::smem_u32(p); }

constexpr int kTcChunk = 128;  // C on the tensor-core path
constexpr int kTcSub = 128;    // secondary chunk c: the default, one GEMM per chunk (16: two-level)
constexpr int kTcBV = 64;      // value columns per walk CTA

// Workspace slices of a tensor-core pass (gla_tc_api.cu). The backward's layout extends the
// forward's, so a forward workspace can be handed to the backward unchanged.
struct TcBuffers {
    __nv_bfloat16 *Qt, *Kt, *P;  // Q~, K~ [BH][L][K]; masked intra-chunk scores [BH][N][128][128]
    float *gam, *hT;             // e^Gamma [BH][N][K]; a copy of the final state
    __nv_bfloat16* states;       // state entering each chunk [BH][N][K][V] (materialised mode, backward)
    float* segbuf;               // segmented state walks: end states and entering states per segment
    __nv_bfloat16* Dbuf;         // backward: D_i [BH][N][K][V]
    float* gpart;                // scalar gate kinds: per-CTA partial sums of the gate gradient
};
TcBuffers tc_carve(const Problem& p, Arena& a, bool bwd);

// Gated slot attention, tensor-core path (gla_gsa_read.cu). For the GLA pass problem p (key width
// m = p.K = 128 slots, value width D = p.V) and chunk states M_[i] [BH][N][m][D] (the slot memory
// entering chunk i), the read of the memory from its value side, in fp32:
//   r_j = e^{B_j} * ( M_[i] x_j^T + sum_{s<=j} (x_j . y_s) w_s e^{-B_s} ),  w = bf16(1 - e^{log a}),
// with B the per-chunk cumsum of log a over the slots (exact log-space terms for a slot whose chunk
// decay passes the range bound). mode 0 (x = q, y = k): s = softmax(r) into s_b (bf16) and s_f
// (fp32). mode 1 (x = dO, y = v): G = s * (r - <s, r>) into s_b (bf16), s read from s_in (fp32).
// Either result x (as stored in bf16) is the query of a GLA layer with key w under the same gate; its
// chunk-local operands come out too, as tc_prep_launch would write them: Qt = x e^{B} [BH][L][m] and
// the masked scores P [BH][N][128][128].
gla_status tc_gsa_slot_read_launch(const Problem& p, const void* x, const void* y, const __nv_bfloat16* M,
                                   const float* la, const float* s_in, __nv_bfloat16* s_b, float* s_f,
                                   __nv_bfloat16* Qt, __nv_bfloat16* P, int mode, cudaStream_t s);
bool tc_gsa_slot_read_supported(const Problem& p);
// The slot gate's preparation for the memories' walks (p: key width m = 128): w = bf16(1 - e^{log a})
// [BH][L][m], the walk operand K~ = w e^{Gamma - B} [BH][L][m] and e^Gamma [BH][N][m], the last two also
// into Kt2 / gam2 when given (the second GLA layer's buffers: the same key and gate).
gla_status tc_gsa_gate_prep_launch(const Problem& p, const float* la, __nv_bfloat16* w, __nv_bfloat16* Kt,
                                   float* gam, __nv_bfloat16* Kt2, float* gam2, cudaStream_t s);

// Chunk-parallel gate preparation (gla_tc_prep.cu): Q~, K~, e^Gamma and the
// masked intra-chunk scores P.
// `la` is the gate argument of kind `gate_kind` (gla_gate.cuh): the kernel reads every kind natively.
gla_status tc_prep_launch(const Problem& p, const void* q, const void* k, const float* la, __nv_bfloat16* Qt,
                          __nv_bfloat16* Kt, __nv_bfloat16* P, float* gam, int gate_kind, cudaStream_t s);

// Two-level intra-chunk scores (gla_tc_twolevel.cu), sub-chunk length 16: overwrites P.
gla_status tc_intra_twolevel_launch(const Problem& p, const void* q, const void* k, const float* la,
                                    __nv_bfloat16* P, cudaStream_t s);

// Row-gated chunk walk (gla_tc_walk.cu). State X [K x 64-column tile] with the
// gate on its rows. Per chunk i (in walk order):
//   Y_i = A2_i X + Pm_i B1_i          (fused / output-only modes)
//   X  <- diag(gam_i) X + A1_i^T B1_i  (fused / states-only modes)
// Forward: A1 = K~, B1 = v, A2 = Q~, Pm = P, forward order, Y = o, X0 = h0.
// dv:      A1 = Q~, B1 = dO, A2 = K~, Pm = P^T, reverse order, Y = dv, X0 = dhT.
enum WalkMode : int { kWalkFused = 0, kWalkStatesOnly = 1, kWalkOutputOnly = 2 };

// A long walk over few heads is split into segments of `len` chunks (walk
// order) that run in parallel: pass 1 walks every segment from a zero state
// (segment 0 from the true initial state) and keeps the end states; a scan
// over the segments turns them into the true state entering each segment
// (S_in[g+1] = diag(prod of e^{Gamma} over segment g) S_in[g] + E[g], fp32);
// pass 2 walks the segments again from those states. A plain walk is one
// segment.
struct WalkSegs {
    int first;              // first segment of this launch
    int len;                // chunks (walk steps) per segment
    int store_all;          // 1: every segment stores its states, 0: segment 0 only, -1: none
    int64_t stride;         // elements between the per-segment [BH][K][V] fp32 blocks of init_seg / fin
    const float* init_seg;  // start states of segments >= 1, indexed by segment (null: zero)
};

struct WalkArgs {
    const __nv_bfloat16* A1;  // [BH][L][K]
    const __nv_bfloat16* B1;  // [BH][L][V]
    const __nv_bfloat16* A2;  // [BH][L][K]
    const __nv_bfloat16* Pm;  // [BH][N][128][128]
    const float* gam;         // [BH][N][K]
    const float* init;        // [BH][K][V] or null
    float* fin;               // [BH][K][V] or null
    float* fin2;              // second copy of the final state, or null
    __nv_bfloat16* Y;         // [BH][L][V]
    __nv_bfloat16* states;    // [BH][N][K][V] bf16 state entering each chunk (written by
                              // states-only mode and, when non-null, by fused mode; read by
                              // output-only mode)
    int mode;
    bool reverse;
    bool p_transposed;
    // fused mode: segments (seg_count > 1: every segment in one launch, segment g > 0 starting from
    // seg_init + g * seg_stride; fin and fin2 are then left to the segment scan)
    int seg_count = 1;
    int seg_len = 0;
    const float* seg_init = nullptr;
    int64_t seg_stride = 0;
};

gla_status tc_walk_launch(const Problem& p, const WalkArgs& a, cudaStream_t s, const char* name);

// Materialised state walk on [128 x 128] tiles with the state accumulated in
// TMEM (gla_tc_states.cu); requires d_v % 128 == 0.
// A walk over few heads and many chunks is split into segments that run in
// parallel (two passes and a scan over the segment end states); `segbuf`
// holds tc_walk_seg_floats(p) floats of workspace (null: never split).
bool tc_states_walk_supported(const Problem& p);
size_t tc_walk_seg_floats(const Problem& p);
// Pass 1 and the scan of a segmented walk for the fused (non-materialised) walks: returns the
// number of segments G (1: not split, nothing launched), their length and the entering states;
// fin / fin2 receive the final state.
int tc_walk_seg_prepare(const Problem& p, const __nv_bfloat16* A, const __nv_bfloat16* B, const float* gam,
                        const float* init, float* fin, float* fin2, float* segbuf, bool reverse, cudaStream_t s,
                        int* len, const float** S_in, int64_t* stride, gla_status* st);
gla_status tc_states_walk_launch(const Problem& p, const __nv_bfloat16* A, const __nv_bfloat16* B, const float* gam,
                                 const float* init, float* fin, float* fin2, __nv_bfloat16* states, float* segbuf,
                                 bool reverse, cudaStream_t s, const char* name);

// The final state of the walk only (nothing stored; few heads: parallel segments and a scan).
gla_status tc_states_walk_final(const Problem& p, const __nv_bfloat16* A, const __nv_bfloat16* B, const float* gam,
                                const float* init, float* fin, float* segbuf, bool reverse, cudaStream_t s,
                                const char* name);

// Chunk-parallel Y_i = A_i X_i + Pm_i B_i from stored bf16 chunk states X
// (gla_tc_out.cu): forward o (A = Q~, Pm = P) and dv (A = K~, Pm = P^T).
// late_wait: the kernel follows, by programmatic dependent launch, a kernel that it does not
// depend on and that triggers its dependents only after its own wait; it then reads its inputs
// at once and waits for that kernel only before it exits.
gla_status tc_chunk_out_launch(const Problem& p, const __nv_bfloat16* A, const __nv_bfloat16* X,
                               const __nv_bfloat16* Pm, const __nv_bfloat16* Bv, bool p_transposed,
                               __nv_bfloat16* Y, bool late_wait, cudaStream_t s, const char* name);

// Backward, chunk-parallel part (gla_tc_bwd.cu): dq, dk and dlog a from dO, v,
// the stored states S_[i] and D_i, Q~ and e^Gamma.
// `la` is the gate argument of kind p.gate. Per-channel kinds write dla (dL/dlog alpha, or dL/dz for
// preact) directly; the scalar kinds write per-CTA partial sums over their 128 channels to
// gpart[(bh * N + i) * (K / 128) + kh][token] (zero past the end of the sequence), which
// tc_gate_grad_partials reduces into the caller's gradient.
gla_status tc_bwd_chunk_launch(const Problem& p, const void* q, const void* k, const float* la, const void* dO,
                               const void* v, const __nv_bfloat16* Qt, const float* gam, const __nv_bfloat16* Sbuf,
                               const __nv_bfloat16* Dbuf, void* dq, void* dk, float* dla, float* gpart,
                               cudaStream_t s);
gla_status tc_gate_grad_partials(const Problem& p, const float* gpart, float* dla, cudaStream_t s);

}  // namespace gla
