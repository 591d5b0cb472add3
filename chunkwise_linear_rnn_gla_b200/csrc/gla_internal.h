// Internal host-side interface between the C ABI (gla_api.cu) and the kernel
// files. Not installed; not part of the ABI.
#pragma once

#include <cuda_runtime.h>
#include <cstddef>
#include <cstdint>

#include "../../include/gla.h"

namespace gla {

// Resolved problem: the descriptor after defaults and checks.
struct Problem {
    int64_t B, H, L, K, V;
    int64_t BH;      // B*H
    int C;           // chunk length
    int c;           // sub-chunk length
    int64_t N;       // number of chunks, ceil(L / C)
    bool bf16;       // element type of q, k, v, o, dO, dq, dk, dv
    int impl;        // GLA_IMPL_SIMT or GLA_IMPL_TC (never AUTO)
    int state_mode;  // never AUTO
    int flags;
    int gate = 0;         // gla_gate: what the caller's log_a holds
    float inv_tau = 0.f;  // GLA_GATE_PREACT: 1 / gate_tau
};

// Bump allocator over the caller's workspace; every slice is 256-B aligned.
// With guards on (GLA_FLAG_CHECKS), every slice is followed by a 256-byte guard
// block that the checking build fills with a pattern before the kernels run
// and verifies after them, so a kernel writing past the end of its slice is
// reported (gla_check_device_error -> GLA_ERR_WORKSPACE).
constexpr int kMaxGuards = 32;
constexpr size_t kGuardBytes = 256;
struct Arena {
    char* base;
    size_t cap;
    size_t used;
    bool guard = false;
    int nguard = 0;
    char* guards[kMaxGuards] = {};
    template <typename T>
    T* take(size_t count) {
        size_t off = (used + 255) & ~size_t(255);
        size_t bytes = count * sizeof(T);
        used = off + bytes;
        if (guard && nguard < kMaxGuards) {
            const size_t g = (used + 255) & ~size_t(255);
            if (base) guards[nguard] = base + g;
            ++nguard;
            used = g + kGuardBytes;
        }
        return base ? reinterpret_cast<T*>(base + off) : nullptr;
    }
};

// Arena over a workspace (base may be null for size queries); guards follow the problem's flags.
Arena make_arena(const Problem& p, void* base, size_t cap);

// ---- launch bookkeeping (gla_api.cu) ------------------------------------
// Every kernel launch goes through launch_begin/launch_end so that the
// launch counter and the optional per-kernel event timing see it.
void launch_begin(const char* name, cudaStream_t s);
gla_status launch_end(const char* name, cudaStream_t s);

// Device-side error word (set by kernels whose bounded waits run out, and by
// the checking build's checks). Bits: tc::kErrWaitTimeout, kErrBadGate,
// kErrNonFinite, kErrGuard.
int* device_error_word();
enum : int { kErrBadGate = 2, kErrNonFinite = 4, kErrGuard = 8 };

// ---- checking build (gla_checks.cu) ------------------------------------------
// Before a pass: every gate must be finite and <= 0 (kErrBadGate); the workspace
// guards are filled. After it: every output element must be finite
// (kErrNonFinite) and every guard intact (kErrGuard).
gla_status check_gates(const float* log_a, int64_t n, cudaStream_t s);
gla_status check_finite(const void* p, int64_t n, bool bf16, cudaStream_t s);
gla_status guards_fill(const Arena& a, cudaStream_t s);
gla_status guards_check(const Arena& a, cudaStream_t s);
bool checks_on(const Problem& p);

// ---- gate kinds (gla_gates.cu) ------------------------------------------------
// Per-channel log alpha [B,H,L,K] from the caller's gate argument, and the caller's gate gradient
// from the per-channel one (scalar / head: sums; preact: dpc and dla are the same buffer, scaled in
// place by sigmoid(-z)/tau).
gla_status gate_expand(const Problem& p, const float* g, float* out, cudaStream_t s);
gla_status gate_grad(const Problem& p, const float* g, const float* dpc, float* dla, cudaStream_t s);

// ---- sequence-sharded evaluation (gla_seq.cu) ---------------------------------
gla_status segment_decay(const Problem& p, const float* log_a, float* a, cudaStream_t s);
gla_status state_combine(int64_t G, int64_t BH, int64_t K, int64_t V, const float* a, const float* U,
                         const float* init, int r, int reverse, float* out, cudaStream_t s);

// ---- SIMT path (gla_simt.cu) ---------------------------------------------
size_t simt_fwd_workspace(const Problem& p);
size_t simt_bwd_workspace(const Problem& p);
void simt_layout(const Problem& p, Arena& a, bool bwd);  // carve `a` as the pass would (guard positions)
gla_status simt_chunk_cumsum(const Problem& p, const float* log_a, float* Bc, cudaStream_t s);
gla_status simt_fwd(const Problem& p, const void* q, const void* k, const void* v, const float* log_a,
                    const float* h0, void* o, float* hT, Arena& ws, cudaStream_t s);
gla_status simt_bwd(const Problem& p, const void* q, const void* k, const void* v, const float* log_a,
                    const float* h0, const void* dO, const float* dhT, void* dq, void* dk, void* dv,
                    float* dlog_a, float* dh0, Arena& ws, cudaStream_t s);

// ---- decode step (gla_step.cu) ---------------------------------------------
gla_status step_launch(const Problem& p, const void* q, const void* k, const void* v, const float* log_a,
                       float* S, void* o, cudaStream_t s);

// ---- tensor-core path (gla_tc_*.cu) -----------------------------------------
bool tc_supported(const Problem& p);
size_t tc_fwd_workspace(const Problem& p);
size_t tc_bwd_workspace(const Problem& p);
void tc_layout(const Problem& p, Arena& a, bool bwd);
gla_status tc_fwd(const Problem& p, const void* q, const void* k, const void* v, const float* log_a,
                  const float* h0, void* o, float* hT, Arena& ws, cudaStream_t s);
// Only the end state of a forward (prep and a walk that stores nothing), and only the gradient at the
// entering state of a backward (prep and the reverse walk): the summaries of sequence-sharded evaluation.
gla_status tc_fwd_final_state(const Problem& p, const void* q, const void* k, const void* v, const float* la,
                              const float* h0, float* hT, Arena& ws, cudaStream_t s);
gla_status tc_bwd_initial_grad(const Problem& p, const void* q, const void* k, const float* la, const void* dO,
                               const float* dhT, float* dh0, Arena& ws, cudaStream_t s);
gla_status tc_bwd(const Problem& p, const void* q, const void* k, const void* v, const float* log_a,
                  const float* h0, const void* dO, const float* dhT, void* dq, void* dk, void* dv,
                  float* dlog_a, float* dh0, Arena& ws, cudaStream_t s);

// ---- gated slot attention (gla_gsa.cu) -------------------------------------------
// The two GLA passes of the method, resolved like any GLA call: A = layer one (GLA key width m, value
// width Dk: the key memory), B = layer two (key width m, value width Dv: the value memory).
// tc: the tensor-core route (bf16, m = 128, both passes on the tensor-core path, materialised states);
// otherwise both passes run on the CUDA-core path in fp32 and io_bf16 says whether the caller's q, k, v,
// o, dO and gradients are bf16 (converted at the boundary).
// preact: the caller's gate argument is z, log a = logsigmoid(z) * inv_tau (expanded into the workspace
// first; the gate gradient is scaled by sigmoid(-z) * inv_tau at the end).
struct GsaProblem {
    Problem A, B;
    int64_t m;
    bool tc;
    bool io_bf16;
    bool preact = false;
    float inv_tau = 0.f;
};
bool gsa_tc_route(const Problem& A, const Problem& B, int64_t m);
// Decode step: both memories Km [BH][m][Dk], Vm [BH][m][Dv] (fp32) updated in place, o [BH][Dv].
bool gsa_step_supported(int64_t m, int64_t Dk, int64_t Dv);
// inv_tau > 0: la holds the pre-activation z, log a = logsigmoid(z) * inv_tau.
gla_status gsa_step(int64_t BH, int64_t m, int64_t Dk, int64_t Dv, bool bf16, const void* q, const void* k,
                    const void* v, const float* la, float inv_tau, float* Km, float* Vm, void* o, cudaStream_t s);
size_t gsa_workspace(const GsaProblem& g, bool bwd);
gla_status gsa_fwd(const GsaProblem& g, const void* q, const void* k, const void* v, const float* la,
                   const float* hk0, const float* hv0, void* o, float* hkT, float* hvT, void* ws, size_t cap,
                   cudaStream_t s);
gla_status gsa_bwd(const GsaProblem& g, const void* q, const void* k, const void* v, const float* la,
                   const float* hk0, const float* hv0, const void* dO, const float* dhkT, const float* dhvT, void* dq,
                   void* dk, void* dv, float* dla, float* dhk0, float* dhv0, bool reuse, void* ws, size_t cap,
                   cudaStream_t s);

}  // namespace gla

// Launch helper: bracket a <<<>>> launch with the bookkeeping hooks and return
// GLA_ERR_CUDA from the enclosing function if the launch failed.
#define GLA_LAUNCH(name, kernel, grid, block, smem, stream, ...)                   \
    do {                                                                           \
        ::gla::launch_begin(name, stream);                                         \
        kernel<<<(grid), (block), (smem), (stream)>>>(__VA_ARGS__);                \
        gla_status _st = ::gla::launch_end(name, stream);                          \
        if (_st != GLA_OK) return _st;                                             \
    } while (0)

// Launch with programmatic dependent launch: the kernel's CTAs may start (and run
// their prologue: barrier init, TMEM allocation, tensor-map prefetch) while the
// previous kernel on the stream drains. Every kernel launched this way executes
// tc::pdl_wait() before it touches global memory that earlier work writes or reads.
#define GLA_LAUNCH_PDL(name, kernel, grid, block, smem, strm_, ...)                              \
    do {                                                                                          \
        ::gla::launch_begin(name, strm_);                                                        \
        cudaLaunchConfig_t _cfg = {};                                                             \
        _cfg.gridDim = dim3(grid);                                                                \
        _cfg.blockDim = dim3(block);                                                              \
        _cfg.dynamicSmemBytes = (smem);                                                           \
        _cfg.stream = (strm_);                                                                   \
        cudaLaunchAttribute _attr[1];                                                             \
        _attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;                         \
        _attr[0].val.programmaticStreamSerializationAllowed = 1;                                  \
        _cfg.attrs = _attr;                                                                       \
        _cfg.numAttrs = 1;                                                                        \
        (void)cudaLaunchKernelEx(&_cfg, kernel, __VA_ARGS__);                                     \
        gla_status _st = ::gla::launch_end(name, strm_);                                         \
        if (_st != GLA_OK) return _st;                                                            \
    } while (0)
