// Checking mode (GLA_FLAG_CHECKS, or every call when built with -DGLA_CHECKS):
// precondition checks on the gates, finiteness checks on the outputs and guard
// blocks after every workspace slice. A failed check sets a bit in the device
// error word (never traps, never stops the pass); gla_check_device_error turns
// the bits into a status after the call.
//
// The gate precondition is the domain of the layer's decay: alpha_t =
// exp(log_a_t) must lie in [0, 1], i.e. log_a finite and <= 0 ("Gated Linear
// Attention Transformers with Hardware-Efficient Training", atlas.scime.ai
// summary, "Approach": the gate is a decay of each key channel).

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "gla_internal.h"

namespace gla {
namespace {

constexpr uint32_t kGuardWord = 0x7FC0DEADu;  // a quiet-NaN bit pattern nothing in the path writes
constexpr int kThreads = 256;

unsigned blocks_for(int64_t n) {
    int64_t b = (n + kThreads * 4 - 1) / (kThreads * 4);
    if (b < 1) b = 1;
    if (b > 148 * 16) b = 148 * 16;  // grid-stride beyond this
    return unsigned(b);
}

// A gate is in its domain when it is finite and <= 0. NaN fails the comparison, +inf and every
// positive value fail it, -inf is caught by the finiteness test.
__device__ __forceinline__ bool gate_ok(float x) { return x <= 0.f && x > -INFINITY; }

__global__ void __launch_bounds__(kThreads) k_check_gates(const float* __restrict__ la, int64_t n, int* err) {
    bool bad = false;
    for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += int64_t(gridDim.x) * blockDim.x)
        bad |= !gate_ok(la[i]);
    if (__syncthreads_or(bad) && threadIdx.x == 0) atomicOr(err, kErrBadGate);
}

template <typename T>
__device__ __forceinline__ float to_f(T x);
template <>
__device__ __forceinline__ float to_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__global__ void __launch_bounds__(kThreads) k_check_finite(const T* __restrict__ p, int64_t n, int* err) {
    bool bad = false;
    for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += int64_t(gridDim.x) * blockDim.x)
        bad |= !isfinite(to_f(p[i]));
    if (__syncthreads_or(bad) && threadIdx.x == 0) atomicOr(err, kErrNonFinite);
}

struct GuardList {
    uint32_t* g[kMaxGuards];
    int n;
};

// one block per guard, one thread per 32-bit word
__global__ void k_guards_fill(GuardList gl) {
    if (int(blockIdx.x) < gl.n && threadIdx.x < kGuardBytes / 4) gl.g[blockIdx.x][threadIdx.x] = kGuardWord;
}

__global__ void k_guards_check(GuardList gl, int* err) {
    if (int(blockIdx.x) < gl.n && threadIdx.x < kGuardBytes / 4 && gl.g[blockIdx.x][threadIdx.x] != kGuardWord)
        atomicOr(err, kErrGuard);
}

GuardList guard_list(const Arena& a) {
    GuardList gl{};
    gl.n = a.nguard < kMaxGuards ? a.nguard : kMaxGuards;
    for (int i = 0; i < gl.n; ++i) gl.g[i] = reinterpret_cast<uint32_t*>(a.guards[i]);
    return gl;
}

}  // namespace

bool checks_on(const Problem& p) {
#ifdef GLA_CHECKS
    (void)p;
    return true;
#else
    return (p.flags & GLA_FLAG_CHECKS) != 0;
#endif
}

Arena make_arena(const Problem& p, void* base, size_t cap) {
    Arena a{static_cast<char*>(base), cap, 0};
    a.guard = checks_on(p);
    return a;
}

gla_status check_gates(const float* log_a, int64_t n, cudaStream_t s) {
    if (n <= 0) return GLA_OK;
    GLA_LAUNCH("check_gates", k_check_gates, blocks_for(n), kThreads, 0, s, log_a, n, device_error_word());
    return GLA_OK;
}

gla_status check_finite(const void* p, int64_t n, bool bf16, cudaStream_t s) {
    if (!p || n <= 0) return GLA_OK;
    if (bf16)
        GLA_LAUNCH("check_finite", k_check_finite<__nv_bfloat16>, blocks_for(n), kThreads, 0, s,
                   static_cast<const __nv_bfloat16*>(p), n, device_error_word());
    else
        GLA_LAUNCH("check_finite", k_check_finite<float>, blocks_for(n), kThreads, 0, s, static_cast<const float*>(p),
                   n, device_error_word());
    return GLA_OK;
}

gla_status guards_fill(const Arena& a, cudaStream_t s) {
    const GuardList gl = guard_list(a);
    if (gl.n == 0) return GLA_OK;
    GLA_LAUNCH("guards_fill", k_guards_fill, unsigned(gl.n), unsigned(kGuardBytes / 4), 0, s, gl);
    return GLA_OK;
}

gla_status guards_check(const Arena& a, cudaStream_t s) {
    const GuardList gl = guard_list(a);
    if (gl.n == 0) return GLA_OK;
    GLA_LAUNCH("guards_check", k_guards_check, unsigned(gl.n), unsigned(kGuardBytes / 4), 0, s, gl,
               device_error_word());
    return GLA_OK;
}

}  // namespace gla
