/*
 * gla.h -- C ABI of libgla: chunkwise gated linear attention (GLA) on NVIDIA
 * B200 (sm_100a).
 *
 * The layer ("Gated Linear Attention Transformers with Hardware-Efficient
 * Training", atlas.scime.ai summary, section "Approach"): per batch b and
 * head h, with a data-dependent gate G_t = alpha_t^T 1 (rank one, constant
 * along the value dimension), i.e. a per-key-channel decay,
 *
 *     S_t = diag(alpha_t) S_{t-1} + k_t^T v_t,      o_t = q_t S_t,
 *
 * alpha_t = exp(log_a_t) in [0,1]^{Dk}, S_{-1} = h0, hT = S_{L-1}. The output
 * reads the state after the update. There is no 1/sqrt(Dk) scale and no
 * normaliser inside the layer. log_a must be finite and <= 0: a gate of
 * exactly zero is passed as a large negative value (e.g. -1e30), not -inf.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Layout: all tensors are dense, row-major, contiguous, on the device:
 *     q, k, log_a, dq, dk, dlog_a : [B, H, L, Dk]
 *     v, o, dO, dv                : [B, H, L, Dv]
 *     h0, hT, dhT, dh0, S         : [B, H, Dk, Dv]   (always fp32)
 * q, k, v, o, dO, dq, dk, dv have the element type `desc->dtype` (fp32 or
 * bf16); log_a, dlog_a and all states are fp32. Every arithmetic step
 * accumulates in fp32.
 * Ownership: the caller allocates and frees every buffer, including the
 * workspace. The library never allocates device memory, never frees, and
 * never synchronises (except gla_check_device_error).
 * Execution: work is enqueued on `stream` (a cudaStream_t; NULL = the legacy
 * default stream) on the current device; calls return before the GPU is
 * done. Outputs must not alias inputs (except S in gla_step, updated in
 * place).
 * Errors: argument checks run on the host before any launch and return a
 * status; nothing is thrown across the ABI. A failed launch returns
 * GLA_ERR_CUDA. Device-side conditions (a bounded wait that ran out) are
 * recorded in a device flag that gla_check_device_error reports.
 * Alignment: device pointers must be 16-byte aligned; the workspace 256-byte
 * aligned.
 */
#ifndef GLA_H_
#define GLA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define GLA_ABI_VERSION 2

typedef enum gla_status {
    GLA_OK = 0,
    GLA_ERR_INVALID_ARG = 1, /* null/misaligned pointer, bad size, bad enum   */
    GLA_ERR_UNSUPPORTED = 2, /* valid request this build has no kernel for    */
    GLA_ERR_WORKSPACE = 3,   /* workspace missing, too small or misaligned    */
    GLA_ERR_CUDA = 4,        /* a CUDA runtime call or kernel launch failed   */
    GLA_ERR_TIMEOUT = 5      /* a device-side bounded wait ran out            */
} gla_status;

typedef enum gla_dtype {
    GLA_DTYPE_F32 = 0,
    GLA_DTYPE_BF16 = 1
} gla_dtype;

/* How the inter-chunk states are handled (the "Approach" section offers both:
 * the per-chunk states may be stored in memory or kept on chip). */
typedef enum gla_state_mode {
    GLA_STATE_AUTO = 0,            /* library picks: materialised              */
    GLA_STATE_MATERIALIZED = 1,    /* write S_[i] of every chunk to workspace  */
    GLA_STATE_NONMATERIALIZED = 2  /* keep S on chip while walking the chunks  */
} gla_state_mode;

/* Which kernel family runs. */
typedef enum gla_impl {
    GLA_IMPL_AUTO = 0,  /* tensor-core path for bf16, CUDA-core path for fp32 */
    GLA_IMPL_SIMT = 1,  /* fp32 CUDA-core kernels for every dtype              */
    GLA_IMPL_TC = 2     /* bf16 tensor-core kernels (tcgen05/TMEM/TMA)         */
} gla_impl;

/* What the `log_a` argument of every entry point holds, and what the
 * backward returns in `dlog_a`. The pages compare the per-channel gate with
 * two coarser decays ("Measured effects" ablations of "Gated Linear Attention
 * Transformers with Hardware-Efficient Training", atlas.scime.ai summary): a
 * decay that depends on the data but is one scalar per head and step, and a
 * fixed decay per head that does not depend on the data. The "Approach"
 * section makes the gate a function of the input; GLA_GATE_PREACT takes that
 * function's argument and applies it inside the kernels.
 *   kind                log_a (fwd/bwd)   log_a (step)   dlog_a (bwd)
 *   GLA_GATE_CHANNEL    [B,H,L,Dk]        [B,H,Dk]       [B,H,L,Dk] dL/dlog_a
 *   GLA_GATE_SCALAR     [B,H,L]           [B,H]          [B,H,L]    dL/dlog_a (summed over channels)
 *   GLA_GATE_HEAD       [H]               [H]            [H]        dL/dlog_a (summed over b, t, channels)
 *   GLA_GATE_PREACT     z [B,H,L,Dk]      z [B,H,Dk]     [B,H,L,Dk] dL/dz
 * CHANNEL, SCALAR and HEAD take log alpha itself (finite, <= 0). PREACT takes
 * any finite z and uses log alpha = logsigmoid(z) / gate_tau (gate_tau > 0),
 * so dL/dz = dL/dlog_alpha * sigmoid(-z) / gate_tau. */
typedef enum gla_gate {
    GLA_GATE_CHANNEL = 0,
    GLA_GATE_SCALAR = 1,
    GLA_GATE_HEAD = 2,
    GLA_GATE_PREACT = 3
} gla_gate;

/* Problem descriptor. B, H, L >= 1; Dk, Dv >= 1 (each path states its own
 * supported set and returns GLA_ERR_UNSUPPORTED outside it). chunk = 0 and
 * subchunk = 0 pick defaults; otherwise chunk must be one of 16, 32, 64, 128
 * and subchunk must divide chunk. The result does not depend on chunk or
 * subchunk beyond rounding. gate = GLA_GATE_CHANNEL and gate_tau = 0 are the
 * per-channel gate of earlier versions of this ABI; gate_tau is read only for
 * GLA_GATE_PREACT. */
typedef struct gla_desc {
    int64_t B, H, L, Dk, Dv;
    int32_t dtype;      /* gla_dtype                                   */
    int32_t chunk;      /* C, the chunk length (0 = default)           */
    int32_t subchunk;   /* c, the secondary chunk length (0 = default) */
    int32_t state_mode; /* gla_state_mode                              */
    int32_t impl;       /* gla_impl                                    */
    int32_t flags;      /* GLA_FLAG_* bits                             */
    int32_t gate;       /* gla_gate: what log_a holds                  */
    float gate_tau;     /* GLA_GATE_PREACT: log alpha = logsigmoid(z) / gate_tau */
} gla_desc;

/* gla_bwd: the workspace still holds what gla_fwd left in it for the same
 * inputs and descriptor, so the backward may reuse those intermediates
 * instead of recomputing them. The caller guarantees that nothing wrote the
 * workspace or the inputs in between. */
#define GLA_FLAG_WS_FROM_FWD 0x1

/* Checking mode (the same as building the library with -DGLA_CHECKS, which
 * turns it on for every call). Each call then also enqueues:
 *  - before the pass, a check that every log_a element is finite and <= 0;
 *  - before the pass, a fill of guard blocks (256 bytes) placed after every
 *    workspace slice, and after the pass a check that they are intact;
 *  - after the pass, a check that every output element is finite.
 * A failed check does not stop the call or trap: it sets the device error
 * flag, and the next gla_check_device_error reports GLA_ERR_INVALID_ARG (a
 * gate outside its domain, or a non-finite output, e.g. from a NaN input) or
 * GLA_ERR_WORKSPACE (a guard block was overwritten: a kernel wrote outside
 * its slice). The workspace sizes include the guard blocks when the flag is
 * set, so a forward and the backward that reuses its workspace must agree on
 * it. Off by default: the checks read every gate and output once more. */
#define GLA_FLAG_CHECKS 0x2

/* Workspace bytes gla_fwd / gla_bwd need for `d` (0 when `d` is invalid).
 * A buffer of gla_bwd_workspace_size bytes also serves gla_fwd, so one
 * workspace can be shared by a forward and the following backward. */
size_t gla_fwd_workspace_size(const gla_desc* d);
size_t gla_bwd_workspace_size(const gla_desc* d);

/* Forward: o[B,H,L,Dv] and, if hT != NULL, hT[B,H,Dk,Dv] = S_{L-1}.
 * h0 may be NULL (zero initial state).
 * Method: per-chunk log-space gate cumsum, inter-chunk state walk and
 * intra-chunk secondary chunking, the chunkwise form of the recurrence
 * ("Approach": I/O-aware chunkwise algorithm, two-level chunking). */
gla_status gla_fwd(const gla_desc* d, const void* q, const void* k, const void* v,
                   const float* log_a, const float* h0, void* o, float* hT,
                   void* workspace, size_t workspace_bytes, void* stream);

/* Backward of L = <dO, o> + <dhT, hT>: dq, dk [B,H,L,Dk], dv [B,H,L,Dv]
 * (dtype), dlog_a [B,H,L,Dk] (fp32), dh0 [B,H,Dk,Dv] (fp32, may be NULL).
 * h0 and dhT may be NULL (zero). The gate gradient is the closed form
 *   dlog_a_t = sum_{s>=t} (q_s*dq_s - k_s*dk_s) + sum_v dhT[:,v]*hT[:,v]
 * (the "Approach" section's closed-form gate gradient, which needs no
 * per-step state). dq, dk, dv are the full gradients. */
gla_status gla_bwd(const gla_desc* d, const void* q, const void* k, const void* v,
                   const float* log_a, const float* h0, const void* dO, const float* dhT,
                   void* dq, void* dk, void* dv, float* dlog_a, float* dh0,
                   void* workspace, size_t workspace_bytes, void* stream);

/* One recurrent decode step for B*H independent states (d->L is ignored):
 * S <- diag(exp(log_a)) S + k^T v (in place), then o = q S.
 * q, k, log_a: [B,H,Dk]; v, o: [B,H,Dv]; S: [B,H,Dk,Dv] fp32. The recurrent
 * form of the layer (podcast.app episode page, summary: the layer read as a
 * gated memory updated once per token). */
gla_status gla_step(const gla_desc* d, const void* q, const void* k, const void* v,
                    const float* log_a, float* S, void* o, void* stream);

/* Per-chunk inclusive log-space gate cumsum: for chunk i and row j,
 * Bcum[t = iC + j] = sum_{r=0..j} max(log_a[iC + r], -200) per key channel,
 * restarting at every chunk boundary (C = the descriptor's chunk). In/out
 * [B,H,L,Dk] fp32. The floor changes no decay factor (e^-200 is 0 in fp32)
 * but keeps a zero gate given as a huge negative number from swallowing the
 * gates after it in the fp32 sum; every chunkwise pass applies it. This is
 * the first stage of every chunkwise pass; it is exported so that it can be
 * checked and timed on its own. */
gla_status gla_chunk_cumsum(const gla_desc* d, const float* log_a, float* Bcum, void* stream);

/* ---- sequence-sharded evaluation --------------------------------------------
 * The state recurrence is affine in the entering state, so a segment of steps
 * maps an entering state X to diag(a) X + U, with a = exp(sum of log alpha over
 * the segment) per key channel and U the segment's end state from a zero start
 * (gla_fwd with h0 = NULL). Segments of one sequence held by different devices
 * exchange (a, U) and combine them; the backward exchanges (a, W) with W the dh0
 * of the segment's gla_bwd with dhT = NULL. The pages carry the recurrent state
 * across training segments ("Gated Linear Attention Transformers with
 * Hardware-Efficient Training", atlas.scime.ai summary, "Measured effects":
 * truncated BPTT); here the segments are shards of one sequence. */

/* The summaries alone, cheaper than the full passes (tensor-core path with
 * materialised states; GLA_ERR_UNSUPPORTED otherwise, and the full pass then
 * gives the same result):
 *  - gla_fwd_final_state: hT of gla_fwd (h0 may be NULL) without computing o
 *    (the preparation and a state walk that stores nothing);
 *  - gla_bwd_initial_grad: dh0 of gla_bwd (dhT may be NULL) without the other
 *    gradients (the preparation and the reverse walk).
 * Workspace: as gla_fwd / gla_bwd for the same descriptor. */
gla_status gla_fwd_final_state(const gla_desc* d, const void* q, const void* k, const void* v,
                               const float* log_a, const float* h0, float* hT,
                               void* workspace, size_t workspace_bytes, void* stream);
gla_status gla_bwd_initial_grad(const gla_desc* d, const void* q, const void* k, const float* log_a,
                                const void* dO, const float* dhT, float* dh0,
                                void* workspace, size_t workspace_bytes, void* stream);

/* a[B,H,Dk] = exp(sum over the descriptor's L steps of log alpha) for the
 * gate argument log_a of kind d->gate (fp32, device). */
gla_status gla_segment_decay(const gla_desc* d, const float* log_a, float* a, void* stream);

/* Combine the summaries of G segments (one after another in a [G][BH][Dk] and
 * U [G][BH][Dk][Dv], fp32, device):
 *   reverse = 0: out = X_r with X_0 = init (NULL: zero), X_{g+1} = diag(a_g) X_g + U_g
 *                (the state entering segment r);
 *   reverse = 1: out = Y_r with Y_{G-1} = init (NULL: zero), Y_{g-1} = diag(a_g) Y_g + U_g
 *                (the gradient arriving at the end of segment r, with U_g = W_g).
 * init and out are [BH][Dk][Dv]; Dv must be a multiple of 4; 0 <= r < G. */
gla_status gla_state_combine(int64_t G, int64_t BH, int64_t Dk, int64_t Dv, const float* a, const float* U,
                             const float* init, int32_t r, int32_t reverse, float* out, void* stream);

/* ---- gated slot attention ---------------------------------------------------
 * The method of the mlsanity card for "Gated Slot Attention for Efficient
 * Linear-Time Sequence Modeling" (abstract): a bounded memory of `slots` (m)
 * slots that a GLA-style data-dependent gate forgets, read by two GLA layers
 * joined by a softmax over the slots. The card prints no equations; the
 * reading built here gives each slot the write weight w_t = 1 - a_t (a slot
 * writes in proportion to what it forgets). Per batch b and head h, with
 * a_t = exp(log_a_t) in (0,1]^m:
 *
 *     Kmem_t = diag(a_t) Kmem_{t-1} + w_t^T k_t        [m x Dk]
 *     Vmem_t = diag(a_t) Vmem_{t-1} + w_t^T v_t        [m x Dv]
 *     s_t    = softmax over the m slots of Kmem_t q_t^T
 *     o_t    = s_t Vmem_t
 *
 * Kmem_{-1} = hk0 and Vmem_{-1} = hv0 (NULL: zero); hkT, hvT are the final
 * memories. Both memories are GLA states over the slot dimension, and the
 * library evaluates the method as GLA passes of its own kernels (layer one's
 * read as the query gradient of a GLA with key w and value k; layer two as a
 * GLA with query s, key w and value v) plus elementwise kernels for w, the
 * softmax, its backward and the gate gradient.
 *
 * Descriptor: B, H, L, Dk (width of q and k), Dv (width of v and o), dtype,
 * chunk, subchunk, impl and state_mode apply to the GLA passes (GLA key width
 * m); `gate` is GLA_GATE_CHANNEL (log_a is the per-slot log gate) or
 * GLA_GATE_PREACT (log_a holds the gate's argument z and log a = logsigmoid(z) / gate_tau; the
 * backward then returns dL/dz in dlog_a), other kinds GLA_ERR_UNSUPPORTED; flags:
 * GLA_FLAG_WS_FROM_FWD (backward only:
 * `workspace` holds the matching gla_gsa_fwd's workspace, same inputs and
 * options) and GLA_FLAG_CHECKS (gate domain and finite outputs, reported by
 * gla_check_device_error). bf16 with m = 128 and Dk, Dv multiples of 64 takes
 * the tensor-core route; every other case the CUDA-core route (gla_gsa_resolve).
 * Layouts (row-major, contiguous, device):
 *     q, k, dq, dk            : [B, H, L, Dk]   (dtype)
 *     v, o, dO, dv            : [B, H, L, Dv]   (dtype)
 *     log_a, dlog_a           : [B, H, L, m]    (fp32)
 *     hk0, hkT, dhkT, dhk0    : [B, H, m, Dk]   (fp32, nullable)
 *     hv0, hvT, dhvT, dhv0    : [B, H, m, Dv]   (fp32, nullable)
 * The backward returns the gradients of <dO, o> + <dhkT, hkT> + <dhvT, hvT>.
 * Errors and ownership as for gla_fwd / gla_bwd; the workspace (caller
 * allocated, 256-byte aligned) holds the two GLA passes' workspaces and the
 * per-slot intermediates (w, s and, in the backward, their gradients). */
/* The route gla_gsa_fwd / gla_gsa_bwd take for (d, slots): *impl = GLA_IMPL_TC (tensor cores:
 * bf16, slots = 128, both GLA passes on the tensor-core path with materialised states, the logits and
 * the read gradient by a fused fp32 slot-read kernel that also prepares the next GLA pass's query
 * operands) or GLA_IMPL_SIMT (both GLA passes on the CUDA
 * cores in fp32; bf16 tensors are converted at the boundary). Returns GLA_ERR_INVALID_ARG /
 * GLA_ERR_UNSUPPORTED like the compute calls. */
gla_status gla_gsa_resolve(const gla_desc* d, int32_t slots, int32_t* impl);
size_t gla_gsa_fwd_workspace_size(const gla_desc* d, int32_t slots);
size_t gla_gsa_bwd_workspace_size(const gla_desc* d, int32_t slots);
gla_status gla_gsa_fwd(const gla_desc* d, int32_t slots, const void* q, const void* k, const void* v,
                       const float* log_a, const float* hk0, const float* hv0, void* o, float* hkT,
                       float* hvT, void* workspace, size_t workspace_bytes, void* stream);
/* One decode step of gated slot attention for a batch of single tokens: q, k [B,H,Dk], v [B,H,Dv]
 * (d->dtype), log_a [B,H,slots] (fp32, or z with GLA_GATE_PREACT), the memories Kmem [B,H,slots,Dk]
 * and Vmem [B,H,slots,Dv] (fp32, updated in place: the step's hkT / hvT), o [B,H,Dv] (d->dtype). d->L is
 * ignored; Dk and Dv multiples of 4. Applied L times from hk0 / hv0 it gives what gla_gsa_fwd
 * gives for those L tokens. GLA_FLAG_CHECKS checks the gate domain and that o and both memories are
 * finite. */
gla_status gla_gsa_step(const gla_desc* d, int32_t slots, const void* q, const void* k, const void* v,
                        const float* log_a, float* Kmem, float* Vmem, void* o, void* stream);
gla_status gla_gsa_bwd(const gla_desc* d, int32_t slots, const void* q, const void* k, const void* v,
                       const float* log_a, const float* hk0, const float* hv0, const void* dO,
                       const float* dhkT, const float* dhvT, void* dq, void* dk, void* dv, float* dlog_a,
                       float* dhk0, float* dhv0, void* workspace, size_t workspace_bytes, void* stream);

/* ---- forward without any allocation ---------------------------------------
 * The paper has no counterpart to this entry point; it exists for callers
 * that cannot allocate device memory or provide a workspace: a plugin under
 * a framework or server that owns every device allocation, a latency-critical
 * loop that must not risk the implicit synchronisation of cudaMalloc/cudaFree,
 * or a C caller with no device memory manager.
 *
 * gla_fwd_noalloc computes exactly what gla_fwd computes (same arguments,
 * same layouts; the CUDA-core kernel path, chosen whatever d->impl says
 * except that GLA_IMPL_TC or GLA_STATE_NONMATERIALIZED return
 * GLA_ERR_UNSUPPORTED), but takes its scratch from a fixed array of
 * GLA_NOALLOC_SCRATCH_BYTES bytes built into the library; it calls no
 * cudaMalloc, cudaFree or other allocating routine.
 *  - Every GPU that loads the library's kernels holds that array until the
 *    process exits.
 *  - A problem whose gla_fwd_workspace_size (with impl = GLA_IMPL_SIMT)
 *    exceeds GLA_NOALLOC_SCRATCH_BYTES is rejected with GLA_ERR_WORKSPACE
 *    before any launch.
 *  - All calls on one device share the array and it keeps the last call's
 *    contents; nothing in it needs clearing, but calls that overlap on the
 *    GPU (other streams or host threads) race and must be serialised.
 *  - The first call on each device looks up the array's device address
 *    (cudaGetSymbolAddress, with that device current), and so does the first
 *    call after the device's context was replaced (cudaDeviceReset): make
 *    those calls before any stream capture begins. */
#define GLA_NOALLOC_SCRATCH_BYTES (16u << 20)
gla_status gla_fwd_noalloc(const gla_desc* d, const void* q, const void* k, const void* v,
                           const float* log_a, const float* h0, void* o, float* hT, void* stream);

/* Blocks until `stream` is idle, then reports (and clears) the device-side
 * error flag: GLA_ERR_TIMEOUT if a bounded wait ran out in any kernel since
 * the last check; else, for calls made in checking mode (GLA_FLAG_CHECKS),
 * GLA_ERR_INVALID_ARG if a gate was outside its domain or an output was not
 * finite, GLA_ERR_WORKSPACE if a workspace guard block was overwritten;
 * GLA_ERR_CUDA on a sticky CUDA error; else GLA_OK. */
gla_status gla_check_device_error(void* stream);

/* The same report under the name the scope table of this layer gives it. */
gla_status gla_last_device_error(void* stream);

/* gla_fwd_workspace_size / gla_bwd_workspace_size under the names the scope
 * table of this layer gives them (identical results). */
size_t gla_fwd_workspace_bytes(const gla_desc* d);
size_t gla_bwd_workspace_bytes(const gla_desc* d);

/* Self-test of the error path: launches one CTA whose mbarrier wait can never
 * complete (nothing arrives on the barrier). The bounded wait gives up after
 * about `limit_cycles` SM cycles (0: 2,000,000, about 1 ms) and records
 * GLA_ERR_TIMEOUT in the device flag, exactly as a stalled kernel of the path
 * would; the kernel then exits normally and the context stays usable. The
 * next gla_check_device_error(stream) reports GLA_ERR_TIMEOUT. Returns
 * GLA_ERR_CUDA if the launch fails. */
gla_status gla_selftest_wait_timeout(long long limit_cycles, void* stream);

/* Static description of a status code (never NULL). */
const char* gla_status_string(gla_status s);

/* GLA_ABI_VERSION of the loaded library. */
int gla_abi_version(void);

/* Chunk and sub-chunk lengths gla_fwd/gla_bwd use for `d` after defaults
 * are applied, and the kernel family (gla_impl) it resolves to; returns
 * GLA_ERR_INVALID_ARG / GLA_ERR_UNSUPPORTED like the compute calls would. */
gla_status gla_resolve(const gla_desc* d, int32_t* chunk, int32_t* subchunk,
                       int32_t* impl, int32_t* state_mode);

/* ---- measurement hooks (host-side counters; off the math path) ---------- */

/* Number of kernels this library has launched since load (or the last
 * reset). */
uint64_t gla_launch_count(void);
void gla_launch_count_reset(void);

/* When enabled (on != 0), every kernel launch is bracketed by a pair of CUDA
 * events recorded on the launching stream, so per-kernel device time can be
 * read back with gla_profile_read. Events are created lazily on the first
 * enabled launch (this is the only place the library creates CUDA objects)
 * and destroyed by gla_profile_reset. */
void gla_profile_enable(int on);

/* Synchronises the recorded events and writes, for up to `cap` kernel
 * names, the name (pointer to a static string), the number of launches and
 * the summed device milliseconds. Returns the number of distinct kernels
 * (which may exceed cap). */
int gla_profile_read(const char** names, uint64_t* launches, double* total_ms, int cap);
void gla_profile_reset(void);

#ifdef __cplusplus
}
#endif

#endif /* GLA_H_ */
