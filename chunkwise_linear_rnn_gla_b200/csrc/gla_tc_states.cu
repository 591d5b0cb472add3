// Materialised inter-chunk states: the sequential walk alone
// ("Gated Linear Attention Transformers with Hardware-Efficient Training",
// atlas.scime.ai summary, "Approach": materialised inter-chunk states).
//
//   forward : S_[0] = h0,  S_[i+1] = diag(e^{Gamma_i}) S_[i] + K~_i^T v_i,   hT = S_[N]
//   backward: D_{N-1} = dhT, D_{i-1} = diag(e^{Gamma_i}) D_i + Q~_i^T dO_i,   dh0 = D_{-1}
// writing the state that enters every chunk to HBM in bf16.
//
// One CTA owns a [128 key channels x BVS value columns] tile of one head's
// state (BVS = 128, or 64 when there are few heads). The chunk products U_i = A_i^T B_i (M = 128 channels, N = 64 values,
// K = 128 tokens, operands by TMA with the 128-byte swizzle) do not depend on
// the state, so the tcgen05 MMAs run up to three chunks ahead of the
// recurrence (three TMEM accumulators); the fp32 state itself lives in the
// registers of BVS / 64 groups of four epilogue warps (thread = key channel,
// 64 values), which per chunk store the bf16 copy of the entering state and
// apply S <- e^{Gamma} S + U. Nothing on the tensor-core side waits for the
// epilogue except the reuse of a TMEM buffer, so the walk runs at the speed
// of its loads. One CTA per SM.

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
constexpr uint32_t PIECE = 16384;
// warp 0 TMA, warp 1 MMA, then one group of four epilogue warps per 64 value columns
template <int BVS>
constexpr int st_threads() { return 64 + 128 * (BVS / 64); }

// Tile of BVS value columns (64 or 128): chunks in flight, bytes per chunk
// (the key-channel pair of A pieces and BVS / 64 value pieces), CTAs per SM.
// The narrow tile is used when the wide grid would leave most SMs idle (few
// heads, long sequences): each walk is then bound by the chunks it has in
// flight, so it keeps four of them.
template <int BVS>
struct StCfg {
    static constexpr int nslot = BVS == 64 ? 4 : 2;
    static constexpr uint32_t slot_bytes = uint32_t(2 + BVS / 64) * PIECE;
    static constexpr int min_blocks = 1;
    // + two staging pieces per epilogue group (double-buffered bf16 state for the TMA stores)
    static constexpr size_t smem = 1024 + size_t(nslot) * slot_bytes + size_t(2 * (BVS / 64)) * PIECE;
    static constexpr uint32_t tmem_cols = 3 * BVS <= 256 ? 256u : 512u;
};

struct StBars {
    uint64_t full[4], empty[4];
    uint64_t u_full[3], u_empty[3], drain;
    uint32_t tmem_slot;
    int abort_flag;
};

constexpr int kMaxSegs = 16;  // segments of a split walk (WalkSegs, gla_tc.h)

// S_in[g] for g = 1 .. G-1 from the pass-1 end states E[g] (E[0] is exact), and the final state.
// One block per state row (head, key channel), one thread per four value columns; the first G
// threads form the decay of every segment (the product of e^{Gamma} over its chunks) first.
template <bool REVERSE>
__global__ void __launch_bounds__(128) k_walk_seg_scan(const float* __restrict__ E, const float* __restrict__ gam,
                                                       float* __restrict__ S_in, float* __restrict__ fin,
                                                       float* __restrict__ fin2, int64_t N, int64_t K, int64_t V,
                                                       int64_t BH, int G, int len) {
    __shared__ float dec[kMaxSegs];
    pdl_wait();  // the end states of pass 1
    const int64_t row = blockIdx.x;  // bh * K + c
    const int64_t bh = row / K, c = row % K;
    const int t = threadIdx.x;
    if (t < G) {
        float d = 1.f;
        const int s_end = (t + 1) * len < N ? (t + 1) * len : int(N);
        for (int st = t * len; st < s_end; ++st) d *= gam[(bh * N + (REVERSE ? N - 1 - st : st)) * K + c];
        dec[t] = d;
    }
    __syncthreads();
    const int64_t stride = BH * K * V;
    for (int64_t v4 = t; v4 < V / 4; v4 += blockDim.x) {
        const int64_t e4 = row * (V / 4) + v4;
        // every segment's end state first (independent loads), then the recurrence over them
        float4 u[kMaxSegs];
#pragma unroll
        for (int g = 0; g < kMaxSegs; ++g)
            if (g < G) u[g] = reinterpret_cast<const float4*>(E + g * stride)[e4];
        float4 x = u[0];
#pragma unroll
        for (int g = 1; g < kMaxSegs; ++g) {
            if (g >= G) break;
            reinterpret_cast<float4*>(S_in + g * stride)[e4] = x;
            const float d = dec[g];
            x = make_float4(fmaf(d, x.x, u[g].x), fmaf(d, x.y, u[g].y), fmaf(d, x.z, u[g].z), fmaf(d, x.w, u[g].w));
        }
        if (fin) reinterpret_cast<float4*>(fin)[e4] = x;
        if (fin2) reinterpret_cast<float4*>(fin2)[e4] = x;
    }
}

template <int BVS, bool REVERSE>
__global__ void __launch_bounds__(st_threads<BVS>(), StCfg<BVS>::min_blocks)
    k_states_walk(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                  const __grid_constant__ CUtensorMap tmS,
                  const float* __restrict__ gam, const float* __restrict__ init, float* __restrict__ fin,
                  float* __restrict__ fin2, __nv_bfloat16* __restrict__ states, int64_t L, int64_t N, int64_t V,
                  int64_t K, int64_t BH, WalkSegs sg, int* err) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    constexpr int NSLOT = StCfg<BVS>::nslot;
    constexpr uint32_t SLOT_BYTES = StCfg<BVS>::slot_bytes;
    StBars& bar = *reinterpret_cast<StBars*>(ring + NSLOT * SLOT_BYTES + 2 * (BVS / 64) * PIECE);
    volatile int* abort_flag = &bar.abort_flag;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int v0 = blockIdx.x * BVS;
    const int kbase = blockIdx.y * 128;
    // blockIdx.z = head + BH * (segment - sg.first); a segment is sg.len consecutive steps of the walk
    const int64_t bh = blockIdx.z % BH;
    const int seg = sg.first + int(blockIdx.z / BH);
    const int s0 = seg * sg.len;
    const int nsteps = int(N) - s0 < sg.len ? int(N) - s0 : sg.len;
    auto chunk_of = [&](int step) -> int { return REVERSE ? int(N) - 1 - (s0 + step) : s0 + step; };
    const bool store = sg.store_all > 0 || (sg.store_all == 0 && seg == 0);
    const float* init_s = seg == 0 ? init : (sg.init_seg ? sg.init_seg + seg * sg.stride : nullptr);
    float* fin_s = fin ? fin + seg * sg.stride : nullptr;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NSLOT; ++s) {
            mbar_init(&bar.full[s], 1);
            mbar_init(&bar.empty[s], 1);
        }
        for (int b = 0; b < 3; ++b) {
            mbar_init(&bar.u_full[b], 1);
            mbar_init(&bar.u_empty[b], 128 * (BVS / 64));
        }
        mbar_init(&bar.drain, 1);
        bar.abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(&bar.tmem_slot, StCfg<BVS>::tmem_cols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bar.tmem_slot;
    // programmatic dependent launch: the prologue above overlapped the previous kernel's tail;
    // nothing below touches global memory before that kernel has completed
    if (threadIdx.x == 0) {  // tensor maps are kernel parameters: fetch them while the previous kernel drains
        tma_prefetch(&tmA);
        tma_prefetch(&tmB);
        tma_prefetch(&tmS);
    }
    pdl_launch_dependents();
    pdl_wait();

    if (warp == 0) {
        if (lane == 0) {
            bool ok = true;
            int step = 0;
            for (; step < nsteps && ok; ++step) {
                const int s = step % NSLOT;
                if (!mbar_wait(&bar.empty[s], uint32_t(((step / NSLOT) & 1) ^ 1), err, abort_flag)) {
                    ok = false;
                    break;
                }
                const int row0 = chunk_of(step) * C;
                uint8_t* st = ring + s * SLOT_BYTES;
                mbar_arrive_expect_tx(&bar.full[s], SLOT_BYTES);
                tma_load_3d(st, &tmA, kbase, row0, int(bh), &bar.full[s]);
                tma_load_3d(st + PIECE, &tmA, kbase + 64, row0, int(bh), &bar.full[s]);
#pragma unroll
                for (int q = 0; q < BVS / 64; ++q)
                    tma_load_3d(st + (2 + q) * PIECE, &tmB, v0 + 64 * q, row0, int(bh), &bar.full[s]);
            }
            if (!ok)
                for (int w = step - NSLOT; w < step; ++w)
                    if (w >= 0) mbar_drain(&bar.full[w % NSLOT], uint32_t((w / NSLOT) & 1));
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // U[c][v] = sum_t A[t][c] B[t][v]: A and B both MN-major (channels / values contiguous)
            const uint32_t id = idesc_bf16_f32(128, BVS, true, true);
            bool ok = true;
            for (int step = 0; step < nsteps && ok; ++step) {
                const int s = step % NSLOT, b = step % 3;
                ok = mbar_wait(&bar.u_empty[b], uint32_t(((step / 3) & 1) ^ 1), err, abort_flag) &&
                     mbar_wait(&bar.full[s], uint32_t((step / NSLOT) & 1), err, abort_flag);
                if (!ok) break;
                tc_fence_after();
                const uint32_t a0 = smem_u32(ring + s * SLOT_BYTES), b0 = a0 + 2 * PIECE;
#pragma unroll
                for (int kk = 0; kk < C / 16; ++kk)
                    mma_bf16(tmem + uint32_t(b * BVS), sdesc_sw128(a0 + kk * 2048, PIECE, 1024),
                             sdesc_sw128(b0 + kk * 2048, PIECE, 1024), id, kk > 0 ? 1u : 0u);
                mma_commit(&bar.u_full[b]);
                mma_commit(&bar.empty[s]);
            }
            mma_commit(&bar.drain);
            mbar_drain(&bar.drain, 0);
        }
    } else {
        // state epilogue: BVS / 64 groups of four warps; thread = key channel (TMEM lane), the 64 value
        // columns of its group in registers
        const int q4 = warp & 3;
        const int grp = (warp - 2) >> 2;
        const int row = 32 * q4 + lane;
        const int64_t c = kbase + row;
        const int col0 = 64 * grp;  // first value column of the group within the tile
        const uint32_t lane_off = uint32_t(32 * q4) << 16;
        float x[64];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            const float4 v4 = init_s ? reinterpret_cast<const float4*>(init_s + (bh * K + c) * V + v0 + col0)[e]
                                     : make_float4(0.f, 0.f, 0.f, 0.f);
            x[4 * e] = v4.x;
            x[4 * e + 1] = v4.y;
            x[4 * e + 2] = v4.z;
            x[4 * e + 3] = v4.w;
        }
        // the bf16 copy of each entering state is staged in shared memory (128-byte swizzle, one
        // piece per group) and written by a TMA store issued by one thread of the group, so the
        // register file never waits on the stores
        uint8_t* stg0 = ring + NSLOT * SLOT_BYTES + 2 * grp * PIECE;
        const bool issuer = row == 0;
        bool ok = true;
        float g_next = gam[(bh * N + chunk_of(0)) * K + c];
        // every epilogue thread passes every named barrier, also after a wait gave up (bar.sync has
        // no time limit); a failed wait only skips the work
        for (int step = 0; step < nsteps; ++step) {
            const int b = step % 3;
            const int ci = chunk_of(step);
            uint8_t* stg = stg0 + (step & 1) * PIECE;
            const float g = g_next;  // loaded one step ahead, off the critical path
            if (step + 1 < nsteps) g_next = gam[(bh * N + chunk_of(step + 1)) * K + c];
            if (issuer) bulk_wait_read_but1();  // the store of two steps ago has read this staging piece
            named_sync(1 + grp, 128);
#pragma unroll
            for (int ch = 0; ch < 8; ++ch)
                *reinterpret_cast<uint4*>(stg + uint32_t(row) * 128u + uint32_t((ch ^ (row & 7)) << 4)) =
                    make_uint4(pack_bf16x2(x[8 * ch], x[8 * ch + 1]), pack_bf16x2(x[8 * ch + 2], x[8 * ch + 3]),
                               pack_bf16x2(x[8 * ch + 4], x[8 * ch + 5]), pack_bf16x2(x[8 * ch + 6], x[8 * ch + 7]));
            fence_proxy_async_smem();
            named_sync(1 + grp, 128);
            if (issuer && ok && store) {
                tma_store_3d(&tmS, v0 + col0, kbase, int(bh * N + ci), stg);
                bulk_commit();
            }
            // tcgen05.ld is warp-collective: the condition must be the same for the whole warp
            ok = __all_sync(0xffffffffu, ok && mbar_wait(&bar.u_full[b], uint32_t((step / 3) & 1), err, abort_flag));
            if (ok) {
                tc_fence_after();
#pragma unroll
                for (int c32 = 0; c32 < 2; ++c32) {
                    float u[32];
                    tmem_ld16(tmem + lane_off + uint32_t(b * BVS + col0 + 32 * c32), u);
                    tmem_ld16(tmem + lane_off + uint32_t(b * BVS + col0 + 32 * c32 + 16), u + 16);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) x[32 * c32 + e] = fmaf(g, x[32 * c32 + e], u[e]);
                }
                tc_fence_before();
                mbar_arrive(&bar.u_empty[b]);
            }
        }
        if (issuer) bulk_wait_read_all();  // the stores finish on their own; the CTA may exit once they have read smem
        if (ok) {
            for (int w = 0; w < 2; ++w) {
                float* f = w ? fin2 : fin_s;
                if (!f) continue;
                float4* d4 = reinterpret_cast<float4*>(f + (bh * K + c) * V + v0 + col0);
#pragma unroll
                for (int e = 0; e < 16; ++e) d4[e] = make_float4(x[4 * e], x[4 * e + 1], x[4 * e + 2], x[4 * e + 3]);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, StCfg<BVS>::tmem_cols);
    }
}

bool map3(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t outer) {
    const uint64_t dims[3] = {inner, rows, outer};
    const uint64_t strides[2] = {inner * 2, inner * rows * 2};
    const uint32_t box[3] = {64, 128, 1};
    return encode_tmap(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

// Tile width and segments of a walk. 128-column tiles halve the re-reads of the key operand through
// L2 when d_v allows and the grid still covers half of the SMs; otherwise 64-column tiles with more
// chunks in flight. Segments: as many as the SMs allow for the CTAs of one segment (at most
// kMaxSegs, each at least four chunks); two passes only pay from three segments on.
struct WalkPlan {
    bool wide;
    int64_t G;
    int len;
};

WalkPlan walk_plan(const Problem& p, int64_t ctas_per_segment_narrow, bool may_split) {
    WalkPlan w{};
    const int64_t sms = sm_count();
    const int64_t wide_ctas = p.BH * (p.K / 128) * (p.V / 128);
    w.wide = p.V % 128 == 0 && 2 * wide_ctas >= sms;
    const int64_t ctas = w.wide ? wide_ctas : ctas_per_segment_narrow;
    w.G = 1;
    if (may_split) {
        w.G = sms / ctas;
        if (w.G > kMaxSegs) w.G = kMaxSegs;
        if (w.G > p.N / 4) w.G = p.N / 4;
        if (w.G < 3) w.G = 1;
    }
    w.len = int((p.N + w.G - 1) / w.G);
    w.G = (p.N + w.len - 1) / w.len;
    return w;
}

gla_status launch_states(const Problem& p, const CUtensorMap* m, bool wide, bool reverse, const float* gam,
                         const float* init, float* fin, float* fin2, __nv_bfloat16* states, const WalkSegs& sg,
                         int64_t nseg, cudaStream_t s, const char* name) {
    const int bvs = wide ? 128 : 64;
    const size_t smem = (wide ? StCfg<128>::smem : StCfg<64>::smem) + sizeof(StBars);
    auto fn = wide ? (reverse ? k_states_walk<128, true> : k_states_walk<128, false>)
                   : (reverse ? k_states_walk<64, true> : k_states_walk<64, false>);
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) != cudaSuccess)
        return GLA_ERR_CUDA;
    const unsigned threads = wide ? st_threads<128>() : st_threads<64>();
    const dim3 grid(unsigned(p.V / bvs), unsigned(p.K / 128), unsigned(p.BH * nseg));
    GLA_LAUNCH_PDL(name, fn, grid, threads, smem, s, m[0], m[1], m[2], gam, init, fin, fin2, states, p.L, p.N, p.V,
                   p.K, p.BH, sg, device_error_word());
    return GLA_OK;
}

gla_status launch_seg_scan(const Problem& p, bool reverse, const float* E, const float* gam, float* S_in, float* fin,
                           float* fin2, int64_t G, int len, cudaStream_t s) {
    auto scan = reverse ? k_walk_seg_scan<true> : k_walk_seg_scan<false>;
    const unsigned threads = unsigned(p.V / 4 < 128 ? p.V / 4 : 128);  // >= 16 >= G
    GLA_LAUNCH_PDL("tc_walk_seg_scan", scan, dim3(unsigned(p.BH * p.K)), threads, 0, s, E, gam, S_in, fin, fin2, p.N,
                   p.K, p.V, p.BH, int(G), len);
    return GLA_OK;
}

bool make_maps(CUtensorMap* m, const Problem& p, const __nv_bfloat16* A, const __nv_bfloat16* B,
               const void* states) {
    memset(m, 0, 3 * sizeof(CUtensorMap));
    return map3(&m[0], A, uint64_t(p.K), uint64_t(p.L), uint64_t(p.BH)) &&
           map3(&m[1], B, uint64_t(p.V), uint64_t(p.L), uint64_t(p.BH)) &&
           map3(&m[2], states, uint64_t(p.V), uint64_t(p.K), uint64_t(p.BH * p.N));
}

}  // namespace

bool tc_states_walk_supported(const Problem& p) { return p.V % 64 == 0; }

size_t tc_walk_seg_floats(const Problem& p) {
    // only walks whose narrow grid covers few SMs are ever split; the size does not depend on the device
    const int64_t narrow_ctas = p.BH * (p.K / 128) * (p.V / 64);
    if (narrow_ctas > 64 || p.N < 12) return 0;
    return size_t(2) * kMaxSegs * size_t(p.BH * p.K * p.V);
}

gla_status tc_states_walk_launch(const Problem& p, const __nv_bfloat16* A, const __nv_bfloat16* B, const float* gam,
                                 const float* init, float* fin, float* fin2, __nv_bfloat16* states, float* segbuf,
                                 bool reverse, cudaStream_t s, const char* name) {
    CUtensorMap m[3];
    if (!make_maps(m, p, A, B, states)) return GLA_ERR_CUDA;
    const WalkPlan w = walk_plan(p, p.BH * (p.K / 128) * (p.V / 64), segbuf != nullptr);
    if (w.G == 1)
        return launch_states(p, m, w.wide, reverse, gam, init, fin, fin2, states, WalkSegs{0, int(p.N), 1, 0, nullptr},
                             1, s, name);
    const int64_t stride = p.BH * p.K * p.V;
    float* E = segbuf;                                  // end state of every segment walked from zero
    float* S_in = segbuf + int64_t(kMaxSegs) * stride;  // true state entering every segment
    gla_status st = launch_states(p, m, w.wide, reverse, gam, init, E, nullptr, states,
                                  WalkSegs{0, w.len, 0, stride, nullptr}, w.G, s, name);
    if (st == GLA_OK) st = launch_seg_scan(p, reverse, E, gam, S_in, fin, fin2, w.G, w.len, s);
    if (st == GLA_OK)
        st = launch_states(p, m, w.wide, reverse, gam, init, nullptr, nullptr, states,
                           WalkSegs{1, w.len, 1, stride, S_in}, w.G - 1, s, name);
    return st;
}

gla_status tc_states_walk_final(const Problem& p, const __nv_bfloat16* A, const __nv_bfloat16* B, const float* gam,
                                const float* init, float* fin, float* segbuf, bool reverse, cudaStream_t s,
                                const char* name) {
    CUtensorMap m[3];
    // nothing is stored: the states map only has to be a valid descriptor
    if (!make_maps(m, p, A, B, A)) return GLA_ERR_CUDA;
    const WalkPlan w = walk_plan(p, p.BH * (p.K / 128) * (p.V / 64), segbuf != nullptr);
    if (w.G == 1)
        return launch_states(p, m, w.wide, reverse, gam, init, fin, nullptr, nullptr,
                             WalkSegs{0, int(p.N), -1, 0, nullptr}, 1, s, name);
    const int64_t stride = p.BH * p.K * p.V;
    float* E = segbuf;
    float* S_in = segbuf + int64_t(kMaxSegs) * stride;
    gla_status st = launch_states(p, m, w.wide, reverse, gam, init, E, nullptr, nullptr,
                                  WalkSegs{0, w.len, -1, stride, nullptr}, w.G, s, name);
    if (st == GLA_OK) st = launch_seg_scan(p, reverse, E, gam, S_in, fin, nullptr, w.G, w.len, s);
    return st;
}

int tc_walk_seg_prepare(const Problem& p, const __nv_bfloat16* A, const __nv_bfloat16* B, const float* gam,
                        const float* init, float* fin, float* fin2, float* segbuf, bool reverse, cudaStream_t s,
                        int* len, const float** S_in_out, int64_t* stride_out, gla_status* st) {
    *st = GLA_OK;
    if (!segbuf) return 1;
    // segments sized for the fused walk's grid (one CTA per head and 64 value columns)
    const WalkPlan w = walk_plan(p, p.BH * (p.V / 64), true);
    if (w.G == 1) return 1;
    CUtensorMap m[3];
    // pass 1 stores nothing; the states map only has to be a valid descriptor
    if (!make_maps(m, p, A, B, segbuf)) {
        *st = GLA_ERR_CUDA;
        return 1;
    }
    const int64_t stride = p.BH * p.K * p.V;
    float* E = segbuf;
    float* S_in = segbuf + int64_t(kMaxSegs) * stride;
    *st = launch_states(p, m, w.wide, reverse, gam, init, E, nullptr, nullptr, WalkSegs{0, w.len, -1, stride, nullptr},
                        w.G, s, reverse ? "tc_walk_seg_dv" : "tc_walk_seg_fwd");
    if (*st == GLA_OK) *st = launch_seg_scan(p, reverse, E, gam, S_in, fin, fin2, w.G, w.len, s);
    *len = w.len;
    *S_in_out = S_in;
    *stride_out = stride;
    return int(w.G);
}

}  // namespace gla
