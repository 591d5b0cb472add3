// Materialised inter-chunk states: the sequential walk alone
// ("Gated Linear Attention Transformers with Hardware-Efficient Training",
// atlas.scime.ai summary, "Approach": materialised inter-chunk states).
//
//   forward : S_[0] = h0,  S_[i+1] = diag(e^{Gamma_i}) S_[i] + K~_i^T v_i,   hT = S_[N]
//   backward: D_{N-1} = dhT, D_{i-1} = diag(e^{Gamma_i}) D_i + Q~_i^T dO_i,   dh0 = D_{-1}
// writing the state that enters every chunk to HBM in bf16.
//
// One CTA owns a [128 key channels x 128 value columns] tile of one head's
// state. The fp32 state lives in TMEM and is updated in place: the epilogue
// writes the bf16 copy of the state entering chunk i, scales the TMEM state
// by e^{Gamma_i}, and the tcgen05 MMA of chunk i (M = 128 channels, N = 128
// values, K = 128 tokens, operands by TMA with the 128-byte swizzle)
// accumulates A_i^T B_i onto it. Compared with 64-column tiles this halves the
// number of CTAs that re-read each A_i tile through L2.

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
constexpr int BVS = 128;  // value columns per CTA
constexpr uint32_t PIECE = 16384;
constexpr int RING = 8;   // 2 chunks of (A pair, B pair)
constexpr int kThreads = 192;

struct StBars {
    uint64_t full[RING], empty[RING];
    uint64_t s_ready, u_done, drain;
    uint32_t tmem_slot;
    int abort_flag;
};

template <bool REVERSE>
__global__ void __launch_bounds__(kThreads, 1)
    k_states_walk(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                  const float* __restrict__ gam, const float* __restrict__ init, float* __restrict__ fin,
                  float* __restrict__ fin2, __nv_bfloat16* __restrict__ states, int64_t L, int64_t N, int64_t V,
                  int64_t K, int* err) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    StBars& bar = *reinterpret_cast<StBars*>(ring + RING * PIECE);
    volatile int* abort_flag = &bar.abort_flag;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int v0 = blockIdx.x * BVS;
    const int kbase = blockIdx.y * 128;
    const int64_t bh = blockIdx.z;
    const int nsteps = int(N);
    auto chunk_of = [&](int step) -> int { return REVERSE ? int(N) - 1 - step : step; };

    if (threadIdx.x == 0) {
        for (int s = 0; s < RING; ++s) {
            mbar_init(&bar.full[s], 1);
            mbar_init(&bar.empty[s], 1);
        }
        mbar_init(&bar.s_ready, 128);
        mbar_init(&bar.u_done, 1);
        mbar_init(&bar.drain, 1);
        bar.abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(&bar.tmem_slot, 128);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bar.tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            tma_prefetch(&tmA);
            tma_prefetch(&tmB);
            uint32_t par = 0, pending = 0, pending_par = 0;
            auto load = [&](int slot, const CUtensorMap* m, int x, int y) -> bool {
                const uint32_t ph = (par >> slot) & 1u;
                if (!mbar_wait(&bar.empty[slot], ph ^ 1u, err, abort_flag)) return false;
                mbar_arrive_expect_tx(&bar.full[slot], PIECE);
                tma_load_3d(ring + slot * PIECE, m, x, y, int(bh), &bar.full[slot]);
                pending |= 1u << slot;
                pending_par = (pending_par & ~(1u << slot)) | (ph << slot);
                par ^= 1u << slot;
                return true;
            };
            bool ok = true;
            for (int step = 0; step < nsteps && ok; ++step) {
                const int row0 = chunk_of(step) * C;
                const int s = (4 * step) % RING;  // A pair at s, B pair at s + 2
                ok = load(s, &tmA, kbase, row0) && load(s + 1, &tmA, kbase + 64, row0) &&
                     load(s + 2, &tmB, v0, row0) && load(s + 3, &tmB, v0 + 64, row0);
            }
            if (!ok)
                for (int s = 0; s < RING; ++s)
                    if ((pending >> s) & 1u) mbar_wait(&bar.full[s], (pending_par >> s) & 1u, nullptr, abort_flag);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t id = idesc_bf16_f32(128, BVS, true, true);
            bool ok = true;
            for (int step = 0; step < nsteps && ok; ++step) {
                const int s = (4 * step) % RING;
                const uint32_t ph = uint32_t((4 * step / RING) & 1);
                ok = mbar_wait(&bar.s_ready, uint32_t(step & 1), err, abort_flag);
                for (int e = 0; e < 4 && ok; ++e) ok = mbar_wait(&bar.full[s + e], ph, err, abort_flag);
                if (!ok) break;
                tc_fence_after();
                const uint32_t a0 = smem_u32(ring + s * PIECE), b0 = smem_u32(ring + (s + 2) * PIECE);
#pragma unroll
                for (int kk = 0; kk < C / 16; ++kk)
                    mma_bf16(tmem, sdesc_sw128(a0 + kk * 2048, PIECE, 1024), sdesc_sw128(b0 + kk * 2048, PIECE, 1024),
                             id, 1u);
                mma_commit(&bar.u_done);
                for (int e = 0; e < 4; ++e) mma_commit(&bar.empty[s + e]);
            }
            mma_commit(&bar.drain);
            mbar_wait(&bar.drain, 0, nullptr, abort_flag, 4000000000LL);
        }
    } else {
        // state epilogue: thread = key channel (TMEM lane), 128 value columns
        const int q = warp & 3;
        const int row = 32 * q + lane;
        const int c = kbase + row;
        const uint32_t lane_off = uint32_t(32 * q) << 16;
        float g = gam[(bh * N + chunk_of(0)) * K + c];
        // S_[first] = init: bf16 copy out, scale, into TMEM
        for (int c16 = 0; c16 < BVS / 16; ++c16) {
            float x[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) x[e] = init ? init[(bh * K + c) * V + v0 + 16 * c16 + e] : 0.f;
            uint4* dst = reinterpret_cast<uint4*>(states + ((bh * N + chunk_of(0)) * K + c) * V + v0 + 16 * c16);
            dst[0] = make_uint4(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]), pack_bf16x2(x[4], x[5]),
                                pack_bf16x2(x[6], x[7]));
            dst[1] = make_uint4(pack_bf16x2(x[8], x[9]), pack_bf16x2(x[10], x[11]), pack_bf16x2(x[12], x[13]),
                                pack_bf16x2(x[14], x[15]));
#pragma unroll
            for (int e = 0; e < 16; ++e) x[e] *= g;
            tmem_st16(tmem + lane_off + uint32_t(16 * c16), x);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bar.s_ready);
        for (int step = 0; step < nsteps; ++step) {
            const bool last = step + 1 == nsteps;
            const float g_next = last ? 0.f : gam[(bh * N + chunk_of(step + 1)) * K + c];
            if (!mbar_wait(&bar.u_done, uint32_t(step & 1), err, abort_flag)) break;
            tc_fence_after();
#pragma unroll
            for (int c32 = 0; c32 < BVS / 32; ++c32) {
                float x[32];
                tmem_ld16(tmem + lane_off + uint32_t(32 * c32), x);
                tmem_ld16(tmem + lane_off + uint32_t(32 * c32 + 16), x + 16);
                tmem_wait_ld();
                if (!last) {
                    uint4* dst =
                        reinterpret_cast<uint4*>(states + ((bh * N + chunk_of(step + 1)) * K + c) * V + v0 + 32 * c32);
#pragma unroll
                    for (int ch = 0; ch < 4; ++ch)
                        dst[ch] = make_uint4(pack_bf16x2(x[8 * ch], x[8 * ch + 1]), pack_bf16x2(x[8 * ch + 2], x[8 * ch + 3]),
                                             pack_bf16x2(x[8 * ch + 4], x[8 * ch + 5]),
                                             pack_bf16x2(x[8 * ch + 6], x[8 * ch + 7]));
#pragma unroll
                    for (int e = 0; e < 32; ++e) x[e] *= g_next;
                    tmem_st16(tmem + lane_off + uint32_t(32 * c32), x);
                    tmem_st16(tmem + lane_off + uint32_t(32 * c32 + 16), x + 16);
                } else {
                    for (int w = 0; w < 2; ++w) {
                        float* f = w ? fin2 : fin;
                        if (!f) continue;
                        float4* d4 = reinterpret_cast<float4*>(f + (bh * K + c) * V + v0 + 32 * c32);
#pragma unroll
                        for (int e = 0; e < 8; ++e) d4[e] = make_float4(x[4 * e], x[4 * e + 1], x[4 * e + 2], x[4 * e + 3]);
                    }
                }
            }
            if (!last) {
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(&bar.s_ready);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 128);
    }
}

bool map3(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t outer) {
    const uint64_t dims[3] = {inner, rows, outer};
    const uint64_t strides[2] = {inner * 2, inner * rows * 2};
    const uint32_t box[3] = {64, 128, 1};
    return encode_tmap(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

}  // namespace

bool tc_states_walk_supported(const Problem& p) { return p.V % BVS == 0; }

gla_status tc_states_walk_launch(const Problem& p, const __nv_bfloat16* A, const __nv_bfloat16* B, const float* gam,
                                 const float* init, float* fin, float* fin2, __nv_bfloat16* states, bool reverse,
                                 cudaStream_t s, const char* name) {
    CUtensorMap m[2];
    memset(m, 0, sizeof(m));
    if (!(map3(&m[0], A, uint64_t(p.K), uint64_t(p.L), uint64_t(p.BH)) &&
          map3(&m[1], B, uint64_t(p.V), uint64_t(p.L), uint64_t(p.BH))))
        return GLA_ERR_CUDA;
    const size_t smem = 1024 + size_t(RING) * PIECE + sizeof(StBars);
    auto fn = reverse ? k_states_walk<true> : k_states_walk<false>;
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) != cudaSuccess)
        return GLA_ERR_CUDA;
    const dim3 grid(unsigned(p.V / BVS), unsigned(p.K / 128), unsigned(p.BH));
    GLA_LAUNCH(name, fn, grid, kThreads, smem, s, m[0], m[1], gam, init, fin, fin2, states, p.L, p.N, p.V, p.K,
               device_error_word());
    return GLA_OK;
}

}  // namespace gla
