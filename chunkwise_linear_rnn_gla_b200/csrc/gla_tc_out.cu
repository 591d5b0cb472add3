// Chunk-parallel output GEMMs from materialised chunk states
// ("Gated Linear Attention Transformers with Hardware-Efficient Training",
// atlas.scime.ai summary, "Approach": materialised inter-chunk states):
//   forward : o_i  = Q~_i S_[i] + P_i   v_i
//   dv      : dv_i = K~_i D_i   + P_i^T dO_i
// Y_i = A_i X_i + Pm_i B_i with X_i a stored bf16 [K x V] chunk state.
//
// Persistent kernel, one CTA per SM. A work item is one chunk and BVO value
// columns (BVO = 64 NQ, up to 256): its fp32 accumulator [128 x BVO] lives in
// TMEM and is double-buffered, so the epilogue of one item overlaps the MMAs
// of the next. Operands arrive by TMA (128-byte swizzle) in groups of 2 + NQ
// pieces of 16 KB through a ring of two groups: per 128 key channels, the two
// A pieces and the NQ state pieces of those channels; then the two Pm pieces
// and the NQ value pieces. The NQ pieces of a group sit side by side, so one
// MN-major descriptor (leading-byte offset = one piece) spans N = BVO and each
// tcgen05.mma computes the whole item width. Items of the same chunk are
// adjacent in the schedule, so the A and Pm tiles they share come from L2.

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
constexpr int kOutThreads = 192;  // warp 0 TMA, warp 1 MMA, warps 2-5 epilogue

struct OutBars {
    uint64_t full[2], empty[2];
    uint64_t o_full[2], o_empty[2];
    uint64_t drain;
    uint32_t tmem_slot;
    int abort_flag;
};

template <int NQ>
struct OutCfg {
    static constexpr int bvo = 64 * NQ;
    static constexpr int group = 2 + NQ;  // pieces per group
    static constexpr uint32_t tmem_cols = uint32_t(2 * 64 * NQ);
    static constexpr size_t smem = 1024 + size_t(2) * group * PIECE + sizeof(OutBars);
};

template <int NH, int NQ, bool PT>
__global__ void __launch_bounds__(kOutThreads, 1)
    k_chunk_out(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmX,
                const __grid_constant__ CUtensorMap tmP, const __grid_constant__ CUtensorMap tmB,
                __nv_bfloat16* __restrict__ Y, int64_t L, int64_t N, int64_t V, int64_t BH, int late_wait,
                int* err) {
    using Cfg = OutCfg<NQ>;
    constexpr int BVO = Cfg::bvo, G = Cfg::group;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    OutBars& bar = *reinterpret_cast<OutBars*>(ring + 2 * G * PIECE);
    volatile int* abort_flag = &bar.abort_flag;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int nvt = int(V / BVO);
    const int64_t n_items_total = BH * N * nvt;
    const int n_items = int((n_items_total - blockIdx.x + gridDim.x - 1) / gridDim.x);
    // item -> (head, chunk, value tile); the value tiles of one chunk are adjacent
    auto decode = [&](int it, int64_t& bh, int& i, int& v0) {
        const int64_t item = int64_t(blockIdx.x) + int64_t(it) * gridDim.x;
        v0 = int(item % nvt) * BVO;
        const int64_t rest = item / nvt;
        i = int(rest % N);
        bh = rest / N;
    };

    if (threadIdx.x == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bar.full[s], 1);
            mbar_init(&bar.empty[s], 1);
            mbar_init(&bar.o_full[s], 1);
            mbar_init(&bar.o_empty[s], 128);
        }
        mbar_init(&bar.drain, 1);
        bar.abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(&bar.tmem_slot, Cfg::tmem_cols);
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
        tma_prefetch(&tmX);
        tma_prefetch(&tmP);
        tma_prefetch(&tmB);
    }
    pdl_launch_dependents();
    // late_wait: launched after a kernel that it does not depend on (every input was complete before
    // that kernel passed its own wait); the blocks start on the SMs that kernel leaves idle, and
    // wait for it only before they exit, so that whatever follows sees both kernels complete
    if (!late_wait) pdl_wait();

    if (warp == 0) {
        if (lane == 0) {
            bool ok = true;
            int gc = 0;  // groups issued
            for (int it = 0; it < n_items && ok; ++it) {
                int64_t bh;
                int i, v0;
                decode(it, bh, i, v0);
                const int zs = int(bh * N + i);
                for (int g = 0; g <= NH && ok; ++g, ++gc) {
                    const int s = gc & 1;
                    if (!mbar_wait(&bar.empty[s], uint32_t(((gc >> 1) & 1) ^ 1), err, abort_flag)) {
                        ok = false;
                        break;
                    }
                    uint8_t* st = ring + s * G * PIECE;
                    mbar_arrive_expect_tx(&bar.full[s], G * PIECE);
                    if (g < NH) {  // A pieces of key channels 128g.., the state rows of those channels
                        tma_load_3d(st, &tmA, 128 * g, i * C, int(bh), &bar.full[s]);
                        tma_load_3d(st + PIECE, &tmA, 128 * g + 64, i * C, int(bh), &bar.full[s]);
#pragma unroll
                        for (int q = 0; q < NQ; ++q)
                            tma_load_3d(st + (2 + q) * PIECE, &tmX, v0 + 64 * q, 128 * g, zs, &bar.full[s]);
                    } else {  // Pm, then the value rows of the chunk
                        tma_load_3d(st, &tmP, 0, 0, zs, &bar.full[s]);
                        tma_load_3d(st + PIECE, &tmP, 64, 0, zs, &bar.full[s]);
#pragma unroll
                        for (int q = 0; q < NQ; ++q)
                            tma_load_3d(st + (2 + q) * PIECE, &tmB, v0 + 64 * q, i * C, int(bh), &bar.full[s]);
                    }
                }
            }
            if (!ok)  // let the copies already issued land before the block exits
                for (int w = gc - 2; w < gc; ++w)
                    if (w >= 0) mbar_drain(&bar.full[w & 1], uint32_t((w >> 1) & 1));
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idAX = idesc_bf16_f32(128, BVO, false, true);
            const uint32_t idPB = idesc_bf16_f32(128, BVO, PT, true);
            bool ok = true;
            int gc = 0;
            for (int it = 0; it < n_items && ok; ++it) {
                const int b = it & 1;
                const uint32_t d = tmem + uint32_t(b * BVO);
                ok = mbar_wait(&bar.o_empty[b], uint32_t(((it >> 1) & 1) ^ 1), err, abort_flag);
                for (int g = 0; g <= NH && ok; ++g, ++gc) {
                    const int s = gc & 1;
                    ok = mbar_wait(&bar.full[s], uint32_t((gc >> 1) & 1), err, abort_flag);
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t st = smem_u32(ring + s * G * PIECE);
                    if (g < NH) {
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk)
                            mma_bf16(d, sdesc_sw128(st + (kk / 4) * PIECE + (kk % 4) * 32, 16, 1024),
                                     sdesc_sw128(st + 2 * PIECE + kk * 2048, PIECE, 1024), idAX,
                                     (g > 0 || kk > 0) ? 1u : 0u);
                    } else {
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk) {
                            const uint64_t ad = PT ? sdesc_sw128(st + kk * 2048, PIECE, 1024)
                                                   : sdesc_sw128(st + (kk / 4) * PIECE + (kk % 4) * 32, 16, 1024);
                            mma_bf16(d, ad, sdesc_sw128(st + 2 * PIECE + kk * 2048, PIECE, 1024), idPB, 1u);
                        }
                    }
                    mma_commit(&bar.empty[s]);
                }
                if (ok) mma_commit(&bar.o_full[b]);
            }
            mma_commit(&bar.drain);
            mbar_drain(&bar.drain, 0);
        }
    } else {
        // epilogue: thread = token row of the item, BVO columns
        const int q4 = warp & 3;
        const int r = 32 * q4 + lane;
        const uint32_t lane_off = uint32_t(32 * q4) << 16;
        for (int it = 0; it < n_items; ++it) {
            const int b = it & 1;
            // tcgen05.ld is warp-collective: the condition must be the same for the whole warp
            if (!__all_sync(0xffffffffu, mbar_wait(&bar.o_full[b], uint32_t((it >> 1) & 1), err, abort_flag))) break;
            tc_fence_after();
            int64_t bh;
            int i, v0;
            decode(it, bh, i, v0);
            const int64_t t = int64_t(i) * C + r;
            __nv_bfloat16* dst = Y + (bh * L + t) * V + v0;
#pragma unroll 1
            for (int c32 = 0; c32 < BVO / 32; ++c32) {
                float y[32];
                tmem_ld16(tmem + lane_off + uint32_t(b * BVO + 32 * c32), y);
                tmem_ld16(tmem + lane_off + uint32_t(b * BVO + 32 * c32 + 16), y + 16);
                tmem_wait_ld();
                if (t < L) {
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        uint32_t w[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) w[e] = pack_bf16x2(y[16 * h + 2 * e], y[16 * h + 2 * e + 1]);
                        st_global_v8(dst + 32 * c32 + 16 * h, w);
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(&bar.o_empty[b]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, Cfg::tmem_cols);
    }
    if (late_wait) pdl_wait();
}

bool map3(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t outer) {
    const uint64_t dims[3] = {inner, rows, outer};
    const uint64_t strides[2] = {inner * 2, inner * rows * 2};
    const uint32_t box[3] = {64, 128, 1};
    return encode_tmap(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

template <int NH, int NQ, bool PT>
gla_status launch_out(const Problem& p, const CUtensorMap* m, __nv_bfloat16* Y, bool late_wait, cudaStream_t s,
                      const char* name) {
    auto fn = k_chunk_out<NH, NQ, PT>;
    const size_t smem = OutCfg<NQ>::smem;
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) != cudaSuccess)
        return GLA_ERR_CUDA;
    const int64_t items = p.BH * p.N * (p.V / OutCfg<NQ>::bvo);
    const int64_t sms = sm_count();
    const unsigned grid = unsigned(items < sms ? items : sms);
    GLA_LAUNCH_PDL(name, fn, dim3(grid), kOutThreads, smem, s, m[0], m[1], m[2], m[3], Y, p.L, p.N, p.V, p.BH,
                   int(late_wait), device_error_word());
    return GLA_OK;
}

template <int NH, bool PT>
gla_status launch_out_nq(const Problem& p, const CUtensorMap* m, __nv_bfloat16* Y, bool lw, cudaStream_t s,
                         const char* name) {
    if (p.V % 256 == 0) return launch_out<NH, 4, PT>(p, m, Y, lw, s, name);
    if (p.V % 128 == 0) return launch_out<NH, 2, PT>(p, m, Y, lw, s, name);
    return launch_out<NH, 1, PT>(p, m, Y, lw, s, name);
}

}  // namespace

gla_status tc_chunk_out_launch(const Problem& p, const __nv_bfloat16* A, const __nv_bfloat16* X,
                               const __nv_bfloat16* Pm, const __nv_bfloat16* Bv, bool p_transposed,
                               __nv_bfloat16* Y, bool late_wait, cudaStream_t s, const char* name) {
    CUtensorMap m[4];
    memset(m, 0, sizeof(m));
    const uint64_t L = uint64_t(p.L), K = uint64_t(p.K), V = uint64_t(p.V), BH = uint64_t(p.BH), N = uint64_t(p.N);
    if (!(map3(&m[0], A, K, L, BH) && map3(&m[1], X, V, K, BH * N) && map3(&m[2], Pm, 128, 128, BH * N) &&
          map3(&m[3], Bv, V, L, BH)))
        return GLA_ERR_CUDA;
    const int NH = int(p.K / 128);
    const bool lw = late_wait;
    if (NH == 1)
        return p_transposed ? launch_out_nq<1, true>(p, m, Y, lw, s, name) : launch_out_nq<1, false>(p, m, Y, lw, s, name);
    if (NH == 2)
        return p_transposed ? launch_out_nq<2, true>(p, m, Y, lw, s, name) : launch_out_nq<2, false>(p, m, Y, lw, s, name);
    return GLA_ERR_UNSUPPORTED;
}

}  // namespace gla
