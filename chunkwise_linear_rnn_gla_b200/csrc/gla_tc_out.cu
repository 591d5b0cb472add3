// Chunk-parallel output GEMMs from materialised chunk states
// ("Gated Linear Attention Transformers with Hardware-Efficient Training",
// atlas.scime.ai summary, "Approach": materialised inter-chunk states):
//   forward : o_i  = Q~_i S_[i] + P_i   v_i
//   dv      : dv_i = K~_i D_i   + P_i^T dO_i
// Y_i = A_i X_i + Pm_i B_i with X_i a stored bf16 [K x V] chunk state. One CTA
// owns a 64-column tile of one head and loops over all chunks; every operand
// of a chunk (A: 2K/128 pieces, X: K/128 pieces, Pm: 2 pieces, B: 1 piece, each
// 128 rows x 128 bytes with the 128-byte swizzle) streams through one TMA ring
// in the order the MMAs consume it; each group of four k-steps waits only for
// its own pieces and releases them as soon as its MMAs complete, so the ring
// stays full and the loads of later chunks overlap the current chunk's
// tcgen05 work. The fp32 accumulator is double-buffered in TMEM and drained
// by four epilogue warps.

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
constexpr int BV = kTcBV;
constexpr uint32_t PIECE = 16384;
constexpr int RING = 6;  // >= the 3 pieces one MMA group holds; two CTAs fit per SM
constexpr int kOutThreads = 192;  // warp 0 TMA, warp 1 MMA, warps 2-5 epilogue

struct OutBars {
    uint64_t full[RING], empty[RING];
    uint64_t o_full[2], o_empty[2];
    uint64_t drain;
    uint32_t tmem_slot;
    int abort_flag;
};

struct OutCursor {
    int pos = 0;
    __device__ int take() {
        const int s = pos;
        pos = (pos + 1) % RING;
        return s;
    }
    __device__ int take_pair() {
        if (pos == RING - 1) pos = 0;
        if (pos & 1) pos = (pos + 1) % RING;
        const int s = pos;
        pos = (pos + 2) % RING;
        return s;
    }
};

template <int NH, bool PT>
__global__ void __launch_bounds__(kOutThreads, 2)
    k_chunk_out(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmX,
                const __grid_constant__ CUtensorMap tmP, const __grid_constant__ CUtensorMap tmB,
                __nv_bfloat16* __restrict__ Y, int64_t L, int64_t N, int64_t V, int* err) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    OutBars& bar = *reinterpret_cast<OutBars*>(ring + RING * PIECE);
    volatile int* abort_flag = &bar.abort_flag;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int v0 = blockIdx.x * BV;
    const int64_t bh = blockIdx.z;
    // chunks i = blockIdx.y, blockIdx.y + gridDim.y, ...
    const int n_items = int((N - blockIdx.y + gridDim.y - 1) / gridDim.y);
    auto chunk_of = [&](int it) -> int { return int(blockIdx.y) + it * int(gridDim.y); };

    if (threadIdx.x == 0) {
        for (int s = 0; s < RING; ++s) {
            mbar_init(&bar.full[s], 1);
            mbar_init(&bar.empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bar.o_full[b], 1);
            mbar_init(&bar.o_empty[b], 128);
        }
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
            tma_prefetch(&tmX);
            tma_prefetch(&tmP);
            tma_prefetch(&tmB);
            OutCursor cur;
            uint32_t par = 0, pending = 0, pending_par = 0;
            auto load = [&](int slot, const CUtensorMap* m, int x, int y, int z) -> bool {
                const uint32_t ph = (par >> slot) & 1u;
                if (!mbar_wait(&bar.empty[slot], ph ^ 1u, err, abort_flag)) return false;
                mbar_arrive_expect_tx(&bar.full[slot], PIECE);
                tma_load_3d(ring + slot * PIECE, m, x, y, z, &bar.full[slot]);
                pending |= 1u << slot;
                pending_par = (pending_par & ~(1u << slot)) | (ph << slot);
                par ^= 1u << slot;
                return true;
            };
            bool ok = true;
            for (int it = 0; it < n_items && ok; ++it) {
                const int i = chunk_of(it);
                const int zs = int(bh * N + i);
                for (int h = 0; h < NH && ok; ++h) {  // X_h, then the two A pieces that pair with it
                    ok = load(cur.take(), &tmX, v0, 128 * h, zs);
                    for (int sub = 0; sub < 2 && ok; ++sub) ok = load(cur.take(), &tmA, 64 * (2 * h + sub), i * C, int(bh));
                }
                if (ok) {
                    const int sp = cur.take_pair();
                    ok = load(sp, &tmP, 0, 0, zs) && load(sp + 1, &tmP, 64, 0, zs);
                }
                if (ok) ok = load(cur.take(), &tmB, v0, i * C, int(bh));
            }
            if (!ok)
                for (int s = 0; s < RING; ++s)
                    if ((pending >> s) & 1u) mbar_wait(&bar.full[s], (pending_par >> s) & 1u, nullptr, abort_flag);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idQS = idesc_bf16_f32(128, BV, false, true);
            const uint32_t idPV = idesc_bf16_f32(128, BV, PT, true);
            OutCursor cur;
            uint32_t par = 0;
            auto wait_full = [&](int slot) -> bool {
                const uint32_t ph = (par >> slot) & 1u;
                par ^= 1u << slot;
                return mbar_wait(&bar.full[slot], ph, err, abort_flag);
            };
            bool ok = true;
            for (int it = 0; it < n_items && ok; ++it) {
                const int b = it & 1;
                const uint32_t d = tmem + uint32_t(b * BV);
                ok = mbar_wait(&bar.o_empty[b], uint32_t(((it >> 1) & 1) ^ 1), err, abort_flag);
                for (int h = 0; h < NH && ok; ++h) {
                    const int sx = cur.take();
                    if (!(ok = wait_full(sx))) break;
                    for (int sub = 0; sub < 2; ++sub) {
                        const int sa = cur.take();
                        if (!(ok = wait_full(sa))) break;
                        tc_fence_after();
                        const uint32_t a0 = smem_u32(ring + sa * PIECE);
                        const uint32_t x0 = smem_u32(ring + sx * PIECE) + sub * 64 * 128;
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            mma_bf16(d, sdesc_sw128(a0 + kk * 32, 16, 1024), sdesc_sw128(x0 + kk * 2048, 16, 1024), idQS,
                                     (h > 0 || sub > 0 || kk > 0) ? 1u : 0u);
                        mma_commit(&bar.empty[sa]);
                    }
                    if (ok) mma_commit(&bar.empty[sx]);
                }
                if (!ok) break;
                const int sp = cur.take_pair();
                const int sb = cur.take();
                ok = wait_full(sp) && wait_full(sp + 1) && wait_full(sb);
                if (!ok) break;
                tc_fence_after();
                const uint32_t p0 = smem_u32(ring + sp * PIECE);
                const uint32_t b0 = smem_u32(ring + sb * PIECE);
#pragma unroll
                for (int kk = 0; kk < C / 16; ++kk) {
                    const uint64_t ad = PT ? sdesc_sw128(p0 + kk * 2048, PIECE, 1024)
                                           : sdesc_sw128(p0 + (kk / 4) * PIECE + (kk % 4) * 32, 16, 1024);
                    mma_bf16(d, ad, sdesc_sw128(b0 + kk * 2048, 16, 1024), idPV, 1u);
                }
                mma_commit(&bar.o_full[b]);
                mma_commit(&bar.empty[sp]);
                mma_commit(&bar.empty[sp + 1]);
                mma_commit(&bar.empty[sb]);
            }
            mma_commit(&bar.drain);
            mbar_wait(&bar.drain, 0, nullptr, abort_flag, 4000000000LL);
        }
    } else {
        const int q = warp & 3;
        const int r = 32 * q + lane;
        const uint32_t lane_off = uint32_t(32 * q) << 16;
        for (int it = 0; it < n_items; ++it) {
            const int b = it & 1;
            if (!mbar_wait(&bar.o_full[b], uint32_t((it >> 1) & 1), err, abort_flag)) break;
            tc_fence_after();
            float y[BV];
#pragma unroll
            for (int c16 = 0; c16 < BV / 16; ++c16) tmem_ld16(tmem + lane_off + uint32_t(b * BV + 16 * c16), y + 16 * c16);
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(&bar.o_empty[b]);
            const int64_t t = int64_t(chunk_of(it)) * C + r;
            if (t < L) {
                uint4* dst = reinterpret_cast<uint4*>(Y + (bh * L + t) * V + v0);
#pragma unroll
                for (int ch = 0; ch < BV / 8; ++ch)
                    dst[ch] = make_uint4(pack_bf16x2(y[8 * ch], y[8 * ch + 1]), pack_bf16x2(y[8 * ch + 2], y[8 * ch + 3]),
                                         pack_bf16x2(y[8 * ch + 4], y[8 * ch + 5]),
                                         pack_bf16x2(y[8 * ch + 6], y[8 * ch + 7]));
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

template <int NH, bool PT>
gla_status launch_out(const Problem& p, const CUtensorMap* m, __nv_bfloat16* Y, cudaStream_t s, const char* name) {
    auto fn = k_chunk_out<NH, PT>;
    const size_t smem = 1024 + size_t(RING) * PIECE + sizeof(OutBars);
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) != cudaSuccess)
        return GLA_ERR_CUDA;
    // one wave of CTAs (two per SM at this shared-memory size); each walks every gy-th chunk
    const int64_t tiles = (p.V / BV) * p.BH;
    int64_t gy = 296 / tiles;
    if (gy > p.N) gy = p.N;
    if (gy < 1) gy = 1;
    const dim3 grid(unsigned(p.V / BV), unsigned(gy), unsigned(p.BH));
    GLA_LAUNCH(name, fn, grid, kOutThreads, smem, s, m[0], m[1], m[2], m[3], Y, p.L, p.N, p.V, device_error_word());
    return GLA_OK;
}

}  // namespace

gla_status tc_chunk_out_launch(const Problem& p, const __nv_bfloat16* A, const __nv_bfloat16* X,
                               const __nv_bfloat16* Pm, const __nv_bfloat16* Bv, bool p_transposed,
                               __nv_bfloat16* Y, cudaStream_t s, const char* name) {
    CUtensorMap m[4];
    memset(m, 0, sizeof(m));
    const uint64_t L = uint64_t(p.L), K = uint64_t(p.K), V = uint64_t(p.V), BH = uint64_t(p.BH), N = uint64_t(p.N);
    if (!(map3(&m[0], A, K, L, BH) && map3(&m[1], X, V, K, BH * N) && map3(&m[2], Pm, 128, 128, BH * N) &&
          map3(&m[3], Bv, V, L, BH)))
        return GLA_ERR_CUDA;
    const int NH = int(p.K / 128);
    if (NH == 1) return p_transposed ? launch_out<1, true>(p, m, Y, s, name) : launch_out<1, false>(p, m, Y, s, name);
    if (NH == 2) return p_transposed ? launch_out<2, true>(p, m, Y, s, name) : launch_out<2, false>(p, m, Y, s, name);
    return GLA_ERR_UNSUPPORTED;
}

}  // namespace gla
