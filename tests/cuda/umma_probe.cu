// Test-only probe of the sm_100a building blocks the tensor-core path uses:
// TMA loads with the 128-byte swizzle, tcgen05.mma (bf16 -> f32, M = 128)
// with every operand-major combination, TMEM allocation and tcgen05.ld.
// One CTA computes D[128 x N] = A[128 x K] * B[K x N]; the test compares it
// with torch.matmul.
//   A K-major : A stored [128][K] (row-major)   A MN-major : A stored [K][128]
//   B K-major : B stored [N][K]                 B MN-major : B stored [K][N]
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "tc_host.h"
#include "tc_prims.cuh"

using namespace gla::tc;

namespace {

__device__ int g_probe_err;

template <bool A_MN, bool B_MN>
__global__ void __launch_bounds__(128) k_probe(const __grid_constant__ CUtensorMap ta,
                                               const __grid_constant__ CUtensorMap tb, float* D, int N, int K) {
    extern __shared__ uint8_t raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
    const uint32_t a_bytes = 128u * K * 2u, b_bytes = uint32_t(N) * K * 2u;
    uint8_t* sA = smem;
    uint8_t* sB = smem + a_bytes;
    uint64_t* bars = reinterpret_cast<uint64_t*>(sB + b_bytes);
    uint32_t* tslot = reinterpret_cast<uint32_t*>(bars + 2);
    __shared__ int abort_flag;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    uint32_t ncols = 32;
    while (ncols < uint32_t(N)) ncols *= 2;
    if (threadIdx.x == 0) {
        abort_flag = 0;
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tslot, ncols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;
    if (threadIdx.x == 0) {
        mbar_arrive_expect_tx(&bars[0], a_bytes + b_bytes);
        if (!A_MN) {
            for (int p = 0; p < K / 64; ++p) tma_load_3d(sA + p * 16384, &ta, 64 * p, 0, 0, &bars[0]);
        } else {
            for (int mb = 0; mb < 2; ++mb) tma_load_3d(sA + mb * K * 128, &ta, 64 * mb, 0, 0, &bars[0]);
        }
        if (!B_MN) {
            for (int p = 0; p < K / 64; ++p) tma_load_3d(sB + p * N * 128, &tb, 64 * p, 0, 0, &bars[0]);
        } else {
            for (int nb = 0; nb < N / 64 || nb == 0; ++nb) tma_load_3d(sB + nb * K * 128, &tb, 64 * nb, 0, 0, &bars[0]);
        }
        if (mbar_wait(&bars[0], 0, &g_probe_err, &abort_flag)) {
            tc_fence_after();
            const uint32_t idesc = idesc_bf16_f32(128, N, A_MN, B_MN);
            for (int kk = 0; kk < K / 16; ++kk) {
                uint64_t ad, bd;
                if (!A_MN) ad = sdesc_sw128(smem_u32(sA + (kk / 4) * 16384 + (kk % 4) * 32), 16, 1024);
                else ad = sdesc_sw128(smem_u32(sA + kk * 2048), K * 128, 1024);
                if (!B_MN) bd = sdesc_sw128(smem_u32(sB + (kk / 4) * N * 128 + (kk % 4) * 32), 16, 1024);
                else bd = sdesc_sw128(smem_u32(sB + kk * 2048), K * 128, 1024);
                mma_bf16(tmem, ad, bd, idesc, kk > 0 ? 1u : 0u);
            }
            mma_commit(&bars[1]);
        }
    }
    __syncwarp();
    if (mbar_wait(&bars[1], 0, &g_probe_err, &abort_flag)) {
        tc_fence_after();
        const int row = warp * 32 + lane;
        for (int c0 = 0; c0 < N; c0 += 16) {
            float v[16];
            tmem_ld16(tmem + (uint32_t(warp * 32) << 16) + uint32_t(c0), v);
            tmem_wait_ld();
            for (int i = 0; i < 16; ++i) D[row * N + c0 + i] = v[i];
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tmem, ncols);
}

bool make_map(CUtensorMap* m, const void* base, int rows, int cols, int box_rows) {
    const uint64_t dims[3] = {uint64_t(cols), uint64_t(rows), 1};
    const uint64_t strides[2] = {uint64_t(cols) * 2, uint64_t(rows) * cols * 2};
    const uint32_t box[3] = {64, uint32_t(box_rows), 1};
    return encode_tmap(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

}  // namespace

// Returns 0 on success, 1 on bad arguments, 2 on encode failure, 3 on a CUDA
// error, 4 on a device wait timeout.
extern "C" int umma_probe(int a_mn, int b_mn, int N, int K, const void* A, const void* B, float* D) {
    if (N < 16 || N > 256 || N % 16 || K < 64 || K > 256 || K % 64) return 1;
    if (b_mn && N % 64) return 1;  // MN-major B pieces are 64 columns wide
    CUtensorMap ta, tb;
    bool ok = a_mn ? make_map(&ta, A, K, 128, K) : make_map(&ta, A, 128, K, 128);
    ok = ok && (b_mn ? make_map(&tb, B, K, N, K) : make_map(&tb, B, N, K, N));
    if (!ok) return 2;
    const size_t smem = 1024 + size_t(128) * K * 2 + size_t(N) * K * 2 + 64;
    void (*fn)(const CUtensorMap, const CUtensorMap, float*, int, int) = nullptr;
    if (!a_mn && !b_mn) fn = k_probe<false, false>;
    if (!a_mn && b_mn) fn = k_probe<false, true>;
    if (a_mn && !b_mn) fn = k_probe<true, false>;
    if (a_mn && b_mn) fn = k_probe<true, true>;
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) != cudaSuccess) return 3;
    fn<<<1, 128, smem>>>(ta, tb, D, N, K);
    if (cudaDeviceSynchronize() != cudaSuccess) return 3;
    int err = 0;
    cudaMemcpyFromSymbol(&err, g_probe_err, sizeof(int));
    return err ? 4 : 0;
}
