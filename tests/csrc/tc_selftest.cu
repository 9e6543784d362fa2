// tc_selftest.cu -- test-only kernel: one tcgen05 MMA chain D (+)= A . B^T with
// A [M,K] and B [N,K] staged in shared memory in the K-major or MN-major
// 128-byte-swizzled layout, so each operand layout used by the KDA kernels can
// be checked against a plain matrix product.
#include <cuda_bf16.h>
#include <stdint.h>

#include "tc_common.cuh"

using namespace kda::tc;

namespace {

__global__ void __launch_bounds__(128) gemm_kernel(const __nv_bfloat16* A, const __nv_bfloat16* B,
                                                   float* D, const float* Dinit, int M, int N,
                                                   int K, int a_mn, int b_mn, int neg, int* err) {
    // a_mn == 2: A is read from TMEM (packed bf16 pairs at columns [256, 256 + K/2))
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint8_t* sA = smem;
    uint8_t* sB = smem + M * K * 2;
    __shared__ uint64_t bar;
    __shared__ uint32_t tbase;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    for (int i = tid; i < M * K; i += 128) {
        const int m = i / K, k = i % K;
        const uint32_t off = a_mn == 1 ? mnmajor_off(k, m, K) : kmajor_off(m, k, M);
        *(__nv_bfloat16*)(sA + off) = A[i];
    }
    for (int i = tid; i < N * K; i += 128) {
        const int n = i / K, k = i % K;
        const uint32_t off = b_mn ? mnmajor_off(k, n, K) : kmajor_off(n, k, N);
        *(__nv_bfloat16*)(sB + off) = B[i];
    }
    uint32_t ncols = a_mn == 2 ? 512 : 32;
    while (ncols < (uint32_t)N) ncols <<= 1;
    if (warp == 0) {
        tmem_alloc(&tbase, ncols);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = tbase;
    // optional initial accumulator
    if (Dinit) {
        for (int c0 = 0; c0 < N; c0 += 16) {
            float v[16];
            for (int j = 0; j < 16; ++j) v[j] = Dinit[(warp * 32 + lane) * N + c0 + j];
            tmem_st16(taddr(tm, warp * 32, c0), v);
        }
        tmem_st_wait();
    }
    if (a_mn == 2) {  // this thread's row of A into TMEM as packed bf16 pairs
        const int m = warp * 32 + lane;
        for (int c0 = 0; c0 < K / 2; c0 += 8) {
            uint32_t u[8];
            for (int j = 0; j < 8; ++j) {
                const __nv_bfloat16 lo = A[m * K + 2 * (c0 + j)], hi = A[m * K + 2 * (c0 + j) + 1];
                u[j] = (uint32_t)__bfloat16_as_ushort(lo) | ((uint32_t)__bfloat16_as_ushort(hi) << 16);
            }
            tmem_st8(taddr(tm, warp * 32, 256 + c0), u);
        }
        tmem_st_wait();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid == 0) {
        const uint32_t id = idesc_bf16(M, N, a_mn == 1, b_mn, neg != 0);
        const uint32_t aB = smem_u32(sA), bB = smem_u32(sB);
        for (int s = 0; s < K / 16; ++s) {
            const uint64_t db = b_mn ? mnmajor_desc(bB, K, s) : kmajor_desc(bB, N, s);
            if (a_mn == 2) {
                mma_bf16_ts(tm, tm + 256 + 8 * s, db, id, (Dinit != nullptr || s > 0) ? 1u : 0u);
            } else {
                const uint64_t da = a_mn ? mnmajor_desc(aB, K, s) : kmajor_desc(aB, M, s);
                mma_bf16(tm, da, db, id, (Dinit != nullptr || s > 0) ? 1u : 0u);
            }
        }
        mma_commit(&bar);
    }
    __syncwarp();
    mbar_wait(&bar, 0, err, 1);
    tc_fence_after();
    for (int c0 = 0; c0 < N; c0 += 16) {
        float v[16];
        tmem_ld16(taddr(tm, warp * 32, c0), v);
        tmem_wait16(v);
        for (int j = 0; j < 16; ++j) D[(warp * 32 + lane) * N + c0 + j] = v[j];
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tm, ncols);
}

}  // namespace

extern "C" int kda_selftest_gemm(const void* A, const void* B, float* D, const float* Dinit, int M,
                                 int N, int K, int a_mn, int b_mn, int neg) {
    if (M != 128 || N < 16 || N > 256 || N % 16 || K % 64 || K > 128) return -1;
    if ((b_mn && N % 64) || (a_mn == 1 && M % 64)) return -1;  // MN-major tiles are whole 64-wide blocks
    if (a_mn == 2 && N > 256) return -1;                          // A from TMEM at columns 256..
    int* err = nullptr;
    cudaMalloc(&err, sizeof(int));
    cudaMemset(err, 0, sizeof(int));
    const int smem = (M * K + N * K) * 2 + 1024;
    cudaFuncSetAttribute(gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    gemm_kernel<<<1, 128, smem>>>((const __nv_bfloat16*)A, (const __nv_bfloat16*)B, D, Dinit, M,
                                  N, K, a_mn, b_mn, neg, err);
    cudaError_t e = cudaDeviceSynchronize();
    int h_err = 0;
    cudaMemcpy(&h_err, err, sizeof(int), cudaMemcpyDeviceToHost);
    cudaFree(err);
    if (e != cudaSuccess) return 1000 + (int)e;
    return h_err;
}
