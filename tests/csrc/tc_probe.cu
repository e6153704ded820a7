// Test-only probe of the tcgen05 building blocks in tc_utils.cuh: fills shared
// memory in the swizzled operand layouts the chunk kernel uses, runs
// tcgen05.mma with the same descriptors, reads the accumulator back from TMEM
// with the same lane/column mapping, and writes D = A * B (fp32) to global
// memory.  The GPU test compares it with a plain matmul.
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../gated_delta_rule_86_b200/csrc/tc_utils.cuh"

using namespace kda;
using namespace kda::tc;

// Byte offset of element (row, col) of a [rows x cols] bf16 tile stored as
// 64-column SW128 blocks (cols % 64 == 0) or one SW64 block (cols == 32).
__device__ uint32_t tile_off(int row, int col, int rows, int cols) {
    if (cols == 32) return sw64(row, col / 8) + (col % 8) * 2;
    return (col / 64) * (rows * 128) + sw128(row, (col % 64) / 8) + (col % 8) * 2;
}

// A: [M][K] if !A_MN else [K][M];  B: [N][K] if !B_MN else [K][N];  D: [M][N] fp32.
template <int M, int N, int K, bool A_MN, bool B_MN>
__global__ void __launch_bounds__(128) probe_kernel(const __nv_bfloat16 *A, const __nv_bfloat16 *B, float *D) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = smem;
    uint8_t *sB = smem + ((M * K * 2 + 1023) / 1024) * 1024;
    __shared__ uint64_t bar;
    __shared__ uint32_t tbase;
    __shared__ int abort_flag;
    const int tid = threadIdx.x, warp = tid / 32;

    for (int i = tid; i < M * K; i += 128) {
        int m = A_MN ? i % M : i / K, k = A_MN ? i / M : i % K;
        uint32_t off = A_MN ? tile_off(k, m, K, M) : tile_off(m, k, M, K);
        *reinterpret_cast<__nv_bfloat16 *>(sA + off) = A[i];
    }
    for (int i = tid; i < N * K; i += 128) {
        int n = B_MN ? i % N : i / K, k = B_MN ? i / N : i % K;
        uint32_t off = B_MN ? tile_off(k, n, K, N) : tile_off(n, k, N, K);
        *reinterpret_cast<__nv_bfloat16 *>(sB + off) = B[i];
    }
    if (tid == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
        abort_flag = 0;
    }
    if (warp == 0) {
        tmem_alloc(&tbase, 512);
        tmem_relinquish();
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tbase;

    if (tid == 0) {
        constexpr uint32_t idesc = make_idesc_bf16(M, N, A_MN, B_MN);
        for (int kk = 0; kk < K / 16; ++kk) {
            uint64_t ad, bd;
            if (A_MN) ad = make_sdesc(smem_u32(sA) + kk * 2048, K * 128, 1024, kSwz128);
            else ad = make_sdesc(smem_u32(sA) + (kk / 4) * (M * 128) + (kk % 4) * 32, 16, 1024, kSwz128);
            if (B_MN) {
                if (N == 32) bd = make_sdesc(smem_u32(sB) + kk * 1024, K * 64, 512, kSwz64);
                else bd = make_sdesc(smem_u32(sB) + kk * 2048, K * 128, 1024, kSwz128);
            } else {
                bd = make_sdesc(smem_u32(sB) + (kk / 4) * (N * 128) + (kk % 4) * 32, 16, 1024, kSwz128);
            }
            mma_f16(tmem, ad, bd, idesc, kk > 0);
        }
        mma_commit(&bar);
    }
    __syncwarp();
    mbar_wait(&bar, 0, &abort_flag);
    tc_fence_after();

    const int lane = tid % 32;
    int row;
    bool valid;
    if (M == 128) { row = warp * 32 + lane; valid = true; }
    else { row = warp * 16 + lane; valid = lane < 16; }
    for (int c0 = 0; c0 < N; c0 += 16) {
        float r[16];
        tmem_ld16(tmem + tmem_lane_base(warp) + c0, r);
        tmem_ld_wait();
        if (valid)
            for (int j = 0; j < 16; ++j) D[row * N + c0 + j] = r[j];
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 512);
}

// A operand in TMEM: thread m writes row m of A (K bf16, two per 32-bit column) with tcgen05.st,
// B [N][K] (K-major) in shared memory; D = A * B^T read back as above.  M = 128.
template <int N, int K>
__global__ void __launch_bounds__(128) probe_tmem_a_kernel(const __nv_bfloat16 *A, const __nv_bfloat16 *B, float *D) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sB = smem;
    __shared__ uint64_t bar;
    __shared__ uint32_t tbase;
    __shared__ int abort_flag;
    const int tid = threadIdx.x, warp = tid / 32;
    constexpr int M = 128;
    for (int i = tid; i < N * K; i += 128) {
        int n = i / K, k = i % K;
        *reinterpret_cast<__nv_bfloat16 *>(sB + tile_off(n, k, N, K)) = B[i];
    }
    if (tid == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
        abort_flag = 0;
    }
    if (warp == 0) {
        tmem_alloc(&tbase, 512);
        tmem_relinquish();
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tbase;
    constexpr uint32_t kAcol = 256;   // A operand columns [256, 256 + K/2)
    {
        const uint32_t *arow = reinterpret_cast<const uint32_t *>(A + tid * K);  // row m = tid
        for (int c0 = 0; c0 < K / 2; c0 += 16) {
            uint32_t u[16];
            for (int j = 0; j < 16; ++j) u[j] = arow[c0 + j];
            tmem_st16(tmem + tmem_lane_base(warp) + kAcol + c0, u);
        }
        tmem_st_wait();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid == 0) {
        constexpr uint32_t idesc = make_idesc_bf16(M, N, false, false);
        for (int kk = 0; kk < K / 16; ++kk) {
            uint64_t bd = make_sdesc(smem_u32(sB) + (kk / 4) * (N * 128) + (kk % 4) * 32, 16, 1024, kSwz128);
            mma_f16_ta(tmem, tmem + kAcol + kk * 8, bd, idesc, kk > 0);
        }
        mma_commit(&bar);
    }
    __syncwarp();
    mbar_wait(&bar, 0, &abort_flag);
    tc_fence_after();
    const int row = warp * 32 + (tid % 32);
    for (int c0 = 0; c0 < N; c0 += 16) {
        float r[16];
        tmem_ld16(tmem + tmem_lane_base(warp) + c0, r);
        tmem_ld_wait();
        for (int j = 0; j < 16; ++j) D[row * N + c0 + j] = r[j];
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 512);
}

template <int N, int K>
static int launch_tmem_a(const void *A, const void *B, void *D) {
    size_t smem = N * K * 2 + 1024;
    auto kern = probe_tmem_a_kernel<N, K>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess) return 1;
    kern<<<1, 128, smem>>>((const __nv_bfloat16 *)A, (const __nv_bfloat16 *)B, (float *)D);
    return cudaGetLastError() == cudaSuccess ? 0 : 2;
}

template <int M, int N, int K, bool A_MN, bool B_MN>
static int launch(const void *A, const void *B, void *D) {
    size_t smem = ((M * K * 2 + 1023) / 1024) * 1024 + N * K * 2 + 1024;
    auto kern = probe_kernel<M, N, K, A_MN, B_MN>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess) return 1;
    kern<<<1, 128, smem>>>((const __nv_bfloat16 *)A, (const __nv_bfloat16 *)B, (float *)D);
    return cudaGetLastError() == cudaSuccess ? 0 : 2;
}

// case ids: see tests/test_gpu_tc_probe.py
extern "C" int tc_probe_run(int case_id, const void *A, const void *B, void *D) {
    switch (case_id) {
        case 0: return launch<64, 64, 128, false, false>(A, B, D);   // A_raw = Kr' Kn'^T
        case 1: return launch<64, 128, 64, false, true>(A, B, D);    // W = (T b) Kg
        case 2: return launch<128, 64, 64, true, true>(A, B, D);     // S += Kd^T U~ (NV = 64)
        case 3: return launch<64, 64, 128, false, true>(A, B, D);    // U~ = U - W S (NV = 64)
        case 4: return launch<64, 32, 128, false, true>(A, B, D);    // NV = 32, SW64 B
        case 5: return launch<128, 32, 64, true, true>(A, B, D);     // NV = 32, SW64 B
        case 6: return launch<128, 128, 64, true, true>(A, B, D);    // NV = 128
        case 7: return launch<64, 128, 128, false, true>(A, B, D);   // NV = 128
        case 8: return launch_tmem_a<64, 64>(A, B, D);               // A in TMEM, K-major B
        case 9: return launch_tmem_a<128, 128>(A, B, D);
        default: return 3;
    }
}
