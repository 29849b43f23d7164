// Layout probe for the tcgen05 building blocks used by the chunked scan:
// one CTA computes D[m][n] = sum_k A[m][k] B[n][k] with a single sequence of
// MMAs, the operands written into shared memory in the requested layout,
// and copies the TMEM accumulator back to global memory.  Every index is
// bounded by M <= 128, N <= 64, K <= 64 (tiles of at most 16 KB).
#include "../../selective_diagonal_state_b200/csrc/umma.cuh"
#include <cuda_bf16.h>

using namespace ssm::umma;

// layout codes: 0 = K-major no swizzle, 1 = MN-major no swizzle,
//               2 = MN-major 128-byte swizzle (64-element rows along MN, rows = K)
//               3 = K-major 128-byte swizzle (64-element rows along K, rows = MN)
__device__ uint32_t place(int code, int mn, int k, int MN, int K) {
    if (code == 0) return off_kmaj(mn, k, 128u, (uint32_t)(K / 8) * 128u);
    if (code == 1) return off_mnmaj(mn, k, (uint32_t)(MN / 8) * 128u, 128u);
    if (code == 3) return off_sw128(mn, k);
    return off_sw128(k, mn);
}
__device__ uint64_t desc_for(int code, uint32_t base, int step, int MN, int K) {
    if (code == 0) return sdesc(base + step * 256u, 128u, (uint32_t)(K / 8) * 128u, LAYOUT_NONE);
    if (code == 1) {
        uint32_t lbo = (uint32_t)(MN / 8) * 128u;
        return sdesc(base + step * 2u * lbo, lbo, 128u, LAYOUT_NONE);
    }
    if (code == 3) return sdesc(base + step * 32u, 16u, 1024u, LAYOUT_SW128);
    return sdesc(base + step * 2048u, 8192u, 1024u, LAYOUT_SW128);
}

extern "C" __global__ void __launch_bounds__(128)
umma_probe(int M, int N, int K, int a_code, int b_code, int d_lane, const float *A,
           const float *B, float *D, int *status) {
    __shared__ __align__(1024) unsigned char sA[16384];
    __shared__ __align__(1024) unsigned char sB[16384];
    __shared__ __align__(8) uint64_t bar;
    __shared__ uint32_t tslot;
    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    for (int i = tid; i < 16384 / 2; i += 128) {
        reinterpret_cast<__nv_bfloat16 *>(sA)[i] = __float2bfloat16(0.f);
        reinterpret_cast<__nv_bfloat16 *>(sB)[i] = __float2bfloat16(0.f);
    }
    __syncthreads();
    for (int i = tid; i < M * K; i += 128) {
        int m = i / K, k = i % K;
        *reinterpret_cast<__nv_bfloat16 *>(sA + place(a_code, m, k, M, K)) = __float2bfloat16(A[i]);
    }
    for (int i = tid; i < N * K; i += 128) {
        int n = i / K, k = i % K;
        *reinterpret_cast<__nv_bfloat16 *>(sB + place(b_code, n, k, N, K)) = __float2bfloat16(B[i]);
    }
    if (warp == 0) tmem_alloc(&tslot, 64);
    if (tid == 0) {
        mbar_init(&bar, 1);
        mbar_fence_init();
    }
    fence_proxy_async();
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tbase = tslot;
    if (tid == 0) {
        const uint32_t id = idesc_bf16(M, N, a_code == 1 || a_code == 2, b_code == 1 || b_code == 2);
        for (int s = 0; s < K / 16; ++s)
            mma_bf16(tmem_addr(tbase, (uint32_t)d_lane, 0), desc_for(a_code, smem_u32(sA), s, M, K),
                     desc_for(b_code, smem_u32(sB), s, N, K), id, s > 0);
        mma_commit(&bar);
    }
    bool ok = mbar_wait(&bar, 0, 1u << 24);
    fence_after_sync();
    if (!ok) {
        if (lane == 0) atomicExch(status, 1);
    } else {
        for (int c = 0; c < N; c += 16) {
            float v[16];
            tmem_ld16(tmem_addr(tbase, 32u * warp, (uint32_t)c), v);
            int row;
            if (M == 128) {
                row = 32 * warp + lane;
            } else {  // M = 64: rows 16w..16w+15 in lanes 32w + d_lane + (0..15)
                int l = lane - d_lane;
                row = (l >= 0 && l < 16) ? 16 * warp + l : -1;
            }
            if (row >= 0)
                for (int j = 0; j < 16; ++j) D[row * N + c + j] = v[j];
        }
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tbase, 64);
}
