// Step 1: block means of Q and K.
//
// Block-level means of Query and Key are the importance estimate of the method (page
// "知识卡片：600倍加速，720p视频实时生成！单卡也能带的动14B模型", 方法/产品要点, bullet
// 动态稀疏量化注意力).  mean[b,h,i,:] = (1/n_i) * sum over the n_i valid tokens t of
// block i of X[b,h,t,:].
//
// HBM-bandwidth bound: every byte of Q and K is read exactly once with 128-bit
// non-coherent loads that skip L1 allocation, and each CTA writes one
// d-wide fp32 row.  One CTA per (tensor, b, h, block); 256 threads; thread t owns the
// 16-byte column chunk t % (d/8) of rows t / (d/8), t / (d/8) + 256/(d/8), ...  All of
// a thread's loads are issued before any is consumed, so 8 x 16 B are in flight per
// thread at block 128.
#pragma once
#include "common.cuh"

namespace sbsa {

__device__ __forceinline__ uint4 ld_stream_v4(const uint4* p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

__device__ __forceinline__ void acc_bf16x8(float (&a)[8], const uint4& w) {
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        a[2 * i] += __uint_as_float(u[i] << 16);
        a[2 * i + 1] += __uint_as_float(u[i] & 0xFFFF0000u);
    }
}

template <int D, int BLK>
__global__ void __launch_bounds__(256) pool_kernel(const uint4* __restrict__ q, const uint4* __restrict__ k,
                                                   float* __restrict__ q_mean, float* __restrict__ k_mean, int L,
                                                   int Lp, int nb, long long units_per_tensor) {
    constexpr int CH = D / 8;          // 16-byte chunks per row
    constexpr int RG = 256 / CH;       // row groups
    constexpr int ITER = BLK / RG;     // rows per thread
    static_assert(BLK % RG == 0, "block must be a multiple of the row-group count");
    __shared__ float red[8][D];

    long long u = blockIdx.x;
    const bool is_k = u >= units_per_tensor;
    if (is_k) u -= units_per_tensor;
    const long long bh = u / nb;
    const int i = static_cast<int>(u % nb);
    const int t0 = i * BLK;
    const int nvalid = min(BLK, L - t0);

    const uint4* src = (is_k ? k : q) + (static_cast<long long>(bh) * Lp + t0) * CH;
    const int c = threadIdx.x % CH;
    const int g = threadIdx.x / CH;

    uint4 w[ITER];
#pragma unroll
    for (int it = 0; it < ITER; ++it) {
        const int r = g + it * RG;
        w[it] = r < nvalid ? ld_stream_v4(src + static_cast<long long>(r) * CH + c) : make_uint4(0, 0, 0, 0);
    }
    float a[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll
    for (int it = 0; it < ITER; ++it) acc_bf16x8(a, w[it]);

    // lanes that share a column chunk: lane ^ CH, lane ^ 2CH, ... within the warp
#pragma unroll
    for (int off = CH; off < 32; off <<= 1)
#pragma unroll
        for (int e = 0; e < 8; ++e) a[e] += __shfl_xor_sync(0xFFFFFFFFu, a[e], off);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    if (lane < CH) {
#pragma unroll
        for (int e = 0; e < 8; ++e) red[warp][lane * 8 + e] = a[e];
    }
    __syncthreads();
    if (threadIdx.x < D) {
        float s = 0.f;
#pragma unroll
        for (int wi = 0; wi < 8; ++wi) s += red[wi][threadIdx.x];
        float* dst = (is_k ? k_mean : q_mean) + u * D;
        dst[threadIdx.x] = s / static_cast<float>(nvalid);
    }
}

}  // namespace sbsa
