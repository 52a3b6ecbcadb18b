// The FP8 path (next step on the path): Q and K per block in e4m3 for the Q.K^T
// tensor-core products, K smoothed first.
//
// The pages feed the sparse mask into an FP8 attention in the style of SageAttention2
// (page "知识卡片：600倍加速，720p视频实时生成！单卡也能带的动14B模型", 方法/产品要点, bullet
// 动态稀疏量化注意力; page "单卡 RTX 5090 跑 Wan2.2-A14B：720p 视频生成只要 3.8 秒", 四步拆解
// item 3) and give no quantization detail.  What is built:
//   key_mean_kernel : the sequence mean of K per (b, h) and channel, from the block
//                     means (weights = valid tokens per block).
//   quantize_kernel : per (tensor, b, h, block): y = x - smooth (K only; the smoothing
//                     vector is normally the key mean, which leaves softmax unchanged),
//                     amax over the block's valid tokens, inv = 448 / amax and
//                     scale = amax / 448 in fp32, code = e4m3(y * inv) rounded to nearest
//                     even and saturated at +-448; padded tokens get code 0.  The code
//                     decisions are these fp32 operations, in this order.
// The attention on the codes is attn_kernel's FP8 form (attn.cuh).
#pragma once
#include "common.cuh"
#include "pool.cuh"
#include "ptx.cuh"
#include "rope.cuh"

namespace sbsa {

// mean[bh][c] = sum_i n_i * block_mean[bh][i][c] / L.  One CTA per (b, h), one thread
// per channel.
__global__ void key_mean_kernel(const float* __restrict__ k_mean, float* __restrict__ out, int d, int nb, int blk,
                                int L) {
    const long long bh = blockIdx.x;
    const int c = threadIdx.x;
    if (c >= d) return;
    const float* m = k_mean + bh * nb * d + c;
    float s = 0.f;
    for (int i = 0; i < nb; ++i) s += static_cast<float>(min(blk, L - i * blk)) * m[static_cast<long long>(i) * d];
    out[bh * d + c] = s / static_cast<float>(L);
}

// Two floats -> two e4m3 codes (lo in the low byte), nearest even, saturating.
__device__ __forceinline__ uint16_t cvt_e4m3x2(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// One CTA per (tensor, b, h, block), 256 threads.  The block's bf16 tile comes into
// shared memory with one bulk copy; thread t owns the 16-byte chunk t % (d/8) of rows
// t / (d/8), t / (d/8) + 256/(d/8), ...: a pass for the block's amax, a pass for the
// codes, 8 codes (8 bytes) stored per chunk.
template <int D, int BLK>
__global__ void __launch_bounds__(256) quantize_kernel(const uint4* __restrict__ q, const uint4* __restrict__ k,
                                                       const float* __restrict__ k_smooth,
                                                       uint2* __restrict__ q8, uint2* __restrict__ k8,
                                                       float* __restrict__ q_scale, float* __restrict__ k_scale,
                                                       int L, int Lp, int nb, long long units_per_tensor,
                                                       unsigned int epoch) {
    constexpr int CH = D / 8;
    constexpr int RG = 256 / CH;
    constexpr int ITER = BLK / RG;
    constexpr uint32_t kTileBytes = BLK * D * 2;
    static_assert(BLK % RG == 0, "block must be a multiple of the row-group count");
    __shared__ __align__(128) uint4 tile[BLK * CH];
    __shared__ float red[8];
    __shared__ __align__(8) uint64_t full;

    long long u = blockIdx.x;
    const bool is_k = u >= units_per_tensor;
    if (is_k) u -= units_per_tensor;
    const long long bh = u / nb;
    const int t0 = static_cast<int>(u % nb) * BLK;
    const int nvalid = min(BLK, L - t0);
    const long long base = (static_cast<long long>(bh) * Lp + t0) * CH;

    if (threadIdx.x == 0) {
        mbar_init(&full, 1);
        fence_mbar_init();
        mbar_arrive_expect_tx(&full, kTileBytes);
        bulk_load_g2s(tile, (is_k ? k : q) + base, kTileBytes, &full);
    }
    const int c = threadIdx.x % CH;
    const int g = threadIdx.x / CH;
    float sm[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) sm[e] = (is_k && k_smooth) ? __ldg(k_smooth + bh * D + 8 * c + e) : 0.f;
    __syncthreads();  // the barrier is initialised before anyone waits on it
    volatile int never = 0;
    // every thread takes the same branch (the later __syncthreads need all of them), so
    // the CTA gives up if any thread's wait ran out
    const bool landed = mbar_wait_bounded(&full, 0, &never, pipe_wait_ns());
    if (__syncthreads_or(landed ? 0 : 1)) {
        if (threadIdx.x == 0) abort_launch(epoch);
        // the copy gets one more bounded wait to land before the shared memory is released
        mbar_wait_bounded(&full, 0, &never, kWaitLimitNs);
        return;
    }
    auto smoothed = [&](int r, float (&y)[8]) {
        const uint4 w = tile[r * CH + c];
        const uint32_t in[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            y[2 * j] = __uint_as_float(in[j] << 16) - sm[2 * j];
            y[2 * j + 1] = __uint_as_float(in[j] & 0xFFFF0000u) - sm[2 * j + 1];
        }
    };
    // block amax over the valid rows
    float amax = 0.f;
#pragma unroll
    for (int it = 0; it < ITER; ++it) {
        const int r = g + it * RG;
        if (r < nvalid) {
            float y[8];
            smoothed(r, y);
#pragma unroll
            for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(y[e]));
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, off));
    if (threadIdx.x % 32 == 0) red[threadIdx.x / 32] = amax;
    __syncthreads();
    amax = red[0];
#pragma unroll
    for (int w = 1; w < 8; ++w) amax = fmaxf(amax, red[w]);
    const float inv = amax > 0.f ? 448.f / amax : 1.f;
    if (threadIdx.x == 0) (is_k ? k_scale : q_scale)[u] = amax > 0.f ? amax / 448.f : 1.f;
    uint2* dst = (is_k ? k8 : q8) + base;  // 8 codes per 16-byte bf16 chunk
#pragma unroll
    for (int it = 0; it < ITER; ++it) {
        const int r = g + it * RG;
        uint2 out = make_uint2(0u, 0u);
        if (r < nvalid) {
            float y[8];
            smoothed(r, y);
            out.x = cvt_e4m3x2(y[0] * inv, y[1] * inv) | (static_cast<uint32_t>(cvt_e4m3x2(y[2] * inv, y[3] * inv)) << 16);
            out.y = cvt_e4m3x2(y[4] * inv, y[5] * inv) | (static_cast<uint32_t>(cvt_e4m3x2(y[6] * inv, y[7] * inv)) << 16);
        }
        dst[static_cast<long long>(r) * CH + c] = out;
    }
}

}  // namespace sbsa
