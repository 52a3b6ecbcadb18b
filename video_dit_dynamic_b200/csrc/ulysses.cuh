// Light-Ulysses sequence parallelism (page "知识卡片：600倍加速，720p视频实时生成！单卡也能带
// 的动14B模型", 方法/产品要点, bullet Light-Ulysses 多卡并行; page "单卡 RTX 5090 跑
// Wan2.2-A14B：720p 视频生成只要 3.8 秒", 四步拆解 item 4): the pre- and post-processing
// around the two all-to-alls of Ulysses-style attention, with an FP8 payload and Q, K, V
// fused into one exchange.
//
// G ranks; rank r holds tokens [r L/G, (r+1) L/G) before the attention and heads
// [r H/G, (r+1) H/G) during it.  A pipeline chunk covers heads h0 .. h0 + hc - 1 of every
// rank's H/G (the head-level pipeline exchanges one chunk while another is attended).
// Every row of d = 128 values crosses as 128 e4m3 codes and one fp32 scale:
//   scale = amax / 448, code = e4m3(x * (448 / amax)) in fp32, nearest even, saturating;
//   an all-zero row has scale 1 and codes 0;  restored value = bf16(code * scale).
//
// Buffers (one chunk, bytes), one slice per peer, slices in rank order, each slice its
// codes followed by its scales:
//   QKV slice for peer j: codes [L/G][3][hc][d], scales [L/G][3][hc]
//   O   slice for peer j: codes [L/G][hc][d],    scales [L/G][hc]
// Layouts around them:
//   x  (fused QKV activation of this rank's tokens)  [L/G][3][H][d] bf16
//   q, k, v (this rank's heads, attention layout)    [H/G][Lp][d] bf16, tokens >= L zero
//   o  (attention output of this rank's heads)       [H/G][Lp][d] bf16
//   y  (all heads of this rank's tokens)             [L/G][H][d] bf16
#pragma once
#include <cuda_bf16.h>

#include "common.cuh"
#include "fp8.cuh"
#include "ptx.cuh"

namespace sbsa {

struct UlyssesDims {
    int G, Lr, L, Lp, H, Hg, h0, hc;
};

// e4m3 code -> exact fp32 value (sign, bias 7, three mantissa bits, subnormals m 2^-9)
__device__ __forceinline__ float e4m3_signed_value(uint32_t code) {
    const uint32_t e = (code >> 3) & 15u, m = code & 7u;
    const float v = e ? __uint_as_float(((e + 120u) << 23) | (m << 20)) : static_cast<float>(m) * 0.001953125f;
    return (code & 0x80u) ? -v : v;
}

// One warp quantizes one row of 128 bf16 values (4 per lane) into 128 codes (4 bytes per
// lane) and one scale (lane 0).
__device__ __forceinline__ void quantize_row_warp(const uint2* __restrict__ src, uint32_t* __restrict__ codes,
                                                  float* __restrict__ scale, int lane) {
    const uint2 w = src[lane];
    float v[4] = {__uint_as_float(w.x << 16), __uint_as_float(w.x & 0xFFFF0000u), __uint_as_float(w.y << 16),
                  __uint_as_float(w.y & 0xFFFF0000u)};
    float amax = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, off));
    const float inv = amax > 0.f ? __fdiv_rn(448.f, amax) : 1.f;
    const uint32_t lo = cvt_e4m3x2(__fmul_rn(v[0], inv), __fmul_rn(v[1], inv));
    const uint32_t hi = cvt_e4m3x2(__fmul_rn(v[2], inv), __fmul_rn(v[3], inv));
    codes[lane] = lo | (hi << 16);
    if (lane == 0) *scale = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
}

// One warp restores one row: 4 codes per lane -> 4 bf16 values.
__device__ __forceinline__ void dequantize_row_warp(const uint32_t* __restrict__ codes, const float* __restrict__ scale,
                                                    uint2* __restrict__ dst, int lane) {
    const uint32_t c = codes[lane];
    const float s = *scale;
    const float v0 = __fmul_rn(e4m3_signed_value(c & 0xFFu), s);
    const float v1 = __fmul_rn(e4m3_signed_value((c >> 8) & 0xFFu), s);
    const float v2 = __fmul_rn(e4m3_signed_value((c >> 16) & 0xFFu), s);
    const float v3 = __fmul_rn(e4m3_signed_value(c >> 24), s);
    dst[lane] = make_uint2(pack_bf16x2(v0, v1), pack_bf16x2(v2, v3));
}

constexpr int kUlyD = 128;          // head_dim handled by these kernels
constexpr int kUlyWarps = 8;        // rows per 256-thread CTA

__host__ __device__ constexpr size_t ulysses_qkv_slice_bytes(const UlyssesDims& u) {
    return static_cast<size_t>(u.Lr) * 3 * u.hc * (kUlyD + 4);
}
__host__ __device__ constexpr size_t ulysses_o_slice_bytes(const UlyssesDims& u) {
    return static_cast<size_t>(u.Lr) * u.hc * (kUlyD + 4);
}

// x [Lr][3][H][d] -> send: slice j holds rows (t, c, hh) of head j Hg + h0 + hh.
__global__ void __launch_bounds__(256) ulysses_pack_qkv_kernel(const __nv_bfloat16* __restrict__ x,
                                                               uint8_t* __restrict__ send, UlyssesDims u) {
    const int lane = threadIdx.x % 32;
    const long long w = blockIdx.x * static_cast<long long>(kUlyWarps) + threadIdx.x / 32;
    const long long per_peer = static_cast<long long>(u.Lr) * 3 * u.hc;
    if (w >= per_peer * u.G) return;
    const int j = static_cast<int>(w / per_peer);
    const long long row = w % per_peer;  // (t * 3 + c) * hc + hh
    const int hh = static_cast<int>(row % u.hc);
    const long long tc = row / u.hc;     // t * 3 + c
    const int h = j * u.Hg + u.h0 + hh;
    const uint2* src = reinterpret_cast<const uint2*>(x + (tc * u.H + h) * kUlyD);
    uint8_t* slice = send + static_cast<size_t>(j) * ulysses_qkv_slice_bytes(u);
    quantize_row_warp(src, reinterpret_cast<uint32_t*>(slice + row * kUlyD),
                      reinterpret_cast<float*>(slice + per_peer * kUlyD) + row, lane);
}

// recv (slice i from rank i) -> q, k, v [Hg][Lp][d]: row (t, c, hh) is token i Lr + t of
// head h0 + hh of tensor c.  Warps past the received rows zero the padded tokens
// [L, Lp) of the chunk's heads.
__global__ void __launch_bounds__(256) ulysses_unpack_qkv_kernel(const uint8_t* __restrict__ recv,
                                                                 __nv_bfloat16* __restrict__ q,
                                                                 __nv_bfloat16* __restrict__ k,
                                                                 __nv_bfloat16* __restrict__ v, UlyssesDims u) {
    const int lane = threadIdx.x % 32;
    const long long w = blockIdx.x * static_cast<long long>(kUlyWarps) + threadIdx.x / 32;
    const long long per_peer = static_cast<long long>(u.Lr) * 3 * u.hc;
    const long long n_rows = per_peer * u.G;
    if (w < n_rows) {
        const int i = static_cast<int>(w / per_peer);
        const long long row = w % per_peer;
        const int hh = static_cast<int>(row % u.hc);
        const long long tc = row / u.hc;
        const int c = static_cast<int>(tc % 3);
        const long long t = tc / 3;
        __nv_bfloat16* dst_t = c == 0 ? q : (c == 1 ? k : v);
        const long long token = static_cast<long long>(i) * u.Lr + t;
        const uint8_t* slice = recv + static_cast<size_t>(i) * ulysses_qkv_slice_bytes(u);
        dequantize_row_warp(reinterpret_cast<const uint32_t*>(slice + row * kUlyD),
                            reinterpret_cast<const float*>(slice + per_peer * kUlyD) + row,
                            reinterpret_cast<uint2*>(dst_t + (static_cast<long long>(u.h0 + hh) * u.Lp + token) * kUlyD),
                            lane);
        return;
    }
    const long long z = w - n_rows;  // padded rows: (c, hh, t - L)
    const long long pad = u.Lp - u.L;
    if (z >= 3 * u.hc * pad) return;
    const int c = static_cast<int>(z / (u.hc * pad));
    const long long rem = z % (u.hc * pad);
    const int hh = static_cast<int>(rem / pad);
    const long long token = u.L + rem % pad;
    __nv_bfloat16* dst_t = c == 0 ? q : (c == 1 ? k : v);
    reinterpret_cast<uint2*>(dst_t + (static_cast<long long>(u.h0 + hh) * u.Lp + token) * kUlyD)[lane] =
        make_uint2(0u, 0u);
}

// o [Hg][Lp][d] -> send: slice j holds rows (t, hh) of token j Lr + t, head h0 + hh.
__global__ void __launch_bounds__(256) ulysses_pack_o_kernel(const __nv_bfloat16* __restrict__ o,
                                                             uint8_t* __restrict__ send, UlyssesDims u) {
    const int lane = threadIdx.x % 32;
    const long long w = blockIdx.x * static_cast<long long>(kUlyWarps) + threadIdx.x / 32;
    const long long per_peer = static_cast<long long>(u.Lr) * u.hc;
    if (w >= per_peer * u.G) return;
    const int j = static_cast<int>(w / per_peer);
    const long long row = w % per_peer;  // t * hc + hh
    const int hh = static_cast<int>(row % u.hc);
    const long long t = row / u.hc;
    const long long token = static_cast<long long>(j) * u.Lr + t;
    const uint2* src = reinterpret_cast<const uint2*>(o + (static_cast<long long>(u.h0 + hh) * u.Lp + token) * kUlyD);
    uint8_t* slice = send + static_cast<size_t>(j) * ulysses_o_slice_bytes(u);
    quantize_row_warp(src, reinterpret_cast<uint32_t*>(slice + row * kUlyD),
                      reinterpret_cast<float*>(slice + per_peer * kUlyD) + row, lane);
}

// recv (slice i from rank i) -> y [Lr][H][d]: row (t, hh) is head i Hg + h0 + hh of
// token t.
__global__ void __launch_bounds__(256) ulysses_unpack_o_kernel(const uint8_t* __restrict__ recv,
                                                               __nv_bfloat16* __restrict__ y, UlyssesDims u) {
    const int lane = threadIdx.x % 32;
    const long long w = blockIdx.x * static_cast<long long>(kUlyWarps) + threadIdx.x / 32;
    const long long per_peer = static_cast<long long>(u.Lr) * u.hc;
    if (w >= per_peer * u.G) return;
    const int i = static_cast<int>(w / per_peer);
    const long long row = w % per_peer;
    const int hh = static_cast<int>(row % u.hc);
    const long long t = row / u.hc;
    const uint8_t* slice = recv + static_cast<size_t>(i) * ulysses_o_slice_bytes(u);
    dequantize_row_warp(reinterpret_cast<const uint32_t*>(slice + row * kUlyD),
                        reinterpret_cast<const float*>(slice + per_peer * kUlyD) + row,
                        reinterpret_cast<uint2*>(y + (t * u.H + i * u.Hg + u.h0 + hh) * kUlyD), lane);
}

}  // namespace sbsa
