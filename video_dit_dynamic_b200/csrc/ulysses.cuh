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
// codes followed by its scales and padded to a multiple of 16 bytes:
//   QKV slice for peer j: codes [L/G][3][hc][d], scales [L/G][3][hc]
//   O   slice for peer j: codes [L/G][hc][d],    scales [L/G][hc]
// Two exchanges are supported: the caller's all-to-all of the send buffers (NCCL), or
// peer puts, where each rank's kernel writes every peer's slice straight into that peer's
// receive buffer (peer-mapped memory over NVLink) and then raises a flag in each peer
// (system-scope release); the receiver waits on its flags (system-scope acquire, bounded)
// before it unpacks.  The receive layout is the same in both.
// Layouts around them:
//   x  (fused QKV activation of this rank's tokens)  [L/G][3][H][d] bf16
//   q, k, v (this rank's heads, attention layout)    [H/G][Lp][d] bf16, tokens >= L zero
//   o  (attention output of this rank's heads)       [H/G][Lp][d] bf16
//   y  (all heads of this rank's tokens)             [L/G][H][d] bf16
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "common.cuh"
#include "fp8.cuh"
#include "ptx.cuh"

namespace sbsa {

// Division of n < 2^31 by an invariant d >= 1 with one 64-bit multiply and a shift
// (Granlund and Montgomery, "Division by invariant integers using multiplication", 1994,
// theorem 4.2 with N = 31): l = ceil(log2 d), s = 31 + l, m = floor(2^s / d) + 1; then
// 2^s < m d <= 2^s + 2^l and floor(n / d) = floor(n m / 2^s) for every n < 2^31.
struct FastDiv {
    unsigned long long m;
    unsigned int s;
};
inline FastDiv make_fastdiv(uint32_t d) {
    unsigned int l = 0;
    while ((1ull << l) < d) ++l;
    const unsigned int s = 31 + l;
    return {(1ull << s) / d + 1, s};
}
__device__ __forceinline__ uint32_t udiv(uint32_t n, const FastDiv& f) {
    return static_cast<uint32_t>((static_cast<unsigned long long>(n) * f.m) >> f.s);
}

struct UlyssesDims {
    int G, Lr, L, Lp, H, Hg, h0, hc;
    // divisors of the row decompositions: rows per peer of a QKV and of an O exchange,
    // the chunk's heads, the padded tokens, and hc times the padded tokens
    FastDiv by_qkv_peer, by_o_peer, by_hc, by_pad, by_pad_hc;
};

// Two e4m3 codes (low byte first) -> their exact values as fp32 (e4m3 is a subset of
// f16, so the hardware conversion to f16 is exact).
__device__ __forceinline__ float2 e4m3x2_to_float2(uint32_t two_codes) {
    uint32_t h2;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(static_cast<uint16_t>(two_codes & 0xFFFFu)));
    return __half22float2(*reinterpret_cast<const __half2*>(&h2));
}

constexpr int kUlyD = 128;          // head_dim handled by these kernels
constexpr int kUlyRowsPerWarp = 16;  // 8 lanes per row (16 values each), 4 rows per step, 4 steps
constexpr int kUlyRowsPerCta = 8 * kUlyRowsPerWarp;

// slices are padded to 16 bytes, so every slice's codes start 16-byte aligned
__host__ __device__ constexpr size_t ulysses_qkv_slice_bytes(const UlyssesDims& u) {
    return (static_cast<size_t>(u.Lr) * 3 * u.hc * (kUlyD + 4) + 15) & ~size_t(15);
}
__host__ __device__ constexpr size_t ulysses_o_slice_bytes(const UlyssesDims& u) {
    return (static_cast<size_t>(u.Lr) * u.hc * (kUlyD + 4) + 15) & ~size_t(15);
}

// Where row `row` of a pack goes and comes from.
struct RowPtrs {
    const uint4* src;  // 8 bf16 per lane (pack) or 8 codes per lane (unpack, as uint2)
    void* dst;
    float* scale;
    bool zero;         // unpack only: a padded token, written as zeros
};

// Row decompositions use 32-bit unsigned arithmetic: the host refuses chunks of 2^31
// rows or more.  Offsets are formed in 64 bits.
__device__ __forceinline__ RowPtrs qkv_pack_row(uint32_t w, const __nv_bfloat16* x, uint8_t* send,
                                                const UlyssesDims& u) {
    const uint32_t per_peer = static_cast<uint32_t>(u.Lr) * 3u * static_cast<uint32_t>(u.hc);
    const uint32_t j = udiv(w, u.by_qkv_peer);
    const uint32_t row = w - j * per_peer;  // (t * 3 + c) * hc + hh
    const uint32_t tc = udiv(row, u.by_hc);
    const uint32_t hh = row - tc * static_cast<uint32_t>(u.hc);
    uint8_t* slice = send + static_cast<size_t>(j) * ulysses_qkv_slice_bytes(u);
    const size_t src = (static_cast<size_t>(tc) * u.H + j * u.Hg + u.h0 + hh) * kUlyD;
    return {reinterpret_cast<const uint4*>(x + src), slice + static_cast<size_t>(row) * kUlyD,
            reinterpret_cast<float*>(slice + static_cast<size_t>(per_peer) * kUlyD) + row, false};
}

__device__ __forceinline__ RowPtrs o_pack_row(uint32_t w, const __nv_bfloat16* o, uint8_t* send,
                                              const UlyssesDims& u) {
    const uint32_t per_peer = static_cast<uint32_t>(u.Lr) * static_cast<uint32_t>(u.hc);
    const uint32_t j = udiv(w, u.by_o_peer);
    const uint32_t row = w - j * per_peer;  // t * hc + hh
    const uint32_t t = udiv(row, u.by_hc);
    const uint32_t hh = row - t * static_cast<uint32_t>(u.hc);
    const size_t token = static_cast<size_t>(j) * u.Lr + t;
    uint8_t* slice = send + static_cast<size_t>(j) * ulysses_o_slice_bytes(u);
    return {reinterpret_cast<const uint4*>(o + (static_cast<size_t>(u.h0 + hh) * u.Lp + token) * kUlyD),
            slice + static_cast<size_t>(row) * kUlyD,
            reinterpret_cast<float*>(slice + static_cast<size_t>(per_peer) * kUlyD) + row, false};
}

// Peer puts: slice j of this rank goes to peer j's receive buffer, at offset
// recv_offset + rank * slice bytes of peer j's exchange allocation.
struct PeerDst {
    const unsigned long long* bases;  // device array of the world's allocation base addresses
    unsigned long long recv_offset;   // byte offset of the receive buffer in each allocation
    int rank;
};

__device__ __forceinline__ RowPtrs qkv_put_row(uint32_t w, const __nv_bfloat16* x, const PeerDst& pd,
                                               const UlyssesDims& u) {
    const uint32_t per_peer = static_cast<uint32_t>(u.Lr) * 3u * static_cast<uint32_t>(u.hc);
    const uint32_t j = udiv(w, u.by_qkv_peer);
    const uint32_t row = w - j * per_peer;  // (t * 3 + c) * hc + hh
    const uint32_t tc = udiv(row, u.by_hc);
    const uint32_t hh = row - tc * static_cast<uint32_t>(u.hc);
    uint8_t* slice = reinterpret_cast<uint8_t*>(__ldg(pd.bases + j) + pd.recv_offset) +
                     static_cast<size_t>(pd.rank) * ulysses_qkv_slice_bytes(u);
    const size_t src = (static_cast<size_t>(tc) * u.H + j * u.Hg + u.h0 + hh) * kUlyD;
    return {reinterpret_cast<const uint4*>(x + src), slice + static_cast<size_t>(row) * kUlyD,
            reinterpret_cast<float*>(slice + static_cast<size_t>(per_peer) * kUlyD) + row, false};
}

__device__ __forceinline__ RowPtrs o_put_row(uint32_t w, const __nv_bfloat16* o, const PeerDst& pd,
                                             const UlyssesDims& u) {
    const uint32_t per_peer = static_cast<uint32_t>(u.Lr) * static_cast<uint32_t>(u.hc);
    const uint32_t j = udiv(w, u.by_o_peer);
    const uint32_t row = w - j * per_peer;  // t * hc + hh
    const uint32_t t = udiv(row, u.by_hc);
    const uint32_t hh = row - t * static_cast<uint32_t>(u.hc);
    const size_t token = static_cast<size_t>(j) * u.Lr + t;
    uint8_t* slice = reinterpret_cast<uint8_t*>(__ldg(pd.bases + j) + pd.recv_offset) +
                     static_cast<size_t>(pd.rank) * ulysses_o_slice_bytes(u);
    return {reinterpret_cast<const uint4*>(o + (static_cast<size_t>(u.h0 + hh) * u.Lp + token) * kUlyD),
            slice + static_cast<size_t>(row) * kUlyD,
            reinterpret_cast<float*>(slice + static_cast<size_t>(per_peer) * kUlyD) + row, false};
}

__device__ __forceinline__ RowPtrs qkv_unpack_row(uint32_t w, const uint8_t* recv, __nv_bfloat16* q,
                                                  __nv_bfloat16* k, __nv_bfloat16* v, const UlyssesDims& u) {
    const uint32_t per_peer = static_cast<uint32_t>(u.Lr) * 3u * static_cast<uint32_t>(u.hc);
    const uint32_t n_rows = per_peer * static_cast<uint32_t>(u.G);
    if (w < n_rows) {
        const uint32_t i = udiv(w, u.by_qkv_peer);
        const uint32_t row = w - i * per_peer;
        const uint32_t tc = udiv(row, u.by_hc);
        const uint32_t hh = row - tc * static_cast<uint32_t>(u.hc);
        const uint32_t t3 = tc / 3u;
        const uint32_t c = tc - 3u * t3;
        __nv_bfloat16* t = c == 0 ? q : (c == 1 ? k : v);
        const size_t token = static_cast<size_t>(i) * u.Lr + t3;
        const uint8_t* slice = recv + static_cast<size_t>(i) * ulysses_qkv_slice_bytes(u);
        return {reinterpret_cast<const uint4*>(slice + static_cast<size_t>(row) * kUlyD),
                t + (static_cast<size_t>(u.h0 + hh) * u.Lp + token) * kUlyD,
                const_cast<float*>(reinterpret_cast<const float*>(slice + static_cast<size_t>(per_peer) * kUlyD)) + row,
                false};
    }
    const uint32_t z = w - n_rows;  // padded rows (c, hh, token - L)
    const uint32_t pad = static_cast<uint32_t>(u.Lp - u.L);
    const uint32_t per_c = static_cast<uint32_t>(u.hc) * pad;
    const uint32_t c = udiv(z, u.by_pad_hc);
    const uint32_t rem = z - c * per_c;
    const uint32_t hh = udiv(rem, u.by_pad);
    __nv_bfloat16* t = c == 0 ? q : (c == 1 ? k : v);
    return {nullptr, t + (static_cast<size_t>(u.h0 + hh) * u.Lp + u.L + (rem - hh * pad)) * kUlyD, nullptr, true};
}

__device__ __forceinline__ RowPtrs o_unpack_row(uint32_t w, const uint8_t* recv, __nv_bfloat16* y,
                                                const UlyssesDims& u) {
    const uint32_t per_peer = static_cast<uint32_t>(u.Lr) * static_cast<uint32_t>(u.hc);
    const uint32_t i = udiv(w, u.by_o_peer);
    const uint32_t row = w - i * per_peer;
    const uint32_t t = udiv(row, u.by_hc);
    const uint32_t hh = row - t * static_cast<uint32_t>(u.hc);
    const uint8_t* slice = recv + static_cast<size_t>(i) * ulysses_o_slice_bytes(u);
    return {reinterpret_cast<const uint4*>(slice + static_cast<size_t>(row) * kUlyD),
            y + (static_cast<size_t>(t) * u.H + i * u.Hg + u.h0 + hh) * kUlyD,
            const_cast<float*>(reinterpret_cast<const float*>(slice + static_cast<size_t>(per_peer) * kUlyD)) + row,
            false};
}

// Quantize rows [first, first + 16) of a pack (rows >= n_rows skipped): step s takes
// rows first + 4 s + lane / 8, and lane l = lane % 8 the values 8 l .. + 7 and
// 64 + 8 l .. + 7 of its row, so that every load and store of a warp covers whole
// 32-byte sectors of four rows; all loads are issued before any is used.
template <typename RowFn>
__device__ __forceinline__ void pack_rows(uint32_t first, uint32_t n_rows, RowFn row_of) {
    const int lane = threadIdx.x % 32, h = lane / 8, l = lane % 8;
    uint4 in[4][2];
    RowPtrs rp[4];
#pragma unroll
    for (int s = 0; s < 4; ++s) {
        const uint32_t w = first + 4u * s + h;
        in[s][0] = in[s][1] = make_uint4(0u, 0u, 0u, 0u);
        if (w < n_rows) {
            rp[s] = row_of(w);
            in[s][0] = __ldg(rp[s].src + l);
            in[s][1] = __ldg(rp[s].src + 8 + l);
        }
    }
#pragma unroll
    for (int s = 0; s < 4; ++s) {
        const uint32_t w = first + 4u * s + h;
        const uint32_t wd[8] = {in[s][0].x, in[s][0].y, in[s][0].z, in[s][0].w,
                                in[s][1].x, in[s][1].y, in[s][1].z, in[s][1].w};
        float vals[16];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            vals[2 * e] = __uint_as_float(wd[e] << 16);
            vals[2 * e + 1] = __uint_as_float(wd[e] & 0xFFFF0000u);
        }
        float amax = 0.f;
#pragma unroll
        for (int e = 0; e < 16; ++e) amax = fmaxf(amax, fabsf(vals[e]));
#pragma unroll
        for (int off = 4; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, off));
        if (w >= n_rows) continue;  // (after the shuffles, which every lane takes part in)
        const float inv = amax > 0.f ? __fdiv_rn(448.f, amax) : 1.f;
        uint32_t c2[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) c2[e] = cvt_e4m3x2(__fmul_rn(vals[2 * e], inv), __fmul_rn(vals[2 * e + 1], inv));
        uint2* dst = reinterpret_cast<uint2*>(rp[s].dst);
        dst[l] = make_uint2(c2[0] | (c2[1] << 16), c2[2] | (c2[3] << 16));
        dst[8 + l] = make_uint2(c2[4] | (c2[5] << 16), c2[6] | (c2[7] << 16));
        if (l == 0) *rp[s].scale = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
    }
}

// Restore rows [first, first + 16) (rows >= n_rows skipped), same thread layout.
template <typename RowFn>
__device__ __forceinline__ void unpack_rows(uint32_t first, uint32_t n_rows, RowFn row_of) {
    const int lane = threadIdx.x % 32, h = lane / 8, l = lane % 8;
    uint2 in[4][2];
    float sc[4];
    RowPtrs rp[4];
#pragma unroll
    for (int s = 0; s < 4; ++s) {
        const uint32_t w = first + 4u * s + h;
        if (w < n_rows) {
            rp[s] = row_of(w);
            if (!rp[s].zero) {
                const uint2* src = reinterpret_cast<const uint2*>(rp[s].src);
                in[s][0] = __ldg(src + l);
                in[s][1] = __ldg(src + 8 + l);
                sc[s] = __ldg(rp[s].scale);
            }
        }
    }
#pragma unroll
    for (int s = 0; s < 4; ++s) {
        const uint32_t w = first + 4u * s + h;
        if (w >= n_rows) continue;
        uint4 out[2] = {make_uint4(0u, 0u, 0u, 0u), make_uint4(0u, 0u, 0u, 0u)};
        if (!rp[s].zero) {
            const float k = sc[s];
#pragma unroll
            for (int p = 0; p < 2; ++p) {
                const float2 a = e4m3x2_to_float2(in[s][p].x), b = e4m3x2_to_float2(in[s][p].x >> 16);
                const float2 c = e4m3x2_to_float2(in[s][p].y), d = e4m3x2_to_float2(in[s][p].y >> 16);
                out[p] = make_uint4(pack_bf16x2(__fmul_rn(a.x, k), __fmul_rn(a.y, k)),
                                    pack_bf16x2(__fmul_rn(b.x, k), __fmul_rn(b.y, k)),
                                    pack_bf16x2(__fmul_rn(c.x, k), __fmul_rn(c.y, k)),
                                    pack_bf16x2(__fmul_rn(d.x, k), __fmul_rn(d.y, k)));
            }
        }
        uint4* dst = reinterpret_cast<uint4*>(rp[s].dst);
        dst[l] = out[0];
        dst[8 + l] = out[1];
    }
}

// x [Lr][3][H][d] -> send: slice j holds rows (t, c, hh) of head j Hg + h0 + hh.
__global__ void __launch_bounds__(256) ulysses_pack_qkv_kernel(const __nv_bfloat16* __restrict__ x,
                                                               uint8_t* __restrict__ send, UlyssesDims u) {
    const uint32_t first = blockIdx.x * kUlyRowsPerCta + (threadIdx.x / 32) * kUlyRowsPerWarp;
    const uint32_t n_rows = static_cast<uint32_t>(u.G) * u.Lr * 3u * u.hc;
    pack_rows(first, n_rows, [&](uint32_t w) { return qkv_pack_row(w, x, send, u); });
}

// recv (slice i from rank i) -> q, k, v [Hg][Lp][d]: row (t, c, hh) is token i Lr + t of
// head h0 + hh of tensor c; after those rows come the padded tokens [L, Lp) of the
// chunk's heads, written as zeros.
__global__ void __launch_bounds__(256) ulysses_unpack_qkv_kernel(const uint8_t* __restrict__ recv,
                                                                 __nv_bfloat16* __restrict__ q,
                                                                 __nv_bfloat16* __restrict__ k,
                                                                 __nv_bfloat16* __restrict__ v, UlyssesDims u) {
    const uint32_t first = blockIdx.x * kUlyRowsPerCta + (threadIdx.x / 32) * kUlyRowsPerWarp;
    const uint32_t n_rows = static_cast<uint32_t>(u.G) * u.Lr * 3u * u.hc + 3u * u.hc * (u.Lp - u.L);
    unpack_rows(first, n_rows, [&](uint32_t w) { return qkv_unpack_row(w, recv, q, k, v, u); });
}

// o [Hg][Lp][d] -> send: slice j holds rows (t, hh) of token j Lr + t, head h0 + hh.
__global__ void __launch_bounds__(256) ulysses_pack_o_kernel(const __nv_bfloat16* __restrict__ o,
                                                             uint8_t* __restrict__ send, UlyssesDims u) {
    const uint32_t first = blockIdx.x * kUlyRowsPerCta + (threadIdx.x / 32) * kUlyRowsPerWarp;
    const uint32_t n_rows = static_cast<uint32_t>(u.G) * u.Lr * u.hc;
    pack_rows(first, n_rows, [&](uint32_t w) { return o_pack_row(w, o, send, u); });
}

// recv (slice i from rank i) -> y [Lr][H][d]: row (t, hh) is head i Hg + h0 + hh of
// token t.
__global__ void __launch_bounds__(256) ulysses_unpack_o_kernel(const uint8_t* __restrict__ recv,
                                                               __nv_bfloat16* __restrict__ y, UlyssesDims u) {
    const uint32_t first = blockIdx.x * kUlyRowsPerCta + (threadIdx.x / 32) * kUlyRowsPerWarp;
    const uint32_t n_rows = static_cast<uint32_t>(u.G) * u.Lr * u.hc;
    unpack_rows(first, n_rows, [&](uint32_t w) { return o_unpack_row(w, recv, y, u); });
}

// The CTA's remote stores, system-wide before it ends: the barrier makes every thread's
// stores observed by thread 0, whose fence.sc.sys is cumulative over them (one fence per
// CTA; one per thread made the put kernels 2.7 times slower).
__device__ __forceinline__ void publish_cta() {
    __syncthreads();
    if (threadIdx.x == 0) __threadfence_system();
}

// x -> every peer's receive buffer (peer puts), published before the CTA ends, so a later
// signal launch may announce it.  A fixed grid strides over the rows, so few CTAs fence.
__global__ void __launch_bounds__(256) ulysses_put_qkv_kernel(const __nv_bfloat16* __restrict__ x, PeerDst pd,
                                                              UlyssesDims u) {
    const uint32_t n_rows = static_cast<uint32_t>(u.G) * u.Lr * 3u * u.hc;
    for (uint32_t base = blockIdx.x * kUlyRowsPerCta; base < n_rows; base += gridDim.x * kUlyRowsPerCta)
        pack_rows(base + (threadIdx.x / 32) * kUlyRowsPerWarp, n_rows,
                  [&](uint32_t w) { return qkv_put_row(w, x, pd, u); });
    publish_cta();
}

__global__ void __launch_bounds__(256) ulysses_put_o_kernel(const __nv_bfloat16* __restrict__ o, PeerDst pd,
                                                            UlyssesDims u) {
    const uint32_t n_rows = static_cast<uint32_t>(u.G) * u.Lr * u.hc;
    for (uint32_t base = blockIdx.x * kUlyRowsPerCta; base < n_rows; base += gridDim.x * kUlyRowsPerCta)
        pack_rows(base + (threadIdx.x / 32) * kUlyRowsPerWarp, n_rows,
                  [&](uint32_t w) { return o_put_row(w, o, pd, u); });
    publish_cta();
}

// Flag word `rank` of the flag array at flag_offset in every peer's allocation := value
// (system-scope release, after this thread's earlier writes and the previous launches'
// on the stream).
__global__ void peer_signal_kernel(const unsigned long long* __restrict__ bases, unsigned long long flag_offset,
                                   int rank, int world, uint32_t value) {
    const int j = blockIdx.x * blockDim.x + threadIdx.x;
    if (j >= world) return;
    uint32_t* f = reinterpret_cast<uint32_t*>(__ldg(bases + j) + flag_offset) + rank;
    asm volatile("fence.sc.sys;" ::: "memory");
    asm volatile("st.release.sys.global.u32 [%0], %1;" ::"l"(f), "r"(value) : "memory");
}

// Wait until flags[0 .. world) all equal value (system-scope acquire), at most limit_ns;
// on running out the launch latches SBSA_ERR_TIMEOUT and returns.
__global__ void peer_wait_kernel(const uint32_t* flags, int world, uint32_t value, unsigned long long limit_ns) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= world) return;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        uint32_t v;
        asm volatile("ld.acquire.sys.global.u32 %0, [%1];" : "=r"(v) : "l"(flags + i) : "memory");
        if (v == value) return;
        if (globaltimer_ns() - t0 > limit_ns) {
            raise_error(kErrTimeout);
            return;
        }
        __nanosleep(256);
    }
}

}  // namespace sbsa
