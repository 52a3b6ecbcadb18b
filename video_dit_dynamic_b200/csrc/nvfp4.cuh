// NVFP4 linear layer (the GEMMs around the attention): both operands in NVFP4 -- E2M1
// values, one E4M3 scale per 16 consecutive elements of a row, one FP32 scale per
// tensor -- multiplied on the tcgen05 block-scaled tensor cores with FP32 accumulation,
// BF16 output and a per-column bias added in the epilogue (page "知识卡片：600倍加速，
// 720p视频实时生成！单卡也能带的动14B模型", 方法/产品要点, bullets NVFP4 量化感知训练 and
// 高效推理算子; page "单卡 RTX 5090 跑 Wan2.2-A14B：720p 视频生成只要 3.8 秒", 四步拆解
// item 2).
//
// Quantization (the pages give no formula; the plainest reading of their description):
//   s     = 2688 / amax(|x|) over the tensor (1 for an all-zero tensor); 2688 = 6 * 448
//   sf_b  = e4m3((amax of block b / 6) * s), nearest even, saturating
//   code  = e2m1(x * (s / sf_b)), nearest even, saturating at +-6 (0 where sf_b = 0)
// every step an fp32 operation in this order.  A value decodes to code * sf_b / s, so
//   C[m][n] = (1 / (s_A s_B)) * sum_k code_A sf_A code_B sf_B + bias[n].
//
// Layouts:
//   codes  [rows][K/2] bytes, element 2i of a row in the low nibble of byte i;
//   scales atoms of 128 rows x 4 blocks (512 bytes; row r at (r % 32) * 16 +
//          ((r % 128) / 32) * 4, block kb at + kb % 4), the K/64 atoms of one 128-row
//          group consecutive; rows padded to a multiple of 128 (scale 0).  One atom is
//          exactly what tcgen05.cp.32x128b.warpx4 moves into four TMEM columns, where the
//          block-scaled MMA reads the scales of row r from column r / 32.
#pragma once
#include <cuda_bf16.h>

#include "common.cuh"
#include "ptx.cuh"
#include "rope.cuh"
#include "tmem_wide.cuh"

namespace sbsa {

constexpr float kNvfp4Range = 2688.f;  // largest e2m1 (6) x largest e4m3 (448)

__device__ __forceinline__ float nvfp4_tensor_scale(float amax) {
    return amax > 0.f ? __fdiv_rn(kNvfp4Range, amax) : 1.f;
}

// e4m3 code (non-negative, finite) -> its exact fp32 value, from the format: bias 7,
// three mantissa bits, subnormals m * 2^-9.
__device__ __forceinline__ float e4m3_value(uint32_t code) {
    const uint32_t e = (code >> 3) & 15u, m = code & 7u;
    return e ? __uint_as_float(((e + 120u) << 23) | (m << 20)) : static_cast<float>(m) * 0.001953125f;
}

// Eight floats -> eight e2m1 codes, v[0] in the lowest nibble (nearest even, saturating).
__device__ __forceinline__ uint32_t cvt_e2m1x8(const float (&v)[8]) {
    uint32_t r;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(r)
        : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
    return r;
}

__host__ __device__ constexpr size_t nvfp4_scale_offset(long long r, int kb, int K) {
    return (static_cast<size_t>(r / 128) * static_cast<size_t>(K / 64) + static_cast<size_t>(kb / 4)) * 512 +
           static_cast<size_t>(r % 32) * 16 + static_cast<size_t>((r % 128) / 32) * 4 + static_cast<size_t>(kb % 4);
}

// ---------------------------------------------------------------- amax
// max |x| over a bf16 tensor of n8 16-byte chunks.  The result is combined with an
// atomicMax on the float's bit pattern (for non-negative floats the bit patterns order
// like the values); *out must hold 0 before the launch.
__global__ void __launch_bounds__(256) nvfp4_amax_kernel(const uint4* __restrict__ x, long long n8,
                                                         unsigned int* __restrict__ out) {
    __shared__ float red[8];
    float m = 0.f;
    for (long long i = blockIdx.x * 256ll + threadIdx.x; i < n8; i += static_cast<long long>(gridDim.x) * 256) {
        const uint4 w = __ldg(x + i);
        const uint32_t v[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            m = fmaxf(m, fabsf(__uint_as_float(v[j] << 16)));
            m = fmaxf(m, fabsf(__uint_as_float(v[j] & 0xFFFF0000u)));
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, off));
    if (threadIdx.x % 32 == 0) red[threadIdx.x / 32] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
#pragma unroll
        for (int w = 1; w < 8; ++w) m = fmaxf(m, red[w]);
        atomicMax(out, __float_as_uint(m));
    }
}

// ---------------------------------------------------------------- quantizer
// One thread per (row, 16-element block) of a [rows][K] bf16 matrix: 32 bytes in,
// 8 bytes of codes and one scale byte out.  Threads for the padding rows (up to a
// multiple of 128) write scale 0.
__global__ void __launch_bounds__(256) nvfp4_quantize_kernel(const uint4* __restrict__ x,
                                                             const float* __restrict__ amax,
                                                             uint2* __restrict__ codes, uint8_t* __restrict__ scales,
                                                             long long rows, int K, long long n_threads) {
    const long long t = blockIdx.x * 256ll + threadIdx.x;
    if (t >= n_threads) return;
    const int kbs = K / 16;
    const long long r = t / kbs;
    const int kb = static_cast<int>(t % kbs);
    const size_t off = nvfp4_scale_offset(r, kb, K);
    if (r >= rows) {
        scales[off] = 0;
        return;
    }
    const float s = nvfp4_tensor_scale(__ldg(amax));
    // row r, elements 16 kb .. 16 kb + 15 are 16-byte chunks 2 t and 2 t + 1
    const uint4 w0 = __ldg(x + 2 * t), w1 = __ldg(x + 2 * t + 1);
    const uint32_t in[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
    float v[16];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        v[2 * j] = __uint_as_float(in[j] << 16);
        v[2 * j + 1] = __uint_as_float(in[j] & 0xFFFF0000u);
    }
    float bmax = 0.f;
#pragma unroll
    for (int j = 0; j < 16; ++j) bmax = fmaxf(bmax, fabsf(v[j]));
    const float scaled = __fmul_rn(__fdiv_rn(bmax, 6.f), s);
    uint16_t sf2;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(sf2) : "f"(0.f), "f"(scaled));
    const uint32_t sf = sf2 & 0xFFu;
    const float sf_f = e4m3_value(sf);
    const float inv = sf_f > 0.f ? __fdiv_rn(s, sf_f) : 0.f;
    float lo[8], hi[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        lo[j] = __fmul_rn(v[j], inv);
        hi[j] = __fmul_rn(v[8 + j], inv);
    }
    codes[t] = make_uint2(cvt_e2m1x8(lo), cvt_e2m1x8(hi));
    scales[off] = static_cast<uint8_t>(sf);
}

// ---------------------------------------------------------------- GEMM
// C[M][N] = alpha * A[M][K] B[N][K]^T + bias[N], A and B NVFP4 (K-major), C bf16.
//
// Persistent: one CTA per SM walks output tiles of 128 x 256 (tile index t -> row
// tile t / tiles_n, column tile t % tiles_n, so the CTAs running at one time share a
// few A row tiles and all of B in L2).  448 threads:
//   warp 0      TMA producer: per K-tile of 256 elements one stage of A (128 rows x
//               128 bytes), B (256 x 128 bytes), their scale atoms (2 KB and 4 KB,
//               contiguous in global memory, one bulk copy per 128-row group) through a
//               four-stage ring;
//   warp 1      TMEM allocation and the one thread that issues the block-scaled MMAs
//               (M = 128, N = 256, K = 64; four per K-tile) and nothing else;
//   warps 2-9   epilogue: warp w reads TMEM lanes 32 (w % 4) .. + 31 and output columns
//               128 ((w - 2) / 4) .. + 127 of the tile, applies alpha and the bias (staged
//               in shared memory while the tile is computed) in one fp32 FMA, rounds to
//               bf16, hands the accumulator back, then stores its rows;
//   warps 10-13 scales: each stage's 12 scale atoms into that stage's TMEM region
//               (tcgen05.st, in the layout tcgen05.cp.32x128b.warpx4 would leave), then
//               its sf_full barrier.
// Measured on the way: scale copies issued with tcgen05.cp by the MMA thread, in order
// with its MMAs, bounded the kernel; stored by warps that also ran the epilogue, they
// queued behind its stores; a bias read from global memory per element made the
// accumulator's hand-back slow.
// TMEM: accumulator in columns 0-255; one scale region of 48 columns per stage from
// column 256 (A scales: four columns per K step, then B scales: eight per K step).
struct Nvfp4GemmParams {
    const uint8_t* sfa;
    const uint8_t* sfb;
    const float* amax_a;
    const float* amax_b;
    const float* bias;  // [N] or null
    __nv_bfloat16* c;   // [M][N]
    int M, N, K;
    int tiles_m, tiles_n;
    unsigned int epoch;
};

constexpr int kFp4TileM = 128;
constexpr int kFp4TileN = 256;
constexpr int kFp4TileK = 256;  // elements: 128 bytes of codes per row
constexpr int kFp4Stages = 4;
constexpr int kFp4ABytes = kFp4TileM * 128;
constexpr int kFp4BBytes = kFp4TileN * 128;
constexpr int kFp4SfaBytes = (kFp4TileM / 128) * 4 * 512;
constexpr int kFp4SfbBytes = (kFp4TileN / 128) * 4 * 512;
constexpr int kFp4StageBytes = kFp4ABytes + kFp4BBytes + kFp4SfaBytes + kFp4SfbBytes;
constexpr int kFp4BiasOff = kFp4Stages * kFp4StageBytes;  // each epilogue warp's 128 bias values of the tile
constexpr int kFp4BarOff = kFp4BiasOff + 8 * 128 * 4;
constexpr uint32_t kFp4SfStageCols = 48;  // A scales (16 columns) then B scales (32) of one K-tile
constexpr int kFp4NumBars = 3 * kFp4Stages + 3;  // full[S], empty[S], sf_full[S], acc_full, acc_empty, drain
constexpr int kFp4SmemBytes = kFp4BarOff + kFp4NumBars * 8 + 16 + 1024;  // + tmem slot, flag, alignment slack
constexpr int kFp4Threads = 448;  // 14 warps: producer, MMA, eight epilogue, four scale warps
constexpr uint32_t kFp4ColSf = 256;  // scale regions from here, one of kFp4SfStageCols per pipeline stage
static_assert(kFp4StageBytes % 1024 == 0, "stages keep the 1024-byte alignment of the swizzled tiles");
static_assert(kFp4SmemBytes <= 232448, "shared memory");

// kind::mxf4nvf4 instruction descriptor: E2M1 A and B (format 1), UE4M3 scales
// (bit 23 = 0), both K-major, dense K = 64, scale-factor ids 0.
__host__ __device__ constexpr uint32_t idesc_nvfp4(int M, int N) {
    return (1u << 7) | (1u << 10) | (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ void umma_nvfp4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                           uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
            d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
        : "memory");
}


__device__ __forceinline__ uint64_t policy_evict_normal() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// One thread's 128 bf16 outputs of a row from column n0 (64 packed pairs).  With
// `wide` (row starts 32-byte aligned, N a multiple of 16) each store is 32 bytes, a
// whole L2 sector: the 16-byte stores of a warp fill half-sectors of 32 rows and cost
// the kernel about 9% (measured).
__device__ __forceinline__ void store_row128(__nv_bfloat16* row, const uint32_t (&v)[64], int n0, int N, bool wide) {
    if (wide) {
#pragma unroll
        for (int j = 0; j < 8; ++j)
            if (n0 + 16 * j < N)
                st_global_v8(row + n0 + 16 * j, v[8 * j], v[8 * j + 1], v[8 * j + 2], v[8 * j + 3], v[8 * j + 4],
                             v[8 * j + 5], v[8 * j + 6], v[8 * j + 7]);
    } else {
        uint4* dst = reinterpret_cast<uint4*>(row + n0);
#pragma unroll
        for (int j = 0; j < 16; ++j)
            if (n0 + 8 * j < N) dst[j] = make_uint4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
    }
}

__global__ void __launch_bounds__(kFp4Threads, 1) nvfp4_gemm_kernel(const __grid_constant__ CUtensorMap map_a,
                                                                    const __grid_constant__ CUtensorMap map_b,
                                                                    const Nvfp4GemmParams p) {
    extern __shared__ __align__(1024) uint8_t fp4_smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(fp4_smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kFp4BarOff);
    uint64_t* full = bars;
    uint64_t* empty = bars + kFp4Stages;
    uint64_t* sf_full = bars + 2 * kFp4Stages;  // a stage's scales are in TMEM
    uint64_t* acc_full = bars + 3 * kFp4Stages;
    uint64_t* acc_empty = acc_full + 1;
    uint64_t* drain = acc_full + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kFp4NumBars);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    // every thread takes the same branch (the barriers below need all of them)
    if (__syncthreads_or(launch_aborted(p.epoch) ? 1 : 0)) return;
    const int num_tiles = p.tiles_m * p.tiles_n;
    const int k_tiles = p.K / kFp4TileK;

    if (threadIdx.x == 0) {
        *abort_flag = 0;
        for (int s = 0; s < kFp4Stages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
            mbar_init(&sf_full[s], 4);  // one arrival per scale-storing warp
        }
        mbar_init(acc_full, 1);
        mbar_init(acc_empty, 8);  // the eight epilogue warps
        mbar_init(drain, 1);
        fence_mbar_init();
        tma_prefetch_desc(&map_a);
        tma_prefetch_desc(&map_b);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    auto give_up = [&]() {
        *abort_flag = 1;
        abort_launch(p.epoch);
    };
    auto wait = [&](uint64_t* bar, uint32_t parity) -> bool {
        if (mbar_wait_bounded(bar, parity, abort_flag, kWaitLimitNs)) return true;
        if (!*abort_flag) give_up();
        return false;
    };

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            const uint64_t pol_a = policy_evict_normal();
            const uint64_t pol_b = policy_evict_last();
            const size_t k_atoms = static_cast<size_t>(p.K / 64);
            const int n_groups = (p.N + 127) / 128;
            int it = 0;
            bool ok = true;
            for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
                const int tm = tile / p.tiles_n;
                const int tn = tile % p.tiles_n;
                const int g0 = tn * (kFp4TileN / 128);
                const int ng = min(kFp4TileN / 128, n_groups - g0);  // B scale groups that exist
                for (int kt = 0; kt < k_tiles; ++kt, ++it) {
                    const int s = it % kFp4Stages;
                    if (!(ok = wait(&empty[s], ((it / kFp4Stages) & 1) ^ 1))) break;
                    uint8_t* st = smem + s * kFp4StageBytes;
                    mbar_arrive_expect_tx(&full[s], kFp4ABytes + kFp4BBytes + kFp4SfaBytes + ng * 2048);
                    tma_load_2d(st, &map_a, &full[s], kt * 128, tm * kFp4TileM, pol_a);
                    tma_load_2d(st + kFp4ABytes, &map_b, &full[s], kt * 128, tn * kFp4TileN, pol_b);
                    bulk_load_g2s(st + kFp4ABytes + kFp4BBytes, p.sfa + (static_cast<size_t>(tm) * k_atoms + 4 * kt) * 512,
                                  2048, &full[s]);
                    for (int g = 0; g < ng; ++g)
                        bulk_load_g2s(st + kFp4ABytes + kFp4BBytes + kFp4SfaBytes + g * 2048,
                                      p.sfb + (static_cast<size_t>(g0 + g) * k_atoms + 4 * kt) * 512, 2048, &full[s]);
                }
            }
            if (!ok) {
                // every issued copy must land before the CTA exits
                volatile int never = 0;
                for (int q = it - kFp4Stages < 0 ? 0 : it - kFp4Stages; q < it; ++q)
                    mbar_wait_bounded(&full[q % kFp4Stages], (q / kFp4Stages) & 1, &never, kWaitLimitNs);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ tensor-pipe issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_nvfp4(kFp4TileM, kFp4TileN);
            int it = 0, tcount = 0;
            bool ok = true;
            for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x, ++tcount) {
                // the epilogue must have read the previous tile's accumulator out of TMEM
                if (tcount > 0 && !(ok = wait(acc_empty, (tcount - 1) & 1))) break;
                tc_fence_after();
                for (int kt = 0; kt < k_tiles; ++kt, ++it) {
                    const int s = it % kFp4Stages;
                    if (!(ok = wait(&full[s], (it / kFp4Stages) & 1))) break;
                    tc_fence_after();
                    const uint32_t st = smem_u32(smem + s * kFp4StageBytes);
                    // the stage's scales were stored into its TMEM region by warps 10-13
                    if (!(ok = wait(&sf_full[s], (it / kFp4Stages) & 1))) break;
                    tc_fence_after();
                    const uint32_t t_sfa = tmem + kFp4ColSf + static_cast<uint32_t>(s) * kFp4SfStageCols;
                    const uint32_t t_sfb = t_sfa + 16;
                    const uint64_t a0 = sdesc_sw128(st, 16, 1024);
                    const uint64_t b0 = sdesc_sw128(st + kFp4ABytes, 16, 1024);
#pragma unroll
                    for (int kb = 0; kb < 4; ++kb) {
                        // K = 64 codes = 32 bytes per step inside the 128-byte swizzled row
                        umma_nvfp4(tmem, a0 + static_cast<uint64_t>((kb * 32) >> 4), b0 + static_cast<uint64_t>((kb * 32) >> 4),
                                   idesc, t_sfa + 4 * kb, t_sfb + 8 * kb, (kt | kb) ? 1u : 0u);
                    }
                    umma_commit(&empty[s]);
                }
                if (ok) umma_commit(acc_full);
            }
            if (!ok) {
                umma_commit(drain);  // wait for every MMA this thread issued
                volatile int never = 0;
                mbar_wait_bounded(drain, 0, &never, kWaitLimitNs);
            }
        }
    } else {
        const int quarter = warp & 3;  // the TMEM lane quarter this warp may access
        if (warp < 10) {
            // ------------------------------------------------------------ epilogue (warps 2-9)
            const int half = (warp - 2) >> 2;
            const uint32_t t_row = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(half * 128);
            const float alpha =
                __frcp_rn(__fmul_rn(nvfp4_tensor_scale(__ldg(p.amax_a)), nvfp4_tensor_scale(__ldg(p.amax_b))));
            const bool wide = (reinterpret_cast<uintptr_t>(p.c) & 31u) == 0 && p.N % 16 == 0;
            // this warp's copy of the tile's 128 bias values (read back as broadcasts)
            const uint32_t bias_w = smem_u32(smem + kFp4BiasOff) + static_cast<uint32_t>((warp - 2) * 128 * 4);
            int tcount = 0;
            for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++tcount) {
                const int tm = tile / p.tiles_n;
                const int tn = tile % p.tiles_n;
                const int n0 = tn * kFp4TileN + half * 128;
                // the bias goes to shared memory while the tile is still being computed
                {
                    float b[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int n = n0 + 4 * lane + e;
                        b[e] = (p.bias && n < p.N) ? __ldg(p.bias + n) : 0.f;
                    }
                    st_shared_v4(bias_w + lane * 16, __float_as_uint(b[0]), __float_as_uint(b[1]), __float_as_uint(b[2]),
                                 __float_as_uint(b[3]));
                    __syncwarp();
                }
                if (!__all_sync(0xFFFFFFFFu, wait(acc_full, tcount & 1))) break;
                tc_fence_after();
                // this warp's 128 columns in two 64-column TMEM loads
                uint32_t packed[64];
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    uint32_t raw[64];
                    tmem_ld64(t_row + c * 64, raw);
#pragma unroll
                    for (int e = 0; e < 64; e += 4) {
                        uint32_t b0, b1, b2, b3;
                        ld_shared_v4(bias_w + (c * 64 + e) * 4, b0, b1, b2, b3);
                        packed[c * 32 + e / 2] = pack_bf16x2(fmaf(__uint_as_float(raw[e]), alpha, __uint_as_float(b0)),
                                                             fmaf(__uint_as_float(raw[e + 1]), alpha, __uint_as_float(b1)));
                        packed[c * 32 + e / 2 + 1] =
                            pack_bf16x2(fmaf(__uint_as_float(raw[e + 2]), alpha, __uint_as_float(b2)),
                                        fmaf(__uint_as_float(raw[e + 3]), alpha, __uint_as_float(b3)));
                    }
                }
                // the accumulator is in registers: the next tile's MMAs may overwrite it
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(acc_empty);
                const long long m = static_cast<long long>(tm) * kFp4TileM + quarter * 32 + lane;
                if (m < p.M) store_row128(p.c + m * p.N, packed, n0, p.N, wide);
                __syncwarp();  // every lane has read the bias before the next tile's is written
            }
        } else {
            // ------------------------------------------------------------ scales (warps 10-13)
            // K-tile i's scales into TMEM region i % S: lane L of quarter q holds, for rows
            // 32 q + L % 32 of A (4 columns per K step) and of B's two 128-row groups
            // (8 columns per K step), the 16 bytes of row L % 32 of each 512-byte atom --
            // the layout tcgen05.cp.32x128b.warpx4 would leave there
            const int my_tiles = static_cast<int>(blockIdx.x) < num_tiles
                                     ? (num_tiles - 1 - static_cast<int>(blockIdx.x)) / static_cast<int>(gridDim.x) + 1
                                     : 0;
            const int total = my_tiles * k_tiles;
            for (int i = 0; i < total; ++i) {
                const int s = i % kFp4Stages;
                if (!__all_sync(0xFFFFFFFFu, wait(&full[s], (i / kFp4Stages) & 1))) break;
                const uint32_t base = smem_u32(smem + s * kFp4StageBytes + kFp4ABytes + kFp4BBytes) + lane * 16;
                uint32_t va[16], vb[32];
#pragma unroll
                for (int kb = 0; kb < 4; ++kb) {
                    ld_shared_v4(base + kb * 512, va[4 * kb], va[4 * kb + 1], va[4 * kb + 2], va[4 * kb + 3]);
#pragma unroll
                    for (int g = 0; g < 2; ++g)
                        ld_shared_v4(base + kFp4SfaBytes + g * 2048 + kb * 512, vb[8 * kb + 4 * g], vb[8 * kb + 4 * g + 1],
                                     vb[8 * kb + 4 * g + 2], vb[8 * kb + 4 * g + 3]);
                }
                const uint32_t t = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + kFp4ColSf +
                                   static_cast<uint32_t>(s) * kFp4SfStageCols;
                tmem_st16(t, va);
                tmem_st32(t + 16, vb);
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sf_full[s]);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ---------------------------------------------------------------- GEMM on CTA pairs
// The same product on pairs of CTAs (clusters of two) with tcgen05's two-CTA MMA: a
// pair owns a 256 x 256 output tile, so each SM loads 38 KB per K-tile instead of the
// 54 KB of a 128 x 256 tile on one CTA, for the same number of MMA cycles (the load
// path, about 61 bytes per clock per SM from L2, bounds the one-CTA kernel).
//   warp 0      (both CTAs) loads this CTA's 128 rows of the tile's A and of its B with
//               two-CTA TMA, whose bytes complete on the leader's stage barrier, and the
//               scales of its A rows and of all 256 B rows with bulk copies on its own
//               barrier;
//   warp 1      (leader) issues the MMAs (tcgen05.mma.cta_group::2, M = 256, N = 256,
//               K = 64), which read A from each CTA's shared memory and B from both and
//               leave rows 128 r .. + 127 of the accumulator in CTA r's TMEM;
//   warps 2-9   (both CTAs) epilogue as in the one-CTA kernel;
//   warps 10-13 (both CTAs) store this CTA's scales into its TMEM.
// The leader's commits arrive on the stage's free barrier and, at the end of a tile, the
// accumulator barrier of both CTAs.  The other CTA's hand-overs to the leader (scales
// stored, accumulator read) are relaxed remote arrivals made after tcgen05.wait::st /
// ::ld returned: with release semantics each took about 1,400 cycles and the kernel ran
// at a third of the speed.
struct Nvfp4Gemm2Params {
    const uint8_t* sfa;
    const uint8_t* sfb;
    const float* amax_a;
    const float* amax_b;
    const float* bias;  // [N] or null
    __nv_bfloat16* c;   // [M][N]
    int M, N, K;
    int tiles_m, tiles_n;   // 256 x 256 tiles
    int groups_a, groups_b; // 128-row scale groups of A and B
    unsigned int epoch;
};

constexpr int kF2Stages = 5;
constexpr int kF2Half = 128 * 128;                   // 128 rows x 128 bytes of codes
constexpr int kF2SfaBytes = 4 * 512;                 // this CTA's A rows, one K-tile
constexpr int kF2SfbBytes = 2 * 4 * 512;             // all 256 B rows of the tile, one K-tile
constexpr int kF2StageBytes = 2 * kF2Half + kF2SfaBytes + kF2SfbBytes;
// each epilogue warp's 4 KB: the tile's 128 bias values while it converts, then 32 rows x 64
// columns of bf16 output at a time for the transposed stores
constexpr int kF2EpiOff = kF2Stages * kF2StageBytes;
constexpr int kF2EpiBytes = 4096;
constexpr int kF2BarOff = kF2EpiOff + 8 * kF2EpiBytes;
// full[S] (leader: both CTAs' codes), sf_in[S] (this CTA's scales landed), sf_full[S]
// (leader: both CTAs' scales in TMEM), empty[S], acc_full, acc_empty, drain
constexpr int kF2NumBars = 4 * kF2Stages + 3;
constexpr int kF2SmemBytes = kF2BarOff + kF2NumBars * 8 + 16 + 1024;
static_assert(kF2StageBytes % 1024 == 0, "stages keep the 1024-byte alignment of the swizzled tiles");
static_assert(kF2SmemBytes <= 232448, "shared memory");
static_assert(kFp4ColSf + kF2Stages * kFp4SfStageCols <= 512, "accumulator and scale regions fit in TMEM");

__device__ __forceinline__ void umma_nvfp4_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                                uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
            d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
        : "memory");
}
// Arrive on the barrier at this shared offset in both CTAs of the pair once the
// tensor-core work issued so far has completed.
__device__ __forceinline__ void umma_commit_pair_both(uint64_t* bar) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
            smem_u32(bar)),
        "h"(static_cast<uint16_t>(0x3))
        : "memory");
}
__device__ __forceinline__ void umma_commit_pair_own(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}
// Two-CTA tiled load into this CTA's shared memory whose bytes complete on the barrier
// at `bar_cluster` (a shared::cluster address, here the leader's).
__device__ __forceinline__ void tma_load_2d_pair(void* smem_dst, const CUtensorMap* map, uint32_t bar_cluster, int x,
                                                 int y, uint64_t cache_policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(x), "r"(y), "l"(cache_policy)
        : "memory");
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kFp4Threads, 1)
    nvfp4_gemm_pair_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                           const Nvfp4Gemm2Params p) {
    extern __shared__ __align__(1024) uint8_t fp4p_smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(fp4p_smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kF2BarOff);
    uint64_t* full = bars;
    uint64_t* sf_in = bars + kF2Stages;
    uint64_t* sf_full = bars + 2 * kF2Stages;
    uint64_t* empty = bars + 3 * kF2Stages;
    uint64_t* acc_full = bars + 4 * kF2Stages;
    uint64_t* acc_empty = acc_full + 1;
    uint64_t* drain = acc_full + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kF2NumBars);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int pair = blockIdx.x / 2;
    const int n_pairs = gridDim.x / 2;
    const int num_tiles = p.tiles_m * p.tiles_n;
    const int k_tiles = p.K / kFp4TileK;
    const int my_tiles = pair < num_tiles ? (num_tiles - 1 - pair) / n_pairs + 1 : 0;

    if (threadIdx.x == 0) {
        *abort_flag = 0;
        for (int s = 0; s < kF2Stages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&sf_in[s], 1);
            mbar_init(&sf_full[s], 8);  // four scale warps in each CTA
            mbar_init(&empty[s], 1);
        }
        mbar_init(acc_full, 1);
        mbar_init(acc_empty, 16);  // eight epilogue warps in each CTA
        mbar_init(drain, 1);
        fence_mbar_init();
        tma_prefetch_desc(&map_a);
        tma_prefetch_desc(&map_b);
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(512)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    cluster_sync_all();  // both CTAs' barriers exist before either uses the other's
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    auto give_up = [&]() {
        *abort_flag = 1;
        abort_launch(p.epoch);
    };
    auto wait = [&](uint64_t* bar, uint32_t parity) -> bool {
        if (mbar_wait_bounded_cluster(bar, parity, abort_flag, kWaitLimitNs)) return true;
        if (!*abort_flag) give_up();
        return false;
    };
    // a hand-over to the leader after this thread waited for its TMEM accesses: a plain
    // arrival in the leader, a relaxed remote one from the other CTA
    auto arrive_leader = [&](uint64_t* bar) {
        if (leader) mbar_arrive(bar);
        else mbar_arrive_cluster_relaxed(mapa_shared(smem_u32(bar), 0));
    };

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer (both CTAs)
        if (lane == 0 && !launch_aborted(p.epoch)) {
            const uint64_t pol_a = policy_evict_normal();
            const uint64_t pol_b = policy_evict_last();
            const size_t k_atoms = static_cast<size_t>(p.K / 64);
            int it = 0;
            bool ok = true;
            for (int tile = pair; ok && tile < num_tiles; tile += n_pairs) {
                const int tm = tile / p.tiles_n;
                const int tn = tile % p.tiles_n;
                // this CTA's rows of the tile's A and B, and the tile's scale groups; groups
                // that do not exist (past the padded rows) are replaced by the last one: they
                // only feed rows and columns that are never stored
                const int ra = tm * 256 + static_cast<int>(rank) * 128;
                const int rb = tn * 256 + static_cast<int>(rank) * 128;
                const size_t ga = static_cast<size_t>(min(tm * 2 + static_cast<int>(rank), p.groups_a - 1));
                const size_t gb0 = static_cast<size_t>(min(tn * 2, p.groups_b - 1));
                const size_t gb1 = static_cast<size_t>(min(tn * 2 + 1, p.groups_b - 1));
                for (int kt = 0; kt < k_tiles; ++kt, ++it) {
                    const int s = it % kF2Stages;
                    if (!(ok = wait(&empty[s], ((it / kF2Stages) & 1) ^ 1))) break;
                    uint8_t* st = smem + s * kF2StageBytes;
                    const uint32_t bar = mapa_shared(smem_u32(&full[s]), 0);
                    if (leader) mbar_arrive_expect_tx(&full[s], 2 * 2 * kF2Half);
                    tma_load_2d_pair(st, &map_a, bar, kt * 128, ra, pol_a);
                    tma_load_2d_pair(st + kF2Half, &map_b, bar, kt * 128, rb, pol_b);
                    mbar_arrive_expect_tx(&sf_in[s], kF2SfaBytes + kF2SfbBytes);
                    bulk_load_g2s(st + 2 * kF2Half, p.sfa + (ga * k_atoms + 4 * kt) * 512, 2048, &sf_in[s]);
                    bulk_load_g2s(st + 2 * kF2Half + kF2SfaBytes, p.sfb + (gb0 * k_atoms + 4 * kt) * 512, 2048, &sf_in[s]);
                    bulk_load_g2s(st + 2 * kF2Half + kF2SfaBytes + 2048, p.sfb + (gb1 * k_atoms + 4 * kt) * 512, 2048,
                                  &sf_in[s]);
                }
            }
            if (!ok) {
                // every copy issued for the stages still pending must land before the pair exits
                volatile int never = 0;
                for (int q = it - kF2Stages < 0 ? 0 : it - kF2Stages; q < it; ++q) {
                    if (leader) mbar_wait_bounded_cluster(&full[q % kF2Stages], (q / kF2Stages) & 1, &never, kWaitLimitNs);
                    mbar_wait_bounded_cluster(&sf_in[q % kF2Stages], (q / kF2Stages) & 1, &never, kWaitLimitNs);
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ tensor-pipe issuer (leader)
        if (lane == 0 && leader && !launch_aborted(p.epoch)) {
            constexpr uint32_t idesc = idesc_nvfp4(256, 256);
            int it = 0, tcount = 0;
            bool ok = true;
            for (int tile = pair; ok && tile < num_tiles; tile += n_pairs, ++tcount) {
                // both CTAs' epilogues must have read the previous tile's accumulator
                if (tcount > 0 && !(ok = wait(acc_empty, (tcount - 1) & 1))) break;
                tc_fence_after();
                for (int kt = 0; kt < k_tiles; ++kt, ++it) {
                    const int s = it % kF2Stages;
                    if (!(ok = wait(&full[s], (it / kF2Stages) & 1))) break;
                    // both CTAs' scales of the stage are in their TMEM regions
                    if (!(ok = wait(&sf_full[s], (it / kF2Stages) & 1))) break;
                    tc_fence_after();
                    const uint32_t st = smem_u32(smem + s * kF2StageBytes);
                    const uint32_t t_sfa = tmem + kFp4ColSf + static_cast<uint32_t>(s) * kFp4SfStageCols;
                    const uint32_t t_sfb = t_sfa + 16;
                    const uint64_t a0 = sdesc_sw128(st, 16, 1024);
                    const uint64_t b0 = sdesc_sw128(st + kF2Half, 16, 1024);
#pragma unroll
                    for (int kb = 0; kb < 4; ++kb)
                        umma_nvfp4_pair(tmem, a0 + static_cast<uint64_t>((kb * 32) >> 4),
                                        b0 + static_cast<uint64_t>((kb * 32) >> 4), idesc, t_sfa + 4 * kb, t_sfb + 8 * kb,
                                        (kt | kb) ? 1u : 0u);
                    umma_commit_pair_both(&empty[s]);
                }
                if (ok) umma_commit_pair_both(acc_full);
            }
            if (!ok) {
                umma_commit_pair_own(drain);  // wait for every MMA this thread issued
                volatile int never = 0;
                mbar_wait_bounded_cluster(drain, 0, &never, kWaitLimitNs);
            }
        }
    } else if (warp < 10) {
        // ------------------------------------------------------------ epilogue (both CTAs)
        const int quarter = warp & 3;
        const int half = (warp - 2) >> 2;
        const uint32_t t_row = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(half * 128);
        const float alpha = __frcp_rn(__fmul_rn(nvfp4_tensor_scale(__ldg(p.amax_a)), nvfp4_tensor_scale(__ldg(p.amax_b))));
        const bool wide = (reinterpret_cast<uintptr_t>(p.c) & 31u) == 0 && p.N % 16 == 0;
        const uint32_t bias_w = smem_u32(smem + kF2EpiOff) + static_cast<uint32_t>((warp - 2) * kF2EpiBytes);
        int tcount = 0;
        for (int tile = pair; tile < num_tiles && !launch_aborted(p.epoch); tile += n_pairs, ++tcount) {
            const int tm = tile / p.tiles_n;
            const int tn = tile % p.tiles_n;
            const int n0 = tn * 256 + half * 128;
            // the bias goes to shared memory while the tile is still being computed
            {
                float b[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int n = n0 + 4 * lane + e;
                    b[e] = (p.bias && n < p.N) ? __ldg(p.bias + n) : 0.f;
                }
                st_shared_v4(bias_w + lane * 16, __float_as_uint(b[0]), __float_as_uint(b[1]), __float_as_uint(b[2]),
                             __float_as_uint(b[3]));
                __syncwarp();
            }
            if (!__all_sync(0xFFFFFFFFu, wait(acc_full, tcount & 1))) break;
            tc_fence_after();
            uint32_t packed[64];
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                uint32_t raw[64];
                tmem_ld64(t_row + c * 64, raw);  // returns after tcgen05.wait::ld
                if (c == 1) {
                    // the whole accumulator is in registers: the next tile's MMAs may
                    // overwrite it while the second half is converted
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) arrive_leader(acc_empty);
                }
#pragma unroll
                for (int e = 0; e < 64; e += 4) {
                    uint32_t b0, b1, b2, b3;
                    ld_shared_v4(bias_w + (c * 64 + e) * 4, b0, b1, b2, b3);
                    packed[c * 32 + e / 2] = pack_bf16x2(fmaf(__uint_as_float(raw[e]), alpha, __uint_as_float(b0)),
                                                         fmaf(__uint_as_float(raw[e + 1]), alpha, __uint_as_float(b1)));
                    packed[c * 32 + e / 2 + 1] = pack_bf16x2(fmaf(__uint_as_float(raw[e + 2]), alpha, __uint_as_float(b2)),
                                                             fmaf(__uint_as_float(raw[e + 3]), alpha, __uint_as_float(b3)));
                }
            }
            const long long m0 = static_cast<long long>(tm) * 256 + static_cast<int>(rank) * 128 + quarter * 32;
            if (wide) {
                // through the warp's buffer, 64 columns at a time: lane r writes row r (16-byte
                // chunk c at position c ^ (r % 8), so the eight rows of a read hit distinct
                // banks), then each store instruction writes 128 bytes of each of 8 rows
                __syncwarp();  // every lane has read the bias
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
#pragma unroll
                    for (int c = 0; c < 8; ++c)
                        st_shared_v4(bias_w + lane * 128 + ((c ^ (lane & 7)) << 4), packed[32 * hh + 4 * c],
                                     packed[32 * hh + 4 * c + 1], packed[32 * hh + 4 * c + 2], packed[32 * hh + 4 * c + 3]);
                    __syncwarp();
                    const int col = n0 + hh * 64 + (lane & 3) * 16;
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int r = i * 8 + (lane >> 2);
                        const int c0 = (lane & 3) * 2;
                        uint32_t w[8];
                        ld_shared_v4(bias_w + r * 128 + ((c0 ^ (r & 7)) << 4), w[0], w[1], w[2], w[3]);
                        ld_shared_v4(bias_w + r * 128 + (((c0 + 1) ^ (r & 7)) << 4), w[4], w[5], w[6], w[7]);
                        if (m0 + r < p.M && col < p.N)
                            st_global_v8(p.c + (m0 + r) * p.N + col, w[0], w[1], w[2], w[3], w[4], w[5], w[6], w[7]);
                    }
                    __syncwarp();  // the buffer is read before it is written again
                }
            } else {
                if (m0 + lane < p.M) store_row128(p.c + (m0 + lane) * p.N, packed, n0, p.N, false);
                __syncwarp();  // every lane has read the bias before the next tile's is written
            }
        }
    } else {
        // ------------------------------------------------------------ scales (warps 10-13, both CTAs)
        // this CTA's scales of K-tile i into its TMEM region i % S, in the layout of the
        // one-CTA kernel (A: its 128 rows; B: all 256 rows of the tile)
        const int quarter = warp & 3;
        const int total = my_tiles * k_tiles;
        for (int i = 0; i < total; ++i) {
            const int s = i % kF2Stages;
            if (!__all_sync(0xFFFFFFFFu, wait(&sf_in[s], (i / kF2Stages) & 1))) break;
            const uint32_t base = smem_u32(smem + s * kF2StageBytes + 2 * kF2Half) + lane * 16;
            uint32_t va[16], vb[32];
#pragma unroll
            for (int kb = 0; kb < 4; ++kb) {
                ld_shared_v4(base + kb * 512, va[4 * kb], va[4 * kb + 1], va[4 * kb + 2], va[4 * kb + 3]);
#pragma unroll
                for (int g = 0; g < 2; ++g)
                    ld_shared_v4(base + kF2SfaBytes + g * 2048 + kb * 512, vb[8 * kb + 4 * g], vb[8 * kb + 4 * g + 1],
                                 vb[8 * kb + 4 * g + 2], vb[8 * kb + 4 * g + 3]);
            }
            const uint32_t t = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + kFp4ColSf +
                               static_cast<uint32_t>(s) * kFp4SfStageCols;
            tmem_st16(t, va);
            tmem_st32(t + 16, vb);
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) arrive_leader(&sf_full[s]);
        }
    }

    // neither CTA releases its shared memory or TMEM while the pair's copies, MMAs or
    // epilogue may still use them
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512) : "memory");
    }
}

}  // namespace sbsa
