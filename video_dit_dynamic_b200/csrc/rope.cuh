// Step 0, fused with step 1: 3D RoPE of Q and K, written back as bf16, and the block
// means of the rotated values.
//
// The pages replace 3D RoPE with a fused kernel to save temporaries and memory round
// trips (page "知识卡片：600倍加速，720p视频实时生成！单卡也能带的动14B模型", 方法/产品要点,
// bullet 高效推理算子; page "单卡 RTX 5090 跑 Wan2.2-A14B：720p 视频生成只要 3.8 秒",
// 四步拆解 item 4 融合内核).  Here the rotation is fused with the block-mean pooling that
// follows it, so Q and K make one trip through HBM for both.
//
// Rotation (the pages give no frequencies; this is the usual 3D split): the head
// dimension is cut into rotation pairs (2p, 2p+1); the first P_T = d/2 - 2 P_H pairs
// turn with the token's frame index, the next P_H = d/6 (integer) with its row index,
// the last P_W = P_H with its column index on the (T, H, W) latent grid (tokens in
// row-major order); pair q of an axis with P pairs turns by pos * theta^(-q/P).
// cos/sin come from a table built once per grid (rope_table_kernel, in double).
// Padded tokens (t >= L) have no grid position; they are passed through unrotated.
//
// HBM-bound: one CTA per (tensor, b, h, block), 256 threads.  The block's tile comes in
// and goes out with one bulk copy each; thread t owns the 16-byte chunk t % (d/8)
// (four rotation pairs) of rows t / (d/8), t / (d/8) + 256/(d/8), ..., rotates it in
// fp32, rounds to bf16 (ties to even) in place, and sums the rounded values of the
// valid rows for the mean.
#pragma once
#include "common.cuh"
#include "pool.cuh"
#include "ptx.cuh"

namespace sbsa {

template <int D>
struct RopeSplit {
    static constexpr int kPairs = D / 2;
    static constexpr int kH = D / 6, kW = D / 6, kT = kPairs - 2 * (D / 6);
};

// Number of float2 entries of the table for head dimension d on a (gt, gh, gw) grid:
// frame rows [gt][P_T], then [gh][P_H], then [gw][P_W].
inline long long rope_table_entries(int d, int gt, int gh, int gw) {
    const int ph = d / 6, pt = d / 2 - 2 * ph;
    return static_cast<long long>(gt) * pt + static_cast<long long>(gh) * ph + static_cast<long long>(gw) * ph;
}

// One thread per entry: (cos, sin) of pos * theta^(-q/P), computed in double.
__global__ void rope_table_kernel(int d, int gt, int gh, int gw, double theta, float2* __restrict__ table,
                                  long long n) {
    const long long e = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x;
    if (e >= n) return;
    const int ph = d / 6, pt = d / 2 - 2 * ph;
    const long long n_t = static_cast<long long>(gt) * pt, n_h = static_cast<long long>(gh) * ph;
    long long idx = e;
    int np;
    if (idx < n_t) {
        np = pt;
    } else if ((idx -= n_t) < n_h) {
        np = ph;
    } else {
        idx -= n_h;
        np = ph;
    }
    const long long pos = idx / np;
    const int q = static_cast<int>(idx % np);
    const double ang = static_cast<double>(pos) * pow(theta, -static_cast<double>(q) / np);
    double s, c;
    sincos(ang, &s, &c);
    table[e] = make_float2(static_cast<float>(c), static_cast<float>(s));
}

__device__ __forceinline__ void bulk_load_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(dst)),
                 "l"(src), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}
__device__ __forceinline__ void bulk_store_s2g(void* dst, const void* src, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(smem_u32(src)),
                 "r"(bytes)
                 : "memory");
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
__device__ __forceinline__ void bulk_store_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}

// The block's BLK x d bf16 tile is contiguous in memory: one bulk copy brings it into
// shared memory, the threads rotate it in place, and one bulk copy writes it back, so
// no register holds data in flight and many CTAs share an SM.  in and out may be the
// same tensor (each tile is read completely before it is written), so they carry no
// __restrict__.
template <int D, int BLK>
__global__ void __launch_bounds__(256) rope_pool_kernel(const uint4* q_in, const uint4* k_in, uint4* q_out,
                                                        uint4* k_out, const float2* __restrict__ table,
                                                        float* __restrict__ q_mean, float* __restrict__ k_mean,
                                                        int L, int Lp, int nb, int gh, int gw, int gt,
                                                        long long units_per_tensor, unsigned int epoch) {
    using S = RopeSplit<D>;
    constexpr int CH = D / 8;          // 16-byte chunks (four pairs each) per row
    constexpr int RG = 256 / CH;       // row groups
    constexpr int ITER = BLK / RG;     // rows per thread
    constexpr uint32_t kTileBytes = BLK * D * 2;
    static_assert(BLK % RG == 0, "block must be a multiple of the row-group count");
    __shared__ __align__(128) uint4 tile[BLK * CH];
    __shared__ float red[8][D];
    __shared__ __align__(8) uint64_t full;

    long long u = blockIdx.x;
    const bool is_k = u >= units_per_tensor;
    if (is_k) u -= units_per_tensor;
    const long long bh = u / nb;
    const int i = static_cast<int>(u % nb);
    const int t0 = i * BLK;
    const int nvalid = min(BLK, L - t0);
    const long long base = (static_cast<long long>(bh) * Lp + t0) * CH;

    if (threadIdx.x == 0) {
        mbar_init(&full, 1);
        fence_mbar_init();
        mbar_arrive_expect_tx(&full, kTileBytes);
        bulk_load_g2s(tile, (is_k ? k_in : q_in) + base, kTileBytes, &full);
    }
    const int c = threadIdx.x % CH;
    const int g = threadIdx.x / CH;

    // the four pairs of this chunk: their axis (0 frame, 1 row, 2 column), the table
    // entry of position 0 and the entries per position step
    int axis[4], entry0[4], step[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int p = 4 * c + j;
        if (p < S::kT) {
            axis[j] = 0;
            entry0[j] = p;
            step[j] = S::kT;
        } else if (p < S::kT + S::kH) {
            axis[j] = 1;
            entry0[j] = gt * S::kT + (p - S::kT);
            step[j] = S::kH;
        } else {
            axis[j] = 2;
            entry0[j] = gt * S::kT + gh * S::kH + (p - S::kT - S::kH);
            step[j] = S::kW;
        }
    }
    // grid position of this thread's first row, then stepped by RG rows (t < L only:
    // padded tokens have no grid position and pass through unrotated)
    const int tf = t0 + g;
    int pf = tf / (gh * gw), ph = (tf / gw) % gh, pw = tf % gw;

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

    float a[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll
    for (int it = 0; it < ITER; ++it) {
        const int r = g + it * RG;
        const bool valid = r < nvalid;
        uint4& cell = tile[r * CH + c];
        const uint4 w = cell;
        const uint32_t in[4] = {w.x, w.y, w.z, w.w};
        uint32_t out[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int pos = axis[j] == 0 ? pf : (axis[j] == 1 ? ph : pw);
            // the index stays inside the table for every row; padded rows use the identity
            const float2 tc = __ldg(table + (valid ? entry0[j] + pos * step[j] : 0));
            const float2 cs = valid ? tc : make_float2(1.f, 0.f);
            const float x = __uint_as_float(in[j] << 16), y = __uint_as_float(in[j] & 0xFFFF0000u);
            out[j] = pack_bf16x2(x * cs.x - y * cs.y, x * cs.y + y * cs.x);
        }
        const uint4 o = make_uint4(out[0], out[1], out[2], out[3]);
        cell = o;
        if (valid) acc_bf16x8(a, o);
        // advance the grid position by RG tokens
        pw += RG;
        while (pw >= gw) {
            pw -= gw;
            if (++ph == gh) {
                ph = 0;
                ++pf;
            }
        }
    }
    fence_proxy_async_smem();  // the rotated tile is read by the async proxy next
    __syncthreads();
    if (threadIdx.x == 0) bulk_store_s2g((is_k ? k_out : q_out) + base, tile, kTileBytes);

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
        float* m = (is_k ? k_mean : q_mean) + u * D;
        m[threadIdx.x] = s / static_cast<float>(nvalid);
    }
    // the tile must stay in shared memory until the bulk store has read it
    if (threadIdx.x == 0) bulk_store_wait_read();
}

}  // namespace sbsa
