// Step 2: block scores and per-query-block top-k with the diagonal forced.
//
// The method keeps only ~10-20% of the key blocks per query block, chosen at run time
// from the block means (page "知识卡片：600倍加速，720p视频实时生成！单卡也能带的动14B模型",
// 方法/产品要点, bullet 动态稀疏量化注意力).  Score of (i, j) = <qmean_i, kmean_j> in
// fp32.  Kept: j = i, plus the k-1 highest-scoring j != i, ties to the lower j; written
// in ascending j order into a CSR list with a uniform row length k.
//
// One CTA per (b*h, tile of QT query blocks), 256 threads.
//   scores : each thread takes one key block j at a time, holds kmean_j in registers
//            and forms its dot product with the QT query means broadcast from shared
//            memory; the fp32 scores go to shared memory as order-preserving uint32 keys.
//   top-k  : one warp per query row.  Lane l holds keys j = l + 32 r.  The (k-1)-th
//            largest key T is found by bisection on the key bits (warp-wide counts,
//            early exit); then keys > T are kept, and keys == T in ascending j until k-1
//            are kept; the output position of each kept j is a ballot prefix count,
//            which yields the ascending order directly.
#pragma once
#include "common.cuh"

namespace sbsa {

// fp32 -> uint32 with the same order (larger float -> larger key).
__device__ __forceinline__ uint32_t order_key(float s) {
    const uint32_t u = __float_as_uint(s);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Keep, for query block i, the diagonal and the k_keep-1 largest of the other keys
// (ties: lower j), writing them in ascending j.  One warp; lane l holds keys
// j = l + 32 s.  The (k-1)-th largest key T is found by bisection on the key bits with
// warp-wide counts, stopping early once exactly k-1 keys lie at or above the candidate.
template <int KPL>
__device__ __forceinline__ void select_row_topk(const uint32_t* __restrict__ keys_row, int nb, int i, int k_keep,
                                                long long row, int32_t* __restrict__ row_ptr,
                                                int32_t* __restrict__ col_idx) {
    const int lane = threadIdx.x % 32;
    const uint32_t lt = lanemask_lt();
    const int kk = k_keep - 1;  // off-diagonal blocks to keep
    uint32_t key[KPL];
#pragma unroll
    for (int s = 0; s < KPL; ++s) {
        const int j = s * 32 + lane;
        // non-candidates (padding, the diagonal) get key 0; every bisection candidate is
        // >= 1, so they never count (a real score's key is >= 1: only the all-ones NaN
        // pattern maps to 0, and it is clamped to 1)
        key[s] = (j < nb && j != i) ? max(keys_row[j], 1u) : 0u;
    }
    // The (k-1)-th largest candidate key T: a search over the key range [lo, hi) with
    // count(key >= lo) >= k-1 > count(key >= hi).  Each probe is placed where the
    // counts at the two ends put it if the keys were spread evenly in between
    // (interpolation), with a halving probe after any interpolation that did not at
    // least halve the range, so the search never takes more than twice the 33 steps
    // of plain bisection.  It stops early when exactly k-1 keys are >= the probe.
    uint32_t T = 0u;
    if (kk > 0) {
        uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
        int nc = 0;
#pragma unroll
        for (int s = 0; s < KPL; ++s) {
            if (key[s] != 0u) {
                kmin = min(kmin, key[s]);
                ++nc;
            }
            kmax = max(kmax, key[s]);
        }
        uint32_t lo = __reduce_min_sync(0xFFFFFFFFu, kmin);
        const uint32_t top = __reduce_max_sync(0xFFFFFFFFu, kmax);
        int c_lo = __reduce_add_sync(0xFFFFFFFFu, nc);  // candidates: count(key >= lo)
        int c_hi = 0;
        // hi = top + 1 as a 64-bit bound: top can be the largest key
        uint64_t hi = static_cast<uint64_t>(top) + 1u;
        bool halve = false;
        T = lo;
#pragma unroll 1
        for (int it = 0; it < 72 && hi - lo > 1u; ++it) {
            const uint64_t range = hi - lo;
            uint64_t off;
            if (halve) {
                off = range >> 1;
            } else {
                const float f = static_cast<float>(c_lo - kk) / static_cast<float>(c_lo - c_hi);
                off = static_cast<uint64_t>(f * static_cast<float>(range));
            }
            off = off < 1u ? 1u : (off > range - 1u ? range - 1u : off);
            const uint32_t cand = static_cast<uint32_t>(lo + off);
            // four independent partial counts keep the add chains short
            int c4[4] = {0, 0, 0, 0};
#pragma unroll
            for (int s = 0; s < KPL; ++s) c4[s & 3] += key[s] >= cand ? 1 : 0;
            const int cnt = __reduce_add_sync(0xFFFFFFFFu, (c4[0] + c4[1]) + (c4[2] + c4[3]));
            if (cnt == kk) {  // {key >= cand} is exactly the top k-1
                T = cand;
                break;
            }
            if (cnt > kk) {
                lo = cand;
                c_lo = cnt;
            } else {
                hi = cand;
                c_hi = cnt;
            }
            T = lo;
            halve = !halve && 2u * (hi - lo) > range;
        }
    }
    int n_gt = 0;
    if (kk > 0) {
        int g4[4] = {0, 0, 0, 0};
#pragma unroll
        for (int s = 0; s < KPL; ++s) g4[s & 3] += key[s] > T ? 1 : 0;
        n_gt = __reduce_add_sync(0xFFFFFFFFu, (g4[0] + g4[1]) + (g4[2] + g4[3]));
    }
    const int need_eq = kk - n_gt;  // how many keys equal to T to keep (lowest j first)
    int32_t* out = col_idx + row * k_keep;
    int pos = 0, eq_seen = 0;
#pragma unroll
    for (int s = 0; s < KPL; ++s) {
        const int j = s * 32 + lane;
        const bool cand = key[s] != 0u;  // j < nb and j != i
        const bool is_eq = kk > 0 && cand && key[s] == T;
        const uint32_t eq_mask = __ballot_sync(0xFFFFFFFFu, is_eq);
        const int eq_rank = eq_seen + __popc(eq_mask & lt);
        const bool keep = (j == i) || (kk > 0 && cand && key[s] > T) || (is_eq && eq_rank < need_eq);
        const uint32_t m = __ballot_sync(0xFFFFFFFFu, keep);
        if (keep) out[pos + __popc(m & lt)] = j;
        pos += __popc(m);
        eq_seen += __popc(eq_mask);
    }
    if (lane == 0) row_ptr[row] = static_cast<int32_t>(row * k_keep);
}

template <int D, int QT, int KPL>
__global__ void __launch_bounds__(256) select_kernel(const float* __restrict__ q_mean,
                                                     const float* __restrict__ k_mean, int nb, int k_keep,
                                                     int32_t* __restrict__ row_ptr, int32_t* __restrict__ col_idx,
                                                     long long n_rows) {
    extern __shared__ __align__(16) uint8_t sel_smem[];
    float* qs = reinterpret_cast<float*>(sel_smem);                    // [QT][D]
    uint32_t* keys = reinterpret_cast<uint32_t*>(qs + QT * D);         // [QT][32*KPL]
    constexpr int NBP = 32 * KPL;

    const long long bh = blockIdx.y;
    const int i0 = blockIdx.x * QT;
    const int nq = min(QT, nb - i0);
    const float* qm = q_mean + (bh * nb + i0) * D;
    const float* km = k_mean + bh * nb * D;

    for (int e = threadIdx.x; e < QT * D; e += blockDim.x) qs[e] = e < nq * D ? qm[e] : 0.f;
    __syncthreads();

    // ---- scores
    for (int j = threadIdx.x; j < nb; j += blockDim.x) {
        float kr[D];
        const float4* kj = reinterpret_cast<const float4*>(km + static_cast<long long>(j) * D);
#pragma unroll
        for (int c4 = 0; c4 < D / 4; ++c4) {
            const float4 t = __ldg(kj + c4);
            kr[4 * c4] = t.x; kr[4 * c4 + 1] = t.y; kr[4 * c4 + 2] = t.z; kr[4 * c4 + 3] = t.w;
        }
#pragma unroll 1
        for (int r = 0; r < QT; ++r) {
            const float4* qr = reinterpret_cast<const float4*>(qs + r * D);
            float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
#pragma unroll
            for (int c4 = 0; c4 < D / 4; ++c4) {
                const float4 t = qr[c4];
                s0 = fmaf(t.x, kr[4 * c4], s0);
                s1 = fmaf(t.y, kr[4 * c4 + 1], s1);
                s2 = fmaf(t.z, kr[4 * c4 + 2], s2);
                s3 = fmaf(t.w, kr[4 * c4 + 3], s3);
            }
            keys[r * NBP + j] = order_key((s0 + s1) + (s2 + s3));
        }
    }
    __syncthreads();

    // ---- top-k per row, one warp per row
    const int warp = threadIdx.x / 32;
    for (int r = warp; r < nq; r += blockDim.x / 32)
        select_row_topk<KPL>(keys + r * NBP, nb, i0 + r, k_keep, bh * nb + i0 + r, row_ptr, col_idx);
    if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) row_ptr[n_rows] = static_cast<int32_t>(n_rows * k_keep);
}

// Scores through a shared-memory, register-blocked fp32 GEMM, for nb <= 1024.
// CTA = (b*h, 32 query blocks), 256 threads.  Key means stream through shared memory
// in chunks of 256 key blocks x 32 channels.  Thread (warp w, lane l) owns query rows
// {l/8 + 4 r : r < 8} and key blocks {256 c + 32 w + l%8 + 8 s : s < 4}; rows and key
// blocks interleave so that each shared-memory load is conflict-free or broadcast.
// Products accumulate over channel pairs with packed fp32x2 FMAs, (even, odd) channel
// partial sums added at the end.  Then one warp per row selects as above.
constexpr int kSelQT = 32;
constexpr int kSelQStride = 132;  // floats per query-mean row in shared memory (128 + 4)
constexpr int kSelKStride = 36;   // floats per key-mean row of a 32-channel chunk (32 + 4)
constexpr int kSelJChunk = 256;
constexpr int kSelCChunk = 32;

template <int KPL>
__global__ void __launch_bounds__(256, 1) select_gemm_kernel(const float* __restrict__ q_mean,
                                                            const float* __restrict__ k_mean, int nb, int k_keep,
                                                            int32_t* __restrict__ row_ptr,
                                                            int32_t* __restrict__ col_idx, long long n_rows) {
    constexpr int D = 128;
    constexpr int NBP = 32 * KPL;
    extern __shared__ __align__(16) uint8_t sel_smem[];
    float* qs = reinterpret_cast<float*>(sel_smem);                        // [32][132]
    float* ks = qs + kSelQT * kSelQStride;                                 // [2][256][36]
    uint32_t* keys = reinterpret_cast<uint32_t*>(ks + 2 * kSelJChunk * kSelKStride);  // [32][NBP]

    const long long bh = blockIdx.y;
    const int i0 = blockIdx.x * kSelQT;
    const int nq = min(kSelQT, nb - i0);
    const float* qm = q_mean + (bh * nb + i0) * D;
    const float* km = k_mean + bh * nb * D;
    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;

    // query means -> qs (rows past nq are zero)
    for (int f = tid; f < kSelQT * D / 4; f += 256) {
        const int r = f / (D / 4), c4 = f % (D / 4);
        const float4 v = r < nq ? __ldg(reinterpret_cast<const float4*>(qm) + f) : make_float4(0.f, 0.f, 0.f, 0.f);
        *reinterpret_cast<float4*>(qs + r * kSelQStride + c4 * 4) = v;
    }

    const int li = lane / 8, lj = lane % 8;
    auto load_chunk = [&](int jc, int cc, float* dst) {
        // 256 key rows x 32 channels = 2048 x 16 B, 8 per thread, asynchronous copies
        // (coalesced along channels; rows past nb are zero-filled)
#pragma unroll
        for (int r = 0; r < 8; ++r) {
            const int f = tid + 256 * r;
            const int row = f / 8, q4 = f % 8;
            const int j = jc + row;
            const float* src = km + static_cast<long long>(j < nb ? j : 0) * D + cc * kSelCChunk + q4 * 4;
            const uint32_t dst_s = smem_u32(dst + row * kSelKStride + q4 * 4);
            const uint32_t bytes = j < nb ? 16u : 0u;
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst_s), "l"(src), "r"(bytes) : "memory");
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };

    for (int jc = 0; jc < nb; jc += kSelJChunk) {
        float2 acc[8][4];
#pragma unroll
        for (int a = 0; a < 8; ++a)
#pragma unroll
            for (int b = 0; b < 4; ++b) acc[a][b] = make_float2(0.f, 0.f);
        __syncthreads();  // previous chunk's readers are done with ks
        if (jc == 0) load_chunk(0, 0, ks);  // later chunks' first slice was prefetched below
        for (int cc = 0; cc < D / kSelCChunk; ++cc) {
            float* cur = ks + (cc & 1) * kSelJChunk * kSelKStride;
            asm volatile("cp.async.wait_group 0;" ::: "memory");
            __syncthreads();  // cur is filled for every thread; the other buffer is free
            if (cc + 1 < D / kSelCChunk)
                load_chunk(jc, cc + 1, ks + ((cc + 1) & 1) * kSelJChunk * kSelKStride);
            else if (jc + kSelJChunk < nb)
                load_chunk(jc + kSelJChunk, 0, ks + ((cc + 1) & 1) * kSelJChunk * kSelKStride);
#pragma unroll
            for (int c = 0; c < kSelCChunk; c += 4) {
                float4 qv[8], kv[4];
#pragma unroll
                for (int a = 0; a < 8; ++a)
                    qv[a] = *reinterpret_cast<const float4*>(qs + (li + 4 * a) * kSelQStride + cc * kSelCChunk + c);
#pragma unroll
                for (int b = 0; b < 4; ++b)
                    kv[b] = *reinterpret_cast<const float4*>(cur + (warp * 32 + lj + 8 * b) * kSelKStride + c);
#pragma unroll
                for (int a = 0; a < 8; ++a)
#pragma unroll
                    for (int b = 0; b < 4; ++b) {
                        acc[a][b] = __ffma2_rn(make_float2(qv[a].x, qv[a].y), make_float2(kv[b].x, kv[b].y), acc[a][b]);
                        acc[a][b] = __ffma2_rn(make_float2(qv[a].z, qv[a].w), make_float2(kv[b].z, kv[b].w), acc[a][b]);
                    }
            }
        }
#pragma unroll
        for (int a = 0; a < 8; ++a)
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                const int j = jc + warp * 32 + lj + 8 * b;
                if (j < NBP) keys[(li + 4 * a) * NBP + j] = order_key(acc[a][b].x + acc[a][b].y);
            }
    }
    __syncthreads();

    for (int r = warp; r < nq; r += 8)
        select_row_topk<KPL>(keys + r * NBP, nb, i0 + r, k_keep, bh * nb + i0 + r, row_ptr, col_idx);
    if (blockIdx.x == 0 && blockIdx.y == 0 && tid == 0) row_ptr[n_rows] = static_cast<int32_t>(n_rows * k_keep);
}

constexpr size_t select_gemm_smem_bytes(int KPL) {
    return (static_cast<size_t>(kSelQT) * kSelQStride + 2ull * kSelJChunk * kSelKStride) * 4 +
           static_cast<size_t>(kSelQT) * 32 * KPL * 4;
}

}  // namespace sbsa
