// Step 2: block scores and per-query-block top-k with the diagonal forced.
//
// The method keeps only ~10-20% of the key blocks per query block, chosen at run time
// from the block means (page "知识卡片：600倍加速，720p视频实时生成！单卡也能带的动14B模型",
// 方法/产品要点, bullet 动态稀疏量化注意力).  Score of (i, j) = <qmean_i, kmean_j> in
// fp32.  Kept: j = i, plus the k-1 highest-scoring j != i, ties to the lower j; written
// in ascending j order into a CSR list with a uniform row length k.
//
// Two kernels share the top-k:
//   select_tc_kernel (head_dim 128, nb <= 1024): scores on the tensor cores in tf32 with
//     an exact three-product split, described above the kernel.
//   select_kernel (other shapes): one CTA per (b*h, tile of QT query blocks); each thread
//     takes one key block j at a time, holds kmean_j in registers and forms its dot
//     product with the QT query means broadcast from shared memory.
// Scores go to shared memory as order-preserving uint32 keys.  Top-k: one warp per
// query row, lane l holding keys j = l + 32 r; the (k-1)-th largest key T comes from a
// search with warp-wide counts, starting at the threshold of the warp's previous
// (neighbouring) row; keys > T are kept, and keys == T in ascending j until k-1 are
// kept; the keep bits are transposed with ballots into one 32-block word per lane, and a
// prefix sum of the words' counts places every kept j in ascending order.
#pragma once
#include <type_traits>

// 1: the tensor-core selection's top-k counts on the floating-point pipe
// (select_row_topk_f); 0: on the integer pipe (select_row_topk).
#ifndef SBSA_SELECT_FCOUNT
#define SBSA_SELECT_FCOUNT 1
#endif

#include "common.cuh"
#include "ptx.cuh"

namespace sbsa {

constexpr bool kSelFloatCount = SBSA_SELECT_FCOUNT != 0;

// fp32 -> uint32 with the same order (larger float -> larger key).
__device__ __forceinline__ uint32_t order_key(float s) {
    const uint32_t u = __float_as_uint(s);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Keep, for query block i, the diagonal and the k_keep-1 largest of the other keys
// (ties: lower j), writing them in ascending j.  One warp; lane l holds keys
// j = l + 32 s.  `hint` carries the threshold key found for the warp's previous row (0
// for none): rows handled one after the other by a warp are neighbouring query blocks,
// whose score rows are alike, so it is tried as the first probe.
template <int KPL>
__device__ __forceinline__ void select_row_topk(const uint32_t* __restrict__ keys_row, int nb, int i, int k_keep,
                                                long long row, int32_t* __restrict__ row_ptr,
                                                int32_t* __restrict__ col_idx, uint32_t& hint) {
    static_assert(KPL <= 64, "at most two output words per lane");
    using Mask = typename std::conditional<(KPL > 32), unsigned long long, uint32_t>::type;
    const int lane = threadIdx.x % 32;
    const uint32_t lt = lanemask_lt();
    const int kk = k_keep - 1;  // off-diagonal blocks to keep
    uint32_t key[KPL];
#pragma unroll
    for (int s = 0; s < KPL; ++s) {
        const int j = s * 32 + lane;
        // non-candidates (padding, the diagonal) get key 0; every search candidate is
        // >= 1, so they never count (a real score's key is >= 1: only the all-ones NaN
        // pattern maps to 0, and it is clamped to 1)
        key[s] = (j < nb && j != i) ? max(keys_row[j], 1u) : 0u;
    }
    // The (k-1)-th largest candidate key T: a search over the key range [lo, hi) with
    // count(key >= lo) >= k-1 > count(key >= hi).  The first probe is the hint when it
    // lies inside the range; then each probe is placed where the counts at the two ends
    // put it if the keys were spread evenly in between (interpolation), with a halving
    // probe after any interpolation that did not at least halve the range, so the search
    // never takes more than twice the 33 steps of plain bisection (plus the hint).  It
    // stops early when exactly k-1 keys are >= the probe ("exact": then no key needs a
    // tie decision).
    uint32_t T = 0u;
    bool exact = kk == 0;
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
        // keys of finite scores are at most 0xFF7FFFFF, so hi = top + 1 fits in 32 bits
        // (the clamp only matters for a NaN score, which the caller rules out)
        uint32_t hi = min(__reduce_max_sync(0xFFFFFFFFu, kmax), 0xFFFFFFFEu) + 1u;
        int c_lo = __reduce_add_sync(0xFFFFFFFFu, nc);  // candidates: count(key >= lo)
        int c_hi = 0;
        bool halve = false;
        bool use_hint = hint > lo && hint < hi;
        T = lo;
#pragma unroll 1
        for (int it = 0; it < 73 && hi - lo > 1u; ++it) {
            const uint32_t range = hi - lo;
            uint32_t cand;
            if (use_hint) {
                cand = hint;
                use_hint = false;
            } else {
                uint32_t off;
                if (halve) {
                    off = range >> 1;
                } else {
                    const float f = __fdividef(static_cast<float>(c_lo - kk), static_cast<float>(c_lo - c_hi));
                    off = static_cast<uint32_t>(f * static_cast<float>(range));
                }
                off = min(max(off, 1u), range - 1u);
                cand = lo + off;
            }
            // four independent partial counts keep the add chains short
            int c4[4] = {0, 0, 0, 0};
#pragma unroll
            for (int s = 0; s < KPL; ++s) c4[s & 3] += key[s] >= cand ? 1 : 0;
            const int cnt = __reduce_add_sync(0xFFFFFFFFu, (c4[0] + c4[1]) + (c4[2] + c4[3]));
            if (cnt == kk) {  // {key >= cand} is exactly the top k-1
                T = cand;
                exact = true;
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
            halve = !halve && 2ull * (hi - lo) > range;
        }
        hint = T;
    }
    // Keep bits of this lane's slots (bit s: j = s*32 + lane).  Keys equal to T are kept
    // lowest j first until k-1 are kept (only needed when the search ended on a key value
    // with ties possible).
    Mask mask = 0u;
    if (exact) {
#pragma unroll
        for (int s = 0; s < KPL; ++s) {
            const int j = s * 32 + lane;
            const bool keep = (j == i) || (kk > 0 && key[s] != 0u && key[s] >= T);
            mask |= keep ? (Mask(1) << s) : Mask(0);
        }
    } else {
        int g4[4] = {0, 0, 0, 0};
#pragma unroll
        for (int s = 0; s < KPL; ++s) g4[s & 3] += key[s] > T ? 1 : 0;
        const int need_eq = kk - __reduce_add_sync(0xFFFFFFFFu, (g4[0] + g4[1]) + (g4[2] + g4[3]));
        int eq_seen = 0;
#pragma unroll
        for (int s = 0; s < KPL; ++s) {
            const int j = s * 32 + lane;
            const bool cand = key[s] != 0u;  // j < nb and j != i
            const bool is_eq = cand && key[s] == T;
            const uint32_t eq_mask = __ballot_sync(0xFFFFFFFFu, is_eq);
            const bool keep = (j == i) || (cand && key[s] > T) || (is_eq && eq_seen + __popc(eq_mask & lt) < need_eq);
            eq_seen += __popc(eq_mask);
            mask |= keep ? (Mask(1) << s) : Mask(0);
        }
    }
    // Transpose the keep bits: lane w gathers word w (and w + 32 when KPL > 32), whose bit
    // l is slot w of lane l, i.e. block j = 32 w + l.  Ascending j is then ascending word,
    // then ascending bit: a prefix sum of the words' counts gives each lane where its
    // blocks go.
    constexpr int NW = (KPL + 31) / 32;
    uint32_t word[NW];
#pragma unroll
    for (int w = 0; w < NW; ++w) word[w] = 0u;
#pragma unroll
    for (int s = 0; s < KPL; ++s) {
        const uint32_t b = __ballot_sync(0xFFFFFFFFu, static_cast<uint32_t>(mask >> s) & 1u);
        word[s / 32] = lane == (s % 32) ? b : word[s / 32];
    }
    int32_t* out = col_idx + row * k_keep;
    int base = 0;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
        const int cnt = __popc(word[w]);
        int incl = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int t = __shfl_up_sync(0xFFFFFFFFu, incl, o);
            if (lane >= o) incl += t;
        }
        int pos = base + incl - cnt;
        uint32_t bits = word[w];
        while (bits) {
            const int b = __ffs(static_cast<int>(bits)) - 1;
            out[pos++] = 32 * (32 * w + lane) + b;
            bits &= bits - 1u;
        }
        base += __shfl_sync(0xFFFFFFFFu, incl, 31);
    }
    if (lane == 0) row_ptr[row] = static_cast<int32_t>(row * k_keep);
    __syncwarp();
}

// The float whose order key is k (k the key of a finite float).
__device__ __forceinline__ float key_float(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

// f with key(s) >= c exactly when s > f, for scores s that are never -0 (the caller adds
// +0 to each): the float whose key is c - 1, stepped one key further down where that
// float is -0, which compares equal to the score +0 whose key is c.
__device__ __forceinline__ float float_below_key(uint32_t c) {
    const uint32_t k = c - 1u;
    return key_float(k == 0x7FFFFFFFu ? k - 1u : k);
}

// select_row_topk with the row's scores kept as floats (the shared-memory row holds their
// bit patterns): the search is the same, over the same order keys, but each probe's count
// of keys >= cand is taken on the floating-point pipe -- key(s) >= cand exactly when
// s > f, f = float_below_key(cand), and s > f exactly when (s - f) * inf
// saturates to 1 (it gives +inf there, -inf below and NaN at equality, which saturate to
// 1, 0 and 0) -- where the integer form spends two integer instructions per key on the
// integer pipe, which the top-k otherwise saturates.  Non-candidates are -inf.
template <int KPL>
__device__ __forceinline__ void select_row_topk_f(const uint32_t* __restrict__ row_bits, int nb, int i, int k_keep,
                                                  long long row, int32_t* __restrict__ row_ptr,
                                                  int32_t* __restrict__ col_idx, uint32_t& hint) {
    static_assert(KPL <= 32, "one output word per lane");
    const int lane = threadIdx.x % 32;
    const uint32_t lt = lanemask_lt();
    const int kk = k_keep - 1;  // off-diagonal blocks to keep
    float sv[KPL];
#pragma unroll
    for (int s = 0; s < KPL; ++s) {
        const int j = s * 32 + lane;
        // + 0 turns a -0 score into +0, so that float order and key order agree
        sv[s] = (j < nb && j != i) ? __fadd_rn(__uint_as_float(row_bits[j]), 0.f) : -INFINITY;
    }
    // The search of select_row_topk over order keys: count(key >= lo) >= k-1 > count(key >= hi).
    uint32_t T = 0u;
    bool exact = kk == 0;
    if (kk > 0) {
        // -inf (the non-candidates) never wins a min over the candidates' +inf start;
        // the max of the non-candidates is -inf, below every candidate
        float fmin = INFINITY, fmax = -INFINITY;
#pragma unroll
        for (int s = 0; s < KPL; ++s) {
            fmin = fminf(fmin, sv[s] == -INFINITY ? INFINITY : sv[s]);
            fmax = fmaxf(fmax, sv[s]);
        }
        uint32_t lo = __reduce_min_sync(0xFFFFFFFFu, order_key(fmin));
        // keys of finite scores are at most 0xFF7FFFFF, so hi = top + 1 fits in 32 bits
        uint32_t hi = min(__reduce_max_sync(0xFFFFFFFFu, order_key(fmax)), 0xFFFFFFFEu) + 1u;
        int c_lo = nb - 1;  // candidates: every block but the diagonal, count(key >= lo)
        int c_hi = 0;
        bool halve = false;
        bool use_hint = hint > lo && hint < hi;
        T = lo;
#pragma unroll 1
        for (int it = 0; it < 73 && hi - lo > 1u; ++it) {
            const uint32_t range = hi - lo;
            uint32_t cand;
            if (use_hint) {
                cand = hint;
                use_hint = false;
            } else {
                uint32_t off;
                if (halve) {
                    off = range >> 1;
                } else {
                    const float f = __fdividef(static_cast<float>(c_lo - kk), static_cast<float>(c_lo - c_hi));
                    off = static_cast<uint32_t>(f * static_cast<float>(range));
                }
                off = min(max(off, 1u), range - 1u);
                cand = lo + off;
            }
            // count(key >= cand) = count(s > f): lo < cand, so cand - 1 is a finite float's key;
            // the differences and the sums two keys at a time (packed fp32)
            const float f = float_below_key(cand);
            const float2 nf2 = make_float2(-f, -f);
            float2 a2[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
            for (int s = 0; s + 1 < KPL; s += 2) {
                const float2 d = __fadd2_rn(make_float2(sv[s], sv[s + 1]), nf2);
                a2[(s >> 1) & 3] = __fadd2_rn(a2[(s >> 1) & 3], make_float2(__saturatef(__fmul_rn(d.x, INFINITY)),
                                                                            __saturatef(__fmul_rn(d.y, INFINITY))));
            }
            const float2 a01 = __fadd2_rn(a2[0], a2[1]), a23 = __fadd2_rn(a2[2], a2[3]);
            const float2 aa = __fadd2_rn(a01, a23);
            const int cnt = __reduce_add_sync(0xFFFFFFFFu, __float2int_rn(aa.x + aa.y));
            if (cnt == kk) {  // {key >= cand} is exactly the top k-1
                T = cand;
                exact = true;
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
            halve = !halve && 2ull * (hi - lo) > range;
        }
        hint = T;
    }
    // Ascending output: the ballot of slot s over the lanes is the 32-block word of blocks
    // 32 s .. 32 s + 31; lane w keeps word w.  The diagonal is added to its word.
    uint32_t word = 0u;
    if (exact) {
        // keep key(s) >= T, i.e. s > the float whose key is T - 1 (T > 0 whenever k > 1)
        const float f = kk > 0 ? float_below_key(T) : INFINITY;
#pragma unroll
        for (int s = 0; s < KPL; ++s) {
            const uint32_t b = __ballot_sync(0xFFFFFFFFu, sv[s] > f);
            word = lane == s ? b : word;
        }
    } else {
        // keys > T kept, and keys == T lowest j first until k-1 are kept
        int g4[4] = {0, 0, 0, 0};
#pragma unroll
        for (int s = 0; s < KPL; ++s) g4[s & 3] += (sv[s] != -INFINITY && order_key(sv[s]) > T) ? 1 : 0;
        const int need_eq = kk - __reduce_add_sync(0xFFFFFFFFu, (g4[0] + g4[1]) + (g4[2] + g4[3]));
        int eq_seen = 0;
#pragma unroll
        for (int s = 0; s < KPL; ++s) {
            const bool cand = sv[s] != -INFINITY;
            const uint32_t key = cand ? order_key(sv[s]) : 0u;
            const bool is_eq = cand && key == T;
            const uint32_t eq_mask = __ballot_sync(0xFFFFFFFFu, is_eq);
            const bool keep = (cand && key > T) || (is_eq && eq_seen + __popc(eq_mask & lt) < need_eq);
            eq_seen += __popc(eq_mask);
            const uint32_t b = __ballot_sync(0xFFFFFFFFu, keep);
            word = lane == s ? b : word;
        }
    }
    if (lane == i / 32) word |= 1u << (i % 32);  // the diagonal
    const int cnt = __popc(word);
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += t;
    }
    int32_t* out = col_idx + row * k_keep;
    int pos = incl - cnt;
    while (word) {
        const int b = __ffs(static_cast<int>(word)) - 1;
        out[pos++] = 32 * lane + b;
        word &= word - 1u;
    }
    if (lane == 0) row_ptr[row] = static_cast<int32_t>(row * k_keep);
    __syncwarp();
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

    // ---- top-k per row, one warp per row; each warp takes neighbouring rows
    const int warp = threadIdx.x / 32;
    constexpr int kRowsPerWarp = QT / 8;
    static_assert(QT % 8 == 0, "eight warps share the rows");
    uint32_t hint = 0u;
#pragma unroll 1
    for (int q = 0; q < kRowsPerWarp; ++q) {
        const int r = warp * kRowsPerWarp + q;
        if (r < nq) select_row_topk<KPL>(keys + r * NBP, nb, i0 + r, k_keep, bh * nb + i0 + r, row_ptr, col_idx, hint);
    }
    if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) row_ptr[n_rows] = static_cast<int32_t>(n_rows * k_keep);
}

// ---------------------------------------------------------------- tensor-core scores
// Scores of 32 query blocks against all key blocks of one (b, h) on the tensor cores, in
// the transposed form S^T = Kmean . Qmean^T: M = 128 key blocks per tile (TMEM lane =
// key block, column = query block), N = 32 query blocks, K = d = 128, kind::tf32.
// fp32 accuracy from three products per K step: each mean x is split exactly into
// x_t = x with its 13 low mantissa bits cleared (a value tf32 holds exactly) and
// x_l = x - x_t; s = k_t.q_t + k_t.q_l + k_l.q_t drops only k_l.q_l and the tf32
// rounding of the small parts, about 2^-19 of |k||q| per product, below the fp32
// rounding of a 128-term sum.  Both parts are written into the operand buffers
// explicitly (x_t over the raw means in place), so the result does not depend on how
// the tensor core converts an fp32 operand that is not already a tf32 value.
//
// CTA = (b*h, 32 query blocks), 320 threads, two CTAs per SM:
//   warp 8  : TMA of the raw means (box 32 channels x rows, 128-byte swizzle: the
//             K-major operand layout): the Q tile once, then K chunks (128 key blocks x
//             32 channels) through a three-slot ring.
//   warp 9  : TMEM allocation (256 columns: 8 key tiles x 32 query blocks) and the thread
//             that issues the MMAs, 12 per chunk ((k_t,q_t), (k_t,q_l), (k_l,q_t) at 4 K
//             steps).
//   warps 0-7: split the Q tile once and every K chunk into (x_t in place, x_l in one of
//             two buffers); then read the scores
//             out of TMEM into shared memory as order-preserving keys, 16 query rows at a
//             time, and run the warp-per-row top-k.
constexpr int kSelTcRows = 32;                  // query blocks per CTA
constexpr int kSelTcThreads = 320;
constexpr int kSelTcTile = 128 * 128;           // bytes of one K chunk (128 rows x 32 fp32)
constexpr int kSelTcQBytes = 4 * 32 * 128;      // Q tile: 4 channel chunks x 32 rows x 128 B
constexpr int kSelTcOffQ = 0, kSelTcOffQl = kSelTcQBytes, kSelTcOffX = 2 * kSelTcQBytes;
constexpr int kSelTcStages = 3;                // raw K chunks in flight
constexpr int kSelTcOffXl = kSelTcOffX + kSelTcStages * kSelTcTile;
constexpr int kSelTcOffBar = kSelTcOffXl + 2 * kSelTcTile;  // 112 KB of operands
// q_full, ql_full, x_full[S], x_empty[S], l_full[2], l_empty[2], done
constexpr int kSelTcNumBars = 2 + 2 * kSelTcStages + 2 + 2 + 1;
// No alignment slack: two CTAs must fit in one SM's 228 KB.  Dynamic shared memory
// starts 1024-byte aligned when the kernel has no static shared memory; the kernel
// checks that, and if it ever is not, latches SBSA_ERR_TIMEOUT and returns at once.
constexpr size_t kSelTcSmemBytes = kSelTcOffBar + kSelTcNumBars * 8 + 16;

constexpr uint32_t idesc_tf32_f32(int M, int N) {
    return (1u << 4) | (2u << 7) | (2u << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
           (static_cast<uint32_t>(M >> 4) << 24);
}
__device__ __forceinline__ void umma_tf32_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                             uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// x with its 13 low mantissa bits cleared (exact in tf32), for four floats
__device__ __forceinline__ float4 tf32_high_part(float4 v) {
    auto hi = [](float x) { return __uint_as_float(__float_as_uint(x) & 0xFFFFE000u); };
    return make_float4(hi(v.x), hi(v.y), hi(v.z), hi(v.w));
}
// x - (x with its 13 low mantissa bits cleared), exact, for four floats
__device__ __forceinline__ float4 tf32_low_part(float4 v, float4 h) {
    return make_float4(v.x - h.x, v.y - h.y, v.z - h.z, v.w - h.w);
}

struct SelTcParams {
    int nb, k_keep;
    long long n_rows;
    unsigned int epoch;
};

template <int KPL>
__global__ void __launch_bounds__(kSelTcThreads, 2) select_tc_kernel(const __grid_constant__ CUtensorMap map_q,
                                                                    const __grid_constant__ CUtensorMap map_k,
                                                                    int32_t* __restrict__ row_ptr,
                                                                    int32_t* __restrict__ col_idx,
                                                                    const SelTcParams p) {
    constexpr int NBP = 32 * KPL;                 // key slots per row (>= nb)
    constexpr int HALF = kSelTcRows / 2;          // query rows per top-k round
    static_assert(HALF * NBP * 4 <= kSelTcOffBar, "keys of one round fit over the operand buffers");
    extern __shared__ __align__(1024) uint8_t sel_tc_raw[];
    uint8_t* smem = sel_tc_raw;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kSelTcOffBar);
    uint64_t* q_full = bars;
    uint64_t* ql_full = bars + 1;
    constexpr int S = kSelTcStages;
    uint64_t* x_full = bars + 2;
    uint64_t* x_empty = x_full + S;
    uint64_t* l_full = x_empty + S;
    uint64_t* l_empty = l_full + 2;
    uint64_t* done = l_empty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kSelTcNumBars);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    uint32_t* keys = reinterpret_cast<uint32_t*>(smem);  // [HALF][NBP], after the MMAs

    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    // every thread takes the same branch (the barriers below need all of them)
    if (__syncthreads_or(launch_aborted(p.epoch) ? 1 : 0)) return;
    if (smem_u32(smem) & 1023u) {  // the swizzled operand layouts need 1024-byte alignment
        if (tid == 0) abort_launch(p.epoch);
        return;
    }
    const int nb = p.nb;
    const long long bh = blockIdx.y;
    const int i0 = blockIdx.x * kSelTcRows;
    const int nq = min(kSelTcRows, nb - i0);
    const int n_tiles = (nb + 127) / 128;
    const int n_chunks = 4 * n_tiles;

    if (tid == 256) {
        *abort_flag = 0;
        // ql_full and l_full[] count the 256 threads that write low parts; the rest one arrival
        for (int b = 0; b < kSelTcNumBars; ++b)
            mbar_init(&bars[b], (&bars[b] == ql_full || &bars[b] == &l_full[0] || &bars[b] == &l_full[1]) ? 256u : 1u);
        fence_mbar_init();
        tma_prefetch_desc(&map_q);
        tma_prefetch_desc(&map_k);
    }
    if (warp == 9) {
        tmem_alloc(tmem_slot, 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint64_t pipe_limit = pipe_wait_ns();  // pipeline waits; the drain keeps kWaitLimitNs
    auto wait = [&](uint64_t* bar, uint32_t parity) -> bool {
        if (mbar_wait_bounded(bar, parity, abort_flag, pipe_limit)) return true;
        if (!*abort_flag) {
            *abort_flag = 1;
            abort_launch(p.epoch);
        }
        return false;
    };
    bool ok = true;

    if (warp == 8) {
        // ---------------------------------------------------------------- TMA
        if (lane == 0) {
            const uint64_t pol = policy_evict_last();
            const int row_q = static_cast<int>(bh * nb + i0), row_k = static_cast<int>(bh * nb);
            mbar_arrive_expect_tx(q_full, kSelTcQBytes);
#pragma unroll
            for (int a = 0; a < 4; ++a) tma_load_2d(smem + kSelTcOffQ + a * 32 * 128, &map_q, q_full, 32 * a, row_q, pol);
            int c = 0;
            for (; c < n_chunks; ++c) {
                const int b = c % S;
                if (c >= S && !(ok = wait(&x_empty[b], ((c - S) / S) & 1))) break;
                mbar_arrive_expect_tx(&x_full[b], kSelTcTile);
                tma_load_2d(smem + kSelTcOffX + b * kSelTcTile, &map_k, &x_full[b], 32 * (c & 3), row_k + 128 * (c >> 2), pol);
            }
            if (!ok) {
                volatile int never = 0;
                mbar_wait_bounded(q_full, 0, &never, kWaitLimitNs);
                for (int q = c - S < 0 ? 0 : c - S; q < c; ++q) mbar_wait_bounded(&x_full[q % S], (q / S) & 1, &never, kWaitLimitNs);
            }
        }
    } else if (warp == 9) {
        // ---------------------------------------------------------------- MMA
        if (lane == 0) {
            constexpr uint32_t id = idesc_tf32_f32(128, kSelTcRows);
            const uint32_t q_addr = smem_u32(smem + kSelTcOffQ), ql_addr = smem_u32(smem + kSelTcOffQl);
            const uint32_t x_addr = smem_u32(smem + kSelTcOffX), xl_addr = smem_u32(smem + kSelTcOffXl);
            ok = wait(q_full, 0) && wait(ql_full, 0);
            for (int c = 0; ok && c < n_chunks; ++c) {
                const int b = c % S, lb = c & 1, t = c >> 2, dc = c & 3;
                if (!(ok = wait(&x_full[b], (c / S) & 1))) break;
                if (!(ok = wait(&l_full[lb], (c >> 1) & 1))) break;
                tc_fence_after();
                const uint32_t d = tmem + t * kSelTcRows;
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
                    const uint64_t xa = sdesc_sw128(x_addr + b * kSelTcTile + ks * 32, 16, 1024);
                    const uint64_t la = sdesc_sw128(xl_addr + lb * kSelTcTile + ks * 32, 16, 1024);
                    const uint64_t qb = sdesc_sw128(q_addr + dc * 32 * 128 + ks * 32, 16, 1024);
                    const uint64_t lb = sdesc_sw128(ql_addr + dc * 32 * 128 + ks * 32, 16, 1024);
                    umma_tf32_ss(d, xa, qb, id, (dc > 0 || ks > 0) ? 1u : 0u);
                    umma_tf32_ss(d, xa, lb, id, 1u);
                    umma_tf32_ss(d, la, qb, id, 1u);
                }
                umma_commit(&x_empty[b]);
                umma_commit(&l_empty[lb]);
            }
            umma_commit(done);  // every MMA this thread issued (also on the error path)
            if (!ok) {
                volatile int never = 0;
                mbar_wait_bounded(done, 0, &never, kWaitLimitNs);
            }
        }
    } else {
        // ---------------------------------------------------------------- low parts
        if ((ok = wait(q_full, 0))) {
#pragma unroll
            for (int u = 0; u < kSelTcQBytes / 16 / 256; ++u) {
                const int f = tid + 256 * u;
                const float4 v = reinterpret_cast<const float4*>(smem + kSelTcOffQ)[f];
                const float4 h = tf32_high_part(v);
                reinterpret_cast<float4*>(smem + kSelTcOffQ)[f] = h;
                reinterpret_cast<float4*>(smem + kSelTcOffQl)[f] = tf32_low_part(v, h);
            }
        }
        fence_proxy_async_smem();
        mbar_arrive(ql_full);
        for (int c = 0; ok && c < n_chunks; ++c) {
            const int b = c % S, lb = c & 1;
            if (!(ok = wait(&x_full[b], (c / S) & 1))) break;
            // the raw chunk in slot b is read by no MMA before l_full[lb] below, so its
            // high parts can be written over it in place
            float4* xs = reinterpret_cast<float4*>(smem + kSelTcOffX + b * kSelTcTile);
            float4 v[kSelTcTile / 16 / 256];
#pragma unroll
            for (int u = 0; u < kSelTcTile / 16 / 256; ++u) {
                const float4 x = xs[tid + 256 * u];
                const float4 h = tf32_high_part(x);
                xs[tid + 256 * u] = h;
                v[u] = tf32_low_part(x, h);
            }
            if (c >= 2 && !(ok = wait(&l_empty[lb], ((c - 2) >> 1) & 1))) break;
#pragma unroll
            for (int u = 0; u < kSelTcTile / 16 / 256; ++u)
                reinterpret_cast<float4*>(smem + kSelTcOffXl + lb * kSelTcTile)[tid + 256 * u] = v[u];
            fence_proxy_async_smem();
            mbar_arrive(&l_full[lb]);
        }
    }
    // ---------------------------------------------------------------- top-k
    // every MMA is done once `done` completes; the operand buffers then hold keys
    if (warp < 8 && ok) ok = wait(done, 0);
    ok = __syncthreads_and(ok ? 1 : 0) != 0;
    tc_fence_after();
    if (ok && warp < 8) {
        const int q4 = warp & 3;  // TMEM lane quarter of this warp
        uint32_t hint = 0u;       // threshold key of this warp's previous row
        for (int round = 0; round < 2; ++round) {
            const int r0 = round * HALF;
            if (r0 < nq) {
                // scores of key blocks 128 t + 32 q4 + lane for query rows r0 .. r0+15
                for (int t = warp >> 2; t < n_tiles; t += 2) {
                    uint32_t v[16];
                    tmem_ld16(tmem + (static_cast<uint32_t>(32 * q4) << 16) + t * kSelTcRows + r0, v);
                    const int j = 128 * t + 32 * q4 + lane;
                    if (j < NBP) {
#pragma unroll
                        for (int c = 0; c < HALF; ++c) keys[c * NBP + j] = kSelFloatCount ? v[c] : order_key(__uint_as_float(v[c]));
                    }
                }
            }
            asm volatile("bar.sync 1, 256;" ::: "memory");
            // each warp takes neighbouring rows (the threshold of one is the first probe of the next)
#pragma unroll 1
            for (int q = 0; q < HALF / 8; ++q) {
                const int r = r0 + warp * (HALF / 8) + q;
                if (r < nq) {
                    if constexpr (kSelFloatCount)
                        select_row_topk_f<KPL>(keys + (r - r0) * NBP, nb, i0 + r, p.k_keep, bh * nb + i0 + r, row_ptr,
                                               col_idx, hint);
                    else
                        select_row_topk<KPL>(keys + (r - r0) * NBP, nb, i0 + r, p.k_keep, bh * nb + i0 + r, row_ptr,
                                             col_idx, hint);
                }
            }
            asm volatile("bar.sync 1, 256;" ::: "memory");
        }
    }
    if (blockIdx.x == 0 && blockIdx.y == 0 && tid == 0) row_ptr[p.n_rows] = static_cast<int32_t>(p.n_rows * p.k_keep);
    tc_fence_before();
    __syncthreads();
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

}  // namespace sbsa
