// Step 3: dense softmax attention inside the kept key blocks, on tcgen05 tensor cores.
//
// The kept blocks are computed densely to keep the GPU's throughput (page "单卡 RTX 5090
// 跑 Wan2.2-A14B：720p 视频生成只要 3.8 秒", 四步拆解 item 3 动态稀疏注意力); unkept blocks
// contribute nothing and the softmax is normalised over the kept keys only.
//
// One CTA per (b, h, query block): a 128-row query tile against its k kept key blocks.
// 352 threads (eleven warps):
//   warps 0-3 / 4-7 (softmax, two warpgroups): warpgroup g handles the kept blocks
//       j = g, g+2, g+4, ...  Thread r owns query row r.  It copies its row of
//       S_j = Q K_j^T out of TMEM and at once hands the S buffer back, keeps its own
//       running max m_g and sum l_g (log2 domain), rescales its row of its own
//       accumulator O_g in TMEM when m_g moves, and writes P_j = exp2(S_j*scale*log2e - m_g)
//       as bf16 into the warpgroup's shared-memory P buffer (the layout a K-major
//       tcgen05 operand with 128-byte swizzle reads).  The two warpgroups never wait on
//       each other per block; at the end each row merges (m_0, l_0, O_0) and
//       (m_1, l_1, O_1) exactly:
//       O = (2^(m_0-M) O_0 + 2^(m_1-M) O_1) / (2^(m_0-M) l_0 + 2^(m_1-M) l_1), M = max.
//   warp 8 streams Q and the K_j / V_j tiles with TMA (128-byte swizzle) into a K ring
//       and a V ring of shared-memory slots.
//   warp 9 allocates 512 TMEM columns; one of its threads issues every S_j = Q K_j^T
//       (both operands in shared memory) into S buffer j&1.
//   warp 10: one thread issues every O_{j&1} += P_j V_j (P and V in shared memory,
//       V an MN-major operand).
// Two issuing threads, each with a single MMA instruction site: a wait in one of them
// (for a K tile, a free S buffer, a P block) leaves the other's MMAs to keep the
// tensor pipe busy, where one thread alternating between the two kinds drains the
// MMA queue at every switch and every wait.  Since the two threads' MMAs are not
// ordered with respect to each other, every hand-over is an mbarrier:
//   s_full[b]  QK_j done (commit)          -> softmax warpgroup b may read S_j
//   s_free[b]  S_j copied to registers      -> QK_{j+2} may overwrite S buffer b
//   p_full[b]  P_j stored (and O_b rescaled) -> PV_j may run
//   pv_done[b] PV_j done (commit)          -> P buffer b is free and O_b is stable
//
// TMEM columns: S buffers at 0 and 128 (BLK fp32 columns each), O_0 at 256 and O_1 at
// 384 (D columns each).
//
// BLK = 64: a CTA takes two neighbouring query blocks, qa = 2i and qa + 1, as the
// two halves of its 128-row tile.  When both kept lists are strictly ascending, in range
// and short enough, the CTA walks their union once (a key block kept by both is
// computed once for all 128 rows); otherwise it walks list a and then list b.  Each
// entry carries which row halves it serves; the rows of the other half see it fully
// masked.  (Unpaired, half of every 128-row product would be for rows discarded.)
//
// Every wait is bounded (the pipeline limit, 1 s unless a test lowered it); a wait that
// runs out latches SBSA_ERR_TIMEOUT, makes every CTA of the launch give up, drains this
// CTA's own copies and MMAs (each drain wait bounded by 1 s) and frees its TMEM before
// returning.
#pragma once
#include <cuda_bf16.h>

#include "common.cuh"
#include "ptx.cuh"
#include "tmem_wide.cuh"

#include <type_traits>

// Fraction of the probabilities (in eighths) computed with the FMA-pipe
// polynomial instead of the MUFU ex2 unit; the two run in parallel, so moving some of
// the work off the MUFU unit (16 results/clk/SM) shortens the softmax.
#ifndef SBSA_POLY_EXP2_EIGHTHS
#define SBSA_POLY_EXP2_EIGHTHS 2
#endif
// The same for the FP8 form, measured fastest with one eighth (2% over two at the
// long-sequence size; the bf16 form is fastest with two: 0 and 1 are slower).
#ifndef SBSA_POLY_EXP2_EIGHTHS_FP8
#define SBSA_POLY_EXP2_EIGHTHS_FP8 1
#endif

// Issue order of the two MMA threads: with m > 0 the thread that issues S_j = Q K_j^T
// waits until O += P_{j-m} V_{j-m} has been issued, which holds the Q K^T thread back so
// that the tensor pipe alternates more between the two kinds; 0 lets it run ahead as far
// as the S buffers allow.  Measured (long-sequence and 480p layers): the bf16 form is
// fastest with 0 (m = 2 and 3 slower); the FP8 form, whose Q K^T MMAs take half as
// long, with 3 (12% fewer cycles than 0; m = 2 slower).
#ifndef SBSA_ATTN_QK_AFTER_PV
#define SBSA_ATTN_QK_AFTER_PV 0
#endif
#ifndef SBSA_ATTN_QK_AFTER_PV_FP8
#define SBSA_ATTN_QK_AFTER_PV_FP8 3
#endif


namespace sbsa {

// Pairs (e, e+1) with e = 2 * (pair index); pair index mod 8 below EIGHTHS use the polynomial.
template <bool FP8>
__host__ __device__ constexpr bool kPolyPair(int e) {
    return ((e >> 1) & 7) < (FP8 ? SBSA_POLY_EXP2_EIGHTHS_FP8 : SBSA_POLY_EXP2_EIGHTHS);
}

// 2^x on the FMA pipe for a pair, x <= 8 (x >= -125 after the clamp; smaller x give
// ~2^-125).  Cody-Waite style split x = n + f with n = rint(x) (the 1.5*2^23 rounding
// trick) and f in [-0.5, 0.5]; 2^f by a cubic fitted for minimal relative error on
// that interval (max relative error 7.5e-5, well inside the bf16 rounding of P); 2^n
// is added to the exponent field with an integer add.
__device__ __forceinline__ float2 exp2_poly2(float2 x) {
    x.x = fmaxf(x.x, -125.f);
    x.y = fmaxf(x.y, -125.f);
    const float2 t = __fadd2_rn(x, make_float2(12582912.f, 12582912.f));  // 1.5*2^23: t holds rint(x)
    const float2 n = __fadd2_rn(t, make_float2(-12582912.f, -12582912.f));
    const float2 f = __ffma2_rn(n, make_float2(-1.f, -1.f), x);
    float2 q = __ffma2_rn(make_float2(0.0551716685f, 0.0551716685f), f, make_float2(0.242611140f, 0.242611140f));
    q = __ffma2_rn(q, f, make_float2(0.693260968f, 0.693260968f));
    q = __ffma2_rn(q, f, make_float2(0.999928057f, 0.999928057f));
    return make_float2(__uint_as_float(__float_as_uint(q.x) + (__float_as_uint(t.x) << 23)),
                       __uint_as_float(__float_as_uint(q.y) + (__float_as_uint(t.y) << 23)));
}

template <int N>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t (&r)[N]) {
    if constexpr (N == 128) tmem_ld128(taddr, r);
    else if constexpr (N == 64) tmem_ld64(taddr, r);
    else if constexpr (N == 32) tmem_ld32(taddr, r);
    else tmem_ld16(taddr, r);
}
template <int N>
__device__ __forceinline__ void tmem_st_cols(uint32_t taddr, const uint32_t (&r)[N]) {
    if constexpr (N == 128) tmem_st128(taddr, r);
    else if constexpr (N == 64) tmem_st64(taddr, r);
    else if constexpr (N == 32) tmem_st32(taddr, r);
    else tmem_st16(taddr, r);
}

// FP8: Q and K arrive as e4m3 codes with one scale per block (fp8.cuh) and S = Q K^T
// runs as kind::f8f6f4 MMAs (K = 32 per instruction, one 128-byte swizzle atom per row
// at d = 128); the logit of block j is S * |scale| * log2(e) * q_scale * k_scale[j].
// Everything from P on is the same as the bf16 form.
template <int D, int BLK, bool FP8 = false>
struct AttnCfg {
    static constexpr int kQKBytes = FP8 ? 1 : 2;     // bytes per Q/K element
    static constexpr int kKTile = BLK * D * kQKBytes;  // bytes of one K tile
    static constexpr int kVTile = BLK * D * 2;         // bytes of one V tile
    static constexpr int kQBytes = 128 * D * kQKBytes;  // bytes of the Q tile
    static constexpr int kQKAtoms = D * kQKBytes / 128;  // 128-byte swizzle atoms per Q/K row
    static constexpr int kQKElemsPerAtom = 128 / kQKBytes;
    static constexpr int kQKSteps = D / (FP8 ? 32 : 16);  // MMAs per S = Q K^T
    static constexpr int kPBytes = 128 * BLK * 2;    // bytes of one P block (bf16)
    static constexpr int kSmemBudget = 224 * 1024;   // Q + two P buffers + the K and V rings
    static constexpr int kStagesRaw = (kSmemBudget - kQBytes - 2 * kPBytes) / (kKTile + kVTile);
    static constexpr int kStages = kStagesRaw > 4 ? 4 : kStagesRaw;  // slots per ring
    static constexpr int kPOff = kQBytes;
    static constexpr int kKOff = kPOff + 2 * kPBytes;
    static constexpr int kVOff = kKOff + kStages * kKTile;
    static constexpr int kBarOff = kVOff + kStages * kVTile;
    // barriers: q_full, k_full[S], k_empty[S], v_full[S], v_empty[S], s_full[2],
    // s_free[2], p_full[2], pv_done[2], drain[2], pv_issued[4]
    static constexpr int kNumBars = 1 + 4 * kStages + 2 * 5 + 4;
    // paired query blocks (BLK = 64): the kept lists copied to shared memory and their
    // union, when each list holds at most kListCap entries
    static constexpr bool kPaired = BLK == 64;
    static constexpr int kListCap = kPaired ? 256 : 0;
    static constexpr int kSeqOff = kBarOff + kNumBars * 8 + 16;  // after the tmem slot and flag
    static constexpr int kSeqBytes = kPaired ? (4 * kListCap + 4) * 4 : 0;  // union, two lists, mode and length
    static constexpr int kSmemBytes = kSeqOff + kSeqBytes + 1024;  // + alignment slack
    static constexpr int kThreads = 352;
    static constexpr uint32_t kColS0 = 0, kColO0 = 256;  // S_b at b*128, O_g at 256 + g*128
    static_assert(kStages >= 2, "need at least two slots per ring");
    static_assert(D == 64 || D == 128, "head_dim");
    static_assert(BLK == 64 || BLK == 128, "block_size");
    static_assert(kSmemBytes <= 232448, "shared memory");
    static_assert(2 * 2 * 128 * 4 <= kPBytes, "merge exchange fits in a P buffer");
    static_assert(!FP8 || D == 128, "the FP8 form needs d = 128 (one 128-byte atom per row)");
};

struct AttnParams {
    const int32_t* row_ptr;
    const int32_t* col_idx;
    __nv_bfloat16* o;
    long long units;   // B * H * nb
    int L, Lp, nb;
    float scale_log2;  // |scale| * log2(e)
    int neg_scale;     // 1 if scale < 0 (logits are then -|scale| * S)
    unsigned int epoch;
    const float* q_scale;  // FP8 form: per (b, h, block) scales of the codes
    const float* k_scale;
    int prefetch_dist;     // units ahead whose Q tile is prefetched into L2 (0: none; the SM count)
    int units_per_bh;      // units per (b, h): nb, or ceil(nb / 2) with paired query blocks
};

// e4m3 x e4m3 -> fp32 instruction descriptor (format 0 = E4M3 for both operands).
__host__ __device__ constexpr uint32_t idesc_e4m3_f32(int M, int N) {
    return (1u << 4) | (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}
__device__ __forceinline__ void umma_f8_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                           uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Synchronise the two softmax warpgroups (warps 0-7) on named barrier 1 (final merge).
__device__ __forceinline__ void softmax_pair_sync() {
    asm volatile("bar.sync 1, 256;" ::: "memory");
}

template <int D, int BLK, bool FP8 = false>
__global__ void __launch_bounds__(352, 1) attn_kernel(const __grid_constant__ CUtensorMap map_q,
                                                      const __grid_constant__ CUtensorMap map_k,
                                                      const __grid_constant__ CUtensorMap map_v,
                                                      const AttnParams p) {
    using C = AttnCfg<D, BLK, FP8>;
    constexpr int NS = C::kStages;
    constexpr int kQkAfterPv = FP8 ? SBSA_ATTN_QK_AFTER_PV_FP8 : SBSA_ATTN_QK_AFTER_PV;
    constexpr int HD = D / 2;    // output columns each warpgroup writes in the merge
    extern __shared__ __align__(1024) uint8_t attn_smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(attn_smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sQ = smem;
    uint8_t* sP = smem + C::kPOff;   // P_b at sP + b * kPBytes
    uint8_t* sK = smem + C::kKOff;
    uint8_t* sV = smem + C::kVOff;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
    uint64_t* q_full = bars;
    uint64_t* k_full = bars + 1;
    uint64_t* k_empty = k_full + NS;
    uint64_t* v_full = k_empty + NS;
    uint64_t* v_empty = v_full + NS;
    uint64_t* s_full = v_empty + NS;
    uint64_t* s_free = s_full + 2;
    uint64_t* p_full = s_free + 2;
    uint64_t* pv_done = p_full + 2;
    uint64_t* drain = pv_done + 2;
    uint64_t* pv_issued = drain + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::kNumBars);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int tid = threadIdx.x;
    const int warp = tid / 32;
    // a CTA that starts after another one of its launch gave up returns at once; every
    // thread takes the same branch (the barriers below need all of them)
    if (__syncthreads_or(launch_aborted(p.epoch) ? 1 : 0)) return;

    const long long unit = blockIdx.x;
    const long long bh = unit / p.units_per_bh;
    // first query block of the tile (paired: qb and qb + 1, when qb + 1 exists)
    const int qb = static_cast<int>(unit % p.units_per_bh) * (C::kPaired ? 2 : 1);
    const bool has_b = C::kPaired && qb + 1 < p.nb;
    const long long row_a = bh * p.nb + qb;
    int rs = __ldg(p.row_ptr + row_a);
    int re = __ldg(p.row_ptr + row_a + 1);
    bool bad_row = rs < 0 || re < rs;
    if (rs < 0 || re < rs) re = rs = 0;
    int rs2 = 0, re2 = 0;  // the second query block's list (paired)
    if (has_b) {
        rs2 = __ldg(p.row_ptr + row_a + 1);
        re2 = __ldg(p.row_ptr + row_a + 2);
        if (rs2 < 0 || re2 < rs2) {
            bad_row = true;
            re2 = rs2 = 0;
        }
    }
    uint32_t* seq = reinterpret_cast<uint32_t*>(smem + C::kSeqOff);  // union: block | halves << 30
    int* list_a = reinterpret_cast<int*>(seq + 2 * C::kListCap);
    int* list_b = list_a + C::kListCap;
    int* seq_info = list_b + C::kListCap;  // [0] 1 = walk the union, [1] entries

    if (tid == 256) {
        *abort_flag = 0;
        mbar_init(q_full, 1);
        for (int s = 0; s < NS; ++s) {
            mbar_init(&k_full[s], 1);
            mbar_init(&k_empty[s], 1);
            mbar_init(&v_full[s], 1);
            mbar_init(&v_empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&s_full[b], 1);
            mbar_init(&s_free[b], 128);
            mbar_init(&p_full[b], 128);
            mbar_init(&pv_done[b], 1);
            mbar_init(&drain[b], 1);
        }
        for (int b = 0; b < 4; ++b) mbar_init(&pv_issued[b], 1);
        fence_mbar_init();
        tma_prefetch_desc(&map_q);
        tma_prefetch_desc(&map_k);
        tma_prefetch_desc(&map_v);
        if (bad_row) raise_error(kErrBadIndex);
    }
    if (warp == 9) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    if constexpr (C::kPaired) {
        if (warp == 8) {
            // the union of the two kept lists, when both are strictly ascending, in range
            // and at most kListCap long (uniform over the warp)
            const int na = re - rs, nb2 = re2 - rs2;
            bool use_union = na <= C::kListCap && nb2 <= C::kListCap;
            if (use_union) {
                bool good = true;
                for (int i = (tid & 31); i < na; i += 32) {
                    const int v = __ldg(p.col_idx + rs + i);
                    list_a[i] = v;
                    good = good && v >= 0 && v < p.nb && (i == 0 || __ldg(p.col_idx + rs + i - 1) < v);
                }
                for (int i = (tid & 31); i < nb2; i += 32) {
                    const int v = __ldg(p.col_idx + rs2 + i);
                    list_b[i] = v;
                    good = good && v >= 0 && v < p.nb && (i == 0 || __ldg(p.col_idx + rs2 + i - 1) < v);
                }
                use_union = __all_sync(0xFFFFFFFFu, good);
            }
            __syncwarp();
            if ((tid & 31) == 0) {
                int o = na + nb2;
                if (use_union) {
                    // merge; every step takes one entry of a or of b or both
                    int i = 0, k2 = 0;
                    o = 0;
                    while (i < na || k2 < nb2) {
                        uint32_t v, halves;
                        if (k2 >= nb2 || (i < na && list_a[i] < list_b[k2])) {
                            v = static_cast<uint32_t>(list_a[i++]);
                            halves = 1u;
                        } else if (i >= na || list_b[k2] < list_a[i]) {
                            v = static_cast<uint32_t>(list_b[k2++]);
                            halves = 2u;
                        } else {
                            v = static_cast<uint32_t>(list_a[i]);
                            ++i;
                            ++k2;
                            halves = 3u;
                        }
                        seq[o++] = v | (halves << 30);
                    }
                }
                seq_info[0] = use_union ? 1 : 0;
                seq_info[1] = o;
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // kept entries of this CTA and, for entry j, its key block and the row halves it
    // serves (bit h: rows 64 h .. 64 h + 63; both bits unpaired)
    const bool walk_union = C::kPaired && seq_info[0] != 0;
    const int n = C::kPaired ? seq_info[1] : re - rs;
    auto entry = [&](int j, uint32_t& halves) -> int {
        if constexpr (C::kPaired) {
            if (walk_union) {
                const uint32_t e = seq[j];
                halves = e >> 30;
                return static_cast<int>(e & 0x3FFFFFFFu);
            }
            const int na = re - rs;
            halves = j < na ? 1u : 2u;
            return j < na ? __ldg(p.col_idx + rs + j) : __ldg(p.col_idx + rs2 + (j - na));
        } else {
            halves = 3u;
            return __ldg(p.col_idx + rs + j);
        }
    };

    auto give_up = [&]() {
        *abort_flag = 1;
        abort_launch(p.epoch);
    };
    const uint64_t pipe_limit = pipe_wait_ns();  // pipeline waits; the drain below keeps kWaitLimitNs
    auto wait = [&](uint64_t* bar, uint32_t parity) -> bool {
        if (mbar_wait_bounded(bar, parity, abort_flag, pipe_limit)) return true;
        if (!*abort_flag) give_up();
        return false;
    };

    if (warp == 8) {
        // ------------------------------------------------------------ TMA producer
        // Order of need: K_0, K_1, then K_{j+2} (wanted as soon as S_j is copied out)
        // before V_j (wanted when P_j is ready).
        if ((tid & 31) == 0 && n > 0) {
            const uint64_t pol_q = policy_evict_first();
            const uint64_t pol_kv = policy_evict_last();
            const int row0 = static_cast<int>(bh * p.Lp);
            mbar_arrive_expect_tx(q_full, C::kQBytes);
#pragma unroll
            for (int a = 0; a < C::kQKAtoms; ++a)
                tma_load_2d(sQ + a * 128 * 128, &map_q, q_full, a * C::kQKElemsPerAtom, row0 + qb * BLK, pol_q);
            // The unit that starts about one CTA lifetime from now (one CTA per SM, units
            // dispatched in order) is unit + prefetch_dist: its Q tile is brought into L2
            // now, so that its first load does not wait for HBM
            const long long u2 = unit + p.prefetch_dist;
            if (p.prefetch_dist > 0 && u2 < p.units) {
                const int qb2 = static_cast<int>(u2 % p.units_per_bh) * (C::kPaired ? 2 : 1);
                const int row2 = static_cast<int>((u2 / p.units_per_bh) * p.Lp + qb2 * BLK);
#pragma unroll
                for (int a = 0; a < C::kQKAtoms; ++a) tma_prefetch_l2_2d(&map_q, a * C::kQKElemsPerAtom, row2);
            }
            int kseq = 0, vseq = 0;
            auto load = [&](int j, bool is_v) -> bool {
                int& seq = is_v ? vseq : kseq;
                const int slot = seq % NS;
                const uint32_t ph = (seq / NS) & 1;
                if (!wait(is_v ? &v_empty[slot] : &k_empty[slot], ph ^ 1)) return false;
                uint32_t halves;
                int blk = entry(j, halves);
                if (blk < 0 || blk >= p.nb) blk = 0;  // masked by the softmax warps
                uint8_t* dst = is_v ? sV + slot * C::kVTile : sK + slot * C::kKTile;
                uint64_t* full = is_v ? &v_full[slot] : &k_full[slot];
                mbar_arrive_expect_tx(full, is_v ? C::kVTile : C::kKTile);
                if (is_v) {
#pragma unroll
                    for (int a = 0; a < D / 64; ++a)
                        tma_load_2d(dst + a * BLK * 128, &map_v, full, a * 64, row0 + blk * BLK, pol_kv);
                } else {
#pragma unroll
                    for (int a = 0; a < C::kQKAtoms; ++a)
                        tma_load_2d(dst + a * BLK * 128, &map_k, full, a * C::kQKElemsPerAtom, row0 + blk * BLK, pol_kv);
                }
                ++seq;
                return true;
            };
            bool ok = load(0, false);
            if (ok && n > 1) ok = load(1, false);
            for (int j = 0; ok && j < n; ++j) {
                if (j + 2 < n) ok = load(j + 2, false);
                if (ok) ok = load(j, true);
            }
            if (!ok) {
                // drain: every issued copy must land before the CTA exits
                volatile int never = 0;
                mbar_wait_bounded(q_full, 0, &never, kWaitLimitNs);
                for (int q = kseq - NS < 0 ? 0 : kseq - NS; q < kseq; ++q)
                    mbar_wait_bounded(&k_full[q % NS], (q / NS) & 1, &never, kWaitLimitNs);
                for (int q = vseq - NS < 0 ? 0 : vseq - NS; q < vseq; ++q)
                    mbar_wait_bounded(&v_full[q % NS], (q / NS) & 1, &never, kWaitLimitNs);
            }
        }
    } else if (warp == 9) {
        // ------------------------------------------------------------ QK issuer
        if ((tid & 31) == 0 && n > 0) {
            constexpr uint32_t idS = FP8 ? idesc_e4m3_f32(128, BLK) : idesc_bf16_f32(128, BLK, false);
            const uint32_t k_addr = smem_u32(sK);
            const uint64_t qdesc0 = sdesc_sw128(smem_u32(sQ), 16, 1024);
            bool ok = wait(q_full, 0);
            for (int j = 0; ok && j < n; ++j) {
                const int slot = j % NS;
                const int b = j & 1;
                if (!(ok = wait(&k_full[slot], (j / NS) & 1))) break;
                if (j >= 2 && !(ok = wait(&s_free[b], ((j - 2) >> 1) & 1))) break;
                if constexpr (kQkAfterPv > 0) {
                    constexpr int m = kQkAfterPv;
                    // PV_{j-m+4}, the next arrival on this barrier, needs QK_{j-m+4} (m <= 4):
                    // the barrier is never a whole phase ahead of this wait
                    static_assert(m <= 4, "pv_issued has four barriers");
                    if (j >= m && !(ok = wait(&pv_issued[(j - m) & 3], ((j - m) >> 2) & 1))) break;
                }
                tc_fence_after();
                const uint64_t kdesc0 = sdesc_sw128(k_addr + slot * C::kKTile, 16, 1024);
                const uint32_t d_s = tmem + C::kColS0 + b * 128;
#pragma unroll
                for (int kk = 0; kk < C::kQKSteps; ++kk) {
                    // only the 14-bit start-address field (bytes / 16) moves between K steps
                    // (32 bytes per step: 16 bf16 or 32 e4m3 elements)
                    const uint64_t da = qdesc0 + static_cast<uint64_t>(((kk / 4) * (128 * 128) + (kk % 4) * 32) >> 4);
                    const uint64_t db = kdesc0 + static_cast<uint64_t>(((kk / 4) * (BLK * 128) + (kk % 4) * 32) >> 4);
                    if constexpr (FP8) umma_f8_ss(d_s, da, db, idS, kk > 0 ? 1u : 0u);
                    else umma_ss(d_s, da, db, idS, kk > 0 ? 1u : 0u);
                }
                umma_commit(&k_empty[slot]);
                umma_commit(&s_full[b]);
            }
            if (!ok) {
                umma_commit(&drain[0]);  // wait for every MMA this thread issued
                volatile int never = 0;
                mbar_wait_bounded(&drain[0], 0, &never, kWaitLimitNs);
            }
        }
    } else if (warp == 10) {
        // ------------------------------------------------------------ PV issuer
        if ((tid & 31) == 0 && n > 0) {
            constexpr uint32_t idO = idesc_bf16_f32(128, D, true);
            const uint32_t v_addr = smem_u32(sV);
            const uint64_t pdesc0 = sdesc_sw128(smem_u32(sP), 16, 1024);
            bool ok = true;
            for (int j = 0; ok && j < n; ++j) {
                const int slot = j % NS;
                const int b = j & 1;
                if (!(ok = wait(&v_full[slot], (j / NS) & 1))) break;
                if (!(ok = wait(&p_full[b], (j >> 1) & 1))) break;
                tc_fence_after();
                const uint64_t vdesc0 = sdesc_sw128(v_addr + slot * C::kVTile, BLK * 128, 1024);
                const uint64_t pdesc = pdesc0 + static_cast<uint64_t>((b * C::kPBytes) >> 4);
                const uint32_t d_o = tmem + C::kColO0 + b * 128;
#pragma unroll
                for (int kk = 0; kk < BLK / 16; ++kk) {
                    const uint64_t da = pdesc + static_cast<uint64_t>(((kk / 4) * (128 * 128) + (kk % 4) * 32) >> 4);
                    const uint64_t db = vdesc0 + static_cast<uint64_t>((kk * 16 * 128) >> 4);
                    umma_ss(d_o, da, db, idO, (j > 1 || kk > 0) ? 1u : 0u);
                }
                umma_commit(&v_empty[slot]);
                umma_commit(&pv_done[b]);
                if constexpr (kQkAfterPv > 0) mbar_arrive(&pv_issued[j & 3]);
            }
            if (!ok) {
                umma_commit(&drain[1]);
                volatile int never = 0;
                mbar_wait_bounded(&drain[1], 0, &never, kWaitLimitNs);
            }
        }
    } else if (warp < 8) {
        // ------------------------------------------------------------ softmax warpgroups
        const int g = warp >> 2;     // this warpgroup's blocks: j = g, g + 2, ...
        const int r = tid & 127;     // row within the 128-row tile
        const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const int t = qb * BLK + r;
        const bool row_in_block = r < BLK || has_b;  // paired: rows BLK.. are block qb + 1
        const uint32_t my_half = static_cast<uint32_t>(r >= 64 ? 2 : 1);
        const bool row_valid = row_in_block && t < p.L;
        // logit scale |scale| * log2(e) > 0; the FP8 form also folds in this query
        // block's scale here and each key block's scale below
        // (paired: rows BLK.. belong to query block qb + 1, whose scale is the next one)
        const float sl2_q = FP8 ? p.scale_log2 * __ldg(p.q_scale + row_a + (r >= BLK && has_b ? 1 : 0)) : p.scale_log2;
        const uint32_t s_col = tmem + lane_base + C::kColS0 + g * 128;
        const uint32_t o_col = tmem + lane_base + C::kColO0 + g * 128;
        // this row of P_g: 128-byte rows, 16-byte chunks swizzled by (row mod 8), one
        // 16 KB region per 64 keys
        const uint32_t p_row = smem_u32(sP + g * C::kPBytes) + r * 128;
        const uint32_t p_swz = static_cast<uint32_t>(r & 7);
        float m = -INFINITY;  // running reference max (log2 domain), possibly stale by < 8
        float l = 0.f;        // this warpgroup's part of the row sum
        bool ok = true;
        // tcgen05.ld/st are warp-collective: every decision that guards one is made
        // warp-uniform (a wait's outcome included); a failed wait skips work but never
        // the final merge barrier.
        auto wait_warp = [&](uint64_t* bar, uint32_t parity) -> bool {
            const bool w = wait(bar, parity);
            return __all_sync(0xFFFFFFFFu, w);
        };
        uint32_t halves_next = 3u;
        int blk_next = g < n ? entry(g, halves_next) : 0;
        float ks_next = 1.f;
        if constexpr (FP8) {
            if (g < n && blk_next >= 0 && blk_next < p.nb) ks_next = __ldg(p.k_scale + bh * p.nb + blk_next);
        }
        for (int j = g; j < n; j += 2) {
            const int blk = blk_next;
            const uint32_t halves = halves_next;
            const float sl2 = sl2_q * ks_next;
            const float2 sl2x2 = make_float2(sl2, sl2);
            if (j + 2 < n) {
                blk_next = entry(j + 2, halves_next);
                if constexpr (FP8) {
                    ks_next = (blk_next >= 0 && blk_next < p.nb) ? __ldg(p.k_scale + bh * p.nb + blk_next) : 1.f;
                }
            }
            if (ok) ok = wait_warp(&s_full[g], (j >> 1) & 1);
            if (!ok) continue;
            tc_fence_after();
            const bool bad = blk < 0 || blk >= p.nb;
            if (bad && r == 0) raise_error(kErrBadIndex);
            // valid keys of the block for this row: none when the entry does not serve its
            // half of the tile (uniform per warp: a warp's 32 rows lie in one half)
            const int nvalid = (bad || (halves & my_half) == 0) ? 0 : min(BLK, p.L - blk * BLK);
            float s[BLK];
            {
                uint32_t raw[BLK];
                tmem_ld_cols<BLK>(s_col, raw);
#pragma unroll
                for (int e = 0; e < BLK; ++e) s[e] = __uint_as_float(raw[e]);
            }
            // S_j is in registers: QK_{j+2} may overwrite the buffer
            tc_fence_before();
            mbar_arrive(&s_free[g]);
            if (p.neg_scale) {
#pragma unroll
                for (int e = 0; e < BLK; ++e) s[e] = -s[e];
            }
            const bool masked = nvalid < BLK;  // padded tail, skipped index or other half (warp-uniform)
            if (masked) {
#pragma unroll
                for (int e = 0; e < BLK; ++e)
                    if (e >= nvalid) s[e] = -INFINITY;
            }
            // block max: eight independent chains of three-input maxima, then a tree
            float mx8[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) mx8[c] = fmaxf(s[c], s[c + 8]);
#pragma unroll
            for (int e = 16; e < BLK; e += 16)
#pragma unroll
                for (int c = 0; c < 8; ++c) mx8[c] = fmax3(mx8[c], s[e + c], s[e + 8 + c]);
            const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                                   fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7]))) * sl2;
            // Lazy rescaling: keep the old reference max unless the block's max exceeds
            // it by more than 8 (values up to 2^8 are safe in bf16 P and fp32 O / l).
            float alpha = 1.f;
            if (mx > m + 8.f) {
                alpha = (m == -INFINITY) ? 0.f : ex2_approx(m - mx);
                m = mx;
            }
            const float neg_m = (m == -INFINITY) ? 0.f : -m;
            const float2 nm2 = make_float2(neg_m, neg_m);
            float2 sum4[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                              make_float2(0.f, 0.f)};
            uint32_t pk[BLK / 2];
            // P for keys [E0, E1): exp2(S * sl2 - m) in fp32, summed, packed to bf16 pairs
            auto exps = [&](auto e0_tag, auto e1_tag) {
                constexpr int E0 = decltype(e0_tag)::value, E1 = decltype(e1_tag)::value;
                if (!masked) {
#pragma unroll
                    for (int e = E0; e < E1; e += 2) {
                        const float2 x = __ffma2_rn(make_float2(s[e], s[e + 1]), sl2x2, nm2);
                        float2 pr;
                        if (kPolyPair<FP8>(e)) {
                            pr = exp2_poly2(x);
                        } else {
                            pr.x = ex2_approx(x.x);
                            pr.y = ex2_approx(x.y);
                        }
                        sum4[(e >> 1) & 3] = __fadd2_rn(sum4[(e >> 1) & 3], pr);
                        pk[e / 2] = pack_bf16x2(pr.x, pr.y);
                    }
                } else {
                    // masked entries are -inf: ex2 gives exactly 0 (the polynomial would not)
#pragma unroll
                    for (int e = E0; e < E1; e += 2) {
                        const float2 x = __ffma2_rn(make_float2(s[e], s[e + 1]), sl2x2, nm2);
                        float2 pr;
                        pr.x = ex2_approx(x.x);
                        pr.y = ex2_approx(x.y);
                        sum4[(e >> 1) & 3] = __fadd2_rn(sum4[(e >> 1) & 3], pr);
                        pk[e / 2] = pack_bf16x2(pr.x, pr.y);
                    }
                }
            };
            // P_j's 16-byte chunks [C0, C1) into P buffer g (128-byte rows, one 16 KB region per 64 keys)
            auto store_p = [&](auto c0_tag, auto c1_tag) {
                constexpr int C0 = decltype(c0_tag)::value, C1 = decltype(c1_tag)::value;
#pragma unroll
                for (int c = C0; c < C1; ++c) {
                    const uint32_t addr = p_row + (c / 8) * (128 * 128) + ((static_cast<uint32_t>(c & 7) ^ p_swz) << 4);
                    st_shared_v4(addr, pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
                }
            };
            // O_g *= alpha when the reference max moved (PV_{j-2} is done)
            auto rescale_o = [&]() {
                if (j > 1 && __any_sync(0xFFFFFFFFu, alpha != 1.f)) {
                    const float2 a2 = make_float2(alpha, alpha);
                    // 32 columns at a time: few registers next to the live S and P values
#pragma unroll 1
                    for (int h = 0; h < D; h += 32) {
                        uint32_t ov[32];
                        tmem_ld_cols<32>(o_col + h, ov);
#pragma unroll
                        for (int e = 0; e < 32; e += 2) {
                            const float2 v = __fmul2_rn(make_float2(__uint_as_float(ov[e]), __uint_as_float(ov[e + 1])), a2);
                            ov[e] = __float_as_uint(v.x);
                            ov[e + 1] = __float_as_uint(v.y);
                        }
                        tmem_st_cols<32>(o_col + h, ov);
                    }
                    tmem_st_wait();
                }
            };
            using I0 = std::integral_constant<int, 0>;
            using IB = std::integral_constant<int, BLK>;
            using C0 = std::integral_constant<int, 0>;
            using CB = std::integral_constant<int, BLK / 8>;
            exps(I0{}, IB{});
            // PV_{j-2} must be done before P buffer g is overwritten or O_g rescaled
            if (j >= 2) {
                ok = wait_warp(&pv_done[g], ((j - 2) >> 1) & 1);
                if (!ok) continue;
            }
            store_p(C0{}, CB{});
            rescale_o();
            const float2 s01 = __fadd2_rn(sum4[0], sum4[1]);
            const float2 s23 = __fadd2_rn(sum4[2], sum4[3]);
            const float2 sall = __fadd2_rn(s01, s23);
            l = l * alpha + (sall.x + sall.y);
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&p_full[g]);
        }
        const bool has_blocks = g < n;
        if (ok && has_blocks) {
            const int j_last = g + ((n - 1 - g) & ~1);  // this warpgroup's last block
            ok = wait_warp(&pv_done[g], (j_last >> 1) & 1);
        }
        ok = __all_sync(0xFFFFFFFFu, ok);
        // ---- merge: row r of (m_0, l_0, O_0) and (m_1, l_1, O_1); warpgroup g writes
        // output columns [g D/2, (g+1) D/2).  The exchange goes through P buffer g,
        // which no MMA reads any more once this warpgroup's last PV is done; after a
        // failed wait it may still be read, so then nothing is exchanged.
        float* xml_mine = reinterpret_cast<float*>(sP + g * C::kPBytes);
        const float* xml_other = reinterpret_cast<const float*>(sP + (g ^ 1) * C::kPBytes);
        if (ok) {
            xml_mine[r] = has_blocks ? m : -INFINITY;
            xml_mine[128 + r] = has_blocks ? l : 0.f;
        }
        tc_fence_before();
        softmax_pair_sync();
        tc_fence_after();
        // a failed wait anywhere in the pair is seen by both warpgroups: the flag is
        // latched before the barrier
        const bool pair_ok = ok && !*abort_flag;
        float mg = -INFINITY, lg = 0.f, mo = -INFINITY, lo = 0.f;
        if (pair_ok) {
            mg = xml_mine[r];
            lg = xml_mine[128 + r];
            mo = xml_other[r];
            lo = xml_other[128 + r];
        }
        const float m0 = g == 0 ? mg : mo, l0 = g == 0 ? lg : lo;
        const float m1 = g == 0 ? mo : mg, l1 = g == 0 ? lo : lg;
        const float M = fmaxf(m0, m1);
        const float w0 = (m0 == -INFINITY) ? 0.f : ex2_approx(m0 - M);
        const float w1 = (m1 == -INFINITY) ? 0.f : ex2_approx(m1 - M);
        const float lt = w0 * l0 + w1 * l1;
        const bool any_pv = n > 0;
        {
            // every lane of the warp runs the TMEM loads (warp-collective); only rows of
            // this query block are stored
            const bool read_o = __all_sync(0xFFFFFFFFu, pair_ok) && any_pv;
            const bool write_o = read_o && row_valid && lt > 0.f;
            const float inv = write_o ? 1.f / lt : 0.f;
            const float c0 = w0 * inv, c1 = w1 * inv;
            const bool use1 = n > 1;  // O_1 holds data only if warpgroup 1 had a block
            uint32_t o0[HD], o1[HD];
            if (read_o) {
                tmem_ld_cols<HD>(tmem + lane_base + C::kColO0 + g * HD, o0);
                if (use1) tmem_ld_cols<HD>(tmem + lane_base + C::kColO0 + 128 + g * HD, o1);
            }
            if (row_in_block) {
                __nv_bfloat16* dst = p.o + (bh * p.Lp + t) * D + g * HD;
                const bool wide = (reinterpret_cast<uintptr_t>(p.o) & 31u) == 0;
#pragma unroll
                for (int e = 0; e < HD; e += 16) {
                    uint32_t w[8];
#pragma unroll
                    for (int q = 0; q < 16; q += 2) {
                        float x0 = write_o ? __uint_as_float(o0[e + q]) * c0 : 0.f;
                        float x1 = write_o ? __uint_as_float(o0[e + q + 1]) * c0 : 0.f;
                        if (write_o && use1) {
                            x0 = fmaf(__uint_as_float(o1[e + q]), c1, x0);
                            x1 = fmaf(__uint_as_float(o1[e + q + 1]), c1, x1);
                        }
                        w[q / 2] = pack_bf16x2(x0, x1);
                    }
                    if (wide) {
                        st_global_v8(dst + e, w[0], w[1], w[2], w[3], w[4], w[5], w[6], w[7]);
                    } else {
                        uint4* d4 = reinterpret_cast<uint4*>(dst + e);
                        d4[0] = make_uint4(w[0], w[1], w[2], w[3]);
                        d4[1] = make_uint4(w[4], w[5], w[6], w[7]);
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace sbsa
