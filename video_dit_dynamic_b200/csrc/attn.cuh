// Step 3: dense softmax attention inside the kept key blocks, on tcgen05 tensor cores.
//
// The kept blocks are computed densely to keep the GPU's throughput (page "单卡 RTX 5090
// 跑 Wan2.2-A14B：720p 视频生成只要 3.8 秒", 四步拆解 item 3 动态稀疏注意力); unkept blocks
// contribute nothing and the softmax is normalised over the kept keys only.
//
// One CTA per (b, h, query block): a 128-row query tile against its k kept key blocks.
// 320 threads (ten warps):
//   warps 0-3 / 4-7 (softmax, two warpgroups): warpgroup g handles the kept blocks
//       j = g, g+2, g+4, ...  Thread r owns query row r: it reads its row of
//       S_j = Q K_j^T from TMEM, keeps its own running max m_g and sum l_g (log2
//       domain), rescales its row of its own accumulator O_g in TMEM when m_g moves,
//       and writes P_j = exp2(S_j*scale*log2e - m_g) as bf16 over the first BLK/2
//       columns of S_j (P aliases S).  The two warpgroups never wait on each other per
//       block; at the end each row merges (m_0, l_0, O_0) and (m_1, l_1, O_1) exactly:
//       O = (2^(m_0-M) O_0 + 2^(m_1-M) O_1) / (2^(m_0-M) l_0 + 2^(m_1-M) l_1), M = max.
//   warp 8 streams Q and the K_j / V_j tiles with TMA (128-byte swizzle) through a ring
//       of shared-memory slots.
//   warp 9 allocates 512 TMEM columns and one of its threads issues tcgen05.mma:
//       S_j = Q K_j^T (both operands in shared memory) into S buffer j&1, and
//       O_{j&1} += P_j V_j (P from TMEM, V an MN-major shared-memory operand).
// Tensor-core order: QK_0, QK_1, PV_0, QK_2, PV_1, QK_3, ... so S_{j+1} is computed
// while a warpgroup works on S_j.  MMAs execute in issue order: QK_{j+2} may reuse S
// buffer j&1 (and the aliased P_j) once PV_j is issued, and the commit that signals
// S_{j+2} also proves PV_j done, so O_{j&1} is stable when its warpgroup rescales it.
// The producer loads K_0, K_1, V_0, K_2, V_1, ... - the same order - over one ring.
//
// TMEM columns: S buffers at 0 and 128 (BLK fp32 columns each, P in the first BLK/2),
// O_0 at 256 and O_1 at 384 (D columns each).  For BLK = 64 the 128-row Q tile also holds the next block's
// 64 rows; those rows are computed and discarded.
//
// Every wait is bounded (kWaitLimitNs); a wait that runs out latches SBSA_ERR_TIMEOUT,
// makes every CTA of the launch give up, drains this CTA's own copies and MMAs and
// frees its TMEM before returning.
#pragma once
#include <cuda_bf16.h>

#include "common.cuh"
#include "ptx.cuh"
#include "tmem_wide.cuh"

// Fraction of the probabilities (in eighths, even) computed with the FMA-pipe
// polynomial instead of the MUFU ex2 unit; the two run in parallel, so moving some of
// the work off the MUFU unit (16 results/clk/SM) shortens the softmax.
#ifndef SBSA_POLY_EXP2_EIGHTHS
#define SBSA_POLY_EXP2_EIGHTHS 0
#endif

namespace sbsa {

// Pairs (e, e+1) with e = 2 * (pair index); pair index mod 4 below EIGHTHS/2 use the polynomial.
__host__ __device__ constexpr bool kPolyPair(int e) { return ((e >> 1) & 3) < SBSA_POLY_EXP2_EIGHTHS / 2; }

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

template <int D, int BLK>
struct AttnCfg {
    static constexpr int kTile = BLK * D * 2;        // bytes of one K or V tile
    static constexpr int kQBytes = 128 * D * 2;      // bytes of the Q tile
    static constexpr int kSmemBudget = 216 * 1024;   // Q tile + ring
    static constexpr int kStagesRaw = (kSmemBudget - kQBytes) / kTile;
    static constexpr int kStages = kStagesRaw > 8 ? 8 : kStagesRaw;
    static constexpr int kRingOff = kQBytes;
    static constexpr int kBarOff = kRingOff + kStages * kTile;
    // barriers: q_full, kv_full[S], kv_empty[S], s_full[2], p_full[2], o_ready[2], drain
    static constexpr int kNumBars = 1 + 2 * kStages + 2 + 2 + 2 + 1;
    // after the barriers: tmem slot + abort flag (16 B), then the per-row (m, l) of
    // each warpgroup for the final merge: [2][2][128] floats
    static constexpr int kXchgOff = kBarOff + kNumBars * 8 + 16;
    static constexpr int kXchgBytes = 2 * 2 * 128 * 4;
    static constexpr int kSmemBytes = kXchgOff + kXchgBytes + 1024;  // + alignment slack
    static constexpr int kThreads = 320;
    static constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO0 = 256, kColO1 = 384;
    static_assert(kStages >= 2, "need at least two ring slots");
    static_assert(D == 64 || D == 128, "head_dim");
    static_assert(BLK == 64 || BLK == 128, "block_size");
    static_assert(kSmemBytes <= 232448, "shared memory");
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
};

// Synchronise the two softmax warpgroups (warps 0-7) on named barrier 1 (final merge).
__device__ __forceinline__ void softmax_pair_sync() {
    asm volatile("bar.sync 1, 256;" ::: "memory");
}

template <int D, int BLK>
__global__ void __launch_bounds__(320, 1) attn_kernel(const __grid_constant__ CUtensorMap map_q,
                                                      const __grid_constant__ CUtensorMap map_k,
                                                      const __grid_constant__ CUtensorMap map_v,
                                                      const AttnParams p) {
    using C = AttnCfg<D, BLK>;
    constexpr int NS = C::kStages;
    constexpr int HD = D / 2;    // output columns each warpgroup writes in the merge
    extern __shared__ __align__(1024) uint8_t attn_smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(attn_smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sQ = smem;
    uint8_t* sRing = smem + C::kRingOff;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
    uint64_t* q_full = bars;
    uint64_t* kv_full = bars + 1;
    uint64_t* kv_empty = kv_full + NS;
    uint64_t* s_full = kv_empty + NS;
    uint64_t* p_full = s_full + 2;
    uint64_t* o_ready = p_full + 2;
    uint64_t* drain = o_ready + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::kNumBars);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    float* xml = reinterpret_cast<float*>(smem + C::kXchgOff);  // [g][m, l][128]

    const int tid = threadIdx.x;
    const int warp = tid / 32;
    if (launch_aborted(p.epoch)) return;

    const long long unit = blockIdx.x;
    const long long bh = unit / p.nb;
    const int qb = static_cast<int>(unit % p.nb);
    int rs = __ldg(p.row_ptr + unit);
    int re = __ldg(p.row_ptr + unit + 1);
    const bool bad_row = rs < 0 || re < rs;
    if (bad_row) re = rs = 0;
    const int n = re - rs;

    if (tid == 256) {
        *abort_flag = 0;
        mbar_init(q_full, 1);
        for (int s = 0; s < NS; ++s) { mbar_init(&kv_full[s], 1); mbar_init(&kv_empty[s], 1); }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&s_full[b], 1);
            mbar_init(&p_full[b], 128);
            mbar_init(&o_ready[b], 1);
        }
        mbar_init(drain, 1);
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
    // ring position of the tiles, in the shared load / MMA order
    //   K_0 -> 0, K_1 -> 1, and for j >= 0: V_j -> 2 + 2j, K_{j+2} -> 3 + 2j
    // (when n == 1: K_0 -> 0, V_0 -> 1)

    if (warp == 8) {
        // ------------------------------------------------------------ TMA producer
        if ((tid & 31) == 0 && n > 0) {
            const uint64_t pol_q = policy_evict_first();
            const uint64_t pol_kv = policy_evict_last();
            const int row0 = static_cast<int>(bh * p.Lp);
            mbar_arrive_expect_tx(q_full, C::kQBytes);
#pragma unroll
            for (int a = 0; a < D / 64; ++a)
                tma_load_2d(sQ + a * 128 * 128, &map_q, q_full, a * 64, row0 + qb * BLK, pol_q);
            int seq = 0;
            bool ok = true;
            auto load = [&](int j, bool is_v) -> bool {
                const int slot = seq % NS;
                const uint32_t ph = (seq / NS) & 1;
                if (!wait(&kv_empty[slot], ph ^ 1)) return false;
                int blk = __ldg(p.col_idx + rs + j);
                if (blk < 0 || blk >= p.nb) blk = 0;  // masked by the softmax warps
                uint8_t* dst = sRing + slot * C::kTile;
                mbar_arrive_expect_tx(&kv_full[slot], C::kTile);
#pragma unroll
                for (int a = 0; a < D / 64; ++a)
                    tma_load_2d(dst + a * BLK * 128, is_v ? &map_v : &map_k, &kv_full[slot], a * 64,
                                row0 + blk * BLK, pol_kv);
                ++seq;
                return true;
            };
            ok = load(0, false);
            if (ok && n > 1) ok = load(1, false);
            for (int j = 0; ok && j < n; ++j) {
                ok = load(j, true);
                if (ok && j + 2 < n) ok = load(j + 2, false);
            }
            if (!ok) {
                // drain: every issued copy must land before the CTA exits
                volatile int never = 0;
                mbar_wait_bounded(q_full, 0, &never, kWaitLimitNs);
                for (int q = seq - NS < 0 ? 0 : seq - NS; q < seq; ++q)
                    mbar_wait_bounded(&kv_full[q % NS], (q / NS) & 1, &never, kWaitLimitNs);
            }
        }
    } else if (warp == 9) {
        // ------------------------------------------------------------ MMA issuer
        if ((tid & 31) == 0 && n > 0) {
            constexpr uint32_t idS = idesc_bf16_f32(128, BLK, false);
            constexpr uint32_t idO = idesc_bf16_f32(128, D, true);
            const uint32_t ring_addr = smem_u32(sRing);
            const uint64_t qdesc0 = sdesc_sw128(smem_u32(sQ), 16, 1024);
            int seq = 0;
            auto issue_qk = [&](int j) -> bool {
                const int slot = seq % NS;
                if (!wait(&kv_full[slot], (seq / NS) & 1)) return false;
                tc_fence_after();
                const uint64_t kdesc0 = sdesc_sw128(ring_addr + slot * C::kTile, 16, 1024);
                const uint32_t d_s = tmem + ((j & 1) ? C::kColS1 : C::kColS0);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    // only the 14-bit start-address field (bytes / 16) moves between K steps
                    const uint64_t da = qdesc0 + static_cast<uint64_t>(((kk / 4) * (128 * 128) + (kk % 4) * 32) >> 4);
                    const uint64_t db = kdesc0 + static_cast<uint64_t>(((kk / 4) * (BLK * 128) + (kk % 4) * 32) >> 4);
                    umma_ss(d_s, da, db, idS, kk > 0 ? 1u : 0u);
                }
                umma_commit(&kv_empty[slot]);
                umma_commit(&s_full[j & 1]);
                ++seq;
                return true;
            };
            bool ok = wait(q_full, 0) && issue_qk(0);
            if (ok && n > 1) ok = issue_qk(1);
            for (int j = 0; ok && j < n; ++j) {
                // V_j first (normally loaded long ago; this wait overlaps QK_{j+1} on the
                // tensor core), then the real dependency: P_j from the softmax warps
                const int slot = seq % NS;
                if (!(ok = wait(&kv_full[slot], (seq / NS) & 1))) break;
                if (!(ok = wait(&p_full[j & 1], (j >> 1) & 1))) break;
                tc_fence_after();
                const uint64_t vdesc0 = sdesc_sw128(ring_addr + slot * C::kTile, BLK * 128, 1024);
                const uint32_t a_p = tmem + ((j & 1) ? C::kColS1 : C::kColS0);
                const uint32_t d_o = tmem + ((j & 1) ? C::kColO1 : C::kColO0);
#pragma unroll
                for (int kk = 0; kk < BLK / 16; ++kk) {
                    const uint64_t db = vdesc0 + static_cast<uint64_t>((kk * 16 * 128) >> 4);
                    umma_ts(d_o, a_p + kk * 8, db, idO, (j > 1 || kk > 0) ? 1u : 0u);
                }
                umma_commit(&kv_empty[slot]);
                if (j + 2 >= n) umma_commit(&o_ready[j & 1]);  // last PV into O_{j&1}
                ++seq;
                if (j + 2 < n) ok = issue_qk(j + 2);
            }
            if (!ok) {
                umma_commit(drain);  // wait for every MMA already issued
                volatile int never = 0;
                mbar_wait_bounded(drain, 0, &never, kWaitLimitNs);
            }
        }
    } else if (warp < 8) {
        // ------------------------------------------------------------ softmax warpgroups
        const int g = warp >> 2;     // this warpgroup's blocks: j = g, g + 2, ...
        const int r = tid & 127;     // row within the 128-row tile
        const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const int t = qb * BLK + r;
        const bool row_in_block = r < BLK;
        const bool row_valid = row_in_block && t < p.L;
        const float sl2 = p.scale_log2;  // |scale| * log2(e) > 0
        const float2 sl2x2 = make_float2(sl2, sl2);
        const uint32_t s_col = tmem + lane_base + (g ? C::kColS1 : C::kColS0);
        const uint32_t o_col = tmem + lane_base + (g ? C::kColO1 : C::kColO0);
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
        int blk_next = g < n ? __ldg(p.col_idx + rs + g) : 0;
        for (int j = g; j < n; j += 2) {
            const int blk = blk_next;
            if (j + 2 < n) blk_next = __ldg(p.col_idx + rs + j + 2);
            if (ok) ok = wait_warp(&s_full[g], (j >> 1) & 1);
            if (!ok) continue;
            tc_fence_after();
            const bool bad = blk < 0 || blk >= p.nb;
            if (bad && r == 0) raise_error(kErrBadIndex);
            const int nvalid = bad ? 0 : min(BLK, p.L - blk * BLK);  // valid keys of the block
            float s[BLK];
            {
                uint32_t raw[BLK];
                tmem_ld_cols<BLK>(s_col, raw);
#pragma unroll
                for (int e = 0; e < BLK; ++e) s[e] = __uint_as_float(raw[e]);
            }
            if (p.neg_scale) {
#pragma unroll
                for (int e = 0; e < BLK; ++e) s[e] = -s[e];
            }
            const bool masked = nvalid < BLK;  // padded tail block or skipped index (uniform)
            if (masked) {
#pragma unroll
                for (int e = 0; e < BLK; ++e)
                    if (e >= nvalid) s[e] = -INFINITY;
            }
            // block max: eight independent chains, then a tree
            float mx8[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) mx8[c] = s[c];
#pragma unroll
            for (int e = 8; e < BLK; ++e) mx8[e & 7] = fmaxf(mx8[e & 7], s[e]);
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
            if (!masked) {
#pragma unroll
                for (int e = 0; e < BLK; e += 2) {
                    const float2 x = __ffma2_rn(make_float2(s[e], s[e + 1]), sl2x2, nm2);
                    float2 pr;
                    if (kPolyPair(e)) {
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
                for (int e = 0; e < BLK; e += 2) {
                    const float2 x = __ffma2_rn(make_float2(s[e], s[e + 1]), sl2x2, nm2);
                    float2 pr;
                    pr.x = ex2_approx(x.x);
                    pr.y = ex2_approx(x.y);
                    sum4[(e >> 1) & 3] = __fadd2_rn(sum4[(e >> 1) & 3], pr);
                    pk[e / 2] = pack_bf16x2(pr.x, pr.y);
                }
            }
            const float2 s01 = __fadd2_rn(sum4[0], sum4[1]);
            const float2 s23 = __fadd2_rn(sum4[2], sum4[3]);
            const float2 sall = __fadd2_rn(s01, s23);
            l = l * alpha + (sall.x + sall.y);
            tmem_st_cols<BLK / 2>(s_col, pk);  // P over the first BLK/2 columns of S
            // O_g already holds every earlier PV of this warpgroup (the commit that
            // signalled S_j covers them): rescale it now that P is out of registers
            if (j > 1 && __any_sync(0xFFFFFFFFu, alpha != 1.f)) {
                const float2 a2 = make_float2(alpha, alpha);
#pragma unroll
                for (int h = 0; h < D; h += 64) {
                    uint32_t ov[D < 64 ? D : 64];
                    tmem_ld_cols<(D < 64 ? D : 64)>(o_col + h, ov);
#pragma unroll
                    for (int e = 0; e < (D < 64 ? D : 64); e += 2) {
                        const float2 v = __fmul2_rn(make_float2(__uint_as_float(ov[e]), __uint_as_float(ov[e + 1])), a2);
                        ov[e] = __float_as_uint(v.x);
                        ov[e + 1] = __float_as_uint(v.y);
                    }
                    tmem_st_cols<(D < 64 ? D : 64)>(o_col + h, ov);
                }
            }
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(&p_full[g]);
        }
        const bool has_blocks = g < n;
        if (ok && has_blocks) ok = wait_warp(&o_ready[g], 0);
        // ---- merge: row r of (m_0, l_0, O_0) and (m_1, l_1, O_1); warpgroup g writes
        // output columns [g D/2, (g+1) D/2)
        xml[(g * 2 + 0) * 128 + r] = has_blocks ? m : -INFINITY;
        xml[(g * 2 + 1) * 128 + r] = has_blocks ? l : 0.f;
        ok = __all_sync(0xFFFFFFFFu, ok);
        tc_fence_before();
        softmax_pair_sync();
        tc_fence_after();
        const float m0 = xml[0 * 128 + r], l0 = xml[1 * 128 + r];
        const float m1 = xml[2 * 128 + r], l1 = xml[3 * 128 + r];
        const float M = fmaxf(m0, m1);
        const float w0 = (m0 == -INFINITY) ? 0.f : ex2_approx(m0 - M);
        const float w1 = (m1 == -INFINITY) ? 0.f : ex2_approx(m1 - M);
        const float lt = w0 * l0 + w1 * l1;
        const bool any_pv = n > 0;
        {
            // every lane of the warp runs the TMEM loads (warp-collective); only rows of
            // this query block are stored
            const bool write_o = ok && any_pv && row_valid && lt > 0.f;
            const float inv = write_o ? 1.f / lt : 0.f;
            const float c0 = w0 * inv, c1 = w1 * inv;
            const bool use1 = n > 1;  // O_1 holds data only if warpgroup 1 had a block
            uint32_t o0[HD], o1[HD];
            if (ok && any_pv) {
                tmem_ld_cols<HD>(tmem + lane_base + C::kColO0 + g * HD, o0);
                if (use1) tmem_ld_cols<HD>(tmem + lane_base + C::kColO1 + g * HD, o1);
            }
            if (row_in_block) {
                uint4* dst = reinterpret_cast<uint4*>(p.o + (bh * p.Lp + t) * D + g * HD);
#pragma unroll
                for (int e = 0; e < HD; e += 8) {
                    float v[8];
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        float x = write_o ? __uint_as_float(o0[e + q]) * c0 : 0.f;
                        if (write_o && use1) x = fmaf(__uint_as_float(o1[e + q]), c1, x);
                        v[q] = x;
                    }
                    uint4 w;
                    w.x = pack_bf16x2(v[0], v[1]);
                    w.y = pack_bf16x2(v[2], v[3]);
                    w.z = pack_bf16x2(v[4], v[5]);
                    w.w = pack_bf16x2(v[6], v[7]);
                    dst[e / 8] = w;
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
