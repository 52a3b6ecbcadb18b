// Step 3: dense softmax attention inside the kept key blocks, on tcgen05 tensor cores.
//
// The kept blocks are computed densely to keep the GPU's throughput (page "单卡 RTX 5090
// 跑 Wan2.2-A14B：720p 视频生成只要 3.8 秒", 四步拆解 item 3 动态稀疏注意力); unkept blocks
// contribute nothing and the softmax is normalised over the kept keys only.
//
// One CTA works on TWO query tiles at once (tile 0 = unit 2c, tile 1 = unit 2c+1,
// units in (b, h, query block) order).  Each tile has its own list of kept key blocks,
// so each has its own K/V stream; the two streams share one ring of shared-memory
// slots.  Interleaving two independent tiles lets the tensor core work on one tile
// while the other tile's softmax runs, and gives every SM sub-partition two softmax
// warps to hide each other's latencies.
//
// 320 threads (ten warps):
//   warpgroup 0 / 1 (softmax of tile 0 / 1): thread r owns query row r.  It reads its
//       row of S = Q K_j^T from TMEM, keeps a running max m and sum l (log2 domain),
//       rescales its row of O in TMEM when m moves, writes P = exp2(S*scale*log2e - m)
//       as bf16 into the first BLK/2 columns of S (P aliases S), and at the end writes
//       O / l as bf16.
//   warp 8 streams Q and the K_j / V_j tiles with TMA (128-byte swizzle);
//       warp 9 allocates 512 TMEM columns and one of its threads issues tcgen05.mma:
//       S = Q K_j^T (both operands in shared memory) and O += P V_j (P from TMEM,
//       V an MN-major shared-memory operand).
// Per tile the tensor-core order is QK_j -> PV_j -> QK_{j+1}; MMAs execute in issue
// order, so QK_{j+1} may overwrite S (and the aliased P) right after PV_j is issued,
// and the commit that signals S_{j+1} also proves PV_j done (O stable to rescale).
// Tiles interleave: QK0_0, QK1_0, PV0_0, QK0_1, PV1_0, QK1_1, PV0_1, ...  The producer
// walks the same sequence (walk_ops), so both sides share one ring order.
//
// TMEM columns: tile t has S at 256 t (BLK fp32 columns; P in its first BLK/2) and O at
// 256 t + 128 (D columns).  For BLK = 64 the 128-row Q tile also holds the next
// block's 64 rows; those rows are computed and discarded.
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
    else tmem_ld32(taddr, r);
}
template <int N>
__device__ __forceinline__ void tmem_st_cols(uint32_t taddr, const uint32_t (&r)[N]) {
    if constexpr (N == 128) tmem_st128(taddr, r);
    else if constexpr (N == 64) tmem_st64(taddr, r);
    else tmem_st32(taddr, r);
}

template <int D, int BLK>
struct AttnCfg {
    static constexpr int kTile = BLK * D * 2;        // bytes of one K or V tile
    static constexpr int kQBytes = 128 * D * 2;      // bytes of one Q tile
    static constexpr int kSmemBudget = 224 * 1024;   // Q tiles + ring
    static constexpr int kStagesRaw = (kSmemBudget - 2 * kQBytes) / kTile;
    static constexpr int kStages = kStagesRaw > 8 ? 8 : kStagesRaw;
    static constexpr int kRingOff = 2 * kQBytes;
    static constexpr int kBarOff = kRingOff + kStages * kTile;
    // barriers: q_full[2], kv_full[S], kv_empty[S], s_full[2], p_full[2], o_ready[2], drain
    static constexpr int kNumBars = 2 + 2 * kStages + 2 + 2 + 2 + 1;
    static constexpr int kSmemBytes = kBarOff + kNumBars * 8 + 16 + 1024;  // + tmem slot/flag + align
    static constexpr int kThreads = 320;
    static_assert(kStages >= 2, "need at least two ring slots");
    static_assert(D == 64 || D == 128, "head_dim");
    static_assert(BLK == 64 || BLK == 128, "block_size");
    static_assert(kSmemBytes <= 232448, "shared memory");
};

__host__ __device__ constexpr uint32_t tmem_col_s(int tile) { return tile ? 256u : 0u; }
__host__ __device__ constexpr uint32_t tmem_col_o(int tile) { return tile ? 384u : 128u; }

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

// Visits the tensor-core operations of the two tiles in issue order:
//   QK(0,0), QK(1,0), then for j = 0, 1, ...: PV(0,j), QK(0,j+1), PV(1,j), QK(1,j+1)
// skipping entries past a tile's list.  The producer and the MMA issuer both walk it,
// so ring slots are filled and drained in the same order.  Every call of f has literal
// tile / is_v arguments, so after inlining its per-tile state stays in registers.
// f(tile, is_v, j) returns false to stop the walk.
template <typename F>
__device__ __forceinline__ bool walk_ops(int n0, int n1, F&& f) {
    if (n0 > 0 && !f(0, false, 0)) return false;
    if (n1 > 0 && !f(1, false, 0)) return false;
    const int nmax = max(n0, n1);
    for (int j = 0; j < nmax; ++j) {
        if (j < n0) {
            if (!f(0, true, j)) return false;
            if (j + 1 < n0 && !f(0, false, j + 1)) return false;
        }
        if (j < n1) {
            if (!f(1, true, j)) return false;
            if (j + 1 < n1 && !f(1, false, j + 1)) return false;
        }
    }
    return true;
}

template <int D, int BLK>
__global__ void __launch_bounds__(320, 1) attn_kernel(const __grid_constant__ CUtensorMap map_q,
                                                      const __grid_constant__ CUtensorMap map_k,
                                                      const __grid_constant__ CUtensorMap map_v,
                                                      const AttnParams p) {
    using C = AttnCfg<D, BLK>;
    constexpr int NS = C::kStages;
    extern __shared__ __align__(1024) uint8_t attn_smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(attn_smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sQ = smem;  // two Q tiles
    uint8_t* sRing = smem + C::kRingOff;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
    uint64_t* q_full = bars;
    uint64_t* kv_full = bars + 2;
    uint64_t* kv_empty = kv_full + NS;
    uint64_t* s_full = kv_empty + NS;
    uint64_t* p_full = s_full + 2;
    uint64_t* o_ready = p_full + 2;
    uint64_t* drain = o_ready + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::kNumBars);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int tid = threadIdx.x;
    const int warp = tid / 32;
    if (launch_aborted(p.epoch)) return;

    // the two units of this CTA and their kept-block lists
    long long unit[2];
    int rs[2], n[2];
    bool bad_row = false;
#pragma unroll
    for (int t = 0; t < 2; ++t) {
        unit[t] = 2ll * blockIdx.x + t;
        rs[t] = 0;
        n[t] = 0;
        if (unit[t] < p.units) {
            const int a = __ldg(p.row_ptr + unit[t]);
            const int b = __ldg(p.row_ptr + unit[t] + 1);
            if (a < 0 || b < a) bad_row = true;
            else { rs[t] = a; n[t] = b - a; }
        }
    }

    if (tid == 256) {
        *abort_flag = 0;
        for (int t = 0; t < 2; ++t) {
            mbar_init(&q_full[t], 1);
            mbar_init(&s_full[t], 1);
            mbar_init(&p_full[t], 128);
            mbar_init(&o_ready[t], 1);
        }
        for (int s = 0; s < NS; ++s) { mbar_init(&kv_full[s], 1); mbar_init(&kv_empty[s], 1); }
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

    if (warp == 8) {
        // ------------------------------------------------------------ TMA producer
        if ((tid & 31) == 0) {
            const uint64_t pol_q = policy_evict_first();
            const uint64_t pol_kv = policy_evict_last();
            int row0[2];
#pragma unroll
            for (int t = 0; t < 2; ++t) {
                const long long bh = unit[t] / p.nb;
                row0[t] = static_cast<int>(bh * p.Lp);
                if (n[t] > 0) {
                    const int qb = static_cast<int>(unit[t] % p.nb);
                    mbar_arrive_expect_tx(&q_full[t], C::kQBytes);
#pragma unroll
                    for (int a = 0; a < D / 64; ++a)
                        tma_load_2d(sQ + t * C::kQBytes + a * 128 * 128, &map_q, &q_full[t], a * 64,
                                    row0[t] + qb * BLK, pol_q);
                }
            }
            const int rs0 = rs[0], rs1 = rs[1], r00 = row0[0], r01 = row0[1];
            int seq = 0;
            const bool ok = walk_ops(n[0], n[1], [&](int tile, bool is_v, int j) -> bool {
                const int slot = seq % NS;
                const uint32_t ph = (seq / NS) & 1;
                if (!wait(&kv_empty[slot], ph ^ 1)) return false;
                int blk = __ldg(p.col_idx + (tile ? rs1 : rs0) + j);
                if (blk < 0 || blk >= p.nb) blk = 0;  // masked by the softmax warps
                uint8_t* dst = sRing + slot * C::kTile;
                mbar_arrive_expect_tx(&kv_full[slot], C::kTile);
#pragma unroll
                for (int a = 0; a < D / 64; ++a)
                    tma_load_2d(dst + a * BLK * 128, is_v ? &map_v : &map_k, &kv_full[slot], a * 64,
                                (tile ? r01 : r00) + blk * BLK, pol_kv);
                ++seq;
                return true;
            });
            if (!ok) {
                // drain: every issued copy must land before the CTA exits
                volatile int never = 0;
                for (int t = 0; t < 2; ++t)
                    if (n[t] > 0) mbar_wait_bounded(&q_full[t], 0, &never, kWaitLimitNs);
                for (int q = seq - NS < 0 ? 0 : seq - NS; q < seq; ++q)
                    mbar_wait_bounded(&kv_full[q % NS], (q / NS) & 1, &never, kWaitLimitNs);
            }
        }
    } else if (warp == 9) {
        // ------------------------------------------------------------ MMA issuer
        if ((tid & 31) == 0) {
            constexpr uint32_t idS = idesc_bf16_f32(128, BLK, false);
            constexpr uint32_t idO = idesc_bf16_f32(128, D, true);
            const uint32_t ring_addr = smem_u32(sRing);
            const int n0 = n[0], n1 = n[1];
            int seq = 0;
            const bool ok = walk_ops(n0, n1, [&](int tile, bool is_v, int j) -> bool {
                const int slot = seq % NS;
                if (is_v) {
                    if (!wait(&p_full[tile], j & 1)) return false;
                } else if (j == 0) {
                    if (!wait(&q_full[tile], 0)) return false;
                }
                if (!wait(&kv_full[slot], (seq / NS) & 1)) return false;
                tc_fence_after();
                const uint32_t tile_addr = ring_addr + slot * C::kTile;
                if (!is_v) {
                    const uint32_t q_addr = smem_u32(sQ) + tile * C::kQBytes;
                    const uint32_t d_s = tmem + tmem_col_s(tile);
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint64_t da = sdesc_sw128(q_addr + (kk / 4) * (128 * 128) + (kk % 4) * 32, 16, 1024);
                        const uint64_t db = sdesc_sw128(tile_addr + (kk / 4) * (BLK * 128) + (kk % 4) * 32, 16, 1024);
                        umma_ss(d_s, da, db, idS, kk > 0 ? 1u : 0u);
                    }
                    umma_commit(&kv_empty[slot]);
                    umma_commit(&s_full[tile]);
                } else {
                    const uint32_t a_p = tmem + tmem_col_s(tile);
#pragma unroll
                    for (int kk = 0; kk < BLK / 16; ++kk) {
                        const uint64_t db = sdesc_sw128(tile_addr + kk * 16 * 128, BLK * 128, 1024);
                        umma_ts(tmem + tmem_col_o(tile), a_p + kk * 8, db, idO, (j > 0 || kk > 0) ? 1u : 0u);
                    }
                    umma_commit(&kv_empty[slot]);
                    if (j == (tile ? n1 : n0) - 1) umma_commit(&o_ready[tile]);
                }
                ++seq;
                return true;
            });
            if (!ok) {
                umma_commit(drain);  // wait for every MMA already issued
                volatile int never = 0;
                mbar_wait_bounded(drain, 0, &never, kWaitLimitNs);
            }
        }
    } else if (warp < 8) {
        // ------------------------------------------------------------ softmax, tile = warpgroup
        const int tile = warp >> 2;
        const int r = tid & 127;  // row within the 128-row tile
        const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const long long my_unit = tile ? unit[1] : unit[0];
        const int my_rs = tile ? rs[1] : rs[0];
        const long long bh = my_unit / p.nb;
        const int qb = static_cast<int>(my_unit % p.nb);
        const int nt = tile ? n[1] : n[0];
        const int t = qb * BLK + r;
        const bool row_in_block = r < BLK && my_unit < p.units;
        const bool row_valid = row_in_block && t < p.L;
        const float sl2 = p.scale_log2;  // |scale| * log2(e) > 0
        const float2 sl2x2 = make_float2(sl2, sl2);
        const uint32_t s_col = tmem + lane_base + tmem_col_s(tile);
        const uint32_t o_col = tmem + lane_base + tmem_col_o(tile);
        float m = -INFINITY;  // running reference max (log2 domain), possibly stale by < 8
        float l = 0.f;
        bool ok = true;
        // tcgen05.ld/st are warp-collective: every decision that guards one is made
        // warp-uniform (a wait's outcome included).
        auto wait_warp = [&](uint64_t* bar, uint32_t parity) -> bool {
            const bool w = wait(bar, parity);
            return __all_sync(0xFFFFFFFFu, w);
        };
        int blk_next = nt > 0 ? __ldg(p.col_idx + my_rs) : 0;
        for (int j = 0; j < nt; ++j) {
            const int blk = blk_next;
            if (j + 1 < nt) blk_next = __ldg(p.col_idx + my_rs + j + 1);
            if (!(ok = wait_warp(&s_full[tile], j & 1))) break;
            tc_fence_after();
            const bool bad = blk < 0 || blk >= p.nb;
            if (bad && r == 0) raise_error(kErrBadIndex);
            const int nvalid = bad ? 0 : min(BLK, p.L - blk * BLK);
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
            // O already holds PV_{j-1} (the commit that signalled S_j covers it); rescale
            // it now that P is out of registers, in halves to bound register use.
            if (j > 0 && __any_sync(0xFFFFFFFFu, alpha != 1.f)) {
                const float2 a2 = make_float2(alpha, alpha);
#pragma unroll
                for (int h = 0; h < D; h += 64) {
                    uint32_t ov[64];
                    tmem_ld64(o_col + h, ov);
#pragma unroll
                    for (int e = 0; e < 64; e += 2) {
                        const float2 v = __fmul2_rn(make_float2(__uint_as_float(ov[e]), __uint_as_float(ov[e + 1])), a2);
                        ov[e] = __float_as_uint(v.x);
                        ov[e + 1] = __float_as_uint(v.y);
                    }
                    tmem_st64(o_col + h, ov);
                }
            }
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(&p_full[tile]);
        }
        if (ok && nt > 0) ok = wait_warp(&o_ready[tile], 0);
        tc_fence_after();
        // epilogue: O / l as bf16; rows past L (and rows with no valid key) are zero
        if (row_in_block) {
            uint4* dst = reinterpret_cast<uint4*>(p.o + (bh * p.Lp + t) * D);
            const bool write_o = ok && nt > 0 && row_valid && l > 0.f;
            const float inv = write_o ? 1.f / l : 0.f;
#pragma unroll
            for (int h = 0; h < D; h += 64) {
                uint32_t ov[64];
                if (nt > 0 && ok) tmem_ld64(o_col + h, ov);
#pragma unroll
                for (int e = 0; e < 64; e += 8) {
                    uint4 w;
                    if (write_o) {
                        w.x = pack_bf16x2(__uint_as_float(ov[e]) * inv, __uint_as_float(ov[e + 1]) * inv);
                        w.y = pack_bf16x2(__uint_as_float(ov[e + 2]) * inv, __uint_as_float(ov[e + 3]) * inv);
                        w.z = pack_bf16x2(__uint_as_float(ov[e + 4]) * inv, __uint_as_float(ov[e + 5]) * inv);
                        w.w = pack_bf16x2(__uint_as_float(ov[e + 6]) * inv, __uint_as_float(ov[e + 7]) * inv);
                    } else {
                        w = make_uint4(0, 0, 0, 0);
                    }
                    dst[(h + e) / 8] = w;
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
