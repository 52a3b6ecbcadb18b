// Step 3: dense softmax attention inside the kept key blocks, on tcgen05 tensor cores.
//
// The kept blocks are computed densely to keep the GPU's throughput (page "单卡 RTX 5090
// 跑 Wan2.2-A14B：720p 视频生成只要 3.8 秒", 四步拆解 item 3 动态稀疏注意力); unkept blocks
// contribute nothing and the softmax is normalised over the kept keys only.
//
// One CTA per (b, h, query block i); 192 threads in three roles:
//   warps 0-3 (softmax): thread r owns query row r of the 128-row tile.  It reads its
//       row of S = Q K_j^T from TMEM, keeps a running max m and sum l (log2 domain),
//       writes P = exp2(S*scale*log2e - m) as bf16 into TMEM, rescales its row of the
//       O accumulator in TMEM when m moves, and finally writes O / l as bf16.
//   warp 4 (load): one thread streams the Q tile and then the K_j / V_j tiles of the
//       kept blocks through a ring of shared-memory slots with TMA (128-byte swizzle).
//   warp 5 (MMA): allocates 512 TMEM columns; one thread issues the tcgen05.mma:
//       S_j = Q K_j^T (A and B from shared memory) into one of two S buffers, and
//       O += P_j V_j (P from TMEM, V from shared memory as an MN-major operand).
// Order on the tensor core: QK_0, QK_1, PV_0, QK_2, PV_1, ...  so S_{j+1} is computed
// while the softmax warps work on S_j.  The load order K_0, K_1, V_0, K_2, V_1, ...
// is the same sequence, so producer and consumer walk one ring.
//
// TMEM columns: S buffers at 0 and 128 (BLK fp32 columns each), O at 256 (D columns),
// P buffers at 384 and 448 (BLK/2 columns each: bf16 pairs, even element low).
// For BLK = 64 the 128-row Q tile also holds the next block's 64 rows; those rows are
// computed and discarded.
//
// Every wait is bounded (kWaitLimitNs); a wait that runs out latches SBSA_ERR_TIMEOUT,
// makes every CTA of the launch give up, drains this CTA's own copies and MMAs and
// frees its TMEM before returning.
#pragma once
#include "common.cuh"
#include "ptx.cuh"

namespace sbsa {

template <int D, int BLK>
struct AttnCfg {
    static constexpr int kTile = BLK * D * 2;      // bytes of one K or V tile
    static constexpr int kQBytes = 128 * D * 2;    // bytes of the Q tile
    static constexpr int kSmemBudget = 200 * 1024; // tiles only
    static constexpr int kStagesRaw = (kSmemBudget - kQBytes) / kTile;
    static constexpr int kStages = kStagesRaw > 8 ? 8 : kStagesRaw;
    static constexpr int kColS0 = 0, kColS1 = 128, kColO = 256, kColP0 = 384, kColP1 = 448;
    static constexpr int kBarOff = kQBytes + kStages * kTile;
    // barriers: q_full, kv_full[S], kv_empty[S], s_full[2], p_full[2], o_ready, drain
    static constexpr int kNumBars = 1 + 2 * kStages + 2 + 2 + 1 + 1;
    static constexpr int kSmemBytes = kBarOff + kNumBars * 8 + 16 + 1024;  // + tmem slot/flag + align
    static_assert(kStages >= 2, "need at least two ring slots");
    static_assert(D == 64 || D == 128, "head_dim");
    static_assert(BLK == 64 || BLK == 128, "block_size");
};

struct AttnParams {
    const int32_t* row_ptr;
    const int32_t* col_idx;
    __nv_bfloat16* o;
    int L, Lp, nb;
    float scale_log2;  // scale * log2(e)
    unsigned int epoch;
};

template <int D, int BLK>
__global__ void __launch_bounds__(192, 1) attn_kernel(const __grid_constant__ CUtensorMap map_q,
                                                      const __grid_constant__ CUtensorMap map_k,
                                                      const __grid_constant__ CUtensorMap map_v,
                                                      const AttnParams p) {
    using C = AttnCfg<D, BLK>;
    constexpr int NS = C::kStages;
    extern __shared__ __align__(1024) uint8_t attn_smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(attn_smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sQ = smem;
    uint8_t* sRing = smem + C::kQBytes;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
    uint64_t* q_full = bars;
    uint64_t* kv_full = bars + 1;
    uint64_t* kv_empty = bars + 1 + NS;
    uint64_t* s_full = bars + 1 + 2 * NS;
    uint64_t* p_full = s_full + 2;
    uint64_t* o_ready = p_full + 2;
    uint64_t* drain = o_ready + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::kNumBars);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int tid = threadIdx.x;
    const int warp = tid / 32;
    const long long unit = blockIdx.x;
    const long long bh = unit / p.nb;
    const int qb = static_cast<int>(unit % p.nb);

    if (launch_aborted(p.epoch)) return;

    if (tid == 128) {
        *abort_flag = 0;
        mbar_init(q_full, 1);
        for (int s = 0; s < NS; ++s) { mbar_init(&kv_full[s], 1); mbar_init(&kv_empty[s], 1); }
        for (int b = 0; b < 2; ++b) { mbar_init(&s_full[b], 1); mbar_init(&p_full[b], 128); }
        mbar_init(o_ready, 1);
        mbar_init(drain, 1);
        fence_mbar_init();
        tma_prefetch_desc(&map_q);
        tma_prefetch_desc(&map_k);
        tma_prefetch_desc(&map_v);
    }
    if (warp == 5) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // the kept-block list of this query block
    int rs = __ldg(p.row_ptr + unit);
    int re = __ldg(p.row_ptr + unit + 1);
    if (rs < 0 || re < rs) {
        if (tid == 0) raise_error(kErrBadIndex);
        re = rs = 0;
    }
    const int n = re - rs;

    auto give_up = [&]() {
        *abort_flag = 1;
        abort_launch(p.epoch);
    };
    auto wait = [&](uint64_t* bar, uint32_t parity) -> bool {
        if (mbar_wait_bounded(bar, parity, abort_flag, kWaitLimitNs)) return true;
        if (!*abort_flag) give_up();
        return false;
    };

    if (warp == 4) {
        // ------------------------------------------------------------ TMA producer
        if ((tid & 31) == 0) {
            const uint64_t pol_q = policy_evict_first();
            const uint64_t pol_kv = policy_evict_last();
            const int row0 = static_cast<int>(bh * p.Lp);
            if (n > 0) {
                mbar_arrive_expect_tx(q_full, C::kQBytes);
#pragma unroll
                for (int a = 0; a < D / 64; ++a)
                    tma_load_2d(sQ + a * 128 * 128, &map_q, q_full, a * 64, row0 + qb * BLK, pol_q);
            }
            int issued_phase[NS];
            bool any_issued[NS];
#pragma unroll
            for (int s = 0; s < NS; ++s) { issued_phase[s] = 0; any_issued[s] = false; }
            const int total = 2 * n;
            bool ok = true;
            for (int s = 0; s < total && ok; ++s) {
                // sequence: K_0, then for j: K_{j+1} (if any), V_j
                int j, is_v;
                if (s == 0) { j = 0; is_v = 0; }
                else {
                    const int jj = (s - 1) / 2;
                    const bool has_next = jj + 1 < n;
                    if (has_next) { if ((s - 1) % 2 == 0) { j = jj + 1; is_v = 0; } else { j = jj; is_v = 1; } }
                    else { j = jj; is_v = 1; }
                }
                const int slot = s % NS;
                const uint32_t ph = (s / NS) & 1;
                if (!wait(&kv_empty[slot], ph ^ 1)) { ok = false; break; }
                int blk = __ldg(p.col_idx + rs + j);
                if (blk < 0 || blk >= p.nb) blk = 0;  // masked by the softmax warps
                uint8_t* dst = sRing + slot * C::kTile;
                mbar_arrive_expect_tx(&kv_full[slot], C::kTile);
#pragma unroll
                for (int a = 0; a < D / 64; ++a)
                    tma_load_2d(dst + a * BLK * 128, is_v ? &map_v : &map_k, &kv_full[slot], a * 64,
                                row0 + blk * BLK, pol_kv);
                issued_phase[slot] = static_cast<int>(ph);
                any_issued[slot] = true;
            }
            if (!ok) {
                // drain: every issued copy must land before the CTA exits
                volatile int never = 0;
                mbar_wait_bounded(q_full, 0, &never, kWaitLimitNs);
                for (int s = 0; s < NS; ++s)
                    if (any_issued[s]) mbar_wait_bounded(&kv_full[s], issued_phase[s], &never, kWaitLimitNs);
            }
        }
    } else if (warp == 5) {
        // ------------------------------------------------------------ MMA issuer
        if ((tid & 31) == 0) {
            constexpr uint32_t idS = idesc_bf16_f32(128, BLK, false);
            constexpr uint32_t idO = idesc_bf16_f32(128, D, true);
            const uint32_t q_addr = smem_u32(sQ);
            const uint32_t ring_addr = smem_u32(sRing);
            int seq = 0;
            bool ok = n == 0 || wait(q_full, 0);  // no Q copy is issued when n == 0
            auto issue_qk = [&](int j) -> bool {
                const int slot = seq % NS;
                if (!wait(&kv_full[slot], (seq / NS) & 1)) return false;
                tc_fence_after();
                const uint32_t kaddr = ring_addr + slot * C::kTile;
                const uint32_t d_s = tmem + ((j & 1) ? C::kColS1 : C::kColS0);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t da = sdesc_sw128(q_addr + (kk / 4) * (128 * 128) + (kk % 4) * 32, 16, 1024);
                    const uint64_t db = sdesc_sw128(kaddr + (kk / 4) * (BLK * 128) + (kk % 4) * 32, 16, 1024);
                    umma_ss(d_s, da, db, idS, kk > 0 ? 1u : 0u);
                }
                umma_commit(&kv_empty[slot]);
                umma_commit(&s_full[j & 1]);
                ++seq;
                return true;
            };
            if (ok && n > 0) ok = issue_qk(0);
            for (int j = 0; j < n && ok; ++j) {
                if (j + 1 < n && !(ok = issue_qk(j + 1))) break;
                if (!(ok = wait(&p_full[j & 1], (j >> 1) & 1))) break;
                const int slot = seq % NS;
                if (!(ok = wait(&kv_full[slot], (seq / NS) & 1))) break;
                tc_fence_after();
                const uint32_t vaddr = ring_addr + slot * C::kTile;
                const uint32_t a_p = tmem + ((j & 1) ? C::kColP1 : C::kColP0);
#pragma unroll
                for (int kk = 0; kk < BLK / 16; ++kk) {
                    const uint64_t db = sdesc_sw128(vaddr + kk * 16 * 128, BLK * 128, 1024);
                    umma_ts(tmem + C::kColO, a_p + kk * 8, db, idO, (j > 0 || kk > 0) ? 1u : 0u);
                }
                umma_commit(&kv_empty[slot]);
                umma_commit(o_ready);
                ++seq;
            }
            if (!ok) {
                umma_commit(drain);  // wait for every MMA already issued
                volatile int never = 0;
                mbar_wait_bounded(drain, 0, &never, kWaitLimitNs);
            }
        }
    } else {
        // ------------------------------------------------------------ softmax warps 0-3
        const int r = tid;  // row within the 128-row tile
        const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
        const int t = qb * BLK + r;
        const bool row_in_block = r < BLK;
        const bool row_valid = row_in_block && t < p.L;
        float m = -INFINITY;  // running max (log2 domain), possibly stale by < 8
        float l = 0.f;
        bool ok = true;
        // tcgen05.ld/st are warp-collective: every decision that guards one is made
        // warp-uniform (a wait's outcome included).
        auto wait_warp = [&](uint64_t* bar, uint32_t parity) -> bool {
            const bool r = wait(bar, parity);
            return __all_sync(0xFFFFFFFFu, r);
        };
        for (int j = 0; j < n; ++j) {
            const int b = j & 1;
            if (!(ok = wait_warp(&s_full[b], (j >> 1) & 1))) break;
            tc_fence_after();
            int blk = __ldg(p.col_idx + rs + j);
            int nvalid;
            if (blk < 0 || blk >= p.nb) {
                if (r == 0) raise_error(kErrBadIndex);
                nvalid = 0;
            } else {
                nvalid = min(BLK, p.L - blk * BLK);
            }
            float x[BLK];
#pragma unroll
            for (int c = 0; c < BLK / 32; ++c) {
                uint32_t v[32];
                tmem_ld32(tmem + lane_base + (b ? C::kColS1 : C::kColS0) + c * 32, v);
#pragma unroll
                for (int e = 0; e < 32; ++e) x[c * 32 + e] = __uint_as_float(v[e]) * p.scale_log2;
            }
            float mx = -INFINITY;
#pragma unroll
            for (int e = 0; e < BLK; ++e) {
                if (e >= nvalid) x[e] = -INFINITY;
                mx = fmaxf(mx, x[e]);
            }
            // Lazy rescaling: keep the old reference max unless the block's max exceeds
            // it by more than 8 (values up to 2^8 are safe in bf16 P and fp32 O / l).
            float alpha = 1.f;
            if (mx > m + 8.f) {
                alpha = (m == -INFINITY) ? 0.f : ex2_approx(m - mx);
                m = mx;
            }
            const float mref = (m == -INFINITY) ? 0.f : m;
            float rowsum = 0.f;
            uint32_t pk[BLK / 2];
#pragma unroll
            for (int e = 0; e < BLK / 2; ++e) {
                const float p0 = ex2_approx(x[2 * e] - mref);
                const float p1 = ex2_approx(x[2 * e + 1] - mref);
                rowsum += p0 + p1;
                pk[e] = pack_bf16x2(p0, p1);
            }
            l = l * alpha + rowsum;
            const uint32_t pcol = tmem + lane_base + (b ? C::kColP1 : C::kColP0);
#pragma unroll
            for (int c = 0; c < BLK / 64; ++c) tmem_st32(pcol + c * 32, *reinterpret_cast<uint32_t(*)[32]>(pk + c * 32));
            if (j > 0) {
                // O must hold PV_{j-1} before it is rescaled (and before P_{j+1} reuses
                // the P buffer PV_{j-1} read).
                if (!(ok = wait_warp(o_ready, (j - 1) & 1))) break;
                tc_fence_after();
                if (__any_sync(0xFFFFFFFFu, alpha != 1.f)) {
#pragma unroll
                    for (int c = 0; c < D / 32; ++c) {
                        uint32_t v[32];
                        tmem_ld32(tmem + lane_base + C::kColO + c * 32, v);
#pragma unroll
                        for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * alpha);
                        tmem_st32(tmem + lane_base + C::kColO + c * 32, v);
                    }
                }
            }
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(&p_full[b]);
        }
        if (ok && n > 0) ok = wait_warp(o_ready, (n - 1) & 1);
        tc_fence_after();
        // epilogue: O / l as bf16; rows past L (and rows with no valid key) are zero
        if (row_in_block) {
            uint4* dst = reinterpret_cast<uint4*>(p.o + (bh * p.Lp + t) * D);
            const bool write_o = ok && n > 0 && row_valid && l > 0.f;
            const float inv = write_o ? 1.f / l : 0.f;
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t v[32];
                if (n > 0 && ok) tmem_ld32(tmem + lane_base + C::kColO + c * 32, v);
#pragma unroll
                for (int e = 0; e < 32; e += 8) {
                    uint4 w;
                    if (write_o) {
                        w.x = pack_bf16x2(__uint_as_float(v[e]) * inv, __uint_as_float(v[e + 1]) * inv);
                        w.y = pack_bf16x2(__uint_as_float(v[e + 2]) * inv, __uint_as_float(v[e + 3]) * inv);
                        w.z = pack_bf16x2(__uint_as_float(v[e + 4]) * inv, __uint_as_float(v[e + 5]) * inv);
                        w.w = pack_bf16x2(__uint_as_float(v[e + 6]) * inv, __uint_as_float(v[e + 7]) * inv);
                    } else {
                        w = make_uint4(0, 0, 0, 0);
                    }
                    dst[(c * 32 + e) / 8] = w;
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 5) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace sbsa
