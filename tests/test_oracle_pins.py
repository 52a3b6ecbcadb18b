"""Pins for the CPU oracle: each check comes from something other than the oracle.

Sources of truth used here:
  * the hand-computed 4-block example in tests/golden/four_block_example.json;
  * closed forms (constant inputs, uniform softmax when Q = 0, block-indicator V);
  * special cases that reduce to a library routine (keep every block -> dense softmax
    attention, computed by torch's fp64 scaled_dot_product_attention);
  * the defining property of a top-k (every kept score >= every dropped one, ties to
    the lower index) and invariances (permuting keys inside a block).

Each is chosen so that a plausible mistake in the oracle -- dividing by the block size
instead of the valid-token count, counting padded keys, dropping the max subtraction,
a transposed operand, an off-by-one in the block gather, a wrong tie order -- fails at
least one test.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from video_dit_dynamic_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "four_block_example.json")


def _golden():
    with open(GOLDEN) as f:
        return json.load(f)


def _arr(x):
    return np.asarray(x, dtype=np.float64)


def _as4(x):  # [L, d] -> [1, 1, L, d]
    return _arr(x)[None, None]


def _sdpa(q, k, v, scale, key_mask=None):
    """Dense softmax attention in fp64 via torch's library routine."""
    tq, tk, tv = (torch.from_numpy(np.asarray(a, dtype=np.float64)) for a in (q, k, v))
    mask = None if key_mask is None else torch.from_numpy(key_mask)
    return torch.nn.functional.scaled_dot_product_attention(
        tq, tk, tv, attn_mask=mask, scale=scale).numpy()


# ---------------------------------------------------------------- pool

def test_pool_hand_example():
    g = _golden()
    qm = oracle.pool(_as4(g["Q"]), g["L"], g["blk"])
    km = oracle.pool(_as4(g["K"]), g["L"], g["blk"])
    np.testing.assert_array_equal(qm[0, 0], _arr(g["qmean"]))
    np.testing.assert_array_equal(km[0, 0], _arr(g["kmean"]))


def test_pool_partial_last_block_ignores_padding():
    g = _golden()
    p = g["partial_block"]
    Q = _arr(g["Q"]).copy()
    K = _arr(g["K"]).copy()
    Q[7] = p["Q_row7_junk"]
    K[7] = p["K_row7_junk"]
    qm = oracle.pool(Q[None, None], p["L"], g["blk"])
    km = oracle.pool(K[None, None], p["L"], g["blk"])
    np.testing.assert_array_equal(qm[0, 0], _arr(p["qmean"]))
    np.testing.assert_array_equal(km[0, 0], _arr(p["kmean"]))


def test_pool_block_constant_input():
    B, H, nb, blk, d = 2, 3, 5, 4, 8
    rng = np.random.default_rng(7)
    c = rng.normal(size=(B, H, nb, d))
    x = np.repeat(c, blk, axis=2)  # every token of block i equals c[..., i, :]
    L = nb * blk - 3               # partial last block: still the constant
    np.testing.assert_allclose(oracle.pool(x, L, blk), c, rtol=0, atol=1e-15)


def test_pool_reads_bf16_bits_exactly():
    # bf16 patterns for 1.0, -2.0, 0.5, 3.0 (sign | exponent | 7-bit mantissa)
    bits = np.array([0x3F80, 0xC000, 0x3F00, 0x4040], dtype=np.uint16).reshape(1, 1, 4, 1)
    qm = oracle.pool(bits, 4, 2)
    np.testing.assert_array_equal(qm.reshape(-1), [(1.0 - 2.0) / 2, (0.5 + 3.0) / 2])


# ---------------------------------------------------------------- select

def test_select_hand_example_with_ties():
    g = _golden()
    qm, km = _arr(g["qmean"])[None, None], _arr(g["kmean"])[None, None]
    for i in range(4):
        s, _ = oracle.score_row(qm[0, 0], km[0, 0], i)
        np.testing.assert_array_equal(s, _arr(g["scores"][i]))
    np.testing.assert_array_equal(oracle.select(qm, km, 2)[0, 0], g["col_idx_k2"])
    np.testing.assert_array_equal(oracle.select(qm, km, 3)[0, 0], g["col_idx_k3"])


def test_select_k_all_and_k_one():
    rng = np.random.default_rng(1)
    qm = rng.normal(size=(1, 2, 9, 4))
    km = rng.normal(size=(1, 2, 9, 4))
    np.testing.assert_array_equal(oracle.select(qm, km, 9), np.broadcast_to(np.arange(9), (1, 2, 9, 9)))
    np.testing.assert_array_equal(oracle.select(qm, km, 1)[..., 0], np.broadcast_to(np.arange(9), (1, 2, 9)))


def test_select_is_a_topk_with_diagonal():
    """Defining property: ascending, contains i, and every kept off-diagonal score is
    >= every dropped score (strictly greater, or equal with a lower index)."""
    rng = np.random.default_rng(2)
    B, H, nb, d, k = 1, 2, 16, 8, 5
    qm = rng.normal(size=(B, H, nb, d))
    km = rng.normal(size=(B, H, nb, d))
    col, kth = oracle.select(qm, km, k, want_kth=True)
    for h in range(H):
        S = qm[0, h] @ km[0, h].T  # independent score computation (numpy matmul)
        for i in range(nb):
            row = col[0, h, i]
            assert list(row) == sorted(set(row)) and i in row and len(row) == k
            kept = [j for j in row if j != i]
            dropped = [j for j in range(nb) if j not in row]
            for a in kept:
                for b in dropped:
                    assert S[i, a] > S[i, b] or (S[i, a] == S[i, b] and a < b)
            assert math.isclose(kth[0, h, i], min(S[i, a] for a in kept), rel_tol=1e-12)


def test_select_exact_ties_prefer_lower_index():
    # key blocks 2, 5 and 7 are identical copies: exact ties between them
    rng = np.random.default_rng(3)
    nb, d = 8, 4
    qm = rng.normal(size=(1, 1, nb, d))
    km = rng.normal(size=(1, 1, nb, d)) * 0.01
    km[0, 0, 5] = km[0, 0, 7] = km[0, 0, 2] = qm[0, 0, 0] * 3.0  # the top score for row 0
    col = oracle.select(qm, km, 3)  # row 0: diag + two of {2, 5, 7}
    np.testing.assert_array_equal(col[0, 0, 0], [0, 2, 5])
    col = oracle.select(qm, km, 2)
    np.testing.assert_array_equal(col[0, 0, 0], [0, 2])


def test_select_rejects_bad_k():
    qm = np.zeros((1, 1, 4, 2))
    with pytest.raises(ValueError):
        oracle.select(qm, qm, 0)
    with pytest.raises(ValueError):
        oracle.select(qm, qm, 5)


def test_keep_blocks_rounding():
    assert [oracle.keep_blocks(256, f) for f in (1.0, 0.5, 0.3, 0.2, 0.1)] == [256, 128, 77, 51, 26]
    assert oracle.keep_blocks(960, 0.1) == 96
    assert oracle.keep_blocks(591, 0.15) == 89
    assert oracle.keep_blocks(16, 0.25) == 4
    assert oracle.keep_blocks(10, 0.0) == 1


# ---------------------------------------------------------------- attention

def test_attention_hand_example_exact_rationals():
    g = _golden()
    q, k, v = _as4(g["Q"]), _as4(g["K"]), _as4(g["V"])
    out, col, qm, km = oracle.forward(q, k, v, g["L"], g["blk"], 2, scale=math.log(2.0))
    np.testing.assert_array_equal(col[0, 0], g["col_idx_k2"])
    want0 = [float(Fraction(s)) for s in g["out_k2_col0"]]
    want1 = [float(Fraction(s)) for s in g["out_k2_col1"]]
    np.testing.assert_allclose(out[0, 0, :, 0], want0, rtol=1e-13, atol=0)
    np.testing.assert_allclose(out[0, 0, :, 1], want1, rtol=1e-13, atol=0)


@pytest.mark.parametrize("L", [96, 90])
def test_attention_keep_all_equals_dense_sdpa(L):
    """k = nb: the sparse path must be dense softmax attention over the valid keys."""
    B, H, blk, d = 1, 2, 16, 8
    Lp = -(-L // blk) * blk
    nb = Lp // blk
    q, k, v = (t.double().numpy() for t in inputs.random_qkv(B, H, Lp, d, L=L, seed=4, dtype=torch.float64))
    k[:, :, L:] = 5.0  # junk in padded keys must not matter
    v[:, :, L:] = 7.0
    out, col, _, _ = oracle.forward(q, k, v, L, blk, nb)
    mask = np.zeros((Lp, Lp), dtype=bool)
    mask[:, :L] = True
    ref = _sdpa(q, k, v, 1.0 / math.sqrt(d), mask)
    np.testing.assert_allclose(out[:, :, :L], ref[:, :, :L], rtol=1e-12, atol=1e-12)
    assert np.all(out[:, :, L:] == 0.0)


def test_attention_k1_is_dense_within_diagonal_block():
    B, H, Lp, blk, d = 1, 1, 64, 16, 8
    q, k, v = (t.numpy() for t in inputs.random_qkv(B, H, Lp, d, seed=5, dtype=torch.float64))
    out, col, _, _ = oracle.forward(q, k, v, Lp, blk, 1)
    for i in range(Lp // blk):
        s = slice(i * blk, (i + 1) * blk)
        ref = _sdpa(q[:, :, s], k[:, :, s], v[:, :, s], 1.0 / math.sqrt(d))
        np.testing.assert_allclose(out[:, :, s], ref, rtol=1e-12, atol=1e-13)


def test_attention_block_indicator_v_pins_the_mask():
    """V[t, c] = 1 if block(t) == c: O[q, c] is the softmax mass on block c, so it is
    0 on dropped blocks, > 0 on kept ones, and sums to 1."""
    B, H, Lp, blk, d, k = 1, 2, 128, 8, 16, 4
    nb = Lp // blk
    q, kk, _ = (t.numpy() for t in inputs.random_qkv(B, H, Lp, d, seed=6, dtype=torch.float64))
    v = np.zeros((B, H, Lp, d))
    for t in range(Lp):
        v[:, :, t, t // blk] = 1.0
    out, col, _, _ = oracle.forward(q, kk, v, Lp, blk, k)
    for h in range(H):
        for t in range(Lp):
            kept = set(col[0, h, t // blk])
            row = out[0, h, t]
            for c in range(nb):
                if c in kept:
                    assert row[c] > 0.0
                else:
                    assert row[c] == 0.0
            assert abs(row.sum() - 1.0) < 1e-13


def test_attention_uniform_when_q_zero():
    """Q = 0: every logit equals, so O is the plain mean of V over the kept valid keys."""
    g = _golden()
    B, H, Lp, blk, d, L, k = 1, 1, 48, 8, 4, 45, 2
    _, kk, v = (t.numpy() for t in inputs.random_qkv(B, H, Lp, d, L=L, seed=8, dtype=torch.float64))
    q = np.zeros_like(kk)
    qm = np.zeros((1, 1, Lp // blk, d))
    km = oracle.pool(kk, L, blk)
    col = oracle.select(qm, km, k)  # all scores 0: diagonal + lowest other index
    rp = oracle.uniform_row_ptr(1, 1, Lp // blk, k)
    out = oracle.attention(q, kk, v, L, blk, rp, col)
    for t in range(L):
        keys = [u for j in col[0, 0, t // blk] for u in range(j * blk, (j + 1) * blk) if u < L]
        np.testing.assert_allclose(out[0, 0, t], v[0, 0, keys].mean(axis=0), rtol=1e-13, atol=1e-14)
    assert g  # golden file present


def test_attention_constant_v():
    B, H, Lp, blk, d = 1, 1, 64, 16, 8
    q, k, _ = (t.numpy() for t in inputs.random_qkv(B, H, Lp, d, seed=9, dtype=torch.float64))
    v = np.broadcast_to(np.arange(d, dtype=np.float64), (B, H, Lp, d)).copy()
    out, _, _, _ = oracle.forward(q, k, v, Lp, blk, 2)
    np.testing.assert_allclose(out, v, rtol=1e-13, atol=1e-13)


def test_attention_invariant_to_key_order_within_block():
    B, H, Lp, blk, d, k = 1, 1, 64, 16, 8, 2
    q, kk, v = (t.numpy() for t in inputs.random_qkv(B, H, Lp, d, seed=10, dtype=torch.float64))
    out1, col1, _, _ = oracle.forward(q, kk, v, Lp, blk, k)
    perm = np.arange(Lp)
    rng = np.random.default_rng(11)
    for i in range(Lp // blk):
        perm[i * blk:(i + 1) * blk] = rng.permutation(np.arange(i * blk, (i + 1) * blk))
    out2, col2, _, _ = oracle.forward(q, kk[:, :, perm], v[:, :, perm], Lp, blk, k)
    np.testing.assert_array_equal(col1, col2)  # block means unchanged by the permutation
    np.testing.assert_allclose(out1, out2, rtol=1e-12, atol=1e-13)


def test_attention_large_logits_need_max_subtraction():
    """Logits of several hundred overflow exp() unless the max is subtracted first."""
    B, H, Lp, blk, d = 1, 1, 32, 8, 8
    q, k, v = (t.numpy() for t in inputs.random_qkv(B, H, Lp, d, seed=12, dtype=torch.float64, q_scale=300.0))
    nb = Lp // blk
    out, _, _, _ = oracle.forward(q, k, v, Lp, blk, nb)
    ref = _sdpa(q, k, v, 1.0 / math.sqrt(d))
    assert np.all(np.isfinite(out))
    np.testing.assert_allclose(out, ref, rtol=1e-10, atol=1e-12)


def test_attention_general_csr_rows():
    """Rows of different lengths, including an empty row (output 0)."""
    B, H, Lp, blk, d = 1, 1, 32, 8, 4
    q, k, v = (t.numpy() for t in inputs.random_qkv(B, H, Lp, d, seed=13, dtype=torch.float64))
    rows = [[0, 3], [], [1, 2, 3], [3]]
    rp = np.cumsum([0] + [len(r) for r in rows]).astype(np.int32)
    ci = np.array([j for r in rows for j in r], dtype=np.int32)
    out = oracle.attention(q, k, v, Lp, blk, rp, ci)
    for i, r in enumerate(rows):
        s = slice(i * blk, (i + 1) * blk)
        if not r:
            assert np.all(out[0, 0, s] == 0.0)
            continue
        keys = np.concatenate([np.arange(j * blk, (j + 1) * blk) for j in r])
        ref = _sdpa(q[:, :, s], k[:, :, keys], v[:, :, keys], 1.0 / math.sqrt(d))
        np.testing.assert_allclose(out[:, :, s], ref, rtol=1e-12, atol=1e-13)


def test_attention_unit_sampling_matches_full():
    B, H, Lp, blk, d, k = 1, 2, 64, 16, 8, 2
    q, kk, v = (t.numpy() for t in inputs.random_qkv(B, H, Lp, d, L=60, seed=14, dtype=torch.float64))
    full, col, _, _ = oracle.forward(q, kk, v, 60, blk, k)
    nb = Lp // blk
    rp = oracle.uniform_row_ptr(B, H, nb, k)
    units = [5, 0, 3, 7]
    part = oracle.attention(q, kk, v, 60, blk, rp, col, units=units)
    for n, u in enumerate(units):
        h, i = divmod(u, nb)
        np.testing.assert_array_equal(part[n], full[0, h, i * blk:(i + 1) * blk])


def test_oracle_accepts_fp32_and_bf16_consistently():
    q, k, v = inputs.random_qkv(1, 1, 64, 8, seed=15, dtype=torch.bfloat16)
    as_f32 = [t.float().numpy() for t in (q, k, v)]
    as_bits = [inputs.bf16_bits(t) for t in (q, k, v)]
    o1, c1, _, _ = oracle.forward(*as_f32, 64, 16, 2)
    o2, c2, _, _ = oracle.forward(*as_bits, 64, 16, 2)
    np.testing.assert_array_equal(c1, c2)
    np.testing.assert_array_equal(o1, o2)


# ---------------------------------------------------------------- step 0: 3D RoPE
# The pages name a fused 3D RoPE kernel (page "知识卡片…", 方法/产品要点, bullet 高效推理算子;
# page "单卡 RTX 5090 跑 Wan2.2-A14B…", 四步拆解 item 4) but give no frequencies; the
# reading (pair split, theta) is stated in sbsa_oracle.c.  These pins fix that reading
# with values worked out by hand and with properties a rotation must have.

def _one_token_grid(d, pos, grid=(4, 4, 8)):
    """x [1,1,Lp,d] with an impulse (1, 0) in every pair of the token at grid position pos."""
    gt, gh, gw = grid
    Lp = gt * gh * gw
    x = np.zeros((1, 1, Lp, d))
    t = (pos[0] * gh + pos[1]) * gw + pos[2]
    x[0, 0, t, 0::2] = 1.0
    return x, t


def test_rope_hand_values_d12():
    # d = 12: 6 pairs, 2 per axis.  theta^(-q/2) at q = 1 is 1/sqrt(10000) = 0.01 exactly,
    # so the column pair q = 1 of a token in column 5 turns by 0.05 rad; q = 0 by 5 rad.
    x, t = _one_token_grid(12, (0, 0, 5))
    r = oracle.rope(x, (4, 4, 8))[0, 0, t]
    cos5, sin5 = 0.28366218546322625, -0.9589242746631385          # cos 5, sin 5
    cos005, sin005 = 0.9987502603949663, 0.04997916927067833      # cos 0.05, sin 0.05
    np.testing.assert_allclose(r[8:10], [cos5, sin5], rtol=0, atol=1e-15)
    np.testing.assert_allclose(r[10:12], [cos005, sin005], rtol=0, atol=1e-15)
    # frame and row pairs: that token is at frame 0, row 0 -> untouched
    np.testing.assert_array_equal(r[0:8], [1, 0, 1, 0, 1, 0, 1, 0])


def test_rope_hand_values_rows_and_frames_d12():
    # frame pairs are the first two, row pairs the next two; q = 0 turns by pos rad
    x, t = _one_token_grid(12, (2, 3, 0))
    r = oracle.rope(x, (4, 4, 8))[0, 0, t]
    np.testing.assert_allclose(r[0:2], [math.cos(2.0), math.sin(2.0)], atol=1e-15)
    np.testing.assert_allclose(r[2:4], [math.cos(0.02), math.sin(0.02)], atol=1e-15)
    np.testing.assert_allclose(r[4:6], [math.cos(3.0), math.sin(3.0)], atol=1e-15)
    np.testing.assert_allclose(r[6:8], [math.cos(0.03), math.sin(0.03)], atol=1e-15)
    np.testing.assert_array_equal(r[8:12], [1, 0, 1, 0])


@pytest.mark.parametrize("d", [64, 128])
def test_rope_axis_split(d):
    # moving a token along one axis changes only that axis' pairs: frame pairs first,
    # then row pairs, then column pairs (d=128: 22 + 21 + 21 pairs; d=64: 12 + 10 + 10)
    pt, ph, pw = oracle.rope_pairs(d)
    assert (pt, ph, pw) == ((22, 21, 21) if d == 128 else (12, 10, 10))
    base = oracle.rope(_one_token_grid(d, (0, 0, 0))[0], (4, 4, 8))[0, 0, 0]
    np.testing.assert_array_equal(base[0::2], 1.0)  # position 0: identity
    for axis, (lo, hi) in enumerate([(0, pt), (pt, pt + ph), (pt + ph, pt + ph + pw)]):
        pos = [0, 0, 0]
        pos[axis] = 1
        x, t = _one_token_grid(d, tuple(pos))
        r = oracle.rope(x, (4, 4, 8))[0, 0, t]
        moved = np.nonzero(np.abs(r[0::2] - 1.0) > 1e-13)[0]
        assert moved.min() == lo and moved.max() == hi - 1


def test_rope_preserves_pair_norms():
    rng = np.random.default_rng(21)
    x = rng.standard_normal((2, 3, 96, 128))
    r = oracle.rope(x, (3, 4, 8))
    n_in = np.hypot(x[..., 0::2], x[..., 1::2])
    n_out = np.hypot(r[..., 0::2], r[..., 1::2])
    np.testing.assert_allclose(n_out, n_in, rtol=1e-13)


def test_rope_dot_product_depends_on_offset_only():
    # <R(m) q, R(n) k> is unchanged when both positions move by the same offset on the
    # grid: rotations that turn with the position make attention translation-invariant
    rng = np.random.default_rng(22)
    d, grid = 64, (4, 4, 8)
    Lp = 4 * 4 * 8
    q = np.zeros((1, 1, Lp, d))
    k = np.zeros((1, 1, Lp, d))
    qv, kv = rng.standard_normal(d), rng.standard_normal(d)

    def t_of(p):
        return (p[0] * 4 + p[1]) * 8 + p[2]

    pairs = [((0, 1, 2), (1, 3, 5)), ((2, 0, 0), (3, 2, 3)), ((1, 1, 1), (2, 3, 4))]
    dots = []
    for a, b in pairs:
        q[:] = 0.0
        k[:] = 0.0
        q[0, 0, t_of(a)] = qv
        k[0, 0, t_of(b)] = kv
        rq, rk = oracle.rope(q, grid)[0, 0, t_of(a)], oracle.rope(k, grid)[0, 0, t_of(b)]
        dots.append(rq @ rk)
    # the three pairs share the offset (1, 2, 3)
    np.testing.assert_allclose(dots, dots[0], rtol=1e-12)
    assert abs(dots[0] - qv @ kv) > 1e-3  # and the rotation is not the identity


def test_rope_pool_means_are_means_of_rounded_outputs():
    x = inputs.random_qkv(1, 2, 64, 12, seed=23, dtype=torch.bfloat16)[0]
    bits, means = oracle.rope_pool(inputs.bf16_bits(x), (2, 4, 8), 60, 16)
    vals = torch.from_numpy(bits.astype(np.int32) << 16).view(torch.float32).double().numpy()
    ref = np.stack([vals[:, :, i * 16:min((i + 1) * 16, 60)].mean(axis=2) for i in range(4)], axis=2)
    np.testing.assert_allclose(means, ref, rtol=1e-13, atol=1e-15)


def test_bf16_rounding_ties_to_even():
    # 1 + 2^-8 is halfway between bf16 1.0 and 1.0078125: to even (1.0); 1 + 3*2^-9 up
    vals = np.array([1.0, 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -9, 1.0 + 3 * 2.0 ** -8, -2.5, 0.0])
    assert [int(b) for b in oracle.bf16_round(vals)] == [0x3F80, 0x3F80, 0x3F81, 0x3F82, 0xC020, 0x0000]


# ---------------------------------------------------------------- FP8 path
# FP8 attention in the style of SageAttention2 (page "知识卡片…", 方法/产品要点, bullet
# 动态稀疏量化注意力; page "单卡 RTX 5090 跑 Wan2.2-A14B…", 四步拆解 item 3).  The reading
# (smoothed K, one scale per block, e4m3 codes) is stated in sbsa_oracle.c.

def test_e4m3_hand_values():
    # e4m3: bias 7, 3 mantissa bits, largest 448 = 1.75 * 2^8, smallest 2^-9
    cases = {448.0: 0x7E, 1.0: 0x38, 0.5: 0x30, 240.0: 0x77, 2.0 ** -6: 0x08, 7 * 2.0 ** -9: 0x07,
             2.0 ** -9: 0x01, -448.0: 0xFE, 0.0: 0x00,
             # halfway cases go to the even mantissa
             1.0625: 0x38, 1.1875: 0x3A, 1.9375: 0x40, 1.5 * 2.0 ** -9: 0x02,
             # beyond the largest finite value: saturate
             500.0: 0x7E, -1e6: 0xFE}
    for v, code in cases.items():
        assert oracle.e4m3_encode(v) == code, (v, hex(oracle.e4m3_encode(v)), hex(code))


def test_e4m3_codes_round_trip():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)  # 0x7F/0xFF: NaN
    vals = oracle.e4m3_decode(codes)
    assert vals.max() == 448.0 and vals.min() == -448.0
    back = np.array([oracle.e4m3_encode(v) for v in vals])
    # +0 and -0 both decode to a zero; everything else comes back to its own code
    nz = codes != 0x80
    np.testing.assert_array_equal(back[nz], codes[nz])
    # the grid: 8 values per binade from 2^-6 on, 2^-9 steps below it
    pos = np.sort(vals[vals > 0])
    assert pos[0] == 2.0 ** -9 and np.allclose(np.diff(pos[:8]), 2.0 ** -9)


def test_quantize_block_scale_and_error_bound():
    rng = np.random.default_rng(31)
    x = rng.standard_normal((1, 2, 96, 16)).astype(np.float32)
    x[0, 1, 40:] *= 1e-3                 # a second block of a different magnitude
    x[:, :, 90:] = 1000.0                # padded tokens hold junk larger than any valid value
    codes, scales = oracle.quantize_fp8(x, 90, 32)
    d = oracle.dequantize_fp8(codes, scales, 32)
    for h in range(2):
        for i in range(3):
            blk = x[0, h, i * 32:min((i + 1) * 32, 90)]
            amax = np.abs(blk).max()
            assert scales[0, h, i] == np.float32(amax) / np.float32(448.0)
            # the largest element lands on +-448 exactly
            c = codes[0, h, i * 32:min((i + 1) * 32, 90)]
            assert np.isin(c, [0x7E, 0xFE]).any()
            # within half a quantum: 2^-4 relative in the normal range, 2^-10 * scale below
            err = np.abs(d[0, h, i * 32:min((i + 1) * 32, 90)] - blk)
            assert np.all(err <= np.maximum(np.abs(blk) * 2.0 ** -4, scales[0, h, i] * 2.0 ** -10) * (1 + 1e-6))
    # padded tokens (t >= 90) are code 0 and do not enter the block's amax
    assert np.all(codes[:, :, 90:] == 0)


def test_smoothing_leaves_attention_unchanged():
    # subtracting one vector from every key adds a per-query constant to the logits
    q, k, v = (t.numpy() for t in inputs.random_qkv(1, 2, 64, 16, L=60, seed=32, dtype=torch.float64))
    mean_k = k[:, :, :60].mean(axis=2, keepdims=True)
    rp = oracle.uniform_row_ptr(1, 2, 4, 2)
    col = oracle.select(oracle.pool(q, 60, 16), oracle.pool(k, 60, 16), 2)
    a = oracle.attention(q, k, v, 60, 16, rp, col)
    b = oracle.attention(q, k - mean_k, v, 60, 16, rp, col)
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)


def test_fp8_attention_is_close_to_exact_attention():
    q, k, v = inputs.random_qkv(1, 2, 128, 64, L=120, seed=33, dtype=torch.bfloat16)
    qb, kb, vb = (inputs.bf16_bits(t) for t in (q, k, v))
    kf = (kb.astype(np.uint32) << 16).view(np.float32)
    smooth = kf[:, :, :120].astype(np.float64).mean(axis=2).astype(np.float32)
    qc, qs = oracle.quantize_fp8(qb, 120, 32)
    kc, ks = oracle.quantize_fp8(kb, 120, 32, smooth)
    rp = oracle.uniform_row_ptr(1, 2, 4, 2)
    col = oracle.select(oracle.pool(qb, 120, 32), oracle.pool(kb, 120, 32), 2)
    exact = oracle.attention(qb, kb, vb, 120, 32, rp, col)
    fp8 = oracle.attention_fp8(qc, qs, kc, ks, vb, 120, 32, rp, col)
    err = np.abs(fp8 - exact)[:, :, :120]
    # logits of d = 64 products of ~N(0,1) values with 2^-4 relative errors per factor
    assert err.max() < 0.1 and err.mean() < 0.01
    assert err.max() > 0  # and the quantization does something


# ---------------------------------------------------------------- NVFP4 (linear layers)

def test_e2m1_hand_values():
    # e2m1: bias 1, one mantissa bit; magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6
    exact = {0.0: 0x0, 0.5: 0x1, 1.0: 0x2, 1.5: 0x3, 2.0: 0x4, 3.0: 0x5, 4.0: 0x6, 6.0: 0x7,
             -0.5: 0x9, -1.5: 0xB, -3.0: 0xD, -6.0: 0xF}
    for v, c in exact.items():
        assert oracle.e2m1_encode(v) == c, v
        assert oracle.e2m1_decode(np.array([c]))[0] == v
    # halfway cases go to the even code (mantissa bit 0)
    ties = {0.25: 0x0, 0.75: 0x2, 1.25: 0x2, 1.75: 0x4, 2.5: 0x4, 3.5: 0x6, 5.0: 0x6, -2.5: 0xC}
    for v, c in ties.items():
        assert oracle.e2m1_encode(v) == c, v
    # nearest, not truncated; beyond 6 saturates
    near = {0.26: 0x1, 1.3: 0x3, 2.6: 0x5, 5.1: 0x7, 6.5: 0x7, 1000.0: 0x7, -7.0: 0xF, 0.2: 0x0}
    for v, c in near.items():
        assert oracle.e2m1_encode(v) == c, v


def test_e2m1_round_trip_and_nearest_by_brute_force():
    codes = np.arange(16)
    vals = oracle.e2m1_decode(codes)
    for c, v in zip(codes, vals):
        if c != 0x8:  # -0 encodes as +0's magnitude with the sign bit
            assert oracle.e2m1_encode(v) == c
    grid = np.unique(vals)
    rng = np.random.default_rng(41)
    for x in rng.uniform(-7, 7, 2000).astype(np.float32):
        got = oracle.e2m1_decode(np.array([oracle.e2m1_encode(x)]))[0]
        best = np.min(np.abs(grid - np.clip(x, -6, 6)))
        assert abs(got - np.clip(x, -6, 6)) == best


def test_nvfp4_sf_layout_hand_offsets():
    K = 256  # 16 blocks per row, 4 atoms of 4 blocks per 128-row group
    # (row, block) -> offset: atom = (row // 128) * (K // 64) + block // 4, then
    # (row % 32) * 16 + ((row % 128) // 32) * 4 + block % 4 inside the 512-byte atom
    cases = {(0, 0): 0, (0, 1): 1, (0, 3): 3, (0, 4): 512, (1, 0): 16, (31, 0): 496, (32, 0): 4,
             (33, 1): 21, (127, 15): 3 * 512 + 31 * 16 + 3 * 4 + 3, (128, 0): 4 * 512, (200, 6): 5 * 512 + 8 * 16 + 2 * 4 + 2}
    for (r, kb), off in cases.items():
        assert oracle.nvfp4_sf_offset(r, kb, K) == off, (r, kb)


def test_nvfp4_nibble_order_and_scales_by_hand():
    # one row, 64 columns; amax 6 -> s = 2688/6 = 448; block 0 amax 6 -> sf = e4m3(448) = 0x7E
    x = np.zeros((1, 64), dtype=np.float32)
    x[0, 0], x[0, 1] = 0.5, 6.0          # codes 1 (low nibble) and 7 (high nibble): byte 0x71
    x[0, 2], x[0, 3] = -1.0, 0.0         # codes 0xA and 0: byte 0x0A
    x[0, 16] = 3.0                       # block 1: amax 3 -> sf = e4m3(0.5 * 448 = 224) = 0x76, code(6) = 7
    codes, sf, s = oracle.nvfp4_quantize(x)
    assert s == np.float32(448.0)
    assert codes[0, 0] == 0x71 and codes[0, 1] == 0x0A and codes[0, 8] == 0x07
    assert sf[0] == 0x7E and sf[1] == 0x76 and sf[2] == 0 and sf[3] == 0
    # rows beyond the matrix (padding up to 128) have scale 0
    assert np.all(sf[16:] == 0) and sf.size == 128 * 4


def test_nvfp4_exactly_representable_inputs_round_trip():
    # x = (e2m1 value) * 2^j with every block holding a +-6 * 2^j: all scales are exact
    rng = np.random.default_rng(42)
    rows, K = 130, 128
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], dtype=np.float64)
    mag = rng.choice(grid, size=(rows, K)) * rng.choice([-1, 1], size=(rows, K))
    j = rng.integers(-6, 3, size=(rows, K // 16))
    j[0, 0] = 3  # the block holding the tensor amax 6 * 2^3
    mag.reshape(rows, K // 16, 16)[:, :, 5] = 6.0
    x = (mag.reshape(rows, K // 16, 16) * np.exp2(j)[:, :, None]).reshape(rows, K)
    codes, sf, s = oracle.nvfp4_quantize(x.astype(np.float32))
    np.testing.assert_array_equal(oracle.nvfp4_dequantize(codes, sf, s), x)


def test_nvfp4_block_scale_and_error_bound():
    rng = np.random.default_rng(43)
    x = rng.standard_normal((40, 192)).astype(np.float32)
    x[3, 16:32] *= 1e-3                    # a block far below the others
    codes, sf, s = oracle.nvfp4_quantize(x)
    amax = np.abs(x).max()
    assert s == np.float32(2688.0) / np.float32(amax)
    d = oracle.nvfp4_dequantize(codes, sf, s)
    for r in range(40):
        for kb in range(192 // 16):
            blk = x[r, kb * 16:(kb + 1) * 16].astype(np.float64)
            sfv = oracle.e4m3_decode(np.array([sf[oracle.nvfp4_sf_offset(r, kb, 192)]]))[0]
            step = sfv / s  # the value of one e2m1 unit in this block
            # the block scale is the e4m3 rounding of (block amax / 6) * s: within 2^-4
            target = float(np.float32(np.float32(np.abs(blk).max()) / np.float32(6.0)) * np.float32(s))
            assert abs(sfv - target) <= target * 2.0 ** -4
            # every element is the nearest of the block's 15 grid values (of x clipped to +-6 steps)
            grid = np.unique(np.concatenate([oracle.e2m1_decode(np.arange(16))])) * step
            got = d[r, kb * 16:(kb + 1) * 16]
            for xv, gv in zip(blk, got):
                assert abs(gv - np.clip(xv, grid[0], grid[-1])) <= np.min(np.abs(grid - xv)) * (1 + 1e-6) + 1e-300


def test_nvfp4_gemm_exact_and_closed_forms():
    rng = np.random.default_rng(44)
    M, N, K = 96, 160, 128             # non-square: a transposed operand cannot pass
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], dtype=np.float64)

    def exact(rows):
        v = rng.choice(grid, size=(rows, K)) * rng.choice([-1, 1], size=(rows, K))
        v.reshape(rows, K // 16, 16)[:, :, 0] = 6.0
        return (v.reshape(rows, K // 16, 16) * np.exp2(rng.integers(-3, 2, size=(rows, K // 16)))[:, :, None]
                ).reshape(rows, K)

    a, b = exact(M), exact(N)
    bias = rng.standard_normal(N)
    qa, qb = oracle.nvfp4_quantize(a.astype(np.float32)), oracle.nvfp4_quantize(b.astype(np.float32))
    c = oracle.nvfp4_gemm(*qa, *qb, bias)
    np.testing.assert_array_equal(c, a @ b.T + bias[None, :])
    # A = 0: every row of C is the bias (a column vector of C per n)
    z = oracle.nvfp4_quantize(np.zeros((M, K), dtype=np.float32))
    np.testing.assert_array_equal(oracle.nvfp4_gemm(*z, *qb, bias), np.broadcast_to(bias, (M, N)))
    # one-hot rows of A pick columns of B_dec
    e = np.zeros((4, K), dtype=np.float32)
    e[np.arange(4), [0, 17, 64, 127]] = 6.0
    qe = oracle.nvfp4_quantize(e)
    bd = oracle.nvfp4_dequantize(*qb)
    np.testing.assert_array_equal(oracle.nvfp4_gemm(*qe, *qb), 6.0 * bd[:, [0, 17, 64, 127]].T)


def test_nvfp4_gemm_close_to_unquantized():
    rng = np.random.default_rng(45)
    a = rng.standard_normal((64, 256)).astype(np.float32)
    b = rng.standard_normal((128, 256)).astype(np.float32)
    c = oracle.nvfp4_gemm(*oracle.nvfp4_quantize(a), *oracle.nvfp4_quantize(b))
    ref = a.astype(np.float64) @ b.T.astype(np.float64)
    rel = np.linalg.norm(c - ref) / np.linalg.norm(ref)
    # per-element relative error of e2m1 with block scales is ~ 1/12 rms; two operands
    assert 0.02 < rel < 0.2, rel


# ---------------------------------------------------------------- Light-Ulysses exchange

def _bits_of(x):
    return (np.asarray(x, dtype=np.float32).view(np.uint32) >> 16).astype(np.uint16)


def test_row_quantizer_scale_and_round_trip():
    rng = np.random.default_rng(51)
    rows = rng.standard_normal((33, 64)).astype(np.float32)
    rows[4] = 0.0
    codes, scales = oracle.quantize_rows_fp8(rows)
    amax = np.abs(rows).max(axis=1)
    np.testing.assert_array_equal(scales[amax > 0], (amax / np.float32(448.0)).astype(np.float32)[amax > 0])
    assert scales[4] == 1.0 and np.all(codes[4] == 0)
    # every row's largest element lands on +-448
    assert np.all(np.isin(codes[amax > 0], [0x7E, 0xFE]).any(axis=1))
    back = (oracle.dequantize_rows_bf16(codes, scales).astype(np.uint32) << 16).view(np.float32)
    err = np.abs(back.astype(np.float64) - rows)
    # e4m3 half-quantum (2^-4 relative, 2^-10 * scale below the normal range) + one bf16 rounding
    bound = np.maximum(np.abs(rows) * 2.0 ** -4, scales[:, None] * 2.0 ** -10) * (1 + 2.0 ** -7) + np.abs(rows) * 2.0 ** -8
    assert np.all(err <= bound)


def test_ulysses_exchange_by_hand():
    # G = 2 ranks, H = 2 heads, L = 4 tokens (2 per rank), d = 2; values exact in e4m3 and bf16:
    # x[t, c, h, :] = [448 * s, 56 * s] with s = 2^-(t + c + h) (one row, one scale each)
    G, H, L, d = 2, 2, 4, 2
    x = np.zeros((L, 3, H, d), dtype=np.float32)
    for t in range(L):
        for c in range(3):
            for h in range(H):
                s = 2.0 ** -(t + c + h)
                x[t, c, h] = [448.0 * s, -56.0 * s]
    shards = [_bits_of(x[0:2]), _bits_of(x[2:4])]
    out = oracle.ulysses_qkv(shards, H, L, Lp=6)
    for r in range(G):
        got = (out[r].astype(np.uint32) << 16).view(np.float32)
        assert got.shape == (3, 1, 6, d)
        # rank r holds head r of all four tokens, padded tokens 4 and 5 zero
        for c in range(3):
            for t in range(L):
                np.testing.assert_array_equal(got[c, 0, t], x[t, c, r])
            assert np.all(got[c, 0, 4:] == 0)
    # the return exchange puts every head of a rank's own tokens back
    o_shards = [out[r][0, :, :, :] for r in range(G)]  # the q rows of each rank's head, as "attention output"
    back = oracle.ulysses_o(o_shards, H, L)
    for r in range(G):
        got = (back[r].astype(np.uint32) << 16).view(np.float32)
        np.testing.assert_array_equal(got, x[2 * r:2 * r + 2, 0, :, :])
