"""GPU parity of the fused 3D RoPE + block-mean kernel against the oracle.

The kernel rotates in fp32 with an fp32 cos/sin table and rounds to bf16; the oracle
rotates in fp64 and rounds once.  Where the two land on different sides of a bf16
rounding boundary they differ by one bf16 step (at most 2^-7 relative), and where the two
products of x cos - y sin cancel, the fp32 evaluation error (a few 2^-24 of the pair's
norm) can exceed that step; the rotated tensors must agree within those bounds
everywhere and exactly almost everywhere.  The block means are checked against the
means of the kernel's own rounded values and, loosely, against the oracle's.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from tests import parity_utils as pu
from video_dit_dynamic_b200 import inputs

pytestmark = pytest.mark.gpu


def _sbsa():
    from video_dit_dynamic_b200 import sbsa
    sbsa.load()
    return sbsa


def _bf16_from_bits(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _run(d, blk, grid, B, H, seed, in_place=False, theta=10000.0):
    sbsa = _sbsa()
    L = grid[0] * grid[1] * grid[2]
    Lp = (L + blk - 1) // blk * blk
    g = torch.Generator(device="cpu").manual_seed(seed)
    q = torch.randn(B, H, Lp, d, generator=g).to(torch.bfloat16).cuda()
    k = torch.randn(B, H, Lp, d, generator=g).to(torch.bfloat16).cuda()
    s = sbsa.make_shape(B, H, L, d, blk)
    nb = Lp // blk
    table = torch.empty(sbsa.sbsa_rope_table_floats(d, grid), dtype=torch.float32, device="cuda")
    sbsa.sbsa_rope_table_init(d, grid, theta, table)
    qi, ki = q.clone(), k.clone()
    qo, ko = (q, k) if in_place else (torch.empty_like(q), torch.empty_like(k))
    qm = torch.empty(B * H * nb * d, dtype=torch.float32, device="cuda")
    km = torch.empty_like(qm)
    sbsa.sbsa_rope_pool_qk(s, grid, table, q, k, qo, ko, qm, km)
    sbsa.sbsa_check()
    return qi, ki, qo, ko, qm.view(B, H, nb, d), km.view(B, H, nb, d), table, L


def _check_tensor(x_in, x_out, means, grid, L, blk, theta=10000.0):
    bits_in = inputs.bf16_bits(x_in.cpu())
    got = inputs.bf16_bits(x_out.cpu())
    ref_bits, ref_means = oracle.rope_pool(bits_in, grid, L, blk, theta)
    g, r = _bf16_from_bits(got), _bf16_from_bits(ref_bits)
    # One bf16 step of the result, plus the fp32 evaluation error of x cos - y sin with an
    # fp32 table (a few 2^-24 of the pair's norm: it dominates only where the two
    # products cancel and the result is small); and rarely any difference at all.
    x = _bf16_from_bits(bits_in)
    pair_norm = np.repeat(np.hypot(x[..., 0::2], x[..., 1::2]), 2, axis=-1)
    diff = np.abs(g - r)
    # one bf16 step is 2^(e-7) for a value in [2^e, 2^(e+1)), at most 2^-7 of the value
    bound = np.maximum(np.abs(r), np.abs(g)) * 2.0 ** -7 + pair_norm * 2.0 ** -21
    assert np.all(diff <= bound), f"worst excess {np.max(diff - bound):.3e}"
    frac = np.mean(got != ref_bits)
    assert frac < 0.01, f"{frac:.4f} of the elements differ by one bf16 step"
    # padded tokens pass through bit for bit
    np.testing.assert_array_equal(got[:, :, L:], bits_in[:, :, L:])
    # means of the kernel's own rounded values, and against the oracle's
    own = oracle.pool(got, L, blk)
    np.testing.assert_allclose(means.cpu().double().numpy(), own, rtol=2e-6, atol=1e-6)
    np.testing.assert_allclose(means.cpu().double().numpy(), ref_means, rtol=0, atol=2e-3)
    return frac


@pytest.mark.parametrize("d,blk,grid,B,H", [(128, 128, (3, 5, 7), 1, 2), (64, 64, (2, 6, 11), 2, 2),
                                           (128, 64, (4, 4, 8), 1, 3), (64, 128, (1, 1, 300), 1, 2),
                                           (128, 128, (21, 30, 52), 1, 1)])
def test_rope_pool_matches_oracle(d, blk, grid, B, H):
    qi, ki, qo, ko, qm, km, _, L = _run(d, blk, grid, B, H, seed=d + blk + grid[2])
    _check_tensor(qi, qo, qm, grid, L, blk)
    _check_tensor(ki, ko, km, grid, L, blk)


def test_rope_pool_in_place_matches_out_of_place():
    args = (128, 128, (3, 8, 9), 1, 2)
    _, _, qo, ko, qm, km, _, _ = _run(*args, seed=3)
    _, _, qi, ki, qm2, km2, _, _ = _run(*args, seed=3, in_place=True)
    assert torch.equal(qo, qi) and torch.equal(ko, ki)
    assert torch.equal(qm, qm2) and torch.equal(km, km2)


def test_rope_table_values():
    sbsa = _sbsa()
    d, grid = 128, (5, 7, 9)
    table = torch.empty(sbsa.sbsa_rope_table_floats(d, grid), dtype=torch.float32, device="cuda")
    sbsa.sbsa_rope_table_init(d, grid, 10000.0, table)
    tab = table.cpu().numpy().reshape(-1, 2).astype(np.float64)
    pt, ph, pw = oracle.rope_pairs(d)
    ref = []
    for n_pos, P in ((grid[0], pt), (grid[1], ph), (grid[2], pw)):
        for pos in range(n_pos):
            for q in range(P):
                a = pos * 10000.0 ** (-q / P)
                ref.append((math.cos(a), math.sin(a)))
    # fp32 rounding of the double values: half an fp32 step
    np.testing.assert_allclose(tab, np.array(ref), rtol=0, atol=2.0 ** -24)


def test_rotated_means_feed_select():
    """rope_pool -> select on the rotated means (the order a DiT layer uses)."""
    sbsa = _sbsa()
    d, blk, grid, H = 128, 128, (4, 8, 16), 2
    qi, ki, qo, ko, qm, km, _, L = _run(d, blk, grid, 1, H, seed=9)
    s = sbsa.make_shape(1, H, L, d, blk)
    nb = qm.shape[2]
    kk = sbsa.sbsa_keep_blocks(nb, 0.5)
    rp, ci = pu.gpu_select(s, qm.reshape(-1), km.reshape(-1), kk)
    qn, kn = qm.double().cpu().numpy(), km.double().cpu().numpy()
    pu.assert_selection_ok(ci.cpu().numpy().reshape(1, H, nb, kk), oracle.select(qn, kn, kk), qn, kn, kk)
