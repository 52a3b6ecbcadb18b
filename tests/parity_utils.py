"""Helpers shared by the GPU parity tests: run the CUDA path through the C ABI and
compare with the CPU oracle under the tolerances the method's target states:

  * block indices: equal to the oracle's, except that blocks whose oracle score lies
    within 1e-5 (relative) of the oracle's k-th score may be swapped.  "Relative" is
    taken against max(|s_k|, sum_c |qmean_ic * kmean_jc|), the second term being the
    magnitude that bounds the rounding error of a dot product whose value is near 0;
  * attention output (bf16, fp32 accumulation) given the oracle's mask: max-abs error
    <= 2e-2 and mean-abs error <= 2e-3 against the fp64 oracle;
  * block means (fp32 accumulation of bf16 values, one rounding per add): within
    rtol 1e-5 / atol 1e-6 of the fp64 oracle.
"""
from __future__ import annotations

import os

import numpy as np
import torch

import oracle
from video_dit_dynamic_b200 import inputs, sbsa

MAX_ABS = 2e-2
MEAN_ABS = 2e-3
TIE_REL = 1e-5

oracle.set_threads(os.cpu_count() or 1)


def require_cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    sbsa.load()


def shape_of(q: torch.Tensor, L: int, blk: int) -> sbsa.Shape:
    B, H, Lp, d = q.shape
    return sbsa.make_shape(B, H, L, d, blk, Lp)


def gpu_pool(shape, q, k):
    rows = shape.batch * shape.heads * shape.num_blocks
    qm = torch.empty(rows * shape.head_dim, dtype=torch.float32, device="cuda")
    km = torch.empty_like(qm)
    sbsa.sbsa_pool_qk(shape, q, k, qm, km)
    return qm.view(shape.batch, shape.heads, shape.num_blocks, shape.head_dim), \
        km.view(shape.batch, shape.heads, shape.num_blocks, shape.head_dim)


def gpu_select(shape, qm, km, k_keep):
    rows = shape.batch * shape.heads * shape.num_blocks
    rp = torch.empty(rows + 1, dtype=torch.int32, device="cuda")
    ci = torch.empty(rows * k_keep, dtype=torch.int32, device="cuda")
    sbsa.sbsa_select_blocks(shape, qm.contiguous(), km.contiguous(), k_keep, rp, ci)
    return rp, ci


def gpu_attention(shape, q, k, v, rp, ci, scale=0.0):
    o = torch.empty_like(q)
    sbsa.sbsa_attention_fwd(shape, q, k, v, rp, ci, scale, o)
    return o


def assert_means_close(gpu, ref):
    np.testing.assert_allclose(gpu.detach().cpu().double().numpy(), ref, rtol=1e-5, atol=1e-6)


def assert_selection_ok(gpu_col: np.ndarray, ora_col: np.ndarray, qmean: np.ndarray, kmean: np.ndarray, k: int,
                        rows=None, stats=None):
    """gpu_col / ora_col: [B,H,nb,k]; qmean/kmean: [B,H,nb,d] float64 (the oracle's).
    Returns the number of rows that differ only by tolerated tie swaps.  If `stats` is a
    dict it receives "swaps" (that count) and "wide_swaps": the rows among them where a
    swapped block's score is further than TIE_REL * |s_k| from the k-th score, i.e. rows
    accepted only through the sum-of-magnitudes term of the bound."""
    B, H, nb, _ = qmean.shape
    g = gpu_col.reshape(B * H, nb, k)
    o = ora_col.reshape(B * H, nb, k)
    # structure: strictly ascending, in range, diagonal present -- every row
    assert np.all(g >= 0) and np.all(g < nb)
    if k > 1:
        assert np.all(np.diff(g, axis=-1) > 0), "GPU block lists must be strictly ascending"
    diag = np.arange(nb)[None, :, None]
    assert np.all(np.any(g == diag, axis=-1)), "diagonal block missing"
    differ = np.nonzero(np.any(g != o, axis=-1))
    qm = qmean.reshape(B * H, nb, -1)
    km = kmean.reshape(B * H, nb, -1)
    swaps = wide = 0
    for bh, i in zip(*differ):
        if rows is not None and (bh, i) not in rows:
            continue
        G, O = set(g[bh, i].tolist()), set(o[bh, i].tolist())
        s = km[bh] @ qm[bh, i]
        a = np.abs(km[bh]) @ np.abs(qm[bh, i])
        sk = min(s[j] for j in O if j != i)
        is_wide = False
        for j in G ^ O:
            bound = TIE_REL * max(abs(sk), a[j])
            assert abs(s[j] - sk) <= bound, (
                f"row (bh={bh}, i={i}): block {j} score {s[j]!r} vs k-th {sk!r} differs by more than the tie bound")
            is_wide |= abs(s[j] - sk) > TIE_REL * abs(sk)
        swaps += 1
        wide += int(is_wide)
    if stats is not None:
        stats["swaps"] = swaps
        stats["wide_swaps"] = wide
    return swaps


def assert_attention_close(gpu_o: torch.Tensor, ref: np.ndarray, what=""):
    g = gpu_o.detach().float().cpu().double().numpy()
    err = np.abs(g - ref)
    mx, mean = float(err.max()), float(err.mean())
    assert np.all(np.isfinite(g)), f"{what}: non-finite output"
    assert mx <= MAX_ABS, f"{what}: max-abs error {mx:.3e} > {MAX_ABS}"
    assert mean <= MEAN_ABS, f"{what}: mean-abs error {mean:.3e} > {MEAN_ABS}"
    return mx, mean


def bits(t: torch.Tensor) -> np.ndarray:
    return inputs.bf16_bits(t)
