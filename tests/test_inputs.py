"""The synthetic input recipe, on the CPU: shapes and padding, seeding, the positional
signal that correlates Q with K (and not with V), and the workload sizes."""
import math

import numpy as np
import torch

from video_dit_dynamic_b200 import inputs


def _small(kind="positional", keep=0.25):
    # a 3 x 4 x 11 grid = 132 tokens, padded to 192 with blocks of 64
    return inputs.Workload("t", 2, 3, (3, 4, 11), 64, 64, keep, kind=kind)


def test_shapes_dtype_and_zero_padding():
    wl = _small()
    assert (wl.seq_len, wl.seq_len_padded, wl.num_blocks) == (132, 192, 3)
    q, k, v = inputs.make_qkv(wl, seed=4)
    for t in (q, k, v):
        assert t.shape == (2, 3, 192, 64) and t.dtype == torch.bfloat16
        assert torch.all(t[:, :, 132:] == 0) and torch.any(t[:, :, :132] != 0)
    qn, _, _ = inputs.make_qkv(_small(kind="normal"), seed=4)
    assert torch.all(qn[:, :, 132:] == 0)


def test_seeding():
    wl = _small()
    a = inputs.make_qkv(wl, seed=1)
    b = inputs.make_qkv(wl, seed=1)
    c = inputs.make_qkv(wl, seed=2)
    assert all(torch.equal(x, y) for x, y in zip(a, b))
    assert not any(torch.equal(x, y) for x, y in zip(a, c))
    # Q, K and V draw independent noise; the heads and batch entries differ
    q, k, v = a
    assert not torch.equal(q, k) and not torch.equal(q[0, 0], q[0, 1]) and not torch.equal(q[0], q[1])


def test_positional_features_follow_the_grid():
    T, Hg, W = 3, 4, 11
    f = inputs.positional_features((T, Hg, W)).double()
    assert f.shape == (T * Hg * W, 6)
    assert torch.allclose(f[0], torch.tensor([0.0, 1.0, 0.0, 1.0, 0.0, 1.0], dtype=torch.float64), atol=1e-7)
    # token index = (t * Hg + h) * W + w, each axis a full period over its extent
    t, h, w = 2, 3, 5
    idx = (t * Hg + h) * W + w
    want = [math.sin(2 * math.pi * t / T), math.cos(2 * math.pi * t / T), math.sin(2 * math.pi * h / Hg),
            math.cos(2 * math.pi * h / Hg), math.sin(2 * math.pi * w / W), math.cos(2 * math.pi * w / W)]
    assert torch.allclose(f[idx], torch.tensor(want, dtype=torch.float64), atol=1e-6)
    assert torch.allclose(f[:, 0::2] ** 2 + f[:, 1::2] ** 2, torch.ones(T * Hg * W, 3, dtype=torch.float64), atol=1e-6)


def test_q_and_k_share_the_positional_signal():
    """The block-mean scores q_i . k_j carry the grid structure the selection ranks by: a
    block scores itself among the highest of its row; V carries none of it, and neither
    do kind="normal" inputs (there the diagonal ranks mid-row, as chance would)."""
    def diag_rank(kind, other):
        wl = inputs.Workload("c", 1, 2, (8, 16, 16), 128, 64, 0.25, kind=kind)  # 2,048 tokens, 32 blocks
        q, k, v = inputs.make_qkv(wl, seed=0)
        m = [t[0].double().view(2, wl.num_blocks, 64, 128).mean(dim=2) for t in (q, k, v)]
        s = m[0] @ m[1 if other == "k" else 2].transpose(1, 2)
        diag = torch.diagonal(s, dim1=1, dim2=2)
        return float((s > diag.unsqueeze(-1)).sum(-1).double().mean())  # higher-scoring blocks per row

    assert diag_rank("positional", "k") < 6
    assert diag_rank("positional", "v") > 10
    assert diag_rank("normal", "k") > 10


def test_workload_sizes():
    w = inputs.WORKLOADS
    assert (w["tiny"].seq_len, w["tiny"].num_blocks) == (1024, 16)
    assert (w["480p"].seq_len, w["480p"].seq_len_padded, w["480p"].num_blocks) == (32760, 32768, 256)
    assert (w["720p"].seq_len, w["720p"].seq_len_padded, w["720p"].num_blocks) == (75600, 75648, 591)
    assert (w["long122880"].seq_len, w["long122880"].num_blocks) == (122880, 960)
    s = inputs.sweep_workload(0.3)
    assert (s.seq_len, s.num_blocks, s.keep, s.heads) == (32768, 256, 0.3, 40)


def test_bf16_bits_round_trip():
    x = torch.tensor([1.0, -2.5, 0.0, 3.140625], dtype=torch.bfloat16)
    bits = inputs.bf16_bits(x)
    assert bits.dtype == np.uint16
    assert list(bits) == [0x3F80, 0xC020, 0x0000, 0x4049]
