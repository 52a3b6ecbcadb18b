"""Block 64: one CTA takes two neighbouring query blocks as the halves of its 128-row tile.

The kernel walks the union of the two kept lists when both are strictly ascending, in
range and at most 256 long (a block kept by both computed once for all 128 rows), and
otherwise list a then list b.  Every case is compared with the oracle given the same
lists: sorted lists that overlap in part, fully or not at all (the union walk), lists
with repeats and in any order, one list over the cap, an odd number of blocks (the last
tile has no second block), and a row pair where one list is empty.
"""
import numpy as np
import pytest
import torch

import oracle
from tests import parity_utils as pu
from video_dit_dynamic_b200 import inputs, sbsa

pytestmark = pytest.mark.gpu


def _run(d, nb, rows, L=None, H=1, seed=41):
    blk = 64
    Lp = nb * blk
    L = Lp - 5 if L is None else L
    q, k, v = inputs.random_qkv(1, H, Lp, d, L=L, seed=seed, device="cuda")
    rp = np.cumsum([0] + [len(x) for x in rows]).astype(np.int32)
    ci = np.array([j for x in rows for j in x], dtype=np.int32)
    s = pu.shape_of(q, L, blk)
    o = pu.gpu_attention(s, q, k, v, torch.from_numpy(rp).cuda(),
                         torch.from_numpy(ci if ci.size else np.zeros(1, np.int32)).cuda())
    sbsa.sbsa_check()
    ref = oracle.attention(pu.bits(q), pu.bits(k), pu.bits(v), L, blk, rp, ci)
    return o, ref


@pytest.mark.parametrize("d", [128, 64])
def test_union_walk_partial_full_and_no_overlap(d):
    pu.require_cuda()
    nb = 12
    rng = np.random.default_rng(42)
    rows = []
    for i in range(0, nb, 2):
        a = sorted(rng.choice(nb, size=5, replace=False).tolist())
        kind = (i // 2) % 3
        if kind == 0:    # partial overlap
            b = sorted(set(a[:2]) | set(rng.choice(nb, size=3, replace=False).tolist()))
        elif kind == 1:  # the same list
            b = list(a)
        else:            # disjoint
            b = sorted(rng.choice([j for j in range(nb) if j not in a], size=4, replace=False).tolist())
        rows += [a, b]
    o, ref = _run(d, nb, rows)
    pu.assert_attention_close(o, ref, "union walk")


def test_repeats_and_any_order_walk_both_lists():
    pu.require_cuda()
    nb = 10
    rng = np.random.default_rng(43)
    rows = []
    for i in range(nb):
        x = rng.integers(0, nb, size=int(rng.integers(1, 8))).tolist()  # repeats, any order
        rows.append(x)
    rows[4] = sorted(set(rows[4]))  # a sorted list paired with an unsorted one
    o, ref = _run(128, nb, rows)
    pu.assert_attention_close(o, ref, "repeats, any order")


def test_list_over_the_union_cap():
    pu.require_cuda()
    nb = 300  # lists of 300 entries: past the 256 the union walk holds
    rows = []
    rng = np.random.default_rng(44)
    for i in range(nb):
        if i in (0, 1):
            rows.append(list(range(nb)))
        else:
            rows.append(sorted(rng.choice(nb, size=3, replace=False).tolist()))
    o, ref = _run(64, nb, rows)
    pu.assert_attention_close(o, ref, "over the cap")


def test_odd_block_count_and_empty_half():
    pu.require_cuda()
    nb = 9  # the last tile has only block 8
    L = nb * 64 - 11
    rng = np.random.default_rng(45)
    rows = [sorted(rng.choice(nb, size=3, replace=False).tolist()) for _ in range(2 * nb)]  # two heads
    rows[2] = []          # head 0, block 2 empty, its partner block 3 not
    rows[nb + 5] = []     # head 1, block 5 empty, its partner block 4 not
    o, ref = _run(128, nb, rows, L=L, H=2)
    pu.assert_attention_close(o, ref, "odd count, empty half")
    for h, i in ((0, 2), (1, 5)):
        assert torch.all(o[0, h, i * 64:(i + 1) * 64] == 0)
    assert torch.all(o[0, :, L:] == 0)
