"""The GPU parity checkers themselves, on the CPU: they must accept exactly what the
tolerances allow and reject the rest (a checker that accepts everything would make every
GPU parity result meaningless)."""
import numpy as np
import pytest
import torch

from tests import parity_utils as pu


def _means():
    # one (b, h), four blocks, d = 2; query block 0 scores key blocks 1 and 2 equally
    qm = np.array([[1.0, 0.0], [0.0, 1.0], [1.0, 1.0], [0.5, -1.0]])[None, None]
    km = np.array([[2.0, 0.0], [1.0, 5.0], [1.0, -3.0], [0.25, 0.0]])[None, None]
    return qm, km


def _oracle_cols(qm, km, k):
    nb = qm.shape[2]
    out = np.empty((1, 1, nb, k), dtype=np.int32)
    for i in range(nb):
        s = km[0, 0] @ qm[0, 0, i]
        others = sorted((j for j in range(nb) if j != i), key=lambda j: (-s[j], j))
        out[0, 0, i] = sorted([i] + others[:k - 1])
    return out


def test_selection_identical_and_tie_swap_accepted():
    qm, km = _means()
    ora = _oracle_cols(qm, km, 2)
    assert pu.assert_selection_ok(ora.copy(), ora, qm, km, 2) == 0
    # row 0: blocks 1 and 2 both score 1.0; the oracle keeps 1 (lower index), taking 2 is a tie swap
    assert list(ora[0, 0, 0]) == [0, 1]
    gpu = ora.copy()
    gpu[0, 0, 0] = [0, 2]
    assert pu.assert_selection_ok(gpu, ora, qm, km, 2) == 1


def test_selection_counts_swaps_that_need_the_magnitude_term():
    # row 0: block 2 scores 1.001 and block 1 scores 1.0, each the sum of two large terms of
    # opposite sign (sum of magnitudes about 2000); taking block 1 instead of 2 is 1e-3 away
    # from the k-th score: beyond 1e-5 * |s_k| but within 1e-5 * 2000
    qm = np.array([[1.0, 1.0], [0.0, 1.0], [1.0, 0.0], [0.5, 0.5]])[None, None]
    km = np.array([[0.0, 0.0], [1000.0, -999.0], [1000.0, -998.999], [0.0, 0.0]])[None, None]
    ora = _oracle_cols(qm, km, 2)
    assert list(ora[0, 0, 0]) == [0, 2]
    gpu = ora.copy()
    gpu[0, 0, 0] = [0, 1]
    st = {}
    assert pu.assert_selection_ok(gpu, ora, qm, km, 2, stats=st) == 1
    assert st == {"swaps": 1, "wide_swaps": 1}
    # an exact tie swap is not a wide one
    qm2, km2 = _means()
    ora2 = _oracle_cols(qm2, km2, 2)
    gpu2 = ora2.copy()
    gpu2[0, 0, 0] = [0, 2]
    st2 = {}
    pu.assert_selection_ok(gpu2, ora2, qm2, km2, 2, stats=st2)
    assert st2 == {"swaps": 1, "wide_swaps": 0}


def test_selection_rejects_real_differences():
    qm, km = _means()
    ora = _oracle_cols(qm, km, 2)
    bad = ora.copy()
    bad[0, 0, 0] = [0, 3]  # block 3 scores 0.25, far from the k-th score 1.0
    with pytest.raises(AssertionError):
        pu.assert_selection_ok(bad, ora, qm, km, 2)
    no_diag = ora.copy()
    no_diag[0, 0, 1] = [0, 2]
    with pytest.raises(AssertionError):
        pu.assert_selection_ok(no_diag, ora, qm, km, 2)
    unsorted = ora.copy()
    unsorted[0, 0, 0] = [1, 0]
    with pytest.raises(AssertionError):
        pu.assert_selection_ok(unsorted, ora, qm, km, 2)
    out_of_range = ora.copy()
    out_of_range[0, 0, 3] = [3, 4]
    with pytest.raises(AssertionError):
        pu.assert_selection_ok(out_of_range, ora, qm, km, 2)


def test_attention_tolerance_bounds():
    ref = np.random.default_rng(0).standard_normal((2, 3, 64, 8))
    exact = torch.from_numpy(ref)
    pu.assert_attention_close(exact, ref)
    one_big = exact.clone()
    one_big[0, 0, 0, 0] += 0.03  # max-abs 3e-2 > 2e-2
    with pytest.raises(AssertionError):
        pu.assert_attention_close(one_big, ref)
    shifted = exact + 3e-3  # every element within the max bound, the mean beyond 2e-3
    with pytest.raises(AssertionError):
        pu.assert_attention_close(shifted, ref)
    within = exact + 1.5e-3
    pu.assert_attention_close(within, ref)
    nan = exact.clone()
    nan[1, 2, 3, 4] = float("nan")
    with pytest.raises(AssertionError):
        pu.assert_attention_close(nan, ref)


def test_mean_tolerance_bounds():
    ref = np.random.default_rng(1).standard_normal((1, 2, 4, 8))
    pu.assert_means_close(torch.from_numpy(ref * (1 + 1e-7)), ref)
    with pytest.raises(AssertionError):
        pu.assert_means_close(torch.from_numpy(ref * (1 + 1e-4)), ref)


def test_nvfp4_gemm_bound():
    """One bf16 rounding of the exact product is accepted; an error of a few bf16 steps is
    not (a dropped or doubled K-block, a wrong scale, would be far larger)."""
    from tests.test_gpu_nvfp4 import _check_gemm
    rng = np.random.default_rng(2)
    a = rng.standard_normal((32, 64))
    b = rng.standard_normal((48, 64))
    ref = a @ b.T
    rounded = torch.from_numpy(ref).to(torch.bfloat16)  # the kernel's output rounding
    assert _check_gemm(rounded, ref, a, b) <= 1.0
    off = torch.from_numpy(ref * (1 + 2.0 ** -5)).to(torch.bfloat16)
    with pytest.raises(AssertionError):
        _check_gemm(off, ref, a, b)
    dropped = torch.from_numpy(a[:, :48] @ b[:, :48].T).to(torch.bfloat16)  # one quarter of K missing
    with pytest.raises(AssertionError):
        _check_gemm(dropped, ref, a, b)


def test_rope_checker():
    """The oracle's own rotation passes; two bf16 steps on one element, one step on 2% of
    the elements, swapped pair members, or a touched padded token do not."""
    import oracle
    from tests.test_gpu_rope import _check_tensor
    from video_dit_dynamic_b200 import inputs
    grid, L, blk = (2, 3, 9), 54, 32
    g = torch.Generator().manual_seed(3)
    x = torch.randn(1, 2, 64, 32, generator=g)
    x[:, :, L:] = 0.5  # padded tokens: passed through
    x = x.to(torch.bfloat16)
    ref_bits, _ = oracle.rope_pool(inputs.bf16_bits(x), grid, L, blk)

    def as_t(bits):
        return torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16)

    def run(bits):
        means = torch.from_numpy(oracle.pool(bits, L, blk))
        return _check_tensor(x, as_t(bits), means, grid, L, blk)

    assert run(ref_bits.copy()) == 0.0
    two_steps = ref_bits.copy()
    two_steps[0, 0, 5, 7] += 2
    with pytest.raises(AssertionError):
        run(two_steps)
    many = ref_bits.copy().reshape(-1)
    idx = np.arange(0, L * 32, 40)  # about 2.5% of the valid elements of the first head, one step each
    many[idx] = many[idx] + 1
    with pytest.raises(AssertionError):
        run(many.reshape(ref_bits.shape))
    swapped = ref_bits.copy()
    swapped[..., 0::2], swapped[..., 1::2] = ref_bits[..., 1::2], ref_bits[..., 0::2]
    with pytest.raises(AssertionError):
        run(swapped)
    padded = ref_bits.copy()
    padded[0, 1, L + 2, 0] ^= 1
    with pytest.raises(AssertionError):
        run(padded)
