"""The kernels' give-up path on the GPU, driven without a stalled pipeline.

Every pipeline wait of the attention, selection, RoPE + pooling and FP8 quantizer
kernels is bounded.  With the pipeline limit lowered to 0 through the C ABI
(sbsa_set_pipeline_wait_ns), a wait whose barrier has not completed at its first test
gives up at once: the kernel latches SBSA_ERR_TIMEOUT, the launch's other CTAs stop,
and each CTA waits (with its own, unchanged limit) for the copies and tensor-core work
it has in flight and releases its tensor memory before it exits.  Each kernel must end
that way, sbsa_check must report SBSA_ERR_TIMEOUT, and with the limit restored the same
calls must match the oracle again: the context and the GPU carry on.  No wait here is
left without a limit, nothing traps and no memory is touched out of bounds.
"""
import numpy as np
import pytest
import torch

import oracle
from tests import parity_utils as pu
from video_dit_dynamic_b200 import inputs

pytestmark = pytest.mark.gpu

DEFAULT_LIMIT_NS = 1_000_000_000


@pytest.fixture
def sbsa():
    pu.require_cuda()
    from video_dit_dynamic_b200 import sbsa as mod
    mod.sbsa_check()  # nothing latched before the test
    yield mod
    mod.sbsa_set_pipeline_wait_ns(DEFAULT_LIMIT_NS)
    torch.cuda.synchronize()


def _expect_timeout(sbsa):
    with pytest.raises(sbsa.SbsaError) as err:
        sbsa.sbsa_check()
    assert err.value.status == 5, err.value  # SBSA_ERR_TIMEOUT


def _case():
    # 2 heads, d = 128, 40 blocks of 128 with a ragged last block, keep 25%
    wl = inputs.Workload("giveup", 1, 2, (1, 1, 5100), 128, 128, 0.25)
    q, k, v = inputs.make_qkv(wl, seed=21, device="cuda")
    return wl, q, k, v


def test_attention_and_select_give_up_then_recover(sbsa):
    wl, q, k, v = _case()
    s = sbsa.make_shape(1, wl.heads, wl.seq_len, wl.head_dim, wl.block)
    nb = s.num_blocks
    kk = sbsa.sbsa_keep_blocks(nb, wl.keep)
    qm, km = pu.gpu_pool(s, q, k)
    sbsa.sbsa_check()
    sbsa.sbsa_set_pipeline_wait_ns(0)
    rp, ci = pu.gpu_select(s, qm, km, kk)
    _expect_timeout(sbsa)
    # the attention, on a valid block list (the oracle's), gives up the same way
    qb, kb, vb = pu.bits(q), pu.bits(k), pu.bits(v)
    qmo, kmo = oracle.pool(qb, wl.seq_len, wl.block), oracle.pool(kb, wl.seq_len, wl.block)
    col = oracle.select(qmo, kmo, kk)
    rpo = oracle.uniform_row_ptr(1, wl.heads, nb, kk)
    rp_d, ci_d = torch.from_numpy(rpo).cuda(), torch.from_numpy(col.reshape(-1)).cuda()
    pu.gpu_attention(s, q, k, v, rp_d, ci_d)
    _expect_timeout(sbsa)
    # limit restored: the same calls complete and match the oracle
    sbsa.sbsa_set_pipeline_wait_ns(DEFAULT_LIMIT_NS)
    rp, ci = pu.gpu_select(s, qm, km, kk)
    o = pu.gpu_attention(s, q, k, v, rp_d, ci_d)
    sbsa.sbsa_check()
    pu.assert_selection_ok(ci.cpu().numpy().reshape(1, wl.heads, nb, kk), col, qmo, kmo, kk)
    ref = oracle.attention(qb, kb, vb, wl.seq_len, wl.block, rpo, col)
    pu.assert_attention_close(o[:, :, :wl.seq_len], ref[:, :, :wl.seq_len], "after the give-up")


def _flush_l2():
    """Write a buffer larger than the 126 MB L2, so the next kernel reads from HBM."""
    torch.empty(256 << 20, dtype=torch.uint8, device="cuda").fill_(1)
    torch.cuda.synchronize()


def test_rope_pool_and_fp8_quantizer_give_up_then_recover(sbsa):
    # the 480p workload (40 heads, 21 x 30 x 52 tokens, 335 MB per tensor): with L2 flushed
    # each CTA's tile comes from HBM, so its first test of the copy barrier finds it
    # still in flight
    wl = inputs.WORKLOADS["480p"]
    q, k, _ = inputs.make_qkv(wl, seed=22, device="cuda")
    grid, d, blk, H = wl.grid, wl.head_dim, wl.block, wl.heads
    s = sbsa.make_shape(1, H, wl.seq_len, d, blk)
    nb = s.num_blocks
    table = torch.empty(sbsa.sbsa_rope_table_floats(d, grid), dtype=torch.float32, device="cuda")
    sbsa.sbsa_rope_table_init(d, grid, 10000.0, table)
    qo, ko = torch.empty_like(q), torch.empty_like(k)
    qm = torch.empty(H * nb * d, dtype=torch.float32, device="cuda")
    km = torch.empty_like(qm)
    q8 = torch.empty(q.numel(), dtype=torch.uint8, device="cuda")
    k8 = torch.empty_like(q8)
    qs = torch.empty(H * nb, dtype=torch.float32, device="cuda")
    ks = torch.empty_like(qs)
    sbsa.sbsa_check()
    sbsa.sbsa_set_pipeline_wait_ns(0)
    _flush_l2()
    sbsa.sbsa_rope_pool_qk(s, grid, table, q, k, qo, ko, qm, km)
    _expect_timeout(sbsa)
    _flush_l2()
    sbsa.sbsa_quantize_qk_fp8(s, q, k, None, q8, k8, qs, ks)
    _expect_timeout(sbsa)
    sbsa.sbsa_set_pipeline_wait_ns(DEFAULT_LIMIT_NS)
    sbsa.sbsa_rope_pool_qk(s, grid, table, q, k, qo, ko, qm, km)
    sbsa.sbsa_quantize_qk_fp8(s, q, k, None, q8, k8, qs, ks)
    sbsa.sbsa_check()
    # the means are the means of the kernel's own rounded output, the rotation within the
    # rope parity bound of the oracle's (heads 0 and H-1), and the FP8 codes and scales
    # the oracle's
    got = pu.bits(qo)
    qin = pu.bits(q)
    np.testing.assert_allclose(qm.cpu().double().numpy().reshape(1, H, nb, d),
                               oracle.pool(got, wl.seq_len, blk), rtol=2e-6, atol=1e-6)
    to_f = lambda b: (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    for h in (0, H - 1):
        ref_bits, _ = oracle.rope_pool(qin[:, h:h + 1], grid, wl.seq_len, blk)
        g, r = to_f(got[:, h:h + 1]), to_f(ref_bits)
        assert np.all(np.abs(g - r) <= np.maximum(np.abs(g), np.abs(r)) * 2.0 ** -7 + 1e-5)
    qc, qsc = oracle.quantize_fp8(qin, wl.seq_len, blk)
    np.testing.assert_array_equal(qs.cpu().numpy().reshape(qsc.shape), qsc)
    gc = q8.cpu().numpy().reshape(qc.shape)
    assert np.all((gc == qc) | (((gc & 0x7F) == 0) & ((qc & 0x7F) == 0)))
