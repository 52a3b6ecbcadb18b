"""GPU parity of the FP8 path against the oracle.

- key mean: against the oracle's block means reduced in fp64 (fp32 sums on the GPU);
- quantization: codes and scales bit for bit against oracle.quantize_fp8 fed the same
  bf16 bits and the same fp32 smoothing vector (both take the code decisions in the
  same fp32 operations);
- attention: against oracle.attention_fp8 on the GPU's own codes and scales, with the
  tolerances of the bf16 attention (the only differences left are fp32 accumulation
  and P rounded to bf16), and loosely against exact attention on the unquantized inputs.
"""
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


def _quantize(sbsa, s, q, k, smooth):
    n = q.numel()
    rows = s.batch * s.heads * s.num_blocks
    q8 = torch.empty(n, dtype=torch.uint8, device="cuda")
    k8 = torch.empty_like(q8)
    qs = torch.empty(rows, dtype=torch.float32, device="cuda")
    ks = torch.empty_like(qs)
    sbsa.sbsa_quantize_qk_fp8(s, q, k, smooth, q8, k8, qs, ks)
    sbsa.sbsa_check()
    return q8, k8, qs, ks


def _means(sbsa, s, q, k):
    rows = s.batch * s.heads * s.num_blocks
    qm = torch.empty(rows * s.head_dim, dtype=torch.float32, device="cuda")
    km = torch.empty_like(qm)
    sbsa.sbsa_pool_qk(s, q, k, qm, km)
    return qm, km


@pytest.mark.parametrize("blk,L,H", [(128, 1000, 2), (64, 777, 3), (128, 4096, 1)])
def test_key_mean(blk, L, H):
    sbsa = _sbsa()
    d = 128
    wl = inputs.Workload("t", 1, H, (1, 1, L), d, blk, 0.2)
    q, k, _ = inputs.make_qkv(wl, seed=blk + L, device="cuda")
    s = sbsa.make_shape(1, H, L, d, blk)
    _, km = _means(sbsa, s, q, k)
    out = torch.empty(H * d, dtype=torch.float32, device="cuda")
    sbsa.sbsa_key_mean(s, km, out)
    kb = inputs.bf16_bits(k)
    kv = (kb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    ref = kv[:, :, :L].mean(axis=2).reshape(-1)
    np.testing.assert_allclose(out.cpu().double().numpy(), ref, rtol=0, atol=2e-6)


@pytest.mark.parametrize("blk,L,H,smooth", [(128, 1000, 2, True), (64, 777, 3, True), (128, 256, 1, False)])
def test_quantize_bit_exact(blk, L, H, smooth):
    sbsa = _sbsa()
    d = 128
    wl = inputs.Workload("t", 1, H, (1, 1, L), d, blk, 0.2)
    q, k, _ = inputs.make_qkv(wl, seed=L + H, device="cuda")
    k = k * 3.0 + 0.5  # a key offset worth smoothing away
    k = k.to(torch.bfloat16)
    s = sbsa.make_shape(1, H, L, d, blk)
    sm = None
    if smooth:
        sm = torch.randn(H * d, generator=torch.Generator().manual_seed(L)).float().cuda() * 0.5
    q8, k8, qs, ks = _quantize(sbsa, s, q, k, sm)
    Lp = s.seq_len_padded
    qc, qsc = oracle.quantize_fp8(inputs.bf16_bits(q), L, blk)
    kc, ksc = oracle.quantize_fp8(inputs.bf16_bits(k), L, blk,
                                  None if sm is None else sm.cpu().numpy().reshape(1, H, d))
    np.testing.assert_array_equal(qs.cpu().numpy().reshape(1, H, -1), qsc)
    np.testing.assert_array_equal(ks.cpu().numpy().reshape(1, H, -1), ksc)
    got_q = q8.cpu().numpy().reshape(1, H, Lp, d)
    got_k = k8.cpu().numpy().reshape(1, H, Lp, d)
    # +0 / -0 may differ where a value rounds to zero; compare the decoded values there
    for got, ref in ((got_q, qc), (got_k, kc)):
        same = (got == ref) | ((got & 0x7F) == 0) & ((ref & 0x7F) == 0)
        assert same.all(), f"{np.count_nonzero(~same)} codes differ"


@pytest.mark.parametrize("blk,L,H,keep", [(128, 1000, 2, 0.3), (64, 700, 2, 0.25), (128, 3000, 2, 0.2)])
def test_fp8_attention_matches_oracle(blk, L, H, keep):
    sbsa = _sbsa()
    d = 128
    wl = inputs.Workload("t", 1, H, (1, 1, L), d, blk, keep)
    q, k, v = inputs.make_qkv(wl, seed=blk * 7 + L, device="cuda")
    s = sbsa.make_shape(1, H, L, d, blk)
    nb, Lp = s.num_blocks, s.seq_len_padded
    qm, km = _means(sbsa, s, q, k)
    kbar = torch.empty(H * d, dtype=torch.float32, device="cuda")
    sbsa.sbsa_key_mean(s, km, kbar)
    q8, k8, qs, ks = _quantize(sbsa, s, q, k, kbar)
    kk = sbsa.sbsa_keep_blocks(nb, keep)
    rp, ci = pu.gpu_select(s, qm, km, kk)
    o = torch.empty_like(q)
    sbsa.sbsa_attention_fwd_fp8(s, q8, k8, v, qs, ks, rp, ci, 0.0, o)
    sbsa.sbsa_check()
    col = ci.cpu().numpy().reshape(1, H, nb, kk)
    rpn = rp.cpu().numpy()
    ref = oracle.attention_fp8(q8.cpu().numpy().reshape(1, H, Lp, d), qs.cpu().numpy().reshape(1, H, nb),
                               k8.cpu().numpy().reshape(1, H, Lp, d), ks.cpu().numpy().reshape(1, H, nb),
                               inputs.bf16_bits(v), L, blk, rpn, col)
    pu.assert_attention_close(o, ref, f"fp8 blk={blk} L={L} keep={keep}")
    # and close to exact attention on the unquantized inputs (smoothing changes nothing,
    # quantization a little)
    exact = oracle.attention(inputs.bf16_bits(q), inputs.bf16_bits(k), inputs.bf16_bits(v), L, blk, rpn, col)
    err = np.abs(o.float().cpu().numpy() - exact)[:, :, :L]
    assert err.max() < 0.1 and err.mean() < 0.01, (err.max(), err.mean())


def test_fp8_path_rejects_head_dim_64():
    sbsa = _sbsa()
    s = sbsa.make_shape(1, 1, 256, 64, 64)
    q = torch.zeros(256 * 64, dtype=torch.bfloat16, device="cuda")
    q8 = torch.zeros(256 * 64, dtype=torch.uint8, device="cuda")
    sc = torch.ones(4, dtype=torch.float32, device="cuda")
    with pytest.raises(sbsa.SbsaError):
        sbsa.sbsa_quantize_qk_fp8(s, q, q, None, q8, q8, sc, sc)
