"""GPU parity of the NVFP4 linear layer (amax, quantizer, block-scaled GEMM) against the oracle.

- amax: exact (a maximum of bf16 values);
- quantizer: codes and scales bit for bit against oracle.nvfp4_quantize on the same bf16
  bits (both sides take every decision in the same fp32 operations; a value that rounds
  to zero may carry either sign);
- GEMM: the GPU kernel fed the ORACLE's codes and scales, against oracle.nvfp4_gemm in
  fp64.  Bound per element: one bf16 rounding of the result (2^-8 relative) plus an
  accumulation term of 2^-16 of sum_k |A_k B_k| (fp32 accumulation of K <= 5120 exact
  products is far below it);
- end to end: GPU amax -> quantize -> GEMM against the oracle's quantize -> GEMM;
- the full-size layer (122,880 x 5,120 activations, 15,360 x 5,120 weights): each tensor's
  amax taken on the host from the full bf16 bits (and the GPU's amax equal to it), sampled
  rows quantized by the oracle with that host amax, and the outputs they produce.
"""
import numpy as np
import pytest
import torch

import oracle
from video_dit_dynamic_b200 import inputs

pytestmark = pytest.mark.gpu

ACC_REL = 2.0 ** -16


def _sbsa():
    from video_dit_dynamic_b200 import sbsa
    sbsa.load()
    return sbsa


def _bf16(rows, cols, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(rows, cols, generator=g) * scale).to(torch.bfloat16)


def _amax_of(x_bits):
    return np.float32(np.abs((x_bits.astype(np.uint32) << 16).view(np.float32)).max())


def _amax_host(x: torch.Tensor) -> np.float32:
    """max |x| of a bf16 tensor from its bits on the host: for non-NaN values the order of
    the magnitude bits (sign cleared) is the order of |x|."""
    bits = inputs.bf16_bits(x.cpu())
    top = np.uint32(np.max(bits & np.uint16(0x7FFF)))
    return np.array([top << np.uint32(16)], dtype=np.uint32).view(np.float32)[0]


def _codes_equal(got, ref):
    """Byte arrays of packed codes, compared nibble by nibble; a nibble may differ only
    as +0 (0x0) against -0 (0x8)."""
    ok = np.ones(got.shape, dtype=bool)
    for shift in (0, 4):
        g, r = (got >> shift) & 15, (ref >> shift) & 15
        ok &= (g == r) | (((g & 7) == 0) & ((r & 7) == 0))
    return ok


def _gpu_quantize(sbsa, x):
    rows, cols = x.shape
    amax = torch.empty(1, dtype=torch.float32, device="cuda")
    codes = torch.empty(rows * cols // 2, dtype=torch.uint8, device="cuda")
    scales = torch.empty(sbsa.sbsa_nvfp4_scale_bytes(rows, cols), dtype=torch.uint8, device="cuda")
    sbsa.sbsa_nvfp4_amax(x, amax)
    sbsa.sbsa_nvfp4_quantize(x, amax, codes, scales)
    return codes, scales, amax


def _check_gemm(c_gpu, ref, a_dec, b_dec):
    g = c_gpu.float().cpu().double().numpy()
    bound = np.abs(ref) * 2.0 ** -8 + ACC_REL * (np.abs(a_dec) @ np.abs(b_dec).T) + 1e-30
    err = np.abs(g - ref)
    assert np.all(np.isfinite(g))
    worst = np.max(err / bound)
    assert worst <= 1.0, f"worst error {worst:.3f} of the bound"
    return worst


@pytest.mark.parametrize("rows,cols", [(300, 512), (128, 64), (1, 256), (1000, 1280)])
def test_amax_and_quantize_bit_exact(rows, cols):
    sbsa = _sbsa()
    x = _bf16(rows, cols, seed=rows + cols)
    x[rows // 2, 3] = 11.5  # the tensor amax away from the first block
    xg = x.cuda()
    codes, scales, amax = _gpu_quantize(sbsa, xg)
    sbsa.sbsa_check()
    bits = inputs.bf16_bits(x)
    assert amax.item() == _amax_of(bits) == np.float32(11.5)
    rc, rs, s = oracle.nvfp4_quantize(bits)
    np.testing.assert_array_equal(scales.cpu().numpy(), rs)
    got = codes.cpu().numpy().reshape(rows, cols // 2)
    ok = _codes_equal(got, rc)
    assert ok.all(), f"{np.count_nonzero(~ok)} code bytes differ"


def test_quantize_all_zero_and_tiny_blocks():
    sbsa = _sbsa()
    x = torch.zeros(130, 128, dtype=torch.bfloat16)
    x[5, :16] = 1e-30  # scale underflows to 0 in e4m3: codes 0
    x[7, 16:32] = torch.linspace(-3, 3, 16).to(torch.bfloat16)
    codes, scales, amax = _gpu_quantize(sbsa, x.cuda())
    bits = inputs.bf16_bits(x)
    rc, rs, _ = oracle.nvfp4_quantize(bits)
    np.testing.assert_array_equal(scales.cpu().numpy(), rs)
    assert _codes_equal(codes.cpu().numpy().reshape(130, 64), rc).all()


@pytest.mark.parametrize("m,n,k,bias", [(128, 256, 256, True), (300, 264, 512, True), (1000, 1024, 1280, False),
                                        (2304, 2560, 512, True)])
def test_gemm_matches_oracle_on_oracle_codes(m, n, k, bias):
    sbsa = _sbsa()
    a = inputs.bf16_bits(_bf16(m, k, seed=m))
    b = inputs.bf16_bits(_bf16(n, k, seed=n + 1, scale=0.05))
    ac, asf, a_s = oracle.nvfp4_quantize(a)
    bc, bsf, b_s = oracle.nvfp4_quantize(b)
    bias_v = np.random.default_rng(m + n).standard_normal(n).astype(np.float32) if bias else None
    ref = oracle.nvfp4_gemm(ac, asf, a_s, bc, bsf, b_s, bias_v)
    dev = lambda arr: torch.from_numpy(np.ascontiguousarray(arr)).cuda()
    c = torch.empty(m, n, dtype=torch.bfloat16, device="cuda")
    sbsa.sbsa_nvfp4_gemm(m, n, k, dev(ac), dev(asf), dev(np.array([_amax_of(a)])), dev(bc), dev(bsf),
                         dev(np.array([_amax_of(b)])), dev(bias_v) if bias else None, c)
    sbsa.sbsa_check()
    _check_gemm(c, ref, oracle.nvfp4_dequantize(ac, asf, a_s), oracle.nvfp4_dequantize(bc, bsf, b_s))


def test_gemm_output_only_16_byte_aligned():
    """C starting 16 bytes past a 32-byte boundary takes the 16-byte store path."""
    sbsa = _sbsa()
    m, n, k = 259, 512, 256
    a = inputs.bf16_bits(_bf16(m, k, seed=41))
    b = inputs.bf16_bits(_bf16(n, k, seed=42, scale=0.05))
    ac, asf, a_s = oracle.nvfp4_quantize(a)
    bc, bsf, b_s = oracle.nvfp4_quantize(b)
    ref = oracle.nvfp4_gemm(ac, asf, a_s, bc, bsf, b_s, None)
    dev = lambda arr: torch.from_numpy(np.ascontiguousarray(arr)).cuda()
    buf = torch.empty(m * n + 32, dtype=torch.bfloat16, device="cuda")
    base = (-buf.data_ptr() // 2) % 16  # elements to the next 32-byte boundary
    c = buf[base + 8:base + 8 + m * n].view(m, n)
    assert c.data_ptr() % 32 == 16
    sbsa.sbsa_nvfp4_gemm(m, n, k, dev(ac), dev(asf), dev(np.array([_amax_of(a)])), dev(bc), dev(bsf),
                         dev(np.array([_amax_of(b)])), None, c)
    sbsa.sbsa_check()
    _check_gemm(c, ref, oracle.nvfp4_dequantize(ac, asf, a_s), oracle.nvfp4_dequantize(bc, bsf, b_s))


def test_gemm_end_to_end_from_bf16():
    sbsa = _sbsa()
    m, n, k = 520, 768, 1024
    a, b = _bf16(m, k, seed=5), _bf16(n, k, seed=6, scale=0.03)
    bias = torch.randn(n, generator=torch.Generator().manual_seed(7)).float()
    ac, asf, aam = _gpu_quantize(sbsa, a.cuda())
    bc, bsf, bam = _gpu_quantize(sbsa, b.cuda())
    c = torch.empty(m, n, dtype=torch.bfloat16, device="cuda")
    sbsa.sbsa_nvfp4_gemm(m, n, k, ac, asf, aam, bc, bsf, bam, bias.cuda(), c)
    sbsa.sbsa_check()
    qa, qb = oracle.nvfp4_quantize(inputs.bf16_bits(a)), oracle.nvfp4_quantize(inputs.bf16_bits(b))
    ref = oracle.nvfp4_gemm(*qa, *qb, bias.numpy())
    _check_gemm(c, ref, oracle.nvfp4_dequantize(*qa), oracle.nvfp4_dequantize(*qb))
    # and the quantized layer stays close to the bf16 layer it replaces
    exact = a.double().numpy() @ b.double().numpy().T + bias.double().numpy()[None, :]
    rel = np.linalg.norm(c.double().cpu().numpy() - exact) / np.linalg.norm(exact)
    assert rel < 0.2, rel


def test_gemm_full_size_sampled():
    """The QKV projection of one layer at the long-sequence size, sampled."""
    sbsa = _sbsa()
    m, n, k = 122880, 15360, 5120
    g = torch.Generator(device="cuda").manual_seed(11)
    a = torch.randn(m, k, generator=g, device="cuda").to(torch.bfloat16)
    b = (torch.randn(n, k, generator=g, device="cuda") * 0.02).to(torch.bfloat16)
    bias = torch.randn(n, generator=g, device="cuda").float()
    ac, asf, aam = _gpu_quantize(sbsa, a)
    bc, bsf, bam = _gpu_quantize(sbsa, b)
    c = torch.empty(m, n, dtype=torch.bfloat16, device="cuda")
    sbsa.sbsa_nvfp4_gemm(m, n, k, ac, asf, aam, bc, bsf, bam, bias, c)
    sbsa.sbsa_check()
    rng = np.random.default_rng(12)
    rows = np.sort(np.concatenate([[0, 127, 128, m - 1], rng.choice(m, 60, replace=False)]))
    cols = np.sort(np.concatenate([[0, 255, 256, n - 1], rng.choice(n, 60, replace=False)]))
    a_s = inputs.bf16_bits(a[torch.from_numpy(rows).cuda()].cpu())
    b_s = inputs.bf16_bits(b[torch.from_numpy(cols).cuda()].cpu())
    # the tensors' amax from the host copies of their bits, independent of the GPU path
    a_amax, b_amax = _amax_host(a), _amax_host(b)
    assert aam.item() == a_amax and bam.item() == b_amax, (aam.item(), a_amax, bam.item(), b_amax)
    qa = oracle.nvfp4_quantize(a_s, amax=float(a_amax))
    qb = oracle.nvfp4_quantize(b_s, amax=float(b_amax))
    # the sampled rows' codes are the GPU's rows
    got_a = ac.view(m, k // 2)[torch.from_numpy(rows).cuda()].cpu().numpy()
    assert _codes_equal(got_a, qa[0]).all()
    ref = oracle.nvfp4_gemm(*qa, *qb, bias.cpu().numpy()[cols])
    got = c[torch.from_numpy(rows).cuda()][:, torch.from_numpy(cols).cuda()]
    _check_gemm(got, ref, oracle.nvfp4_dequantize(*qa), oracle.nvfp4_dequantize(*qb))
