"""GPU parity of the NEXT rows at the sizes bench.py times them: batch 1, 40 heads,
d = 128, block 128, on the long-sequence grid 24 x 64 x 80 (L = 122,880) and the 480p
grid 21 x 30 x 52 (L = 32,760, a ragged last block).

- FP8 path (page "知识卡片：600倍加速，720p视频实时生成！单卡也能带的动14B模型", 方法/产品要点,
  bullet 动态稀疏量化注意力): the key mean against the fp64 mean of K on the host; codes and
  scales of EVERY block of Q and K bit for bit against the oracle's quantizer, both fed the
  same host-made smoothing vector; the attention, given the oracle's mask, on sampled
  (head, query block) units that include the first, the last and interior blocks, against
  the oracle's FP8 attention on the oracle's codes.
- fused 3D RoPE + pooling (same page, bullet 高效推理算子): every block mean against the
  means of the kernel's own rounded output, and whole heads (first, last, one random) of
  the rotated Q and K against the oracle's rotation.
- Light-Ulysses pre/post-processing (same page, bullet Light-Ulysses 多卡并行): the whole
  layer with 1 rank (the bench's configuration) and 8 ranks emulated on one GPU, through
  the all-to-all form (pack, re-slice, unpack) and the peer-put form (every rank's put
  kernel writing into the 8 local receive buffers); the two forms equal bit for bit,
  and sampled rows of each exchange bit for bit against the oracle's row quantizer.
"""
import numpy as np
import pytest
import torch

import oracle
from tests import parity_utils as pu
from video_dit_dynamic_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sbsa():
    pu.require_cuda()
    from video_dit_dynamic_b200 import sbsa as mod
    return mod


def _f64(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _sample_units(H, nb, n, seed):
    rng = np.random.default_rng(seed)
    units = {0, nb - 1, (H - 1) * nb, H * nb - 1, nb // 2}
    while len(units) < n:
        units.add(int(rng.integers(0, H * nb)))
    return sorted(units)


# ---------------------------------------------------------------------------- FP8 path
_FP8_WORKLOADS = {
    "long122880": inputs.WORKLOADS["long122880"],
    # blocks of 64 on the 480p grid: the attention runs as paired 128-row tiles
    "480p_b64": inputs.Workload("480p_b64", 1, 40, (21, 30, 52), 128, 64, 0.2),
}


@pytest.mark.parametrize("name", list(_FP8_WORKLOADS))
def test_fp8_path_full_size(sbsa, name):
    wl = _FP8_WORKLOADS[name]
    B, H, d, blk = wl.batch, wl.heads, wl.head_dim, wl.block
    L, Lp, nb = wl.seq_len, wl.seq_len_padded, wl.num_blocks
    kk = sbsa.sbsa_keep_blocks(nb, wl.keep)
    s = sbsa.make_shape(B, H, L, d, blk)
    q, k, v = inputs.make_qkv(wl, seed=0, device="cuda")
    qb, kb = pu.bits(q), pu.bits(k)
    rows = B * H * nb
    # the GPU's key mean (from its block means) against the fp64 mean of K on the host
    qm = torch.empty(rows * d, dtype=torch.float32, device="cuda")
    km = torch.empty_like(qm)
    sbsa.sbsa_pool_qk(s, q, k, qm, km)
    kbar_gpu = torch.empty(B * H * d, dtype=torch.float32, device="cuda")
    sbsa.sbsa_key_mean(s, km, kbar_gpu)
    sbsa.sbsa_check()
    kbar_host = np.stack([_f64(kb[0, h, :L]).mean(axis=0) for h in range(H)])[None]  # [1, H, d] fp64
    np.testing.assert_allclose(kbar_gpu.cpu().double().numpy().reshape(1, H, d), kbar_host, rtol=0, atol=2e-6)
    # codes and scales of every block, with the host's smoothing vector on both sides
    smooth = kbar_host.astype(np.float32)
    q8 = torch.empty(q.numel(), dtype=torch.uint8, device="cuda")
    k8 = torch.empty_like(q8)
    qs = torch.empty(rows, dtype=torch.float32, device="cuda")
    ks = torch.empty_like(qs)
    sbsa.sbsa_quantize_qk_fp8(s, q, k, torch.from_numpy(smooth.reshape(-1)).cuda(), q8, k8, qs, ks)
    sbsa.sbsa_check()
    qc, qsc = oracle.quantize_fp8(qb, L, blk)
    kc, ksc = oracle.quantize_fp8(kb, L, blk, smooth)
    np.testing.assert_array_equal(qs.cpu().numpy().reshape(B, H, nb), qsc)
    np.testing.assert_array_equal(ks.cpu().numpy().reshape(B, H, nb), ksc)
    for got_t, ref in ((q8, qc), (k8, kc)):
        got = got_t.cpu().numpy().reshape(ref.shape)
        # +0 / -0 may differ where a value rounds to zero
        same = (got == ref) | (((got & 0x7F) == 0) & ((ref & 0x7F) == 0))
        assert same.all(), f"{np.count_nonzero(~same)} codes differ"
    del q8, k8
    # attention given the oracle's mask, on the oracle's codes (equal to the GPU's, above)
    qmo, kmo = oracle.pool(qb, L, blk), oracle.pool(kb, L, blk)
    col = oracle.select(qmo, kmo, kk)
    rp = oracle.uniform_row_ptr(B, H, nb, kk)
    q8o = torch.from_numpy(qc.reshape(-1)).cuda()
    k8o = torch.from_numpy(kc.reshape(-1)).cuda()
    o = torch.empty_like(q)
    sbsa.sbsa_attention_fwd_fp8(s, q8o, k8o, v, torch.from_numpy(qsc.reshape(-1)).cuda(),
                                torch.from_numpy(ksc.reshape(-1)).cuda(), torch.from_numpy(rp).cuda(),
                                torch.from_numpy(col.reshape(-1)).cuda(), 0.0, o)
    sbsa.sbsa_check()
    vb = pu.bits(v)
    units = _sample_units(H, nb, 64, seed=7)
    got = o.view(H * nb, blk, d)[torch.tensor(units, device="cuda")]
    ref = np.empty((len(units), blk, d))
    for h in sorted({u // nb for u in units}):
        idx = [n for n, u in enumerate(units) if u // nb == h]
        loc = [units[n] - h * nb for n in idx]
        ref[idx] = oracle.attention_fp8(qc[:, h:h + 1], qsc[:, h:h + 1], kc[:, h:h + 1], ksc[:, h:h + 1],
                                        vb[:, h:h + 1], L, blk, oracle.uniform_row_ptr(1, 1, nb, kk),
                                        col[:, h:h + 1], units=loc)
    pu.assert_attention_close(got, ref, "fp8 attention, %s sampled units" % name)


# ---------------------------------------------------------------------------- RoPE + pool
@pytest.mark.parametrize("name", ["480p", "long122880"])
def test_rope_pool_full_size(sbsa, name):
    wl = inputs.WORKLOADS[name]
    B, H, d, blk, grid = wl.batch, wl.heads, wl.head_dim, wl.block, wl.grid
    L, Lp, nb = wl.seq_len, wl.seq_len_padded, wl.num_blocks
    s = sbsa.make_shape(B, H, L, d, blk)
    q, k, _ = inputs.make_qkv(wl, seed=0, device="cuda")
    table = torch.empty(sbsa.sbsa_rope_table_floats(d, grid), dtype=torch.float32, device="cuda")
    sbsa.sbsa_rope_table_init(d, grid, 10000.0, table)
    qo, ko = torch.empty_like(q), torch.empty_like(k)
    qm = torch.empty(B * H * nb * d, dtype=torch.float32, device="cuda")
    km = torch.empty_like(qm)
    sbsa.sbsa_rope_pool_qk(s, grid, table, q, k, qo, ko, qm, km)
    sbsa.sbsa_check()
    heads = sorted({0, H - 1, int(np.random.default_rng(L).integers(1, H - 1))})
    for x_in, x_out, means in ((q, qo, qm), (k, ko, km)):
        bits_in, got = pu.bits(x_in), pu.bits(x_out)
        # every block mean: the means of the kernel's own rounded output
        own = oracle.pool(got, L, blk)
        np.testing.assert_allclose(means.cpu().double().numpy().reshape(own.shape), own, rtol=2e-6, atol=1e-6)
        # padded tokens pass through bit for bit
        np.testing.assert_array_equal(got[:, :, L:], bits_in[:, :, L:])
        for h in heads:
            ref_bits, ref_means = oracle.rope_pool(bits_in[:, h:h + 1], grid, L, blk)
            g, r = _f64(got[:, h:h + 1]), _f64(ref_bits)
            x = _f64(bits_in[:, h:h + 1])
            pair_norm = np.repeat(np.hypot(x[..., 0::2], x[..., 1::2]), 2, axis=-1)
            bound = np.maximum(np.abs(r), np.abs(g)) * 2.0 ** -7 + pair_norm * 2.0 ** -21
            diff = np.abs(g - r)
            assert np.all(diff <= bound), f"{name} head {h}: worst excess {np.max(diff - bound):.3e}"
            frac = np.mean(got[:, h:h + 1] != ref_bits)
            assert frac < 0.01, f"{name} head {h}: {frac:.4f} of the elements differ by one bf16 step"
            np.testing.assert_allclose(means.cpu().double().numpy().reshape(own.shape)[:, h:h + 1], ref_means,
                                       rtol=0, atol=2e-3)


# ---------------------------------------------------------------------------- Light-Ulysses
def _rows_oracle(rows_bits: np.ndarray) -> np.ndarray:
    """Each row crosses as e4m3 codes with one scale and comes back as bf16."""
    return oracle.dequantize_rows_bf16(*oracle.quantize_rows_fp8(rows_bits))


@pytest.mark.parametrize("G", [1, 8])
def test_ulysses_whole_layer(sbsa, G):
    wl = inputs.WORKLOADS["long122880"]
    L, Lp, H, d = wl.seq_len, wl.seq_len_padded, wl.heads, wl.head_dim
    Lr, Hg = L // G, H // G
    shape = sbsa.make_ulysses_shape(G, L, Lp, H, d)
    g = torch.Generator(device="cuda").manual_seed(200)
    x = torch.randn(L, 3, H, d, generator=g, device="cuda")
    x = (x * torch.exp(torch.randn(L, 3, H, 1, generator=g, device="cuda"))).to(torch.bfloat16)
    x[5, 2, 3] = 0  # an all-zero row
    xs = [x[r * Lr:(r + 1) * Lr] for r in range(G)]
    nbytes = sbsa.sbsa_ulysses_qkv_bytes(shape, Hg)
    n = nbytes // G
    # all-to-all form: pack, re-slice, unpack
    sends = [torch.empty(nbytes, dtype=torch.uint8, device="cuda") for _ in range(G)]
    for r in range(G):
        sbsa.sbsa_ulysses_pack_qkv(shape, 0, Hg, xs[r], sends[r])
    recvs = [torch.cat([sends[i][j * n:(j + 1) * n] for i in range(G)]) for j in range(G)]
    del sends
    outs = [[torch.empty(Hg, Lp, d, dtype=torch.bfloat16, device="cuda") for _ in range(3)] for _ in range(G)]
    for r in range(G):
        sbsa.sbsa_ulysses_unpack_qkv(shape, 0, Hg, recvs[r], *outs[r])
    sbsa.sbsa_check()
    # peer-put form: every rank writes straight into the G receive buffers
    pbufs = [torch.empty(nbytes, dtype=torch.uint8, device="cuda") for _ in range(G)]
    bases = torch.tensor([b.data_ptr() for b in pbufs], dtype=torch.int64, device="cuda")
    for r in range(G):
        sbsa.sbsa_ulysses_put_qkv(shape, 0, Hg, xs[r], bases, 0, r)
    outs_p = [[torch.empty(Hg, Lp, d, dtype=torch.bfloat16, device="cuda") for _ in range(3)] for _ in range(G)]
    for r in range(G):
        sbsa.sbsa_ulysses_unpack_qkv(shape, 0, Hg, pbufs[r], *outs_p[r])
    sbsa.sbsa_check()
    for r in range(G):
        for c in range(3):
            assert torch.equal(outs[r][c], outs_p[r][c]), f"rank {r} tensor {c}: put and all-to-all differ"
    del pbufs, outs_p, recvs
    # sampled (token, q/k/v, head) rows against the oracle, at their destination
    rng = np.random.default_rng(G)
    edge_t = sorted({0, Lr - 1, Lr % L, L - 1})
    edge_h = sorted({0, Hg - 1, Hg % H, H - 1})
    samp = [(t, c, h) for t in edge_t for c in range(3) for h in edge_h] + [(5, 2, 3)]
    samp += [(int(rng.integers(L)), int(rng.integers(3)), int(rng.integers(H))) for _ in range(4096)]
    tt = torch.tensor([p[0] for p in samp], device="cuda")
    cc = torch.tensor([p[1] for p in samp], device="cuda")
    hh = torch.tensor([p[2] for p in samp], device="cuda")
    src = pu.bits(x[tt, cc, hh])
    ref = _rows_oracle(src)
    got = np.stack([pu.bits(outs[h // Hg][c][h % Hg, t]) for t, c, h in samp])
    np.testing.assert_array_equal(got, ref)
    # the return exchange: rank r's "attention output" (its unpacked q) back to token shards
    obytes = sbsa.sbsa_ulysses_o_bytes(shape, Hg)
    m = obytes // G
    osend = [torch.empty(obytes, dtype=torch.uint8, device="cuda") for _ in range(G)]
    for r in range(G):
        sbsa.sbsa_ulysses_pack_o(shape, 0, Hg, outs[r][0], osend[r])
    orecv = [torch.cat([osend[i][j * m:(j + 1) * m] for i in range(G)]) for j in range(G)]
    del osend
    ys = [torch.empty(Lr, H, d, dtype=torch.bfloat16, device="cuda") for _ in range(G)]
    for r in range(G):
        sbsa.sbsa_ulysses_unpack_o(shape, 0, Hg, orecv[r], ys[r])
    sbsa.sbsa_check()
    del orecv
    obufs = [torch.empty(obytes, dtype=torch.uint8, device="cuda") for _ in range(G)]
    obases = torch.tensor([b.data_ptr() for b in obufs], dtype=torch.int64, device="cuda")
    for r in range(G):
        sbsa.sbsa_ulysses_put_o(shape, 0, Hg, outs[r][0], obases, 0, r)
    ys_p = [torch.empty(Lr, H, d, dtype=torch.bfloat16, device="cuda") for _ in range(G)]
    for r in range(G):
        sbsa.sbsa_ulysses_unpack_o(shape, 0, Hg, obufs[r], ys_p[r])
    sbsa.sbsa_check()
    for r in range(G):
        assert torch.equal(ys[r], ys_p[r]), f"rank {r}: put_o and the all-to-all differ"
    osamp = [(t, h) for t in edge_t for h in edge_h]
    osamp += [(int(rng.integers(L)), int(rng.integers(H))) for _ in range(4096)]
    src = np.stack([pu.bits(outs[h // Hg][0][h % Hg, t]) for t, h in osamp])
    ref = _rows_oracle(src)
    got = np.stack([pu.bits(ys[t // Lr][t % Lr, h]) for t, h in osamp])
    np.testing.assert_array_equal(got, ref)
