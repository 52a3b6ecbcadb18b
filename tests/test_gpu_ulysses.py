"""GPU parity of the Light-Ulysses pre/post-processing kernels against the oracle.

The kernels of G ranks run on one GPU: every emulated rank packs its send buffer, the
all-to-all is a re-slicing of those buffers in the test (slice j of rank i's send buffer
is slice i of rank j's receive buffer), and every rank unpacks.  Codes and scales decide
integers in the same fp32 operations on both sides, so the restored bf16 values are
compared bit for bit.  One rank runs LightUlysses end to end through the library.
"""
import numpy as np
import pytest
import torch

import oracle
from video_dit_dynamic_b200 import inputs

pytestmark = pytest.mark.gpu


def _sbsa():
    from video_dit_dynamic_b200 import sbsa
    sbsa.load()
    return sbsa


def _shards(G, L, H, d, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(L, 3, H, d, generator=g) * torch.exp(torch.randn(L, 3, H, 1, generator=g))
    x[3, 1, 0] = 0.0  # an all-zero row
    x = x.to(torch.bfloat16)
    return [x[r * (L // G):(r + 1) * (L // G)].contiguous() for r in range(G)]


def _exchange(sends, G):
    """all-to-all of equal slices: rank j receives slice j of every rank's buffer."""
    n = sends[0].numel() // G
    return [torch.cat([sends[i][j * n:(j + 1) * n] for i in range(G)]) for j in range(G)]


@pytest.mark.parametrize("G,L,H,Lp,chunks", [(2, 200, 4, 256, [(0, 2)]), (4, 400, 8, 512, [(0, 1), (1, 1)]),
                                             (1, 130, 2, 256, [(0, 2)]), (2, 256, 6, 256, [(0, 2), (2, 1)])])
def test_qkv_and_o_exchange_bit_exact(G, L, H, Lp, chunks):
    sbsa = _sbsa()
    d = 128
    shape = sbsa.make_ulysses_shape(G, L, Lp, H, d)
    shards = _shards(G, L, H, d, seed=G * 100 + L)
    ref = oracle.ulysses_qkv([inputs.bf16_bits(s) for s in shards], H, L, Lp)
    Hg = H // G
    outs = [[torch.full((Hg, Lp, d), 7.0, dtype=torch.bfloat16, device="cuda") for _ in range(3)] for _ in range(G)]
    for h0, hc in chunks:
        nbytes = sbsa.sbsa_ulysses_qkv_bytes(shape, hc)
        sends = []
        for r in range(G):
            send = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
            sbsa.sbsa_ulysses_pack_qkv(shape, h0, hc, shards[r].cuda(), send)
            sends.append(send)
        for r, recv in enumerate(_exchange(sends, G)):
            sbsa.sbsa_ulysses_unpack_qkv(shape, h0, hc, recv, *outs[r])
    sbsa.sbsa_check()
    covered = sorted(h for h0, hc in chunks for h in range(h0, h0 + hc))
    for r in range(G):
        for c in range(3):
            got = inputs.bf16_bits(outs[r][c].cpu())
            np.testing.assert_array_equal(got[covered], ref[r][c][covered])
    # the return exchange of an oracle-made attention output
    o_ref = [ref[r][0] for r in range(G)]  # any [Hg, Lp, d] bf16 tensor per rank
    y_ref = oracle.ulysses_o(o_ref, H, L)
    ys = [torch.zeros(L // G, H, d, dtype=torch.bfloat16, device="cuda") for _ in range(G)]
    for h0, hc in chunks:
        nbytes = sbsa.sbsa_ulysses_o_bytes(shape, hc)
        sends = []
        for r in range(G):
            send = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
            o = torch.from_numpy(o_ref[r].view(np.int16)).view(torch.bfloat16).cuda()
            sbsa.sbsa_ulysses_pack_o(shape, h0, hc, o, send)
            sends.append(send)
        for r, recv in enumerate(_exchange(sends, G)):
            sbsa.sbsa_ulysses_unpack_o(shape, h0, hc, recv, ys[r])
    sbsa.sbsa_check()
    heads = sorted(i * Hg + h for i in range(G) for h in covered)
    for r in range(G):
        np.testing.assert_array_equal(inputs.bf16_bits(ys[r].cpu())[:, heads], y_ref[r][:, heads])


def test_light_ulysses_single_rank_end_to_end():
    from video_dit_dynamic_b200 import ulysses
    _sbsa()
    L, Lp, H, d = 500, 512, 4, 128
    x = _shards(1, L, H, d, seed=3)[0].cuda()
    ys = []
    for hc in (4, 1, 3):
        plan = ulysses.UlyssesPlan(world=1, tokens=L, tokens_padded=Lp, heads=H, head_dim=d, head_chunk=hc)
        lu = ulysses.LightUlysses(plan, group=None, keep=1.0)
        ys.append(lu.forward(x))
        torch.cuda.synchronize()
        # the exchanged q, k, v are the oracle's, bit for bit
        ref = oracle.ulysses_qkv([inputs.bf16_bits(x.cpu())], H, L, Lp)[0]
        for c, t in enumerate((lu.q, lu.k, lu.v)):
            np.testing.assert_array_equal(inputs.bf16_bits(t.cpu()), ref[c])
    # the head-level pipeline does not change the result
    assert torch.equal(ys[0], ys[1]) and torch.equal(ys[0], ys[2])
    # against the oracle's layer: exchange -> dense attention (keep = 1) -> bf16 -> return
    ref = oracle.ulysses_qkv([inputs.bf16_bits(x.cpu())], H, L, Lp)[0]
    nb = Lp // 128
    rp = oracle.uniform_row_ptr(1, H, nb, nb)
    col = np.broadcast_to(np.arange(nb, dtype=np.int32), (1, H, nb, nb)).copy()
    o = oracle.attention(ref[0][None], ref[1][None], ref[2][None], L, 128, rp, col)[0]
    y_ref = oracle.ulysses_o([oracle.bf16_round(o)], H, L)[0]
    yr = (y_ref.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    yg = ys[0].float().cpu().double().numpy()
    # attention tolerance, plus one e4m3 quantum of each side's row (both outputs cross as FP8)
    row_max = np.abs(yr).max(axis=2, keepdims=True)
    assert np.all(np.abs(yg - yr) <= 2e-2 + row_max * 2.0 ** -3)
    assert np.mean(np.abs(yg - yr)) < 2e-3


@pytest.mark.parametrize("G,L,H,Lp,hc", [(2, 256, 4, 256, 1), (4, 400, 8, 512, 1), (2, 250, 6, 256, 2),
                                         (2, 256, 8, 256, 1)])  # 4 chunks: buffers reused within a call
def test_peer_put_exchange_emulated_ranks(G, L, H, Lp, hc):
    """The peer-put exchange with G ranks emulated on one GPU (their allocations are local
    buffers, every rank's step runs before the next step): q, k, v bit-exact with the
    oracle's exchange, the layer within the attention tolerance of the oracle's, and a
    second call (buffers reused, acknowledgements awaited) identical to the first."""
    from video_dit_dynamic_b200 import ulysses
    sbsa = _sbsa()
    d = 128
    plan = ulysses.UlyssesPlan(world=G, tokens=L, tokens_padded=Lp, heads=H, head_dim=d, head_chunk=hc)
    exs = ulysses.PeerExchange.emulated(plan, "cuda", timeout_s=5.0)
    layers = [ulysses.LightUlysses(plan, keep=1.0, exchange=exs[r]) for r in range(G)]
    shards = _shards(G, L, H, d, seed=G * 7 + L)
    xs = [s.cuda() for s in shards]
    ys = [y.clone() for y in ulysses.lockstep_forward(layers, xs)]
    sbsa.sbsa_check()
    ref = oracle.ulysses_qkv([inputs.bf16_bits(s) for s in shards], H, L, Lp)
    for r in range(G):
        for c, t in enumerate((layers[r].q, layers[r].k, layers[r].v)):
            np.testing.assert_array_equal(inputs.bf16_bits(t.cpu()), ref[r][c])
    ys2 = ulysses.lockstep_forward(layers, xs)
    sbsa.sbsa_check()
    for r in range(G):
        assert torch.equal(ys[r], ys2[r])
    # the oracle's layer: exchange -> dense attention (keep = 1) per rank -> bf16 -> return
    nb = Lp // 128
    Hg = H // G
    rp = oracle.uniform_row_ptr(1, Hg, nb, nb)
    col = np.broadcast_to(np.arange(nb, dtype=np.int32), (1, Hg, nb, nb)).copy()
    os_ = [oracle.bf16_round(oracle.attention(ref[r][0][None], ref[r][1][None], ref[r][2][None], L, 128, rp, col)[0])
           for r in range(G)]
    y_ref = oracle.ulysses_o(os_, H, L)
    for r in range(G):
        yr = (y_ref[r].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        yg = ys[r].float().cpu().double().numpy()
        row_max = np.abs(yr).max(axis=2, keepdims=True)
        assert np.all(np.abs(yg - yr) <= 2e-2 + row_max * 2.0 ** -3)
        assert np.mean(np.abs(yg - yr)) < 2e-3


def test_peer_wait_gives_up_without_a_fault():
    """A wait on a flag nothing sets ends after its limit with SBSA_ERR_TIMEOUT from
    sbsa_check; the context stays usable."""
    sbsa = _sbsa()
    flags = torch.zeros(4, dtype=torch.int32, device="cuda")
    sbsa.sbsa_peer_wait(flags, 4, 12345, timeout_s=0.05)
    with pytest.raises(sbsa.SbsaError) as err:
        sbsa.sbsa_check()
    assert err.value.status == 5  # SBSA_ERR_TIMEOUT
    # flags that are set end the wait at once, and the next launches run normally
    bases = torch.tensor([flags.data_ptr()] * 4, dtype=torch.int64, device="cuda")  # four "peers", one array
    for i in range(4):
        sbsa.sbsa_peer_signal(bases, 0, i, 4, 777)
    sbsa.sbsa_peer_wait(flags, 4, 777, timeout_s=5.0)
    sbsa.sbsa_check()
    assert torch.all(flags == 777)
