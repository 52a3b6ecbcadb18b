"""GPU parity: each kernel, called through the C ABI, against the CPU oracle on the
same seeded inputs, at sizes the oracle finishes in seconds that span several tiles
and ragged tails, plus edge cases (k = 1, k = nb, exact ties, variable-length and
empty CSR rows, out-of-range indices, large logits)."""
import math

import numpy as np
import pytest
import torch

import oracle
from tests import parity_utils as pu
from video_dit_dynamic_b200 import inputs, sbsa

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    pu.require_cuda()


# ---------------------------------------------------------------- pool

@pytest.mark.parametrize("d,blk,L,H", [(64, 64, 1000, 3), (128, 128, 1000, 3), (64, 128, 777, 2),
                                       (128, 64, 2048, 2), (128, 128, 128, 1), (64, 64, 1, 1)])
def test_pool_matches_oracle(d, blk, L, H):
    Lp = -(-L // blk) * blk
    q, k, _ = inputs.random_qkv(1, H, Lp, d, L=L, seed=100 + d + blk, device="cuda")
    # junk in padded tokens must be ignored
    q[:, :, L:] = 3.0
    k[:, :, L:] = -3.0
    s = pu.shape_of(q, L, blk)
    qm, km = pu.gpu_pool(s, q, k)
    pu.assert_means_close(qm, oracle.pool(pu.bits(q), L, blk))
    pu.assert_means_close(km, oracle.pool(pu.bits(k), L, blk))


# ---------------------------------------------------------------- select

def _random_means(B, H, nb, d, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    qm = torch.randn(B, H, nb, d, generator=g, device="cuda")
    km = torch.randn(B, H, nb, d, generator=g, device="cuda")
    return qm, km


@pytest.mark.parametrize("nb,k,d", [(1, 1, 64), (5, 2, 64), (33, 7, 128), (64, 64, 64), (100, 1, 128),
                                    (96, 96, 128), (257, 51, 128), (700, 70, 128), (960, 96, 128),
                                    (1024, 100, 128), (1500, 150, 64), (2048, 205, 128)])
def test_select_matches_oracle(nb, k, d):
    B, H = 1, 2
    qm, km = _random_means(B, H, nb, d, seed=nb * 7 + k)
    s = sbsa.make_shape(B, H, nb * 64, d, 64)
    rp, ci = pu.gpu_select(s, qm, km, k)
    qn, kn = qm.double().cpu().numpy(), km.double().cpu().numpy()
    ref = oracle.select(qn, kn, k)
    assert np.array_equal(rp.cpu().numpy(), np.arange(B * H * nb + 1) * k)
    pu.assert_selection_ok(ci.cpu().numpy().reshape(B, H, nb, k), ref, qn, kn, k)


@pytest.mark.parametrize("d", [64, 128])
def test_select_exact_ties_prefer_lower_index(d):
    nb, k = 40, 4
    qm, km = _random_means(1, 1, nb, d, seed=5)
    km *= 0.01
    for j in (3, 17, 29, 31, 39):  # identical key blocks: exact ties in every row's ranking
        km[0, 0, j] = qm[0, 0, 0] * 2.0
    s = sbsa.make_shape(1, 1, nb * 64, d, 64)
    _, ci = pu.gpu_select(s, qm, km, k)
    got = ci.cpu().numpy().reshape(nb, k)
    ref = oracle.select(qm.double().cpu().numpy(), km.double().cpu().numpy(), k)[0, 0]
    # row 0: the five tied copies outscore every other block; the three lowest win (exact
    # ties survive the tensor-core path too: equal means give bit-equal scores)
    np.testing.assert_array_equal(got[0], ref[0])
    np.testing.assert_array_equal(got[0], [0, 3, 17, 29])
    np.testing.assert_array_equal(got, ref)


@pytest.mark.parametrize("d", [64, 128])
def test_select_threshold_among_zero_scores(d):
    """Scores exactly 0 (from +0 and -0 key means) around the k-th place: every zero ties,
    and the lowest indices win, as in the oracle (which compares in fp64, where -0 == +0)."""
    nb, k = 48, 15
    qm = torch.full((1, 1, nb, d), 0.25, device="cuda")
    km = torch.zeros(1, 1, nb, d, device="cuda")
    km[0, 0, :10] = torch.linspace(1.0, 2.0, 10, device="cuda")[:, None]   # positive scores
    km[0, 0, 10:20] = -0.0                                                  # -0 scores
    km[0, 0, 30:] = -torch.linspace(1.0, 2.0, nb - 30, device="cuda")[:, None]  # negative scores
    s = sbsa.make_shape(1, 1, nb * 64, d, 64)
    _, ci = pu.gpu_select(s, qm, km, k)
    sbsa.sbsa_check()
    got = ci.cpu().numpy().reshape(1, 1, nb, k)
    qn, kn = qm.double().cpu().numpy(), km.double().cpu().numpy()
    ref = oracle.select(qn, kn, k)
    if d == 128:
        # the tensor-core path compares scores as floats after adding +0: exact agreement
        np.testing.assert_array_equal(got, ref)
    else:
        pu.assert_selection_ok(got, ref, qn, kn, k)


@pytest.mark.parametrize("scale", [1e-3, 1e4])
def test_select_scaled_means(scale):
    """The tf32 split of the scores is exact at any magnitude: scaled means select alike."""
    nb, k, d = 300, 30, 128
    qm, km = _random_means(1, 2, nb, d, seed=11)
    qm *= scale
    km *= scale
    s = sbsa.make_shape(1, 2, nb * 64, d, 64)
    rp, ci = pu.gpu_select(s, qm, km, k)
    qn, kn = qm.double().cpu().numpy(), km.double().cpu().numpy()
    pu.assert_selection_ok(ci.cpu().numpy().reshape(1, 2, nb, k), oracle.select(qn, kn, k), qn, kn, k)


def test_select_validate_csr_accepts_output():
    nb, k = 77, 9
    qm, km = _random_means(2, 3, nb, 128, seed=9)
    s = sbsa.make_shape(2, 3, nb * 128 - 5, 128, 128)
    rp, ci = pu.gpu_select(s, qm, km, k)
    assert sbsa.sbsa_validate_csr(s, rp, ci, ci.numel(), require_diagonal=True)
    bad = ci.clone()
    bad[5] = nb  # out of range
    assert not sbsa.sbsa_validate_csr(s, rp, bad, bad.numel())
    bad = ci.clone()
    bad[k:2 * k] = bad[k:2 * k].flip(0)  # not ascending
    assert not sbsa.sbsa_validate_csr(s, rp, bad, bad.numel())


# ---------------------------------------------------------------- attention

def _oracle_mask(q, k, L, blk, kk):
    qm = oracle.pool(pu.bits(q), L, blk)
    km = oracle.pool(pu.bits(k), L, blk)
    col = oracle.select(qm, km, kk)
    B, H, nb, _ = qm.shape
    rp = oracle.uniform_row_ptr(B, H, nb, kk)
    return rp, col, qm, km


@pytest.mark.parametrize("d,blk,L,H,keep", [(64, 64, 1024, 2, 0.25), (128, 128, 1000, 2, 0.3),
                                            (64, 128, 1500, 2, 0.5), (128, 64, 900, 1, 0.2),
                                            (128, 128, 2048, 1, 1.0), (64, 64, 1024, 2, 1.0)])
def test_attention_matches_oracle_given_oracle_mask(d, blk, L, H, keep):
    Lp = -(-L // blk) * blk
    q, k, v = inputs.random_qkv(1, H, Lp, d, L=L, seed=200 + d + blk + L, device="cuda")
    k[:, :, L:] = 9.0  # padded keys hold junk and must be masked
    v[:, :, L:] = 9.0
    nb = Lp // blk
    kk = oracle.keep_blocks(nb, keep)
    rp, col, _, _ = _oracle_mask(q, k, L, blk, kk)
    s = pu.shape_of(q, L, blk)
    o = pu.gpu_attention(s, q, k, v, torch.from_numpy(rp).cuda(), torch.from_numpy(col.reshape(-1)).cuda())
    ref = oracle.attention(pu.bits(q), pu.bits(k), pu.bits(v), L, blk, rp, col)
    pu.assert_attention_close(o, ref, f"d={d} blk={blk} L={L} keep={keep}")
    assert torch.all(o[:, :, L:] == 0)
    sbsa.sbsa_check()


def test_attention_tiny_workload_keep_all_is_dense():
    wl = inputs.WORKLOADS["tiny"]
    q, k, v = inputs.make_qkv(wl, seed=0, device="cuda")
    L, blk, nb = wl.seq_len, wl.block, wl.num_blocks
    rp = oracle.uniform_row_ptr(1, wl.heads, nb, nb)
    col = np.tile(np.arange(nb, dtype=np.int32), (1, wl.heads, nb, 1))
    s = pu.shape_of(q, L, blk)
    o = pu.gpu_attention(s, q, k, v, torch.from_numpy(rp).cuda(), torch.from_numpy(col.reshape(-1)).cuda())
    # dense softmax attention (torch fp64 library routine) on the same bf16 values
    ref = torch.nn.functional.scaled_dot_product_attention(q.double().cpu(), k.double().cpu(), v.double().cpu())
    pu.assert_attention_close(o, ref.numpy(), "keep=1 vs dense")


def test_attention_large_logits():
    d, blk, L = 128, 128, 1024
    q, k, v = inputs.random_qkv(1, 2, L, d, seed=31, device="cuda", q_scale=20.0)
    kk = 3
    rp, col, _, _ = _oracle_mask(q, k, L, blk, kk)
    s = pu.shape_of(q, L, blk)
    o = pu.gpu_attention(s, q, k, v, torch.from_numpy(rp).cuda(), torch.from_numpy(col.reshape(-1)).cuda())
    ref = oracle.attention(pu.bits(q), pu.bits(k), pu.bits(v), L, blk, rp, col)
    pu.assert_attention_close(o, ref, "Q x20")


def test_attention_explicit_scale():
    d, blk, L = 64, 64, 640
    q, k, v = inputs.random_qkv(1, 1, L, d, seed=32, device="cuda")
    rp, col, _, _ = _oracle_mask(q, k, L, blk, 4)
    s = pu.shape_of(q, L, blk)
    o = pu.gpu_attention(s, q, k, v, torch.from_numpy(rp).cuda(), torch.from_numpy(col.reshape(-1)).cuda(),
                         scale=0.05)
    ref = oracle.attention(pu.bits(q), pu.bits(k), pu.bits(v), L, blk, rp, col, scale=0.05)
    pu.assert_attention_close(o, ref, "scale=0.05")


@pytest.mark.parametrize("d,blk", [(128, 128), (64, 64), (128, 64)])
def test_attention_negative_scale(d, blk):
    """A negative logit scale (the logits are -|scale|.S: the softmax favours the lowest
    scores), through the unpaired and the paired (block 64) tiles."""
    L = 9 * blk - 13
    q, k, v = inputs.random_qkv(1, 2, 9 * blk, d, L=L, seed=36, device="cuda")
    rp, col, _, _ = _oracle_mask(q, k, L, blk, 3)
    s = pu.shape_of(q, L, blk)
    o = pu.gpu_attention(s, q, k, v, torch.from_numpy(rp).cuda(), torch.from_numpy(col.reshape(-1)).cuda(),
                         scale=-0.09)
    ref = oracle.attention(pu.bits(q), pu.bits(k), pu.bits(v), L, blk, rp, col, scale=-0.09)
    pu.assert_attention_close(o, ref, "scale=-0.09")


@pytest.mark.parametrize("d,blk", [(128, 128), (64, 64)])
def test_attention_variable_and_empty_rows(d, blk):
    H, nb = 2, 9
    L = nb * blk - 7
    Lp = nb * blk
    q, k, v = inputs.random_qkv(1, H, Lp, d, L=L, seed=33, device="cuda")
    rng = np.random.default_rng(34)
    rows = []
    for r in range(H * nb):
        n = int(rng.integers(0, nb + 1)) if r % 5 else 0  # every fifth row empty
        rows.append(sorted(rng.choice(nb, size=n, replace=False).tolist()))
    rp = np.cumsum([0] + [len(x) for x in rows]).astype(np.int32)
    ci = np.array([j for x in rows for j in x], dtype=np.int32)
    s = pu.shape_of(q, L, blk)
    o = pu.gpu_attention(s, q, k, v, torch.from_numpy(rp).cuda(),
                         torch.from_numpy(ci if ci.size else np.zeros(1, np.int32)).cuda())
    ref = oracle.attention(pu.bits(q), pu.bits(k), pu.bits(v), L, blk, rp, ci)
    pu.assert_attention_close(o, ref, "variable rows")
    for r, x in enumerate(rows):
        if not x:
            h, i = divmod(r, nb)
            assert torch.all(o[0, h, i * blk:(i + 1) * blk] == 0)
    sbsa.sbsa_check()


@pytest.mark.parametrize("d", [128, 64])
def test_attention_unsorted_and_repeated_lists(d):
    """Lists in any order, with repeats (a block listed twice counts twice, as in the
    oracle), at blocks of 128."""
    blk, H, nb = 128, 2, 7
    L = nb * blk - 3
    q, k, v = inputs.random_qkv(1, H, nb * blk, d, L=L, seed=38, device="cuda")
    rng = np.random.default_rng(39)
    rows = [rng.integers(0, nb, size=int(rng.integers(1, 9))).tolist() for _ in range(H * nb)]
    rp = np.cumsum([0] + [len(x) for x in rows]).astype(np.int32)
    ci = np.array([j for x in rows for j in x], dtype=np.int32)
    s = pu.shape_of(q, L, blk)
    o = pu.gpu_attention(s, q, k, v, torch.from_numpy(rp).cuda(), torch.from_numpy(ci).cuda())
    sbsa.sbsa_check()
    ref = oracle.attention(pu.bits(q), pu.bits(k), pu.bits(v), L, blk, rp, ci)
    pu.assert_attention_close(o, ref, "unsorted, repeated")


def test_attention_out_of_range_index_is_skipped_and_reported():
    d, blk, nb = 64, 64, 6
    L = nb * blk
    q, k, v = inputs.random_qkv(1, 1, L, d, seed=35, device="cuda")
    rows = [[0, 2], [1, 99], [2, -1, 4], [3], [4, 5], [5, 1000000]]
    rp = np.cumsum([0] + [len(x) for x in rows]).astype(np.int32)
    ci = np.array([j for x in rows for j in x], dtype=np.int32)
    s = pu.shape_of(q, L, blk)
    sbsa.sbsa_check()  # clear anything left over
    o = pu.gpu_attention(s, q, k, v, torch.from_numpy(rp).cuda(), torch.from_numpy(ci).cuda())
    with pytest.raises(sbsa.SbsaError) as e:
        sbsa.sbsa_check()
    assert e.value.status == 6
    clean = [[j for j in x if 0 <= j < nb] for x in rows]
    rp2 = np.cumsum([0] + [len(x) for x in clean]).astype(np.int32)
    ci2 = np.array([j for x in clean for j in x], dtype=np.int32)
    ref = oracle.attention(pu.bits(q), pu.bits(k), pu.bits(v), L, blk, rp2, ci2)
    pu.assert_attention_close(o, ref, "bad indices skipped")
    sbsa.sbsa_check()  # the word was cleared


# ---------------------------------------------------------------- fused forward

@pytest.mark.parametrize("wl_name", ["tiny"])
def test_forward_tiny_workload(wl_name):
    wl = inputs.WORKLOADS[wl_name]
    q, k, v = inputs.make_qkv(wl, seed=0, device="cuda")
    L, blk, nb = wl.seq_len, wl.block, wl.num_blocks
    kk = sbsa.sbsa_keep_blocks(nb, wl.keep)
    assert kk == 4
    s = pu.shape_of(q, L, blk)
    o = torch.empty_like(q)
    col = torch.empty(wl.heads * nb * kk, dtype=torch.int32, device="cuda")
    ws = sbsa.alloc_workspace(s, kk)
    sbsa.sbsa_forward(s, q, k, v, kk, 0.0, o, col, ws)
    sbsa.sbsa_check()
    ref_o, ref_col, qm, km = oracle.forward(pu.bits(q), pu.bits(k), pu.bits(v), L, blk, kk)
    gcol = col.cpu().numpy().reshape(1, wl.heads, nb, kk)
    pu.assert_selection_ok(gcol, ref_col, qm, km, kk)
    # attention given the GPU's (tie-equivalent) mask
    rp = oracle.uniform_row_ptr(1, wl.heads, nb, kk)
    ref = oracle.attention(pu.bits(q), pu.bits(k), pu.bits(v), L, blk, rp, gcol)
    pu.assert_attention_close(o, ref, "forward tiny")
    if np.array_equal(gcol, ref_col):
        pu.assert_attention_close(o, ref_o, "forward tiny vs oracle forward")


@pytest.mark.parametrize("d,blk,L,H,keep", [(128, 128, 3000, 3, 0.2), (64, 64, 2500, 2, 0.1),
                                            (128, 64, 1999, 2, 0.15)])
def test_forward_ragged_positional(d, blk, L, H, keep):
    wl = inputs.Workload("t", 1, H, (1, 1, L), d, blk, keep)
    q, k, v = inputs.make_qkv(wl, seed=3, device="cuda")
    nb = wl.num_blocks
    kk = sbsa.sbsa_keep_blocks(nb, keep)
    s = pu.shape_of(q, L, blk)
    o = torch.empty_like(q)
    col = torch.empty(H * nb * kk, dtype=torch.int32, device="cuda")
    sbsa.sbsa_forward(s, q, k, v, kk, 0.0, o, col, sbsa.alloc_workspace(s, kk))
    sbsa.sbsa_check()
    ref_o, ref_col, qm, km = oracle.forward(pu.bits(q), pu.bits(k), pu.bits(v), L, blk, kk)
    gcol = col.cpu().numpy().reshape(1, H, nb, kk)
    pu.assert_selection_ok(gcol, ref_col, qm, km, kk)
    rp = oracle.uniform_row_ptr(1, H, nb, kk)
    ref = oracle.attention(pu.bits(q), pu.bits(k), pu.bits(v), L, blk, rp, gcol)
    pu.assert_attention_close(o, ref, "forward ragged")


def test_forward_from_host_matches_device_path():
    wl = inputs.WORKLOADS["tiny"]
    q, k, v = inputs.make_qkv(wl, seed=1, device="cpu")
    qh, kh, vh = (t.pin_memory() for t in (q, k, v))
    s = sbsa.make_shape(1, wl.heads, wl.seq_len, wl.head_dim, wl.block)
    kk = sbsa.sbsa_keep_blocks(wl.num_blocks, wl.keep)
    oh = sbsa.forward_from_host(s, qh, kh, vh, kk)
    torch.cuda.synchronize()
    od = torch.empty_like(q, device="cuda")
    sbsa.sbsa_forward(s, q.cuda(), k.cuda(), v.cuda(), kk, 0.0, od, None, sbsa.alloc_workspace(s, kk))
    torch.cuda.synchronize()
    assert torch.equal(oh, od.cpu())
    assert math.isfinite(float(oh.float().abs().max()))


@pytest.mark.parametrize("head_chunk", [None, 1, 3, 10])
def test_forward_from_host_chunked_pipeline(head_chunk):
    """The copy/compute/copy pipeline over head chunks gives the one-call result bit for
    bit, also when the chunks do not divide the heads, and when called back to back."""
    B, H, L, d, blk = 2, 5, 700, 128, 128
    s = sbsa.make_shape(B, H, L, d, blk)
    q, k, v = inputs.random_qkv(B, H, s.seq_len_padded, d, L=L, seed=21)
    qh, kh, vh = (t.pin_memory() for t in (q, k, v))
    kk = sbsa.sbsa_keep_blocks(s.num_blocks, 0.5)
    od = torch.empty_like(q, device="cuda")
    sbsa.sbsa_forward(s, q.cuda(), k.cuda(), v.cuda(), kk, 0.0, od, None, sbsa.alloc_workspace(s, kk))
    bufs = (torch.empty_like(od), torch.empty_like(od), torch.empty_like(od), torch.empty_like(od),
            sbsa.alloc_workspace(s, kk))
    outs = [sbsa.forward_from_host(s, qh, kh, vh, kk, device_buffers=bufs, head_chunk=head_chunk) for _ in range(2)]
    torch.cuda.synchronize()
    sbsa.sbsa_check()
    ref = od.cpu()
    for oh in outs:
        assert torch.equal(oh, ref)


@pytest.mark.parametrize("d,blk", [(128, 128), (128, 64), (64, 64)])
def test_forward_batch_two(d, blk):
    """B = 2: sbsa_forward (pool, select, attention) over two batch entries of three heads
    against the oracle on the whole output, and sbsa_forward_host chunked over the six
    (batch, head) pairs bit-equal to it."""
    B, H = 2, 3
    L = 11 * blk - 9
    s = sbsa.make_shape(B, H, L, d, blk)
    q, k, v = inputs.random_qkv(B, H, s.seq_len_padded, d, L=L, seed=37)
    kk = sbsa.sbsa_keep_blocks(s.num_blocks, 0.3)
    o = torch.empty_like(q, device="cuda")
    col = torch.empty(B * H * s.num_blocks * kk, dtype=torch.int32, device="cuda")
    sbsa.sbsa_forward(s, q.cuda(), k.cuda(), v.cuda(), kk, 0.0, o, col, sbsa.alloc_workspace(s, kk))
    sbsa.sbsa_check()
    qb, kb, vb = pu.bits(q), pu.bits(k), pu.bits(v)
    qm, km = oracle.pool(qb, L, blk), oracle.pool(kb, L, blk)
    ref_col = oracle.select(qm, km, kk)
    pu.assert_selection_ok(col.cpu().numpy().reshape(ref_col.shape), ref_col, qm, km, kk)
    rp = oracle.uniform_row_ptr(B, H, s.num_blocks, kk)
    ref = oracle.attention(qb, kb, vb, L, blk, rp, col.cpu().numpy())
    pu.assert_attention_close(o, ref, "B = 2")
    oh = torch.empty(q.shape, dtype=torch.bfloat16).pin_memory()
    dq, dk, dv, do = (torch.empty_like(o) for _ in range(4))
    st = torch.cuda.current_stream()
    sbsa.sbsa_forward_host(s, q.pin_memory(), k.pin_memory(), v.pin_memory(), kk, 0.0, oh, dq, dk, dv, do,
                           sbsa.alloc_workspace(s, kk), pairs_per_chunk=2, stream=st,
                           h2d_stream=torch.cuda.Stream(), d2h_stream=torch.cuda.Stream())
    st.synchronize()
    sbsa.sbsa_check()
    assert torch.equal(oh, o.cpu())


@pytest.mark.parametrize("pinned,copy_streams", [(True, True), (False, False)])
def test_forward_host_entry_point(pinned, copy_streams):
    """sbsa_forward_host through the C ABI: pinned host memory with separate copy streams,
    and pageable host memory with every copy on the compute stream; both bit-equal to
    sbsa_forward, with the selection written nowhere else."""
    B, H, L, d, blk = 1, 6, 1500, 64, 64
    s = sbsa.make_shape(B, H, L, d, blk)
    q, k, v = inputs.random_qkv(B, H, s.seq_len_padded, d, L=L, seed=33)
    kk = sbsa.sbsa_keep_blocks(s.num_blocks, 0.3)
    od = torch.empty_like(q, device="cuda")
    sbsa.sbsa_forward(s, q.cuda(), k.cuda(), v.cuda(), kk, 0.0, od, None, sbsa.alloc_workspace(s, kk))
    hq, hk, hv = ((t.pin_memory() if pinned else t.clone()) for t in (q, k, v))
    oh = torch.full(q.shape, 3.0, dtype=torch.bfloat16, pin_memory=pinned)
    dq, dk, dv, do = (torch.empty_like(od) for _ in range(4))
    ws = sbsa.alloc_workspace(s, kk)
    side = (torch.cuda.Stream(), torch.cuda.Stream()) if copy_streams else (None, None)
    st = torch.cuda.current_stream()
    sbsa.sbsa_forward_host(s, hq, hk, hv, kk, 0.0, oh, dq, dk, dv, do, ws, pairs_per_chunk=4, stream=st,
                           h2d_stream=side[0], d2h_stream=side[1])
    st.synchronize()
    sbsa.sbsa_check()
    assert torch.equal(oh, od.cpu())
