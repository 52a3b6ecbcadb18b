"""The allocation-free forward entry point, checked against sbsa_forward.

sbsa_forward_noalloc serves callers that cannot call cudaMalloc -- a plug-in inside
an engine that owns all device memory, or a latency-critical loop where an allocation
would synchronize the device.  Its block means and block lists live in the library's
fixed 16 MiB scratch array instead of a caller workspace.  Here it must give the
same kept blocks and the same output (within the parity tolerance) as sbsa_forward,
on two calls in a row with different shapes and inputs, so that what the first call
leaves in the shared scratch cannot leak into the second; and it must refuse a shape
whose scratch need exceeds the array.

This file is named to be collected last."""
import ctypes

import pytest
import torch

from tests import parity_utils as pu
from video_dit_dynamic_b200 import inputs, sbsa

pytestmark = pytest.mark.gpu


def _run_both(wl, seed):
    q, k, v = inputs.make_qkv(wl, seed=seed, device="cuda")
    nb = wl.num_blocks
    kk = sbsa.sbsa_keep_blocks(nb, wl.keep)
    s = sbsa.make_shape(wl.batch, wl.heads, wl.seq_len, wl.head_dim, wl.block)
    assert sbsa.sbsa_workspace_bytes(s, kk) <= 16 << 20
    o_ref = torch.empty_like(q)
    col_ref = torch.empty(wl.batch * wl.heads * nb * kk, dtype=torch.int32, device="cuda")
    sbsa.sbsa_forward(s, q, k, v, kk, 0.0, o_ref, col_ref, sbsa.alloc_workspace(s, kk))
    o = torch.full_like(q, float("nan"))
    col = torch.full_like(col_ref, -1)
    sbsa.sbsa_forward_noalloc(s, q, k, v, kk, 0.0, o, col)
    sbsa.sbsa_check()
    return o, col, o_ref, col_ref


def test_noalloc_matches_forward_on_two_calls_in_a_row():
    pu.require_cuda()
    first = inputs.WORKLOADS["480p"]  # 40 heads x 256 blocks: 12.6 MB of scratch
    second = inputs.Workload("ragged", 1, 6, (1, 1, 4999), 64, 64, 0.15)
    for wl, seed in ((first, 0), (second, 1)):
        o, col, o_ref, col_ref = _run_both(wl, seed)
        assert torch.equal(col, col_ref), f"{wl.name}: kept blocks differ"
        pu.assert_attention_close(o, o_ref.double().cpu().numpy(), f"{wl.name}: noalloc vs forward")


def test_noalloc_rejects_shapes_beyond_its_scratch():
    pu.require_cuda()
    wl = inputs.WORKLOADS["720p"]  # needs about 26 MB of scratch
    s = sbsa.make_shape(wl.batch, wl.heads, wl.seq_len, wl.head_dim, wl.block)
    kk = sbsa.sbsa_keep_blocks(wl.num_blocks, wl.keep)
    assert sbsa.sbsa_workspace_bytes(s, kk) > 16 << 20
    x = torch.zeros(16, dtype=torch.bfloat16, device="cuda")  # never touched: rejected first
    lib = sbsa.load()
    st = lib.sbsa_forward_noalloc(ctypes.byref(s), x.data_ptr(), x.data_ptr(), x.data_ptr(), kk, 0.0,
                                  x.data_ptr(), None, None)
    assert st == 3  # SBSA_ERR_WORKSPACE
    with pytest.raises(sbsa.SbsaError) as e:
        sbsa._raise_on(st)
    assert "16777216" in str(e.value)
