"""Light-Ulysses orchestration on two real processes (gloo, CPU).

`LightUlysses` drives the head-level pipeline: pack -> asynchronous all-to-all ->
unpack -> attend -> pack -> all-to-all back -> unpack, two exchange buffers of each
kind in flight.  Here its kernels are replaced, in the test only, by the oracle's
arithmetic on CPU tensors, so two gloo ranks run the real buffer handling, chunking,
ordering and collectives, and the result must equal the oracle's layer exactly.
"""
import datetime
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _u16(t):
    return t.view(torch.int16).numpy().view(np.uint16)


class OracleOps:
    """The five per-rank operations of LightUlysses written with the oracle on CPU tensors
    (test double; the library's CudaOps run them on the GPU)."""

    def __init__(self, plan, block):
        import oracle
        self.o_ = oracle
        self.p = plan
        self.block = block

    def _slices(self, buf, slice_bytes, rows, d):
        G = self.p.world
        a = buf.numpy()
        for j in range(G):
            base = j * slice_bytes
            codes = a[base:base + rows * d].reshape(rows, d)
            scales = a[base + rows * d:base + rows * (d + 4)].view(np.float32)
            yield j, codes, scales

    def pack_qkv(self, h0, n, x, send):
        p, d = self.p, self.p.head_dim
        xb = _u16(x)  # [Lr, 3, H, d]
        rows = p.tokens_local * 3 * n
        for j, codes, scales in self._slices(send, p.qkv_slice_bytes(n), rows, d):
            hs = slice(j * p.heads_local + h0, j * p.heads_local + h0 + n)
            c, s = self.o_.quantize_rows_fp8(np.ascontiguousarray(xb[:, :, hs, :]).reshape(rows, d))
            codes[:] = c
            scales[:] = s

    def unpack_qkv(self, h0, n, recv, q, k, v):
        p, d = self.p, self.p.head_dim
        rows = p.tokens_local * 3 * n
        outs = [_u16(q), _u16(k), _u16(v)]
        for i, codes, scales in self._slices(recv, p.qkv_slice_bytes(n), rows, d):
            deq = self.o_.dequantize_rows_bf16(codes, scales).reshape(p.tokens_local, 3, n, d)
            for c in range(3):
                outs[c][h0:h0 + n, i * p.tokens_local:(i + 1) * p.tokens_local] = deq[:, c].transpose(1, 0, 2)
        for t in outs:
            t[h0:h0 + n, p.tokens:] = 0

    def attend(self, h0, n, q, k, v, o):
        p, blk = self.p, self.block
        nb = p.tokens_padded // blk
        rp = self.o_.uniform_row_ptr(1, n, nb, nb)
        col = np.broadcast_to(np.arange(nb, dtype=np.int32), (1, n, nb, nb)).copy()
        res = self.o_.attention(_u16(q)[None, h0:h0 + n].copy(), _u16(k)[None, h0:h0 + n].copy(),
                                _u16(v)[None, h0:h0 + n].copy(), p.tokens, blk, rp, col)[0]
        _u16(o)[h0:h0 + n] = self.o_.bf16_round(res)

    def pack_o(self, h0, n, o, send):
        p, d = self.p, self.p.head_dim
        ob = _u16(o)
        rows = p.tokens_local * n
        for j, codes, scales in self._slices(send, p.o_slice_bytes(n), rows, d):
            blk = ob[h0:h0 + n, j * p.tokens_local:(j + 1) * p.tokens_local].transpose(1, 0, 2)
            c, s = self.o_.quantize_rows_fp8(np.ascontiguousarray(blk).reshape(rows, d))
            codes[:] = c
            scales[:] = s

    def unpack_o(self, h0, n, recv, y):
        p, d = self.p, self.p.head_dim
        rows = p.tokens_local * n
        yb = _u16(y)
        for i, codes, scales in self._slices(recv, p.o_slice_bytes(n), rows, d):
            deq = self.o_.dequantize_rows_bf16(codes, scales).reshape(p.tokens_local, n, d)
            yb[:, i * p.heads_local + h0:i * p.heads_local + h0 + n] = deq


G, L, LP, H, D, BLK = 2, 96, 128, 4, 128, 32


def _layer_input():
    g = torch.Generator().manual_seed(77)
    return (torch.randn(L, 3, H, D, generator=g) * 0.7).to(torch.bfloat16)


def _rank_main(rank, world, port, head_chunk, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    from video_dit_dynamic_b200 import ulysses
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        plan = ulysses.UlyssesPlan(world=world, tokens=L, tokens_padded=LP, heads=H, head_dim=D, head_chunk=head_chunk)
        lu = ulysses.LightUlysses(plan, group=dist.group.WORLD, device="cpu", ops=OracleOps(plan, BLK))
        x = _layer_input()[rank * (L // world):(rank + 1) * (L // world)].contiguous()
        y = lu.forward(x)
        out.put((rank, _u16(y).copy()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("head_chunk", [2, 1])
def test_two_rank_light_ulysses_matches_oracle_layer(head_chunk):
    import oracle
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, G, port, head_chunk, q)) for r in range(G)]
    for p in procs:
        p.start()
    results = dict(q.get(timeout=240) for _ in range(G))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # the oracle's layer: exchange, dense attention per rank, bf16, return exchange
    x = _layer_input()
    shards = [_u16(x[r * (L // G):(r + 1) * (L // G)].contiguous()) for r in range(G)]
    qkv = oracle.ulysses_qkv(shards, H, L, LP)
    nb = LP // BLK
    o = []
    for r in range(G):
        rp = oracle.uniform_row_ptr(1, H // G, nb, nb)
        col = np.broadcast_to(np.arange(nb, dtype=np.int32), (1, H // G, nb, nb)).copy()
        res = oracle.attention(qkv[r][0][None], qkv[r][1][None], qkv[r][2][None], L, BLK, rp, col)[0]
        o.append(oracle.bf16_round(res))
    y_ref = oracle.ulysses_o(o, H, L)
    for r in range(G):
        np.testing.assert_array_equal(results[r], y_ref[r])
