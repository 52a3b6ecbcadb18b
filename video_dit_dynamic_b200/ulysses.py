"""Light-Ulysses: Ulysses-style sequence parallelism around the sparse attention.

Page "知识卡片：600倍加速，720p视频实时生成！单卡也能带的动14B模型", 方法/产品要点, bullet
Light-Ulysses 多卡并行, and page "单卡 RTX 5090 跑 Wan2.2-A14B：720p 视频生成只要 3.8 秒",
四步拆解 item 4: FP8 communication, Q, K and V fused into one all-to-all, fused pre- and
post-processing kernels, and a head-level asynchronous pipeline.

One process per GPU.  Rank r holds a contiguous shard of L/G tokens of the fused QKV
activation, [L/G, 3, H, d] (the QKV projection's output).  `LightUlysses.forward` runs,
for each chunk of heads:

  pack   (library kernel: rows -> e4m3 codes + one scale each, ordered by peer)
  all-to-all over NCCL, asynchronous
  unpack (library kernel: -> q, k, v of this rank's heads in the attention's layout)
  the sparse attention on this chunk's heads (pool -> select -> attend)
  pack the output, all-to-all back, unpack into [L/G, H, d]

and the exchange of chunk c + 1 is in flight while chunk c is attended.  The kernels are
in the sbsa library; this module holds buffers, the order of the steps and the
collective calls.  Tokens and heads must divide by the world size.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch
import torch.distributed as dist

from . import sbsa


class _Done:
    def wait(self):
        return None


@dataclass
class UlyssesPlan:
    """Sizes of one Light-Ulysses layer on `world` ranks."""
    world: int
    tokens: int
    tokens_padded: int
    heads: int
    head_dim: int
    head_chunk: int

    def __post_init__(self):
        if self.tokens % self.world or self.heads % self.world:
            raise ValueError("tokens and heads must be multiples of the world size")
        if self.tokens_padded < self.tokens:
            raise ValueError("tokens_padded < tokens")
        hg = self.heads // self.world
        if not 1 <= self.head_chunk <= hg:
            raise ValueError(f"head_chunk must be in [1, {hg}]")

    @property
    def tokens_local(self) -> int:
        return self.tokens // self.world

    @property
    def heads_local(self) -> int:
        return self.heads // self.world

    def chunks(self):
        """(head0, count) of every step of the head-level pipeline."""
        hg = self.heads_local
        return [(h0, min(self.head_chunk, hg - h0)) for h0 in range(0, hg, self.head_chunk)]

    def qkv_slice_bytes(self, count: int) -> int:
        # codes then scales, padded to 16 bytes (the library's slice layout)
        return (self.tokens_local * 3 * count * (self.head_dim + 4) + 15) // 16 * 16

    def o_slice_bytes(self, count: int) -> int:
        return (self.tokens_local * count * (self.head_dim + 4) + 15) // 16 * 16


class CudaOps:
    """The library kernels for one rank: pack/unpack of both exchanges and the sparse
    attention on a chunk of this rank's heads."""

    def __init__(self, plan: UlyssesPlan, block: int, keep: float, scale: float, device):
        self.plan = plan
        self.block = block
        self.scale = scale
        self.full = sbsa.make_ulysses_shape(plan.world, plan.tokens, plan.tokens_padded, plan.heads, plan.head_dim)
        self.nb = plan.tokens_padded // block
        self.k_keep = sbsa.sbsa_keep_blocks(self.nb, keep)
        shape = sbsa.make_shape(1, plan.head_chunk, plan.tokens, plan.head_dim, block, plan.tokens_padded)
        self.workspace = sbsa.alloc_workspace(shape, self.k_keep, device=device)

    def pack_qkv(self, h0, n, x, send):
        sbsa.sbsa_ulysses_pack_qkv(self.full, h0, n, x, send)

    def unpack_qkv(self, h0, n, recv, q, k, v):
        sbsa.sbsa_ulysses_unpack_qkv(self.full, h0, n, recv, q, k, v)

    def pack_o(self, h0, n, o, send):
        sbsa.sbsa_ulysses_pack_o(self.full, h0, n, o, send)

    def unpack_o(self, h0, n, recv, y):
        sbsa.sbsa_ulysses_unpack_o(self.full, h0, n, recv, y)

    def attend(self, h0, n, q, k, v, o):
        p = self.plan
        shape = sbsa.make_shape(1, n, p.tokens, p.head_dim, self.block, p.tokens_padded)
        sbsa.sbsa_forward(shape, q[h0:h0 + n], k[h0:h0 + n], v[h0:h0 + n], self.k_keep, self.scale,
                          o[h0:h0 + n], None, self.workspace)


class LightUlysses:
    """Sequence-parallel sparse attention of one layer on every rank of `group`.

    forward(x) takes this rank's [L/G, 3, H, d] bf16 activation and returns its
    [L/G, H, d] attention output.  `ops` defaults to the library kernels; `group=None`
    runs a single rank without a collective."""

    def __init__(self, plan: UlyssesPlan, group=None, device=None, block: int = 128, keep: float = 0.1,
                 scale: float = 0.0, ops=None, dtype=torch.bfloat16):
        self.plan = plan
        self.group = group
        if group is not None and dist.get_world_size(group) != plan.world:
            raise ValueError("plan.world differs from the group's size")
        if group is None and plan.world != 1:
            raise ValueError("a world larger than 1 needs a process group")
        self.device = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
        self.ops = ops if ops is not None else CudaOps(plan, block, keep, scale, self.device)
        hc = plan.head_chunk
        u8 = dict(dtype=torch.uint8, device=self.device)
        # two of each exchange buffer: one chunk in flight while the other is consumed
        self.send_qkv = [torch.empty(plan.world * plan.qkv_slice_bytes(hc), **u8) for _ in range(2)]
        self.recv_qkv = [torch.empty_like(b) for b in self.send_qkv]
        self.send_o = [torch.empty(plan.world * plan.o_slice_bytes(hc), **u8) for _ in range(2)]
        self.recv_o = [torch.empty_like(b) for b in self.send_o]
        att = (plan.heads_local, plan.tokens_padded, plan.head_dim)
        self.q, self.k, self.v, self.o = (torch.empty(att, dtype=dtype, device=self.device) for _ in range(4))

    def _exchange(self, recv, send, nbytes):
        if self.group is None:
            recv[:nbytes].copy_(send[:nbytes])
            return _Done()
        return dist.all_to_all_single(recv[:nbytes], send[:nbytes], group=self.group, async_op=True)

    def forward(self, x, y=None):
        p = self.plan
        if y is None:
            y = torch.empty((p.tokens_local, p.heads, p.head_dim), dtype=x.dtype, device=x.device)
        chunks = p.chunks()
        pending = {}

        def start(ci):
            h0, n = chunks[ci]
            b = ci % 2
            self.ops.pack_qkv(h0, n, x, self.send_qkv[b])
            pending[ci] = self._exchange(self.recv_qkv[b], self.send_qkv[b], p.world * p.qkv_slice_bytes(n))

        out_pending = None
        start(0)
        for ci, (h0, n) in enumerate(chunks):
            b = ci % 2
            if ci + 1 < len(chunks):
                start(ci + 1)  # the next chunk crosses while this one is attended
            pending.pop(ci).wait()
            self.ops.unpack_qkv(h0, n, self.recv_qkv[b], self.q, self.k, self.v)
            self.ops.attend(h0, n, self.q, self.k, self.v, self.o)
            if out_pending is not None:
                # the previous chunk's output exchange must end before its buffers are reused
                pci, ph0, pn, handle = out_pending
                handle.wait()
                self.ops.unpack_o(ph0, pn, self.recv_o[pci % 2], y)
            self.ops.pack_o(h0, n, self.o, self.send_o[b])
            out_pending = (ci, h0, n, self._exchange(self.recv_o[b], self.send_o[b], p.world * p.o_slice_bytes(n)))
        pci, ph0, pn, handle = out_pending
        handle.wait()
        self.ops.unpack_o(ph0, pn, self.recv_o[pci % 2], y)
        return y
