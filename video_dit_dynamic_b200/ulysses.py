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

Two exchanges: NCCL's all_to_all_single of packed send buffers, or `PeerExchange`, where
the packing kernel writes every peer's slice straight into that peer's receive buffer in
peer-mapped (symmetric) memory and raises a flag there; the receiver waits for all of its
flags on the device, unpacks, and acknowledges, so that a buffer is rewritten only after
every peer has read it.
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


class PeerExchange:
    """Receive buffers and flags of the peer-put exchange, for one rank.

    One allocation per rank, with the same layout on every rank (byte offsets, each a
    multiple of 16):
      qkv receive buffers  [2][world * qkv slice]  (chunk c uses buffer c % 2)
      o receive buffers    [2][world * o slice]
      flags                uint32 [2 exchanges (qkv, o)][2 buffers][2 kinds (data, ack)][world]
    `local` is this rank's allocation (uint8 CUDA tensor, flags zero at start) and `bases`
    an int64 CUDA tensor of the world's allocation addresses as mapped on this rank.
    Flag values are epochs: (call << 16) + chunk + 1, never 0 and never repeated."""

    def __init__(self, plan: UlyssesPlan, local: torch.Tensor, bases: torch.Tensor, rank: int,
                 timeout_s: float = 10.0, keepalive=None):
        self.plan = plan
        self.rank = rank
        self.local = local
        self.bases = bases
        self.timeout_s = timeout_s
        self._keepalive = keepalive  # the symmetric-memory handle, if any
        lay = self.layout(plan)
        if local.numel() < lay["total"]:
            raise ValueError("exchange allocation too small")
        self.qkv_off, self.o_off, self.flag_off = lay["qkv"], lay["o"], lay["flags"]
        self.full = sbsa.make_ulysses_shape(plan.world, plan.tokens, plan.tokens_padded, plan.heads, plan.head_dim)
        self.last_epoch = {}  # (exchange, buffer) -> epoch of the buffer's last write
        self.calls = 0        # forwards through this allocation, by every layer that uses it

    def new_call(self) -> int:
        """The number of the next forward through this allocation: epochs stay distinct when
        several layers share it (every rank counts the same calls in the same order)."""
        self.calls += 1
        return self.calls

    @staticmethod
    def layout(plan: UlyssesPlan) -> dict:
        hc, w = plan.head_chunk, plan.world
        qkv_b = w * plan.qkv_slice_bytes(hc)
        o_b = w * plan.o_slice_bytes(hc)
        qkv = [0, qkv_b]
        o = [2 * qkv_b, 2 * qkv_b + o_b]
        flags = 2 * qkv_b + 2 * o_b
        return {"qkv": qkv, "o": o, "flags": flags, "total": flags + 2 * 2 * 2 * w * 4}

    def flag_offset(self, exchange: int, buf: int, kind: int) -> int:
        return self.flag_off + ((exchange * 2 + buf) * 2 + kind) * self.plan.world * 4

    def _flags(self, exchange: int, buf: int, kind: int) -> torch.Tensor:
        o = self.flag_offset(exchange, buf, kind)
        return self.local[o:o + 4 * self.plan.world].view(torch.int32)

    def _recv(self, exchange: int, buf: int, count: int) -> torch.Tensor:
        p = self.plan
        size = p.world * (p.qkv_slice_bytes(count) if exchange == 0 else p.o_slice_bytes(count))
        o = (self.qkv_off if exchange == 0 else self.o_off)[buf]
        return self.local[o:o + size]

    def send(self, exchange: int, chunk: int, h0: int, n: int, src: torch.Tensor, epoch: int):
        """Pack `src` (x for qkv, o for the output) into every peer's buffer chunk % 2, after
        every peer has read what was last written there, then raise the data flags."""
        p, b = self.plan, chunk % 2
        prev = self.last_epoch.get((exchange, b))
        if prev is not None:
            sbsa.sbsa_peer_wait(self._flags(exchange, b, 1), p.world, prev, self.timeout_s)
        off = (self.qkv_off if exchange == 0 else self.o_off)[b]
        put = sbsa.sbsa_ulysses_put_qkv if exchange == 0 else sbsa.sbsa_ulysses_put_o
        put(self.full, h0, n, src, self.bases, off, self.rank)
        sbsa.sbsa_peer_signal(self.bases, self.flag_offset(exchange, b, 0), self.rank, p.world, epoch)
        self.last_epoch[(exchange, b)] = epoch

    def recv(self, exchange: int, chunk: int, h0: int, n: int, dst, epoch: int):
        """Wait for every peer's slice of chunk `chunk`, unpack it into `dst` ((q, k, v) or y)
        and acknowledge to every peer."""
        p, b = self.plan, chunk % 2
        sbsa.sbsa_peer_wait(self._flags(exchange, b, 0), p.world, epoch, self.timeout_s)
        if exchange == 0:
            sbsa.sbsa_ulysses_unpack_qkv(self.full, h0, n, self._recv(0, b, n), *dst)
        else:
            sbsa.sbsa_ulysses_unpack_o(self.full, h0, n, self._recv(1, b, n), dst)
        sbsa.sbsa_peer_signal(self.bases, self.flag_offset(exchange, b, 1), self.rank, p.world, epoch)

    @classmethod
    def from_symmetric_memory(cls, plan: UlyssesPlan, group, device, timeout_s: float = 10.0) -> "PeerExchange":
        """The allocation in torch's symmetric memory (peer-mapped over NVLink), one per rank
        of `group`; collective: every rank of the group calls it."""
        import torch.distributed._symmetric_memory as symm_mem
        group = group if group is not None else dist.group.WORLD
        if hasattr(symm_mem, "enable_symm_mem_for_group"):
            symm_mem.enable_symm_mem_for_group(group.group_name)
        local = symm_mem.empty(cls.layout(plan)["total"], dtype=torch.uint8, device=device)
        local.zero_()
        handle = symm_mem.rendezvous(local, group)
        bases = torch.tensor([int(a) for a in handle.buffer_ptrs], dtype=torch.int64, device=device)
        torch.cuda.synchronize(device)
        dist.barrier(group=group)  # every rank's flags are zero before any rank signals
        return cls(plan, local, bases, dist.get_rank(group), timeout_s, keepalive=handle)

    @classmethod
    def emulated(cls, plan: UlyssesPlan, device, timeout_s: float = 10.0) -> list:
        """`world` exchanges whose allocations are buffers of this one GPU, for running every
        rank in one process with `lockstep_forward` (no rank ever waits for a later launch)."""
        size = cls.layout(plan)["total"]
        locals_ = [torch.zeros(size, dtype=torch.uint8, device=device) for _ in range(plan.world)]
        bases = torch.tensor([t.data_ptr() for t in locals_], dtype=torch.int64, device=device)
        return [cls(plan, locals_[r], bases, r, timeout_s) for r in range(plan.world)]


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
    runs a single rank without a collective.  With `exchange` (a PeerExchange) the
    exchanges are peer puts instead of NCCL all-to-alls."""

    def __init__(self, plan: UlyssesPlan, group=None, device=None, block: int = 128, keep: float = 0.1,
                 scale: float = 0.0, ops=None, dtype=torch.bfloat16, exchange: PeerExchange | None = None):
        self.plan = plan
        self.group = group
        self.peer = exchange
        self._call = 0
        if exchange is not None and exchange.plan != plan:
            raise ValueError("the exchange was laid out for another plan")
        if exchange is None:
            if group is not None and dist.get_world_size(group) != plan.world:
                raise ValueError("plan.world differs from the group's size")
            if group is None and plan.world != 1:
                raise ValueError("a world larger than 1 needs a process group or a PeerExchange")
        self.device = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
        self.ops = ops if ops is not None else CudaOps(plan, block, keep, scale, self.device)
        hc = plan.head_chunk
        u8 = dict(dtype=torch.uint8, device=self.device)
        if exchange is None:
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

    def steps(self):
        """The schedule of one forward: (step, chunk) in launch order.  Chunk c + 1's QKV
        exchange is started before chunk c is attended; chunk c - 1's output is received
        after chunk c is attended."""
        n = len(self.plan.chunks())
        out = [("send_qkv", 0)]
        for ci in range(n):
            if ci + 1 < n:
                out.append(("send_qkv", ci + 1))
            out += [("recv_qkv", ci), ("attend", ci)]
            if ci >= 1:
                out.append(("recv_o", ci - 1))
            out.append(("send_o", ci))
        out.append(("recv_o", n - 1))
        return out

    def begin(self, x, y=None):
        p = self.plan
        if y is None:
            y = torch.empty((p.tokens_local, p.heads, p.head_dim), dtype=x.dtype, device=x.device)
        self._x, self._y = x, y
        self._call = self.peer.new_call() if self.peer is not None else self._call + 1
        self._pending = {}
        return y

    def run(self, step: str, ci: int):
        p = self.plan
        h0, n = p.chunks()[ci]
        b = ci % 2
        epoch = ((self._call & 0xFFFF) << 16) + ci + 1
        if step == "attend":
            self.ops.attend(h0, n, self.q, self.k, self.v, self.o)
        elif self.peer is not None:
            if step == "send_qkv":
                self.peer.send(0, ci, h0, n, self._x, epoch)
            elif step == "recv_qkv":
                self.peer.recv(0, ci, h0, n, (self.q, self.k, self.v), epoch)
            elif step == "send_o":
                self.peer.send(1, ci, h0, n, self.o, epoch)
            else:
                self.peer.recv(1, ci, h0, n, self._y, epoch)
        elif step == "send_qkv":
            self.ops.pack_qkv(h0, n, self._x, self.send_qkv[b])
            self._pending[("qkv", ci)] = self._exchange(self.recv_qkv[b], self.send_qkv[b],
                                                        p.world * p.qkv_slice_bytes(n))
        elif step == "recv_qkv":
            self._pending.pop(("qkv", ci)).wait()
            self.ops.unpack_qkv(h0, n, self.recv_qkv[b], self.q, self.k, self.v)
        elif step == "send_o":
            self.ops.pack_o(h0, n, self.o, self.send_o[b])
            self._pending[("o", ci)] = self._exchange(self.recv_o[b], self.send_o[b], p.world * p.o_slice_bytes(n))
        else:
            # the exchange of chunk ci must end before its buffers are reused (chunk ci + 2)
            self._pending.pop(("o", ci)).wait()
            self.ops.unpack_o(h0, n, self.recv_o[b], self._y)

    def forward(self, x, y=None):
        y = self.begin(x, y)
        for step, ci in self.steps():
            self.run(step, ci)
        return y


def lockstep_forward(layers, xs, ys=None):
    """Every rank's forward in one process, step by step across the ranks (rank 0's step,
    rank 1's step, ..., then the next step): the ranks of `PeerExchange.emulated` on one
    GPU, where each wait is already satisfied by earlier launches on the stream."""
    ys = [layer.begin(x, None if ys is None else ys[r]) for r, (layer, x) in enumerate(zip(layers, xs))]
    for step, ci in layers[0].steps():
        for layer in layers:
            layer.run(step, ci)
    return ys
