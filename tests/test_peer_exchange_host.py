"""Host logic of the peer-put exchange (PeerExchange + LightUlysses steps), on the CPU.

The device calls are replaced by fakes over a simulated memory: a signal writes flag
words into every peer's allocation, a wait asserts that its flags already hold the
awaited epoch (the lockstep order must satisfy every wait with earlier launches), a put
records which writer's chunk sits in each slot of each peer's receive buffer, and an
unpack checks that it reads exactly the chunk the flags announced, from every writer.
"""
import pytest
import torch

from video_dit_dynamic_b200 import sbsa, ulysses


class FakeDevice:
    def __init__(self, exchanges):
        self.ex = exchanges
        self.flags = {}      # (rank, byte offset) -> value
        self.slots = {}      # (rank, exchange, buffer, writer) -> (chunk epoch, head0, count)
        self.last_wait = {}  # rank -> (flag byte offset, value) of its latest wait
        self.log = []

    def _owner(self, t):
        for r, e in enumerate(self.ex):
            base = e.local.data_ptr()
            if base <= t.data_ptr() < base + e.local.numel():
                return r, t.data_ptr() - base
        raise AssertionError("tensor outside every allocation")

    def signal(self, bases, flag_offset, rank, world, value, stream=None):
        for j in range(world):
            self.flags[(j, flag_offset + 4 * rank)] = value
        self.log.append(("signal", rank, flag_offset, value))

    def wait(self, flags, world, value, timeout_s=10.0, stream=None):
        r, off = self._owner(flags)
        for i in range(world):
            got = self.flags.get((r, off + 4 * i), 0)
            assert got == value, f"rank {r} waits for {value:#x} at flag {i}, finds {got:#x}"
        self.last_wait[r] = (off, value)

    def _put(self, exchange, shape, head0, n, src, bases, offset, rank, stream=None):
        e = self.ex[rank]
        buf = (e.qkv_off if exchange == 0 else e.o_off).index(offset)
        epoch = e._pending_epoch  # set by the wrapper below
        for j in range(shape.world):
            key = (j, exchange, buf, rank)
            prev = self.slots.get(key)
            if prev is not None:
                # the writer waited, just before, for every reader's acknowledgement of the
                # previous chunk in this buffer, and they have all acknowledged it
                assert self.last_wait.get(rank) == (e.flag_offset(exchange, buf, 1), prev[0])
                assert self.flags.get((rank, e.flag_offset(exchange, buf, 1) + 4 * j), 0) == prev[0]
            self.slots[key] = (epoch, head0, n)

    def _unpack(self, exchange, rank, recv, head0, n):
        e = self.ex[rank]
        r, off = self._owner(recv)
        assert r == rank
        buf = (e.qkv_off if exchange == 0 else e.o_off).index(off)
        want = e._pending_epoch
        # the reader waited, just before, for every writer's data flag of this chunk
        assert self.last_wait.get(rank) == (e.flag_offset(exchange, buf, 0), want)
        for writer in range(e.plan.world):
            assert self.slots[(rank, exchange, buf, writer)] == (want, head0, n)


@pytest.mark.parametrize("world,heads,head_chunk,calls", [(2, 4, 1, 2), (4, 8, 1, 1), (2, 6, 2, 3), (3, 3, 1, 2),
                                                             (2, 12, 1, 2), (3, 12, 1, 1)])
def test_lockstep_schedule_satisfies_every_wait_and_never_overwrites_unread_data(monkeypatch, world, heads,
                                                                                   head_chunk, calls):
    tokens = 8 * world
    plan = ulysses.UlyssesPlan(world, tokens, tokens, heads, 128, head_chunk)
    size = ulysses.PeerExchange.layout(plan)["total"]
    locals_ = [torch.zeros(size, dtype=torch.uint8) for _ in range(world)]
    bases = torch.tensor([t.data_ptr() for t in locals_], dtype=torch.int64)
    exs = [ulysses.PeerExchange(plan, locals_[r], bases, r) for r in range(world)]
    dev = FakeDevice(exs)

    # epochs reach the fakes through the exchange object (send/recv pass them to signal/wait)
    orig_send, orig_recv = ulysses.PeerExchange.send, ulysses.PeerExchange.recv

    def send(self, exchange, chunk, h0, n, src, epoch):
        self._pending_epoch = epoch
        return orig_send(self, exchange, chunk, h0, n, src, epoch)

    def recv(self, exchange, chunk, h0, n, dst, epoch):
        self._pending_epoch = epoch
        return orig_recv(self, exchange, chunk, h0, n, dst, epoch)

    monkeypatch.setattr(ulysses.PeerExchange, "send", send)
    monkeypatch.setattr(ulysses.PeerExchange, "recv", recv)
    monkeypatch.setattr(sbsa, "sbsa_peer_signal", dev.signal)
    monkeypatch.setattr(sbsa, "sbsa_peer_wait", dev.wait)
    monkeypatch.setattr(sbsa, "sbsa_ulysses_put_qkv",
                        lambda shape, h0, n, src, b, off, rank, stream=None: dev._put(0, shape, h0, n, src, b, off, rank))
    monkeypatch.setattr(sbsa, "sbsa_ulysses_put_o",
                        lambda shape, h0, n, src, b, off, rank, stream=None: dev._put(1, shape, h0, n, src, b, off, rank))

    class Ops:
        def __init__(self, rank):
            self.rank = rank

        def attend(self, h0, n, q, k, v, o):
            pass

    layers = [ulysses.LightUlysses(plan, device="cpu", ops=Ops(r), exchange=exs[r]) for r in range(world)]

    def unpack_qkv(shape, h0, n, recv_t, q, k, v, stream=None):
        dev._unpack(0, dev._owner(recv_t)[0], recv_t, h0, n)

    def unpack_o(shape, h0, n, recv_t, y, stream=None):
        dev._unpack(1, dev._owner(recv_t)[0], recv_t, h0, n)

    monkeypatch.setattr(sbsa, "sbsa_ulysses_unpack_qkv", unpack_qkv)
    monkeypatch.setattr(sbsa, "sbsa_ulysses_unpack_o", unpack_o)
    xs = [torch.zeros(plan.tokens_local, 3, heads, 128, dtype=torch.bfloat16) for _ in range(world)]
    for _ in range(calls):  # later calls reuse the buffers across the call boundary
        ulysses.lockstep_forward(layers, xs)
    n_chunks = len(plan.chunks())
    # every chunk was signalled twice per exchange kind (data and ack) by every rank
    assert sum(1 for e in dev.log if e[0] == "signal") == calls * n_chunks * 2 * 2 * world


def test_steps_cover_every_chunk_in_order():
    plan = ulysses.UlyssesPlan(2, 16, 16, 8, 128, 1)  # 4 chunks
    layer = ulysses.LightUlysses.__new__(ulysses.LightUlysses)
    layer.plan = plan
    steps = layer.steps()
    n = len(plan.chunks())
    for kind in ("send_qkv", "recv_qkv", "attend", "send_o", "recv_o"):
        assert [c for k, c in steps if k == kind] == list(range(n))
    pos = {s: i for i, s in enumerate(steps)}
    for c in range(n):
        assert pos[("send_qkv", c)] < pos[("recv_qkv", c)] < pos[("attend", c)] < pos[("send_o", c)] < pos[("recv_o", c)]
        if c + 1 < n:
            assert pos[("send_qkv", c + 1)] < pos[("attend", c)]  # the next exchange overlaps this attention


def test_layers_sharing_an_exchange_get_distinct_epochs(monkeypatch):
    """Two layers over one allocation: the second layer's chunks must not match the first
    layer's flags (the call counter lives in the exchange)."""
    plan = ulysses.UlyssesPlan(1, 8, 8, 2, 128, 1)
    size = ulysses.PeerExchange.layout(plan)["total"]
    ex = ulysses.PeerExchange(plan, torch.zeros(size, dtype=torch.uint8), torch.zeros(1, dtype=torch.int64), 0)
    seen = []
    monkeypatch.setattr(ulysses.PeerExchange, "send", lambda self, e, c, h0, n, src, epoch: seen.append((e, epoch)))
    monkeypatch.setattr(ulysses.PeerExchange, "recv", lambda self, e, c, h0, n, dst, epoch: None)

    class Ops:
        def attend(self, *a):
            pass

    a = ulysses.LightUlysses(plan, device="cpu", ops=Ops(), exchange=ex)
    b = ulysses.LightUlysses(plan, device="cpu", ops=Ops(), exchange=ex)
    x = torch.zeros(8, 3, 2, 128, dtype=torch.bfloat16)
    a.forward(x)
    b.forward(x)
    a.forward(x)
    # the two exchanges keep separate flags; within each, every epoch is new
    assert len(seen) == len(set(seen)) == 3 * 2 * 2  # 3 calls x 2 chunks x (qkv, o)
    other = ulysses.UlyssesPlan(1, 8, 8, 2, 128, 2)
    with pytest.raises(ValueError):
        ulysses.LightUlysses(other, device="cpu", ops=Ops(), exchange=ex)
