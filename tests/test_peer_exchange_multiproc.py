"""The peer-put exchange's schedule with every rank in its own process, on the CPU.

Each process runs its own LightUlysses.forward (not lockstep), as ranks on separate GPUs
do; the device calls are replaced by fakes over shared memory: a signal writes flag words
into the peers' flag arrays, a wait blocks until its flags hold the epoch (or fails after
a timeout), a put stamps (writer, epoch) markers into every peer's receive slots and an
unpack checks that each slot holds this chunk's marker from every writer.  Finishing
without a timeout shows the schedule is free of cross-rank deadlock; the markers show no
buffer is read before it is written or rewritten before it is read.
"""
import multiprocessing as mp
import time

import numpy as np
import pytest

N_FLAGS = 2 * 2 * 2  # exchanges x buffers x kinds


def _rank_main(rank, world, heads, head_chunk, calls, shm_name, out):
    import torch

    from multiprocessing import shared_memory
    from video_dit_dynamic_b200 import sbsa, ulysses

    shm = shared_memory.SharedMemory(name=shm_name)
    try:
        # flags[r][kind_index][writer], slots[r][exchange][buffer][writer] (epochs)
        flags = np.ndarray((world, N_FLAGS, world), dtype=np.uint32, buffer=shm.buf, offset=0)
        slots = np.ndarray((world, 2, 2, world), dtype=np.uint32, buffer=shm.buf, offset=flags.nbytes)
        ready = np.ndarray((world,), dtype=np.uint32, buffer=shm.buf, offset=flags.nbytes + slots.nbytes)
        tokens = 8 * world
        plan = ulysses.UlyssesPlan(world, tokens, tokens, heads, 128, head_chunk)
        size = ulysses.PeerExchange.layout(plan)["total"]
        local = torch.zeros(size, dtype=torch.uint8)
        ex = ulysses.PeerExchange(plan, local, torch.zeros(world, dtype=torch.int64), rank)

        def index_of(flag_offset):
            k = (flag_offset - ex.flag_off) // (4 * world)
            assert 0 <= k < N_FLAGS and ex.flag_off + k * 4 * world == flag_offset
            return k

        def signal(bases, flag_offset, r, w, value, stream=None):
            k = index_of(flag_offset)
            for j in range(w):
                flags[j, k, r] = value

        def wait(flag_view, w, value, timeout_s=10.0, stream=None):
            k = index_of(flag_view.data_ptr() - local.data_ptr())
            t0 = time.monotonic()
            while not np.all(flags[rank, k] == value):
                if time.monotonic() - t0 > 60.0:
                    raise TimeoutError(f"rank {rank} waits on flag set {k} for {value:#x}: {flags[rank, k]}")
                time.sleep(0.0005)

        state = {}

        def put(exchange):
            def f(shape, h0, n, src, bases, offset, r, stream=None):
                b = (ex.qkv_off if exchange == 0 else ex.o_off).index(offset)
                for j in range(world):
                    slots[j, exchange, b, r] = state["epoch"]
            return f

        def unpack(exchange):
            def f(shape, h0, n, recv, *dst, stream=None):
                b = (ex.qkv_off if exchange == 0 else ex.o_off).index(recv.data_ptr() - local.data_ptr())
                # a slow reader: a writer that did not wait for its acknowledgement overwrites
                # the slots in the meantime
                time.sleep(0.003 * ((rank + state["epoch"]) % 2))
                got = slots[rank, exchange, b].copy()
                assert np.all(got == state["epoch"]), f"rank {rank} reads {got}, wants {state['epoch']:#x}"
            return f

        orig_send, orig_recv = ulysses.PeerExchange.send, ulysses.PeerExchange.recv

        def send(self, exchange, chunk, h0, n, src, epoch):
            state["epoch"] = epoch
            return orig_send(self, exchange, chunk, h0, n, src, epoch)

        def recv(self, exchange, chunk, h0, n, dst, epoch):
            state["epoch"] = epoch
            return orig_recv(self, exchange, chunk, h0, n, dst, epoch)

        ulysses.PeerExchange.send, ulysses.PeerExchange.recv = send, recv
        sbsa.sbsa_peer_signal, sbsa.sbsa_peer_wait = signal, wait
        sbsa.sbsa_ulysses_put_qkv, sbsa.sbsa_ulysses_put_o = put(0), put(1)
        sbsa.sbsa_ulysses_unpack_qkv, sbsa.sbsa_ulysses_unpack_o = unpack(0), unpack(1)

        class Ops:
            def attend(self, h0, n, q, k, v, o):
                time.sleep(0.001 * ((rank + h0) % 3))  # ranks drift apart

        layer = ulysses.LightUlysses(plan, device="cpu", ops=Ops(), exchange=ex)
        x = torch.zeros(plan.tokens_local, 3, heads, 128, dtype=torch.bfloat16)
        # start together: process start-up (imports) must not count against the waits
        ready[rank] = 1
        t0 = time.monotonic()
        while not np.all(ready == 1):
            if time.monotonic() - t0 > 300.0:
                raise TimeoutError("not every rank started")
            time.sleep(0.001)
        for _ in range(calls):
            layer.forward(x)
        out.put((rank, "ok"))
    except BaseException as e:  # reported to the parent
        out.put((rank, f"{type(e).__name__}: {e}"))
    finally:
        shm.close()


# 4-6 chunks per call: a buffer comes round again within a call (chunk c + 2), which is
# where a writer that skipped the acknowledgement wait would overwrite unread data
@pytest.mark.parametrize("world,heads,head_chunk,calls", [(2, 12, 1, 2), (3, 12, 1, 2), (4, 24, 1, 1)])
def test_every_rank_runs_its_own_schedule_without_deadlock(world, heads, head_chunk, calls):
    from multiprocessing import shared_memory
    nbytes = world * N_FLAGS * world * 4 + world * 2 * 2 * world * 4 + world * 4
    shm = shared_memory.SharedMemory(create=True, size=nbytes)
    try:
        np.ndarray((nbytes,), dtype=np.uint8, buffer=shm.buf)[:] = 0
        ctx = mp.get_context("spawn")
        out = ctx.Queue()
        procs = [ctx.Process(target=_rank_main, args=(r, world, heads, head_chunk, calls, shm.name, out))
                 for r in range(world)]
        for p in procs:
            p.start()
        results = dict(out.get(timeout=600) for _ in range(world))
        for p in procs:
            p.join(timeout=60)
        assert all(v == "ok" for v in results.values()), results
    finally:
        shm.close()
        shm.unlink()
