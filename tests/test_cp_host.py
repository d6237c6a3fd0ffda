"""Host side of context parallelism, on CPU: the connection of the ranks of one sequence.

cp_connect_ranks publishes each rank's gather-buffer and flag handles, collects every
rank's, maps the others' and hands the library one address per rank (its own buffers at its
own index). Here two gloo ranks exchange the handles through torch.distributed; the
library's IPC calls and the handle are stand-ins (no GPU), so what is checked is the
exchange: which address ends up at which index, and the refusal of an incomplete set of
ranks."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import recurrent_depth_transformer_b200 as R


class FakeHandle:
    """cp_buffers / cp_connect of a rank whose buffers sit at 1000 (rank + 1) and + 100."""

    def __init__(self, rank):
        self.rank = rank
        self.connected = None

    def cp_buffers(self):
        base = 1000 * (self.rank + 1)
        return base, 4096, base + 100, 256

    def cp_connect(self, peer_kv, peer_flags):
        self.connected = (list(peer_kv), list(peer_flags))


def fake_get(addr):          # a 64-byte "handle" that names the address
    return int(addr).to_bytes(64, "little")


def fake_open(handle):       # "mapping" another process's allocation moves it
    return int.from_bytes(handle, "little") + 7


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)

    def all_gather(obj):
        out = [None] * world
        dist.all_gather_object(out, obj)
        return out

    h = FakeHandle(rank)
    opened = R.cp_connect_ranks(h, rank, world, all_gather, get_handle=fake_get, open_handle=fake_open)
    q.put((rank, h.connected, sorted(opened)))
    dist.barrier()
    dist.destroy_process_group()


def test_two_ranks_connect_to_each_others_buffers():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = dict((r, (c, o)) for r, c, o in (q.get(timeout=10) for _ in range(2)))
    # rank 0: its own buffers as they are, rank 1's as mapped here (+ 7)
    assert res[0][0] == ([1000, 2007], [1100, 2107])
    assert res[1][0] == ([1007, 2000], [1107, 2100])
    assert res[0][1] == [2007, 2107] and res[1][1] == [1007, 1107]   # what to close later


def test_incomplete_or_duplicate_ranks_are_refused():
    h = FakeHandle(0)
    with pytest.raises(RuntimeError, match="expected ranks 0 .. 2"):
        R.cp_connect_ranks(h, 0, 3, lambda obj: [obj, (1, b"", b"")], get_handle=fake_get, open_handle=fake_open)
    with pytest.raises(RuntimeError, match="expected ranks 0 .. 1"):
        R.cp_connect_ranks(h, 0, 2, lambda obj: [obj, obj], get_handle=fake_get, open_handle=fake_open)
    assert h.connected is None
