"""Host logic of the neuron-sharded layer's peer exchange, on CPU.

The exchange itself is one CUDA kernel (tested on a GPU by emulating the
ranks in one cooperative launch); here, without a GPU: the descriptor lists
every rank's buffers in rank order, validation rejects bad groups, and two
gloo ranks building a PeerGroup through a fake IPC layer each end up with
their own buffers in their own slot and the peer's mapped buffers in the
peer's slot, closing exactly what they opened."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

from activation_sparse_ffn_predict_b200 import _lib as L
from activation_sparse_ffn_predict_b200 import shard as SH


def test_exchange_sizes():
    pub, nflag = SH.exchange_sizes(8192, 4)
    assert pub == 2 * 4 * 8192 * 4 and nflag == 256 * 4
    assert SH.exchange_sizes(1096, 1) == (2 * 1096 * 4, 35)      # ragged last column block


def test_descriptor_in_rank_order():
    g = SH.group_descriptor(3, 1, 4, 1024, [16, 32, 48], [64, 80, 96], 112)
    assert (g.world, g.rank, g.max_batch, g.d) == (3, 1, 4, 1024)
    assert [g.pub[r] for r in range(3)] == [16, 32, 48]
    assert [g.flag[r] for r in range(3)] == [64, 80, 96]
    assert g.epoch == 112
    assert all(not g.pub[r] for r in range(3, L.ASF_MAX_PEERS))


@pytest.mark.parametrize("bad", [
    dict(world=0), dict(world=L.ASF_MAX_PEERS + 1), dict(rank=-1), dict(rank=2),
    dict(pub=[16]), dict(flag=[64, 0]), dict(epoch=0)])
def test_descriptor_rejects_bad_groups(bad):
    args = dict(world=2, rank=0, max_batch=1, d=64, pub=[16, 32], flag=[64, 80], epoch=112)
    args.update(bad)
    with pytest.raises(ValueError):
        SH.group_descriptor(**args)


class FakeIpc:
    """Pointers derived from (rank, buffer kind); handles name them."""

    def __init__(self, rank):
        self.rank, self.next, self.closed, self.freed, self.opened = rank, 0, [], [], []

    def malloc_zeroed(self, nbytes):
        self.next += 1
        return (self.rank + 1) * 0x1000000 + self.next * 0x1000

    def handle(self, ptr):
        return ptr.to_bytes(8, "little") + bytes(56)

    def open(self, handle):
        ptr = int.from_bytes(handle[:8], "little")
        self.opened.append(ptr)
        return ptr + 0x100000000          # this process's mapping of the peer's buffer

    def close(self, ptr):
        self.closed.append(ptr)

    def free(self, ptr):
        self.freed.append(ptr)

    def synchronize(self):
        pass


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ipc = FakeIpc(rank)
        pg = SH.PeerGroup(d=4096, max_batch=2, ipc=ipc)
        g = pg.desc
        out = (rank, g.world, g.rank, [g.pub[r] for r in range(world)], [g.flag[r] for r in range(world)],
               g.epoch, list(pg.own), list(pg.opened))
        pg.close()
        q.put(out + (ipc.closed, ipc.freed))
    finally:
        dist.destroy_process_group()


def test_peer_group_maps_every_rank_on_two_gloo_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(world):
        r = q.get(timeout=120)
        res[r[0]] = r
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    own = {r: res[r][6] for r in range(world)}
    for r in range(world):
        _, w, rk, pub, flag, epoch, mine, opened, closed, freed = res[r]
        assert (w, rk) == (world, r)
        for h in range(world):
            if h == r:
                assert pub[h] == own[r][0] and flag[h] == own[r][1]
            else:                          # the peer's buffers, as mapped in this process
                assert pub[h] == own[h][0] + 0x100000000 and flag[h] == own[h][1] + 0x100000000
        assert epoch == own[r][2]          # counters are never shared
        assert sorted(closed) == sorted(opened) and sorted(freed) == sorted(own[r])
