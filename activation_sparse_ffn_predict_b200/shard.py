"""Neuron-sharded layer across G GPUs (one process per GPU).

The FFN's neurons are split across ranks -- the neuron partitioning that the
PowerInfer_x64 page lists among its multi-GPU coordination modes (its
architecture and tech-stack paragraph): rank g holds the predictor's W2/b2 rows and
the gate/up/down rows of its own neurons, while W1/b1 (the predictor's first
layer, over the whole input) are replicated.  Each rank predicts the activity
of its own neurons and gathers only those rows with the same one-call layer
(asf_predict_sparse_ffn) as the single-GPU path, giving a partial y over its
neurons; one all-reduce (sum) of y [B, d] fp32 per layer combines the ranks.

A neuron's prediction depends only on x and its own W2 row, so the union of
the ranks' lists (mapped back to global ids) is exactly the single-GPU list,
and the sum of the partial outputs is the single-GPU y up to the order of the
fp32 additions.

Ownership deals blocks of `block` consecutive rows round-robin, so a
hot-first storage order (the offline permutation) spreads hot rows evenly
instead of giving them all to rank 0.  The shards' rows are gathered once,
offline, with the library's own row-gather kernel.
"""
from __future__ import annotations

import numpy as np
import torch
import torch.distributed as dist

from .api import (FFN, Predictor, Workspace, asf_gather_rows, asf_predict_sparse_ffn, pack_layer)


def shard_rows(n: int, world: int, rank: int, block: int = 32) -> np.ndarray:
    """Global ids (ascending, int32) of the neurons rank owns: blocks of
    `block` consecutive rows dealt round-robin over the world's ranks."""
    if not (0 <= rank < world) or n < 0 or block < 1:
        raise ValueError("need 0 <= rank < world, n >= 0 and block >= 1")
    nb = (n + block - 1) // block
    mine = np.arange(rank, nb, world, dtype=np.int64)
    rows = (mine[:, None] * block + np.arange(block, dtype=np.int64)[None, :]).ravel()
    return rows[rows < n].astype(np.int32)


def _gather_vector(v: torch.Tensor, rows: torch.Tensor) -> torch.Tensor:
    """v[rows] for a 1-D fp32 device vector, through the library's gather kernel."""
    out = torch.empty(rows.shape[0], dtype=v.dtype, device=v.device)
    if rows.shape[0]:
        asf_gather_rows(v.reshape(-1, 1), out.reshape(-1, 1), rows)
    return out


def _gather_matrix(W: torch.Tensor, rows: torch.Tensor) -> torch.Tensor:
    out = torch.empty(rows.shape[0], W.shape[1], dtype=W.dtype, device=W.device)
    if rows.shape[0]:
        asf_gather_rows(W, out, rows)
    return out


class NeuronShard:
    """One rank's part of one layer (``synthetic.LayerWeights``-like ``w`` on
    this rank's device): the predictor over its neurons and its FFN rows in the
    neuron-major packed layout."""

    def __init__(self, w, rank: int, world: int, block: int = 32):
        n = int(w.W2.shape[0])
        dev = w.W2.device
        self.rank, self.world = rank, world
        self.rows_host = shard_rows(n, world, rank, block)
        self.rows = torch.from_numpy(self.rows_host).to(dev)
        if self.rows.shape[0] == 0:
            raise ValueError("this rank owns no neurons: use fewer ranks or a smaller block")
        self.W2 = _gather_matrix(w.W2, self.rows)
        self.b2 = _gather_vector(w.b2, self.rows)
        self.bias = _gather_vector(w.bias, self.rows)
        self.packed = pack_layer(w.act, w.Wg, w.Wu, w.WdT, perm=self.rows)
        self.pred = Predictor(w.W1, w.b1, self.W2, self.b2)
        self.ffn = FFN.packed(w.act, self.packed, self.bias)
        self.n_local = int(self.rows.shape[0])

    def workspace(self, max_batch: int) -> Workspace:
        return Workspace(self.pred, self.ffn, max_batch)

    def global_ids(self, idx: torch.Tensor, count: int) -> torch.Tensor:
        """This rank's active neurons as global ids (ascending: the ownership
        map is increasing, so the local order is kept)."""
        return self.rows.index_select(0, idx[:count].long())


def combine_partials(y: torch.Tensor, group=None) -> torch.Tensor:
    """Sum the ranks' partial outputs in place (one all-reduce of y [B, d]);
    a no-op without an initialised process group of more than one rank."""
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(y, op=dist.ReduceOp.SUM, group=group)
    return y


def _torch_stream(stream):
    """A torch stream object for a stream argument (None, torch stream or raw handle)."""
    if stream is None or isinstance(stream, torch.cuda.Stream):
        return stream
    return torch.cuda.ExternalStream(int(stream))


def sharded_layer(shard: NeuronShard, x: torch.Tensor, tau: float, idx: torch.Tensor, count: torch.Tensor,
                  y: torch.Tensor, ws: Workspace, group=None, stream=None) -> torch.Tensor:
    """One layer on this rank: predict and gather its own neurons (idx/count
    in local ids), then combine y over the ranks.  With a stream, the layer's
    kernels and the all-reduce are both enqueued on it (a collective orders
    against torch's current stream, so it is made current for the call)."""
    ts = _torch_stream(stream)
    asf_predict_sparse_ffn(shard.pred, shard.ffn, x, tau, idx, count, y, ws, ts)
    if ts is None:
        return combine_partials(y, group)
    with torch.cuda.stream(ts):
        return combine_partials(y, group)


def merge_lists(per_rank: list) -> np.ndarray:
    """The single-GPU list from the ranks' global-id lists (host arrays)."""
    if not per_rank:
        return np.zeros(0, dtype=np.int32)
    return np.sort(np.concatenate([np.asarray(p, dtype=np.int64) for p in per_rank])).astype(np.int32)



# --------------------------------------------------------------------------- #
# the ranks' partial outputs exchanged over peer memory (one kernel, no NCCL)  #
# --------------------------------------------------------------------------- #
def exchange_sizes(d: int, max_batch: int):
    """(publication bytes, flag words) of one rank's exchange buffers."""
    nbx = (d + 31) // 32
    return 2 * max_batch * d * 4, nbx * max_batch


def group_descriptor(world: int, rank: int, max_batch: int, d: int, pub, flag, epoch):
    """The asf_peer_group of this rank: every rank's buffer pointers in rank order."""
    from ._lib import ASF_MAX_PEERS, asf_peer_group
    if not (1 <= world <= ASF_MAX_PEERS) or not (0 <= rank < world):
        raise ValueError(f"need 1 <= world <= {ASF_MAX_PEERS} and 0 <= rank < world")
    if len(pub) != world or len(flag) != world:
        raise ValueError("one publication buffer and one flag array per rank")
    if any(not p for p in pub) or any(not f for f in flag) or not epoch:
        raise ValueError("null exchange buffer")
    g = asf_peer_group()
    g.world, g.rank, g.max_batch, g.d = world, rank, max_batch, d
    for r in range(world):
        g.pub[r] = int(pub[r])
        g.flag[r] = int(flag[r])
    g.epoch = int(epoch)
    return g


class CudaIpc:
    """Device buffers from cudaMalloc (so an IPC handle names exactly the
    buffer) and the CUDA IPC calls that share them between processes."""

    def __init__(self):
        from cuda.bindings import runtime as rt
        self.rt = rt

    def _ok(self, res, what):
        err = res[0] if isinstance(res, tuple) else res
        if err != self.rt.cudaError_t.cudaSuccess:
            raise RuntimeError(f"{what} failed: {err}")
        return res[1] if isinstance(res, tuple) and len(res) > 1 else None

    def malloc_zeroed(self, nbytes: int) -> int:
        ptr = int(self._ok(self.rt.cudaMalloc(nbytes), "cudaMalloc"))
        self._ok(self.rt.cudaMemset(ptr, 0, nbytes), "cudaMemset")
        return ptr

    def handle(self, ptr: int) -> bytes:
        return bytes(self._ok(self.rt.cudaIpcGetMemHandle(ptr), "cudaIpcGetMemHandle").reserved)

    def open(self, handle: bytes) -> int:
        h = self.rt.cudaIpcMemHandle_t()
        h.reserved = handle
        return int(self._ok(self.rt.cudaIpcOpenMemHandle(h, self.rt.cudaIpcMemLazyEnablePeerAccess),
                            "cudaIpcOpenMemHandle"))

    def close(self, ptr: int) -> None:
        self._ok(self.rt.cudaIpcCloseMemHandle(ptr), "cudaIpcCloseMemHandle")

    def free(self, ptr: int) -> None:
        self._ok(self.rt.cudaFree(ptr), "cudaFree")

    def synchronize(self) -> None:
        self._ok(self.rt.cudaDeviceSynchronize(), "cudaDeviceSynchronize")


class PeerGroup:
    """The exchange buffers of the ranks of a torch.distributed group, one
    process per GPU: this rank's publication buffer, flag words and call
    counters, and the other ranks' buffers mapped here through CUDA IPC.
    ``desc`` is the asf_peer_group the exchanging calls take."""

    def __init__(self, d: int, max_batch: int, group=None, ipc=None):
        self.world = dist.get_world_size(group) if dist.is_initialized() else 1
        self.rank = dist.get_rank(group) if dist.is_initialized() else 0
        self.ipc = ipc if ipc is not None else CudaIpc()
        pub_bytes, nflag = exchange_sizes(d, max_batch)
        self.own = [self.ipc.malloc_zeroed(pub_bytes), self.ipc.malloc_zeroed(4 * nflag),
                    self.ipc.malloc_zeroed(4 * nflag)]        # publication, flags, counters
        self.ipc.synchronize()                                  # zeroed before any peer can look
        mine = (self.ipc.handle(self.own[0]), self.ipc.handle(self.own[1]))
        handles = [None] * self.world
        if self.world > 1:
            dist.all_gather_object(handles, mine, group=group)
        else:
            handles[0] = mine
        self.opened = []
        pub, flag = [], []
        for r in range(self.world):
            if r == self.rank:
                pub.append(self.own[0])
                flag.append(self.own[1])
            else:
                p, f = self.ipc.open(handles[r][0]), self.ipc.open(handles[r][1])
                self.opened += [p, f]
                pub.append(p)
                flag.append(f)
        self.desc = group_descriptor(self.world, self.rank, max_batch, d, pub, flag, self.own[2])
        if self.world > 1:
            dist.barrier(group=group)       # every rank mapped every buffer before the first exchange

    def close(self) -> None:
        for p in self.opened:
            self.ipc.close(p)
        for p in self.own:
            self.ipc.free(p)
        self.opened, self.own = [], []


class EmulatedGroup:
    """Every rank of a group held by one process on one GPU (torch buffers):
    for exercising the exchange kernel without several GPUs
    (asf_reduce_exchange with local_ranks == world)."""

    def __init__(self, world: int, d: int, max_batch: int, device=None):
        pub_bytes, nflag = exchange_sizes(d, max_batch)
        dev = device if device is not None else torch.device("cuda")
        self.pub = [torch.zeros(pub_bytes // 4, dtype=torch.float32, device=dev) for _ in range(world)]
        self.flag = [torch.zeros(nflag, dtype=torch.int32, device=dev) for _ in range(world)]
        self.epoch = torch.zeros(world * nflag, dtype=torch.int32, device=dev)
        self.desc = group_descriptor(world, 0, max_batch, d, [t.data_ptr() for t in self.pub],
                                     [t.data_ptr() for t in self.flag], self.epoch.data_ptr())


def sharded_layer_exchange(shard: NeuronShard, x: torch.Tensor, tau: float, idx: torch.Tensor,
                           count: torch.Tensor, y: torch.Tensor, ws: Workspace, peers: PeerGroup,
                           stream=None) -> torch.Tensor:
    """One layer on this rank with y summed over the ranks inside the layer's
    last kernel (peer memory; no separate collective)."""
    from .api import asf_predict_sparse_ffn_exchange
    asf_predict_sparse_ffn_exchange(shard.pred, shard.ffn, x, tau, idx, count, y, ws, peers.desc,
                                    _torch_stream(stream))
    return y
