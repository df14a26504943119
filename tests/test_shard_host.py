"""Neuron-sharded layer, host side (CPU): the ownership map partitions the
neurons and stays balanced under a hot-first order, the ranks' oracle results
recombine to the single-GPU oracle result, and the all-reduce that combines
the ranks' partial outputs works across two gloo ranks."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle as O
import synthetic as S
from activation_sparse_ffn_predict_b200 import shard as SH


def shard_arrays(h, rows):
    pick = lambda a: None if a is None else a[rows]
    return {k: (pick(v) if k in ("W2", "b2", "Wg", "Wu", "WdT", "bias") else v) for k, v in h.items()}


@pytest.mark.parametrize("n", [1, 31, 32, 33, 1376, 11008])
@pytest.mark.parametrize("world", [1, 2, 3, 8])
@pytest.mark.parametrize("block", [1, 32])
def test_ownership_partitions_and_balances(n, world, block):
    parts = [SH.shard_rows(n, world, g, block) for g in range(world)]
    allrows = np.concatenate(parts)
    assert np.array_equal(np.sort(allrows), np.arange(n))          # every neuron exactly once
    for p in parts:
        assert np.all(np.diff(p) > 0)                                 # ascending: local order = global order
    sizes = [p.size for p in parts]
    assert max(sizes) - min(sizes) <= block                           # within one block


def test_hot_first_order_is_spread_over_ranks():
    # the offline permutation stores the hottest 20% first; every rank must get
    # its share of them
    n, world = 11008, 8
    hot = n // 5
    for g in range(world):
        rows = SH.shard_rows(n, world, g)
        share = np.count_nonzero(rows < hot) / hot
        assert abs(share - 1 / world) < 0.01


def test_invalid_arguments():
    with pytest.raises(ValueError):
        SH.shard_rows(10, 2, 2)
    with pytest.raises(ValueError):
        SH.shard_rows(10, 2, 0, block=0)
    assert SH.merge_lists([]).size == 0


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("B", [1, 4])
def test_oracle_shards_recombine_to_single_gpu_layer(world, B):
    cfg = S.get("tiny_reglu_f32")
    h = S.layer_weights(cfg, 0).numpy()
    X = S.layer_tokens(cfg, 0, B).numpy()
    ref_idx = O.predict(h["W1"], h["b1"], h["W2"], h["b2"], X, cfg.tau)[0]
    ref_y = O.sparse_ffn(h["act"], h["Wg"], h["Wu"], h["WdT"], h["bias"], X, ref_idx)
    lists, y = [], np.zeros_like(ref_y)
    for g in range(world):
        rows = SH.shard_rows(cfg.n, world, g)
        s = shard_arrays(h, rows)
        loc = O.predict(s["W1"], s["b1"], s["W2"], s["b2"], X, cfg.tau)[0]
        lists.append(rows[loc])
        y += O.sparse_ffn(s["act"], s["Wg"], s["Wu"], s["WdT"], s["bias"], X, loc)
    np.testing.assert_array_equal(SH.merge_lists(lists), ref_idx)
    np.testing.assert_allclose(y, ref_y, rtol=1e-12, atol=1e-12 * np.abs(ref_y).max())


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        cfg = S.get("tiny_reglu_f32")
        h = S.layer_weights(cfg, 0).numpy()
        X = S.layer_tokens(cfg, 0, 2).numpy()
        s = shard_arrays(h, SH.shard_rows(cfg.n, world, rank))
        loc = O.predict(s["W1"], s["b1"], s["W2"], s["b2"], X, cfg.tau)[0]
        y = torch.from_numpy(O.sparse_ffn(s["act"], s["Wg"], s["Wu"], s["WdT"], s["bias"], X, loc))
        SH.combine_partials(y)
        q.put((rank, y.numpy()))
    finally:
        dist.destroy_process_group()


def test_all_reduce_combines_two_gloo_ranks():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    cfg = S.get("tiny_reglu_f32")
    h = S.layer_weights(cfg, 0).numpy()
    X = S.layer_tokens(cfg, 0, 2).numpy()
    ref_idx = O.predict(h["W1"], h["b1"], h["W2"], h["b2"], X, cfg.tau)[0]
    ref_y = O.sparse_ffn(h["act"], h["Wg"], h["Wu"], h["WdT"], h["bias"], X, ref_idx)
    for r in range(world):
        np.testing.assert_allclose(res[r], ref_y, rtol=1e-12, atol=1e-12 * np.abs(ref_y).max())
    np.testing.assert_array_equal(res[0], res[1])     # every rank holds the same sum


def test_combine_is_a_no_op_without_a_group():
    y = torch.arange(6.0).reshape(2, 3)
    assert torch.equal(SH.combine_partials(y.clone()), y)
