"""Tensor parallelism, host side ("深入解析Llama MLP模块" page §6.3): the weight slicing
of tp_shard_weights and the decomposition it relies on, checked with the fp64 oracle:
the ranks' attention partials plus X give X', their MLP partials of X' plus X' give
the block output, and their caches are the block's KV heads (prefill and a decode
step, GQA, 2 and 4 ranks). Then the same with a real all-reduce over two gloo ranks
(world size 2, CPU), each rank computing only its own slice."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import block as ob
from synth import BlockConfig, make_decode_x, make_weights, make_x

CFG = BlockConfig("tp", d=64, n_heads=8, n_kv_heads=4, head_dim=8, f=96, B=2, T=9, dtype="f32",
                  gain="1+N(0,0.1)")


def _shards(W, world):
    from llama_pre_norm_b200 import tp_shard_weights

    return [tp_shard_weights(W, r, world, CFG.n_heads, CFG.n_kv_heads, CFG.head_dim) for r in range(world)]


@pytest.mark.parametrize("world", [2, 4])
def test_tp_partials_sum_to_the_block(world):
    W = make_weights(CFG)
    X = make_x(CFG)
    a = (CFG.eps, CFG.rope_base)
    full = ob.block_prefill(X, W, CFG.n_heads, CFG.n_kv_heads, CFG.head_dim, *a)
    hs, ks = CFG.n_heads // world, CFG.n_kv_heads // world
    shards = _shards(W, world)
    assert all(Ws["wq"].shape == (hs * CFG.head_dim, CFG.d) for Ws in shards)
    assert all(Ws["w_down"].shape == (CFG.d, CFG.f // world) for Ws in shards)
    parts = [ob.tp_attention_partial(X, Ws, hs, ks, CFG.head_dim, *a) for Ws in shards]
    x1 = ob._f64(X) + sum(p["o"] for p in parts)
    np.testing.assert_allclose(x1, full["x1"], rtol=0, atol=1e-12)
    y = x1 + sum(ob.tp_mlp_partial(x1, Ws, CFG.eps) for Ws in shards)
    np.testing.assert_allclose(y, full["y"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(np.concatenate([p["k"] for p in parts], axis=1), full["k"], atol=1e-12)
    np.testing.assert_allclose(np.concatenate([p["v"] for p in parts], axis=1), full["v"], atol=1e-12)
    x = make_decode_x(CFG, 0)
    L = [CFG.T] * CFG.B
    fd = ob.block_decode(x, W, CFG.n_heads, CFG.n_kv_heads, CFG.head_dim, *a, full["k"], full["v"], L)
    dp = [ob.tp_attention_partial_decode(x, Ws, hs, ks, CFG.head_dim, *a, p["k"], p["v"], L)
          for Ws, p in zip(shards, parts)]
    x1d = ob._f64(x) + sum(p["o"] for p in dp)
    yd = x1d + sum(ob.tp_mlp_partial(x1d, Ws, CFG.eps) for Ws in shards)
    np.testing.assert_allclose(yd, fd["y"], rtol=0, atol=1e-12)


def test_tp_shard_weights_rejects_uneven_splits():
    from llama_pre_norm_b200 import tp_shard_weights

    with pytest.raises(ValueError):
        tp_shard_weights(make_weights(CFG), 0, 3, CFG.n_heads, CFG.n_kv_heads, CFG.head_dim)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    W = make_weights(CFG)
    X = make_x(CFG)
    a = (CFG.eps, CFG.rope_base)
    Ws = _shards(W, world)[rank]
    hs, ks = CFG.n_heads // world, CFG.n_kv_heads // world
    o = torch.from_numpy(ob.tp_attention_partial(X, Ws, hs, ks, CFG.head_dim, *a)["o"])
    dist.all_reduce(o)  # the attention branch, complete on every rank
    x1 = ob._f64(X) + o.numpy()
    m = torch.from_numpy(ob.tp_mlp_partial(x1, Ws, CFG.eps))
    dist.all_reduce(m)
    y = x1 + m.numpy()
    full = ob.block_prefill(X, W, CFG.n_heads, CFG.n_kv_heads, CFG.head_dim, *a)
    q.put((rank, float(np.max(np.abs(y - full["y"])))))
    dist.barrier()
    dist.destroy_process_group()


def test_tp_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    assert [r for r, _ in res] == [0, 1]
    assert all(err < 1e-12 for _, err in res)
