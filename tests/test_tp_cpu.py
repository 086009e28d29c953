"""Tensor-parallel MLRA-4 and GLA-2 on CPU ranks (gloo).

Each rank takes its shard of one seeded problem (shared_kv_caches_b200.tp),
solves it with the fp64 oracle standing in for the library (no GPU here), and
the collective assembles the result: an all-reduce of the four MLRA branch
outputs, an all-gather of the two GLA groups' heads.  Every rank must end with
the oracle's answer for the whole, unsharded problem.  The shard slicing
itself is checked against the cache layout on one process.
"""

import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

from shared_kv_caches_b200 import tp as TP
from shared_kv_caches_b200 import workloads as W

SHAPES = {
    "mlra4": W.WORKLOADS["mlra_128k"].replace(batch=2, num_q_heads=8, ctx=(40, 150)),
    "gla2": W.WORKLOADS["gla"].replace(batch=2, num_q_heads=8, ctx=(40, 150)),
}


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, name, q):
    import torch.distributed as dist

    from oracle import oracle
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        x = W.make_inputs(SHAPES[name], seed=5)
        out, lse = TP.tp_decode(x, rank, world, compute=oracle.decode)
        q.put((rank, out, lse))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("name,world", [("mlra4", 4), ("gla2", 2), ("mlra4", 2)])
def test_tp_ranks_reassemble_the_whole_problem(oracle_mod, name, world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, name, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=180) for _ in procs), key=lambda t: t[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    x = W.make_inputs(SHAPES[name], seed=5)
    ref_out, ref_lse = oracle_mod.decode(x)
    for rank, out, lse in res:
        assert out.shape == ref_out.shape and lse.shape == ref_lse.shape
        np.testing.assert_allclose(out, ref_out, rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=1e-12)


def test_shard_columns_and_queries():
    s = SHAPES["mlra4"]
    x = W.make_inputs(s, seed=3)
    dn, dr = s.d_nope, s.d_rope
    for r in range(4):
        y = TP.shard_inputs(x, r, 4)
        assert y["shape"].num_kv == 1 and y["shape"].out_dtype == "fp32"
        assert y["kv"].shape[-1] == dn + dr == y["shape"].row_elems
        np.testing.assert_array_equal(y["kv"][..., :dn], x["kv"][..., r * dn:(r + 1) * dn])
        np.testing.assert_array_equal(y["kv"][..., dn:], x["kv"][..., 4 * dn:])
        np.testing.assert_array_equal(y["q_nope"][:, :, 0], x["q_nope"][:, :, r])
    g = SHAPES["gla2"]
    x = W.make_inputs(g, seed=3)
    hpr = g.num_q_heads // 2
    for r in range(2):
        y = TP.shard_inputs(x, r, 2)
        assert y["shape"].num_q_heads == hpr and y["shape"].num_kv == 1
        np.testing.assert_array_equal(y["kv"][..., :g.d_nope], x["kv"][..., r * g.d_nope:(r + 1) * g.d_nope])
        np.testing.assert_array_equal(y["q_nope"], x["q_nope"][:, r * hpr:(r + 1) * hpr])


def test_bad_splits_are_refused():
    with pytest.raises(ValueError):
        TP.units_per_rank(SHAPES["mlra4"], 3)
    with pytest.raises(ValueError):
        TP.units_per_rank(W.WORKLOADS["gqa"], 2)
    with pytest.raises(ValueError):
        TP.shard_inputs(W.make_inputs(SHAPES["gla2"], seed=1), 2, 2)
