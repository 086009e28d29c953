"""Multi-rank bench plumbing on CPU: two gloo ranks reduce their timings with
max / sum and draw distinct batches (data parallel over sequences)."""

import os
import socket

import numpy as np
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch.distributed as dist

    from shared_kv_caches_b200 import benchutil as BU
    from shared_kv_caches_b200 import workloads as W
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    mx = BU.max_over_ranks(10.0 + rank)
    sm = BU.sum_over_ranks(1.0 + rank)
    x = W.make_inputs(W.WORKLOADS["gqa"].replace(batch=4, ctx=(10, 500)), seed=BU.rank_seed(0, rank))
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, mx, sm, x["seq_lens"].tolist(), int(x["q_nope"][0, 0, 0])))


def test_two_gloo_ranks_reduce_and_shard():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [11.0, 11.0]
    assert [r[2] for r in res] == [3.0, 3.0]
    assert res[0][3] != res[1][3] or res[0][4] != res[1][4]   # each rank has its own batch


def test_single_process_reductions_are_identity():
    from shared_kv_caches_b200 import benchutil as BU
    assert BU.max_over_ranks(3.5) == 3.5
    assert BU.sum_over_ranks(2.0) == 2.0


def test_step_cost_counts():
    from shared_kv_caches_b200 import benchutil as BU
    from shared_kv_caches_b200 import workloads as W
    s = W.WORKLOADS["mla"]
    c = BU.step_cost(s.replace(batch=2), np.array([64, 100]))
    assert c["kv_bytes"] == 164 * 1152
    assert c["flops"] == 164 * 128 * 2 * (576 + 512)
    s = W.WORKLOADS["gqa"]
    c = BU.step_cost(s.replace(batch=1), np.array([10]))
    assert c["kv_bytes"] == 10 * 4096
    s = W.WORKLOADS["mlra_1m"]
    assert BU.flops_per_token(s) == 128 * 4 * 2 * (192 + 128)
