"""The multi-rank path: sequences sharded across 2 gloo ranks on CPU, no exchange.

Each rank takes its shard of a packed varlen batch, runs the recurrence on it
(here the fp64 oracle stands in for the per-GPU library, on CPU), and the
gathered per-sequence results must equal a single-process run. The max-over-ranks
timing reduction used by bench.py is checked too.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from gated_delta_rule_62_b200.sharding import gather_shard, partition_sequences


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _case():
    from tests.pins import random_case
    lens = [5, 0, 17, 3, 9, 1, 12]
    T = sum(lens)
    q, k, v, la, beta, _ = random_case(77, T=T, H=2, dk=4, dv=3)
    r = np.random.default_rng(78)
    s0 = r.standard_normal((len(lens), 2, 4, 3))
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    return lens, cu, q, k, v, la, beta, s0


def _worker(rank, world, port, out):
    import oracle
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        lens, cu, q, k, v, la, beta, s0 = _case()
        shards = partition_sequences(lens, world)
        mine = shards[rank]
        idx, sub = gather_shard(cu, mine)
        o, s = oracle.forward(q[idx], k[idx], v[idx], la[idx], beta[idx], s0[mine], sub)
        results = [None] * world
        dist.all_gather_object(results, {"seqs": mine, "out": o, "state": s, "sub": sub})
        t = torch.tensor([float(rank + 1)], dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        if rank == 0:
            out.put((results, float(t.item())))
    finally:
        dist.destroy_process_group()


def test_partition_is_a_balanced_cover():
    lens = [512, 65536, 700, 30000, 1, 0, 4096, 2048, 9999]
    for w in (1, 2, 3, 8):
        shards = partition_sequences(lens, w)
        flat = sorted(i for s in shards for i in s)
        assert flat == list(range(len(lens)))
        loads = [sum(lens[i] for i in s) for s in shards]
        assert max(loads) - min(loads) <= max(lens)


@pytest.mark.timeout(120)
def test_two_gloo_ranks_match_single_process():
    import oracle
    oracle.build()
    ctx = mp.get_context("spawn")
    q_ = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q_)) for r in range(2)]
    for p in procs:
        p.start()
    results, tmax = q_.get(timeout=100)
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    assert tmax == 2.0
    lens, cu, q, k, v, la, beta, s0 = _case()
    ref_o, ref_s = oracle.forward(q, k, v, la, beta, s0, cu)
    seen = []
    for r in results:
        for j, n in enumerate(r["seqs"]):
            a, b = r["sub"][j], r["sub"][j + 1]
            np.testing.assert_allclose(r["out"][a:b], ref_o[cu[n]:cu[n + 1]], atol=1e-12, rtol=0)
            np.testing.assert_allclose(r["state"][j], ref_s[n], atol=1e-12, rtol=0)
            seen.append(n)
    assert sorted(seen) == list(range(len(lens)))
