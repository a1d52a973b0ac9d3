"""The N > 1 bench path on CPU: world-size-2 gloo process groups.  The path has
no exchange step (independent replicas), so what ranks share is host logic:
the max-over-ranks timing reduction and identical plans on every replica."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        import bench
        import synth
        from prefill_decode_b200 import build
        build.build()
        import prefill_decode_b200 as pod
        got = bench.reduce_max(10.0 + rank, dist, "cpu")
        w = synth.llama3_8b_mix()
        lens = synth._draw_lengths(__import__("numpy").random.default_rng(w.seed), w)
        plan = pod.Plan(w.num_q_heads, w.num_kv_heads, w.head_dim, w.prefill_len, w.prefill_ctx + w.prefill_len,
                        lens, num_sms=148)
        digests = [None] * world
        dist.all_gather_object(digests, bench.plan_digest(plan))
        q.put((rank, got, digests))
    finally:
        dist.destroy_process_group()


def test_two_rank_reduce_and_identical_plans():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, digests in res:
        assert got == 11.0
        assert len(set(digests)) == 1


def test_reduce_max_without_process_group():
    import bench
    assert bench.reduce_max(3.5, None, "cpu") == 3.5
