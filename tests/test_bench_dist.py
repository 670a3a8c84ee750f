"""The bench's multi-GPU arithmetic on CPU: two gloo ranks stand in for two
GPUs (replicas only -- the layer forward has no exchange step, so the only
cross-rank operations are the barrier and the max-over-ranks timing)."""
import os
import socket
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local = [10.0 + rank, 100.0 - rank]            # rank-dependent step / e2e times (ms)
        t, e = bench.reduce_max_over_ranks(local)
        dist.barrier()
        q.put((rank, t, e, bench.job_tokens_per_s(world, 8, 1000, t)))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, t, e, tps in res:
        assert t == 11.0 and e == 100.0          # the slowest rank decides
        assert tps == pytest.approx(2 * 8 * 1000 / 0.011)


def test_reference_arm_other_ranks_exit_without_work(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    from mixture_experts_layer_43_b200 import synth
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "1")
    args = bench.main.__globals__["argparse"].Namespace(steps=5, warmup=3, seed=0)
    assert bench.run_reference(args, synth.WORKLOADS["tiny_T4_d256_E8k2_F512"]) == 0


def test_reduce_is_identity_without_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_max_over_ranks([1.5, 2.5]) == [1.5, 2.5]
    assert bench.job_tokens_per_s(1, 8, 100, 50.0) == pytest.approx(16000.0)
