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


def test_reference_arm_prints_one_contract_line():
    """`bench.py --impl reference` runs the oracle on the host (no GPU): one
    JSON line with the contract's keys, its own cpu_baseline and an e2e
    block with no host-device copies."""
    import json
    import subprocess
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "tiny_T4_d256_E8k2_F512", "--steps", "3", "--warmup", "3"],
                       capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["steps"] == 3 and d["warmup"] == 3
    assert d["value"] > 0 and d["unit"] == "tokens/s" and d["higher_is_better"] is True
    assert d["config"]["workload"] == "tiny_T4_d256_E8k2_F512"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}


def test_profile_traffic_is_null_unless_the_capture_matches_the_sources(tmp_path, monkeypatch):
    """`roofline.traffic` comes from a committed ncu summary only while that
    summary's source hash equals the current kernel sources' hash."""
    sys.path.insert(0, ROOT)
    import bench
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    p = tmp_path / "profiles" / "k__w.txt"
    p.write_text("# command: ...\nkernel_source_sha256: abc\ndram_bytes_per_launch: 1234\n")
    assert bench._profile_traffic("k", "w", "abc") == 1234.0
    assert bench._profile_traffic("k", "w", "abd") is None          # sources changed since
    assert bench._profile_traffic("k", "other", "abc") is None      # no capture for it
    p.write_text("kernel_source_sha256: abc\n")
    assert bench._profile_traffic("k", "w", "abc") is None          # capture without the figure


def test_committed_profiles_name_the_hash_of_their_sources():
    """Every committed decode / prefill DRAM summary records the hash of the
    sources of its kernel (so the bench can tell whether it still applies),
    and none carries a hand-written note about a recomputed hash."""
    import glob
    sys.path.insert(0, ROOT)
    files = glob.glob(os.path.join(ROOT, "profiles", "*.txt"))
    assert files
    for f in files:
        txt = open(f).read()
        assert "kernel_source_sha256:" in txt, f
        assert "recomputed" not in txt, f
        sha = [ln.split(":", 1)[1].strip() for ln in txt.splitlines()
               if ln.startswith("kernel_source_sha256:")][0]
        assert len(sha) == 64 and all(c in "0123456789abcdef" for c in sha), f
