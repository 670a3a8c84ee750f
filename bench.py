#!/usr/bin/env python
"""Benchmark of the MoE SwiGLU layer forward pass on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl b200|reference]
                    [--workload NAME] [--instances M]

A step is one whole layer call (router, top-k, buckets, every active routed
and shared expert, weighted combine) over one batch of seeded synthetic
input.  The default workload is the Mixtral-8x7B-shaped decode layer
(T=8, d=4096, E=8, k=2, F=14336, bf16), whose 2.8 GB of expert weights are
far larger than the 126 MB L2, so every step streams its weights from HBM.
Workloads whose weights fit in L2 rotate through M distinct layer instances
(--instances) so that each step reads cold weights.

Rank 0 prints one JSON line.  With N > 1 (torchrun, one process per GPU)
every rank runs an independent replica (the layer forward has no exchange
step: replicas only); the time is the max over ranks.

--impl reference times the fp64 CPU oracle instead (rank 0 only), one token
of the same workload per step, on the host cores.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from mixture_experts_layer_43_b200 import synth  # noqa: E402

METRIC = "MoE layer tokens/s; achieved HBM GB/s (T≤8) or TFLOPS (T=4096) vs peak"
DEFAULT_WORKLOAD = "mixtral_T8_d4096_E8k2_F14336"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
REF_BUDGET_S = 150.0


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return (float(j["hbm_gbs"]), float(j["bf16_tflops"]),
                float(j.get("bf16_tflops_sustained", j["bf16_tflops"])), "measured")
    return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


def _profile_traffic(kernel: str, workload: str, src_sha: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel source; else None."""
    path = os.path.join(ROOT, "profiles", f"{kernel}__{workload}.txt")
    if not os.path.exists(path):
        return None
    vals = {}
    with open(path) as f:
        for ln in f:
            if ":" in ln and not ln.startswith("#"):
                k, v = ln.split(":", 1)
                vals[k.strip()] = v.strip()
    if vals.get("kernel_source_sha256") != src_sha:
        return None
    try:
        return float(vals["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


def _kernel_src_sha(files):
    import hashlib
    h = hashlib.sha256()
    for fn in files:
        with open(os.path.join(ROOT, "mixture_experts_layer_43_b200", "csrc", fn), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


class ClockSampler:
    """nvidia-smi samples of the SM clock and throttle reasons while running."""

    FIELDS = ("uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid: str, period_ms: int = 100):
        self.uuid = uuid
        self.period_ms = period_ms
        self.proc = None
        self.path = None

    def __enter__(self):
        import tempfile
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 f"-lms", str(self.period_ms), "-f", self.path],
                stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None or not self.path or not os.path.exists(self.path):
            return None
        rows = []
        with open(self.path) as f:
            for ln in f:
                parts = [p.strip() for p in ln.split(",")]
                if len(parts) < 9:
                    continue
                if self.uuid and parts[0] != self.uuid:
                    continue
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        try:
            sm = [float(r[1]) for r in rows]
            mx = max(float(r[2]) for r in rows)
        except ValueError:
            return None
        reasons = set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for r in rows:
            for n, v in zip(names, r[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(rows)}


def reduce_max_over_ranks(values, device=None):
    """Each value's maximum over all ranks: a multi-GPU job is as slow as its
    slowest replica.  Identity without an initialised process group."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def job_tokens_per_s(world_size: int, tokens_per_step: int, steps: int, t_max_ms: float) -> float:
    """Whole-job throughput of `world_size` replicas that each ran `steps`
    layer calls of `tokens_per_step` tokens in at most `t_max_ms`."""
    return world_size * tokens_per_step * steps / (t_max_ms / 1e3)


def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def _active_bytes(sh, counts, n_shared):
    """Algorithmic bytes of one experts launch: every distinct active routed
    expert and every shared expert read once, x read, out written."""
    act = int(np.count_nonzero(counts))
    per = synth.weight_bytes_per_expert(sh)
    shared = n_shared * synth.weight_bytes_per_expert(sh, sh.Fs) if n_shared else 0
    return act * per + shared + sh.T * sh.d * 2 + sh.T * sh.d * 4, act


def _expert_flops(sh, counts, n_shared):
    """Algorithmic FLOPs of the expert stage: 2 per multiply-add of the three
    expert matrices for every (token, routed expert) pair and every (token,
    shared expert) pair."""
    routed = int(np.sum(counts)) * 2 * 3 * sh.F * sh.d
    shared = sh.T * n_shared * 2 * 3 * sh.Fs * sh.d if n_shared else 0
    return routed + shared


def _cpu_baseline(inp, sh, budget_s=12.0, max_s=30.0):
    import oracle
    n_threads = oracle.max_threads()
    t0 = time.perf_counter()
    done = 0
    while True:
        oracle.forward(inp, tokens=[done % sh.T])
        done += 1
        el = time.perf_counter() - t0
        if el >= budget_s or el >= max_s:
            break
    return {"value": done / el, "unit": "tokens/s", "cores": n_threads, "kind": "oracle",
            "sample": (f"{done} tokens of the {sh.name} batch, one fp64 oracle call per "
                       f"token (routing + every selected and shared expert), {el:.1f} s")}


def run_reference(args, sh):
    ws, rank, _ = _dist()
    if rank != 0:
        return 0
    import oracle
    inp = synth.make_inputs(sh, seed=args.seed)
    n_threads = oracle.max_threads()
    for i in range(args.warmup):
        oracle.forward(inp, tokens=[i % sh.T])
    t0 = time.perf_counter()
    steps = 0
    while steps < args.steps:
        oracle.forward(inp, tokens=[steps % sh.T])
        steps += 1
        if time.perf_counter() - t0 > REF_BUDGET_S:
            break
    el = time.perf_counter() - t0
    val = steps / el
    line = {
        "impl": "reference", "metric": METRIC, "value": val, "unit": "tokens/s",
        "n_gpus": ws, "steps": steps, "steps_requested": args.steps, "warmup": args.warmup,
        "ms_per_step": el / steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": sh.name, "shape": synth.describe(sh),
                   "sample_per_step": "one token of the batch"},
        "cpu_baseline": {"value": val, "unit": "tokens/s", "cores": n_threads, "kind": "oracle",
                         "sample": f"{steps} steps of one token each, fp64 oracle"},
        "e2e": {"value": val, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# Every seeded workload of the layer measured by the default run, under the
# same protocol (CUDA-graph replays, cold weights, events on the launching
# stream): the decode layers of the Mixtral-8x7B and 35B-A3B shapes (bf16
# and Q4_0, T = 1 and 8), the tiny parity layer, and the DeepSeek-MoE-16B
# prefill layer.  The first is the headline line's workload.
ALL_WORKLOADS = ("mixtral_T8_d4096_E8k2_F14336", "tiny_T4_d256_E8k2_F512",
                 "a3b_T1_d2048_E256k8_F512_S1", "a3b_q4_T1_d2048_E256k8_F512_S1",
                 "a3b_q4_T8_d2048_E256k8_F512_S1", "deepseek_T4096_d2048_E64k6_F1408_S2",
                 # the other weight formats of the 35B-A3B model's mix, and the
                 # prefill layer with fp16 down matrices (h in fp16)
                 "a3b_T8_d2048_E256k8_F512_S1", "a3b_q8_T8_d2048_E256k8_F512_S1",
                 "a3b_q5_T8_d2048_E256k8_F512_S1", "a3b_q6_T8_d2048_E256k8_F512_S1",
                 "deepseek_f16down_T4096_d2048_E64k6_F1408_S2")
MIN_TIMED_MS = 150.0      # per-workload entries time at least this long (clock samples)


class _Setup:
    """A workload resident on the device: layer instances, x, out, plan."""

    def __init__(self, sh, args, dev, stream, host_inputs):
        import torch
        from mixture_experts_layer_43_b200 import binding as B
        from mixture_experts_layer_43_b200 import device as D
        self.sh, self.dev, self.stream = sh, dev, stream
        if host_inputs:
            self.base = synth.make_inputs(sh, seed=args.seed)
            first = D.DeviceLayer(self.base, device=str(dev))
            x_bits = self.base.x
        else:
            self.base = None
            first = D.random_layer(sh, seed=args.seed, device=str(dev))
            x_bits = synth.make_inputs(sh, seed=args.seed, x_only=True).x
        self.x_bits = x_bits
        E_act = sh.E * (1.0 - (1.0 - sh.k / sh.E) ** sh.T)
        active_est = (E_act * synth.weight_bytes_per_expert(sh) + sh.S * (
            synth.weight_bytes_per_expert(sh, sh.Fs) if sh.S else 0) + sh.E * sh.d * 4)
        self.per_inst = first.weight_bytes() + sh.E * sh.d * 4
        # distinct device copies, enough that the weights one step reads are
        # cold in L2 (>= 4x L2 over the rotation)
        n_inst = args.instances or int(min(128, max(1, -(-4 * L2_BYTES // int(active_est)))))
        self.n_inst = max(1, min(n_inst, int(40e9 // self.per_inst)))
        self.layers = [first] + [first.clone() for _ in range(1, self.n_inst)]
        torch.cuda.synchronize(dev)
        self.x = D.upload_x(x_bits, dev)
        self.out = torch.empty((sh.T, sh.d), dtype=torch.float32, device=dev)
        self.plan = B.moe_plan_create(first.config(sh.T))
        self.routing = D.Routing(sh.T, sh.k, sh.E, dev)
        self.prefill = sh.T > B.MOE_DECODE_MAX_T and sh.wfmt in (synth.WFMT_BF16,
                                                                synth.WFMT_BF16_F16DOWN)

    def step(self, i, ev_a=None, ev_b=None):
        """One layer call.  Decode: moe_forward (the single fused launch),
        events around it.  Prefill: router + scatter, then events around the
        two GEMM launches."""
        from mixture_experts_layer_43_b200 import binding as B
        sh, L, st = self.sh, self.layers[i % self.n_inst], self.stream.cuda_stream
        xp, op = self.x.data_ptr(), self.out.data_ptr()
        if not self.prefill:
            if ev_a is not None:
                ev_a.record(self.stream)
            B.moe_forward(self.plan, L.weights, xp, sh.T, sh.k, sh.wfmt, op, None, st)
            if ev_b is not None:
                ev_b.record(self.stream)
            return
        B.moe_route(self.plan, L.weights, xp, sh.T, sh.k, sh.wfmt, op, st)
        if ev_a is not None:
            ev_a.record(self.stream)
        B.moe_experts(self.plan, L.weights, xp, sh.T, sh.k, sh.wfmt, op, st)
        if ev_b is not None:
            ev_b.record(self.stream)

    def destroy(self):
        from mixture_experts_layer_43_b200 import binding as B
        B.moe_plan_destroy(self.plan)
        self.layers = []


def _measure(su: "_Setup", args, uuid, exact_steps=None, min_ms=0.0, ws=1):
    """Time one workload.  exact_steps: time exactly that many steps (the
    headline line); else at least --steps steps and at least min_ms.
    Returns the measurement as a dict (max over ranks where it matters)."""
    import torch
    from mixture_experts_layer_43_b200 import binding as B
    sh, dev, stream = su.sh, su.dev, su.stream
    T, st = sh.T, stream.cuda_stream
    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            su.step(i)
        # algorithmic bytes and FLOPs: from each instance's own routing on this x
        act_bytes, acts, act_flops = [], [], []
        for i in range(su.n_inst):
            B.moe_forward(su.plan, su.layers[i].weights, su.x.data_ptr(), T, sh.k, sh.wfmt,
                          su.out.data_ptr(), su.routing.struct, st)
            stream.synchronize()
            cnt = su.routing.counts.cpu().numpy()
            b, a = _active_bytes(sh, cnt, su.layers[i].n_shared)
            act_bytes.append(b)
            acts.append(a)
            act_flops.append(_expert_flops(sh, cnt, su.layers[i].n_shared))
        launches_per_step = B.moe_last_launch_count(su.plan)
        status = B.moe_get_device_status(su.plan)
        if status != B.MOE_OK:
            raise RuntimeError(f"{sh.name}: device status after warm-up: "
                               + B.moe_status_string(status))

        # The timed loop replays a CUDA graph of S whole steps (router +
        # experts per step, cycling the instances), so host launch overhead
        # cannot starve the GPU.  A second graph of S steps carries an event
        # node on each side of every experts launch, for that kernel's own
        # duration.
        S = su.n_inst * max(1, -(-32 // su.n_inst))
        g_steps = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_steps, stream=stream):
            for i in range(S):
                su.step(i)
        ev_a = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(S)]
        ev_b = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(S)]
        g_kern = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_kern, stream=stream):
            for i in range(S):
                su.step(i, ev_a[i], ev_b[i])
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        for _ in range(2):
            g_steps.replay()
            g_kern.replay()
        t0.record(stream)
        g_steps.replay()
        t1.record(stream)
        torch.cuda.synchronize(dev)
        est_ms = max(t0.elapsed_time(t1) / S, 1e-4)
        if exact_steps is not None:
            K = exact_steps
        else:
            K = max(args.steps, int(math.ceil(min_ms / est_ms)))
        R, rem = divmod(K, S)
        g_rem = None
        if rem:
            g_rem = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g_rem, stream=stream):
                for i in range(rem):
                    su.step(i)
            g_rem.replay()
        t_start = torch.cuda.Event(enable_timing=True)
        t_end = torch.cuda.Event(enable_timing=True)
        if ws > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize(dev)
        with ClockSampler(uuid) as clk:
            t_start.record(stream)
            for _ in range(R):
                g_steps.replay()
            if g_rem is not None:
                g_rem.replay()
            t_end.record(stream)
            torch.cuda.synchronize(dev)
            kern_ms = []
            for _ in range(max(1, min(R, 8))):
                g_kern.replay()
                torch.cuda.synchronize(dev)
                kern_ms += [a.elapsed_time(b) for a, b in zip(ev_a, ev_b)]
        if ws > 1:
            torch.distributed.barrier()
        clocks = clk.summary()
        total_ms = t_start.elapsed_time(t_end)
        status = B.moe_get_device_status(su.plan)
        if status != B.MOE_OK:
            raise RuntimeError(f"{sh.name}: device status after timing: "
                               + B.moe_status_string(status))
        del g_steps, g_kern, g_rem

        # e2e: pinned host x in, pinned host out back, every step, through
        # the public moe_forward call
        x_host = torch.from_numpy(su.x_bits.view(np.int16)).pin_memory()
        out_host = torch.empty((T, sh.d), dtype=torch.float32).pin_memory()
        e_start = torch.cuda.Event(enable_timing=True)
        e_end = torch.cuda.Event(enable_timing=True)
        K2 = max(1, K // 4)
        torch.cuda.synchronize(dev)
        e_start.record(stream)
        for i in range(K2):
            su.x.copy_(x_host, non_blocking=True)
            B.moe_forward(su.plan, su.layers[i % su.n_inst].weights, su.x.data_ptr(), T, sh.k,
                          sh.wfmt, su.out.data_ptr(), None, st)
            out_host.copy_(su.out, non_blocking=True)
        e_end.record(stream)
        torch.cuda.synchronize(dev)
        e2e_ms = e_start.elapsed_time(e_end)

    t_max, e2e_max = reduce_max_over_ranks([total_ms, e2e_ms], device=dev)
    return {"K": K, "K2": K2, "S": S, "t_max": t_max, "e2e_max": e2e_max, "kern_ms": kern_ms,
            "launches": launches_per_step * K, "launches_per_step": launches_per_step,
            "act_bytes": act_bytes, "acts": acts, "act_flops": act_flops, "clocks": clocks}


def _entry(su: "_Setup", m: dict, ws: int, peaks):
    """The JSON fields of one measured workload."""
    from mixture_experts_layer_43_b200 import binding as B  # noqa: F401
    hbm_gbs, bf16_tf, bf16_tf_sus, peak_src = peaks
    sh, K, n_inst = su.sh, m["K"], su.n_inst
    T = sh.T
    tokens_per_s = job_tokens_per_s(ws, T, K, m["t_max"])
    kern_evt_s = float(np.mean(m["kern_ms"])) / 1e3
    # A decode step is exactly one launch (the fused kernel), so its duration
    # is the graph step time (event nodes around such short kernels add
    # their own overhead); prefill: event nodes around the two GEMM launches.
    kern_avg_s = kern_evt_s if su.prefill else min(kern_evt_s, m["t_max"] / K / 1e3)
    alg_bytes = float(np.mean([m["act_bytes"][i % n_inst] for i in range(K)]))
    alg_flops = float(np.mean([m["act_flops"][i % n_inst] for i in range(K)]))
    if su.prefill:
        src_sha = _kernel_src_sha(["prefill.cu", "moe_internal.cuh"])
        achieved = alg_flops / kern_avg_s / 1e12
        roof = {"bound": "tensor", "kernel": "prefill_gemm_kernel (gate/up + down launches)",
                "achieved": achieved, "peak": bf16_tf_sus, "unit": "TFLOP/s",
                "frac": achieved / bf16_tf_sus,
                "traffic": _profile_traffic("prefill_gemm_kernel", sh.name, src_sha),
                "algorithmic_flops_per_launch": alg_flops,
                "kernel_ms_avg": kern_avg_s * 1e3,
                "frac_of_burst_peak": achieved / bf16_tf,
                "peak_source": (f"{peak_src} (MEASURED_PEAKS.json bf16_tflops_sustained; "
                                "the GEMMs run inside a seconds-long loop)")}
        l2 = (f"inputs larger than L2: each step reads {su.per_inst / 1e9:.2f} GB of expert "
              f"weights and {T * sh.d * 2 / 1e6:.1f} MB of x; {n_inst} instance(s)")
    else:
        src_sha = _kernel_src_sha(["decode.cu", "moe_internal.cuh"])
        alg_bytes += sh.E * sh.d * 4            # the fused kernel also reads the router
        achieved = alg_bytes / kern_avg_s / 1e9
        roof = {"bound": "hbm", "kernel": "decode_fused_kernel (whole layer, one launch)",
                "achieved": achieved, "peak": hbm_gbs, "unit": "GB/s",
                "frac": achieved / hbm_gbs,
                "traffic": _profile_traffic("decode_fused_kernel", sh.name, src_sha),
                "algorithmic_bytes_per_launch": alg_bytes,
                "kernel_ms_avg": kern_avg_s * 1e3,
                "kernel_ms_event_nodes": kern_evt_s * 1e3,
                "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs, copy)"}
        l2 = ("inputs larger than L2: each step streams "
              f"{alg_bytes / 1e9:.3f} GB of distinct expert weights; "
              f"{n_inst} layer instance(s) rotated")
    return {
        "value": tokens_per_s, "unit": "tokens/s", "steps": K, "ms_per_step": m["t_max"] / K,
        "dtype": _dtype(sh),
        "config": {"workload": sh.name, "shape": synth.describe(sh), "T": T,
                   "instances": n_inst, "graph_steps": m["S"],
                   "timing": ("CUDA-graph replays of whole steps; kernel time from event "
                              "nodes in a second graph around each moe_forward (decode: the "
                              "single fused kernel) or moe_experts (prefill: the two GEMMs)"),
                   "l2": l2,
                   "active_experts_per_step": float(np.mean(m["acts"])),
                   "weights": ("host-generated by synth" if su.base is not None else
                               "drawn on the device with the workload's distributions")},
        "roofline": roof,
        "e2e": {"value": job_tokens_per_s(ws, T, m["K2"], m["e2e_max"]), "unit": "tokens/s",
                "h2d_bytes_per_step": T * sh.d * 2, "d2h_bytes_per_step": T * sh.d * 4},
        "gpu_launches": m["launches"],
        "clocks": m["clocks"],
    }


def _dtype(sh):
    return {synth.WFMT_BF16: "bf16", synth.WFMT_Q4_0: "q4_0/bf16",
            synth.WFMT_Q8_0: "q8_0/bf16", synth.WFMT_Q5_0: "q5_0/bf16",
            synth.WFMT_Q6_K: "q6_k/bf16", synth.WFMT_BF16_F16DOWN: "bf16 (fp16 down)"}[sh.wfmt]


def _read_stream_gbs(dev, stream) -> float:
    """A read-only streaming reference measured on this GPU: torch.sum over
    4 GiB of float32 resident on the device (each byte read once), best of
    five timed with CUDA events on the launching stream.  The copy peak reads
    and writes every byte; a read-only stream could run faster, and the
    decode kernel only reads weights, so both are reported."""
    import torch
    n = (4 << 30) // 4
    buf = torch.ones(n, dtype=torch.float32, device=dev)
    best = float("inf")
    with torch.cuda.stream(stream):
        for _ in range(2):
            buf.sum()
        for _ in range(5):
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            buf.sum()
            b.record(stream)
            stream.synchronize()
            best = min(best, a.elapsed_time(b))
    del buf
    torch.cuda.empty_cache()
    return (4 << 30) / (best / 1e3) / 1e9


def run_b200(args, sh):
    import torch

    ws, rank, local = _dist()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if ws > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    peaks = _peaks()
    stream = torch.cuda.Stream(device=dev)
    uuid = str(torch.cuda.get_device_properties(dev).uuid)
    if uuid and not uuid.startswith("GPU-"):
        uuid = "GPU-" + uuid

    # the headline workload: exactly --steps timed steps
    su = _Setup(sh, args, dev, stream, host_inputs=True)
    m = _measure(su, args, uuid, exact_steps=max(1, args.steps), ws=ws)
    head = _entry(su, m, ws, peaks)
    base = su.base
    su.destroy()
    del su
    torch.cuda.empty_cache()

    # the other seeded workloads, each its own entry
    configs = {}
    if not args.only_workload:
        for name in ALL_WORKLOADS:
            if name == sh.name:
                continue
            wsh = synth.WORKLOADS[name]
            small = wsh.name.startswith("tiny")
            su = _Setup(wsh, args, dev, stream, host_inputs=small)
            mm = _measure(su, args, uuid, min_ms=MIN_TIMED_MS, ws=ws)
            configs[name] = _entry(su, mm, ws, peaks)
            su.destroy()
            del su
            torch.cuda.empty_cache()

    line = {
        "metric": METRIC, "value": head["value"], "unit": "tokens/s", "n_gpus": ws,
        "steps": head["steps"], "steps_requested": args.steps, "warmup": args.warmup,
        "ms_per_step": head["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": head["dtype"],
        "data": "synthetic (seeded N(0,0.02) weights, N(0,1) x; no trained weights)",
        "config": dict(head["config"],
                       parallelism=f"replicas x{ws}" if ws > 1 else "single GPU"),
        "roofline": head["roofline"],
        "e2e": head["e2e"],
        "gpu_launches": head["gpu_launches"],
        "clocks": head["clocks"],
    }
    if not head["roofline"]["unit"] == "TFLOP/s":
        rs = _read_stream_gbs(dev, stream)
        line["roofline"] = dict(line["roofline"], read_stream_gbs=rs,
                                frac_of_read_stream=line["roofline"]["achieved"] / rs,
                                read_stream_note=("reference: torch.sum over 4 GiB of float32 on "
                                                  "this GPU, read-only; frac stays against the "
                                                  "copy peak"))
    if configs:
        configs[sh.name] = {k: head[k] for k in head}
        line["configs"] = configs
        line["configs_note"] = (
            "one entry per seeded workload, keyed by workload name, each timed with the same "
            f"protocol; entries other than the headline time max(--steps, {MIN_TIMED_MS:.0f} ms "
            "worth of) steps so the clock sampler sees the timed region")
    if ws == 1 and rank == 0 and not args.no_cpu_baseline:
        line["cpu_baseline"] = _cpu_baseline(base, sh)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    return 0


def run_sweep(args):
    """Achieved HBM bandwidth of the fused decode kernel against the bytes
    one launch reads (the pages' bandwidth-vs-bytes-per-kernel measurement,
    cold data): a T=8, d=4096, E=8, k=2 layer with F from 32 to 14336, each
    point timed on a rotation of layer copies larger than 4x L2.  Prints one
    JSON line per point."""
    import torch
    from mixture_experts_layer_43_b200 import binding as B
    from mixture_experts_layer_43_b200 import device as D
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    hbm_gbs = _peaks()[0]
    stream = torch.cuda.Stream(device=dev)
    st = stream.cuda_stream
    for F in (32, 64, 128, 256, 512, 1024, 2048, 4096, 8192, 14336):
        sh = synth.MoEShape(f"sweep_F{F}", T=8, d=4096, E=8, k=2, F=F)
        base, xb = D.random_bf16_layer(sh, seed=args.seed, device=str(dev))
        x = D.upload_x(xb, dev)
        out = torch.empty((sh.T, sh.d), dtype=torch.float32, device=dev)
        plan = B.moe_plan_create(base.config(sh.T))
        routing = D.Routing(sh.T, sh.k, sh.E, dev)
        with torch.cuda.stream(stream):
            B.moe_forward(plan, base.weights, x.data_ptr(), sh.T, sh.k, sh.wfmt, out.data_ptr(), routing.struct, st)
        stream.synchronize()
        act, n_act = _active_bytes(sh, routing.counts.cpu().numpy(), 0)
        act += sh.E * sh.d * 4
        n_inst = int(min(256, max(1, -(-4 * L2_BYTES // act))))
        n_inst = max(1, min(n_inst, int(40e9 // (base.weight_bytes() + 1))))
        layers = [base] + [base.clone() for _ in range(n_inst - 1)]
        S = n_inst * max(1, -(-64 // n_inst))
        with torch.cuda.stream(stream):
            for i in range(args.warmup):
                B.moe_forward(plan, layers[i % n_inst].weights, x.data_ptr(), sh.T, sh.k, sh.wfmt, out.data_ptr(), None, st)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                for i in range(S):
                    B.moe_forward(plan, layers[i % n_inst].weights, x.data_ptr(), sh.T, sh.k,
                                  sh.wfmt, out.data_ptr(), None, st)
            g.replay()
            stream.synchronize()
            R = max(3, min(200, -(-args.steps // S)))
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(R):
                g.replay()
            b.record(stream)
            stream.synchronize()
        us = a.elapsed_time(b) * 1e3 / (R * S)
        gbs = act / (us * 1e-6) / 1e9
        print(json.dumps({"sweep": "bytes_per_launch", "F": F, "bytes_per_launch": act,
                          "active_experts": n_act, "us_per_launch": us, "achieved_gbs": gbs,
                          "frac_of_peak": gbs / hbm_gbs, "instances": n_inst}), flush=True)
        del g
        B.moe_plan_destroy(plan)
        del layers, base
        torch.cuda.empty_cache()
    return 0


def run_sweep_t(args):
    """Decode vs prefill regime on the 35B-A3B-shaped bf16 layer (d=2048,
    E=256, k=8, F=512, 1 shared expert) for T = 1..8 (both regimes run
    there) and the prefill regime for T = 16..256: time per layer call and
    tokens/s, one JSON line per (regime, T), timed on rotated layer copies."""
    import torch
    from mixture_experts_layer_43_b200 import binding as B
    from mixture_experts_layer_43_b200 import device as D
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.Stream(device=dev)
    st = stream.cuda_stream
    t_max = 256
    sh = synth.MoEShape("a3b_sweep_T", T=t_max, d=2048, E=256, k=8, F=512, S=1, Fs=512)
    base, xb = D.random_bf16_layer(sh, seed=args.seed, device=str(dev))
    n_inst = 24
    layers = [base] + [base.clone() for _ in range(n_inst - 1)]
    x = D.upload_x(xb, dev)
    out = torch.empty((t_max, sh.d), dtype=torch.float32, device=dev)
    plans = {r: B.moe_plan_create(base.config(t_max if r == B.MOE_REGIME_PREFILL else 8, r))
             for r in (B.MOE_REGIME_DECODE, B.MOE_REGIME_PREFILL)}
    points = [(B.MOE_REGIME_DECODE, T) for T in range(1, 9)] + \
             [(B.MOE_REGIME_PREFILL, T) for T in (1, 2, 4, 8, 16, 32, 64, 128, 256)]
    for regime, T in points:
        plan = plans[regime]
        S = n_inst * 2
        with torch.cuda.stream(stream):
            for i in range(args.warmup):
                B.moe_forward(plan, layers[i % n_inst].weights, x.data_ptr(), T, sh.k, sh.wfmt, out.data_ptr(), None, st)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                for i in range(S):
                    B.moe_forward(plan, layers[i % n_inst].weights, x.data_ptr(), T, sh.k, sh.wfmt, out.data_ptr(),
                                  None, st)
            g.replay()
            stream.synchronize()
            R = 20
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(R):
                g.replay()
            b.record(stream)
            stream.synchronize()
        us = a.elapsed_time(b) * 1e3 / (R * S)
        print(json.dumps({"sweep": "tokens_per_call", "regime": "decode" if regime == 1 else "prefill",
                          "T": T, "us_per_call": us, "tokens_per_s": T / (us * 1e-6)}), flush=True)
        del g
    for p in plans.values():
        B.moe_plan_destroy(p)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__,
                                 formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=("b200", "reference"), default="b200")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(synth.WORKLOADS))
    ap.add_argument("--instances", type=int, default=0)
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--only-workload", action="store_true",
                    help="measure only --workload (no per-workload `configs` entries)")
    ap.add_argument("--sweep-bytes", action="store_true",
                    help="bandwidth vs bytes per launch of the decode kernel, one JSON line per point")
    ap.add_argument("--sweep-t", action="store_true",
                    help="decode vs prefill regime over tokens per call, one JSON line per point")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.sweep_bytes:
        return run_sweep(args)
    if args.sweep_t:
        return run_sweep_t(args)
    sh = synth.WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, sh)
    return run_b200(args, sh)


if __name__ == "__main__":
    sys.exit(main())
