"""GPU parity of the decode regime (T <= 8): the C-ABI call against the fp64
oracle on seeded inputs, at the full sizes of the decode workloads and at
small shapes that cover ragged tails, k = E, E = 1, several shared experts
and T = 0."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from mixture_experts_layer_43_b200 import binding as B
from mixture_experts_layer_43_b200 import device as D
from mixture_experts_layer_43_b200 import synth

from gpu_util import DECODE_TRIPWIRE, compare, run_gpu, run_gpu_split

pytestmark = pytest.mark.gpu

W = synth.WORKLOADS
SMALL = [
    # ragged: d = 3 x 128 (partial stages), F = 3 slices of 32, Fs != F
    synth.MoEShape("ragged_bf16", T=3, d=384, E=5, k=3, F=96, S=1, Fs=64),
    synth.MoEShape("ragged_q4", T=3, d=384, E=5, k=3, F=96, S=1, Fs=64, wfmt=synth.WFMT_Q4_0),
    synth.MoEShape("k_eq_E", T=2, d=256, E=4, k=4, F=64),
    synth.MoEShape("one_expert", T=5, d=128, E=1, k=1, F=32),
    synth.MoEShape("two_shared", T=6, d=256, E=16, k=2, F=64, S=2, Fs=96),
    synth.MoEShape("two_shared_q4", T=7, d=256, E=16, k=2, F=64, S=2, Fs=96,
                   wfmt=synth.WFMT_Q4_0),
    synth.MoEShape("multi_unit", T=8, d=1024, E=8, k=2, F=2048, S=1, Fs=512),
    synth.MoEShape("multi_unit_q4", T=8, d=1024, E=8, k=2, F=2048, S=1, Fs=512,
                   wfmt=synth.WFMT_Q4_0),
    synth.MoEShape("biased", T=8, d=512, E=64, k=6, F=128, S=2, Fs=128, zipf_bias=1.1),
    synth.MoEShape("ragged_q8", T=3, d=384, E=5, k=3, F=96, S=1, Fs=64, wfmt=synth.WFMT_Q8_0),
    synth.MoEShape("two_shared_q8", T=7, d=256, E=16, k=2, F=64, S=2, Fs=96,
                   wfmt=synth.WFMT_Q8_0),
    synth.MoEShape("multi_unit_q8", T=8, d=1024, E=8, k=2, F=2048, S=1, Fs=512,
                   wfmt=synth.WFMT_Q8_0),
    # Q8_0 with 72 block columns (two phase-A chunks per row group, the second
    # partial) and at the interface's limits
    synth.MoEShape("chunked_q8", T=5, d=2304, E=8, k=2, F=96, S=1, Fs=64, wfmt=synth.WFMT_Q8_0),
    synth.MoEShape("max_limits_q8", T=8, d=256, E=1024, k=16, F=64, S=8, Fs=32,
                   wfmt=synth.WFMT_Q8_0),
    # the interface's limits: E = 1024 experts, k = 16, 8 shared experts, T = 8
    # (128 token-expert pairs, a 32-word expert mask, the widest register top-k)
    synth.MoEShape("max_limits", T=8, d=256, E=1024, k=16, F=64, S=8, Fs=32),
    synth.MoEShape("max_limits_q4", T=8, d=256, E=1024, k=16, F=64, S=8, Fs=32,
                   wfmt=synth.WFMT_Q4_0),
    # Q5_0: 32-row slices with a partial last down box (d = 384), two shared
    # experts of another size, 64-row slices over several stages, the limits
    synth.MoEShape("ragged_q5", T=3, d=384, E=5, k=3, F=96, S=1, Fs=64, wfmt=synth.WFMT_Q5_0),
    synth.MoEShape("two_shared_q5", T=7, d=256, E=16, k=2, F=64, S=2, Fs=96,
                   wfmt=synth.WFMT_Q5_0),
    synth.MoEShape("multi_unit_q5", T=8, d=1024, E=8, k=2, F=2048, S=1, Fs=512,
                   wfmt=synth.WFMT_Q5_0),
    synth.MoEShape("max_limits_q5", T=8, d=256, E=1024, k=16, F=64, S=8, Fs=32,
                   wfmt=synth.WFMT_Q5_0),
    # q6_K (256-wide super-blocks): 24 block columns (a partial warp split), 72 block
    # columns (two phase-A chunks, the second one partial), the interface limits
    synth.MoEShape("ragged_q6", T=3, d=768, E=5, k=3, F=256, S=1, Fs=512, wfmt=synth.WFMT_Q6_K),
    synth.MoEShape("chunked_q6", T=5, d=2304, E=8, k=2, F=512, S=1, Fs=256,
                   wfmt=synth.WFMT_Q6_K),
    synth.MoEShape("max_limits_q6", T=8, d=256, E=1024, k=16, F=256, S=8, Fs=256,
                   wfmt=synth.WFMT_Q6_K),
    # Q4_0 with 72 block columns: two phase-A chunks per row group
    synth.MoEShape("chunked_q4", T=5, d=2304, E=8, k=2, F=96, S=1, Fs=64, wfmt=synth.WFMT_Q4_0),
    # bf16 gate/up with fp16 down matrices (h in fp16): 32- and 64-row slices
    synth.MoEShape("ragged_f16down", T=3, d=384, E=5, k=3, F=96, S=1, Fs=64,
                   wfmt=synth.WFMT_BF16_F16DOWN),
    synth.MoEShape("multi_unit_f16down", T=8, d=1024, E=8, k=2, F=2048, S=1, Fs=512,
                   wfmt=synth.WFMT_BF16_F16DOWN),
]


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def _check(sh, seed=0, T=None, split=False):
    """split=False: moe_forward (the single fused cooperative launch);
    split=True: moe_route + moe_experts (router kernel, then experts kernel)."""
    inp = synth.make_inputs(sh, seed=seed)
    layer = D.DeviceLayer(inp)
    T = sh.T if T is None else T
    if split:
        out, routing, launches = run_gpu_split(layer, inp.x, T)
        assert launches == 2
    else:
        out, routing, launches = run_gpu(layer, inp.x, T)
        assert launches == 1
    sub = synth.MoEInputs(sh, inp.x[:T], inp.router_w, inp.router_b, inp.gate, inp.up,
                          inp.down, inp.shared_gate, inp.shared_up, inp.shared_down)
    res = oracle.forward(sub)
    return compare(sub, out, routing, res, tripwire=DECODE_TRIPWIRE)


@pytest.mark.parametrize("name", ["tiny_T4_d256_E8k2_F512", "a3b_T1_d2048_E256k8_F512_S1",
                                  "a3b_q4_T1_d2048_E256k8_F512_S1",
                                  "a3b_q4_T8_d2048_E256k8_F512_S1",
                                  "a3b_T8_d2048_E256k8_F512_S1",
                                  "a3b_q8_T1_d2048_E256k8_F512_S1",
                                  "a3b_q8_T8_d2048_E256k8_F512_S1",
                                  "a3b_q5_T1_d2048_E256k8_F512_S1",
                                  "a3b_q5_T8_d2048_E256k8_F512_S1",
                                  "a3b_q6_T1_d2048_E256k8_F512_S1",
                                  "a3b_q6_T8_d2048_E256k8_F512_S1"])
def test_decode_workloads_full_size(name):
    err = _check(W[name])
    print(f"{name}: rel L2 {err:.3e}")


def test_decode_mixtral_full_size():
    err = _check(W["mixtral_T8_d4096_E8k2_F14336"])
    print(f"mixtral: rel L2 {err:.3e}")


@pytest.mark.parametrize("sh", SMALL, ids=[s.name for s in SMALL])
def test_decode_small_shapes(sh):
    _check(sh, seed=1)


# Router widths and top-k sizes that select every variant of the warp top-k:
# logits per lane 2, 4 and 8 (E = 40, 100, 200; 1024 is max_limits above)
# with 2, 4 and 16 unrolled selection rounds (k = 2, 3, 12)
TOPK_SHAPES = [
    synth.MoEShape("topk_E40_k2", T=6, d=256, E=40, k=2, F=64, S=1, Fs=64),
    synth.MoEShape("topk_E100_k3", T=4, d=256, E=100, k=3, F=64, S=1, Fs=64),
    synth.MoEShape("topk_E200_k12", T=8, d=256, E=200, k=12, F=64, S=1, Fs=64),
    synth.MoEShape("topk_E200_k12_q4", T=3, d=256, E=200, k=12, F=64, S=1, Fs=64,
                   wfmt=synth.WFMT_Q4_0),
]


@pytest.mark.parametrize("sh", TOPK_SHAPES, ids=[s.name for s in TOPK_SHAPES])
def test_decode_topk_variants(sh):
    _check(sh, seed=5)


SPLIT = SMALL[:6] + [SMALL[10], SMALL[-4], W["a3b_q4_T8_d2048_E256k8_F512_S1"],
                     W["a3b_q6_T8_d2048_E256k8_F512_S1"], W["a3b_q8_T8_d2048_E256k8_F512_S1"]]


@pytest.mark.parametrize("sh", SPLIT, ids=[s.name for s in SPLIT])
def test_decode_two_launch_path(sh):
    _check(sh, seed=5, split=True)


@pytest.mark.parametrize("T", [1, 2, 5, 8])
def test_decode_every_T(T):
    _check(synth.MoEShape("tsweep", T=8, d=512, E=32, k=4, F=256, S=1, Fs=256), seed=2, T=T)


def test_decode_T0_enqueues_nothing():
    sh = synth.MoEShape("t0", T=1, d=256, E=4, k=2, F=64)
    inp = synth.make_inputs(sh)
    layer = D.DeviceLayer(inp)
    plan = B.moe_plan_create(layer.config(4))
    try:
        out = torch.full((1, sh.d), 7.0, device="cuda")
        x = D.upload_x(inp.x, "cuda")
        B.moe_forward(plan, layer.weights, x.data_ptr(), 0, sh.k, sh.wfmt, out.data_ptr())
        assert B.moe_last_launch_count(plan) == 0
        torch.cuda.synchronize()
        assert torch.all(out == 7.0)
    finally:
        B.moe_plan_destroy(plan)


def test_decode_repeatable():
    """Routing is bitwise repeatable; the output differs at most by the order
    of the fp32 atomic additions of the combine."""
    sh = synth.MoEShape("rep", T=8, d=1024, E=32, k=4, F=512, S=1, Fs=512)
    inp = synth.make_inputs(sh, seed=4)
    layer = D.DeviceLayer(inp)
    plan = B.moe_plan_create(layer.config(8))
    try:
        o1, r1, _ = run_gpu(layer, inp.x, 8, plan=plan)
        o2, r2, _ = run_gpu(layer, inp.x, 8, plan=plan)
    finally:
        B.moe_plan_destroy(plan)
    for a, b in zip(r1, r2):
        assert np.array_equal(a, b)
    assert np.max(np.abs(o1 - o2)) <= 1e-5 * np.max(np.abs(o1))


def test_decode_invalid_call_enqueues_nothing():
    sh = synth.MoEShape("bad", T=2, d=256, E=4, k=2, F=64)
    inp = synth.make_inputs(sh)
    layer = D.DeviceLayer(inp)
    plan = B.moe_plan_create(layer.config(2))
    try:
        x = D.upload_x(inp.x, "cuda")
        out = torch.zeros((2, sh.d), device="cuda")
        with pytest.raises(B.MoeError) as e:
            B.moe_forward(plan, layer.weights, x.data_ptr(), 3, sh.k, sh.wfmt, out.data_ptr())  # T > t_max
        assert e.value.status == B.MOE_ERR_INVALID_ARG
        with pytest.raises(B.MoeError):
            B.moe_forward(plan, layer.weights, x.data_ptr() + 2, 2, sh.k, sh.wfmt,
                          out.data_ptr())                                  # misaligned
        w = B.moe_weights_t()
        w.router_w = layer.weights.router_w
        with pytest.raises(B.MoeError):
            B.moe_forward(plan, w, x.data_ptr(), 2, sh.k, sh.wfmt, out.data_ptr())  # missing weights
        # k and the weight format restate the plan's: a mismatch is rejected
        for k, wfmt in ((sh.k + 1, sh.wfmt), (sh.k - 1, sh.wfmt), (sh.k, B.MOE_WFMT_Q4_0),
                        (sh.k, 7)):
            for call in (B.moe_forward, B.moe_route, B.moe_experts):
                with pytest.raises(B.MoeError) as e:
                    call(plan, layer.weights, x.data_ptr(), 2, k, wfmt, out.data_ptr())
                assert e.value.status == B.MOE_ERR_INVALID_ARG
        torch.cuda.synchronize()
        assert torch.all(out == 0.0)                                      # nothing ran
        assert B.moe_get_device_status(plan) == B.MOE_OK
    finally:
        B.moe_plan_destroy(plan)


def test_plan_reused_across_token_counts():
    """One plan, consecutive fused launches with T = 8, 1, 5, 8, 2, 8 and a
    fresh x each time: every call matches the oracle.  (A launch publishes
    router logits for all 8 token rows, tagged with the launch; rows beyond
    its own T must never pass for a later launch's.)"""
    sh8 = synth.MoEShape("reuse", T=8, d=512, E=64, k=6, F=128, S=1, Fs=128)
    base = synth.make_inputs(sh8, seed=41)
    layer = D.DeviceLayer(base)
    plan = B.moe_plan_create(layer.config(8))
    try:
        for j, T in enumerate((8, 1, 5, 8, 2, 8)):
            xb = synth.make_inputs(sh8, seed=200 + j, x_only=True).x[:T]
            inp = dataclasses.replace(base, shape=dataclasses.replace(sh8, T=T), x=xb)
            got, routing, launches = run_gpu(layer, xb, T, plan=plan)
            assert launches == 1
            compare(inp, got, routing, oracle.forward(inp))
    finally:
        B.moe_plan_destroy(plan)
