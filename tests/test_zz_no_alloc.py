"""moe_route_noalloc: the routing step for callers that cannot allocate
device memory (engines that forbid cudaMalloc on their serving path, plugin
enqueue steps that may only launch work).  Its scratch lives in a static
device array of the library instead of a plan workspace.

Checked through the C ABI on two calls in a row with different batches:
  * against the existing plan-based entry point (moe_route +
    moe_routing_get): ids, counts, offsets and slot order bit-exact, weights
    within the parity tests' routing tolerance, `out` zero-filled;
  * against the fp64 oracle's router and bucketing directly;
  * a call after the first one allocates no device memory (free memory and
    torch's allocator both unchanged across it);
  * its sticky error word reads clean through moe_route_noalloc_status.
This file sorts last so that a run stopping at the first failure has run
every other test before it."""
import numpy as np
import pytest
import torch

import oracle
from mixture_experts_layer_43_b200 import binding as B
from mixture_experts_layer_43_b200 import device as D
from mixture_experts_layer_43_b200 import synth

from gpu_util import W_ABS, check_tie_choice, w_rtol, waived_tokens

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def _routing_planned(layer, x_bits, T):
    sh = layer.shape
    plan = B.moe_plan_create(layer.config(T, B.MOE_REGIME_DECODE))
    try:
        x = D.upload_x(x_bits, "cuda")
        out = torch.full((T, sh.d), 3.0, device="cuda")
        r = D.Routing(T, sh.k, sh.E, "cuda")
        st = torch.cuda.current_stream().cuda_stream
        B.moe_route(plan, layer.weights, x.data_ptr(), T, sh.k, sh.wfmt, out.data_ptr(), st)
        B.moe_routing_get(plan, T, r.struct, st)
        torch.cuda.synchronize()
        return r.numpy(), out.cpu().numpy()
    finally:
        B.moe_plan_destroy(plan)


def _routing_noalloc(layer, x_bits, T):
    sh = layer.shape
    x = D.upload_x(x_bits, "cuda")
    out = torch.full((T, sh.d), 3.0, device="cuda")
    r = D.Routing(T, sh.k, sh.E, "cuda")
    B.moe_route_noalloc(layer.config(T), layer.weights, x.data_ptr(), T, out.data_ptr(),
                        r.struct, torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    return r.numpy(), out.cpu().numpy()


SHAPE = synth.MoEShape("noalloc", T=8, d=2048, E=256, k=8, F=32, S=1, Fs=32, zipf_bias=1.1)


def test_route_noalloc_matches_planned_route_twice():
    inp = synth.make_inputs(SHAPE, seed=21)
    layer = D.DeviceLayer(inp)
    other = synth.make_inputs(SHAPE, seed=22).x
    for x_bits, T in ((inp.x, 8), (other[:5], 5)):
        want, want_out = _routing_planned(layer, x_bits, T)
        got, got_out = _routing_noalloc(layer, x_bits, T)
        ids, w, counts, offsets, slot_pair = got
        assert np.array_equal(ids, want[0])
        np.testing.assert_allclose(w, want[1], rtol=w_rtol(SHAPE.d), atol=W_ABS)
        assert np.array_equal(counts, want[2])
        assert np.array_equal(offsets, want[3])
        assert np.array_equal(slot_pair, want[4])
        assert np.all(got_out == 0.0) and np.all(want_out == 0.0)
    assert B.moe_route_noalloc_status() == B.MOE_OK


def test_route_noalloc_matches_oracle_twice():
    inp = synth.make_inputs(SHAPE, seed=23)
    layer = D.DeviceLayer(inp)
    other = synth.make_inputs(SHAPE, seed=24).x
    for x_bits, T in ((inp.x, 8), (other[:3], 3)):
        (ids, w, counts, offsets, slot_pair), _ = _routing_noalloc(layer, x_bits, T)
        logits, o_ids, o_w = oracle.route(x_bits, inp.router_w, inp.router_b, SHAPE.k)
        waived = waived_tokens(logits, SHAPE.k)
        ok = np.all(ids == o_ids, axis=1)
        assert np.all(ok | waived)
        for t in np.where(~ok)[0]:
            check_tie_choice(logits[t], ids[t], SHAPE.k)
        np.testing.assert_allclose(w[ok], o_w[ok], rtol=w_rtol(SHAPE.d), atol=W_ABS)
        c, o, sp = oracle.buckets(ids.astype(np.int32), SHAPE.E)
        assert np.array_equal(counts, c)
        assert np.array_equal(offsets, o)
        assert np.array_equal(slot_pair, sp)
    assert B.moe_route_noalloc_status() == B.MOE_OK


def test_route_noalloc_allocates_nothing_after_first_call():
    inp = synth.make_inputs(SHAPE, seed=25)
    layer = D.DeviceLayer(inp)
    T = 8
    x = D.upload_x(inp.x, "cuda")
    out = torch.empty((T, SHAPE.d), device="cuda")
    r = D.Routing(T, SHAPE.k, SHAPE.E, "cuda")
    cfg = layer.config(T)
    st = torch.cuda.current_stream().cuda_stream
    # the first call may load the library's module (lazy loading): a warm-up
    B.moe_route_noalloc(cfg, layer.weights, x.data_ptr(), T, out.data_ptr(), r.struct, st)
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    torch0 = torch.cuda.memory_allocated()
    for _ in range(3):
        B.moe_route_noalloc(cfg, layer.weights, x.data_ptr(), T, out.data_ptr(), r.struct, st)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert torch.cuda.memory_allocated() == torch0
    assert free1 >= free0, f"device free memory fell by {free0 - free1} bytes"
    assert B.moe_route_noalloc_status() == B.MOE_OK


def test_route_noalloc_rejects_too_many_tokens():
    sh = synth.MoEShape("noalloc_big", T=9, d=256, E=8, k=2, F=32)
    inp = synth.make_inputs(sh, seed=1)
    layer = D.DeviceLayer(inp)
    x = D.upload_x(inp.x, "cuda")
    out = torch.zeros((9, sh.d), device="cuda")
    r = D.Routing(9, sh.k, sh.E, "cuda")
    with pytest.raises(B.MoeError) as e:
        B.moe_route_noalloc(layer.config(9), layer.weights, x.data_ptr(), 9, out.data_ptr(),
                            r.struct, 0)
    assert e.value.status == B.MOE_ERR_INVALID_ARG
