"""Failure detection without a GPU fault: a bounded device wait that runs out
reports MOE_ERR_TIMEOUT through the host, the context stays usable and the
plan recovers.  The fused decode kernel's wait for the other CTAs' router
logits is made to run out by a launch ticket count from which the CTAs derive
different tags (a flag nothing sets); nothing traps, faults or hangs."""
import numpy as np
import pytest
import torch

import oracle
from mixture_experts_layer_43_b200 import binding as B
from mixture_experts_layer_43_b200 import device as D
from mixture_experts_layer_43_b200 import synth

from gpu_util import compare, run_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def test_routing_wait_timeout_is_reported_and_recovered():
    sh = synth.MoEShape("stall", T=4, d=256, E=8, k=2, F=128, S=1, Fs=64)
    inp = synth.make_inputs(sh, seed=31)
    layer = D.DeviceLayer(inp)
    plan = B.moe_plan_create(layer.config(sh.T))
    try:
        x = D.upload_x(inp.x, "cuda")
        out = torch.zeros((sh.T, sh.d), device="cuda")
        st = torch.cuda.current_stream().cuda_stream
        B.moe_debug_stall_barrier(plan, st)
        B.moe_forward(plan, layer.weights, x.data_ptr(), sh.T, sh.k, sh.wfmt, out.data_ptr(), None, st)
        assert B.moe_last_launch_count(plan) == 1
        torch.cuda.synchronize()                       # the launch ends by itself
        # a second call before the status is read must not compute on the
        # ticket count the timeout left mid-round: it skips its work and its out
        # is NaN, never a plausible wrong value
        out2 = torch.zeros((sh.T, sh.d), device="cuda")
        B.moe_forward(plan, layer.weights, x.data_ptr(), sh.T, sh.k, sh.wfmt, out2.data_ptr(),
                      None, st)
        torch.cuda.synchronize()
        assert torch.all(torch.isnan(out2))
        assert B.moe_get_device_status(plan) == B.MOE_ERR_TIMEOUT
        assert B.moe_get_device_status(plan) == B.MOE_OK   # read-and-clear
        # the context and the plan are usable again: full parity on the next call
        got, routing, launches = run_gpu(layer, inp.x, sh.T, plan=plan)
        res = oracle.forward(inp)
        compare(inp, got, routing, res)
    finally:
        B.moe_plan_destroy(plan)
