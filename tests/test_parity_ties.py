"""The tie rule on the GPU: among equal router logits the lower expert index
wins, and each token's experts come out in descending-logit order.  These
cases are exact ties, which the near-tie waiver of the other parity tests
would excuse; here the ids must match the oracle's bit for bit.

  * a zero router: every logit is exactly 0, so every token must pick experts
    0..k-1 with weights 1/k;
  * a router whose second half of rows repeats the first half: each token's
    logits come in equal pairs (e, e + E/2), computed the same way on both
    sides, so the lower index must come first within each pair.
Both regimes (the fused decode launch and the prefill kernels) are covered."""
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


CASES = [
    (synth.MoEShape("tie_decode", T=8, d=512, E=16, k=4, F=64, S=1, Fs=64),
     B.MOE_REGIME_DECODE),
    (synth.MoEShape("tie_decode_E256", T=3, d=256, E=256, k=8, F=32), B.MOE_REGIME_DECODE),
    (synth.MoEShape("tie_prefill", T=96, d=256, E=16, k=4, F=128, S=1, Fs=128),
     B.MOE_REGIME_PREFILL),
]


def _run(inp, regime):
    layer = D.DeviceLayer(inp)
    return run_gpu(layer, inp.x, inp.shape.T, regime=regime)


def _compare(inp, out, routing, res, regime):
    return compare(inp, out, routing, res, prefill=regime == B.MOE_REGIME_PREFILL)


@pytest.mark.parametrize("sh,regime", CASES, ids=[c[0].name for c in CASES])
def test_zero_router_picks_lowest_indices(sh, regime):
    inp = synth.make_inputs(sh, seed=12)
    inp.router_w = np.zeros_like(inp.router_w)
    out, routing, _ = _run(inp, regime)
    ids, w = routing[0], routing[1]
    want = np.tile(np.arange(sh.k, dtype=np.int32), (sh.T, 1))
    assert np.array_equal(ids, want)
    np.testing.assert_allclose(w, 1.0 / sh.k, rtol=1e-6)
    res = oracle.forward(inp)
    assert np.array_equal(res[1], want)                     # the oracle agrees
    _compare(inp, out, routing, res, regime)


@pytest.mark.parametrize("sh,regime", CASES, ids=[c[0].name for c in CASES])
def test_duplicated_router_rows_pick_lower_index_first(sh, regime):
    inp = synth.make_inputs(sh, seed=13)
    half = sh.E // 2
    inp.router_w = np.ascontiguousarray(np.concatenate([inp.router_w[:half]] * 2))
    out, routing, _ = _run(inp, regime)
    ids = routing[0]
    res = oracle.forward(inp)
    o_ids, lg = res[1], res[3]
    # tokens whose top-k is made of whole pairs and whose k-th and (k+1)-th
    # distinct logits are well apart: the order is fixed by the tie rule alone
    s = -np.sort(-lg, axis=1)
    sep = (s[:, sh.k - 1] - s[:, sh.k]) > 1e-4 * np.abs(s[:, sh.k - 1])
    assert sep.sum() >= sh.T // 2
    for t in np.where(sep)[0]:
        assert np.array_equal(ids[t], o_ids[t]), (t, ids[t], o_ids[t])
        for j in range(0, sh.k, 2):                         # (e, e + E/2) pairs, e first
            assert ids[t, j] + half == ids[t, j + 1], ids[t]
    _compare(inp, out, routing, res, regime)
