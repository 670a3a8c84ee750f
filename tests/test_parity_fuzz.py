"""Seeded random layer shapes in both regimes against the fp64 oracle: a net
for the combinations the hand-picked cases do not name -- ragged T, E and k,
odd widths, zero to two shared experts, every decode weight format, and
prefill experts whose tails fall on either side of the swapped-tile limit.
The bar is the one of the other parity tests (gpu_util.compare): ids, buckets
and slot order exact, routing weights within the fp32 bound, `out` within
the format's relative L2 bound (decode also under its 1e-4 tripwire)."""
import numpy as np
import pytest
import torch

import oracle
from mixture_experts_layer_43_b200 import binding as B
from mixture_experts_layer_43_b200 import device as D
from mixture_experts_layer_43_b200 import synth

from gpu_util import DECODE_TRIPWIRE, compare, run_gpu

pytestmark = pytest.mark.gpu

FORMATS = [synth.WFMT_BF16, synth.WFMT_Q4_0, synth.WFMT_Q8_0, synth.WFMT_Q5_0,
           synth.WFMT_Q6_K, synth.WFMT_BF16_F16DOWN]


def _decode_shapes(n, seed):
    rng = np.random.default_rng(seed)
    out = []
    for i in range(n):
        wfmt = FORMATS[i % len(FORMATS)]
        if wfmt == synth.WFMT_Q6_K:
            d = int(rng.choice([256, 512]))
            F = 256
            Fs = int(rng.choice([256, 512]))
        else:
            d = int(rng.choice([128, 256, 384, 512]))
            F = int(rng.choice([32, 64, 96, 160]))
            Fs = int(rng.choice([32, 64, 128]))
        E = int(rng.integers(1, 301))
        k = int(rng.integers(1, min(E, 16) + 1))
        S = int(rng.integers(0, 3))
        T = int(rng.integers(1, 9))
        out.append(synth.MoEShape(f"fuzz_dec{i}", T=T, d=d, E=E, k=k, F=F, S=S,
                                  Fs=Fs if S else 0, wfmt=wfmt))
    return out


def _prefill_shapes(n, seed):
    rng = np.random.default_rng(seed)
    out = []
    for i in range(n):
        wfmt = synth.WFMT_BF16_F16DOWN if i % 3 == 2 else synth.WFMT_BF16
        E = int(rng.integers(1, 65))
        k = int(rng.integers(1, min(E, 8) + 1))
        S = int(rng.integers(0, 3))
        out.append(synth.MoEShape(
            f"fuzz_pf{i}", T=int(rng.integers(9, 401)), d=int(rng.choice([256, 512])), E=E,
            k=k, F=int(rng.choice([64, 128, 192, 320])), S=S,
            Fs=int(rng.choice([64, 128])) if S else 0, wfmt=wfmt,
            zipf_bias=1.1 if i % 2 else 0.0))
    return out


DECODE = _decode_shapes(12, 20261203)
PREFILL = _prefill_shapes(8, 20261204)


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


@pytest.mark.parametrize("sh", DECODE, ids=[s.name for s in DECODE])
def test_fuzz_decode(sh):
    inp = synth.make_inputs(sh, seed=7)
    layer = D.DeviceLayer(inp)
    out, routing, launches = run_gpu(layer, inp.x, sh.T)
    assert launches == 1
    compare(inp, out, routing, oracle.forward(inp), tripwire=DECODE_TRIPWIRE)


@pytest.mark.parametrize("sh", PREFILL, ids=[s.name for s in PREFILL])
def test_fuzz_prefill(sh):
    inp = synth.make_inputs(sh, seed=7)
    layer = D.DeviceLayer(inp)
    out, routing, launches = run_gpu(layer, inp.x, sh.T, regime=B.MOE_REGIME_PREFILL)
    assert launches == 4
    compare(inp, out, routing, oracle.forward(inp), prefill=True)
