"""Helpers of the GPU parity tests: run the layer through the C ABI and compare
it element by element with the fp64 oracle on the same seeded inputs.

Acceptance (the contract of the layer):
  * expert ids bit-exact, except for a token whose oracle gap between the
    k-th and (k+1)-th largest logit is below 1e-5 * |k-th logit| (a near tie
    that fp32 and fp64 may order differently); there the GPU's experts must
    still lie inside the tie band;
  * counts, offsets and the slot order bit-exact against the oracle's
    bucketing of the GPU's own ids (they are a pure function of the ids);
  * routing weights within relative c*sqrt(d)*2^-24: the GPU sums the d
    products of a logit in fp32, whose rounding error grows like sqrt(d)*2^-24
    times the partial sums (|partial sums| <~ 1 here), and a renormalised
    weight's relative error is the difference of two such logit errors.
    c = 5 for the decode router (fp32 FMA; observed 1.6 at d = 2048) and
    c = 24 for the prefill router, whose tensor-core accumulation of the
    three exact bf16 parts rounds its fp32 sums less tightly (observed 10.3 on
    the DeepSeek-shaped layer at d = 2048): a margin of 2 to 3 each;
  * out within relative L2 2e-3 (bf16 weights, also with fp16 down matrices)
    or 5e-3 (Q4_0, Q8_0, Q5_0 and q6_K weights) over every token: a token whose ids differ from the oracle's
    (a waived near tie) is compared with the oracle evaluated on the GPU's own
    ids and weights.  Callers may add a tighter tripwire: the decode kernels
    measure about 5e-6 in every format, so a regression of 20x fails long
    before the contract bound would.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from mixture_experts_layer_43_b200 import binding as B
from mixture_experts_layer_43_b200 import device as D
from mixture_experts_layer_43_b200 import synth

TOL = {synth.WFMT_BF16: 2e-3, synth.WFMT_Q4_0: 5e-3, synth.WFMT_Q8_0: 5e-3,
       synth.WFMT_Q5_0: 5e-3, synth.WFMT_Q6_K: 5e-3, synth.WFMT_BF16_F16DOWN: 2e-3}
GAP_REL = 1e-5
W_ABS = 1e-7


DECODE_TRIPWIRE = 1e-4


def w_rtol(d: int, prefill: bool = False) -> float:
    """Relative tolerance of the renormalised routing weights (see above)."""
    return (24.0 if prefill else 5.0) * np.sqrt(d) * 2.0 ** -24


def run_gpu(layer: D.DeviceLayer, x_bits: np.ndarray, T: int, regime=B.MOE_REGIME_AUTO,
            plan=None, out=None):
    """One moe_forward through the C ABI; returns (out fp32 [T][d], routing
    tables as numpy, launches)."""
    sh = layer.shape
    own_plan = plan is None
    if own_plan:
        plan = B.moe_plan_create(layer.config(max(T, 1), regime))
    try:
        x = D.upload_x(x_bits[:T] if T else x_bits[:1], layer.device)
        if out is None:
            out = torch.full((max(T, 1), sh.d), float("nan"), dtype=torch.float32,
                             device=layer.device)
        r = D.Routing(max(T, 1), sh.k, sh.E, layer.device)
        st = torch.cuda.current_stream(layer.device).cuda_stream
        B.moe_forward(plan, layer.weights, x.data_ptr(), T, sh.k, sh.wfmt, out.data_ptr(), r.struct, st)
        launches = B.moe_last_launch_count(plan)
        torch.cuda.synchronize(layer.device)
        status = B.moe_get_device_status(plan)
        assert status == B.MOE_OK, B.moe_status_string(status)
        return out[:T].cpu().numpy().astype(np.float64), r.numpy(), launches
    finally:
        if own_plan:
            B.moe_plan_destroy(plan)


def run_gpu_split(layer: D.DeviceLayer, x_bits: np.ndarray, T: int, regime=B.MOE_REGIME_AUTO):
    """The same layer through moe_route + moe_experts (the two-launch path)."""
    sh = layer.shape
    plan = B.moe_plan_create(layer.config(max(T, 1), regime))
    try:
        x = D.upload_x(x_bits[:T], layer.device)
        out = torch.full((T, sh.d), float("nan"), dtype=torch.float32, device=layer.device)
        r = D.Routing(T, sh.k, sh.E, layer.device)
        st = torch.cuda.current_stream(layer.device).cuda_stream
        B.moe_route(plan, layer.weights, x.data_ptr(), T, sh.k, sh.wfmt, out.data_ptr(), st)
        n1 = B.moe_last_launch_count(plan)
        B.moe_experts(plan, layer.weights, x.data_ptr(), T, sh.k, sh.wfmt, out.data_ptr(), st)
        n2 = B.moe_last_launch_count(plan)
        B.moe_routing_get(plan, T, r.struct, st)
        torch.cuda.synchronize(layer.device)
        assert B.moe_get_device_status(plan) == B.MOE_OK
        return out.cpu().numpy().astype(np.float64), r.numpy(), n1 + n2
    finally:
        B.moe_plan_destroy(plan)


def waived_tokens(logits: np.ndarray, k: int) -> np.ndarray:
    """Tokens whose k-th / (k+1)-th oracle logits nearly tie."""
    T, E = logits.shape
    if k >= E:
        return np.zeros(T, bool)
    s = -np.sort(-logits, axis=1)
    gap = s[:, k - 1] - s[:, k]
    return gap < GAP_REL * np.abs(s[:, k - 1])


def check_tie_choice(logits: np.ndarray, ids, k: int):
    """On a waived near-tie token the GPU may order the tied experts
    differently, but every expert it picked must lie in the tie band of the
    oracle's k-th largest logit, and the picks must be distinct."""
    s = -np.sort(-logits)
    kth = s[k - 1]
    band = GAP_REL * abs(kth)
    assert len(set(np.asarray(ids).tolist())) == k
    assert all(logits[e] >= kth - band for e in ids), (ids, kth)


def compare(inp: synth.MoEInputs, gpu_out, routing, oracle_res, tokens=None, tol=None,
            tripwire=None, prefill=False):
    """Check one GPU call against the oracle; returns the relative L2 error
    over every token checked."""
    sh = inp.shape
    o_out, o_ids, o_w, o_logits = oracle_res
    ids, w, counts, offsets, slot_pair = routing
    T = gpu_out.shape[0]
    tok = np.arange(T) if tokens is None else np.asarray(tokens)
    g_ids, g_w, g_out = ids[tok], w[tok], gpu_out[tok]
    waived = waived_tokens(o_logits, sh.k)
    ok_ids = np.all(g_ids == o_ids, axis=1)
    assert np.all(ok_ids | waived), (
        f"expert ids differ on non-tied tokens {np.where(~ok_ids & ~waived)[0].tolist()}")
    for t in range(len(tok)):                     # ids valid and distinct everywhere
        assert len(set(g_ids[t].tolist())) == sh.k and g_ids[t].min() >= 0 and g_ids[t].max() < sh.E
    np.testing.assert_allclose(g_w[ok_ids], o_w[ok_ids], rtol=w_rtol(sh.d, prefill), atol=W_ABS)
    # buckets are a pure function of the ids: compare with the oracle's
    if tokens is None:
        c, o, sp = oracle.buckets(ids.astype(np.int32), sh.E)
        assert np.array_equal(counts, c)
        assert np.array_equal(offsets, o)
        assert np.array_equal(slot_pair, sp)
    ref = np.array(o_out, dtype=np.float64, copy=True)
    flip = np.where(~ok_ids)[0]
    if len(flip):
        for i in flip:
            check_tie_choice(o_logits[i], g_ids[i], sh.k)
        ref[flip] = oracle.forward_routed(inp, g_ids[flip], g_w[flip].astype(np.float64),
                                          tokens=tok[flip])
    err = float(np.linalg.norm(g_out - ref) / max(np.linalg.norm(ref), 1e-300))
    lim = TOL[sh.wfmt] if tol is None else tol
    assert err <= lim, f"relative L2 error {err:.3e} > {lim:.1e}"
    if tripwire is not None:
        assert err <= tripwire, f"relative L2 error {err:.3e} above the regression tripwire {tripwire:.1e}"
    assert np.all(np.isfinite(gpu_out))
    return err
