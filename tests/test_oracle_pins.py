"""Pins for the fp64 oracle: each test checks it against something other
than itself -- brute force on tiny inputs, closed forms, library routines or
hand-built fixtures -- so that a dropped term, a wrong sign or index, or a
transposed operand anywhere in the oracle fails at least one of them.

The layer these pins describe: router logits, softmax over all experts, top-k
with renormalised weights, per-expert bucketing, SwiGLU experts over the
selected and the always-on shared experts, weighted combine ("Fused MoE
Triton kernel: 5 launches instead of 24" page, list of fused steps; "CUDA:
fuse shared experts into MMVQ" page, section on shared experts).
"""
import itertools
import json
import math
import os
import struct

import numpy as np
import pytest
import torch

import oracle
from mixture_experts_layer_43_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- decoders
def test_bf16_decode_matches_torch_all_patterns():
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).double().numpy()
    got = np.array([oracle.bf16_to_f64(int(b)) for b in bits])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    # signed zeros too
    assert math.copysign(1.0, oracle.bf16_to_f64(0x8000)) == -1.0


def test_fp16_decode_matches_numpy_all_patterns():
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([oracle.fp16_to_f64(int(b)) for b in bits])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


def test_f16down_inputs_are_the_bf16_draws_rounded_to_fp16():
    """The fp16 down matrices of the BF16_F16DOWN format are the bf16 draws
    of the bf16 layer rounded to fp16 (torch's conversion), exactly equal
    wherever 2^-17 <= |w| <= 65504 (every such bf16 value is an fp16 value)."""
    sh = synth.MoEShape("conv", T=2, d=256, E=3, k=2, F=64, S=1, Fs=32)
    a = synth.make_inputs(sh, seed=9)
    b = synth.make_inputs(sh.replace(wfmt=synth.WFMT_BF16_F16DOWN), seed=9)
    assert np.array_equal(a.gate, b.gate) and np.array_equal(a.up, b.up)
    for bf, f16 in ((a.down, b.down), (a.shared_down, b.shared_down)):
        t = torch.from_numpy(np.ascontiguousarray(bf).view(np.int16)).view(torch.bfloat16)
        want = t.to(torch.float16).view(torch.int16).numpy().view(np.uint16)
        assert np.array_equal(f16, want)
        v = t.double().numpy()
        ok = (np.abs(v) >= 2.0 ** -17) | (v == 0)
        assert np.array_equal(f16.view(np.float16).astype(np.float64)[ok], v[ok])


def test_golden_fixtures_match_their_encoder():
    """The committed fixtures are exactly what make_golden.py (plain struct
    packing of the hand-chosen codes, no oracle code) writes."""
    import subprocess
    import sys
    r = subprocess.run([sys.executable, os.path.join(GOLDEN, "make_golden.py"), "--check"],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stdout + r.stderr


def test_q4_0_golden_blocks():
    g = json.load(open(os.path.join(GOLDEN, "q4_0_blocks.json")))
    for blk in g["blocks"]:
        raw = np.array(blk["bytes"], dtype=np.uint8)
        got = oracle.dequant(oracle.WFMT_Q4_0, raw, 1, 32)[0]
        scale = float(np.array([blk["scale_bits"]], np.uint16).view(np.float16)[0])
        want = np.array([scale * (q - 8) for q in blk["codes"]], dtype=np.float64)
        assert np.array_equal(got, want), blk["name"]


def test_q4_0_rows_are_independent_blocks():
    """A multi-row, multi-block matrix dequantises block by block in row-major
    block order (checked against Python's own IEEE half decoder)."""
    rng = np.random.default_rng(5)
    rows, k = 3, 96
    blocks = synth.q4_0_blocks(rng, rows, k, 0.01)
    got = oracle.dequant(oracle.WFMT_Q4_0, blocks, rows, k)
    for r in range(rows):
        for b in range(k // 32):
            raw = bytes(blocks[r, b])
            (scale,) = struct.unpack("<e", raw[:2])
            for j in range(16):
                lo, hi = raw[2 + j] & 15, raw[2 + j] >> 4
                assert got[r, 32 * b + j] == scale * (lo - 8)
                assert got[r, 32 * b + 16 + j] == scale * (hi - 8)


def test_q8_0_golden_blocks():
    g = json.load(open(os.path.join(GOLDEN, "q8_0_blocks.json")))
    for blk in g["blocks"]:
        raw = np.array(blk["bytes"], dtype=np.uint8)
        got = oracle.dequant(oracle.WFMT_Q8_0, raw, 1, 32)[0]
        scale = float(np.array([blk["scale_bits"]], np.uint16).view(np.float16)[0])
        want = np.array([scale * q for q in blk["codes"]], dtype=np.float64)
        assert np.array_equal(got, want), blk["name"]


def test_q8_0_rows_are_independent_blocks():
    """A multi-row, multi-block Q8_0 matrix dequantises block by block in
    row-major block order (checked with Python's struct decoders)."""
    rng = np.random.default_rng(6)
    rows, k = 3, 96
    blocks = synth.q8_0_blocks(rng, rows, k, 0.01)
    got = oracle.dequant(oracle.WFMT_Q8_0, blocks, rows, k)
    for r in range(rows):
        for b in range(k // 32):
            raw = bytes(blocks[r, b])
            (scale,) = struct.unpack("<e", raw[:2])
            codes = struct.unpack("<32b", raw[2:])
            for j in range(32):
                assert got[r, 32 * b + j] == scale * codes[j]


def test_q5_0_golden_blocks():
    g = json.load(open(os.path.join(GOLDEN, "q5_0_blocks.json")))
    for blk in g["blocks"]:
        raw = np.array(blk["bytes"], dtype=np.uint8)
        got = oracle.dequant(oracle.WFMT_Q5_0, raw, 1, 32)[0]
        scale = float(np.array([blk["scale_bits"]], np.uint16).view(np.float16)[0])
        want = np.array([scale * (q - 16) for q in blk["codes"]], dtype=np.float64)
        assert np.array_equal(got, want), blk["name"]


def _q5_codes(raw):
    """The 32 codes of one canonical Q5_0 block, with Python's struct and
    integer operations: bit j of the little-endian word after the scale is
    element j's fifth bit."""
    (qh,) = struct.unpack("<I", raw[2:6])
    qs = raw[6:22]
    low = [c & 15 for c in qs] + [c >> 4 for c in qs]
    return [low[j] + 16 * ((qh >> j) & 1) for j in range(32)]


def test_q5_0_rows_are_independent_blocks():
    """A multi-row, multi-block Q5_0 matrix dequantises block by block in
    row-major block order (checked with Python's struct decoders)."""
    rng = np.random.default_rng(7)
    rows, k = 3, 96
    blocks = synth.q5_0_blocks(rng, rows, k, 0.01)
    got = oracle.dequant(oracle.WFMT_Q5_0, blocks, rows, k)
    seen = set()
    for r in range(rows):
        for b in range(k // 32):
            raw = bytes(blocks[r, b])
            (scale,) = struct.unpack("<e", raw[:2])
            for j, q in enumerate(_q5_codes(raw)):
                assert got[r, 32 * b + j] == scale * (q - 16)
                seen.add(q)
    assert min(seen) < 16 <= max(seen)     # both values of the fifth bit occur


# ------------------------------------------------- pure-Python brute force
def test_q6_k_golden_blocks():
    g = json.load(open(os.path.join(GOLDEN, "q6_k_blocks.json")))
    for blk in g["blocks"]:
        raw = np.array(blk["bytes"], dtype=np.uint8)
        got = oracle.dequant(oracle.WFMT_Q6_K, raw, 1, 256)[0]
        scale = float(np.array([blk["scale_bits"]], np.uint16).view(np.float16)[0])
        want = np.array([scale * blk["sub_scales"][i // 16] * (q - 32)
                         for i, q in enumerate(blk["codes"])], dtype=np.float64)
        assert np.array_equal(got, want), blk["name"]


def _q6_codes(raw):
    """The 256 codes and 16 sub-scales of one canonical q6_K super-block,
    decoded with Python's struct and integer operations, element by element
    from the layout statement: element i = 128 h + 32 c + l."""
    ql, qh = raw[:128], raw[128:192]
    subs = struct.unpack("<16b", raw[192:208])
    codes = []
    for i in range(256):
        h, r = divmod(i, 128)
        c, l = divmod(r, 32)
        byte = ql[64 * h + 32 * (c % 2) + l]
        low = (byte >> 4) if c >= 2 else (byte & 15)
        high = (qh[32 * h + l] >> (2 * c)) & 3
        codes.append(low + 16 * high)
    return codes, subs


def test_q6_k_rows_are_independent_blocks():
    """A multi-row, multi-super-block q6_K matrix dequantises super-block by
    super-block in row-major order (checked with Python's struct decoders)."""
    rng = np.random.default_rng(8)
    rows, k = 2, 512
    blocks = synth.q6_k_blocks(rng, rows, k, 0.01)
    got = oracle.dequant(oracle.WFMT_Q6_K, blocks, rows, k)
    for r in range(rows):
        for b in range(k // 256):
            raw = bytes(blocks[r, b])
            (scale,) = struct.unpack("<e", raw[208:210])
            codes, subs = _q6_codes(raw)
            for i in range(256):
                assert got[r, 256 * b + i] == scale * subs[i // 16] * (codes[i] - 32)


def test_q6_k_rejects_ragged_rows():
    with pytest.raises(ValueError):
        oracle.dequant(oracle.WFMT_Q6_K, np.zeros(420, np.uint8), 1, 288)


def _bf16(b):
    return struct.unpack(">f", struct.pack(">I", int(b) << 16))[0]


def _q4_rows(blocks):
    """Pure-Python decode of canonical Q4_0 rows -> list of lists."""
    out = []
    for row in blocks:
        vals = []
        for blk in row:
            raw = bytes(blk)
            (sc,) = struct.unpack("<e", raw[:2])
            lo = [sc * ((c & 15) - 8) for c in raw[2:]]
            hi = [sc * ((c >> 4) - 8) for c in raw[2:]]
            vals.extend(lo + hi)
        out.append(vals)
    return out


def _q8_rows(blocks):
    """Pure-Python decode of canonical Q8_0 rows -> list of lists."""
    out = []
    for row in blocks:
        vals = []
        for blk in row:
            raw = bytes(blk)
            (sc,) = struct.unpack("<e", raw[:2])
            vals.extend(sc * q for q in struct.unpack("<32b", raw[2:]))
        out.append(vals)
    return out


def _q5_rows(blocks):
    """Pure-Python decode of canonical Q5_0 rows -> list of lists."""
    out = []
    for row in blocks:
        vals = []
        for blk in row:
            raw = bytes(blk)
            (sc,) = struct.unpack("<e", raw[:2])
            vals.extend(sc * (q - 16) for q in _q5_codes(raw))
        out.append(vals)
    return out


def _q6_rows(blocks):
    """Pure-Python decode of canonical q6_K rows -> list of lists."""
    out = []
    for row in blocks:
        vals = []
        for blk in row:
            raw = bytes(blk)
            (sc,) = struct.unpack("<e", raw[208:210])
            codes, subs = _q6_codes(raw)
            vals.extend(sc * subs[i // 16] * (q - 32) for i, q in enumerate(codes))
        out.append(vals)
    return out


_F16_ROWS = "f16"      # down matrices of the BF16_F16DOWN format: IEEE fp16 bits


def _mat(inp_arr, wfmt, m, rows, cols):
    if wfmt == _F16_ROWS:
        a = inp_arr[m]
        return [[struct.unpack("<e", struct.pack("<H", int(a[r, c])))[0] for c in range(cols)]
                for r in range(rows)]
    if wfmt in (synth.WFMT_BF16, synth.WFMT_BF16_F16DOWN):
        a = inp_arr[m]
        return [[_bf16(a[r, c]) for c in range(cols)] for r in range(rows)]
    if wfmt == synth.WFMT_Q6_K:
        return _q6_rows(inp_arr[m])
    if wfmt == synth.WFMT_Q4_0:
        return _q4_rows(inp_arr[m])
    if wfmt == synth.WFMT_Q5_0:
        return _q5_rows(inp_arr[m])
    return _q8_rows(inp_arr[m])


def _brute_layer(inp):
    """Top-k by enumerating all k-subsets (the subset with the largest summed
    logit), softmax over all experts, renormalise, dense SwiGLU by scalar
    loops.  Independent of the C oracle in every step."""
    sh = inp.shape
    T, d = inp.x.shape
    xs = [[_bf16(inp.x[t, i]) for i in range(d)] for t in range(T)]
    wr = inp.router_w.astype(np.float64)
    br = None if inp.router_b is None else inp.router_b.astype(np.float64)

    def ffn(gate, up, down, F, xt):
        h = []
        for f in range(F):
            g = sum(gate[f][i] * xt[i] for i in range(d))
            u = sum(up[f][i] * xt[i] for i in range(d))
            h.append(g / (1.0 + math.exp(-g)) * u)
        return [sum(down[j][f] * h[f] for f in range(F)) for j in range(d)]

    dfmt = _F16_ROWS if sh.wfmt == synth.WFMT_BF16_F16DOWN else sh.wfmt
    experts = [(_mat(inp.gate, sh.wfmt, e, sh.F, d), _mat(inp.up, sh.wfmt, e, sh.F, d),
                _mat(inp.down, dfmt, e, d, sh.F)) for e in range(sh.E)]
    shared = []
    if inp.shared_gate is not None:
        shared = [(_mat(inp.shared_gate, sh.wfmt, s, sh.Fs, d),
                   _mat(inp.shared_up, sh.wfmt, s, sh.Fs, d),
                   _mat(inp.shared_down, dfmt, s, d, sh.Fs)) for s in range(sh.S)]
    outs, sets, weights = [], [], []
    for t in range(T):
        xt = xs[t]
        lg = [sum(xt[i] * float(wr[e, i]) for i in range(d)) + (0.0 if br is None else float(br[e]))
              for e in range(sh.E)]
        best = max(itertools.combinations(range(sh.E), sh.k),
                   key=lambda c: sum(lg[e] for e in c))
        m = max(lg)
        z = sum(math.exp(v - m) for v in lg)
        p = [math.exp(v - m) / z for v in lg]
        ps = sum(p[e] for e in best)
        w = {e: p[e] / ps for e in best}
        o = [0.0] * d
        for e in best:
            y = ffn(*experts[e], sh.F, xt)
            o = [o[j] + w[e] * y[j] for j in range(d)]
        for s in range(len(shared)):
            y = ffn(*shared[s], sh.Fs, xt)
            o = [o[j] + y[j] for j in range(d)]
        outs.append(o)
        sets.append(best)
        weights.append(w)
    return np.array(outs), sets, weights, lg


TINY = [
    synth.MoEShape("bf16_noshared", T=3, d=16, E=6, k=2, F=8),
    synth.MoEShape("bf16_shared", T=2, d=12, E=5, k=3, F=6, S=2, Fs=4),
    synth.MoEShape("bf16_bias", T=3, d=8, E=7, k=2, F=5, S=1, Fs=3, zipf_bias=1.1),
    synth.MoEShape("q4_shared", T=2, d=32, E=4, k=2, F=32, S=1, Fs=32,
                   wfmt=synth.WFMT_Q4_0),
    synth.MoEShape("q8_shared", T=2, d=32, E=4, k=2, F=32, S=1, Fs=32,
                   wfmt=synth.WFMT_Q8_0),
    synth.MoEShape("q5_shared", T=2, d=32, E=4, k=2, F=32, S=1, Fs=32,
                   wfmt=synth.WFMT_Q5_0),
    synth.MoEShape("q6_shared", T=2, d=256, E=3, k=2, F=256, S=1, Fs=256,
                   wfmt=synth.WFMT_Q6_K),
    synth.MoEShape("f16down_shared", T=2, d=12, E=5, k=2, F=6, S=1, Fs=4,
                   wfmt=synth.WFMT_BF16_F16DOWN),
]


@pytest.mark.parametrize("sh", TINY, ids=[s.name for s in TINY])
def test_brute_force_tiny(sh):
    # A larger weight std makes the logits spread and the SwiGLU nonlinear.
    sh = sh.replace(w_std=0.5, wr_std=0.5, q4_scale_std=0.05, q8_scale_std=0.004,
                    q5_scale_std=0.025, q6_scale_std=2e-4)
    inp = synth.make_inputs(sh, seed=11)
    out, ids, w, logits = oracle.forward(inp)
    bout, bsets, bw, _ = _brute_layer(inp)
    scale = np.abs(bout).max()
    assert scale > 0
    np.testing.assert_allclose(out, bout, rtol=1e-12, atol=1e-12 * scale)
    for t in range(sh.T):
        assert sorted(ids[t].tolist()) == sorted(bsets[t])
        # returned in descending-logit order
        lg = logits[t][ids[t]]
        assert np.all(np.diff(lg) <= 0)
        for j, e in enumerate(ids[t]):
            assert abs(w[t, j] - bw[t][e]) < 1e-14
        assert abs(w[t].sum() - 1.0) < 1e-15 and np.all(w[t] > 0)


def _f64_stack(arr, wfmt, rows, cols):
    """Dequantise a stack with torch/numpy (library decoders, not the oracle)."""
    if wfmt == _F16_ROWS:
        return np.ascontiguousarray(arr).view(np.float16).astype(np.float64).reshape(-1, rows, cols)
    if wfmt in (synth.WFMT_BF16, synth.WFMT_BF16_F16DOWN):
        t = torch.from_numpy(np.ascontiguousarray(arr).view(np.int16)).view(torch.bfloat16)
        return t.double().numpy().reshape(-1, rows, cols)
    if wfmt == synth.WFMT_Q8_0:
        a = np.ascontiguousarray(arr).reshape(-1, rows, cols // 32, 34)
        sc = a[..., :2].copy().view(np.float16)[..., 0].astype(np.float64)
        q = a[..., 2:].copy().view(np.int8).astype(np.float64)
        return (q * sc[..., None]).reshape(-1, rows, cols)
    if wfmt == synth.WFMT_Q6_K:
        a = np.ascontiguousarray(arr).reshape(-1, rows, cols // 256, 210)
        d = a[..., 208:210].copy().view(np.float16)[..., 0].astype(np.float64)
        sub = a[..., 192:208].copy().view(np.int8).astype(np.float64)          # [..][16]
        ql = a[..., :128].reshape(a.shape[:-1] + (2, 2, 32))                  # [h][c%2][l]
        qh = a[..., 128:192].reshape(a.shape[:-1] + (2, 32))                  # [h][l]
        low = np.stack([ql[..., 0, :] & 15, ql[..., 1, :] & 15,
                        ql[..., 0, :] >> 4, ql[..., 1, :] >> 4], axis=-2)      # [h][c][l]
        high = np.stack([(qh >> (2 * c)) & 3 for c in range(4)], axis=-2)      # [h][c][l]
        q = (low.astype(np.float64) + 16.0 * high).reshape(a.shape[:-1] + (256,)) - 32.0
        w = q * np.repeat(sub, 16, axis=-1) * d[..., None]
        return w.reshape(-1, rows, cols)
    if wfmt == synth.WFMT_Q5_0:
        a = np.ascontiguousarray(arr).reshape(-1, rows, cols // 32, 22)
        sc = a[..., :2].copy().view(np.float16)[..., 0].astype(np.float64)
        qh = a[..., 2:6].copy().view("<u4")[..., 0]
        fifth = (qh[..., None] >> np.arange(32, dtype=np.uint32)) & 1
        low = np.concatenate([a[..., 6:] & 15, a[..., 6:] >> 4], axis=-1)
        q = low.astype(np.float64) + 16.0 * fifth - 16.0
        return (q * sc[..., None]).reshape(-1, rows, cols)
    a = np.ascontiguousarray(arr).reshape(-1, rows, cols // 32, 18)
    sc = a[..., :2].copy().view(np.float16)[..., 0].astype(np.float64)
    lo = (a[..., 2:] & 15).astype(np.float64) - 8
    hi = (a[..., 2:] >> 4).astype(np.float64) - 8
    q = np.concatenate([lo, hi], axis=-1)
    return (q * sc[..., None]).reshape(-1, rows, cols)


def _np_ffn(g, u, dn, x):
    """SwiGLU FFN with numpy float64 matmuls: x [T][d] -> [T][d]."""
    a = x @ g.T
    b = x @ u.T
    h = a / (1.0 + np.exp(-a)) * b
    return h @ dn.T


def _x64(inp):
    return torch.from_numpy(inp.x.view(np.int16)).view(torch.bfloat16).double().numpy()


@pytest.mark.parametrize("wfmt", [synth.WFMT_BF16, synth.WFMT_Q4_0, synth.WFMT_Q8_0,
                                  synth.WFMT_Q5_0, synth.WFMT_Q6_K, synth.WFMT_BF16_F16DOWN])
def test_k_equals_E_is_dense_softmax_mixture(wfmt):
    big = wfmt == synth.WFMT_Q6_K          # 256-weight super-blocks
    sh = synth.MoEShape("dense", T=5, d=256 if big else 64, E=4, k=4, F=256 if big else 32,
                        wfmt=wfmt, wr_std=0.2 if not big else 0.1, w_std=0.2,
                        q4_scale_std=0.02, q8_scale_std=0.002, q5_scale_std=0.01,
                        q6_scale_std=1e-4)
    inp = synth.make_inputs(sh, seed=3)
    out, ids, w, logits = oracle.forward(inp)
    x = _x64(inp)
    G = _f64_stack(inp.gate, wfmt, sh.F, sh.d)
    U = _f64_stack(inp.up, wfmt, sh.F, sh.d)
    D = _f64_stack(inp.down, _F16_ROWS if wfmt == synth.WFMT_BF16_F16DOWN else wfmt, sh.d, sh.F)
    lg = x @ inp.router_w.astype(np.float64).T
    p = np.exp(lg - lg.max(1, keepdims=True))
    p /= p.sum(1, keepdims=True)
    want = sum(p[:, e:e + 1] * _np_ffn(G[e], U[e], D[e], x) for e in range(sh.E))
    np.testing.assert_allclose(out, want, rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(logits, lg, rtol=1e-13, atol=1e-13)


def test_one_hot_router_reduces_to_single_ffn():
    sh = synth.MoEShape("onehot", T=4, d=64, E=6, k=1, F=24, w_std=0.2)
    inp = synth.make_inputs(sh, seed=4)
    x = _x64(inp)
    wr = np.zeros((sh.E, sh.d), np.float32)
    star = 4
    # logit of expert 4 = 0.5 * |x|^2 (>= 50 for these x), all others 0
    wr[star] = (0.5 * x[0]).astype(np.float32)
    inp.x[:] = inp.x[0]
    inp.router_w = wr
    x = _x64(inp)
    out, ids, w, logits = oracle.forward(inp)
    assert np.all(ids[:, 0] == star) and np.all(w == 1.0)
    assert logits[0, star] - np.delete(logits[0], star).max() >= 20
    G = _f64_stack(inp.gate, 0, sh.F, sh.d)[star]
    U = _f64_stack(inp.up, 0, sh.F, sh.d)[star]
    D = _f64_stack(inp.down, 0, sh.d, sh.F)[star]
    np.testing.assert_allclose(out, _np_ffn(G, U, D, x), rtol=1e-12, atol=1e-14)
    # k = 2: the second weight is p2/(p1+p2) = 1/(1+e^gap), a closed form
    inp2 = synth.MoEInputs(sh.replace(k=2), inp.x, wr, None, inp.gate, inp.up,
                           inp.down, None, None, None)
    _, ids2, w2, lg2 = oracle.forward(inp2)
    gap = lg2[0, ids2[0, 0]] - lg2[0, ids2[0, 1]]
    assert ids2[0, 0] == star
    assert abs(w2[0, 1] - 1.0 / (1.0 + math.exp(gap))) < 1e-15


def test_single_expert_is_plain_swiglu():
    sh = synth.MoEShape("e1", T=6, d=48, E=1, k=1, F=40, w_std=0.3)
    inp = synth.make_inputs(sh, seed=5)
    out, ids, w, _ = oracle.forward(inp)
    x = _x64(inp)
    G, U, D = (_f64_stack(inp.gate, 0, 40, 48)[0], _f64_stack(inp.up, 0, 40, 48)[0],
               _f64_stack(inp.down, 0, 48, 40)[0])
    assert np.all(ids == 0) and np.all(w == 1.0)
    np.testing.assert_allclose(out, _np_ffn(G, U, D, x), rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("wfmt", [synth.WFMT_BF16, synth.WFMT_Q4_0])
def test_forward_routed_is_weighted_sum_of_ffns(wfmt):
    """Steps 6-7 with routing given from outside: arbitrary ids (repeats and
    any order allowed by the definition) and weights, plus the shared
    experts, against numpy float64 matmuls."""
    sh = synth.MoEShape("routed", T=4, d=64, E=5, k=3, F=32, S=1, Fs=32, wfmt=wfmt,
                        w_std=0.2, q4_scale_std=0.02)
    inp = synth.make_inputs(sh, seed=8)
    ids = np.array([[4, 0, 2], [1, 1, 3], [2, 4, 0], [3, 0, 1]], dtype=np.int32)
    w = np.array([[0.5, 0.25, 0.25], [0.125, 0.375, 0.5], [1.0, 0.0, 0.0],
                  [0.3, 0.3, 0.4]])
    x = _x64(inp)
    G = _f64_stack(inp.gate, wfmt, sh.F, sh.d)
    U = _f64_stack(inp.up, wfmt, sh.F, sh.d)
    D = _f64_stack(inp.down, wfmt, sh.d, sh.F)
    want = _np_ffn(_f64_stack(inp.shared_gate, wfmt, sh.Fs, sh.d)[0],
                   _f64_stack(inp.shared_up, wfmt, sh.Fs, sh.d)[0],
                   _f64_stack(inp.shared_down, wfmt, sh.d, sh.Fs)[0], x)
    for t in range(sh.T):
        for j in range(sh.k):
            e = ids[t, j]
            want[t] += w[t, j] * _np_ffn(G[e], U[e], D[e], x[t:t + 1])[0]
    got = oracle.forward_routed(inp, ids, w)
    np.testing.assert_allclose(got, want, rtol=1e-11, atol=1e-13)
    # a subset of tokens, in any order
    sub = oracle.forward_routed(inp, ids[[3, 1]], w[[3, 1]], tokens=[3, 1])
    np.testing.assert_allclose(sub, want[[3, 1]], rtol=1e-11, atol=1e-13)


def test_shared_only_when_routed_down_is_zero():
    sh = synth.MoEShape("sh", T=3, d=32, E=5, k=2, F=16, S=2, Fs=8, w_std=0.3)
    inp = synth.make_inputs(sh, seed=6)
    inp.down = np.zeros_like(inp.down)
    out, _, _, _ = oracle.forward(inp)
    x = _x64(inp)
    want = np.zeros_like(out)
    for s in range(2):
        want += _np_ffn(_f64_stack(inp.shared_gate, 0, 8, 32)[s],
                        _f64_stack(inp.shared_up, 0, 8, 32)[s],
                        _f64_stack(inp.shared_down, 0, 32, 8)[s], x)
    np.testing.assert_allclose(out, want, rtol=1e-12, atol=1e-14)


def test_two_shared_equal_one_concatenated():
    """Two shared experts of hidden size Fs equal one of hidden size 2*Fs whose
    gate/up rows and down columns are the concatenation."""
    sh = synth.MoEShape("cat", T=3, d=16, E=3, k=1, F=8, S=2, Fs=4, w_std=0.3)
    inp = synth.make_inputs(sh, seed=7)
    out, _, _, _ = oracle.forward(inp)
    cat = synth.MoEInputs(sh.replace(S=1, Fs=8), inp.x, inp.router_w, None, inp.gate,
                          inp.up, inp.down, inp.shared_gate.reshape(1, 8, 16).copy(),
                          inp.shared_up.reshape(1, 8, 16).copy(),
                          np.concatenate([inp.shared_down[0], inp.shared_down[1]],
                                         axis=1)[None].copy())
    out2, _, _, _ = oracle.forward(cat)
    np.testing.assert_allclose(out, out2, rtol=1e-13, atol=1e-15)


def test_expert_permutation_invariance():
    sh = synth.MoEShape("perm", T=5, d=32, E=6, k=2, F=12, S=1, Fs=8, w_std=0.3,
                        wr_std=0.3, zipf_bias=1.1)
    inp = synth.make_inputs(sh, seed=8)
    out, ids, w, _ = oracle.forward(inp)
    perm = np.array([3, 0, 5, 1, 4, 2])          # new expert i = old expert perm[i]
    inv = np.argsort(perm)
    pinp = synth.MoEInputs(sh, inp.x, inp.router_w[perm].copy(), inp.router_b[perm].copy(),
                           inp.gate[perm].copy(), inp.up[perm].copy(), inp.down[perm].copy(),
                           inp.shared_gate, inp.shared_up, inp.shared_down)
    pout, pids, pw, _ = oracle.forward(pinp)
    np.testing.assert_allclose(pout, out, rtol=1e-13, atol=1e-15)
    assert np.array_equal(perm[pids], ids)
    np.testing.assert_allclose(pw, w, rtol=1e-15)
    assert np.array_equal(inv[ids], pids)


def test_tie_break_lower_index():
    """Equal logits: the lower expert index is taken first."""
    sh = synth.MoEShape("tie", T=1, d=8, E=5, k=2, F=4)
    inp = synth.make_inputs(sh, seed=9)
    wr = np.zeros((5, 8), np.float32)      # all logits 0
    _, ids, w = oracle.route(inp.x, wr, None, 2)
    assert ids.tolist() == [[0, 1]] and np.allclose(w, 0.5)
    b = np.array([0, 1, 0, 1, 1], np.float32)
    _, ids, _ = oracle.route(inp.x, wr, b, 3)
    assert ids.tolist() == [[1, 3, 4]]


def test_softmax_renormalisation_closed_form():
    """Two experts with logits (1, 0) and k = 2: weights e/(1+e), 1/(1+e);
    k = 1 of three experts with logits (0, 1, 1): expert 1, weight 1."""
    x = synth.f32_to_bf16_bits(np.array([[1.0, 0.0]], np.float32))
    wr = np.array([[1.0, 0.0], [0.0, 0.0]], np.float32)
    _, ids, w = oracle.route(x, wr, None, 2)
    assert ids.tolist() == [[0, 1]]
    assert abs(w[0, 0] - math.e / (1 + math.e)) < 1e-16
    assert abs(w[0, 1] - 1 / (1 + math.e)) < 1e-16
    wr3 = np.array([[0.0, 0.0], [1.0, 0.0], [1.0, 0.0]], np.float32)
    _, ids, w = oracle.route(x, wr3, None, 1)
    assert ids.tolist() == [[1]] and w[0, 0] == 1.0


def test_swiglu_closed_form():
    """d = 2, F = 1, one expert: gate pre-activation 2, up 3, down (0.5, -1):
    out = (0.5, -1) * 3 * 2/(1+e^-2)."""
    sh = synth.MoEShape("cf", T=1, d=2, E=1, k=1, F=1)
    bf = synth.f32_to_bf16_bits
    x = bf(np.array([[1.0, 2.0]], np.float32))
    g = bf(np.array([[[2.0, 0.0]]], np.float32))
    u = bf(np.array([[[1.0, 1.0]]], np.float32))
    dn = bf(np.array([[[0.5], [-1.0]]], np.float32))
    inp = synth.MoEInputs(sh, x, np.zeros((1, 2), np.float32), None, g, u, dn,
                          None, None, None)
    out, _, _, _ = oracle.forward(inp)
    h = 3.0 * 2.0 / (1.0 + math.exp(-2.0))
    assert out[0, 0] == 0.5 * h and out[0, 1] == -h


def _brute_buckets(ids, E):
    T, k = ids.shape
    pairs = [(int(ids[t, j]), t, t * k + j) for t in range(T) for j in range(k)]
    order = sorted(pairs)                   # by expert, then token
    counts = [sum(1 for p in pairs if p[0] == e) for e in range(E)]
    offs = [0]
    for c in counts:
        offs.append(offs[-1] + c)
    return counts, offs, [p[2] for p in order]


@pytest.mark.parametrize("T,k,E,seed", [(1, 8, 256, 0), (8, 2, 8, 1), (37, 6, 64, 2),
                                        (0, 2, 8, 3), (64, 8, 256, 4)])
def test_buckets_match_sort(T, k, E, seed):
    rng = np.random.default_rng(seed)
    ids = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]) \
        if T else np.zeros((0, k), np.int32)
    ids = ids.astype(np.int32).reshape(T, k)
    counts, offs, slot_pair = oracle.buckets(ids, E)
    bc, bo, bs = _brute_buckets(ids, E)
    assert counts.tolist() == bc and offs.tolist() == bo and slot_pair.tolist() == bs
    assert offs[-1] == T * k and counts.sum() == T * k
    assert sorted(slot_pair.tolist()) == list(range(T * k))


def test_zipf_bias_values():
    b = synth.zipf_log_bias(64, 1.1)
    p = np.exp(b.astype(np.float64))
    assert abs(p.sum() - 1) < 1e-6 and np.all(np.diff(b) < 0)
    assert abs((b[0] - b[1]) - 1.1 * math.log(2)) < 1e-6
