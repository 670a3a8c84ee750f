"""fp64 CPU oracle for the MoE SwiGLU layer forward pass (ctypes wrapper).

TEST INFRASTRUCTURE ONLY: the test suite, the smoke check and the
benchmark's CPU-baseline leg are the only callers.  The CUDA product path
never imports this package, and this package never imports the product.

The arithmetic lives in moe_oracle.c (plain C, OpenMP over rows); this file
only compiles it, loads it and marshals numpy arrays.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

WFMT_BF16 = 0
WFMT_Q4_0 = 1
WFMT_Q8_0 = 2
WFMT_Q5_0 = 3
WFMT_Q6_K = 4
WFMT_BF16_F16DOWN = 5


def build(force: bool = False) -> str:
    """Compile moe_oracle.c into liboracle.so next to it (gcc, OpenMP)."""
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    tmp = _LIB + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c99",
           "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", tmp, "-lm"]
    subprocess.check_call(cmd)
    os.replace(tmp, _LIB)
    return _LIB


def _bind(path: str):
    L = ctypes.CDLL(path)
    P = ctypes.c_void_p
    I = ctypes.c_int
    L.oracle_bf16_to_f64.argtypes = [ctypes.c_uint16]
    L.oracle_bf16_to_f64.restype = ctypes.c_double
    L.oracle_fp16_to_f64.argtypes = [ctypes.c_uint16]
    L.oracle_fp16_to_f64.restype = ctypes.c_double
    L.oracle_dequant_rows.argtypes = [I, P, ctypes.c_int64, ctypes.c_int64, P]
    L.oracle_dequant_rows.restype = None
    L.oracle_route.argtypes = [I, I, I, I, P, P, P, P, P, P]
    L.oracle_route.restype = I
    L.oracle_buckets.argtypes = [I, I, I, P, P, P, P]
    L.oracle_buckets.restype = I
    L.oracle_forward.argtypes = [I] * 7 + [P, I] + [P] * 8 + [P, I] + [P] * 4 + [I]
    L.oracle_forward.restype = I
    L.oracle_forward_routed.argtypes = [I] * 7 + [P, I] + [P] * 6 + [P, I, P, P, P, I]
    L.oracle_forward_routed.restype = I
    L.oracle_max_threads.argtypes = []
    L.oracle_max_threads.restype = I
    return L


def lib():
    """The oracle library built from moe_oracle.c."""
    global _lib
    if _lib is None:
        build()
        _lib = _bind(_LIB)
    return _lib


def build_variant(src_text: str, out_path: str) -> str:
    """Compile a modified copy of the oracle source (used by the tests that
    check the pins catch planted mistakes).  Returns the library path."""
    c_path = out_path[:-3] + ".c"
    with open(c_path, "w") as f:
        f.write(src_text)
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared",
                           "-std=c99", "-ffp-contract=off", c_path, "-o",
                           out_path, "-lm"])
    return out_path


def source() -> str:
    with open(_SRC) as f:
        return f.read()


_active = None     # a library bound with _bind, overriding lib() when set


def use(path: Optional[str]):
    """Route the module-level functions to another build of the oracle
    (None restores the default)."""
    global _active
    _active = None if path is None else _bind(path)


def _L():
    return _active if _active is not None else lib()


def _p(a: Optional[np.ndarray]):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data


def bf16_to_f64(bits: int) -> float:
    return _L().oracle_bf16_to_f64(int(bits))


def fp16_to_f64(bits: int) -> float:
    return _L().oracle_fp16_to_f64(int(bits))


def dequant(wfmt: int, w: np.ndarray, rows: int, k: int) -> np.ndarray:
    """Rows x k matrix of a bf16 (uint16 bits), canonical-Q4_0, canonical-Q8_0,
    canonical-Q5_0 or canonical-q6_K array, fp64."""
    # (bytes per block, weights per block)
    blocks = {WFMT_BF16: None, WFMT_Q4_0: (18, 32), WFMT_Q8_0: (34, 32), WFMT_Q5_0: (22, 32),
              WFMT_Q6_K: (210, 256)}
    if wfmt not in blocks:
        raise ValueError(f"unknown weight format {wfmt}")
    nb = blocks[wfmt]
    need = rows * k * 2 if nb is None else rows * (k // nb[1]) * nb[0]
    if (nb is not None and k % nb[1]) or np.asarray(w).nbytes < need:
        raise ValueError("array too small for the requested rows x k")
    out = np.empty((rows, k), dtype=np.float64)
    _L().oracle_dequant_rows(wfmt, _p(np.ascontiguousarray(w)), rows, k, _p(out))
    return out


def route(x: np.ndarray, router_w: np.ndarray, router_b: Optional[np.ndarray],
          k: int):
    """Logits (fp64 [T][E]), top-k ids (int32 [T][k]) and renormalised
    weights (fp64 [T][k]) for every token of x."""
    T, d = x.shape
    E = router_w.shape[0]
    logits = np.empty((T, E), dtype=np.float64)
    ids = np.empty((T, k), dtype=np.int32)
    w = np.empty((T, k), dtype=np.float64)
    rb = None if router_b is None else np.ascontiguousarray(router_b, np.float32)
    rc = _L().oracle_route(T, d, E, k, _p(np.ascontiguousarray(x)),
                            _p(np.ascontiguousarray(router_w, np.float32)),
                            _p(rb), _p(logits), _p(ids), _p(w))
    if rc:
        raise ValueError(f"oracle_route failed ({rc})")
    return logits, ids, w


def buckets(ids: np.ndarray, E: int):
    """Per-expert counts, exclusive offsets (E+1) and the stable slot order
    (slot -> pair index t*k+j)."""
    T, k = ids.shape
    counts = np.empty(E, dtype=np.int32)
    offsets = np.empty(E + 1, dtype=np.int32)
    slot_pair = np.empty(T * k, dtype=np.int32)
    rc = _L().oracle_buckets(T, k, E, _p(np.ascontiguousarray(ids, np.int32)),
                              _p(counts), _p(offsets), _p(slot_pair))
    if rc:
        raise ValueError(f"oracle_buckets failed ({rc})")
    return counts, offsets, slot_pair


def forward(inp, tokens: Optional[Sequence[int]] = None, n_threads: int = 0):
    """Layer output (fp64 [n][d]) for the listed tokens (default: all),
    with ids (int32 [n][k]), weights (fp64 [n][k]) and logits (fp64 [n][E]).

    `inp` is a synth.MoEInputs (or anything with the same attributes)."""
    sh = inp.shape
    T = inp.x.shape[0]
    tok = None
    n = T
    if tokens is not None:
        tok = np.ascontiguousarray(np.asarray(tokens, dtype=np.int32))
        n = tok.shape[0]
    out = np.empty((n, sh.d), dtype=np.float64)
    ids = np.empty((n, sh.k), dtype=np.int32)
    w = np.empty((n, sh.k), dtype=np.float64)
    logits = np.empty((n, sh.E), dtype=np.float64)
    rb = None if inp.router_b is None else np.ascontiguousarray(inp.router_b, np.float32)
    S = sh.S if inp.shared_gate is not None else 0
    rc = _L().oracle_forward(
        sh.d, sh.E, sh.k, sh.F, S, sh.Fs if S else 0, sh.wfmt,
        _p(np.ascontiguousarray(inp.x)), T,
        _p(np.ascontiguousarray(inp.router_w, np.float32)), _p(rb),
        _p(inp.gate), _p(inp.up), _p(inp.down),
        _p(inp.shared_gate), _p(inp.shared_up), _p(inp.shared_down),
        _p(tok), n, _p(out), _p(ids), _p(w), _p(logits), int(n_threads))
    if rc:
        raise ValueError(f"oracle_forward failed ({rc})")
    return out, ids, w, logits


def forward_routed(inp, ids: np.ndarray, w: np.ndarray,
                   tokens: Optional[Sequence[int]] = None, n_threads: int = 0) -> np.ndarray:
    """Layer output (fp64 [n][d]) for the listed tokens (default: all) with
    the routing given by ids (int [n][k]) and weights ([n][k]) instead of the
    oracle's own router: steps 6-7 only."""
    sh = inp.shape
    T = inp.x.shape[0]
    tok = None
    n = T
    if tokens is not None:
        tok = np.ascontiguousarray(np.asarray(tokens, dtype=np.int32))
        n = tok.shape[0]
    ids = np.ascontiguousarray(np.asarray(ids, dtype=np.int32).reshape(n, sh.k))
    w = np.ascontiguousarray(np.asarray(w, dtype=np.float64).reshape(n, sh.k))
    out = np.empty((n, sh.d), dtype=np.float64)
    S = sh.S if inp.shared_gate is not None else 0
    rc = _L().oracle_forward_routed(
        sh.d, sh.E, sh.k, sh.F, S, sh.Fs if S else 0, sh.wfmt,
        _p(np.ascontiguousarray(inp.x)), T,
        _p(inp.gate), _p(inp.up), _p(inp.down),
        _p(inp.shared_gate), _p(inp.shared_up), _p(inp.shared_down),
        _p(tok), n, _p(ids), _p(w), _p(out), int(n_threads))
    if rc:
        raise ValueError(f"oracle_forward_routed failed ({rc})")
    return out


def max_threads() -> int:
    return _L().oracle_max_threads()
