"""Thin ctypes binding of libmoe_b200.so (include/moe.h).

Argument marshalling only: every step of the layer runs in the library's
CUDA kernels.  The functions keep the C names; device pointers are passed as
Python ints (e.g. torch.Tensor.data_ptr()), streams as ints (cudaStream_t).
A missing or unloadable library raises: there is no CPU fallback.
"""
from __future__ import annotations

import ctypes
import os
import re
from typing import Optional

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmoe_b200.so")
HEADER = os.path.join(os.path.dirname(_PKG), "include", "moe.h")

MOE_OK = 0
MOE_ERR_INVALID_ARG = 1
MOE_ERR_UNSUPPORTED = 2
MOE_ERR_CUDA = 3
MOE_ERR_OOM = 4
MOE_ERR_DEVICE_FLAG = 5
MOE_ERR_TIMEOUT = 6

MOE_WFMT_BF16 = 0
MOE_WFMT_Q4_0 = 1
MOE_WFMT_Q8_0 = 2
MOE_WFMT_Q5_0 = 3
MOE_WFMT_Q6_K = 4
MOE_WFMT_BF16_F16DOWN = 5
MOE_REGIME_AUTO = 0
MOE_REGIME_DECODE = 1
MOE_REGIME_PREFILL = 2
MOE_DECODE_MAX_T = 8


class MoeError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {moe_status_string(status)} ({status})")


class moe_config_t(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "t_max", "d_model", "d_ff", "n_experts", "top_k", "n_shared", "d_ff_shared",
        "wfmt", "regime", "device")]


class moe_matrix_t(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("scales", ctypes.c_void_p)]


class moe_weights_t(ctypes.Structure):
    _fields_ = [("router_w", ctypes.c_void_p), ("router_b", ctypes.c_void_p),
                ("gate", moe_matrix_t), ("up", moe_matrix_t), ("down", moe_matrix_t),
                ("shared_gate", moe_matrix_t), ("shared_up", moe_matrix_t),
                ("shared_down", moe_matrix_t)]


class moe_routing_t(ctypes.Structure):
    _fields_ = [("ids", ctypes.c_void_p), ("weights", ctypes.c_void_p),
                ("counts", ctypes.c_void_p), ("offsets", ctypes.c_void_p),
                ("slot_pair", ctypes.c_void_p)]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libmoe_b200.so (raises if it is missing)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"{LIB_PATH} is missing; build it with "
            "`python -m mixture_experts_layer_43_b200.build` (nvcc, sm_100a)")
    L = ctypes.CDLL(LIB_PATH)
    P, I32, I64, S = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_int
    L.moe_status_string.argtypes = [S]
    L.moe_status_string.restype = ctypes.c_char_p
    L.moe_plan_create.argtypes = [ctypes.POINTER(moe_config_t), ctypes.POINTER(P)]
    L.moe_plan_create.restype = S
    L.moe_plan_destroy.argtypes = [P]
    L.moe_plan_destroy.restype = None
    L.moe_forward.argtypes = [P, ctypes.POINTER(moe_weights_t), P, I32, I32, I32, P,
                              ctypes.POINTER(moe_routing_t), P]
    L.moe_forward.restype = S
    for name in ("moe_route", "moe_experts"):
        getattr(L, name).argtypes = [P, ctypes.POINTER(moe_weights_t), P, I32, I32, I32, P, P]
        getattr(L, name).restype = S
    L.moe_route_noalloc.argtypes = [ctypes.POINTER(moe_config_t), ctypes.POINTER(moe_weights_t),
                                    P, I32, P, ctypes.POINTER(moe_routing_t), P]
    L.moe_route_noalloc.restype = S
    L.moe_route_noalloc_status.argtypes = []
    L.moe_route_noalloc_status.restype = S
    L.moe_routing_get.argtypes = [P, I32, ctypes.POINTER(moe_routing_t), P]
    L.moe_routing_get.restype = S
    L.moe_last_launch_count.argtypes = [P]
    L.moe_last_launch_count.restype = I32
    L.moe_get_device_status.argtypes = [P]
    L.moe_get_device_status.restype = S
    L.moe_debug_stall_barrier.argtypes = [P, P]
    L.moe_debug_stall_barrier.restype = S
    L.moe_q4_0_packed_bytes.argtypes = [I64, I64, I64, ctypes.POINTER(ctypes.c_size_t),
                                        ctypes.POINTER(ctypes.c_size_t)]
    L.moe_q4_0_packed_bytes.restype = S
    L.moe_q4_0_pack.argtypes = [P, I64, I64, I64, P, P, P]
    L.moe_q4_0_pack.restype = S
    L.moe_q8_0_packed_bytes.argtypes = [I64, I64, I64, ctypes.POINTER(ctypes.c_size_t),
                                        ctypes.POINTER(ctypes.c_size_t)]
    L.moe_q8_0_packed_bytes.restype = S
    L.moe_q8_0_pack.argtypes = [P, I64, I64, I64, P, P, P]
    L.moe_q8_0_pack.restype = S
    L.moe_q5_0_packed_bytes.argtypes = [I64, I64, I64, ctypes.POINTER(ctypes.c_size_t),
                                        ctypes.POINTER(ctypes.c_size_t)]
    L.moe_q5_0_packed_bytes.restype = S
    L.moe_q5_0_pack.argtypes = [P, I64, I64, I64, P, P, P]
    L.moe_q5_0_pack.restype = S
    L.moe_q6_k_packed_bytes.argtypes = [I64, I64, I64, ctypes.POINTER(ctypes.c_size_t),
                                        ctypes.POINTER(ctypes.c_size_t)]
    L.moe_q6_k_packed_bytes.restype = S
    L.moe_q6_k_pack.argtypes = [P, I64, I64, I64, P, P, P]
    L.moe_q6_k_pack.restype = S
    L.moe_bf16_to_f16.argtypes = [P, I64, P, P]
    L.moe_bf16_to_f16.restype = S
    _lib = L
    return L


def header_functions() -> list:
    """Names of the functions include/moe.h declares."""
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[\w]+\s*\*?\s*(moe_\w+)\s*\(", src, flags=re.M)))


def _check(status: int, what: str):
    if status != MOE_OK:
        raise MoeError(status, what)


def moe_status_string(status: int) -> str:
    return lib().moe_status_string(int(status)).decode()


def moe_plan_create(cfg: moe_config_t) -> int:
    plan = ctypes.c_void_p()
    _check(lib().moe_plan_create(ctypes.byref(cfg), ctypes.byref(plan)), "moe_plan_create")
    return plan.value


def moe_plan_destroy(plan: int) -> None:
    lib().moe_plan_destroy(plan)


def moe_forward(plan: int, w: moe_weights_t, x: int, T: int, top_k: int, wfmt: int, out: int,
                routing: Optional[moe_routing_t] = None, stream: int = 0) -> None:
    _check(lib().moe_forward(plan, ctypes.byref(w), x, T, top_k, wfmt, out,
                             ctypes.byref(routing) if routing is not None else None, stream),
           "moe_forward")


def moe_route(plan: int, w: moe_weights_t, x: int, T: int, top_k: int, wfmt: int, out: int,
              stream: int = 0) -> None:
    _check(lib().moe_route(plan, ctypes.byref(w), x, T, top_k, wfmt, out, stream), "moe_route")


def moe_experts(plan: int, w: moe_weights_t, x: int, T: int, top_k: int, wfmt: int, out: int,
                stream: int = 0) -> None:
    _check(lib().moe_experts(plan, ctypes.byref(w), x, T, top_k, wfmt, out, stream),
           "moe_experts")


def moe_route_noalloc(cfg: moe_config_t, w: moe_weights_t, x: int, T: int, out: int,
                      routing: moe_routing_t, stream: int = 0) -> None:
    """moe_route without a plan: scratch in the library's static device array."""
    _check(lib().moe_route_noalloc(ctypes.byref(cfg), ctypes.byref(w), x, T, out,
                                   ctypes.byref(routing), stream), "moe_route_noalloc")


def moe_route_noalloc_status() -> int:
    """Raw status of moe_route_noalloc's sticky error word on the current
    device (not raised)."""
    return lib().moe_route_noalloc_status()


def moe_routing_get(plan: int, T: int, routing: moe_routing_t, stream: int = 0) -> None:
    _check(lib().moe_routing_get(plan, T, ctypes.byref(routing), stream), "moe_routing_get")


def moe_last_launch_count(plan: int) -> int:
    return lib().moe_last_launch_count(plan)


def moe_get_device_status(plan: int) -> int:
    """Raw status of the sticky device error word (not raised)."""
    return lib().moe_get_device_status(plan)


def moe_debug_stall_barrier(plan: int, stream: int = 0) -> None:
    _check(lib().moe_debug_stall_barrier(plan, stream), "moe_debug_stall_barrier")


def moe_q4_0_packed_bytes(n_mats: int, rows: int, k: int):
    cb, sb = ctypes.c_size_t(), ctypes.c_size_t()
    _check(lib().moe_q4_0_packed_bytes(n_mats, rows, k, ctypes.byref(cb), ctypes.byref(sb)),
           "moe_q4_0_packed_bytes")
    return cb.value, sb.value


def moe_q4_0_pack(blocks: int, n_mats: int, rows: int, k: int, codes: int, scales: int,
                  stream: int = 0) -> None:
    _check(lib().moe_q4_0_pack(blocks, n_mats, rows, k, codes, scales, stream), "moe_q4_0_pack")


def moe_q8_0_packed_bytes(n_mats: int, rows: int, k: int):
    cb, sb = ctypes.c_size_t(), ctypes.c_size_t()
    _check(lib().moe_q8_0_packed_bytes(n_mats, rows, k, ctypes.byref(cb), ctypes.byref(sb)),
           "moe_q8_0_packed_bytes")
    return cb.value, sb.value


def moe_q8_0_pack(blocks: int, n_mats: int, rows: int, k: int, codes: int, scales: int,
                  stream: int = 0) -> None:
    _check(lib().moe_q8_0_pack(blocks, n_mats, rows, k, codes, scales, stream), "moe_q8_0_pack")


def moe_q5_0_packed_bytes(n_mats: int, rows: int, k: int):
    cb, sb = ctypes.c_size_t(), ctypes.c_size_t()
    _check(lib().moe_q5_0_packed_bytes(n_mats, rows, k, ctypes.byref(cb), ctypes.byref(sb)),
           "moe_q5_0_packed_bytes")
    return cb.value, sb.value


def moe_q5_0_pack(blocks: int, n_mats: int, rows: int, k: int, codes: int, scales: int,
                  stream: int = 0) -> None:
    _check(lib().moe_q5_0_pack(blocks, n_mats, rows, k, codes, scales, stream), "moe_q5_0_pack")


def moe_q6_k_packed_bytes(n_mats: int, rows: int, k: int):
    cb, sb = ctypes.c_size_t(), ctypes.c_size_t()
    _check(lib().moe_q6_k_packed_bytes(n_mats, rows, k, ctypes.byref(cb), ctypes.byref(sb)),
           "moe_q6_k_packed_bytes")
    return cb.value, sb.value


def moe_q6_k_pack(blocks: int, n_mats: int, rows: int, k: int, codes: int, scales: int,
                  stream: int = 0) -> None:
    _check(lib().moe_q6_k_pack(blocks, n_mats, rows, k, codes, scales, stream), "moe_q6_k_pack")


def moe_bf16_to_f16(src: int, n: int, dst: int, stream: int = 0) -> None:
    _check(lib().moe_bf16_to_f16(src, n, dst, stream), "moe_bf16_to_f16")
