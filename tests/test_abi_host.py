"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every function include/moe.h declares, and rejects invalid arguments before
touching CUDA."""
import ctypes
import subprocess

import pytest

from mixture_experts_layer_43_b200 import binding as B
from mixture_experts_layer_43_b200 import build as build_mod


@pytest.fixture(scope="module")
def L():
    build_mod.build()
    return B.lib()


def test_exports_every_declared_function(L):
    names = B.header_functions()
    assert len(names) >= 11
    for n in names:
        assert hasattr(L, n), f"{n} declared in include/moe.h but not exported"
    out = subprocess.run(["nm", "-D", "--defined-only", B.LIB_PATH], capture_output=True,
                         text=True).stdout
    exported = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    assert set(names) <= exported
    # nothing else with the public prefix is exported
    assert {n for n in exported if n.startswith("moe_")} == set(names)


def test_status_strings(L):
    for s in range(7):
        assert B.moe_status_string(s)
    assert B.moe_status_string(99) == "unknown status"


def _cfg(**kw):
    base = dict(t_max=8, d_model=256, d_ff=512, n_experts=8, top_k=2, n_shared=0,
                d_ff_shared=0, wfmt=0, regime=0, device=0)
    base.update(kw)
    return B.moe_config_t(**base)


@pytest.mark.parametrize("kw", [
    dict(t_max=0), dict(d_model=100), dict(d_model=192), dict(d_ff=48), dict(n_experts=0),
    dict(n_experts=2000), dict(top_k=0), dict(top_k=9), dict(n_experts=32, top_k=17),
    dict(n_shared=-1), dict(n_shared=9), dict(n_shared=1, d_ff_shared=0),
    dict(n_shared=1, d_ff_shared=40), dict(wfmt=6), dict(regime=3), dict(device=-1),
])
def test_plan_create_rejects_bad_config(L, kw):
    plan = ctypes.c_void_p(123)
    s = L.moe_plan_create(ctypes.byref(_cfg(**kw)), ctypes.byref(plan))
    assert s == B.MOE_ERR_INVALID_ARG
    assert plan.value is None


def test_plan_create_q4_prefill_unsupported(L):
    plan = ctypes.c_void_p()
    s = L.moe_plan_create(ctypes.byref(_cfg(wfmt=1, regime=2)), ctypes.byref(plan))
    assert s == B.MOE_ERR_UNSUPPORTED
    s = L.moe_plan_create(ctypes.byref(_cfg(wfmt=2, regime=2)), ctypes.byref(plan))
    assert s == B.MOE_ERR_UNSUPPORTED
    s = L.moe_plan_create(ctypes.byref(_cfg(wfmt=3, regime=2)), ctypes.byref(plan))
    assert s == B.MOE_ERR_UNSUPPORTED
    # bf16 with fp16 down matrices is a valid prefill format (without a GPU the
    # call gets past the argument checks and fails at the device query)
    s = L.moe_plan_create(ctypes.byref(_cfg(wfmt=5, regime=2)), ctypes.byref(plan))
    assert s not in (B.MOE_ERR_UNSUPPORTED, B.MOE_ERR_INVALID_ARG)
    # 6 is not a format of this ABI
    s = L.moe_plan_create(ctypes.byref(_cfg(wfmt=6)), ctypes.byref(plan))
    assert s == B.MOE_ERR_INVALID_ARG
    # q6_K needs 256-multiples along every reduction dim, and runs in decode only
    s = L.moe_plan_create(ctypes.byref(_cfg(wfmt=4, d_model=384)), ctypes.byref(plan))
    assert s == B.MOE_ERR_INVALID_ARG
    s = L.moe_plan_create(ctypes.byref(_cfg(wfmt=4, regime=2, d_model=256, d_ff=256)),
                          ctypes.byref(plan))
    assert s == B.MOE_ERR_UNSUPPORTED


def test_q6_packed_bytes(L):
    assert B.moe_q6_k_packed_bytes(2, 32, 512) == (2 * 32 * 16 * 16, 2 * 2 * 16 * 160 + 2 * 2 * 32 * 2)
    for bad in ((1, 32, 288), (1, 24, 256), (-1, 16, 256)):
        with pytest.raises(B.MoeError):
            B.moe_q6_k_packed_bytes(*bad)
    assert L.moe_q6_k_pack(None, 1, 16, 288, None, None, None) == B.MOE_ERR_INVALID_ARG
    assert L.moe_q6_k_pack(None, 1, 16, 256, None, None, None) == B.MOE_ERR_INVALID_ARG


def test_bf16_to_f16_rejects_bad_args_without_gpu(L):
    assert L.moe_bf16_to_f16(None, -1, None, None) == B.MOE_ERR_INVALID_ARG
    assert L.moe_bf16_to_f16(None, 4, None, None) == B.MOE_ERR_INVALID_ARG
    assert L.moe_bf16_to_f16(None, 0, None, None) == B.MOE_OK
    assert L.moe_bf16_to_f16(ctypes.c_void_p(0x1001), 4, ctypes.c_void_p(0x2000), None) == \
        B.MOE_ERR_INVALID_ARG


def test_null_arguments(L):
    assert L.moe_plan_create(None, None) == B.MOE_ERR_INVALID_ARG
    w = B.moe_weights_t()
    assert L.moe_forward(None, ctypes.byref(w), None, 1, 2, 0, None, None, None) == \
        B.MOE_ERR_INVALID_ARG
    assert L.moe_route(None, ctypes.byref(w), None, 1, 2, 0, None, None) == B.MOE_ERR_INVALID_ARG
    assert L.moe_experts(None, None, None, 1, 2, 0, None, None) == B.MOE_ERR_INVALID_ARG
    assert L.moe_routing_get(None, 1, None, None) == B.MOE_ERR_INVALID_ARG
    assert L.moe_get_device_status(None) == B.MOE_ERR_INVALID_ARG
    assert L.moe_last_launch_count(None) == -1
    L.moe_plan_destroy(None)


def test_q4_packed_bytes(L):
    assert B.moe_q4_0_packed_bytes(256, 512, 2048) == (256 * 512 * 64 * 16, 256 * 512 * 64 * 2)
    assert B.moe_q4_0_packed_bytes(0, 5, 32) == (0, 0)
    cb = ctypes.c_size_t()
    assert L.moe_q4_0_packed_bytes(1, 1, 33, ctypes.byref(cb), None) == B.MOE_ERR_INVALID_ARG
    assert L.moe_q4_0_packed_bytes(-1, 1, 32, None, None) == B.MOE_ERR_INVALID_ARG


def test_q4_pack_rejects_bad_args_without_gpu(L):
    assert L.moe_q4_0_pack(None, 1, 1, 33, None, None, None) == B.MOE_ERR_INVALID_ARG
    assert L.moe_q4_0_pack(None, 1, 1, 32, None, None, None) == B.MOE_ERR_INVALID_ARG
    # misaligned destination
    assert L.moe_q4_0_pack(16, 1, 1, 32, 17, 32, None) == B.MOE_ERR_INVALID_ARG
    # empty is a no-op
    assert L.moe_q4_0_pack(None, 0, 4, 32, None, None, None) == B.MOE_OK


def test_q8_packed_bytes(L):
    assert B.moe_q8_0_packed_bytes(256, 512, 2048) == (256 * 512 * 64 * 32, 256 * 512 * 64 * 2)
    assert B.moe_q8_0_packed_bytes(0, 5, 32) == (0, 0)
    cb = ctypes.c_size_t()
    assert L.moe_q8_0_packed_bytes(1, 1, 33, ctypes.byref(cb), None) == B.MOE_ERR_INVALID_ARG
    assert L.moe_q8_0_packed_bytes(-1, 1, 32, None, None) == B.MOE_ERR_INVALID_ARG


def test_q8_pack_rejects_bad_args_without_gpu(L):
    assert L.moe_q8_0_pack(None, 1, 1, 33, None, None, None) == B.MOE_ERR_INVALID_ARG
    assert L.moe_q8_0_pack(None, 1, 1, 32, None, None, None) == B.MOE_ERR_INVALID_ARG
    assert L.moe_q8_0_pack(16, 1, 1, 32, 17, 32, None) == B.MOE_ERR_INVALID_ARG
    assert L.moe_q8_0_pack(None, 0, 4, 32, None, None, None) == B.MOE_OK


def test_q5_packed_bytes(L):
    # 16 code bytes and 6 bytes of scale + fifth bits per block
    assert B.moe_q5_0_packed_bytes(256, 512, 2048) == (256 * 512 * 64 * 16, 256 * 512 * 64 * 6)
    assert B.moe_q5_0_packed_bytes(0, 8, 32) == (0, 0)
    cb = ctypes.c_size_t()
    assert L.moe_q5_0_packed_bytes(1, 8, 33, ctypes.byref(cb), None) == B.MOE_ERR_INVALID_ARG
    assert L.moe_q5_0_packed_bytes(-1, 8, 32, None, None) == B.MOE_ERR_INVALID_ARG
    # records of 8 rows: rows must be a multiple of 8
    assert L.moe_q5_0_packed_bytes(1, 12, 32, ctypes.byref(cb), None) == B.MOE_ERR_INVALID_ARG


def test_q5_pack_rejects_bad_args_without_gpu(L):
    assert L.moe_q5_0_pack(None, 1, 8, 33, None, None, None) == B.MOE_ERR_INVALID_ARG
    assert L.moe_q5_0_pack(None, 1, 8, 32, None, None, None) == B.MOE_ERR_INVALID_ARG
    assert L.moe_q5_0_pack(None, 1, 4, 32, None, None, None) == B.MOE_ERR_INVALID_ARG
    assert L.moe_q5_0_pack(16, 1, 8, 32, 17, 32, None) == B.MOE_ERR_INVALID_ARG
    assert L.moe_q5_0_pack(None, 0, 8, 32, None, None, None) == B.MOE_OK

