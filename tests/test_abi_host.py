"""Host-side checks of the C ABI: the library builds, loads, exports every entry
point include/moe.h declares, and rejects bad arguments before touching a GPU."""
import ctypes
import os
import re

import pytest

import routed_expert_ffn_sqrtsoftplus_b200 as moe
from routed_expert_ffn_sqrtsoftplus_b200 import build as moe_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    moe_build.build()
    return moe.lib()


def _declared():
    names = []
    for h in os.listdir(os.path.join(ROOT, "include")):
        if h.endswith(".h"):
            with open(os.path.join(ROOT, "include", h)) as f:
                names += re.findall(r"MOE_API\s+[^;(]*?\b(moe_\w+)\s*\(", f.read())
    return names


def test_every_declared_symbol_is_exported(L):
    declared = _declared()
    assert len(declared) >= 16
    for name in declared:
        assert hasattr(L, name), name
    assert set(moe.EXPORTED) <= set(declared)


def test_exports_are_exactly_the_header(L):
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", moe.LIB_PATH], capture_output=True, text=True).stdout
    exported = {l.split()[-1] for l in out.splitlines() if " T " in l}
    assert exported == set(_declared())


def test_abi_version_and_strings(L):
    assert L.moe_abi_version() == 4
    assert L.moe_status_string(moe.MOE_OK) == b"MOE_OK"
    assert L.moe_status_string(moe.MOE_ERR_TIMEOUT) == b"MOE_ERR_TIMEOUT"
    assert L.moe_num_kernel_kinds() == len(moe.kernel_names())
    assert "gemm_gateup" in moe.kernel_names() and "gemm_down" in moe.kernel_names()
    assert L.moe_kernel_name(-1) is None


def _cfg(**kw):
    base = dict(hidden=512, inter=256, n_routed=32, n_shared=1, top_k=6, max_tokens=64, route_scale=1.5,
                swiglu_limit=10.0, expert_dtype=0)
    base.update(kw)
    return moe._Config(*[base[f] for f, _ in moe._Config._fields_])


FAKE = 0x10000  # 16-byte aligned; never dereferenced because validation fails first


def _w(**kw):
    d = dict(router_w=FAKE, router_bias=None, w1=FAKE, w3=FAKE, w2=FAKE, s1=None, s3=None, s2=None,
             sh_w1=FAKE, sh_w3=FAKE, sh_w2=FAKE)
    d.update(kw)
    return moe._Weights(*[d[f] for f, _ in moe._Weights._fields_])


@pytest.mark.parametrize("kw,expect", [
    (dict(top_k=0), moe.MOE_ERR_INVALID_ARG),
    (dict(top_k=33, n_routed=64), moe.MOE_ERR_UNSUPPORTED),
    (dict(top_k=7, n_routed=6), moe.MOE_ERR_INVALID_ARG),
    (dict(hidden=500), moe.MOE_ERR_UNSUPPORTED),
    (dict(inter=200), moe.MOE_ERR_UNSUPPORTED),
    (dict(n_routed=513), moe.MOE_ERR_UNSUPPORTED),
    (dict(max_tokens=0), moe.MOE_ERR_INVALID_ARG),
    (dict(max_tokens=70000), moe.MOE_ERR_UNSUPPORTED),
    (dict(route_scale=float("nan")), moe.MOE_ERR_INVALID_ARG),
    (dict(route_scale=0.0), moe.MOE_ERR_INVALID_ARG),
    (dict(swiglu_limit=-1.0), moe.MOE_ERR_INVALID_ARG),
    (dict(swiglu_limit=float("nan")), moe.MOE_ERR_INVALID_ARG),
    (dict(n_shared=-1), moe.MOE_ERR_INVALID_ARG),
    (dict(expert_dtype=7), moe.MOE_ERR_INVALID_ARG),
])
def test_create_rejects_bad_config(L, kw, expect):
    h = ctypes.c_void_p(123)
    st = L.moe_create(ctypes.byref(_cfg(**kw)), ctypes.byref(_w()), None, ctypes.byref(h))
    assert st == expect
    assert not h.value


@pytest.mark.parametrize("wkw", [dict(router_w=None), dict(w1=None), dict(w2=FAKE + 4), dict(sh_w3=None),
                                 dict(router_bias=FAKE + 8)])
def test_create_rejects_bad_pointers(L, wkw):
    h = ctypes.c_void_p(None)
    assert L.moe_create(ctypes.byref(_cfg()), ctypes.byref(_w(**wkw)), None, ctypes.byref(h)) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_create(None, ctypes.byref(_w()), None, ctypes.byref(h)) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_create(ctypes.byref(_cfg()), None, None, ctypes.byref(h)) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_create(ctypes.byref(_cfg()), ctypes.byref(_w()), None, None) == moe.MOE_ERR_INVALID_ARG


def test_create_ep_rejects_bad_windows(L):
    h = ctypes.c_void_p()
    E = _cfg().n_routed
    for b, c in ((-1, 2), (0, 0), (E - 1, 2), (E, 1)):
        assert L.moe_create_ep(ctypes.byref(_cfg()), ctypes.byref(_w()), b, c, None, ctypes.byref(h)) == \
            moe.MOE_ERR_INVALID_ARG
        assert not h.value


def test_null_handle_calls(L):
    assert L.moe_forward(None, FAKE, 1, FAKE, None, None, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_forward_host(None, FAKE, 1, FAKE, None, None, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_forward_host_async(None, FAKE, 1, FAKE, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_forward_host_wait(None, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_get_status(None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_inspect(None, 0, FAKE, 4, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_set_wait_timeout(None, 10) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_profile_begin(None, 1) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_get_info(None, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_set_hash_table(None, FAKE, 10, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_forward_hashed(None, FAKE, FAKE, 1, FAKE, None, None, None) == moe.MOE_ERR_INVALID_ARG
    L.moe_destroy(None)  # no-op


def test_quantize_rejects_bad_shapes(L):
    assert L.moe_quantize_mxfp4(FAKE, 4, 33, FAKE, FAKE, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_quantize_mxfp4(FAKE, -1, 32, FAKE, FAKE, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_quantize_mxfp4(None, 4, 32, FAKE, FAKE, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_quantize_mxfp4(FAKE + 2, 4, 32, FAKE, FAKE, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_quantize_mxfp4(FAKE, 0, 32, FAKE, FAKE, None) == moe.MOE_OK


def test_quantize_mxfp8_rejects_bad_shapes(L):
    assert L.moe_quantize_mxfp8(FAKE, 4, 33, FAKE, FAKE, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_quantize_mxfp8(FAKE, -1, 32, FAKE, FAKE, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_quantize_mxfp8(None, 4, 32, FAKE, FAKE, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_quantize_mxfp8(FAKE, 4, 32, FAKE + 4, FAKE, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_quantize_mxfp8(FAKE, 0, 32, FAKE, FAKE, None) == moe.MOE_OK


def test_binding_refuses_cpu_tensors(L):
    import torch
    with pytest.raises(ValueError):
        moe.quantize_mxfp4(torch.zeros(4, 32, dtype=torch.bfloat16))
