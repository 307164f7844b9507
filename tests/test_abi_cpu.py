"""C-ABI boundary checks that need no GPU: the library loads, exports every
symbol include/svdq.h declares, and host-side validation rejects bad calls
before touching the device."""
import ctypes
import os
import re

import numpy as np
import pytest

from bit_diffusion_transformer_w4a4_b200 import svdq
from bit_diffusion_transformer_w4a4_b200 import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_functions():
    src = open(os.path.join(ROOT, "include", "svdq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(svdq_\w+)\s*\(", src)))


def test_library_exports_every_header_symbol():
    L = svdq.lib()
    names = header_functions()
    assert len(names) >= 12
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(svdq.EXPORTED)


def test_status_strings_and_version():
    L = svdq.lib()
    for code, name in svdq.STATUS.items():
        assert L.svdq_status_string(code).decode() == name
    assert b"sm_100a" in L.svdq_version()


def _desc(**kw):
    lay = W.Layer("t", M=64, K=256, N=128, r=16, variant=W.INT4, config_id=9)
    pw = W.synthetic_packed(lay)
    keep = [pw.lam, pw.L1, pw.L2, pw.codes, pw.scales]
    d = svdq.WeightDesc(kw.get("variant", 0), kw.get("K", 256), kw.get("N", 128),
                        kw.get("r", 16), kw.get("max_M", 64), kw.get("flags", 0),
                        pw.lam.ctypes.data, pw.L1.ctypes.data, pw.L2.ctypes.data,
                        pw.codes.ctypes.data, pw.scales.ctypes.data, 0)
    return d, keep


@pytest.mark.parametrize("kw,code", [
    (dict(variant=5), 1), (dict(flags=8), 1),
    (dict(K=200), 2), (dict(K=64), 2), (dict(N=100), 2), (dict(r=24), 2), (dict(max_M=0), 2),
])
def test_load_validation(kw, code):
    L = svdq.lib()
    d, keep = _desc(**kw)
    h = ctypes.c_void_p(0)
    assert L.svdq_weights_load(ctypes.byref(d), ctypes.byref(h), None) == code
    assert not h.value


def test_null_arguments():
    L = svdq.lib()
    h = ctypes.c_void_p(0)
    assert L.svdq_weights_load(None, ctypes.byref(h), None) == 1
    d, keep = _desc()
    assert L.svdq_weights_load(ctypes.byref(d), None, None) == 1
    assert L.svdq_weights_free(None) == 0
    assert L.svdq_linear_forward(None, None, None, 1, None) == 1
    assert L.svdq_quantize_act_lowrank_down(None, None, 1, None, None, None, None) == 1
    assert L.svdq_w4a4_gemm_lowrank_up(None, None, None, None, 1, None, None) == 1
    assert L.svdq_device_status(None, None) == 1
    assert L.svdq_debug_set_fault(None, 1, 10) == 1
    assert L.svdq_set_deterministic(None, 1) == 1
    assert L.svdq_device_error_site(None, None, None) == 1
    n = ctypes.c_size_t(0)
    assert L.svdq_act_scales_bytes(None, 1, ctypes.byref(n)) == 1


def test_nonpositive_lambda_rejected():
    L = svdq.lib()
    d, keep = _desc()
    keep[0][3] = 0.0
    h = ctypes.c_void_p(0)
    assert L.svdq_weights_load(ctypes.byref(d), ctypes.byref(h), None) == 1


def test_no_gpu_no_fallback():
    """Without an sm_100 device the library refuses; nothing runs on the CPU."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    L = svdq.lib()
    d, keep = _desc()
    h = ctypes.c_void_p(0)
    assert L.svdq_weights_load(ctypes.byref(d), ctypes.byref(h), None) == 4
    n = (ctypes.c_ulonglong * 2)()
    assert L.svdq_selftest_division(1, n) == 4


def _awq_desc(**kw):
    lay = W.AWQLayer("t", M=2, K=128, N=16, config_id=93)
    p = W.synthetic_awq(lay)
    zeros = kw.get("zeros", p.zeros)
    keep = [p.a, p.codes, p.scales, zeros]
    d = svdq.AWQDesc(kw.get("K", 128), kw.get("N", 16), kw.get("max_M", 2),
                     p.a.ctypes.data, p.codes.ctypes.data, p.scales.ctypes.data, zeros.ctypes.data, 0)
    return d, keep


@pytest.mark.parametrize("kw,code", [
    ({"K": 96}, 2), ({"K": 0}, 2), ({"N": 0}, 2), ({"max_M": 0}, 2),
    ({"zeros": np.full((16, 2), 16, np.uint8)}, 1),
])
def test_awq_load_validation(kw, code):
    """Host-side validation of svdq_awq_load runs before any device work."""
    L = svdq.lib()
    d, keep = _awq_desc(**kw)
    h = ctypes.c_void_p(0)
    assert L.svdq_awq_load(ctypes.byref(d), ctypes.byref(h), None) == code
    assert not h.value
    assert L.svdq_awq_free(None) == 0


@pytest.mark.parametrize("kw,code", [
    ({"variant": 0, "flags": 8}, 1),           # QKV epilogue: NVFP4 only
    ({"variant": 1, "flags": 8 | 1}, 1),       # not with GELU
    ({"variant": 1, "flags": 8, "N": 256}, 2),  # N must be a multiple of 3 x 128
])
def test_qkv_flag_validation(kw, code):
    L = svdq.lib()
    variant = kw["variant"]
    N = kw.get("N", 384)
    lay = W.Layer("t", M=64, K=256, N=N, r=16, variant=variant, config_id=9)
    pw = W.synthetic_packed(lay)
    g = np.full(128, 0x3F80, np.uint16)
    d = svdq.WeightDesc(variant, 256, N, 16, 64, kw["flags"], pw.lam.ctypes.data, pw.L1.ctypes.data,
                        pw.L2.ctypes.data, pw.codes.ctypes.data, pw.scales.ctypes.data, 0, 0,
                        g.ctypes.data, g.ctypes.data, 1e-6)
    h = ctypes.c_void_p(0)
    assert L.svdq_weights_load(ctypes.byref(d), ctypes.byref(h), None) == code
    assert not h.value
