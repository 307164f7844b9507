"""GPU parity at the workloads' full sizes, in the launch configuration the
benchmark times.  Every token row goes through both kernels on the GPU and
every row is compared with the oracle: activation codes and scales
bit-exact, T within the fp32-accumulation bound, Y within the layer's bars
(the oracle's fp64 GEMM runs in row blocks)."""
import numpy as np
import pytest

from bit_diffusion_transformer_w4a4_b200 import svdq
from bit_diffusion_transformer_w4a4_b200 import workloads as W
from oracle import forward as O
from oracle import prep as P
import parity as PT

pytestmark = pytest.mark.gpu

WL = W.workloads()
CASES = [(name, i) for name, layers in WL.items() for i in range(len(layers))]


def _check_all_rows(h, pw, x, layer, label):
    got = PT.gpu_forward(h, x, layer.M)
    act = PT.oracle_act_all(pw, x)
    tb = PT.t_bound_all(pw, x) if layer.r > 0 else None
    PT.check_act(got, act, r=layer.r, label=label, tb=tb)
    y, Y = PT.oracle_y_all(pw, act)
    PT.check_y(got["Y"], y, Y, label=label)


@pytest.mark.parametrize("name,li", CASES, ids=[f"{n}-{i}" for n, i in CASES])
def test_workload_full_size(name, li):
    layer = WL[name][li]
    x = W.activations(layer)
    if name in ("tiny",):
        pw = P.prepare(x, W.weight(layer), layer.r, layer.variant, gelu=layer.gelu)
    else:
        pw = W.synthetic_packed(layer)
    h = svdq.SVDQWeights(pw, layer.M)
    _check_all_rows(h, pw, x, layer, f"{name}[{li}]")
    h.close()


@pytest.mark.parametrize("name,opts", [("qkv_int4", {}), ("qkv_int4", {"int4_f16": True}),
                                       ("fc1_nvfp4", {})], ids=["qkv_int4", "qkv_int4-f16", "fc1_nvfp4"])
def test_workload_with_svd_prep(name, opts):
    """Full-size layer whose weights come from the oracle's calibration, SVD
    and residual quantisation (the method's own weight distribution); the INT4
    layer also through the fp16-operand GEMM.  All rows."""
    layer = WL[name][0]
    x = W.activations(layer)
    pw = P.prepare(x, W.weight(layer), layer.r, layer.variant, gelu=layer.gelu)
    h = svdq.SVDQWeights(pw, layer.M, **opts)
    _check_all_rows(h, pw, x, layer, f"{name} prepped{' f16' if opts else ''}")
    h.close()


INT4_CASES = [(n, i) for n, i in CASES if WL[n][i].variant == W.INT4]


@pytest.mark.parametrize("name,li", INT4_CASES, ids=[f"{n}-{i}" for n, i in INT4_CASES])
def test_workload_full_size_int4_f16(name, li):
    """Every INT4 workload layer at full size through the fp16-operand GEMM
    (SVDQ_INT4_F16), all rows against the oracle."""
    layer = WL[name][li]
    x = W.activations(layer)
    pw = W.synthetic_packed(layer)
    h = svdq.SVDQWeights(pw, layer.M, int4_f16=True)
    _check_all_rows(h, pw, x, layer, f"{name}[{li}] f16")
    h.close()
