"""GPU parity at the workloads' full sizes, in the launch configuration the
benchmark times: every token row goes through both kernels on the GPU; the
oracle recomputes a sample of rows (first, last, and random ones) and those
are compared -- codes and scales bit-exact, T and Y within the stated bars."""
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


def _rows(M, n=96, seed=0):
    g = np.random.default_rng(seed)
    r = np.unique(np.concatenate([[0, 1, M // 2, M - 1], g.choice(M, min(n, M), replace=False)]))
    return r


@pytest.mark.parametrize("name,li", CASES, ids=[f"{n}-{i}" for n, i in CASES])
def test_workload_full_size(name, li):
    layer = WL[name][li]
    x = W.activations(layer)
    if name in ("tiny",):
        pw = P.prepare(x, W.weight(layer), layer.r, layer.variant, gelu=layer.gelu)
    else:
        pw = W.synthetic_packed(layer)
    h = svdq.SVDQWeights(pw, layer.M)
    got = PT.gpu_forward(h, x, layer.M)
    rows = _rows(layer.M)
    ref = O.linear_forward(x, pw, rows=rows)
    tb = None
    if layer.r > 0:
        inv = (np.float32(1) / pw.lam).astype(np.float32)
        xp = O.smooth_activations(x[rows], inv).astype(np.float64)
        tb = PT.t_bound(xp, W.bf16_bits_to_f32(pw.L1).astype(np.float64))
    PT.check_act(got, ref, rows=rows, r=layer.r, label=f"{name}[{li}]", tb=tb)
    PT.check_y(got["Y"][rows], ref["y"], ref["Y"], label=f"{name}[{li}]")
    h.close()


@pytest.mark.parametrize("name,opts", [("qkv_int4", {}), ("qkv_int4", {"int4_f16": True}),
                                       ("fc1_nvfp4", {})], ids=["qkv_int4", "qkv_int4-f16", "fc1_nvfp4"])
def test_workload_with_svd_prep(name, opts):
    """Full-size layer whose weights come from the oracle's calibration, SVD
    and residual quantisation (the method's own weight distribution); the INT4
    layer also through the fp16-operand GEMM."""
    layer = WL[name][0]
    x = W.activations(layer)
    pw = P.prepare(x, W.weight(layer), layer.r, layer.variant, gelu=layer.gelu)
    h = svdq.SVDQWeights(pw, layer.M, **opts)
    got = PT.gpu_forward(h, x, layer.M, two_calls=False)
    rows = _rows(layer.M, 64, seed=1)
    ref = O.linear_forward(x, pw, rows=rows)
    PT.check_y(got["Y"][rows], ref["y"], ref["Y"], label=f"{name} prepped")
    h.close()


INT4_CASES = [(n, i) for n, i in CASES if WL[n][i].variant == W.INT4]


@pytest.mark.parametrize("name,li", INT4_CASES, ids=[f"{n}-{i}" for n, i in INT4_CASES])
def test_workload_full_size_int4_f16(name, li):
    """Every INT4 workload layer at full size through the fp16-operand GEMM
    (SVDQ_INT4_F16), sampled rows against the oracle."""
    layer = WL[name][li]
    x = W.activations(layer)
    pw = W.synthetic_packed(layer)
    h = svdq.SVDQWeights(pw, layer.M, int4_f16=True)
    got = PT.gpu_forward(h, x, layer.M)
    rows = _rows(layer.M, seed=2)
    ref = O.linear_forward(x, pw, rows=rows)
    PT.check_y(got["Y"][rows], ref["y"], ref["Y"], label=f"{name}[{li}] f16")
    h.close()
