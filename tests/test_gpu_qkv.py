"""GPU parity of the fused QKV epilogue (SVDQ_EPI_QKV_NORM_ROPE: per-head
RMS normalisation of Q and K, rotary embedding of their interleaved pairs,
V untouched) against the oracle: NVFP4 on SM pairs and on single SMs, with
bias, ragged M, several tiles per CTA, and the layer's own all-row check at
a 2048-px block's qkv shape with the benchmark's inputs."""
import math

import numpy as np
import pytest

from bit_diffusion_transformer_w4a4_b200 import svdq
from bit_diffusion_transformer_w4a4_b200 import workloads as W
from oracle import formats as F
from oracle import forward as O
from oracle import prep as P
from oracle import qkv as Q
import parity as PT

pytestmark = pytest.mark.gpu


def _rope_table(M, seed=0):
    """Angles of a 2-D position grid (the caller's; FLUX-style): token m at
    (m // 64, m % 64), pair frequencies 10000^(-i/32) split over two axes."""
    i = np.arange(64)
    freq = 10000.0 ** (-(i % 32) / 32.0)
    m = np.arange(M)
    pos = np.where(i[None, :] < 32, (m // 64)[:, None], (m % 64)[:, None]).astype(np.float64)
    ang = pos * freq[None, :] + 0.1 * seed
    return np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)


def _run(M, H, r, opts, with_bias=True, seed=0, pw_kind="prep"):
    import torch
    N = 3 * H * 128
    lay = W.Layer("qkv", M=M, K=512, N=N, r=r, variant=W.NVFP4, bias=with_bias, config_id=99, layer_id=H)
    x = W.activations(lay)
    if pw_kind == "prep":
        pw = P.prepare(x, W.weight(lay), r, W.NVFP4, bias_bits=W.bias(lay))
    else:
        pw = W.synthetic_packed(lay)
    g = np.random.default_rng(seed + 5)
    gq = F.bf16_bits(1 + 0.2 * g.standard_normal(128))
    gk = F.bf16_bits(1 + 0.2 * g.standard_normal(128))
    cos, sin = _rope_table(M, seed)
    rope = np.stack([cos, sin], axis=-1).reshape(M, 128)
    h = svdq.SVDQWeights(pw, M, qkv_norm=(gq, gk, 1e-6), **opts)
    xd = PT.to_dev(x.view(np.int16)).view(torch.bfloat16)
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    h.linear_forward_qkv(xd, PT.to_dev(rope), y, M)
    torch.cuda.synchronize()
    assert h.device_status() == 0
    Y = PT.from_dev(y.view(torch.int16)).view(np.uint16)
    h.close()
    ref = O.linear_forward(x, pw)              # the plain layer's y (fp64, pre-rounding)
    yq, Yq = Q.qkv_epilogue(ref["y"], gq, gk, cos.astype(np.float64), sin.astype(np.float64))
    return Y, yq, Yq


@pytest.mark.parametrize("opts", [{}, {"single_sm": True}], ids=["pair", "1sm"])
@pytest.mark.parametrize("M,H,r", [(300, 2, 32), (129, 1, 16), (640, 3, 0), (1, 1, 32)])
def test_qkv_epilogue(opts, M, H, r):
    Y, yq, Yq = _run(M, H, r, opts)
    PT.check_y(Y, yq, Yq, label=f"qkv M{M} H{H} r{r} {opts}")


def test_qkv_epilogue_many_tiles():
    """More tiles than SM pairs: the per-head exchange barriers run through
    several phases per CTA."""
    Y, yq, Yq = _run(2048, 8, 32, {}, pw_kind="synthetic")
    PT.check_y(Y, yq, Yq, label="qkv many tiles")


def test_qkv_plain_calls_refused():
    """A QKV handle needs the rotary table: the plain entry points refuse it."""
    import torch
    lay = W.Layer("qkv", M=128, K=256, N=384, r=16, variant=W.NVFP4, config_id=99)
    pw = W.synthetic_packed(lay)
    ones = F.bf16_bits(np.ones(128))
    h = svdq.SVDQWeights(pw, 128, qkv_norm=(ones, ones, 1e-6))
    x = torch.zeros((128, 256), dtype=torch.bfloat16, device="cuda")
    y = torch.empty((128, 384), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(svdq.SvdqError):
        h.linear_forward(x, y, 128)
    h.close()


def test_qkv_epilogue_block_full_size():
    """The 2048-px block's qkv layer (M16896 K3072 N9216 r32, NVFP4, SM pairs)
    with the benchmark's norm weights and rotary table, in the launch
    configuration the benchmark times: every row against the oracle."""
    import torch
    lay = W.workloads()["block_2048px"][0]
    assert lay.name.endswith("qkv") and lay.variant == W.NVFP4
    x = W.activations(lay)
    pw = W.synthetic_packed(lay)
    gq, gk, rope = W.qkv_epilogue_inputs(lay.M, 0)
    h = svdq.SVDQWeights(pw, lay.M, qkv_norm=(gq, gk, 1e-6))
    xd = PT.to_dev(x.view(np.int16)).view(torch.bfloat16)
    y = torch.empty((lay.M, lay.N), dtype=torch.bfloat16, device="cuda")
    h.linear_forward_qkv(xd, PT.to_dev(rope), y, lay.M)
    torch.cuda.synchronize()
    assert h.device_status() == 0
    Y = PT.from_dev(y.view(torch.int16)).view(np.uint16)
    h.close()
    act = PT.oracle_act_all(pw, x)
    acc, _ = PT.oracle_y_all(pw, act)
    yq, Yq = Q.qkv_epilogue(acc, gq, gk, rope[:, 0::2].astype(np.float64), rope[:, 1::2].astype(np.float64))
    PT.check_y(Y, yq, Yq, label="qkv block 2048px")
