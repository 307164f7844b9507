"""Pins of the QKV-epilogue oracle (CPU only): unit RMS per normalised head,
rotation keeps each pair's norm, cos = 1 / sin = 0 is the identity, a
quarter turn maps (a, b) to (-b, a), V is untouched, and an explicit-loop
restatement on a small case."""
import math

import numpy as np

from oracle import formats as F
from oracle import qkv as Q

D = Q.HEAD_DIM


def _case(M=5, H=2, seed=40):
    g = np.random.default_rng(seed)
    acc = g.standard_normal((M, 3 * H * D)) * np.exp(g.normal(0, 1, (M, 1)))
    gq = F.bf16_bits(1 + 0.1 * g.standard_normal(D))
    gk = F.bf16_bits(1 + 0.1 * g.standard_normal(D))
    ang = g.uniform(-math.pi, math.pi, (M, D // 2))
    return acc, gq, gk, np.cos(ang), np.sin(ang)


def test_rms_norm_unit_rms():
    acc, gq, gk, c, s = _case()
    HD = acc.shape[1] // 3
    ones = np.ones(D)
    n = Q.rms_norm_heads(acc[:, :HD], ones, eps=0.0).reshape(acc.shape[0], -1, D)
    assert np.allclose(np.sqrt(np.mean(n * n, axis=2)), 1.0, rtol=1e-14)
    # eps: a zero head stays zero, a tiny head is damped
    z = Q.rms_norm_heads(np.zeros((1, D)), ones)
    assert np.all(z == 0)


def test_rope_rotation_properties():
    acc, gq, gk, c, s = _case(seed=41)
    HD = acc.shape[1] // 3
    v = acc[:, :HD]
    r = Q.rope_heads(v, c, s)
    pv = v.reshape(v.shape[0], -1, D // 2, 2)
    pr = r.reshape(v.shape[0], -1, D // 2, 2)
    assert np.allclose(np.hypot(pv[..., 0], pv[..., 1]), np.hypot(pr[..., 0], pr[..., 1]), rtol=1e-13)
    ident = Q.rope_heads(v, np.ones_like(c), np.zeros_like(s))
    assert np.array_equal(ident, v)
    qt = Q.rope_heads(v, np.zeros_like(c), np.ones_like(s)).reshape(pv.shape)
    assert np.array_equal(qt[..., 0], -pv[..., 1]) and np.array_equal(qt[..., 1], pv[..., 0])
    # rotating by theta then by -theta is the identity
    back = Q.rope_heads(r, c, -s)
    assert np.allclose(back, v, rtol=1e-12, atol=1e-12)


def test_epilogue_explicit_loops():
    acc, gq, gk, c, s = _case(M=3, H=2, seed=42)
    y, Y = Q.qkv_epilogue(acc, gq, gk, c, s)
    M, N = acc.shape
    HD = N // 3
    gqv, gkv = F.bf16_from_bits(gq), F.bf16_from_bits(gk)
    for m in range(M):
        for part, gv in ((0, gqv), (1, gkv)):
            for h in range(HD // D):
                col0 = part * HD + h * D
                head = [acc[m, col0 + d] for d in range(D)]
                rms = math.sqrt(sum(x * x for x in head) / D + Q.EPS)
                nrm = [head[d] / rms * gv[d] for d in range(D)]
                for i in range(D // 2):
                    a, b = nrm[2 * i], nrm[2 * i + 1]
                    ea = a * c[m, i] - b * s[m, i]
                    eb = a * s[m, i] + b * c[m, i]
                    assert abs(y[m, col0 + 2 * i] - ea) <= 1e-12 * (1 + abs(ea))
                    assert abs(y[m, col0 + 2 * i + 1] - eb) <= 1e-12 * (1 + abs(eb))
        assert np.array_equal(y[m, 2 * HD:], acc[m, 2 * HD:])
    assert np.array_equal(Y, F.bf16_bits(y))
