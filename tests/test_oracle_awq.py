"""Pins of the AWQ W4A16 oracle (CPU only) against what the definition and
the mathematics fix: on-grid round trip and error bound of the asymmetric
4-bit quantiser, the all-zero group, the activation-aware scaling
invariance, the special case that reduces the layer to an integer matrix
product, and an exact-rational brute force with its own loops."""
from fractions import Fraction

import numpy as np
import pytest

from oracle import awq as A
from oracle import formats as F

G = A.G_AWQ


def test_quantizer_grid_roundtrip():
    """Groups built as (q - z) s with q covering 0..15, an integer z and a
    bf16 s come back unchanged: codes, scales and zeros bit for bit."""
    g = np.random.default_rng(20)
    N, ng = 32, 6
    q = g.integers(0, 16, (N, ng, G))
    q[:, :, 0] = 0
    q[:, :, 1] = 15                                    # the group spans the code range
    z = g.integers(0, 16, (N, ng))
    s = F.bf16_round(np.exp(g.normal(-4, 1, (N, ng))))
    w = ((q - z[:, :, None]) * s[:, :, None]).reshape(N, ng * G)
    codes, sb, zz = A.quantize_groups(w)
    assert np.array_equal(F.bf16_from_bits(sb), s)
    assert np.array_equal(zz, z)
    assert np.array_equal(codes.reshape(N, ng, G), q)
    assert np.array_equal(A.dequantize(codes, sb, zz), w)


def test_quantizer_error_bound_and_zero_group():
    g = np.random.default_rng(21)
    N, K = 64, 8 * G
    w = g.standard_normal((N, K)) * np.exp(g.normal(0, 1, (N, 1))) + g.normal(0, 0.5, (N, 1))
    w[3, :G] = 0.0                                     # all-zero group
    w[4, G:2 * G] = 0.75                               # constant group: range [0, 0.75]
    codes, sb, zz = A.quantize_groups(w)
    deq = A.dequantize(codes, sb, zz)
    s = np.repeat(F.bf16_from_bits(sb), G, axis=1)
    assert codes.max() <= 15 and zz.max() <= 15
    # rounding to the grid: at most half a step, plus half a step where the
    # rounded zero point moves the grid's end inside the group's range
    assert np.all(np.abs(w - deq) <= s * (1 + 1e-12))
    inner = np.abs(w - deq) <= s / 2 * (1 + 1e-12)
    assert inner.mean() > 0.99
    assert np.all(codes[3, :G] == 0) and sb[3, 0] == 0 and zz[3, 0] == 0
    assert np.all(deq[3, :G] == 0.0)
    assert zz[4, 1] == 0 and np.all(np.abs(deq[4, G:2 * G] - 0.75) <= F.bf16_from_bits(sb[4, 1]) / 2)


def test_channel_factor_scaling_invariance():
    g = np.random.default_rng(22)
    x = g.standard_normal((16, 128))
    x[:, 5] *= 30
    x[:, 7] = 0.0                                      # zero channel -> factor 1
    w = g.standard_normal((128, 40)) * 0.02
    a = A.channel_factors(x).astype(np.float64)
    assert a[7] == 1.0
    assert a[5] == np.float32(np.mean(np.abs(x[:, 5])) ** 0.5)
    lhs = (x / a[None, :]) @ (a[:, None] * w)
    assert np.allclose(lhs, x @ w, rtol=1e-13, atol=1e-15)


def test_integer_special_case():
    """a = 1, s = 1, z = 8: y = x (q - 8)^T, an integer matrix product."""
    g = np.random.default_rng(23)
    M, K, N = 5, 2 * G, 12
    xi = g.integers(-20, 21, (M, K))
    q = g.integers(0, 16, (N, K)).astype(np.uint8)
    p = A.PreparedAWQ(K=K, N=N, a=np.ones(K, np.float32), codes=F.pack_nibbles(q),
                      scales=F.bf16_bits(np.ones((N, K // G))), zeros=np.full((N, K // G), 8, np.uint8),
                      bias=None)
    y, Y = A.forward(F.bf16_bits(xi.astype(np.float64)), p)
    ref = xi.astype(np.int64) @ (q.astype(np.int64) - 8).T
    assert np.array_equal(y, ref.astype(np.float64))


def _f32(fr: Fraction) -> Fraction:
    return Fraction(float(np.float32(float(fr)))) if fr != 0 else Fraction(0)


@pytest.mark.parametrize("with_bias", [False, True])
def test_brute_force_forward(with_bias):
    """Exact rationals, explicit loops: x' = fp32(x * fp32(1/a)), then
    sum_g s sum_k x' (q - z) (+ bias)."""
    g = np.random.default_rng(24 + with_bias)
    M, K, N = 3, 2 * G, 5
    x = g.standard_normal((M, K))
    x[:, 2] *= 20
    x_bits = F.bf16_bits(x)
    w = g.standard_normal((K, N)) * 0.05
    bias_bits = F.bf16_bits(g.standard_normal(N)) if with_bias else None
    p = A.prepare(x_bits, w, bias_bits=bias_bits)
    y, Y = A.forward(x_bits, p)

    xv = F.bf16_from_bits(x_bits)
    inv = [Fraction(float(np.float32(1.0) / np.float32(v))) for v in p.a]
    nib = F.unpack_nibbles(p.codes)
    sv = F.bf16_from_bits(p.scales)
    for m in range(M):
        xp = [_f32(Fraction(float(xv[m, k])) * inv[k]) for k in range(K)]
        for n in range(N):
            acc = Fraction(0)
            for gi in range(K // G):
                part = sum(xp[k] * (int(nib[n, k]) - int(p.zeros[n, gi])) for k in range(gi * G, gi * G + G))
                acc += Fraction(float(sv[n, gi])) * part
            if with_bias:
                acc += Fraction(float(F.bf16_from_bits(bias_bits)[n]))
            assert abs(float(acc) - y[m, n]) <= 1e-12 * max(1.0, abs(float(acc)))
    assert np.array_equal(Y, F.bf16_bits(y))
