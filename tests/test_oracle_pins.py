"""Pins of the oracle's weight prep and forward against what the method and
the mathematics fix (CPU only).

* exact reconstruction when r = min(K, N) (residual zero, Y = X W);
* smoothing invariance (X diag(l)^-1)(diag(l) W) = X W;
* Eckart-Young: the rank-r residual norm equals the tail singular values;
* low-rank branch alone reconstructs L1 L2 (lambda = 1, X = I, zero codes);
* quantiser round-trip of on-grid groups and its error bound;
* brute force on 8x8 problems in exact rational arithmetic, sharing no code
  with the oracle (its own rounding, its own loops).
"""
import math
from fractions import Fraction

import numpy as np
import pytest

from oracle import formats as F
from oracle import forward as O
from oracle import prep as P

INT4, NVFP4 = O.INT4, O.NVFP4


def test_exact_reconstruction_full_rank():
    g = np.random.default_rng(3)
    K, N, M = 24, 16, 10
    x = g.standard_normal((M, K))
    x[:, 3] *= 20
    w = g.standard_normal((K, N)) * 0.02
    lam = P.calibrate_lambda(x, w)
    w_hat = lam.astype(np.float64)[:, None] * w
    L1, L2, S = P.svd_factors(w_hat, min(K, N))
    R = w_hat - L1 @ L2
    assert np.abs(R).max() < 1e-13
    y = O.exact_forward(x, lam, L1, L2, R)
    ref = x @ w
    assert np.abs(y - ref).max() <= 1e-12 * np.abs(ref).max()


def test_smoothing_invariance():
    g = np.random.default_rng(4)
    x = g.standard_normal((7, 32))
    x[:, [1, 9]] *= 20
    w = g.standard_normal((32, 12)) * 0.02
    w[[1, 9], :] *= 8
    lam = P.calibrate_lambda(x, w).astype(np.float64)
    lhs = (x / lam[None, :]) @ (lam[:, None] * w)
    assert np.allclose(lhs, x @ w, rtol=1e-13, atol=1e-15)
    # lambda balances the two maxima: max|X'_k| == max|W_hat_k| when alpha = 0.5
    xs = np.abs(x / lam[None, :]).max(0)
    ws = np.abs(lam[:, None] * w).max(1)
    assert np.allclose(xs, ws, rtol=1e-6)


@pytest.mark.parametrize("r", [1, 4, 8])
def test_eckart_young(r):
    g = np.random.default_rng(5)
    w_hat = g.standard_normal((20, 30))
    L1, L2, S = P.svd_factors(w_hat, r)
    resid = np.linalg.norm(w_hat - L1 @ L2) ** 2
    assert abs(resid - np.sum(S[r:] ** 2)) <= 1e-10 * np.sum(S ** 2)
    # L1 L2 is the product the method fixes; the sqrt split balances the norms
    assert np.allclose(np.linalg.norm(L1, axis=0), np.linalg.norm(L2, axis=1))


def test_prep_residual_absorbs_factor_rounding():
    g = np.random.default_rng(6)
    K, N = 128, 64
    x_bits = F.bf16_bits(g.standard_normal((16, K)))
    w = F.bf16_round(g.standard_normal((K, N)) * 0.02)
    pw = P.prepare(x_bits, w, r=8, variant=INT4)
    recon = F.bf16_from_bits(pw.L1) @ F.bf16_from_bits(pw.L2) + pw.R
    assert np.allclose(recon, pw.w_hat, rtol=0, atol=1e-15)


@pytest.mark.parametrize("variant", [INT4, NVFP4])
def test_lowrank_branch_alone(variant):
    g = np.random.default_rng(7)
    G = O.GROUP[variant]
    K, N, r = 2 * G, 48, 6
    x_bits = F.bf16_bits(np.eye(K))               # X = I_K, exact in bf16
    inv_lam = np.ones(K, dtype=np.float32)        # lambda = 1
    L1 = F.bf16_bits(g.standard_normal((K, r)))
    L2 = F.bf16_bits(g.standard_normal((r, N)))
    codes, scales, T = O.quantize_act_lowrank_down(x_bits, inv_lam, L1, variant)
    assert np.array_equal(T, F.bf16_from_bits(L1).astype(np.float32))
    w_codes = np.zeros((N, K // 2), dtype=np.uint8)          # residual codes all zero
    w_scales = (F.bf16_bits(np.ones((N, K // G))) if variant == INT4
                else F.e4m3_encode(np.ones((N, K // G))))
    y, Y = O.gemm_lowrank_up(codes, scales, T, w_codes, w_scales, L2, variant)
    ref = F.bf16_from_bits(L1) @ F.bf16_from_bits(L2)
    assert np.abs(y - ref).max() <= 1e-12 * np.abs(ref).max()


@pytest.mark.parametrize("variant", [INT4, NVFP4])
def test_quantizer_grid_roundtrip(variant):
    g = np.random.default_rng(8)
    G = O.GROUP[variant]
    rows, ng = 64, 4
    if variant == INT4:
        q = g.integers(-7, 8, (rows, ng, G)).astype(np.float64)
        q[:, :, 0] = 7 * np.where(g.random((rows, ng)) < 0.5, 1, -1)     # amax = 7 s
        s = np.ldexp(g.integers(8, 16, (rows, ng)), g.integers(-8, 2, (rows, ng)))
    else:
        q = F.e2m1_decode(g.integers(0, 16, (rows, ng, G)).astype(np.uint8))
        q[:, :, 0] = 6 * np.where(g.random((rows, ng)) < 0.5, 1, -1)     # amax = 6 s
        s = np.ldexp(g.integers(8, 16, (rows, ng)), g.integers(-9, -2, (rows, ng)))   # E4M3 normals
    xv = (q * s[:, :, None]).reshape(rows, ng * G)
    assert np.array_equal(F.bf16_round(xv), xv)                      # on the bf16 grid
    nib, sc = O.quantize_groups(xv.astype(np.float32), variant)
    if variant == INT4:
        assert np.array_equal(F.bf16_from_bits(sc), s)
        assert np.array_equal(F.int4_decode(nib), q.reshape(rows, -1))
    else:
        assert np.array_equal(F.e4m3_decode(sc), s)
        got = F.e2m1_decode(nib)
        assert np.array_equal(np.abs(got), np.abs(q.reshape(rows, -1)))
    # the weight-side quantiser (fp64) obeys the same rule
    nib_w, sc_w = P.quantize_weight_groups(xv, variant)
    assert np.array_equal(nib_w, nib) and np.array_equal(sc_w, sc)


@pytest.mark.parametrize("variant", [INT4, NVFP4])
def test_quantizer_error_bound(variant):
    g = np.random.default_rng(9)
    G = O.GROUP[variant]
    x = g.standard_normal((128, 8 * G)) * np.exp(g.normal(0, 2, (128, 1)))
    xv = F.bf16_round(x).astype(np.float32)
    nib, sc = O.quantize_groups(xv, variant)
    deq = O.dequantize(nib, sc, variant)
    if variant == INT4:
        s = np.repeat(F.bf16_from_bits(sc), G, axis=1)
        assert np.all(np.abs(xv - deq) <= s / 2 * (1 + 1e-12))
    else:
        s = np.repeat(F.e4m3_decode(sc), G, axis=1)
        # the bound holds while the group scale is an E4M3 normal (>= 2^-6);
        # below that the scale loses precision and large values saturate at 6
        ok = s >= 2.0 ** -6
        assert ok.mean() > 0.5
        v = np.abs(xv) / s
        half = np.where(v < 2, 0.25, np.where(v < 4, 0.5, 1.0))      # half the local spacing
        err = np.abs(np.abs(xv) - np.abs(deq))
        assert np.all(err[ok] <= (s * half)[ok] * (1 + 1e-12))
        sub = (~ok) & (s > 0) & (v > 6.5)
        assert np.all(np.abs(deq[sub]) == 6 * s[sub])


# ------------------------------------------------------------------ brute force
def _rne(fr: Fraction, p: int, emin: int, maxf: Fraction, sat: bool) -> Fraction:
    """Exact round-half-even of a rational to a p-bit binary format."""
    if fr == 0:
        return Fraction(0)
    sign = -1 if fr < 0 else 1
    a = abs(fr)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    e = max(e, emin)                       # leading-bit exponent, clamped for subnormals
    ulp = Fraction(2) ** (e - p + 1)
    k = a / ulp
    n = math.floor(k)
    rem = k - n
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and n % 2 == 1):
        n += 1
    q = n * ulp
    if q > maxf:
        q = maxf if sat else Fraction(10) ** 400
    return sign * q


def _f32(fr):   return _rne(fr, 24, -126, Fraction(2) ** 128, False)
def _bf16(fr):  return _rne(fr, 8, -126, Fraction(2) ** 128, False)
def _e4m3(fr):  return _rne(fr, 4, -6, Fraction(448), True)
def _e2m1(fr):  return _rne(fr, 2, 0, Fraction(6), True)


def _brute_layer(x, inv_lam, L1, L2, wq, ws, variant, gelu, bias=None):
    """Pure-python exact restatement: lists of Fractions, explicit loops.
    The bias (if any) is added to the accumulator before GELU."""
    G = O.GROUP[variant]
    M, K = len(x), len(x[0])
    N, r = len(wq), len(L2)
    xp = [[_bf16(_f32(x[m][k] * inv_lam[k])) for k in range(K)] for m in range(M)]
    qx, sx = [], []
    for m in range(M):
        qrow, srow = [], []
        for g0 in range(0, K, G):
            a = max(abs(v) for v in xp[m][g0:g0 + G])
            s = _bf16(_f32(a / 7)) if variant == INT4 else _e4m3(_f32(a / 6))
            srow.append(s)
            for k in range(g0, g0 + G):
                if s == 0:
                    qrow.append(Fraction(0))
                elif variant == INT4:
                    v = _f32(xp[m][k] / s)
                    n = math.floor(v)
                    rem = v - n
                    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and n % 2):
                        n += 1
                    qrow.append(Fraction(max(-8, min(7, n))))
                else:
                    qrow.append(_e2m1(_f32(xp[m][k] / s)))
        qx.append(qrow)
        sx.append(srow)
    T = [[_f32(sum(xp[m][k] * L1[k][j] for k in range(K))) for j in range(r)] for m in range(M)]
    y = []
    for m in range(M):
        row = []
        for n in range(N):
            acc = Fraction(0)
            for gi, g0 in enumerate(range(0, K, G)):
                acc += sx[m][gi] * ws[n][gi] * sum(qx[m][k] * wq[n][k] for k in range(g0, g0 + G))
            acc += sum(T[m][j] * L2[j][n] for j in range(r))
            if bias is not None:
                acc += bias[n]
            a = float(acc)
            if gelu:
                a = 0.5 * a * (1 + math.tanh(math.sqrt(2 / math.pi) * (a + 0.044715 * a ** 3)))
            row.append(a)
        y.append(row)
    return qx, sx, T, y


@pytest.mark.parametrize("variant,scale_exp", [(INT4, 0), (NVFP4, 0), (NVFP4, -7)])
@pytest.mark.parametrize("gelu,with_bias", [(False, False), (True, False), (False, True),
                                            (True, True)])
def test_brute_force_8x8(variant, scale_exp, gelu, with_bias):
    """scale_exp: the NVFP4 weights' per-tensor scale 2^e (weights q s 2^e)."""
    g = np.random.default_rng(10 + variant + 2 * gelu + 4 * with_bias - scale_exp)
    G = O.GROUP[variant]
    M = N = 8
    K, r = G, 3
    x = g.standard_normal((M, K))
    x[:, 2] *= 20
    x[1, :] = 0.0                       # an all-zero group: scale 0, codes +0
    x[2, :] *= 1e-3                     # small values, negative ones round to -0 in E2M1
    x_bits = F.bf16_bits(x)
    lam = np.exp(g.normal(0, 1, K)).astype(np.float32)
    inv_lam = (np.float32(1) / lam).astype(np.float32)
    L1b = F.bf16_bits(g.standard_normal((K, r)) * 0.3)
    L2b = F.bf16_bits(g.standard_normal((r, N)) * 0.3)
    if variant == INT4:
        wq_nib = F.int4_encode(g.integers(-7, 8, (N, K)))
        ws = F.bf16_bits(np.exp(g.normal(-3, 0.5, (N, K // G))))
        wsv = F.bf16_from_bits(ws)
        wqv = F.int4_decode(wq_nib)
    else:
        wq_nib = g.integers(0, 16, (N, K)).astype(np.uint8)
        ws = F.e4m3_encode(np.exp(g.normal(-3, 0.5, (N, K // G))))
        wsv = F.e4m3_decode(ws)
        wqv = F.e2m1_decode(wq_nib)
    # a bias large enough to move GELU's operating point (bf16 values)
    bias_bits = F.bf16_bits(g.standard_normal(N) * 2.0) if with_bias else None
    codes, scales, T = O.quantize_act_lowrank_down(x_bits, inv_lam, L1b, variant)
    y, Y = O.gemm_lowrank_up(codes, scales, T, F.pack_nibbles(wq_nib), ws, L2b, variant,
                             bias_bits=bias_bits, gelu=gelu, w_scale_exp=scale_exp)
    wsv = wsv * 2.0 ** scale_exp

    fr = lambda a: [[Fraction(float(v)) for v in row] for row in a]
    qx, sx, Tb, yb = _brute_layer(
        fr(F.bf16_from_bits(x_bits)), [Fraction(float(v)) for v in inv_lam],
        fr(F.bf16_from_bits(L1b)), fr(F.bf16_from_bits(L2b)), fr(wqv), fr(wsv), variant, gelu,
        None if bias_bits is None else [Fraction(float(v)) for v in F.bf16_from_bits(bias_bits)])

    nib = F.unpack_nibbles(codes)
    dq = F.int4_decode(nib) if variant == INT4 else F.e2m1_decode(nib)
    assert np.array_equal(dq, np.array([[float(v) for v in row] for row in qx]))
    sv = F.bf16_from_bits(scales) if variant == INT4 else F.e4m3_decode(scales)
    assert np.array_equal(sv, np.array([[float(v) for v in row] for row in sx]))
    assert np.array_equal(T.astype(np.float64), np.array([[float(v) for v in row] for row in Tb]))
    yb = np.array(yb)
    assert np.abs(y - yb).max() <= 1e-12 * max(1.0, np.abs(yb).max())
    Yb = np.array([[float(_bf16(Fraction(v))) for v in row] for row in yb])
    assert np.array_equal(F.bf16_from_bits(Y), Yb)
    if variant == NVFP4:
        # the all-zero row has scale 0 and +0 codes
        assert np.all(nib[1] == 0) and np.all(sv[1] == 0)


# ------------------------------------------------------------ GELU (tanh form)
def test_gelu_tanh_against_torch_and_identities():
    """The oracle's GELU against an independent implementation (torch's
    tanh-approximate GELU, fp64 on the CPU) over a dense grid and at large
    magnitudes, and against what the formula fixes: GELU(0) = 0, the odd-part
    identity GELU(x) - GELU(-x) = x (tanh is odd), GELU(x) -> x for large x
    and -> -0 for very negative x."""
    import torch
    xs = np.concatenate([np.linspace(-12.0, 12.0, 48001),
                         [-1e300, -1e150, -1e30, -1e6, -60.0, -30.0, 30.0, 60.0, 1e6, 1e30,
                          1e150, 1e300]])
    ref = torch.nn.functional.gelu(torch.from_numpy(xs), approximate="tanh").numpy()
    got = O.gelu_tanh(xs)
    fin = np.abs(xs) < 1e100
    # 1 + tanh(u) cancels for negative x in both implementations: compare in
    # absolute terms, a few fp64 ulps of max(1, |x|)
    assert np.all(np.abs(got[fin] - ref[fin]) <= 4e-15 * np.maximum(1.0, np.abs(xs[fin])))
    assert np.all(got[xs >= 30] == xs[xs >= 30])           # tanh(u) == 1 in fp64
    assert np.all(got[xs <= -30] == 0.0)
    g = np.linspace(-6.0, 6.0, 1201)
    assert O.gelu_tanh(0.0) == 0.0
    assert np.allclose(O.gelu_tanh(g) - O.gelu_tanh(-g), g, rtol=0, atol=1e-15)
    # the slope at 0 is 1/2 (d/dx of 0.5 x (1 + tanh(c x + ...)) at 0)
    h = 1e-7
    assert abs((O.gelu_tanh(h) - O.gelu_tanh(-h)) / (2 * h) - 0.5) < 1e-8


# ------------------------------------------------- smoothing factor edge rules
def test_lambda_edge_rules():
    """lambda = 1 where either calibration maximum is zero; lambda clamped to
    [2^-20, 2^20]; otherwise max|X_k|^0.5 / max|W_k|^0.5 (alpha = 0.5)."""
    x = np.ones((4, 6))
    w = np.ones((6, 3))
    x[:, 0] = 0.0                      # all-zero activation channel
    w[1, :] = 0.0                      # all-zero weight row
    x[:, 2] = 2.0 ** 50                # would give 2^25 / 2^-25 = 2^50: clamped
    w[2, :] = 2.0 ** -50
    x[:, 3] = 2.0 ** -50               # 2^-50: clamped at the bottom
    w[3, :] = 2.0 ** 50
    x[:, 4] = 16.0                     # plain case: sqrt(16) / sqrt(4) = 2
    w[4, :] = -4.0
    lam = P.calibrate_lambda(x, w)
    assert lam.dtype == np.float32
    assert lam[0] == 1.0 and lam[1] == 1.0
    assert lam[2] == np.float32(2.0 ** 20) and lam[3] == np.float32(2.0 ** -20)
    assert lam[4] == 2.0 and lam[5] == 1.0


# ------------------------------------- the whole weight preparation at full rank
@pytest.mark.parametrize("K,N,variant", [(128, 64, INT4), (64, 128, INT4), (48, 32, NVFP4),
                                         (32, 80, NVFP4)])
def test_prepare_full_rank_reconstructs_xw(K, N, variant):
    """prepare() end to end with r = min(K, N) and K != N: calibration, row
    smoothing, SVD, bf16 factors and the residual over the stored factors.
    With the fp64 residual the exact-arithmetic layer reproduces X W to fp64
    rounding (the residual then holds only the factor rounding), the residual
    codes are grouped along K per output feature, and the quantised forward
    stays within the bf16 rounding of X'."""
    g = np.random.default_rng(11 + K + N)
    M = 24
    x = g.standard_normal((M, K))
    x[:, 1] *= 20
    w = F.bf16_round(g.standard_normal((K, N)) * 0.02)
    w[1, :] *= 8
    x_bits = F.bf16_bits(x)
    r = min(K, N)
    pw = P.prepare(x_bits, w, r=r, variant=variant)
    xv = F.bf16_from_bits(x_bits)
    L1 = F.bf16_from_bits(pw.L1)
    L2 = F.bf16_from_bits(pw.L2)
    assert L1.shape == (K, r) and L2.shape == (r, N)
    # the factors are full rank, so the residual is only their bf16 rounding
    assert np.linalg.norm(pw.R) <= 2.0 ** -7 * np.linalg.norm(pw.w_hat)
    y = O.exact_forward(xv, pw.lam, L1, L2, pw.R)
    ref = xv @ w
    assert np.abs(y - ref).max() <= 1e-12 * np.abs(ref).max()
    # residual codes: [N, K/2] bytes, groups of G along K for each output n
    G = O.GROUP[variant]
    assert pw.codes.shape == (N, K // 2) and pw.scales.shape == (N, K // G)
    deq = O.dequantize(F.unpack_nibbles(pw.codes), pw.scales, variant)     # [N, K]
    if variant == INT4:
        s = np.repeat(F.bf16_from_bits(pw.scales), G, axis=1)
        assert np.all(np.abs(pw.R.T - deq) <= s / 2 * (1 + 1e-12))
    else:
        # with no per-tensor scale the tiny residual's E4M3 group scales are
        # mostly subnormal or zero: zero scales mean amax / 6 rounded to 0
        # (amax <= 6 * 2^-10); elsewhere codes stay within +-6 s with R's sign,
        # and normal scales bound the error by s (half the widest E2M1 gap)
        s = np.repeat(F.e4m3_decode(pw.scales), G, axis=1)
        Rt = pw.R.T
        assert np.all(np.abs(Rt[s == 0]) <= 6 * 2.0 ** -10)
        assert np.all(np.abs(deq) <= 6 * s)
        assert np.all((deq == 0) | (np.sign(deq) == np.sign(Rt)))
        nrm = s >= 2.0 ** -6
        assert np.all(np.abs(Rt - deq)[nrm] <= s[nrm])
    # quantised forward: the residual is tiny, the rest is X' in bf16 and T in fp32
    out = O.linear_forward(x_bits, pw)
    e = np.linalg.norm(out["y"] - ref) / np.linalg.norm(ref)
    assert e < 1e-2, e


# --------------------------------------- NVFP4 per-tensor second-level scale
def test_tensor_scale_exponent():
    """e is the smallest integer with max|R| / 6 <= 448 * 2^e."""
    assert P.tensor_scale_exponent(np.zeros((4, 4))) == 0
    for e in (-20, -10, -1, 0, 3):
        R = np.full((2, 2), 2688.0 * 2.0 ** e)          # max|R| / 6 = 448 * 2^e exactly
        assert P.tensor_scale_exponent(R) == e
        R[0, 0] = np.nextafter(R[0, 0], np.inf)          # just above: one more
        assert P.tensor_scale_exponent(R) == e + 1
        R = -np.full((3,), 2688.0 * 2.0 ** e * 0.75)     # sign does not matter
        assert P.tensor_scale_exponent(R) == e


def test_tensor_scale_quantisation():
    """With the per-tensor scale a small residual keeps normal E4M3 group
    scales (no zero or subnormal scales where global scale 1 has many), no
    scale saturates, and each group obeys the E2M1 rounding bound; e = 0
    reproduces the plain quantiser bit for bit."""
    g = np.random.default_rng(31)
    N, K = 64, 256
    Rt = g.standard_normal((N, K)) * 3e-3
    Rt[5, 16:32] = 0.0                                   # an all-zero group
    e = P.tensor_scale_exponent(Rt)
    assert e < -5
    nib0, sc0 = P.quantize_weight_groups(Rt, NVFP4)
    nib, sc = P.quantize_weight_groups(Rt, NVFP4, e)
    s0 = F.e4m3_decode(sc0)
    s = F.e4m3_decode(sc)
    assert (s0 < 2.0 ** -6).mean() > 0.9                 # global scale 1: subnormal or zero
    live = np.abs(Rt).reshape(N, K // 16, 16).max(axis=2) > 0
    assert np.all(s[live] >= 2.0 ** -6) and np.all(s <= 448.0)
    assert np.all(s[~live] == 0)
    deq = O.dequantize(nib, sc, NVFP4, e)
    full = np.repeat(s * 2.0 ** e, 16, axis=1)
    v = np.abs(Rt) / np.where(full > 0, full, 1.0)
    half = np.where(v < 2, 0.25, np.where(v < 4, 0.5, 1.0))
    assert np.all(np.abs(np.abs(Rt) - np.abs(deq)) <= full * half * (1 + 1e-12))
    assert np.linalg.norm(Rt - deq) < 0.2 * np.linalg.norm(Rt - O.dequantize(nib0, sc0, NVFP4))
    nib_z, sc_z = P.quantize_weight_groups(Rt, NVFP4, 0)
    assert np.array_equal(nib_z, nib0) and np.array_equal(sc_z, sc0)
