"""Runtime forward of the SVDQuant W4A4 linear layer (the GPU parity target).

Test infrastructure only (see ``oracle/__init__.py``).

    Y = (X diag(lambda)^-1) L1 L2  +  Q4(X diag(lambda)^-1) Q4(R)

[Lite] "The Mechanics of 4-Bit Efficiency and SVDQuant": activation outliers
are moved into the weights, the weights become a 16-bit low-rank branch plus a
4-bit residual, and both weights and activations of the residual branch are
4-bit (W4A4).  [Apatero] "O que e Nunchaku...": the low-rank down projection
consumes the same activations as the quantiser, the up projection is added to
the 4-bit product.

Steps (in the order the layer applies them), with the reading taken where the
pages say nothing:
  s1  X' = bf16_RN( fp32(X) *_RN inv_lambda )            (X' held in bf16)
  s2  a  = max |X'| over each group of G along K           (per token)
  s3  INT4:  s = bf16_RN( fp32(a) /_RN 7 )
      NVFP4: s = E4M3_RN_satfinite( fp32(a) /_RN 6 )
  s4  v = fp32(x') /_RN s;  INT4 q = clamp(rint(v), -8, 7);
      NVFP4 q = E2M1_RN_satfinite(v);  s == 0 gives q = +0
  s5  T = X' L1, summed exactly (fp64), stored fp32
  s6  acc = sum_g s_x s_w sum_{k in g} q_x q_w  +  T L2  (+ bias)   (fp64)
      (an NVFP4 weight with a per-tensor scale 2^e has s_w = E4M3 scale * 2^e)
  s7  y = GELU_tanh(acc) when the layer has GELU;  Y = bf16_RN(y)

Parity: pinned by brute force on 8x8 problems, by the exact-reconstruction
case r = min(K, N), by the low-rank-only identity case and by the quantiser
round-trip / error-bound properties (tests/test_oracle_pins.py).
"""
from __future__ import annotations

import numpy as np

from . import formats as F

INT4, NVFP4 = 0, 1
GROUP = {INT4: 64, NVFP4: 16}


def smooth_activations(x_bits: np.ndarray, inv_lam: np.ndarray) -> np.ndarray:
    """s1: X' = bf16(fp32(X) * inv_lambda), returned as fp32 values."""
    x = F.bf16_from_bits(x_bits).astype(np.float32)
    xs = x * np.asarray(inv_lam, dtype=np.float32)[None, :]      # fp32 multiply, RN
    return F.bf16_round(xs).astype(np.float32)


def quantize_groups(xp: np.ndarray, variant: int):
    """s2-s4 on fp32 values [rows, K]: returns (nibbles [rows,K], scales).

    scales: INT4 -> bf16 bit patterns [rows, K/64]; NVFP4 -> E4M3 bytes
    [rows, K/16].  Division is IEEE fp32 round-to-nearest (numpy float32).
    """
    G = GROUP[variant]
    rows, K = xp.shape
    g = xp.reshape(rows, K // G, G).astype(np.float32)
    a = np.max(np.abs(g), axis=2)                                 # exact
    if variant == INT4:
        s = F.bf16_round(a / np.float32(7.0)).astype(np.float32)  # fp32 div, then bf16 RNE
        s_store = F.bf16_bits(s)
    else:
        s = F.e4m3_round(a / np.float32(6.0)).astype(np.float32)
        s_store = F.e4m3_encode(s)
    nz = s > 0
    v = np.zeros_like(g)
    with np.errstate(divide="ignore", invalid="ignore"):
        v = np.where(nz[:, :, None], g / np.where(nz, s, np.float32(1))[:, :, None], np.float32(0))
    v = v.astype(np.float32)                                      # fp32 quotient, RN
    if variant == INT4:
        nib = F.int4_encode(v)
    else:
        nib = F.e2m1_encode(v)
        nib = np.where(nz[:, :, None], nib, np.uint8(0))          # s == 0 -> +0 codes
    return nib.reshape(rows, K).astype(np.uint8), s_store


def dequantize(nib: np.ndarray, scales: np.ndarray, variant: int, scale_exp: int = 0) -> np.ndarray:
    """nibbles [rows,K] + scales (times 2^scale_exp) -> exact fp64 values q*s."""
    G = GROUP[variant]
    rows, K = nib.shape
    if variant == INT4:
        q = F.int4_decode(nib)
        s = F.bf16_from_bits(scales)
    else:
        q = F.e2m1_decode(nib)
        s = np.ldexp(F.e4m3_decode(scales), scale_exp)
    return (q.reshape(rows, K // G, G) * s[:, :, None]).reshape(rows, K)


def quantize_act_lowrank_down(x_bits, inv_lam, L1_bits, variant):
    """Activation side (steps s1-s5).

    Returns (codes uint8 [M,K/2], scales, T fp32 [M,r]).
    """
    xp = smooth_activations(x_bits, inv_lam)
    nib, scales = quantize_groups(xp, variant)
    L1 = F.bf16_from_bits(L1_bits)
    if L1.shape[1] == 0:
        T = np.zeros((xp.shape[0], 0), dtype=np.float32)
    else:
        T = (xp.astype(np.float64) @ L1).astype(np.float32)      # fp64 sum, fp32 store
    return F.pack_nibbles(nib), scales, T


def gelu_tanh(x):
    """GELU, tanh form: 0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3)))."""
    x = np.asarray(x, dtype=np.float64)
    # x^3 overflows to +-inf for |x| > ~1e102; tanh(+-inf) = +-1 gives the
    # limits x and 0, so the overflow is harmless and not reported
    with np.errstate(over="ignore"):
        return 0.5 * x * (1.0 + np.tanh(np.sqrt(2.0 / np.pi) * (x + 0.044715 * x ** 3)))


def gemm_lowrank_up(codes, scales, T, w_codes, w_scales, L2_bits, variant,
                    bias_bits=None, gelu=False, rows=None, w_scale_exp: int = 0):
    """Weight side (steps s6-s7).

    codes [M,K/2], scales (activation), T fp32 [M,r]; w_codes [N,K/2],
    w_scales [N,K/G], L2 bf16 bits [r,N].  ``rows`` optionally restricts the
    computation to a subset of token rows.  Returns (y fp64 [M,N], Y bf16 bits).
    """
    if rows is not None:
        codes, scales, T = codes[rows], scales[rows], T[rows]
    xa = dequantize(F.unpack_nibbles(codes), scales, variant)
    wq = dequantize(F.unpack_nibbles(w_codes), w_scales, variant, w_scale_exp)
    acc = xa @ wq.T
    L2 = F.bf16_from_bits(L2_bits)
    if L2.shape[0] > 0:
        acc = acc + np.asarray(T, dtype=np.float64) @ L2
    if bias_bits is not None:
        acc = acc + F.bf16_from_bits(bias_bits)[None, :]
    y = gelu_tanh(acc) if gelu else acc
    return y, F.bf16_bits(y)


def linear_forward(x_bits, pw, rows=None):
    """Whole layer for a packed-weight record ``pw`` (fields as in the load
    descriptor: lam, L1, L2, codes, scales, bias, gelu, variant).

    Returns dict with codes, scales, T (all rows) and y, Y (selected rows).
    """
    inv_lam = (np.float32(1.0) / np.asarray(pw.lam, dtype=np.float32)).astype(np.float32)
    if rows is not None:
        x_bits = x_bits[rows]
    codes, scales, T = quantize_act_lowrank_down(x_bits, inv_lam, pw.L1, pw.variant)
    y, Y = gemm_lowrank_up(codes, scales, T, pw.codes, pw.scales, pw.L2, pw.variant,
                           pw.bias, pw.gelu, w_scale_exp=getattr(pw, "w_scale_exp", 0))
    return {"codes": codes, "scales": scales, "T": T, "y": y, "Y": Y}


def exact_forward(x, lam, L1, L2, Rq=None, bias=None, gelu=False):
    """Exact-arithmetic reading of the layer (no bf16 on X', fp64 factors):
    y = (X diag(lambda)^-1) L1 L2 + (X diag(lambda)^-1) R  (+bias, GELU).

    Used by the reconstruction pins; ``Rq`` is an fp64 residual (or None).
    """
    xs = np.asarray(x, dtype=np.float64) / np.asarray(lam, dtype=np.float64)[None, :]
    acc = (xs @ L1) @ L2 if L1.shape[1] else np.zeros((xs.shape[0], L2.shape[1]))
    if Rq is not None:
        acc = acc + xs @ Rq
    if bias is not None:
        acc = acc + bias[None, :]
    return gelu_tanh(acc) if gelu else acc
