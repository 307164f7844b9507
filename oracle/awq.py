"""AWQ W4A16 linear layer: 4-bit weights, 16-bit activations.

Test infrastructure only (see ``oracle/__init__.py``).

"Nunchaku Lite: the 50% VRAM reduction now integrated into Diffusers"
(axbrief.com), section "The Mechanics of 4-Bit Efficiency and SVDQuant":
besides SVDQW4A4Linear, the runtime patching installs ``AWQW4A16Linear``
layers with 4-bit weights and 16-bit activations; section "The Trade-off
Between Fused Kernels and Generality": the generic scanner gives repeated
transformer blocks SVDQ W4A4 and modulation linear layers AWQ W4A16.

The pages name the layer and nothing of its arithmetic.  Readings taken here
(the plainest ones consistent with "activation-aware weight quantisation,
4-bit weights, 16-bit activations"):

  a1  activation-aware channel factors a_k = (mean_m |X[m,k]|)^alpha,
      alpha = 0.5, fp64, stored fp32; a_k = 1 if the mean is 0; clamped to
      [2^-20, 2^20].  The weight rows are scaled W_hat = diag(a) W and the
      runtime divides the activations by a (multiplies by fp32(1/a)).
  a2  groups of G = 64 along K per output feature n (the INT4 group of the
      W4A4 layer); asymmetric unsigned 4-bit codes with an integer zero
      point.  With lo = min(0, min_g w) and hi = max(0, max_g w) (the range
      always holds 0, so 0 is exact and a constant group has a scale):
        s = bf16_RN((hi - lo) / 15)     (fp64 division, then bf16)
        z = clamp(RNE(-lo / s), 0, 15)  (an integer)
        q = clamp(RNE(w / s) + z, 0, 15)
      s == 0 (an all-zero group) gives z = 0, q = 0.  Dequantised weight
      w = (q - z) s, exact in fp64.
  a3  runtime: x' = fp32(x) *_RN fp32(1/a_k) (kept in fp32: the activations
      stay 16-bit, no activation quantisation);
        y[m,n] = sum_g s[n,g] sum_{k in g} x'[m,k] (q[n,k] - z[n,g]) (+ bias)
      summed exactly (fp64); Y = bf16_RN(y).

Parity: pinned by an exact-rational brute force on small problems, the
on-grid round trip and error bound of the quantiser, the scaling
invariance of a1, and the special case s = 1, z = 8, a = 1 that reduces the
layer to an integer matrix product (tests/test_oracle_awq.py).
"""
from __future__ import annotations

import numpy as np

from . import formats as F

G_AWQ = 64


def channel_factors(x, alpha: float = 0.5) -> np.ndarray:
    """a1: activation-aware per-input-channel factors (fp32)."""
    m = np.mean(np.abs(np.asarray(x, dtype=np.float64)), axis=0)
    a = np.ones_like(m)
    ok = m > 0
    a[ok] = m[ok] ** alpha
    return np.clip(a, 2.0 ** -20, 2.0 ** 20).astype(np.float32)


def quantize_groups(wt: np.ndarray):
    """a2 on W_hat^T [N, K] (fp64): returns (codes [N, K] uint8 0..15,
    scales bf16 bits [N, K/G], zeros uint8 [N, K/G])."""
    N, K = wt.shape
    g = np.asarray(wt, dtype=np.float64).reshape(N, K // G_AWQ, G_AWQ)
    lo = np.minimum(g.min(axis=2), 0.0)
    hi = np.maximum(g.max(axis=2), 0.0)
    s = F.bf16_round((hi - lo) / 15.0)
    nz = s > 0
    sd = np.where(nz, s, 1.0)
    z = np.where(nz, np.clip(np.rint(-lo / sd), 0, 15), 0.0)
    q = np.clip(np.rint(g / sd[:, :, None]) + z[:, :, None], 0, 15)
    q = np.where(nz[:, :, None], q, 0.0)
    return (q.reshape(N, K).astype(np.uint8), F.bf16_bits(s), z.astype(np.uint8))


def dequantize(codes: np.ndarray, scales_bits: np.ndarray, zeros: np.ndarray) -> np.ndarray:
    """codes [N, K] + bf16 scales + integer zeros -> exact fp64 weights [N, K]."""
    N, K = codes.shape
    s = F.bf16_from_bits(scales_bits)
    q = codes.astype(np.float64).reshape(N, K // G_AWQ, G_AWQ)
    return ((q - zeros.astype(np.float64)[:, :, None]) * s[:, :, None]).reshape(N, K)


class PreparedAWQ:
    """Pre-packed AWQ W4A16 weights (the library's load format).
    a       fp32 [K]        channel factors (the runtime multiplies by 1/a)
    codes   u8 [N, K/2]     4-bit codes 0..15, element 2j in the low nibble
    scales  bf16 bits [N, K/64]
    zeros   u8 [N, K/64]    integer zero points 0..15
    bias    bf16 bits [N] or None
    """

    def __init__(self, **kw):
        self.__dict__.update(kw)


def prepare(x_bits: np.ndarray, w: np.ndarray, alpha: float = 0.5, bias_bits=None) -> PreparedAWQ:
    """a1-a2 for W [K, N] calibrated on X (bf16 bits)."""
    x = F.bf16_from_bits(x_bits)
    w = np.asarray(w, dtype=np.float64)
    K, N = w.shape
    a = channel_factors(x, alpha)
    w_hat = a.astype(np.float64)[:, None] * w
    q, s, z = quantize_groups(w_hat.T.copy())
    return PreparedAWQ(K=K, N=N, a=a, codes=F.pack_nibbles(q), scales=s, zeros=z,
                       bias=bias_bits, w_hat=w_hat)


def forward(x_bits: np.ndarray, p, rows=None):
    """a3: returns (y fp64 [M, N], Y bf16 bits)."""
    if rows is not None:
        x_bits = x_bits[rows]
    inv = (np.float32(1.0) / np.asarray(p.a, dtype=np.float32)).astype(np.float32)
    xp = (F.bf16_from_bits(x_bits).astype(np.float32) * inv[None, :]).astype(np.float32)
    wq = dequantize(F.unpack_nibbles(p.codes), p.scales, p.zeros)
    y = xp.astype(np.float64) @ wq.T
    if p.bias is not None:
        y = y + F.bf16_from_bits(p.bias)[None, :]
    return y, F.bf16_bits(y)
