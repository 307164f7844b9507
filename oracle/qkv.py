"""QKV projection epilogue: per-head RMS normalisation of Q and K and rotary
position embedding, applied to the output of the SVDQuant W4A4 layer.

Test infrastructure only (see ``oracle/__init__.py``).

"Nunchaku Lite: the 50% VRAM reduction now integrated into Diffusers"
(axbrief.com), section "The Trade-off Between Fused Kernels and
Generality": the original engine's fused path bundles the QKV projection,
Q/K normalisation and rotary embeddings into one kernel, with the Q, K and V
projections merged into one ``to_qkv`` module.

The pages name the operations and nothing of their arithmetic.  Readings
taken here (the conventions of the FLUX-class DiT the pages target):

  q1  the merged projection's N = 3 H D output columns are [Q | K | V], head h
      of Q being columns h D .. h D + D - 1 (likewise K, V), D = 128;
  q2  RMS normalisation of each head of Q and of K over its D features:
        v <- v / sqrt(mean(v^2) + eps) * g,   eps = 1e-6,
      with learned per-feature weights g_q, g_k (bf16 [D]); V is unchanged;
  q3  rotary embedding of the normalised Q and K heads on interleaved pairs
      (2i, 2i+1), i < D/2, by the angle of token m and pair i, given as a
      table of cos and sin [M, D/2] (positions and frequencies are the
      caller's: FLUX derives them from three position axes):
        (a, b) <- (a cos - b sin, a sin + b cos);
  q4  the epilogue works on the layer's accumulator (after the per-tensor
      scale and bias; no GELU), in fp64 here, and rounds once to bf16.

Parity: pinned by the invariants of each step (unit RMS of the normalised
head up to g, pair norms kept by the rotation, the identity and the quarter
turn as special cases, V untouched) and an explicit-loop restatement on
small inputs (tests/test_oracle_qkv.py).
"""
from __future__ import annotations

import numpy as np

from . import formats as F

HEAD_DIM = 128
EPS = 1e-6


def rms_norm_heads(v: np.ndarray, g: np.ndarray, eps: float = EPS) -> np.ndarray:
    """q2 on [M, H*D] (fp64): each D-wide head normalised, times g [D]."""
    M, HD = v.shape
    h = v.reshape(M, HD // HEAD_DIM, HEAD_DIM)
    ms = np.mean(h * h, axis=2, keepdims=True)
    return (h / np.sqrt(ms + eps) * np.asarray(g, dtype=np.float64)[None, None, :]).reshape(M, HD)


def rope_heads(v: np.ndarray, cos: np.ndarray, sin: np.ndarray) -> np.ndarray:
    """q3 on [M, H*D]: pairs (2i, 2i+1) of every head rotated by token m's
    angle for pair i (cos, sin [M, D/2])."""
    M, HD = v.shape
    h = v.reshape(M, HD // HEAD_DIM, HEAD_DIM // 2, 2)
    a, b = h[..., 0], h[..., 1]
    c = np.asarray(cos, dtype=np.float64)[:, None, :]
    s = np.asarray(sin, dtype=np.float64)[:, None, :]
    out = np.stack([a * c - b * s, a * s + b * c], axis=-1)
    return out.reshape(M, HD)


def qkv_epilogue(acc: np.ndarray, gq_bits, gk_bits, cos, sin, eps: float = EPS):
    """q1-q4: acc [M, 3 H D] (fp64, the layer's pre-rounding output) ->
    (y fp64, Y bf16 bits)."""
    M, N = acc.shape
    HD = N // 3
    gq = F.bf16_from_bits(gq_bits)
    gk = F.bf16_from_bits(gk_bits)
    q = rope_heads(rms_norm_heads(acc[:, :HD], gq, eps), cos, sin)
    k = rope_heads(rms_norm_heads(acc[:, HD:2 * HD], gk, eps), cos, sin)
    y = np.concatenate([q, k, acc[:, 2 * HD:]], axis=1)
    return y, F.bf16_bits(y)
