"""Host-side weight preparation (offline compression) of SVDQuant.

Test infrastructure only (see ``oracle/__init__.py``).  Its outputs are the
pre-packed weights the CUDA library loads, so GPU and oracle always see the
same bytes.

[Lite] "The Mechanics of 4-Bit Efficiency and SVDQuant": activation outliers
are shifted into the weights, then the weight is decomposed into a 16-bit
low-rank branch and a 4-bit residual.  [Apatero] "O que e Nunchaku...": the
low-rank branch comes from a singular value decomposition.  [Lite] "Hardware
Specialization and the Compression Workflow": inspect -> calibrate ->
quantize -> package; INT4 or NVFP4 precision.

  c2  lambda_k = (max_m |X[m,k]|)^alpha / (max_n |W[k,n]|)^(1-alpha), alpha=0.5,
      fp64, stored fp32; lambda_k = 1 if either max is 0; clamp [2^-20, 2^20]
  c3  W_hat = diag(lambda) W  (fp64, with the stored fp32 lambda)
  c4  W_hat = U S V^T;  L1 = U_r S_r^(1/2),  L2 = S_r^(1/2) V_r^T  -> bf16 RN
  c5  R = W_hat - bf16(L1) bf16(L2)   (fp64; the residual absorbs factor rounding)
  c6  per output column n, groups of G along K: s = amax/7 -> bf16 (INT4) or
      amax/6 -> E4M3 (NVFP4), codes = round(R/s) in fp64 (same rule as the
      runtime activation quantiser, in fp64)
  c7  NVFP4 with a per-tensor second-level scale (optional): a power of two
      2^e with e the smallest integer such that max|R| / 6 <= 448 * 2^e (e = 0
      when R = 0); group scales s = E4M3_RN_satfinite((amax / 6) * 2^-e), codes
      = E2M1_RN_satfinite(R / (s 2^e)); a weight dequantises to q s 2^e.
      Reading: the pages name NVFP4 but not its second level; the format's own
      tensor scale is an fp32 value, taken here as a power of two so that the
      scaling stays exact through the low-rank branch (the GEMM scales its
      accumulator by 2^e and the low-rank operand T by 2^-e).

Parity: smoothing invariance, the Eckart-Young residual norm and exact
reconstruction at r = min(K, N) are pinned in tests/test_oracle_pins.py.
"""
from __future__ import annotations

import numpy as np

from . import formats as F
from .forward import GROUP, INT4, NVFP4


def calibrate_lambda(x: np.ndarray, w: np.ndarray, alpha: float = 0.5) -> np.ndarray:
    """c2: per-input-channel smoothing factors (fp32)."""
    ax = np.max(np.abs(np.asarray(x, dtype=np.float64)), axis=0)
    aw = np.max(np.abs(np.asarray(w, dtype=np.float64)), axis=1)
    lam = np.ones_like(ax)
    ok = (ax > 0) & (aw > 0)
    lam[ok] = ax[ok] ** alpha / aw[ok] ** (1.0 - alpha)
    lam = np.clip(lam, 2.0 ** -20, 2.0 ** 20)
    return lam.astype(np.float32)


def svd_factors(w_hat: np.ndarray, r: int):
    """c4: rank-r factors with the singular values split evenly (fp64).

    Returns (L1 [K,r], L2 [r,N], singular values)."""
    U, S, Vt = np.linalg.svd(w_hat, full_matrices=False)
    rs = np.sqrt(S[:r])
    return U[:, :r] * rs[None, :], rs[:, None] * Vt[:r, :], S


def tensor_scale_exponent(R: np.ndarray) -> int:
    """c7: the smallest integer e with max|R| / 6 <= 448 * 2^e (0 for R = 0)."""
    amax = float(np.max(np.abs(R))) if R.size else 0.0
    if amax == 0.0:
        return 0
    t = amax / 6.0 / 448.0
    m, x = np.frexp(t)                       # t = m 2^x, 0.5 <= m < 1
    return int(x - 1) if m == 0.5 else int(x)


def quantize_weight_groups(Rt: np.ndarray, variant: int, scale_exp: int = 0):
    """c6 (and c7 when scale_exp != 0) on R^T [N,K] (fp64): returns
    (nibbles [N,K], scales)."""
    G = GROUP[variant]
    N, K = Rt.shape
    g = Rt.reshape(N, K // G, G)
    a = np.max(np.abs(g), axis=2)
    if variant == INT4:
        assert scale_exp == 0, "the per-tensor scale is an NVFP4 option"
        s = F.bf16_round(a / 7.0)
        s_store = F.bf16_bits(s)
    else:
        s = F.e4m3_round(np.ldexp(a / 6.0, -scale_exp))
        s_store = F.e4m3_encode(s)
        s = np.ldexp(s, scale_exp)               # the group's full scale s 2^e
    nz = s > 0
    with np.errstate(divide="ignore", invalid="ignore"):
        v = np.where(nz[:, :, None], g / np.where(nz, s, 1.0)[:, :, None], 0.0)
    nib = F.int4_encode(v) if variant == INT4 else F.e2m1_encode(v)
    nib = np.where(nz[:, :, None], nib, np.uint8(0))
    return nib.reshape(N, K).astype(np.uint8), s_store


class Prepared:
    """Pre-packed weights (same fields as the library's load descriptor)."""

    def __init__(self, **kw):
        self.__dict__.update(kw)


def prepare(x_bits: np.ndarray, w: np.ndarray, r: int, variant: int,
            alpha: float = 0.5, bias_bits=None, gelu: bool = False,
            tensor_scale: bool = False) -> Prepared:
    """c2-c6 (c7 with ``tensor_scale``, NVFP4 only) for weight W [K,N] (fp64
    values) calibrated on X (bf16 bits)."""
    x = F.bf16_from_bits(x_bits)
    w = np.asarray(w, dtype=np.float64)
    K, N = w.shape
    lam = calibrate_lambda(x, w, alpha)
    w_hat = lam.astype(np.float64)[:, None] * w
    if r > 0:
        L1, L2, S = svd_factors(w_hat, r)
        L1b, L2b = F.bf16_bits(L1), F.bf16_bits(L2)
        R = w_hat - F.bf16_from_bits(L1b) @ F.bf16_from_bits(L2b)
    else:
        S = None
        L1b = np.zeros((K, 0), dtype=np.uint16)
        L2b = np.zeros((0, N), dtype=np.uint16)
        R = w_hat
    e = tensor_scale_exponent(R) if tensor_scale else 0
    nib, scales = quantize_weight_groups(R.T.copy(), variant, e)
    return Prepared(variant=variant, K=K, N=N, r=r, lam=lam, L1=L1b, L2=L2b,
                    codes=F.pack_nibbles(nib), scales=scales, bias=bias_bits,
                    gelu=gelu, R=R, S=S, w_hat=w_hat, w_scale_exp=e)
