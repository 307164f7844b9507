"""Seeded synthetic inputs for the SVDQuant W4A4 linear layer.

This module only draws random numbers and formats them (bf16 bit patterns,
raw 4-bit code nibbles, raw E4M3 scale bytes).  It performs none of the
method's arithmetic: no smoothing, no SVD, no quantisation rule.  Both the
CUDA path (benchmarks) and the CPU oracle (tests) take their inputs from here.

Workload shapes follow the DiT-style layers that the method is used on
(FLUX-class transformer, hidden 3072, 4096 image + 512 text tokens at 1024 px,
16384 + 512 at 2048 px).  Distributions: activations ~N(0,1) with a small set
of outlier channels scaled x20, weights ~N(0, 0.02^2) with the same input rows
scaled x8 -- the "outliers in weights and activations" situation that the
SVDQuant mechanics section of the Nunchaku Lite article describes.

RNG: numpy PCG64, ``default_rng([seed, config_id, tensor_id])``, fp32 draws
rounded to bf16 (round-to-nearest-even, done by torch's cast).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

INT4 = 0   # SVDQ_INT4_G64_BF16
NVFP4 = 1  # SVDQ_NVFP4_G16_E4M3
GROUP = {INT4: 64, NVFP4: 16}
VARIANT_NAME = {INT4: "int4_g64_bf16", NVFP4: "nvfp4_g16_e4m3"}


@dataclass(frozen=True)
class Layer:
    """One linear layer of a workload: x[M,K] @ W[K,N]."""
    name: str
    M: int
    K: int
    N: int
    r: int
    variant: int
    gelu: bool = False
    bias: bool = False
    weight_kind: str = "gauss"      # "gauss" | "lowrank128"
    outlier_frac: float = 0.01      # fraction of input channels that are outliers
    n_outliers: int | None = None   # explicit count (overrides the fraction)
    config_id: int = 0
    layer_id: int = 0

    @property
    def G(self) -> int:
        return GROUP[self.variant]

    def outlier_count(self) -> int:
        if self.n_outliers is not None:
            return self.n_outliers
        return int(math.floor(self.outlier_frac * self.K + 0.5))

    def flops(self) -> int:
        """Algorithmic FLOPs: 4-bit GEMM plus both low-rank projections."""
        return 2 * self.M * self.K * self.N + 2 * self.M * self.r * (self.K + self.N)


def _layers_cfg5(M: int = 16896) -> list[Layer]:
    base = dict(M=M, r=32, variant=NVFP4, config_id=5)
    return [
        Layer("block.qkv", K=3072, N=9216, layer_id=0, **base),
        Layer("block.out", K=3072, N=3072, layer_id=1, **base),
        Layer("block.fc1", K=3072, N=12288, gelu=True, layer_id=2, **base),
        Layer("block.fc2", K=12288, N=3072, layer_id=3, **base),
    ]


def workloads() -> dict[str, list[Layer]]:
    """All named workloads.  Each is a list of layers run back to back."""
    w: dict[str, list[Layer]] = {}
    w["tiny"] = [Layer("tiny", M=64, K=256, N=256, r=16, variant=INT4,
                       n_outliers=4, config_id=1)]
    w["qkv_int4"] = [Layer("qkv", M=4608, K=3072, N=9216, r=32, variant=INT4,
                           config_id=2)]
    w["fc1_nvfp4"] = [Layer("fc1", M=4608, K=3072, N=12288, r=32, variant=NVFP4,
                            gelu=True, config_id=3, layer_id=0)]
    w["fc2_nvfp4"] = [Layer("fc2", M=4608, K=12288, N=3072, r=32, variant=NVFP4,
                            config_id=3, layer_id=1)]
    for v in (NVFP4, INT4):
        for r in (0, 16, 32, 64, 128):
            w[f"sweep_{VARIANT_NAME[v]}_r{r}"] = [
                Layer(f"sweep_r{r}", M=4608, K=3072, N=3072, r=r, variant=v,
                      weight_kind="lowrank128", config_id=4, layer_id=10 * v + r // 16)]
    w["block_2048px"] = _layers_cfg5()
    return w


def _rng(seed: int, config_id: int, tensor_id: int) -> np.random.Generator:
    return np.random.default_rng([seed, config_id, tensor_id])


def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """fp32 array -> bf16 bit patterns (uint16) via torch's RNE cast."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> fp32 values (exact widening)."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def outlier_channels(layer: Layer, seed: int = 0) -> np.ndarray:
    """First n entries of a seeded permutation of the K input channels."""
    perm = _rng(seed, layer.config_id, 1000 + layer.layer_id).permutation(layer.K)
    return np.sort(perm[: layer.outlier_count()])


def activations(layer: Layer, seed: int = 0, M: int | None = None) -> np.ndarray:
    """X [M,K] as bf16 bits: N(0,1), outlier channels x20."""
    M = layer.M if M is None else M
    g = _rng(seed, layer.config_id, 10 * layer.layer_id + 1)
    x = g.standard_normal((M, layer.K), dtype=np.float32)
    x[:, outlier_channels(layer, seed)] *= np.float32(20.0)
    return to_bf16_bits(x)


def weight(layer: Layer, seed: int = 0) -> np.ndarray:
    """W [K,N] as fp32 values already on the bf16 grid."""
    K, N = layer.K, layer.N
    g = _rng(seed, layer.config_id, 10 * layer.layer_id + 2)
    if layer.weight_kind == "gauss":
        w = g.standard_normal((K, N), dtype=np.float32) * np.float32(0.02)
        w[outlier_channels(layer, seed), :] *= np.float32(8.0)
    elif layer.weight_kind == "lowrank128":
        # rank-128 structure with singular values sigma_1 / i (sigma_1 = 48 gives
        # an entry rms near 0.02), plus N(0, 0.01^2) noise
        rk = min(128, K, N)
        u, _ = np.linalg.qr(g.standard_normal((K, rk)))
        v, _ = np.linalg.qr(g.standard_normal((N, rk)))
        sig = 48.0 / np.arange(1, rk + 1)
        w = ((u * sig) @ v.T).astype(np.float32)
        w += g.standard_normal((K, N), dtype=np.float32) * np.float32(0.01)
    else:
        raise ValueError(layer.weight_kind)
    return bf16_bits_to_f32(to_bf16_bits(w))


def bias(layer: Layer, seed: int = 0) -> np.ndarray | None:
    if not layer.bias:
        return None
    g = _rng(seed, layer.config_id, 10 * layer.layer_id + 3)
    return to_bf16_bits(g.standard_normal(layer.N, dtype=np.float32) * np.float32(0.1))


@dataclass
class PackedWeights:
    """Pre-packed weights in the library's load format (host numpy arrays).

    lam     fp32 [K]           smoothing factors lambda
    L1      bf16 bits [K, r]   low-rank down factor
    L2      bf16 bits [r, N]   low-rank up factor
    codes   uint8 [N, K/2]     residual 4-bit codes, even k in the low nibble
    scales  INT4: bf16 bits [N, K/64]; NVFP4: E4M3 bytes [N, K/16]
    bias    bf16 bits [N] or None
    """
    variant: int
    K: int
    N: int
    r: int
    lam: np.ndarray
    L1: np.ndarray
    L2: np.ndarray
    codes: np.ndarray
    scales: np.ndarray
    bias: np.ndarray | None = None
    gelu: bool = False
    meta: dict = field(default_factory=dict)
    w_scale_exp: int = 0        # NVFP4 per-tensor scale 2^e of the residual weights


def synthetic_packed(layer: Layer, seed: int = 0, int4_min: int = -7) -> PackedWeights:
    """Random pre-packed weights with realistic magnitudes, for timing runs.

    Codes are raw nibbles drawn from a discretised bell shape, scales are raw
    bf16 / E4M3 bit patterns drawn from a band of magnitudes, lambda is
    log-normal with the outlier channels larger.  No quantisation or SVD is
    performed -- the bit patterns are sampled directly.  INT4 codes are drawn
    in [int4_min, 7]; -8 is a valid code of the format that the amax/7 rule
    never produces, so it only appears when int4_min = -8.
    """
    K, N, r, G = layer.K, layer.N, layer.r, layer.G
    g = _rng(seed, layer.config_id, 10 * layer.layer_id + 7)
    lam = np.exp(g.normal(np.log(6.0), 0.25, K)).astype(np.float32)
    lam[outlier_channels(layer, seed)] *= np.float32(5.0)
    L1 = to_bf16_bits(g.standard_normal((K, r), dtype=np.float32) * np.float32(0.05))
    L2 = to_bf16_bits(g.standard_normal((r, N), dtype=np.float32) * np.float32(0.05))
    if layer.variant == INT4:
        q = np.clip(np.rint(g.normal(0.0, 2.5, (N, K))), int4_min, 7).astype(np.int8)
        nib = (q.astype(np.int16) & 0xF).astype(np.uint8)
        scales = to_bf16_bits(np.exp(g.normal(np.log(0.02), 0.3, (N, K // G))).astype(np.float32))
    else:
        # sign bit + magnitude index 0..7 with a bell-shaped histogram
        mag = np.minimum(np.abs(g.normal(0.0, 2.5, (N, K))).astype(np.int64), 7).astype(np.uint8)
        sign = (g.random((N, K)) < 0.5).astype(np.uint8) << 3
        nib = mag | sign
        # E4M3 bytes with exponent field 3..5 and a random mantissa: 0.0625..0.47
        scales = ((g.integers(3, 6, (N, K // G)) << 3) | g.integers(0, 8, (N, K // G))).astype(np.uint8)
    codes = (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)
    return PackedWeights(layer.variant, K, N, r, lam, L1, L2, codes, scales,
                         bias(layer, seed), layer.gelu, {"source": "synthetic"})


def qkv_epilogue_inputs(M: int, seed: int = 0):
    """Inputs of the fused QKV epilogue for M tokens: the Q and K norm
    weights (bf16 bits [128], around 1) and the caller's rotary table
    [M, 128] fp32 of (cos, sin) per interleaved pair.  Angles: token m sits
    at (m // 64, m % 64) on a 2-D grid; pair i turns at 10000^(-(i mod 32)/32)
    per unit of the row coordinate (pairs 0-31) or the column (32-63)."""
    g = _rng(seed, 91, 0)
    gq = to_bf16_bits(np.float32(1) + np.float32(0.2) * g.standard_normal(128, dtype=np.float32))
    gk = to_bf16_bits(np.float32(1) + np.float32(0.2) * g.standard_normal(128, dtype=np.float32))
    i = np.arange(64)
    freq = 10000.0 ** (-(i % 32) / 32.0)
    m = np.arange(M)
    pos = np.where(i[None, :] < 32, (m // 64)[:, None], (m % 64)[:, None]).astype(np.float64)
    ang = pos * freq[None, :]
    rope = np.stack([np.cos(ang), np.sin(ang)], axis=-1).reshape(M, 128).astype(np.float32)
    return gq, gk, rope


# ------------------------------------------------------------ AWQ W4A16 layers
@dataclass(frozen=True)
class AWQLayer:
    """A W4A16 modulation linear: x[M,K] @ W[K,N] with M = tokens per call
    (one conditioning vector per image: the batch)."""
    name: str
    M: int
    K: int
    N: int
    bias: bool = True
    config_id: int = 90
    layer_id: int = 0

    def flops(self) -> int:
        return 2 * self.M * self.K * self.N

    def weight_bytes(self) -> int:
        """Bytes of the packed weights: codes, bf16 scales and u8 zeros."""
        return self.N * self.K // 2 + self.N * (self.K // 64) * 3


def awq_workloads() -> dict[str, AWQLayer]:
    """DiT adaLN modulation (hidden 3072 -> 6 x 3072) at batch 1, 2 (CFG) and 4."""
    return {f"awq_mod_m{m}": AWQLayer(f"mod_m{m}", M=m, K=3072, N=18432, layer_id=m) for m in (1, 2, 4)}


def awq_activations(layer: AWQLayer, seed: int = 0) -> np.ndarray:
    """x [M,K] bf16 bits ~N(0,1) (a SiLU'd conditioning embedding's scale)."""
    g = _rng(seed, layer.config_id, 10 * layer.layer_id + 1)
    return to_bf16_bits(g.standard_normal((layer.M, layer.K), dtype=np.float32))


def awq_weight(layer: AWQLayer, seed: int = 0) -> np.ndarray:
    """W [K,N] fp32 on the bf16 grid ~N(0, 0.02^2)."""
    g = _rng(seed, layer.config_id, 10 * layer.layer_id + 2)
    w = g.standard_normal((layer.K, layer.N), dtype=np.float32) * np.float32(0.02)
    return bf16_bits_to_f32(to_bf16_bits(w))


@dataclass
class PackedAWQ:
    """AWQ W4A16 load format (host arrays): a fp32 [K]; codes u8 [N, K/2]
    (element 2j low nibble, 0..15); scales bf16 bits [N, K/64]; zeros u8
    [N, K/64] (0..15); bias bf16 bits [N] or None."""
    K: int
    N: int
    a: np.ndarray
    codes: np.ndarray
    scales: np.ndarray
    zeros: np.ndarray
    bias: np.ndarray | None = None


def synthetic_awq(layer: AWQLayer, seed: int = 0) -> PackedAWQ:
    """Random AWQ-packed weights for timing runs, sampled as raw bit patterns:
    codes 0..15 bell-shaped around the zero point, zero points 6..9, bf16
    scales in a band around 0.005, log-normal channel factors."""
    K, N = layer.K, layer.N
    g = _rng(seed, layer.config_id, 10 * layer.layer_id + 7)
    a = np.exp(g.normal(0.0, 0.3, K)).astype(np.float32)
    zeros = g.integers(6, 10, (N, K // 64)).astype(np.uint8)
    q = np.clip(np.rint(g.normal(0.0, 3.0, (N, K)) + np.repeat(zeros, 64, axis=1)), 0, 15).astype(np.uint8)
    codes = (q[:, 0::2] | (q[:, 1::2] << 4)).astype(np.uint8)
    scales = to_bf16_bits(np.exp(g.normal(np.log(0.005), 0.3, (N, K // 64))).astype(np.float32))
    b = None
    if layer.bias:
        b = to_bf16_bits(_rng(seed, layer.config_id, 10 * layer.layer_id + 3)
                         .standard_normal(N, dtype=np.float32) * np.float32(0.1))
    return PackedAWQ(K, N, a, codes, scales, zeros, b)
