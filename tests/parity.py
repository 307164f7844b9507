"""Helpers shared by the GPU parity tests: run the CUDA path through the C ABI
and the CPU oracle on the same seeded inputs, and compare them.

Bars (the layer's stated tolerances):
  * activation codes and scales: bit-exact;
  * T = X' L1: ||dT||_F <= 4 sqrt(K) 2^-24 || |X'| |L1| ||_F, the fp32
    accumulation bound for a K-term dot product (t_bound); small-K cases
    also meet relative Frobenius <= 1e-5;
  * Y: relative Frobenius error <= 1e-3 against the oracle's bf16-rounded Y,
    and, against the unrounded oracle y, max over elements of the error
    beyond the bf16 output rounding, max(|Y - y| - ulp_bf16(y)/2, 0),
    <= 2e-2 * rms(y).  (A bf16 output cannot be closer to y than half an
    ulp; at |y| >= 32 that half ulp alone exceeds 0.02 * rms for typical
    layers, so the bar is read as applying to the error beyond it.)
"""
from __future__ import annotations

import numpy as np

from bit_diffusion_transformer_w4a4_b200 import svdq
from bit_diffusion_transformer_w4a4_b200 import workloads as W
from oracle import formats as F
from oracle import forward as O

T_REL = 1e-5
Y_REL = 1e-3
Y_MAXABS_RMS = 2e-2

# (label, quantity, measured, bar) of every bar checked in this process; the
# terminal summary (tests/conftest.py) prints them with the margin left.
MARGINS: list[tuple[str, str, float, float]] = []


def record(label: str, what: str, value: float, bar: float) -> None:
    MARGINS.append((label, what, float(value), float(bar)))


def torch_mod():
    import torch
    return torch


def to_dev(a: np.ndarray):
    torch = torch_mod()
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def from_dev(t) -> np.ndarray:
    return t.cpu().numpy()


def tile_nvfp4_scales(canon: np.ndarray, M: int, K: int) -> np.ndarray:
    """Canonical [M x K/16] E4M3 -> the library's tiled activation layout."""
    mp = (M + 127) // 128 * 128
    out = np.zeros(mp * (K // 16), dtype=np.uint8)
    m = np.arange(M)[:, None]
    b = np.arange(K // 16)[None, :]
    off = ((m // 128) * (K // 64) + b // 4) * 512 + (m % 32) * 16 + ((m // 32) % 4) * 4 + b % 4
    out[off] = canon
    return out


def gpu_forward(h: svdq.SVDQWeights, x_bits: np.ndarray, M: int, two_calls: bool = True):
    """Run the layer on the GPU.  Returns codes, canonical scales, T, Y bits."""
    torch = torch_mod()
    x = to_dev(x_bits.view(np.int16)).view(torch.bfloat16)
    y = torch.empty((M, h.N), dtype=torch.bfloat16, device="cuda")
    codes, scales, t = h.alloc_act(M)
    if two_calls:
        h.quantize_act_lowrank_down(x, M, codes, scales, t)
        h.w4a4_gemm_lowrank_up(codes, scales, t, M, y)
    else:
        h.linear_forward(x, y, M)
    torch.cuda.synchronize()
    st = h.device_status()
    assert st == 0, svdq.STATUS.get(st)
    Y = from_dev(y.view(torch.int16)).view(np.uint16)
    if not two_calls:          # the fused call keeps its intermediates internal
        return {"Y": Y}
    sc = from_dev(scales)
    if h.variant == W.NVFP4:
        sc = svdq.untile_nvfp4_scales(sc, M, h.K)
    else:
        sc = sc.view(np.uint16).reshape(M, h.K // 64)
    return {"codes": from_dev(codes), "scales": sc, "T": from_dev(t)[:, :h.r], "Y": Y}


def rel_fro(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    den = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / den) if den > 0 else float(np.linalg.norm(a - b))


def t_bound(xp: np.ndarray, L1: np.ndarray) -> float:
    """Frobenius bound for T = X' L1 accumulated in fp32 on the tensor cores:
    4 sqrt(K) 2^-24 || |X'| |L1| ||_F (a random-walk bound on K fp32 roundings,
    each relative to the magnitude of the partial sums)."""
    K = xp.shape[1]
    return 4.0 * np.sqrt(K) * 2.0 ** -24 * float(np.linalg.norm(np.abs(xp) @ np.abs(L1)))


def check_act(got: dict, ref: dict, rows=None, r: int = 0, label: str = "", tb: float | None = None):
    sel = slice(None) if rows is None else rows
    gc, gs = got["codes"][sel], got["scales"][sel]
    bad_c = np.argwhere(gc != ref["codes"])
    bad_s = np.argwhere(gs != ref["scales"])
    assert len(bad_c) == 0, f"{label}: {len(bad_c)} code bytes differ, first {bad_c[:4].tolist()} " \
        f"gpu {gc[tuple(bad_c[0])]:#04x} oracle {ref['codes'][tuple(bad_c[0])]:#04x}"
    assert len(bad_s) == 0, f"{label}: {len(bad_s)} scales differ, first {bad_s[:4].tolist()}"
    if r > 0:
        d = float(np.linalg.norm(got["T"][sel].astype(np.float64) - ref["T"]))
        if tb is None:
            e = rel_fro(got["T"][sel], ref["T"])
            record(label, "T rel Frobenius", e, T_REL)
            assert e <= T_REL, f"{label}: T rel err {e:.3e}"
        else:
            record(label, "||dT|| / fp32 bound", d / tb if tb > 0 else 0.0, 1.0)
            assert d <= tb, f"{label}: ||dT|| {d:.3e} > fp32 accumulation bound {tb:.3e}"


def check_y(Y_gpu_bits: np.ndarray, y_ref: np.ndarray, Y_ref_bits: np.ndarray, label: str = ""):
    yg = F.bf16_from_bits(Y_gpu_bits)
    yr = F.bf16_from_bits(Y_ref_bits)
    y_ref = np.asarray(y_ref, dtype=np.float64)
    assert np.all(np.isfinite(yg)), f"{label}: non-finite output"
    e = rel_fro(yg, yr)
    rms = float(np.sqrt(np.mean(y_ref ** 2)))
    # error beyond the bf16 output rounding itself (half a bf16 ulp of y)
    excess = np.maximum(np.abs(yg - y_ref) - bf16_half_ulp(y_ref), 0.0)
    mx = float(np.max(excess)) if yg.size else 0.0
    record(label, "Y rel Frobenius", e, Y_REL)
    record(label, "Y max excess / rms", mx / rms if rms > 0 else 0.0, Y_MAXABS_RMS)
    assert e <= Y_REL, f"{label}: Y rel Frobenius {e:.3e} > {Y_REL}"
    assert mx <= Y_MAXABS_RMS * rms, f"{label}: max|dY| beyond bf16 rounding {mx:.3e} > " \
        f"{Y_MAXABS_RMS} * rms {rms:.3e}"
    return e, mx / rms if rms > 0 else 0.0


def bf16_half_ulp(y: np.ndarray) -> np.ndarray:
    """Half the bf16 spacing at |y| (the largest error of a correct rounding)."""
    _, ex = np.frexp(np.abs(y))
    return np.ldexp(1.0, np.maximum(ex - 1, -126) - 8)


def oracle_rows(pw, x_bits: np.ndarray, rows: np.ndarray) -> dict:
    return O.linear_forward(x_bits, pw, rows=rows)


def oracle_act_all(pw, x_bits: np.ndarray, chunk: int = 2048) -> dict:
    """The oracle's activation side (codes, canonical scales, T) on every
    token row, computed in row blocks to bound host memory."""
    inv = (np.float32(1) / np.asarray(pw.lam, dtype=np.float32)).astype(np.float32)
    parts = [O.quantize_act_lowrank_down(x_bits[i:i + chunk], inv, pw.L1, pw.variant)
             for i in range(0, x_bits.shape[0], chunk)]
    return {"codes": np.concatenate([p[0] for p in parts]),
            "scales": np.concatenate([p[1] for p in parts]),
            "T": np.concatenate([p[2] for p in parts])}


def oracle_y_all(pw, act: dict, chunk: int = 2048):
    """The oracle's weight side on every row (y fp64, Y bf16 bits), from the
    oracle's own activation codes, scales and T, in row blocks."""
    ys, Ys = [], []
    for i in range(0, act["codes"].shape[0], chunk):
        y, Y = O.gemm_lowrank_up(act["codes"][i:i + chunk], act["scales"][i:i + chunk],
                                 act["T"][i:i + chunk], pw.codes, pw.scales, pw.L2, pw.variant,
                                 pw.bias, pw.gelu)
        ys.append(y)
        Ys.append(Y)
    return np.concatenate(ys), np.concatenate(Ys)


def t_bound_all(pw, x_bits: np.ndarray, chunk: int = 2048) -> float:
    """t_bound over every row, accumulated in row blocks."""
    inv = (np.float32(1) / np.asarray(pw.lam, dtype=np.float32)).astype(np.float32)
    L1 = np.abs(F.bf16_from_bits(pw.L1))
    K = x_bits.shape[1]
    acc = 0.0
    for i in range(0, x_bits.shape[0], chunk):
        xp = np.abs(O.smooth_activations(x_bits[i:i + chunk], inv).astype(np.float64))
        acc += float(np.sum((xp @ L1) ** 2))
    return 4.0 * np.sqrt(K) * 2.0 ** -24 * np.sqrt(acc)
