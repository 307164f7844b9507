"""Helpers shared by the GPU parity tests: run the CUDA path through the C ABI
and the CPU oracle on the same seeded inputs, and compare them.

Bars (the layer's stated tolerances):
  * activation codes and scales: bit-exact;
  * T = X' L1: relative Frobenius error <= 1e-5;
  * Y: relative Frobenius error <= 1e-3 against the oracle's bf16-rounded Y,
    and max |Y - y| <= 2e-2 * rms(y) against the unrounded oracle y.
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
    sc = from_dev(scales)
    if h.variant == W.NVFP4:
        sc = svdq.untile_nvfp4_scales(sc, M, h.K)
    else:
        sc = sc.view(np.uint16).reshape(M, h.K // 64)
    return {"codes": from_dev(codes), "scales": sc, "T": from_dev(t)[:, :h.r],
            "Y": from_dev(y.view(torch.int16)).view(np.uint16)}


def rel_fro(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    den = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / den) if den > 0 else float(np.linalg.norm(a - b))


def check_act(got: dict, ref: dict, rows=None, r: int = 0, label: str = ""):
    sel = slice(None) if rows is None else rows
    gc, gs = got["codes"][sel], got["scales"][sel]
    bad_c = np.argwhere(gc != ref["codes"])
    bad_s = np.argwhere(gs != ref["scales"])
    assert len(bad_c) == 0, f"{label}: {len(bad_c)} code bytes differ, first {bad_c[:4].tolist()} " \
        f"gpu {gc[tuple(bad_c[0])]:#04x} oracle {ref['codes'][tuple(bad_c[0])]:#04x}"
    assert len(bad_s) == 0, f"{label}: {len(bad_s)} scales differ, first {bad_s[:4].tolist()}"
    if r > 0:
        e = rel_fro(got["T"][sel], ref["T"])
        assert e <= T_REL, f"{label}: T rel err {e:.3e}"


def check_y(Y_gpu_bits: np.ndarray, y_ref: np.ndarray, Y_ref_bits: np.ndarray, label: str = ""):
    yg = F.bf16_from_bits(Y_gpu_bits)
    yr = F.bf16_from_bits(Y_ref_bits)
    assert np.all(np.isfinite(yg)), f"{label}: non-finite output"
    e = rel_fro(yg, yr)
    rms = float(np.sqrt(np.mean(np.asarray(y_ref, dtype=np.float64) ** 2)))
    mx = float(np.max(np.abs(yg - y_ref))) if yg.size else 0.0
    assert e <= Y_REL, f"{label}: Y rel Frobenius {e:.3e} > {Y_REL}"
    assert mx <= Y_MAXABS_RMS * rms, f"{label}: max|dY| {mx:.3e} > {Y_MAXABS_RMS} * rms {rms:.3e}"
    return e, mx / rms if rms > 0 else 0.0


def oracle_rows(pw, x_bits: np.ndarray, rows: np.ndarray) -> dict:
    return O.linear_forward(x_bits, pw, rows=rows)
