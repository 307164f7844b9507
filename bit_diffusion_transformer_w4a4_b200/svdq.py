"""Python binding of libsvdq (include/svdq.h) -- argument marshalling only.

Every step of the layer runs in the library's CUDA kernels; this module only
converts numpy / torch buffers into pointers, passes the current CUDA stream
and raises on non-OK status codes.  There is no CPU fallback: if the shared
library is missing or the device is not an sm_100 GPU, calls raise.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

INT4 = 0
NVFP4 = 1
EPI_GELU = 1
GEMM_SINGLE_SM = 2
INT4_F16 = 4
EPI_QKV_NORM_ROPE = 8

STATUS = {
    0: "SVDQ_OK", 1: "SVDQ_ERR_INVALID_ARG", 2: "SVDQ_ERR_SHAPE", 3: "SVDQ_ERR_ALIGNMENT",
    4: "SVDQ_ERR_UNSUPPORTED_DEVICE", 5: "SVDQ_ERR_OOM", 6: "SVDQ_ERR_CUDA",
    7: "SVDQ_ERR_DEVICE_TIMEOUT", 8: "SVDQ_ERR_RANGE",
}

EXPORTED = [
    "svdq_weights_load", "svdq_weights_free", "svdq_act_scales_bytes",
    "svdq_quantize_act_lowrank_down", "svdq_w4a4_gemm_lowrank_up", "svdq_linear_forward",
    "svdq_linear_forward_host", "svdq_device_status", "svdq_debug_set_fault",
    "svdq_selftest_division", "svdq_status_string", "svdq_version",
    "svdq_quantize_act_lowrank_down_static",
    "svdq_awq_load", "svdq_awq_free", "svdq_awq_w4a16_forward",
    "svdq_prep_calibrate", "svdq_prep_lowrank", "svdq_prep_residual_quantize",
    "svdq_w4a4_gemm_lowrank_up_qkv", "svdq_linear_forward_qkv",
    "svdq_w4a4_gemm_lowrank_up_chain", "svdq_linear_forward_chain", "svdq_device_error_site",
    "svdq_set_deterministic",
]


class SvdqError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {STATUS.get(code, code)}")


class WeightDesc(ctypes.Structure):
    _fields_ = [
        ("variant", ctypes.c_int),
        ("K", ctypes.c_int64), ("N", ctypes.c_int64), ("r", ctypes.c_int64),
        ("max_M", ctypes.c_int64),
        ("flags", ctypes.c_uint32),
        ("lam", ctypes.c_void_p), ("L1", ctypes.c_void_p), ("L2", ctypes.c_void_p),
        ("w_codes", ctypes.c_void_p), ("w_scales", ctypes.c_void_p), ("bias", ctypes.c_void_p),
        ("w_scale_exp", ctypes.c_int32),
        ("q_norm", ctypes.c_void_p), ("k_norm", ctypes.c_void_p), ("norm_eps", ctypes.c_float),
    ]


class AWQDesc(ctypes.Structure):
    _fields_ = [
        ("K", ctypes.c_int64), ("N", ctypes.c_int64), ("max_M", ctypes.c_int64),
        ("a", ctypes.c_void_p), ("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p),
        ("zeros", ctypes.c_void_p), ("bias", ctypes.c_void_p),
    ]


_LIB = None


def lib(build_if_missing: bool = True) -> ctypes.CDLL:
    """Load libsvdq.so (building it first when absent or stale)."""
    global _LIB
    if _LIB is not None:
        return _LIB
    path = _build.LIB
    if build_if_missing and _build.stale():
        _build.build()
    if not os.path.exists(path):
        raise OSError(f"libsvdq.so not found at {path}; run python -m "
                      "bit_diffusion_transformer_w4a4_b200.build")
    L = ctypes.CDLL(path)
    vp, i64, st = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    L.svdq_weights_load.argtypes = [ctypes.POINTER(WeightDesc), ctypes.POINTER(vp), vp]
    L.svdq_weights_free.argtypes = [vp]
    L.svdq_act_scales_bytes.argtypes = [vp, i64, ctypes.POINTER(ctypes.c_size_t)]
    L.svdq_quantize_act_lowrank_down.argtypes = [vp, vp, i64, vp, vp, vp, vp]
    L.svdq_w4a4_gemm_lowrank_up.argtypes = [vp, vp, vp, vp, i64, vp, vp]
    L.svdq_linear_forward.argtypes = [vp, vp, vp, i64, vp]
    L.svdq_linear_forward_host.argtypes = [vp, vp, vp, i64, vp]
    L.svdq_device_status.argtypes = [vp, vp]
    L.svdq_debug_set_fault.argtypes = [vp, ctypes.c_uint32, ctypes.c_uint32]
    L.svdq_selftest_division.argtypes = [ctypes.c_int, ctypes.c_void_p]
    L.svdq_w4a4_gemm_lowrank_up_qkv.argtypes = [vp, vp, vp, vp, i64, vp, vp, vp]
    L.svdq_w4a4_gemm_lowrank_up_chain.argtypes = [vp, vp, vp, vp, i64, vp, vp, vp, vp, vp, vp]
    L.svdq_linear_forward_chain.argtypes = [vp, vp, vp, vp, i64, vp]
    L.svdq_device_error_site.argtypes = [vp, vp, ctypes.POINTER(ctypes.c_int)]
    L.svdq_set_deterministic.argtypes = [vp, ctypes.c_int]
    L.svdq_linear_forward_qkv.argtypes = [vp, vp, vp, vp, i64, vp]
    L.svdq_awq_load.argtypes = [ctypes.POINTER(AWQDesc), ctypes.POINTER(vp), vp]
    L.svdq_awq_free.argtypes = [vp]
    L.svdq_awq_w4a16_forward.argtypes = [vp, vp, vp, i64, vp]
    L.svdq_prep_calibrate.argtypes = [vp, i64, vp, i64, i64, ctypes.c_float, vp, vp]
    L.svdq_prep_lowrank.argtypes = [vp, vp, i64, i64, i64, vp, i64, ctypes.c_int, vp, vp, vp]
    L.svdq_prep_residual_quantize.argtypes = [st, vp, vp, vp, vp, i64, i64, i64, ctypes.c_int, vp, vp,
                                              ctypes.POINTER(ctypes.c_int32), vp]
    L.svdq_quantize_act_lowrank_down_static.argtypes = [st, i64, i64, vp, vp, vp, i64, vp, vp, vp, vp, vp]
    L.svdq_status_string.argtypes = [st]
    L.svdq_status_string.restype = ctypes.c_char_p
    L.svdq_version.restype = ctypes.c_char_p
    for name in EXPORTED:
        f = getattr(L, name)
        if f.restype is None or f.restype is ctypes.c_int:
            f.restype = st
    _LIB = L
    return L


def _check(code: int, where: str) -> None:
    if code != 0:
        raise SvdqError(code, where)


def _ptr(a) -> int:
    """Device or host address of a torch tensor / numpy array (None -> 0)."""
    if a is None:
        return 0
    if isinstance(a, np.ndarray):
        return a.ctypes.data
    return a.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        import torch
        if not torch.cuda.is_available():
            return 0            # the library itself reports the missing device
        return torch.cuda.current_stream().cuda_stream
    return int(stream)


def selftest_division(variant: int) -> tuple[int, int]:
    """(code mismatches, normal-range quotient mismatches) -- both 0 expected."""
    n = (ctypes.c_ulonglong * 2)()
    _check(lib().svdq_selftest_division(variant, n), "svdq_selftest_division")
    return int(n[0]), int(n[1])


class SVDQWeights:
    """A loaded layer: owns a library handle (``svdq_weights_t``)."""

    def __init__(self, pw, max_M: int, stream=None, single_sm: bool = False,
                 int4_f16: bool = False, qkv_norm=None):
        """``pw`` has fields variant, K, N, r, lam, L1, L2, codes, scales, bias, gelu
        (host numpy arrays in the formats of ``svdq_weight_desc``).  ``single_sm``
        sets SVDQ_GEMM_SINGLE_SM (NVFP4 GEMM on single SMs; by default it runs on
        pairs of SMs when M > 128).  ``int4_f16`` sets SVDQ_INT4_F16 (INT4 GEMM as
        one fp16 GEMM of the exactly dequantised operands).  ``qkv_norm`` =
        (q_norm bf16 [128], k_norm bf16 [128], eps) sets SVDQ_EPI_QKV_NORM_ROPE."""
        self._keep = [np.ascontiguousarray(pw.lam, dtype=np.float32),
                      np.ascontiguousarray(pw.L1, dtype=np.uint16),
                      np.ascontiguousarray(pw.L2, dtype=np.uint16),
                      np.ascontiguousarray(pw.codes, dtype=np.uint8),
                      np.ascontiguousarray(pw.scales),
                      None if pw.bias is None else np.ascontiguousarray(pw.bias, dtype=np.uint16)]
        lam, L1, L2, codes, scales, bias = self._keep
        qn = kn = None
        eps = 0.0
        if qkv_norm is not None:
            qn = np.ascontiguousarray(qkv_norm[0], dtype=np.uint16)
            kn = np.ascontiguousarray(qkv_norm[1], dtype=np.uint16)
            eps = float(qkv_norm[2])
            self._keep += [qn, kn]
        self.qkv = qkv_norm is not None
        self.variant, self.K, self.N, self.r = int(pw.variant), int(pw.K), int(pw.N), int(pw.r)
        self.max_M = int(max_M)
        self.gelu = bool(pw.gelu)
        d = WeightDesc(self.variant, self.K, self.N, self.r, self.max_M,
                       (EPI_GELU if self.gelu else 0) | (GEMM_SINGLE_SM if single_sm else 0)
                       | (INT4_F16 if int4_f16 else 0) | (EPI_QKV_NORM_ROPE if self.qkv else 0),
                       _ptr(lam), _ptr(L1) if self.r else 0, _ptr(L2) if self.r else 0,
                       _ptr(codes), _ptr(scales), _ptr(bias), int(getattr(pw, "w_scale_exp", 0)),
                       _ptr(qn), _ptr(kn), eps)
        h = ctypes.c_void_p(0)
        self._lib = lib()
        _check(self._lib.svdq_weights_load(ctypes.byref(d), ctypes.byref(h), _stream(stream)),
               "svdq_weights_load")
        self.handle = h

    @property
    def G(self) -> int:
        return 64 if self.variant == INT4 else 16

    def act_scales_bytes(self, M: int) -> int:
        n = ctypes.c_size_t(0)
        _check(self._lib.svdq_act_scales_bytes(self.handle, M, ctypes.byref(n)), "svdq_act_scales_bytes")
        return int(n.value)

    # --------------------------------------------------------------- the calls
    def quantize_act_lowrank_down(self, x, M, act_codes, act_scales, t, stream=None):
        _check(self._lib.svdq_quantize_act_lowrank_down(
            self.handle, _ptr(x), int(M), _ptr(act_codes), _ptr(act_scales), _ptr(t),
            _stream(stream)), "svdq_quantize_act_lowrank_down")

    def w4a4_gemm_lowrank_up(self, act_codes, act_scales, t, M, y, stream=None):
        _check(self._lib.svdq_w4a4_gemm_lowrank_up(
            self.handle, _ptr(act_codes), _ptr(act_scales), _ptr(t), int(M), _ptr(y),
            _stream(stream)), "svdq_w4a4_gemm_lowrank_up")

    def w4a4_gemm_lowrank_up_qkv(self, act_codes, act_scales, t, M, rope, y, stream=None):
        _check(self._lib.svdq_w4a4_gemm_lowrank_up_qkv(
            self.handle, _ptr(act_codes), _ptr(act_scales), _ptr(t), int(M), _ptr(rope), _ptr(y),
            _stream(stream)), "svdq_w4a4_gemm_lowrank_up_qkv")

    def linear_forward_qkv(self, x, rope, y, M, stream=None):
        _check(self._lib.svdq_linear_forward_qkv(self.handle, _ptr(x), _ptr(rope), _ptr(y), int(M),
                                                 _stream(stream)), "svdq_linear_forward_qkv")

    def linear_forward(self, x, y, M, stream=None):
        _check(self._lib.svdq_linear_forward(self.handle, _ptr(x), _ptr(y), int(M), _stream(stream)),
               "svdq_linear_forward")

    def linear_forward_host(self, x_host, y_host, M, stream=None):
        _check(self._lib.svdq_linear_forward_host(self.handle, _ptr(x_host), _ptr(y_host), int(M),
                                                  _stream(stream)), "svdq_linear_forward_host")

    def device_status(self, stream=None) -> int:
        return int(self._lib.svdq_device_status(self.handle, _stream(stream)))

    def device_error_site(self, stream=None) -> int:
        """Wait-site code of the first expired bounded wait (0 if none)."""
        v = ctypes.c_int(0)
        _check(self._lib.svdq_device_error_site(self.handle, _stream(stream), ctypes.byref(v)),
               "svdq_device_error_site")
        return int(v.value)

    def set_deterministic(self, on: bool = True) -> None:
        """Sum kernel 1's split partial T tiles in a fixed order (bit-reproducible
        T and Y) instead of with fp32 reductions."""
        _check(self._lib.svdq_set_deterministic(self.handle, 1 if on else 0), "svdq_set_deterministic")

    def debug_set_fault(self, mask: int, timeout_us: int) -> None:
        _check(self._lib.svdq_debug_set_fault(self.handle, mask, timeout_us), "svdq_debug_set_fault")

    # ------------------------------------------------------- torch conveniences
    def alloc_act(self, M: int, device="cuda"):
        """Allocate (codes, scales, t) device buffers for M tokens."""
        import torch
        codes = torch.empty((M, self.K // 2), dtype=torch.uint8, device=device)
        scales = torch.empty(self.act_scales_bytes(M), dtype=torch.uint8, device=device)
        t = torch.empty((M, max(self.r, 1)), dtype=torch.float32, device=device)
        return codes, scales, t

    def close(self) -> None:
        if getattr(self, "handle", None) is not None and self.handle.value:
            self._lib.svdq_weights_free(self.handle)
            self.handle = ctypes.c_void_p(0)

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class AWQWeights:
    """A loaded AWQ W4A16 layer: owns a library handle (``svdq_awq_t``)."""

    def __init__(self, p, max_M: int, stream=None):
        """``p`` has fields K, N, a, codes, scales, zeros, bias (host numpy
        arrays in the formats of ``svdq_awq_desc``)."""
        self._keep = [np.ascontiguousarray(p.a, dtype=np.float32),
                      np.ascontiguousarray(p.codes, dtype=np.uint8),
                      np.ascontiguousarray(p.scales, dtype=np.uint16),
                      np.ascontiguousarray(p.zeros, dtype=np.uint8),
                      None if p.bias is None else np.ascontiguousarray(p.bias, dtype=np.uint16)]
        a, codes, scales, zeros, bias = self._keep
        self.K, self.N, self.max_M = int(p.K), int(p.N), int(max_M)
        d = AWQDesc(self.K, self.N, self.max_M, _ptr(a), _ptr(codes), _ptr(scales), _ptr(zeros),
                    _ptr(bias))
        h = ctypes.c_void_p(0)
        self._lib = lib()
        _check(self._lib.svdq_awq_load(ctypes.byref(d), ctypes.byref(h), _stream(stream)), "svdq_awq_load")
        self.handle = h

    def forward(self, x, y, M, stream=None):
        _check(self._lib.svdq_awq_w4a16_forward(self.handle, _ptr(x), _ptr(y), int(M), _stream(stream)),
               "svdq_awq_w4a16_forward")

    def close(self) -> None:
        if getattr(self, "handle", None) is not None and self.handle.value:
            self._lib.svdq_awq_free(self.handle)
            self.handle = ctypes.c_void_p(0)

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


# ------------------------------------------------------------- weight prep
def prep_calibrate(x, M, w, K, N, lam, alpha=0.5, stream=None):
    """lambda (fp32 [K], written) from calibration activations x (bf16
    [M x K]) and the weight w (bf16 [K x N]), all device tensors."""
    _check(lib().svdq_prep_calibrate(_ptr(x), int(M), _ptr(w), int(K), int(N), float(alpha), _ptr(lam),
                                     _stream(stream)), "svdq_prep_calibrate")


def prep_lowrank(w, lam, K, N, r, omega, l, power_iters, L1, L2, stream=None):
    """Rank-r bf16 factors L1 [K x r], L2 [r x N] (written) of diag(lam) w by
    a randomized SVD with the caller's Gaussian test matrix omega (fp32
    [N x l])."""
    _check(lib().svdq_prep_lowrank(_ptr(w), _ptr(lam), int(K), int(N), int(r), _ptr(omega), int(l),
                                   int(power_iters), _ptr(L1), _ptr(L2), _stream(stream)), "svdq_prep_lowrank")


def prep_residual_quantize(variant, w, lam, L1, L2, K, N, r, codes, scales, tensor_scale=False,
                           stream=None) -> int:
    """Codes [N x K/2] and scales [N x K/G] (written) of the residual
    diag(lam) w - L1 L2; returns the per-tensor scale exponent (0 without
    tensor_scale)."""
    e = ctypes.c_int32(0)
    _check(lib().svdq_prep_residual_quantize(int(variant), _ptr(w), _ptr(lam), _ptr(L1), _ptr(L2), int(K),
                                             int(N), int(r), int(bool(tensor_scale)), _ptr(codes),
                                             _ptr(scales), ctypes.byref(e), _stream(stream)),
           "svdq_prep_residual_quantize")
    return int(e.value)


def gemm_lowrank_up_chain(h1, act_codes, act_scales, t, M, y1, h2, codes2, scales2, t2, stream=None):
    """h1's kernel 2 with h2's activation side in its epilogue (see
    svdq_w4a4_gemm_lowrank_up_chain); y1 may be None."""
    _check(lib().svdq_w4a4_gemm_lowrank_up_chain(
        h1.handle, _ptr(act_codes), _ptr(act_scales), _ptr(t), int(M), _ptr(y1), h2.handle, _ptr(codes2),
        _ptr(scales2), _ptr(t2), _stream(stream)), "svdq_w4a4_gemm_lowrank_up_chain")


def linear_forward_chain(h1, h2, x, y2, M, stream=None):
    """y2 = fc2(fc1(x)) with fc2's activation side fused into fc1's GEMM."""
    _check(lib().svdq_linear_forward_chain(h1.handle, h2.handle, _ptr(x), _ptr(y2), int(M), _stream(stream)),
           "svdq_linear_forward_chain")


def untile_nvfp4_scales(buf: np.ndarray, M: int, K: int) -> np.ndarray:
    """Tensor-core tiled E4M3 activation scales -> canonical [M x K/16]."""
    buf = np.asarray(buf, dtype=np.uint8)
    m = np.arange(M)[:, None]
    b = np.arange(K // 16)[None, :]
    off = ((m // 128) * (K // 64) + b // 4) * 512 + (m % 32) * 16 + ((m // 32) % 4) * 4 + b % 4
    return buf[off]
