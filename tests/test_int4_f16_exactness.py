"""The arithmetic fact behind the fp16-operand INT4 GEMM (SVDQ_INT4_F16):
a bf16 scale s times a 4-bit code q is exactly an fp16 value while
2^-17 <= s and |q s| <= 65504, so the GEMM of the dequantised fp16 operands
computes the same sum of exact products as the per-group int8 form.  Checked
exhaustively over every bf16 scale in the range and every code, and at the
edges where it stops holding.  CPU only."""
import numpy as np


def _bf16_values(lo, hi):
    """Every positive finite bf16 value in [lo, hi], as float64."""
    bits = np.arange(0x0001, 0x7F80, dtype=np.uint32) << 16
    v = bits.view(np.float32).astype(np.float64)
    return v[(v >= lo) & (v <= hi)]


def _exact_in_fp16(x):
    return np.asarray(x, dtype=np.float16).astype(np.float64) == x


def test_activation_codes_times_scales_are_fp16_values():
    s = _bf16_values(2.0 ** -17, 9357.0)          # the activation-scale range the kernel accepts
    assert s.size > 3000
    q = np.arange(-7, 8, dtype=np.float64)         # activation codes: |q| <= 7 (scale = amax / 7)
    prod = s[:, None] * q[None, :]
    assert np.all(_exact_in_fp16(prod))
    assert np.all(_exact_in_fp16(s))               # the scale itself converts exactly


def test_weight_codes_including_minus_eight():
    s = _bf16_values(2.0 ** -17, 65504.0 / 8)
    q = np.arange(-8, 8, dtype=np.float64)
    assert np.all(_exact_in_fp16(s[:, None] * q[None, :]))


def test_bounds_are_tight():
    # just above the activation bound 7 s overflows fp16
    above = _bf16_values(9357.0, 1e6)
    above = above[above > 9357.0]
    with np.errstate(over="ignore"):
        assert not np.isfinite(np.float16(7.0 * above[0]))
    assert np.isfinite(np.float16(7.0 * 9344.0))   # the largest bf16 value <= 9357
    # below 2^-17 an 8-bit scale can lose low bits in fp16's subnormal range
    tiny = _bf16_values(2.0 ** -24, 2.0 ** -17)
    tiny = tiny[tiny < 2.0 ** -17]
    assert not np.all(_exact_in_fp16(tiny[:, None] * np.arange(1, 8)[None, :]))


def test_products_are_exact_in_the_fp32_accumulator():
    # fp16 x fp16 products have at most 22 significant bits: exact in fp32
    rng = np.random.default_rng(0)
    a = rng.standard_normal(4096).astype(np.float16).astype(np.float64)
    b = rng.standard_normal(4096).astype(np.float16).astype(np.float64)
    p = a * b
    assert np.all(p.astype(np.float32).astype(np.float64) == p)
