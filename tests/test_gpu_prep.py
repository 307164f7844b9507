"""GPU weight preparation (through the C ABI) against the CPU oracle:
calibration factors bit-exact, residual codes and scales bit-exact given the
oracle's factors (INT4, NVFP4, NVFP4 with the per-tensor scale), the
randomized SVD within a small factor of the exact truncated SVD's residual
(Eckart-Young optimum), and a layer prepared end to end on the GPU as
accurate against X W as one prepared by the oracle."""
import numpy as np
import pytest

from bit_diffusion_transformer_w4a4_b200 import svdq
from bit_diffusion_transformer_w4a4_b200 import workloads as W
from oracle import forward as O
from oracle import formats as F
from oracle import prep as P
import parity as PT

pytestmark = pytest.mark.gpu
INT4, NVFP4 = W.INT4, W.NVFP4


def _dev(a):
    return PT.to_dev(np.ascontiguousarray(a))


def _bf16_dev(bits):
    import torch
    return _dev(bits.view(np.int16)).view(torch.bfloat16)


def test_calibrate_matches_oracle():
    import torch
    lay = W.Layer("cal", M=777, K=1024, N=640, r=32, variant=NVFP4, config_id=95)
    x = W.activations(lay)
    w = W.weight(lay)
    xv = W.bf16_bits_to_f32(x).copy()
    xv[:, 5] = 0.0                          # zero activation channel -> 1
    wv = w.copy()
    wv[9, :] = 0.0                          # zero weight row -> 1
    xv[:, 17] *= 2.0 ** 60                  # clamped at 2^20
    wv[17, :] *= 2.0 ** -60
    x = W.to_bf16_bits(xv)
    wb = W.to_bf16_bits(wv)
    lam = torch.empty(lay.K, dtype=torch.float32, device="cuda")
    svdq.prep_calibrate(_bf16_dev(x), lay.M, _bf16_dev(wb), lay.K, lay.N, lam)
    torch.cuda.synchronize()
    ref = P.calibrate_lambda(F.bf16_from_bits(x), F.bf16_from_bits(wb))
    got = lam.cpu().numpy()
    assert np.array_equal(got, ref)
    assert got[5] == 1.0 and got[9] == 1.0 and got[17] == np.float32(2.0 ** 20)


@pytest.mark.parametrize("variant,tensor_scale,r", [(INT4, False, 32), (INT4, False, 0), (NVFP4, False, 32),
                                                    (NVFP4, True, 32), (NVFP4, True, 0)])
def test_residual_quantize_matches_oracle(variant, tensor_scale, r):
    """Given the oracle's lambda and bf16 factors, the GPU's residual codes
    and scales equal the oracle's bit for bit (R in fp64 on both sides)."""
    import torch
    lay = W.Layer("rq", M=256, K=1024, N=600, r=r, variant=variant, config_id=96)
    x = W.activations(lay)
    w = W.weight(lay)
    pw = P.prepare(x, w, r, variant, tensor_scale=tensor_scale)
    G = O.GROUP[variant]
    codes = torch.empty((lay.N, lay.K // 2), dtype=torch.uint8, device="cuda")
    sb = 2 if variant == INT4 else 1
    scales = torch.empty(lay.N * (lay.K // G) * sb, dtype=torch.uint8, device="cuda")
    L1 = _dev(pw.L1) if r else None
    L2 = _dev(pw.L2) if r else None
    e = svdq.prep_residual_quantize(variant, _bf16_dev(W.to_bf16_bits(w)), _dev(pw.lam), L1, L2, lay.K,
                                    lay.N, r, codes, scales, tensor_scale=tensor_scale)
    torch.cuda.synchronize()
    assert e == pw.w_scale_exp
    got_c = codes.cpu().numpy()
    got_s = scales.cpu().numpy()
    got_s = got_s.view(np.uint16).reshape(lay.N, -1) if variant == INT4 else got_s.reshape(lay.N, -1)
    bad_c = int((got_c != pw.codes).sum())
    bad_s = int((got_s != pw.scales).sum())
    assert bad_c == 0 and bad_s == 0, (bad_c, bad_s)


@pytest.mark.parametrize("r,power_iters", [(32, 1), (32, 2), (128, 2)])
def test_randomized_svd_near_optimal(r, power_iters):
    """lowrank128 weights (singular values 48/i plus noise): the GPU factors'
    residual ||W_hat - L1 L2||_F is within 2% of the exact truncated SVD's
    (the oracle's prepare(), bf16 factors as well); r = 128 runs a sketch of
    144 columns."""
    import torch
    lay = W.Layer("rs", M=512, K=1024, N=768, r=r, variant=NVFP4, weight_kind="lowrank128", config_id=97)
    x = W.activations(lay)
    w = W.weight(lay)
    pw = P.prepare(x, w, lay.r, NVFP4)
    l = lay.r + 16
    omega = np.random.default_rng(123).standard_normal((lay.N, l)).astype(np.float32)
    L1 = torch.empty((lay.K, lay.r), dtype=torch.int16, device="cuda")
    L2 = torch.empty((lay.r, lay.N), dtype=torch.int16, device="cuda")
    svdq.prep_lowrank(_bf16_dev(W.to_bf16_bits(w)), _dev(pw.lam), lay.K, lay.N, lay.r, _dev(omega), l,
                      power_iters, L1, L2)
    torch.cuda.synchronize()
    l1 = F.bf16_from_bits(L1.cpu().numpy().view(np.uint16))
    l2 = F.bf16_from_bits(L2.cpu().numpy().view(np.uint16))
    res_gpu = np.linalg.norm(pw.w_hat - l1 @ l2)
    res_ora = np.linalg.norm(pw.R)
    opt = np.sqrt(np.sum(pw.S[lay.r:] ** 2))
    PT.record(f"rsvd r{r} q{power_iters}", "residual / optimum", res_gpu / opt, 1.02)
    assert res_ora <= 1.001 * opt
    assert res_gpu <= 1.02 * opt, (res_gpu / opt, res_ora / opt)


@pytest.mark.parametrize("variant,tensor_scale", [(INT4, False), (NVFP4, False), (NVFP4, True)])
def test_gpu_prepared_layer_accuracy(variant, tensor_scale):
    """Calibration, randomized SVD and residual quantisation on the GPU, then
    the layer: its error against X W matches that of the oracle-prepared
    layer (the scheme's quantisation error) within 10%."""
    import torch
    lay = W.Layer("gp", M=512, K=1024, N=768, r=32, variant=variant, weight_kind="lowrank128", config_id=98)
    x = W.activations(lay)
    w = W.weight(lay)
    G = O.GROUP[variant]
    xd, wd = _bf16_dev(x), _bf16_dev(W.to_bf16_bits(w))
    lam = torch.empty(lay.K, dtype=torch.float32, device="cuda")
    svdq.prep_calibrate(xd, lay.M, wd, lay.K, lay.N, lam)
    l = lay.r + 16
    omega = np.random.default_rng(7).standard_normal((lay.N, l)).astype(np.float32)
    L1 = torch.empty((lay.K, lay.r), dtype=torch.int16, device="cuda")
    L2 = torch.empty((lay.r, lay.N), dtype=torch.int16, device="cuda")
    svdq.prep_lowrank(wd, lam, lay.K, lay.N, lay.r, _dev(omega), l, 2, L1, L2)
    codes = torch.empty((lay.N, lay.K // 2), dtype=torch.uint8, device="cuda")
    sb = 2 if variant == INT4 else 1
    scales = torch.empty(lay.N * (lay.K // G) * sb, dtype=torch.uint8, device="cuda")
    e = svdq.prep_residual_quantize(variant, wd, lam, L1, L2, lay.K, lay.N, lay.r, codes, scales,
                                    tensor_scale=tensor_scale)
    torch.cuda.synchronize()
    sc = scales.cpu().numpy()
    pw = W.PackedWeights(variant, lay.K, lay.N, lay.r, lam.cpu().numpy(), L1.cpu().numpy().view(np.uint16),
                         L2.cpu().numpy().view(np.uint16), codes.cpu().numpy(),
                         sc.view(np.uint16).reshape(lay.N, -1) if variant == INT4 else sc.reshape(lay.N, -1),
                         w_scale_exp=e)
    h = svdq.SVDQWeights(pw, lay.M)
    got = PT.gpu_forward(h, x, lay.M)
    h.close()
    ref = F.bf16_from_bits(x) @ w
    e_gpu = PT.rel_fro(F.bf16_from_bits(got["Y"]), ref)
    po = P.prepare(x, w, lay.r, variant, tensor_scale=tensor_scale)
    e_ora = PT.rel_fro(O.linear_forward(x, po)["y"], ref)
    PT.record(f"gpu prep v{variant} ts{int(tensor_scale)}", "scheme err / oracle's", e_gpu / e_ora, 1.1)
    assert e_gpu <= 1.1 * e_ora + 1e-4, (e_gpu, e_ora)
