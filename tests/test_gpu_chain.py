"""GPU checks of the fused DiT-MLP pair (fc2's activation side in fc1's GEMM
epilogue, svdq_w4a4_gemm_lowrank_up_chain / svdq_linear_forward_chain):

* against the library's own two-kernel path on the same inputs: fc2's
  activation codes and scales bit-identical, T2 within the fp32
  accumulation bound, fc1's optional output y1 bit-identical;
* against the oracle layer by layer: fc1's stored output against the oracle
  fc1, and the chain's fc2 output against the oracle fc2 fed with that same
  fc1 output, each within the layer's bars."""
import numpy as np
import pytest

from bit_diffusion_transformer_w4a4_b200 import svdq
from bit_diffusion_transformer_w4a4_b200 import workloads as W
from oracle import forward as O
from oracle import prep as P
import parity as PT

pytestmark = pytest.mark.gpu


def _pair(M, K, N1, r1, r2, seed=0, prepped=True):
    l1 = W.Layer("fc1", M=M, K=K, N=N1, r=r1, variant=W.NVFP4, gelu=True, bias=True, config_id=88, layer_id=0)
    l2 = W.Layer("fc2", M=M, K=N1, N=K, r=r2, variant=W.NVFP4, config_id=88, layer_id=1)
    x = W.activations(l1, seed)
    if prepped:
        pw1 = P.prepare(x, W.weight(l1, seed), r1, W.NVFP4, bias_bits=W.bias(l1, seed), gelu=True)
        y1 = O.linear_forward(x, pw1)["Y"]          # the oracle fc1's output calibrates fc2
        pw2 = P.prepare(y1, W.weight(l2, seed), r2, W.NVFP4)
    else:
        pw1, pw2 = W.synthetic_packed(l1, seed), W.synthetic_packed(l2, seed)
    return l1, l2, x, pw1, pw2


@pytest.mark.parametrize("M,K,N1,r1,r2", [(300, 512, 1024, 32, 32), (129, 256, 512, 0, 16),
                                          (1000, 384, 2048, 32, 16)])
def test_chain_matches_two_kernel_path(M, K, N1, r1, r2):
    import torch
    l1, l2, x, pw1, pw2 = _pair(M, K, N1, r1, r2, prepped=False)
    h1 = svdq.SVDQWeights(pw1, M)
    h2 = svdq.SVDQWeights(pw2, M)
    xd = PT.to_dev(x.view(np.int16)).view(torch.bfloat16)
    # two-kernel path: fc1 -> y1 (bf16) -> fc2's activation kernel
    c1, s1, t1 = h1.alloc_act(M)
    h1.quantize_act_lowrank_down(xd, M, c1, s1, t1)
    y1 = torch.empty((M, N1), dtype=torch.bfloat16, device="cuda")
    h1.w4a4_gemm_lowrank_up(c1, s1, t1, M, y1)
    c2, s2, t2 = h2.alloc_act(M)
    h2.quantize_act_lowrank_down(y1, M, c2, s2, t2)
    # fused: fc2's activation side in fc1's epilogue
    y1f = torch.empty_like(y1)
    c2f, s2f, t2f = h2.alloc_act(M)
    svdq.gemm_lowrank_up_chain(h1, c1, s1, t1, M, y1f, h2, c2f, s2f, t2f)
    torch.cuda.synchronize()
    assert h1.device_status() == 0 and h2.device_status() == 0
    assert torch.equal(y1f, y1)
    assert torch.equal(c2f, c2)
    # scales: the tiled layout pads the row blocks; compare the M rows
    ua = svdq.untile_nvfp4_scales(PT.from_dev(s2f), M, N1)
    ub = svdq.untile_nvfp4_scales(PT.from_dev(s2), M, N1)
    assert np.array_equal(ua, ub)
    d = float(torch.linalg.norm(t2f[:, :r2].double() - t2[:, :r2].double()))
    y1v = W.bf16_bits_to_f32(PT.from_dev(y1.view(torch.int16)).view(np.uint16)).astype(np.float64)
    xp = O.smooth_activations(W.to_bf16_bits(y1v.astype(np.float32)),
                              (np.float32(1) / pw2.lam).astype(np.float32)).astype(np.float64)
    tb = 2 * PT.t_bound(xp, W.bf16_bits_to_f32(pw2.L1).astype(np.float64))
    PT.record(f"chain M{M} N1{N1}", "||dT2|| / fp32 bound", d / tb, 1.0)
    assert d <= tb
    # the whole chain through the workspaces gives the same fc2 output
    y2a = torch.empty((M, K), dtype=torch.bfloat16, device="cuda")
    h2.w4a4_gemm_lowrank_up(c2, s2, t2, M, y2a)
    y2b = torch.empty_like(y2a)
    svdq.linear_forward_chain(h1, h2, xd, y2b, M)
    torch.cuda.synchronize()
    assert h1.device_status() == 0 and h2.device_status() == 0
    a = y2a.double()
    assert float(torch.linalg.norm(y2b.double() - a) / torch.linalg.norm(a)) <= 1e-3
    h1.close()
    h2.close()


@pytest.mark.parametrize("M", [256, 700])
def test_chain_against_oracle(M):
    """fc2(fc1(x)) through the fused kernels against the oracle, layer by
    layer on the same inputs: fc1's bf16 output y1 (stored by the fused
    kernel) against the oracle fc1 on x, and the chain's fc2 output against
    the oracle fc2 on that same y1.  fc2 quantises its input to 4 bits, so a
    one-ulp difference in y1 (fp32 against fp64 accumulation) may move an
    E4M3 group scale or an E2M1 code and fc2's output by more than the
    single-layer bars; each layer is held to its bars given its input."""
    import torch
    K, N1 = 256, 1024
    l1, l2, x, pw1, pw2 = _pair(M, K, N1, 32, 32)
    h1 = svdq.SVDQWeights(pw1, M)
    h2 = svdq.SVDQWeights(pw2, M)
    xd = PT.to_dev(x.view(np.int16)).view(torch.bfloat16)
    y2 = torch.empty((M, K), dtype=torch.bfloat16, device="cuda")
    svdq.linear_forward_chain(h1, h2, xd, y2, M)
    # the same fc1 pass with its output stored
    c1, s1, t1 = h1.alloc_act(M)
    h1.quantize_act_lowrank_down(xd, M, c1, s1, t1)
    y1 = torch.empty((M, N1), dtype=torch.bfloat16, device="cuda")
    c2, s2, t2 = h2.alloc_act(M)
    svdq.gemm_lowrank_up_chain(h1, c1, s1, t1, M, y1, h2, c2, s2, t2)
    torch.cuda.synchronize()
    assert h1.device_status() == 0 and h2.device_status() == 0
    Y1 = PT.from_dev(y1.view(torch.int16)).view(np.uint16)
    ref1 = O.linear_forward(x, pw1)
    PT.check_y(Y1, ref1["y"], ref1["Y"], label=f"chain fc1 vs oracle M{M}")
    Yg = PT.from_dev(y2.view(torch.int16)).view(np.uint16)
    ref2 = O.linear_forward(Y1, pw2)
    PT.check_y(Yg, ref2["y"], ref2["Y"], label=f"chain fc2 vs oracle M{M}")
    h1.close()
    h2.close()


def test_chain_refuses_bad_pairs():
    lay1 = W.Layer("a", M=128, K=256, N=384, r=32, variant=W.NVFP4, config_id=89)
    lay2 = W.Layer("b", M=128, K=384, N=256, r=32, variant=W.NVFP4, config_id=89)
    h1 = svdq.SVDQWeights(W.synthetic_packed(lay1), 128)
    h2 = svdq.SVDQWeights(W.synthetic_packed(lay2), 128)
    import torch
    x = torch.zeros((128, 256), dtype=torch.bfloat16, device="cuda")
    y = torch.empty((128, 256), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(svdq.SvdqError):      # N1 = 384 is not a multiple of 256
        svdq.linear_forward_chain(h1, h2, x, y, 128)
    h1.close()
    h2.close()
