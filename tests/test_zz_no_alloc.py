"""The allocation-free activation-kernel entry point.

Callers that cannot let a library allocate device memory (code inside a
CUDA-graph capture, runtimes that own a fixed memory pool, processes with a
hard memory budget) use svdq_quantize_act_lowrank_down_static: they pass
every buffer themselves, and the split-K scratch comes from a static device
array of the library.  This file checks, through the C ABI, that its outputs
equal those of the handle-based svdq_quantize_act_lowrank_down on the same
inputs, on two calls in a row (the static scratch keeps the previous call's
contents), and that oversize requests are refused before any work.

The file name makes pytest collect it last.
"""
import ctypes

import numpy as np
import pytest

from bit_diffusion_transformer_w4a4_b200 import svdq
from bit_diffusion_transformer_w4a4_b200 import workloads as W
import parity as PT

pytestmark = pytest.mark.gpu


def _static_call(L, lay, inv_d, l1t_d, x_d, codes, scales, t, err_d):
    import torch
    st = torch.cuda.current_stream().cuda_stream
    return L.svdq_quantize_act_lowrank_down_static(
        lay.variant, lay.K, lay.r, inv_d.data_ptr(), l1t_d.data_ptr() if lay.r else 0,
        x_d.data_ptr(), lay.M, codes.data_ptr(), scales.data_ptr(),
        t.data_ptr() if lay.r else 0, err_d.data_ptr(), st)


@pytest.mark.parametrize("variant", [W.INT4, W.NVFP4])
@pytest.mark.parametrize("M,K,r", [(4608, 3072, 32), (300, 512, 128), (64, 256, 16), (200, 384, 0)])
def test_static_scratch_matches_handle_path(variant, M, K, r):
    import torch
    lay = W.Layer("noalloc", M=M, K=K, N=256, r=r, variant=variant, config_id=80, layer_id=r)
    pw = W.synthetic_packed(lay)
    x = W.activations(lay)
    h = svdq.SVDQWeights(pw, M)
    ref = PT.gpu_forward(h, x, M)            # handle-based kernel 1 (and kernel 2)

    L = svdq.lib()
    inv = (np.float32(1) / pw.lam).astype(np.float32)
    inv_d = torch.from_numpy(inv).cuda()
    l1t_d = torch.from_numpy(np.ascontiguousarray(pw.L1.T).view(np.int16)).cuda()
    x_d = torch.from_numpy(x.view(np.int16)).cuda()
    err_d = torch.zeros(1, dtype=torch.int32, device="cuda")
    for call in range(2):
        codes, scales, t = h.alloc_act(M)
        codes.fill_(0xA5)
        scales.fill_(0xA5)
        t.fill_(float("nan"))
        assert _static_call(L, lay, inv_d, l1t_d, x_d, codes, scales, t, err_d) == 0
        torch.cuda.synchronize()
        assert int(err_d.item()) == 0
        got_codes = codes.cpu().numpy()
        sc = scales.cpu().numpy()
        sc = (svdq.untile_nvfp4_scales(sc, M, K) if variant == W.NVFP4
              else sc.view(np.uint16).reshape(M, K // 64))
        assert np.array_equal(got_codes, ref["codes"]), f"call {call}: codes differ"
        assert np.array_equal(sc, ref["scales"]), f"call {call}: scales differ"
        if r:
            T = t.cpu().numpy()[:, :r]
            assert PT.rel_fro(T, ref["T"]) <= PT.T_REL, f"call {call}: T differs"
    h.close()


def test_static_scratch_refuses_oversize():
    L = svdq.lib()
    # M beyond the counters' capacity: refused before any pointer is touched
    fake = ctypes.c_void_p(16)
    assert L.svdq_quantize_act_lowrank_down_static(
        W.NVFP4, 3072, 32, fake, fake, fake, 4096 * 128 + 1, fake, fake, fake, None, None) == 2
    assert L.svdq_quantize_act_lowrank_down_static(
        W.NVFP4, 3000, 32, fake, fake, fake, 128, fake, fake, fake, None, None) == 2


def test_static_scratch_null_error_word():
    """device_error may be NULL (timeouts are then not reported to anyone):
    the outputs of a normal call are the same."""
    import torch
    M, K, r = 384, 512, 32
    lay = W.Layer("noalloc0", M=M, K=K, N=256, r=r, variant=W.NVFP4, config_id=81)
    pw = W.synthetic_packed(lay)
    x = W.activations(lay)
    h = svdq.SVDQWeights(pw, M)
    ref = PT.gpu_forward(h, x, M)
    L = svdq.lib()
    inv_d = torch.from_numpy((np.float32(1) / pw.lam).astype(np.float32)).cuda()
    l1t_d = torch.from_numpy(np.ascontiguousarray(pw.L1.T).view(np.int16)).cuda()
    x_d = torch.from_numpy(x.view(np.int16)).cuda()
    codes, scales, t = h.alloc_act(M)
    st = torch.cuda.current_stream().cuda_stream
    assert L.svdq_quantize_act_lowrank_down_static(
        lay.variant, K, r, inv_d.data_ptr(), l1t_d.data_ptr(), x_d.data_ptr(), M, codes.data_ptr(),
        scales.data_ptr(), t.data_ptr(), None, st) == 0
    torch.cuda.synchronize()
    assert np.array_equal(codes.cpu().numpy(), ref["codes"])
    assert np.array_equal(svdq.untile_nvfp4_scales(scales.cpu().numpy(), M, K), ref["scales"])
    assert PT.rel_fro(t.cpu().numpy()[:, :r], ref["T"]) <= PT.T_REL
    h.close()
