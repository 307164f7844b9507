"""GPU parity: the CUDA path, called through the C ABI, against the CPU oracle
on the same seeded inputs.  Needs an sm_100 GPU (marked gpu)."""
import copy

import numpy as np
import pytest

from bit_diffusion_transformer_w4a4_b200 import svdq
from bit_diffusion_transformer_w4a4_b200 import workloads as W
from oracle import forward as O
from oracle import prep as P
import parity as PT

pytestmark = pytest.mark.gpu
INT4, NVFP4 = W.INT4, W.NVFP4


def _prepped(M, K, N, r, variant, gelu=False, with_bias=False, seed=0, cid=50):
    lay = W.Layer("t", M=M, K=K, N=N, r=r, variant=variant, gelu=gelu, bias=with_bias,
                  config_id=cid, layer_id=K // 64 + N + r)
    x = W.activations(lay, seed)
    w = W.weight(lay, seed)
    pw = P.prepare(x, w, r, variant, bias_bits=W.bias(lay, seed), gelu=gelu)
    return lay, x, pw


@pytest.mark.parametrize("variant", [INT4, NVFP4])
def test_division_selftest_exhaustive(variant):
    bad_codes, bad_quotients = svdq.selftest_division(variant)
    assert bad_codes == 0 and bad_quotients == 0, (bad_codes, bad_quotients)


@pytest.mark.parametrize("variant", [INT4, NVFP4])
@pytest.mark.parametrize("r", [0, 16, 32, 64, 128])
@pytest.mark.parametrize("M,K", [(200, 512), (64, 256), (1, 128), (384, 1024)])
def test_activation_kernel(variant, r, M, K):
    lay, x, pw = _prepped(M, K, 256, r, variant)
    h = svdq.SVDQWeights(pw, M)
    got = PT.gpu_forward(h, x, M)
    inv = (np.float32(1) / pw.lam).astype(np.float32)
    codes, scales, T = O.quantize_act_lowrank_down(x, inv, pw.L1, variant)
    PT.check_act(got, {"codes": codes, "scales": scales, "T": T}, r=r, label=f"v{variant} r{r} M{M} K{K}")


# Every kernel-2 implementation: INT4 as per-group int8 MMAs (default) or as
# one fp16 GEMM of the dequantised operands (SVDQ_INT4_F16); NVFP4 on SM pairs
# for M > 128 (default) or on single SMs (SVDQ_GEMM_SINGLE_SM).
KERNELS = [(INT4, {}), (INT4, {"int4_f16": True}), (NVFP4, {}), (NVFP4, {"single_sm": True})]
KIDS = ["int4", "int4-f16", "nvfp4-pair", "nvfp4-1sm"]


@pytest.mark.parametrize("variant,opts", KERNELS, ids=KIDS)
@pytest.mark.parametrize("r", [0, 16, 32, 128])
def test_gemm_isolated(variant, opts, r):
    """Kernel 2 alone, fed the oracle's activation codes / scales / T."""
    import torch
    M, K, N = 300, 512, 512
    lay, x, pw = _prepped(M, K, N, r, variant)
    inv = (np.float32(1) / pw.lam).astype(np.float32)
    codes, scales, T = O.quantize_act_lowrank_down(x, inv, pw.L1, variant)
    y_ref, Y_ref = O.gemm_lowrank_up(codes, scales, T, pw.codes, pw.scales, pw.L2, variant)
    h = svdq.SVDQWeights(pw, M, **opts)
    sc = PT.tile_nvfp4_scales(scales, M, K) if variant == NVFP4 else scales.view(np.uint8).reshape(-1)
    tt = np.zeros((M, max(r, 1)), dtype=np.float32)
    tt[:, :r] = T
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    h.w4a4_gemm_lowrank_up(PT.to_dev(codes), PT.to_dev(sc), PT.to_dev(tt), M, y)
    torch.cuda.synchronize()
    assert h.device_status() == 0
    Yg = PT.from_dev(y.view(torch.int16)).view(np.uint16)
    PT.check_y(Yg, y_ref, Y_ref, label=f"gemm v{variant} r{r}")


@pytest.mark.parametrize("variant,opts", KERNELS, ids=KIDS)
@pytest.mark.parametrize("gelu,with_bias", [(False, False), (True, True), (False, True)])
@pytest.mark.parametrize("M,K,N,r", [(300, 512, 448, 32), (129, 1024, 272, 16), (513, 384, 768, 64),
                                     (640, 768, 528, 128)])
def test_forward_small(variant, opts, gelu, with_bias, M, K, N, r):
    """Ragged M and N (partial tiles), several K tiles, bias and GELU."""
    lay, x, pw = _prepped(M, K, N, r, variant, gelu=gelu, with_bias=with_bias)
    h = svdq.SVDQWeights(pw, M, **opts)
    h.set_deterministic()  # the two entry points are compared bit for bit below
    got = PT.gpu_forward(h, x, M)
    ref = O.linear_forward(x, pw)
    PT.check_act(got, ref, r=r, label="fwd")
    PT.check_y(got["Y"], ref["y"], ref["Y"], label=f"fwd v{variant} M{M} N{N}")
    # the fused entry point runs the same kernels: identical bits
    got2 = PT.gpu_forward(h, x, M, two_calls=False)
    assert np.array_equal(got2["Y"], got["Y"])


@pytest.mark.parametrize("variant,opts", KERNELS, ids=KIDS)
def test_several_tiles_per_cta(variant, opts):
    """More tiles than CTAs (or SM pairs): every persistent CTA takes two or
    three tiles, so stage-ring phases, both accumulators and the low-rank
    operand carry across tiles.  Ragged M and N."""
    M, K, N, r = 2000, 256, 4848, 32
    lay, x, pw = _prepped(M, K, N, r, variant, gelu=True, with_bias=True, cid=66)
    h = svdq.SVDQWeights(pw, M, **opts)
    got = PT.gpu_forward(h, x, M)
    rows = np.unique(np.concatenate([np.arange(0, M, 7), [M - 1]]))
    ref = O.linear_forward(x, pw, rows=rows)
    PT.check_y(got["Y"][rows], ref["y"], ref["Y"], label=f"multi-tile v{variant} {opts}")


def test_quantizer_edge_values():
    """All-zero groups, tiny values whose sign survives rounding to zero, huge
    outliers that saturate E4M3 scales, and exact ties."""
    M, K, N, r = 128, 256, 256, 16
    for variant in (INT4, NVFP4):
        lay = W.Layer("edge", M=M, K=K, N=N, r=r, variant=variant, config_id=60)
        pw = W.synthetic_packed(lay)
        pw.lam[:] = 1.0
        x = W.bf16_bits_to_f32(W.activations(lay)).copy()
        x[0, :] = 0.0                              # every group zero -> scale 0
        x[1, :] *= 1e-30                           # subnormal-ish scales
        x[2, :16] = [-0.0, 0.0, -1e-3, 1e-3] * 4   # signed zeros / tiny
        x[3, :] = 5000.0                           # NVFP4 scale saturates at 448
        x[4, :64] = np.arange(64) * 0.25 - 8.0     # many exact ties
        xb = W.to_bf16_bits(x)
        h = svdq.SVDQWeights(pw, M)
        got = PT.gpu_forward(h, xb, M)
        ref = O.linear_forward(xb, pw)
        PT.check_act(got, ref, r=r, label=f"edge v{variant}")


@pytest.mark.parametrize("variant,opts", [(INT4, {}), (NVFP4, {}), (INT4, {"int4_f16": True})],
                         ids=["int4", "nvfp4", "int4-f16"])
@pytest.mark.parametrize("M", [100, 256, 1300, 1536])
def test_host_entry_point_matches_device(variant, opts, M):
    """The host-buffer entry point gives the device entry point's Y bit for
    bit (deterministic T): one chunk on single SMs (M = 100), one chunk
    (256), five chunks with a last one of 276 rows (1300), six chunks of 256
    rows (1536)."""
    import torch
    K, N, r = 512, 512, 32
    lay = W.Layer("host", M=M, K=K, N=N, r=r, variant=variant, config_id=61)
    pw = W.synthetic_packed(lay)
    x = W.activations(lay)
    h = svdq.SVDQWeights(pw, M, **opts)
    h.set_deterministic()
    dev = PT.gpu_forward(h, x, M, two_calls=False)
    xh = torch.from_numpy(x.view(np.int16)).pin_memory()
    yh = torch.empty((M, N), dtype=torch.int16).pin_memory()
    h.linear_forward_host(xh, yh, M)
    torch.cuda.synchronize()
    assert np.array_equal(yh.numpy().view(np.uint16), dev["Y"])


@pytest.mark.parametrize("variant,opts", KERNELS, ids=KIDS)
@pytest.mark.parametrize("mask", [1, 2])
def test_bounded_wait_reports_timeout(variant, opts, mask):
    """A pipeline stage that is never filled: the kernel's bounded wait expires,
    the call reports SVDQ_ERR_DEVICE_TIMEOUT and the context stays usable."""
    M, K, N, r = 256, 1024, 512, 32
    lay = W.Layer("fault", M=M, K=K, N=N, r=r, variant=variant, config_id=62)
    pw = W.synthetic_packed(lay)
    x = W.activations(lay)
    h = svdq.SVDQWeights(pw, M, **opts)
    h.set_deterministic()
    ok = PT.gpu_forward(h, x, M)
    h.debug_set_fault(mask, 20000)                 # 20 ms limit
    import torch
    xd = PT.to_dev(x.view(np.int16)).view(torch.bfloat16)
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    h.linear_forward(xd, y, M)
    # the wait that expired first: kernel 1's sites are 0x1xx, kernel 2's 0x2xx / 0x3xx
    site = h.device_error_site()
    assert (site >> 8) == 1 if mask == 2 else (site >> 8) in (2, 3), hex(site)
    assert h.device_status() == 7                 # SVDQ_ERR_DEVICE_TIMEOUT
    h.debug_set_fault(0, 0)
    again = PT.gpu_forward(h, x, M)
    assert np.array_equal(again["Y"], ok["Y"])


@pytest.mark.parametrize("M", [129, 256, 1000])
def test_pair_and_single_sm_agree(M):
    """The SM-pair and single-SM NVFP4 GEMMs on the same inputs: both within
    the bar of the oracle, and equal to each other up to fp32 summation order."""
    K, N, r = 1024, 768, 32
    lay = W.Layer("pair", M=M, K=K, N=N, r=r, variant=NVFP4, gelu=True, bias=True, config_id=63)
    pw = W.synthetic_packed(lay)
    x = W.activations(lay)
    hp = svdq.SVDQWeights(pw, M)
    hs = svdq.SVDQWeights(pw, M, single_sm=True)
    a = PT.gpu_forward(hp, x, M)
    b = PT.gpu_forward(hs, x, M)
    ref = O.linear_forward(x, pw)
    PT.check_y(a["Y"], ref["y"], ref["Y"], label=f"pair M{M}")
    PT.check_y(b["Y"], ref["y"], ref["Y"], label=f"1sm M{M}")
    ya = W.bf16_bits_to_f32(a["Y"]).astype(np.float64)
    yb = W.bf16_bits_to_f32(b["Y"]).astype(np.float64)
    assert np.linalg.norm(ya - yb) <= 1e-3 * np.linalg.norm(yb)


@pytest.mark.parametrize("M,K,N,r", [(300, 512, 448, 32), (1000, 1024, 768, 64)])
def test_int4_f16_and_int8_agree(M, K, N, r):
    """The two INT4 GEMMs compute the same sum of exact products: equal up to
    fp32 summation order."""
    lay = W.Layer("i4h", M=M, K=K, N=N, r=r, variant=INT4, gelu=True, bias=True, config_id=64)
    pw = W.synthetic_packed(lay)
    x = W.activations(lay)
    a = PT.gpu_forward(svdq.SVDQWeights(pw, M), x, M)
    b = PT.gpu_forward(svdq.SVDQWeights(pw, M, int4_f16=True), x, M)
    assert np.array_equal(a["codes"], b["codes"])
    ya = W.bf16_bits_to_f32(a["Y"]).astype(np.float64)
    yb = W.bf16_bits_to_f32(b["Y"]).astype(np.float64)
    assert np.linalg.norm(ya - yb) <= 1e-3 * np.linalg.norm(ya)


def test_int4_f16_range_errors():
    """Weights whose dequantised values are not fp16 values are refused at
    load; an activation scale above the fp16 bound is reported after the call."""
    import torch
    M, K, N, r = 256, 512, 256, 16
    lay = W.Layer("i4r", M=M, K=K, N=N, r=r, variant=INT4, config_id=65)
    pw = W.synthetic_packed(lay)
    big = copy.deepcopy(pw)
    big.scales = big.scales.copy()
    big.scales.reshape(-1)[5] = 0x4900          # bf16 2^19: 7 * 2^19 > 65504
    with pytest.raises(svdq.SvdqError) as e:
        svdq.SVDQWeights(big, M, int4_f16=True)
    assert "SVDQ_ERR_RANGE" in str(e.value)
    svdq.SVDQWeights(big, M).close()            # the int8 path takes any scale
    h = svdq.SVDQWeights(pw, M, int4_f16=True)
    x = W.bf16_bits_to_f32(W.activations(lay)).copy()
    x[7, :64] = 1.0e7                            # smoothed scale ~1e7 / (7 lambda) > 9357
    xd = PT.to_dev(W.to_bf16_bits(x).view(np.int16)).view(torch.bfloat16)
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    h.linear_forward(xd, y, M)
    torch.cuda.synchronize()
    assert h.device_status() == 8                # SVDQ_ERR_RANGE
    ok = PT.gpu_forward(h, W.activations(lay), M)
    assert h.device_status() == 0
    ref = O.linear_forward(W.activations(lay), pw)
    PT.check_y(ok["Y"], ref["y"], ref["Y"], label="after range error")


@pytest.mark.parametrize("opts", [{}, {"int4_f16": True}], ids=["int4", "int4-f16"])
def test_int4_weight_code_minus8(opts):
    """INT4 weight codes span the whole format, -8..7 (the amax/7 rule never
    produces -8, but the format and the load call accept it): the int8 unpack
    must sign-extend 0x8 to -8, and with fp16 operands -8 s must stay exact."""
    M, K, N, r = 300, 512, 528, 32
    lay = W.Layer("i4m8", M=M, K=K, N=N, r=r, variant=INT4, gelu=True, bias=True, config_id=67)
    pw = W.synthetic_packed(lay, int4_min=-8)
    nib = np.stack([pw.codes & 0xF, pw.codes >> 4], axis=-1)
    assert (nib == 8).sum() >= 100                   # -8 occurs (about 0.14% of codes)
    x = W.activations(lay)
    h = svdq.SVDQWeights(pw, M, **opts)
    got = PT.gpu_forward(h, x, M)
    ref = O.linear_forward(x, pw)
    PT.check_act(got, ref, r=r, label="int4 -8")
    PT.check_y(got["Y"], ref["y"], ref["Y"], label=f"int4 -8 {opts}")
    h.close()


@pytest.mark.parametrize("opts", [{}, {"single_sm": True}], ids=["nvfp4-pair", "nvfp4-1sm"])
@pytest.mark.parametrize("M,K,N,r", [(300, 512, 448, 32), (129, 1024, 272, 0)])
def test_nvfp4_tensor_scale(opts, M, K, N, r):
    """NVFP4 weights with a per-tensor second-level scale 2^e (e < 0 for these
    residuals): the GEMM scales its accumulator by 2^e and T by 2^-e; Y within
    the bars of the oracle, whose weights dequantise to q s 2^e."""
    lay, x, _ = _prepped(M, K, N, r, NVFP4, gelu=True, with_bias=True, cid=68)
    pw = P.prepare(x, W.weight(lay), r, NVFP4, bias_bits=W.bias(lay), gelu=True, tensor_scale=True)
    assert pw.w_scale_exp < 0
    h = svdq.SVDQWeights(pw, M, **opts)
    got = PT.gpu_forward(h, x, M)
    ref = O.linear_forward(x, pw)
    PT.check_act(got, ref, r=r, label="tensor scale")
    PT.check_y(got["Y"], ref["y"], ref["Y"], label=f"tensor scale e{pw.w_scale_exp} {opts}")
    h.close()


def test_handles_loaded_from_two_threads():
    """Two threads load handles and run the layer at the same time (first
    calls race on the per-device shared-memory opt-in); both results equal a
    single-threaded run."""
    import threading
    import torch
    M, K, N, r = 256, 512, 512, 32
    cases = []
    for i, variant in enumerate((NVFP4, INT4)):
        lay = W.Layer("thr", M=M, K=K, N=N, r=r, variant=variant, config_id=69, layer_id=i)
        cases.append((lay, W.synthetic_packed(lay), W.activations(lay)))
    ref = []
    for lay, pw, x in cases:
        h = svdq.SVDQWeights(pw, M)
        h.set_deterministic()
        ref.append(PT.gpu_forward(h, x, M)["Y"])
        h.close()
    out = [None, None]
    err = []

    def work(i):
        try:
            torch.cuda.set_device(0)
            lay, pw, x = cases[i]
            s = torch.cuda.Stream()
            with torch.cuda.stream(s):
                h = svdq.SVDQWeights(pw, M)
                h.set_deterministic()
                out[i] = PT.gpu_forward(h, x, M)["Y"]
                h.close()
        except Exception as e:  # reported below
            err.append(e)

    th = [threading.Thread(target=work, args=(i,)) for i in range(2)]
    for t in th:
        t.start()
    for t in th:
        t.join()
    assert not err, err
    for i in range(2):
        assert np.array_equal(out[i], ref[i])


@pytest.mark.parametrize("variant", [NVFP4, INT4])
def test_split_t_reduction_modes(variant):
    """Kernel 1's split partial T tiles added into T with fp32 reductions (the
    default) against the fixed-order sum (svdq_set_deterministic): codes and
    scales identical, T within the fp32 accumulation bound of the oracle's
    exact T, and the deterministic mode repeats its bits."""
    import torch
    M, K, N, r = 1000, 3072, 512, 32   # 8 row blocks: the K range is split
    lay = W.Layer("tsum", M=M, K=K, N=N, r=r, variant=variant, config_id=70)
    pw = W.synthetic_packed(lay)
    x = W.activations(lay)
    h = svdq.SVDQWeights(pw, M)
    fast = PT.gpu_forward(h, x, M)
    h.set_deterministic()
    det1 = PT.gpu_forward(h, x, M)
    det2 = PT.gpu_forward(h, x, M)
    h.set_deterministic(False)
    fast2 = PT.gpu_forward(h, x, M)
    h.close()
    assert np.array_equal(fast["codes"], det1["codes"]) and np.array_equal(fast["scales"], det1["scales"])
    assert np.array_equal(det1["T"], det2["T"]) and np.array_equal(det1["Y"], det2["Y"])
    xp = O.smooth_activations(x, (np.float32(1) / pw.lam).astype(np.float32)).astype(np.float64)
    l1 = W.bf16_bits_to_f32(pw.L1).astype(np.float64)
    tb = PT.t_bound(xp, l1)
    texact = xp @ l1
    for got, label in ((fast, "reductions"), (det1, "fixed order"), (fast2, "reductions again")):
        d = float(np.linalg.norm(got["T"].astype(np.float64) - texact))
        PT.record(f"T {label} v{variant}", "||dT|| / fp32 bound", d / tb, 1.0)
        assert d <= tb, (label, d, tb)
