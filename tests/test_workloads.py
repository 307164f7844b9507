"""Seeded input generators: determinism, shapes and distributions (CPU)."""
import numpy as np

from bit_diffusion_transformer_w4a4_b200 import workloads as W


def test_all_workloads_defined():
    wl = W.workloads()
    assert set(["tiny", "qkv_int4", "fc1_nvfp4", "fc2_nvfp4", "block_2048px"]) <= set(wl)
    assert sum(k.startswith("sweep_") for k in wl) == 10
    fc1 = wl["fc1_nvfp4"][0]
    assert (fc1.M, fc1.K, fc1.N, fc1.r, fc1.variant, fc1.gelu) == (4608, 3072, 12288, 32, W.NVFP4, True)
    assert [l.N for l in wl["block_2048px"]] == [9216, 3072, 12288, 3072]
    assert wl["tiny"][0].outlier_count() == 4 and wl["qkv_int4"][0].outlier_count() == 31


def test_determinism_and_outliers():
    lay = W.Layer("t", M=64, K=256, N=128, r=16, variant=W.INT4, n_outliers=4, config_id=1)
    a, b = W.activations(lay), W.activations(lay)
    assert a.dtype == np.uint16 and np.array_equal(a, b)
    x = W.bf16_bits_to_f32(a)
    oc = W.outlier_channels(lay)
    assert len(oc) == 4
    rest = np.setdiff1d(np.arange(256), oc)
    assert 10 < np.abs(x[:, oc]).std() / np.abs(x[:, rest]).std() < 40
    w = W.weight(lay)
    assert np.array_equal(W.bf16_bits_to_f32(W.to_bf16_bits(w)), w)   # on the bf16 grid
    assert abs(w[rest].std() - 0.02) < 0.002


def test_synthetic_packed_shapes():
    for v in (W.INT4, W.NVFP4):
        lay = W.Layer("t", M=128, K=256, N=64, r=32, variant=v, config_id=9)
        pw = W.synthetic_packed(lay)
        G = W.GROUP[v]
        assert pw.codes.shape == (64, 128) and pw.codes.dtype == np.uint8
        assert pw.scales.shape == (64, 256 // G)
        assert pw.L1.shape == (256, 32) and pw.L2.shape == (32, 64)
        assert pw.lam.dtype == np.float32 and np.all(pw.lam > 0)


def test_qkv_epilogue_inputs():
    gq, gk, rope = W.qkv_epilogue_inputs(300)
    assert gq.dtype == np.uint16 and gq.shape == (128,) and not np.array_equal(gq, gk)
    g = W.bf16_bits_to_f32(gq)
    assert 0.3 < g.min() and g.max() < 1.8
    assert rope.shape == (300, 128) and rope.dtype == np.float32
    c, s = rope[:, 0::2].astype(np.float64), rope[:, 1::2].astype(np.float64)
    assert np.abs(c * c + s * s - 1).max() < 1e-6
    # token 65 sits at grid (1, 1): pair 0 turns by 1 radian, pair 32 too
    assert abs(c[65, 0] - np.cos(1.0)) < 1e-7 and abs(s[65, 32] - np.sin(1.0)) < 1e-7
    assert np.all(c[0] == 1) and np.all(s[0] == 0)
    assert np.array_equal(W.qkv_epilogue_inputs(300)[2], rope)
