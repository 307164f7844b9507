"""GPU parity of the AWQ W4A16 linear (through the C ABI) against the CPU
oracle: ragged N, every token-block width, K from one group to 12288,
with and without bias, weights from the oracle's own AWQ preparation and
synthetic bit patterns (zero points across 0..15, codes 0 and 15)."""
import numpy as np
import pytest

from bit_diffusion_transformer_w4a4_b200 import svdq
from bit_diffusion_transformer_w4a4_b200 import workloads as W
from oracle import awq as A
import parity as PT

pytestmark = pytest.mark.gpu


def _run(p, x_bits, M, N):
    import torch
    h = svdq.AWQWeights(p, M)
    x = PT.to_dev(x_bits.view(np.int16)).view(torch.bfloat16)
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    y.fill_(float("nan"))
    h.forward(x, y, M)
    torch.cuda.synchronize()
    h.close()
    return PT.from_dev(y.view(torch.int16)).view(np.uint16)


@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 8, 9, 17])
@pytest.mark.parametrize("K,N", [(64, 40), (3072, 1000), (1024, 3077)])
@pytest.mark.parametrize("with_bias", [False, True])
def test_awq_prepared(M, K, N, with_bias):
    lay = W.AWQLayer("t", M=M, K=K, N=N, bias=with_bias, config_id=91, layer_id=K // 64 + N)
    x = W.awq_activations(lay)
    w = W.awq_weight(lay)
    bias = W.synthetic_awq(lay).bias if with_bias else None
    p = A.prepare(x, w, bias_bits=bias)
    Y = _run(p, x, M, N)
    y, Yr = A.forward(x, p)
    PT.check_y(Y, y, Yr, label=f"awq M{M} K{K} N{N} b{int(with_bias)}")


@pytest.mark.parametrize("name", list(W.awq_workloads()))
def test_awq_workload_full_size(name):
    lay = W.awq_workloads()[name]
    p = W.synthetic_awq(lay)
    p.zeros[0, :] = 0                       # extreme zero points
    p.zeros[1, :] = 15
    x = W.awq_activations(lay)
    Y = _run(p, x, lay.M, lay.N)
    y, Yr = A.forward(x, p)
    PT.check_y(Y, y, Yr, label=f"awq {name}")


def test_awq_large_K():
    lay = W.AWQLayer("kbig", M=2, K=12288, N=3072, config_id=92)
    p = W.synthetic_awq(lay)
    x = W.awq_activations(lay)
    Y = _run(p, x, lay.M, lay.N)
    y, Yr = A.forward(x, p)
    PT.check_y(Y, y, Yr, label="awq K12288")
