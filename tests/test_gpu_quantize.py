"""GPU parity of quantize/pack and dequantize: bit-exact against the oracle.

Packed codes, scales and zeros are integer or once-rounded results, so the
CUDA path must reproduce the oracle's bytes exactly, on every shape, group
size and mode, including ragged and degenerate inputs and the full-size
workload matrices."""
import numpy as np
import pytest
import torch

import oracle
import workloads
import weight_only_quantization_rtn_b200 as w4
from weight_only_quantization_rtn_b200 import build as w4build

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    w4build.build()
    oracle.build()
    yield
    assert w4.device_error() == 0


def _run_and_compare(Wc: torch.Tensor, g: int, sym: bool):
    W = Wc.cuda()
    P, S, Z = w4.quantize(W, g, sym)
    Wh = w4.dequantize(P, S, Z, g, sym)
    torch.cuda.synchronize()
    Wb = workloads.bits(Wc)
    rP, rS, rZ = oracle.quantize(Wb, g, sym)
    assert np.array_equal(P.cpu().numpy(), rP), "packed codes differ"
    assert np.array_equal(workloads.bits(S), rS), "scales differ"
    assert np.array_equal(workloads.bits(Z), rZ), "zeros differ"
    rWh = oracle.dequantize(rP, rS, rZ, Wc.shape[1], g, sym)
    assert np.array_equal(workloads.bits(Wh), rWh), "dequantized weights differ"


@pytest.mark.parametrize("sym", [False, True])
@pytest.mark.parametrize("g", [32, 64, 128])
@pytest.mark.parametrize("N,K", [(1, 128), (7, 384), (33, 256), (256, 256), (130, 1152),
                                 (517, 640)])
def test_quantize_bit_exact_small(N, K, g, sym):
    if K % g:
        pytest.skip("K not a multiple of g")
    W = workloads.make_weight(N, K, 0.02, seed=N * 7 + K + g, outlier_frac=0.02,
                              outlier_scale=20.0)
    _run_and_compare(W, g, sym)


def test_tiny_config_bit_exact():
    layer = workloads.TINY.layers[0]
    _run_and_compare(layer.weight(), 128, False)


def _degenerate_rows(K):
    rows = []
    rows.append(np.zeros(K))                                      # all zero: s = 0
    rows.append(np.abs(np.random.default_rng(1).standard_normal(K)) + 0.5)   # all positive
    rows.append(-np.abs(np.random.default_rng(2).standard_normal(K)) - 0.5)  # all negative
    rows.append(np.full(K, 0.375))                                # constant
    r = np.zeros(K)
    r[5] = -2.5
    rows.append(r)                                                # one nonzero
    t = np.tile([-0.625, 0.375, 0.0, 3.125], K // 4)              # ties under s = 0.25
    rows.append(t)
    rows.append(np.random.default_rng(3).standard_normal(K) * 2.0 ** 100)
    rows.append(np.random.default_rng(4).standard_normal(K) * 2.0 ** -100)
    rows.append(np.random.default_rng(5).standard_normal(K) * 1e-39)      # bf16 subnormals
    return torch.tensor(np.stack(rows), dtype=torch.float32).to(torch.bfloat16)


@pytest.mark.parametrize("sym", [False, True])
@pytest.mark.parametrize("g", [32, 128, 160])     # 160 = K: per-channel
def test_degenerate_groups(g, sym):
    """All-zero groups, one-sided groups, constant groups, exact ties, huge and
    tiny magnitudes, a single nonzero element."""
    K = 4 * g if g != 160 else 160
    _run_and_compare(_degenerate_rows(K), g, sym)


# ------------------------------------------------------------------ per-channel (g = K)
@pytest.mark.parametrize("sym", [False, True])
@pytest.mark.parametrize("N,K", [(1, 160), (7, 96), (33, 416), (130, 4096), (517, 1056),
                                 (64, 11008), (1500, 256)])
def test_per_channel_bit_exact(N, K, sym):
    """g = K: one scale and zero per row (a block-wide range reduction per row);
    1500 rows exceed the row kernel's grid, so CTAs loop over rows."""
    W = workloads.make_weight(N, K, 0.02, seed=N + 3 * K, outlier_frac=0.02, outlier_scale=20.0)
    _run_and_compare(W, K, sym)


@pytest.mark.parametrize("sym", [False, True])
@pytest.mark.parametrize("layer_idx", [0, 1])
def test_per_channel_7b_shaped_bit_exact(layer_idx, sym):
    layer = workloads.DECODE_7B.layers[layer_idx]
    _run_and_compare(layer.weight(), layer.K, sym)


@pytest.mark.parametrize("layer_idx", [0, 1])
def test_7b_shaped_matrices_bit_exact(layer_idx):
    layer = workloads.DECODE_7B.layers[layer_idx]
    _run_and_compare(layer.weight(), 128, False)


@pytest.mark.parametrize("sym", [False, True])
@pytest.mark.parametrize("layer_idx", [0, 1])
def test_70b_shaped_matrices_bit_exact(layer_idx, sym):
    layer = workloads.DECODE_70B.layers[layer_idx]
    _run_and_compare(layer.weight(), 128, sym)


@pytest.mark.parametrize("sym", [False, True])
@pytest.mark.parametrize("g", [32, 64, 128])
def test_crossover_matrix_bit_exact(g, sym):
    layer = workloads.CROSSOVER.layers[0]
    _run_and_compare(layer.weight(), g, sym)


def test_quantize_is_deterministic_and_stream_ordered():
    W = workloads.make_weight(300, 1024, 0.02, seed=77).cuda()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        a = w4.quantize(W, 64, False)
        b = w4.quantize(W, 64, False)
    s.synchronize()
    for x, y in zip(a, b):
        assert torch.equal(x, y)
