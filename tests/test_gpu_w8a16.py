"""GPU parity of the W8A16 path (8-bit codes, one per byte) against the oracle.

Codes, scales, zeros and the dequantized weights are integer or once-rounded
results and must match the oracle's bytes exactly; the fused GEMM (the GEMV for
M ≤ 16, the tensor-core kernel above) must meet the same bars as the INT4 GEMM
(tests/helpers.py), and is bit-exact on one-hot activations."""
import numpy as np
import pytest
import torch

import oracle
import workloads
import weight_only_quantization_rtn_b200 as w4
from weight_only_quantization_rtn_b200 import build as w4build
from helpers import assert_y_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    w4build.build()
    oracle.build()
    yield
    assert w4.device_error() == 0


def _quantize_and_compare(Wc: torch.Tensor, g: int, sym: bool):
    C, S, Z = w4.quantize8(Wc.cuda(), g, sym)
    Wh = w4.dequantize8(C, S, Z, g, sym)
    torch.cuda.synchronize()
    rC, rS, rZ = oracle.quantize8(workloads.bits(Wc), g, sym)
    assert np.array_equal(C.cpu().numpy(), rC), "codes differ"
    assert np.array_equal(workloads.bits(S), rS), "scales differ"
    assert np.array_equal(workloads.bits(Z), rZ), "zeros differ"
    rWh = oracle.dequantize8(rC, rS, rZ, g, sym)
    assert np.array_equal(workloads.bits(Wh), rWh), "dequantized weights differ"
    return C, S, Z


@pytest.mark.parametrize("sym", [False, True])
@pytest.mark.parametrize("g", [32, 64, 128, 0])          # 0: per-channel, g = K
@pytest.mark.parametrize("N,K", [(1, 128), (7, 384), (33, 256), (130, 1152), (517, 640),
                                 (1500, 256)])
def test_w8_quantize_bit_exact(N, K, g, sym):
    gg = K if g == 0 else g
    if K % gg:
        pytest.skip("K not a multiple of g")
    W = workloads.make_weight(N, K, 0.02, seed=N * 5 + K + g, outlier_frac=0.02,
                              outlier_scale=20.0)
    _quantize_and_compare(W, gg, sym)


@pytest.mark.parametrize("sym", [False, True])
@pytest.mark.parametrize("g", [32, 128, 160])            # 160 = K: per-channel
def test_w8_degenerate_groups(g, sym):
    K = 4 * g if g != 160 else 160
    rows = [np.zeros(K),
            np.abs(np.random.default_rng(1).standard_normal(K)) + 0.5,
            -np.abs(np.random.default_rng(2).standard_normal(K)) - 0.5,
            np.full(K, 0.375),
            np.tile([-4.0, 0.03125, 0.09375, -0.15625, 1.28125, 11.9375, 0.0, 0.0], K // 8),
            np.random.default_rng(3).standard_normal(K) * 2.0 ** 100,
            np.random.default_rng(4).standard_normal(K) * 2.0 ** -100,
            np.random.default_rng(5).standard_normal(K) * 1e-39]
    W = torch.tensor(np.stack(rows), dtype=torch.float32).to(torch.bfloat16)
    _quantize_and_compare(W, g, sym)


@pytest.mark.parametrize("sym", [False, True])
@pytest.mark.parametrize("li", [0, 1])
def test_w8_7b_shaped_matrices_bit_exact(li, sym):
    layer = workloads.DECODE_7B.layers[li]
    _quantize_and_compare(layer.weight(), 128, sym)


def _check_gemm(M, N, K, g, sym, seed):
    W = workloads.make_weight(N, K, 0.02, seed, outlier_frac=0.01, outlier_scale=20.0)
    C, S, Z = w4.quantize8(W.cuda(), g, sym)
    X = workloads.make_activation(M, K, seed + 1, outlier_frac=0.01, outlier_mode="set")
    Y = w4.gemm8(X.cuda(), C, S, Z, g, sym)
    torch.cuda.synchronize()
    ref = oracle.gemm_w8a16(workloads.bits(X), C.cpu().numpy(), workloads.bits(S),
                            workloads.bits(Z), g, sym)
    assert_y_close(workloads.bits(Y), ref, f"W8 M={M} N={N} K={K} g={g} sym={sym}")


@pytest.mark.parametrize("sym", [False, True])
@pytest.mark.parametrize("g", [32, 64, 128, 0])
@pytest.mark.parametrize("M,N,K", [(1, 256, 256), (1, 1, 128), (2, 37, 384), (3, 100, 1152),
                                   (5, 64, 224), (8, 128, 4096), (13, 257, 1024),
                                   (16, 512, 2048)])
def test_w8_gemm_small(M, N, K, g, sym):
    gg = K if g == 0 else g
    if K % gg:
        pytest.skip("K not a multiple of g")
    _check_gemm(M, N, K, gg, sym, seed=M + N + K)


@pytest.mark.parametrize("sym", [False, True])
@pytest.mark.parametrize("g", [32, 128, 512])             # 512 = K: per-channel
def test_w8_one_hot_activations_select_dequantized_weights_bit_exact(g, sym):
    N, K = 160, 512
    W = workloads.make_weight(N, K, 0.02, seed=17)
    C, S, Z = w4.quantize8(W.cuda(), g, sym)
    Wh = w4.dequantize8(C, S, Z, g, sym)
    for start in range(0, K, 16):
        kk = torch.arange(start, start + 16)
        X = torch.zeros(16, K, dtype=torch.bfloat16)
        X[torch.arange(16), kk] = 1.0
        Y = w4.gemm8(X.cuda(), C, S, Z, g, sym)
        assert torch.equal(Y, Wh[:, kk.cuda()].t().contiguous()), f"k in {start}..{start + 15}"


def test_w8_gemm_deterministic_and_7b_full_size():
    layer = workloads.DECODE_7B.layers[1]                 # K = 11008, N = 4096
    W = layer.weight()
    C, S, Z = w4.quantize8(W.cuda(), 128, False)
    X = layer.activation(4)
    ys = [w4.gemm8(X.cuda(), C, S, Z, 128, False) for _ in range(3)]
    assert all(torch.equal(ys[0], y) for y in ys[1:])
    rng = np.random.default_rng(7)
    ms = rng.integers(0, 4, 2048)
    ns = rng.integers(0, layer.N, 2048)
    ms[:4], ns[:4] = [0, 3, 0, 3], [0, 0, layer.N - 1, layer.N - 1]
    ref = oracle.gemm_w8a16_sampled(workloads.bits(X), C.cpu().numpy(), workloads.bits(S),
                                    workloads.bits(Z), 128, False, ms, ns)
    assert_y_close(workloads.bits(ys[0])[ms, ns], ref, "W8 7B-shaped layer M=4")


@pytest.mark.parametrize("sym", [False, True])
@pytest.mark.parametrize("M", [1, 9, 16])
def test_w8_forced_paths_agree_with_the_oracle(M, sym):
    """w8a16_gemm_ex: the decode and tensor-core kernels both run M <= 16 and both
    match the oracle; the static-weights flag changes no bit."""
    N, K, g = 700, 2304, 64
    W = workloads.make_weight(N, K, 0.02, 31, outlier_frac=0.01, outlier_scale=20.0)
    C, S, Z = w4.quantize8(W.cuda(), g, sym)
    X = workloads.make_activation(M, K, 32, outlier_frac=0.01, outlier_mode="set")
    ref = oracle.gemm_w8a16(workloads.bits(X), C.cpu().numpy(), workloads.bits(S),
                            workloads.bits(Z), g, sym)
    ys = {}
    for path in ("decode", "tensorcore"):
        ys[path] = w4.gemm8(X.cuda(), C, S, Z, g, sym, path=path)
        torch.cuda.synchronize()
        assert_y_close(workloads.bits(ys[path]), ref, f"W8 {path} M={M} sym={sym}")
    Yst = w4.gemm8(X.cuda(), C, S, Z, g, sym, path="decode", static_weights=True)
    assert torch.equal(Yst, ys["decode"])


@pytest.mark.parametrize("sym", [False, True])
@pytest.mark.parametrize("li", [0, 1])
def test_w8_decode_70b_full_size(li, sym):
    """The decode kernel with 8-bit codes on a 70B-shaped layer (M=1; the stream-K
    partition splits row blocks between CTAs), on sampled outputs including the
    last row."""
    layer = workloads.DECODE_70B.layers[li]
    W, X = layer.weight(), layer.activation(1)
    C, S, Z = w4.quantize8(W.cuda(), 128, sym)
    Y = w4.gemm8(X.cuda(), C, S, Z, 128, sym)
    torch.cuda.synchronize()
    rng = np.random.default_rng(13 + li)
    ns = rng.integers(0, layer.N, 1024)
    ns[:2] = [0, layer.N - 1]
    ms = np.zeros_like(ns)
    ref = oracle.gemm_w8a16_sampled(workloads.bits(X), C.cpu().numpy(), workloads.bits(S),
                                    workloads.bits(Z), 128, sym, ms, ns)
    assert_y_close(workloads.bits(Y)[ms, ns], ref, f"W8 70B-shaped layer {li} sym={sym}")
    assert w4.device_error() == 0


@pytest.mark.parametrize("sym", [False, True])
@pytest.mark.parametrize("g", [32, 64, 128, 0])
@pytest.mark.parametrize("M,N,K", [(17, 128, 96), (33, 384, 512), (48, 1000, 4352),
                                   (129, 64, 4096), (300, 700, 1056), (600, 1000, 1024)])
def test_w8_gemm_tensorcore(M, N, K, g, sym):
    """M > 16: the tensor-core kernel with 8-bit codes (64-byte code rows per K
    block, 64-byte swizzle), unsplit and split-K tiles, ragged N, M and K."""
    gg = K if g == 0 else g
    if K % gg:
        pytest.skip("K not a multiple of g")
    _check_gemm(M, N, K, gg, sym, seed=3 * M + N + K)


@pytest.mark.parametrize("sym", [False, True])
@pytest.mark.parametrize("g", [32, 128, 512])
def test_w8_tensorcore_one_hot_bit_exact(g, sym):
    """32 one-hot activation rows (M > 16, so the tensor-core kernel): each output
    is one dequantized weight, exactly."""
    N, K = 160, 512
    W = workloads.make_weight(N, K, 0.02, seed=23)
    C, S, Z = w4.quantize8(W.cuda(), g, sym)
    Wh = w4.dequantize8(C, S, Z, g, sym)
    for start in range(0, K, 32):
        kk = torch.arange(start, start + 32)
        X = torch.zeros(32, K, dtype=torch.bfloat16)
        X[torch.arange(32), kk] = 1.0
        Y = w4.gemm8(X.cuda(), C, S, Z, g, sym)
        assert torch.equal(Y, Wh[:, kk.cuda()].t().contiguous()), f"k in {start}..{start + 31}"


def test_w8_prefill_full_size():
    layer = workloads.PREFILL.layers[0]                   # M=2048, K=N=8192
    W, X = layer.weight(), layer.activation(2048)
    C, S, Z = w4.quantize8(W.cuda(), 128, False)
    ys = [w4.gemm8(X.cuda(), C, S, Z, 128, False) for _ in range(2)]
    assert torch.equal(ys[0], ys[1])
    rng = np.random.default_rng(11)
    ms = rng.integers(0, 2048, 2048)
    ns = rng.integers(0, layer.N, 2048)
    ms[:4], ns[:4] = [0, 2047, 0, 2047], [0, 0, layer.N - 1, layer.N - 1]
    ref = oracle.gemm_w8a16_sampled(workloads.bits(X), C.cpu().numpy(), workloads.bits(S),
                                    workloads.bits(Z), 128, False, ms, ns)
    assert_y_close(workloads.bits(ys[0])[ms, ns], ref, "W8 prefill M=2048")
