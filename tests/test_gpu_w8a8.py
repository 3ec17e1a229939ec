"""W8A8 on the GPU against the oracle: per-token INT8 activations bit-exact
(codes and binary32 scales), the INT8 tensor-core GEMM within the GEMM
tolerance of the other parity tests (the exact integer sum times the two
scales, rounded to bf16)."""
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
    w4.lib()


def _acts(M, K, seed):
    X = workloads.make_activation(M, K, seed, outlier_frac=0.01, outlier_mode="set")
    if M > 2:
        X[2] = 0.0                                         # an all-zero token
    if M > 1:
        X[1] *= 2.0 ** -40                                 # a tiny-magnitude token
    return X


# K = 8192 fills the four register chunks per thread exactly; 8224, 11008 and
# 28672 run the sixteen-chunk kernel with a ragged last chunk set; 32800 is
# past the register cache (the row is read twice).
@pytest.mark.parametrize("M,K", [(1, 32), (5, 96), (7, 4096), (300, 1056), (2, 11008), (64, 256),
                                 (3, 8192), (4, 8224), (3, 28672), (3, 32768), (3, 32800)])
def test_quantize_act8_bit_exact(M, K):
    X = _acts(M, K, seed=M + K)
    q, s = w4.quantize_act8(X.cuda())
    torch.cuda.synchronize()
    q_ref, s_ref = oracle.quantize_act8(workloads.bits(X))
    assert np.array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    assert np.array_equal(q.cpu().numpy(), q_ref)


def _weights(N, K, seed):
    W = workloads.make_weight(N, K, 0.02, seed, outlier_frac=0.01, outlier_scale=20.0)
    C, S, _ = w4.quantize8(W.cuda(), K, True)               # symmetric, one scale per row
    return C, S


@pytest.mark.parametrize("M", [1, 3, 64, 65, 128, 129, 256, 300])
@pytest.mark.parametrize("N,K", [(100, 32), (257, 1056), (1, 96), (384, 4096)])
def test_w8a8_gemm_small(M, N, K):
    X = _acts(M, K, seed=M + N)
    C, S = _weights(N, K, seed=N + K)
    qx, sx = w4.quantize_act8(X.cuda())
    Y = w4.gemm_w8a8(qx, sx, C, S)
    torch.cuda.synchronize()
    q_ref, s_ref = oracle.quantize_act8(workloads.bits(X))
    Y64 = oracle.gemm_w8a8(q_ref, s_ref, C.cpu().numpy(), workloads.bits(S))
    assert_y_close(workloads.bits(Y), Y64, f"W8A8 M={M} N={N} K={K}")


def test_w8a8_one_hot_tokens():
    """One-hot tokens: each output is 127·q_w[n, k]·s_w[n]·s_x[m], so every code
    of a weight column shows up in Y."""
    N, K = 160, 512
    C, S = _weights(N, K, seed=17)
    X = torch.zeros(64, K, dtype=torch.bfloat16)
    kk = torch.arange(64) * 7 % K
    X[torch.arange(64), kk] = torch.linspace(-3.0, 3.0, 64).to(torch.bfloat16) + 0.25
    Y = w4.linear_w8a8(X.cuda(), C, S)
    torch.cuda.synchronize()
    Y64 = oracle.gemm_w8a8_from_bf16(workloads.bits(X), C.cpu().numpy(), workloads.bits(S))
    assert_y_close(workloads.bits(Y), Y64, "W8A8 one-hot tokens")


def test_w8a8_deterministic_and_prefill_full_size():
    layer = workloads.PREFILL.layers[0]                     # M=2048, K=N=8192
    W, X = layer.weight(), layer.activation(2048)
    C, S = w4.quantize8(W.cuda(), layer.K, True)[:2]
    Xd = X.cuda()
    ys = [w4.linear_w8a8(Xd, C, S) for _ in range(2)]
    torch.cuda.synchronize()
    assert torch.equal(ys[0], ys[1])
    q_ref, s_ref = oracle.quantize_act8(workloads.bits(X))
    qx, sx = w4.quantize_act8(Xd)
    assert np.array_equal(qx.cpu().numpy(), q_ref)
    rng = np.random.default_rng(11)
    ms = rng.integers(0, 2048, 2048)
    ns = rng.integers(0, layer.N, 2048)
    ms[:4], ns[:4] = [0, 2047, 0, 2047], [0, 0, layer.N - 1, layer.N - 1]
    ref = oracle.gemm_w8a8_sampled(q_ref, s_ref, C.cpu().numpy(), workloads.bits(S), ms, ns)
    assert_y_close(workloads.bits(ys[0])[ms, ns], ref, "W8A8 prefill M=2048")
    assert w4.device_error() == 0
