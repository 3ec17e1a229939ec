"""GPU parity of the GEMM with a per-input-channel activation scale
(w4a16_gemm_act_scaled): Y = X'·Ŵᵀ with X'[m, k] = bf16_rn(X[m, k]·a[k]), the
activation half of the equivalent scaling of "推理优化中“用精度换性能“的核心技术：
量化", §5.2 and §6.2.  Compared with the oracle's gemm_w4a16_act_scaled (the
oracle's scale_activations, then its binary64 matmul) under the GEMM tolerance of
the other parity tests, through both kernels (M ≤ 16 runs the decode kernel,
whose helper warp scales X; larger M the tensor-core kernel, whose dequantizing
warps scale the X tile); bit-exact where the result is exact."""
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


def _case(M, N, K, g, sym, seed):
    W = workloads.make_weight(N, K, 0.02, seed, outlier_frac=0.01, outlier_scale=20.0)
    P, S, Z = w4.quantize(W.cuda(), g, sym)
    X = workloads.make_activation(M, K, seed + 1, outlier_frac=0.01, outlier_mode="set")
    a = workloads.make_act_scale(K, seed + 2)
    return P, S, Z, X, a


SHAPES = [(1, 256, 256), (2, 37, 384), (3, 100, 1152), (8, 128, 4096), (13, 257, 1024),
          (16, 512, 2048), (17, 200, 256), (64, 129, 640), (200, 384, 2048), (300, 130, 1024)]


@pytest.mark.parametrize("sym", [False, True])
@pytest.mark.parametrize("g", [32, 128, 0])          # 0: per-channel (g = K)
@pytest.mark.parametrize("M,N,K", SHAPES)
def test_act_scaled_matches_oracle(M, N, K, g, sym):
    g = K if g == 0 else g
    if K % g:
        pytest.skip("K not a multiple of g")
    P, S, Z, X, a = _case(M, N, K, g, sym, seed=M + 2 * N + K)
    Y = w4.gemm(X.cuda(), P, S, Z, g, sym, act_scale=a.cuda())
    torch.cuda.synchronize()
    Y64 = oracle.gemm_w4a16_act_scaled(workloads.bits(X), workloads.bits(a), P.cpu().numpy(),
                                       workloads.bits(S), workloads.bits(Z), g, sym)
    assert_y_close(workloads.bits(Y), Y64, f"M={M} N={N} K={K} g={g} sym={sym}")


@pytest.mark.parametrize("M", [1, 12, 48, 256])
def test_unit_scale_is_the_plain_gemm(M):
    """a = 1: x·1 = x exactly, so the result is bit-identical to w4a16_gemm."""
    N, K, g = 300, 2048, 128
    P, S, Z, X, _ = _case(M, N, K, g, False, seed=7 + M)
    ones = torch.ones(K, dtype=torch.bfloat16, device="cuda")
    Xd = X.cuda()
    assert torch.equal(w4.gemm(Xd, P, S, Z, g, False, act_scale=ones), w4.gemm(Xd, P, S, Z, g, False))


@pytest.mark.parametrize("M", [16, 32])              # decode kernel, tensor-core kernel
@pytest.mark.parametrize("sym", [False, True])
def test_one_hot_power_of_two_scale_is_exact(M, sym):
    """X one-hot and a[k] a power of two: Y[m, n] = Ŵ[n, k_m]·a[k_m] exactly (one
    nonzero product, scaled by a power of two), checked bit for bit."""
    N, K, g = 160, 512, 64
    P, S, Z, _, _ = _case(1, N, K, g, sym, seed=21)
    Wh = w4.dequantize(P, S, Z, g, sym).float()
    e = torch.randint(-3, 4, (K,), generator=torch.Generator().manual_seed(5))
    a = torch.exp2(e.float()).to(torch.bfloat16)
    for start in range(0, K, M):
        ks = torch.arange(start, min(start + M, K))
        X = torch.zeros(M, K, dtype=torch.bfloat16)
        X[torch.arange(ks.numel()), ks] = 1.0
        Y = w4.gemm(X.cuda(), P, S, Z, g, sym, act_scale=a.cuda())
        ref = (Wh[:, ks.cuda()] * a.float().cuda()[ks.cuda()]).t().to(torch.bfloat16)
        assert torch.equal(Y[:ks.numel()], ref), f"k in {start}..{start + M - 1}"


def test_act_scaled_full_size_sampled():
    """A 70B-shaped layer at M=1 (decode kernel) and the prefill shape (tensor
    cores, split tail) on sampled outputs the oracle computes one by one."""
    for (M, N, K) in ((1, 28672, 8192), (2048, 8192, 8192)):
        P, S, Z, X, a = _case(M, N, K, 128, False, seed=31)
        Y = w4.gemm(X.cuda(), P, S, Z, 128, False, act_scale=a.cuda())
        torch.cuda.synchronize()
        rng = np.random.default_rng(M)
        ms = rng.integers(0, M, 1024)
        ns = rng.integers(0, N, 1024)
        ms[:2], ns[:2] = [0, M - 1], [0, N - 1]
        Xs = oracle.scale_activations(workloads.bits(X), workloads.bits(a))
        y64 = oracle.gemm_sampled(Xs, P.cpu().numpy(), workloads.bits(S), workloads.bits(Z), 128,
                                  False, ms, ns)
        yb = workloads.bits(Y)[ms, ns]
        assert_y_close(yb, y64, f"M={M} N={N} K={K}")


def test_deterministic():
    P, S, Z, X, a = _case(8, 1000, 4096, 128, False, seed=3)
    Xd, ad = X.cuda(), a.cuda()
    ys = [w4.gemm(Xd, P, S, Z, 128, False, act_scale=ad) for _ in range(3)]
    assert all(torch.equal(ys[0], y) for y in ys[1:])
