"""GPU parity of the fused W4A16 GEMM against the oracle.

Y is compared with the oracle's binary64 matmul Y64 over the dequantized
weights: max|Y − Y64| ≤ 4e-3·max|Y64| and ‖Y − bf16(Y64)‖_F ≤ 1e-3·‖bf16(Y64)‖_F
(tests/helpers.py explains which reference each bar uses).  Where a result is exact (one-hot activations
select single dequantized weights) the comparison is bit-exact.  Both kernels
(decode and tensor-core) are forced at the same shapes; the full-size
workloads run in the launch configuration the benchmark times and are checked
on sampled outputs the oracle computes one by one."""
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


def _quantized(N, K, g, sym, seed, outlier=True):
    W = workloads.make_weight(N, K, 0.02, seed, outlier_frac=0.01 if outlier else 0.0,
                              outlier_scale=20.0)
    Wd = W.cuda()
    P, S, Z = w4.quantize(Wd, g, sym)
    return P, S, Z


def _assert_quantized_like_oracle(W, P, S, Z, g, sym, what=""):
    """The GPU's packed codes, scales and zeros equal the oracle's quantization of
    the same W bit for bit, so a GEMM check against the oracle runs end to end
    from W (the reference below uses the oracle's own codes)."""
    rP, rS, rZ = oracle.quantize(workloads.bits(W), g, sym)
    assert np.array_equal(P.cpu().numpy(), rP), f"packed codes differ {what}"
    assert np.array_equal(workloads.bits(S), rS), f"scales differ {what}"
    assert np.array_equal(workloads.bits(Z), rZ), f"zeros differ {what}"
    return rP, rS, rZ


def _check_full(M, N, K, g, sym, path, seed=0, ctas=0, x_outliers=True):
    W = workloads.make_weight(N, K, 0.02, seed, outlier_frac=0.01, outlier_scale=20.0)
    P, S, Z = w4.quantize(W.cuda(), g, sym)
    rP, rS, rZ = _assert_quantized_like_oracle(W, P, S, Z, g, sym, f"N={N} K={K} g={g} sym={sym}")
    X = workloads.make_activation(M, K, seed + 1, outlier_frac=0.01 if x_outliers else 0.0,
                                  outlier_mode="set")
    Y = w4.gemm(X.cuda(), P, S, Z, g, sym, path=path, ctas=ctas)
    torch.cuda.synchronize()
    Y64 = oracle.gemm_w4a16(workloads.bits(X), rP, rS, rZ, g, sym)
    assert_y_close(workloads.bits(Y), Y64, f"M={M} N={N} K={K} g={g} sym={sym} {path}")
    return Y


# ------------------------------------------------------------------ small shapes, both paths
DECODE_SHAPES = [(1, 256, 256), (1, 1, 128), (2, 37, 384), (3, 100, 1152), (5, 64, 32 * 7),
                 (8, 128, 4096), (9, 96, 640), (13, 257, 1024), (16, 512, 2048)]


@pytest.mark.parametrize("sym", [False, True])
@pytest.mark.parametrize("g", [32, 64, 128])
@pytest.mark.parametrize("M,N,K", DECODE_SHAPES)
def test_decode_path_small(M, N, K, g, sym):
    if K % g:
        pytest.skip("K not a multiple of g")
    _check_full(M, N, K, g, sym, "decode", seed=M + N + K)


@pytest.mark.parametrize("ctas", [1, 2, 3, 5, 7, 13, 40, 97, 300])
@pytest.mark.parametrize("M", [1, 12])
def test_decode_stream_k_partitions(ctas, M):
    """Many persistent-grid sizes: row blocks split 0..n times between CTAs, their
    parts added by each row block's first owner; two calls in a row reuse the
    workspace (its flags must read as consumed again after every call)."""
    _check_full(M, 300, 1024 * 5 + 256, 128, False, "decode", seed=5, ctas=ctas)
    _check_full(M, 300, 1024 * 5 + 256, 128, False, "decode", seed=6, ctas=ctas)


TC_SHAPES = [(1, 128, 64 * 3), (17, 200, 256), (32, 128, 128), (33, 384, 512), (64, 129, 96),
             (100, 256, 1024), (128, 640, 320), (200, 128, 2048), (256, 256, 256),
             (257, 384, 768), (300, 130, 128 * 5), (600, 1000, 1024)]


@pytest.mark.parametrize("sym", [False, True])
@pytest.mark.parametrize("g", [32, 64, 128])
@pytest.mark.parametrize("M,N,K", TC_SHAPES)
def test_tensorcore_path_small(M, N, K, g, sym):
    if K % g:
        pytest.skip("K not a multiple of g")
    _check_full(M, N, K, g, sym, "tensorcore", seed=M * 3 + N + K)


# ------------------------------------------------------------------ exact special cases
@pytest.mark.parametrize("path", ["decode", "tensorcore"])
@pytest.mark.parametrize("sym", [False, True])
@pytest.mark.parametrize("g", [32, 128, 512])     # 512 = K: per-channel
def test_one_hot_activations_select_dequantized_weights_bit_exact(path, sym, g):
    """X = one-hot rows: Y[m, n] = Ŵ[n, k_m] exactly (a single nonzero product,
    exact in fp32, and already a bf16 value), so the fused dequantization of
    every code position is checked bit for bit."""
    N, K = 160, 512
    P, S, Z = _quantized(N, K, g, sym, seed=11)
    Wh = w4.dequantize(P, S, Z, g, sym)
    ks = torch.arange(0, K, dtype=torch.long)
    for start in range(0, K, 16):
        kk = ks[start:start + 16]
        X = torch.zeros(kk.numel(), K, dtype=torch.bfloat16)
        X[torch.arange(kk.numel()), kk] = 1.0
        Y = w4.gemm(X.cuda(), P, S, Z, g, sym, path=path)
        assert torch.equal(Y, Wh[:, kk.cuda()].t().contiguous()), f"k in {start}..{start + 15}"


# ------------------------------------------------------------------ per-channel (g = K)
PC_DECODE_SHAPES = [(1, 256, 256), (1, 1, 160), (3, 100, 1152), (8, 128, 4096), (13, 257, 1056),
                    (16, 64, 11008)]
PC_TC_SHAPES = [(17, 128, 96), (48, 1000, 4352), (129, 64, 4096), (300, 700, 1056)]


@pytest.mark.parametrize("sym", [False, True])
@pytest.mark.parametrize("M,N,K", PC_DECODE_SHAPES)
def test_per_channel_decode(M, N, K, sym):
    """g = K: one scale and zero per weight row, through the decode kernel."""
    _check_full(M, N, K, K, sym, "decode", seed=2 * M + N + K)


@pytest.mark.parametrize("sym", [False, True])
@pytest.mark.parametrize("M,N,K", PC_TC_SHAPES)
def test_per_channel_tensorcore(M, N, K, sym):
    """g = K through the tensor-core kernel, split-K and unsplit tiles."""
    _check_full(M, N, K, K, sym, "tensorcore", seed=3 * M + N + K)


@pytest.mark.parametrize("ctas", [3, 97])
def test_per_channel_decode_partitions(ctas):
    _check_full(5, 300, 1024 * 5 + 256, 1024 * 5 + 256, False, "decode", seed=8, ctas=ctas)


@pytest.mark.parametrize("path", ["decode", "tensorcore"])
def test_deterministic_bitwise(path):
    P, S, Z = _quantized(1000, 4096, 128, False, seed=3)
    X = workloads.make_activation(16, 4096, 4).cuda()
    ys = [w4.gemm(X, P, S, Z, 128, False, path=path) for _ in range(3)]
    assert all(torch.equal(ys[0], y) for y in ys[1:])


@pytest.mark.parametrize("M,N,K,g,sym", [(1, 28672, 8192, 128, False), (4, 4096, 11008, 128, True),
                                         (16, 11008, 4096, 64, False), (3, 1000, 2304, 32, True),
                                         (1, 4096, 11008, 11008, False)])
def test_static_weights_flag_matches_plain_call(M, N, K, g, sym):
    """W4A16_STATIC_WEIGHTS only moves the weight stream ahead of the dependency
    wait: a chain of calls on two sets of fixed weights (each call following a
    GEMM that does not write them) gives the same bits as the plain calls."""
    sets = [_quantized(N, K, g, sym, seed=40 + i) for i in range(2)]
    torch.cuda.synchronize()                      # the quantizer is done with the weights
    X = workloads.make_activation(M, K, 41, outlier_frac=0.01, outlier_mode="set").cuda()
    plain = [w4.gemm(X, *sets[i % 2], g, sym, path="decode") for i in range(4)]
    static = [w4.gemm(X, *sets[i % 2], g, sym, path="decode", static_weights=True) for i in range(4)]
    torch.cuda.synchronize()
    for a, b in zip(plain, static):
        assert torch.equal(a, b)
    assert w4.device_error() == 0


@pytest.mark.parametrize("M,N,K,g,sym", [
    (300, 10240, 2048, 32, False),    # 160 tiles: 148 unsplit + a 12-tile tail split 8 ways
    (2048, 8192, 2048, 128, True),    # 512 tiles: 444 unsplit + a 68-tile tail split 2 ways
    (48, 1000, 4352, 64, False),      # 8 tiles, all split (ragged N, K not a slab multiple)
])
def test_tensorcore_head_and_split_tail(M, N, K, g, sym):
    """Tiles that run unsplit and tiles whose K is split (partials added by the
    reduce kernel) both match the oracle on sampled outputs, including the last
    rows and columns, and two runs are bitwise identical."""
    plan = w4.plan(M, N, K, g, sym, path="tensorcore")
    assert plan["kernels"] >= 2 and plan["workspace_bytes"] > 0
    P, S, Z = _quantized(N, K, g, sym, seed=M)
    X = workloads.make_activation(M, K, M + 1, outlier_frac=0.01, outlier_mode="set")
    Xd = X.cuda()
    Y = w4.gemm(Xd, P, S, Z, g, sym, path="tensorcore")
    Y2 = w4.gemm(Xd, P, S, Z, g, sym, path="tensorcore")
    torch.cuda.synchronize()
    assert torch.equal(Y, Y2)
    rng = np.random.default_rng(M)
    ms = rng.integers(0, M, 2048)
    ns = rng.integers(0, N, 2048)
    ms[:4] = [0, M - 1, 0, M - 1]
    ns[:4] = [0, 0, N - 1, N - 1]
    ref = oracle.gemm_sampled(workloads.bits(X), P.cpu().numpy(), workloads.bits(S),
                              workloads.bits(Z), g, sym, ms, ns)
    assert_y_close(workloads.bits(Y)[ms, ns], ref, f"M={M} N={N} K={K} g={g} sym={sym}")


def test_paths_agree_closely():
    P, S, Z = _quantized(384, 2048, 64, True, seed=8)
    X = workloads.make_activation(16, 2048, 9, outlier_frac=0.01, outlier_mode="set").cuda()
    a = w4.gemm(X, P, S, Z, 64, True, path="decode").float()
    b = w4.gemm(X, P, S, Z, 64, True, path="tensorcore").float()
    assert torch.max(torch.abs(a - b)) <= 4e-3 * torch.max(torch.abs(a))


def test_empty_problems_are_noops():
    P, S, Z = _quantized(64, 256, 128, False, seed=1)
    Y = w4.gemm(torch.empty(0, 256, dtype=torch.bfloat16, device="cuda"), P, S, Z, 128, False)
    assert Y.shape == (0, 64)


def test_host_buffers_end_to_end():
    P, S, Z = _quantized(256, 512, 128, False, seed=12)
    X = workloads.make_activation(2, 512, 13).pin_memory()
    Y = w4.gemm(X, P, S, Z, 128, False)                 # page-locked: w4a16_gemm_host
    assert not Y.is_cuda
    Yd = w4.gemm(X.cuda(), P, S, Z, 128, False)
    assert torch.equal(Y, Yd.cpu())
    Yp = w4.gemm(X.clone(), P, S, Z, 128, False)        # pageable X: the torch copy path
    assert not Yp.is_cuda and torch.equal(Yp, Y)


@pytest.mark.parametrize("M,g,sym", [(1, 128, False), (16, 64, True), (40, 32, False), (300, 128, True)])
def test_host_buffer_chain_matches_device(M, g, sym):
    """Several host-buffer calls queued on one stream (both kernels, one sync at
    the end, reused device scratch) give the device path's bits, each into its
    own page-locked output."""
    layers = [(1152, 768), (768, 1000), (1152, 640)]      # (K, N); K a multiple of every g
    weights = [_quantized(N, K, g, sym, seed=70 + i) for i, (K, N) in enumerate(layers)]
    xs = [workloads.make_activation(M, K, 80 + i).pin_memory() for i, (K, N) in enumerate(layers)]
    torch.cuda.synchronize()          # the weights are written before the chain starts
    outs = []
    for (K, N), (P, S, Z), X in zip(layers, weights, xs):
        Yh = torch.empty(M, N, dtype=torch.bfloat16, pin_memory=True)
        outs.append(w4.gemm(X, P, S, Z, g, sym, out=Yh, sync=False, static_weights=True))
    torch.cuda.synchronize()
    for Yh, (P, S, Z), X in zip(outs, weights, xs):
        assert torch.equal(Yh, w4.gemm(X.cuda(), P, S, Z, g, sym).cpu())


# ------------------------------------------------------------------ full-size workloads
_oracle_codes: dict = {}


def _check_sampled(layer, M, g, sym, path="auto", n_samples=3072, seed=0):
    W = layer.weight()
    X = layer.activation(M)
    P, S, Z = w4.quantize(W.cuda(), g, sym)
    key = (layer.name, layer.N, layer.K, g, sym)
    if key not in _oracle_codes:           # the oracle quantizes each full-size matrix once
        _oracle_codes[key] = _assert_quantized_like_oracle(W, P, S, Z, g, sym, str(key))
    else:
        rP, rS, rZ = _oracle_codes[key]
        assert np.array_equal(P.cpu().numpy(), rP) and np.array_equal(workloads.bits(S), rS) \
            and np.array_equal(workloads.bits(Z), rZ), f"codes differ {key}"
    rP, rS, rZ = _oracle_codes[key]
    Y = w4.gemm(X.cuda(), P, S, Z, g, sym, path=path)
    torch.cuda.synchronize()
    rng = np.random.default_rng(seed + M)
    N = layer.N
    ms = rng.integers(0, M, n_samples)
    ns = rng.integers(0, N, n_samples)
    # always include the first and last rows/columns
    ms[:4] = [0, M - 1, 0, M - 1]
    ns[:4] = [0, 0, N - 1, N - 1]
    ref = oracle.gemm_sampled(workloads.bits(X), rP, rS, rZ, g, sym, ms, ns)
    got = workloads.bits(Y)[ms, ns]
    assert_y_close(got, ref, f"{layer.name} M={M} g={g} sym={sym}")


@pytest.mark.parametrize("M", workloads.DECODE_7B.Ms)
@pytest.mark.parametrize("li", [0, 1])
def test_7b_decode_full_size(li, M):
    _check_sampled(workloads.DECODE_7B.layers[li], M, 128, False)


@pytest.mark.parametrize("sym", [False, True])
@pytest.mark.parametrize("M", workloads.DECODE_70B.Ms)
@pytest.mark.parametrize("li", [0, 1])
def test_70b_decode_full_size(li, M, sym):
    _check_sampled(workloads.DECODE_70B.layers[li], M, 128, sym)


def test_prefill_full_size():
    _check_sampled(workloads.PREFILL.layers[0], 2048, 128, False, n_samples=4096)


@pytest.mark.parametrize("sym", [False, True])
@pytest.mark.parametrize("g", [32, 64, 128])
@pytest.mark.parametrize("M", workloads.CROSSOVER.Ms)
def test_crossover_full_size(M, g, sym):
    """Every point of the crossover workload (K=N=8192, each M, g and mode) in the
    dispatch the benchmark times."""
    _check_sampled(workloads.CROSSOVER.layers[0], M, g, sym, n_samples=2048)


@pytest.mark.parametrize("li", [0, 1])
def test_per_channel_7b_decode_full_size(li):
    layer = workloads.DECODE_7B.layers[li]
    _check_sampled(layer, 1, layer.K, False)


@pytest.mark.parametrize("li", [0, 1])
def test_per_channel_70b_decode_full_size(li):
    layer = workloads.DECODE_70B.layers[li]
    _check_sampled(layer, 2, layer.K, True)


def test_per_channel_prefill_full_size():
    layer = workloads.PREFILL.layers[0]
    _check_sampled(layer, 2048, layer.K, False, n_samples=2048)


def test_tiny_config_full_compare():
    layer = workloads.TINY.layers[0]
    for path in ("decode", "tensorcore"):
        W = layer.weight()
        X = layer.activation(1)
        P, S, Z = w4.quantize(W.cuda(), 128, False)
        Y = w4.gemm(X.cuda(), P, S, Z, 128, False, path=path)
        ref = oracle.gemm_w4a16(workloads.bits(X), P.cpu().numpy(), workloads.bits(S),
                                workloads.bits(Z), 128, False)
        assert_y_close(workloads.bits(Y), ref, f"tiny {path}")


def test_sharded_layer_on_one_rank_nccl():
    """The N-sharded layer's GPU path (fused kernel + NCCL all-gather) on a
    one-rank NCCL group: the rank owns every row and the result matches the
    oracle like the plain GEMM."""
    import os
    import torch.distributed as dist
    from weight_only_quantization_rtn_b200 import sharded
    N, K, M, g = 1000, 2048, 3, 128
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    os.environ.setdefault("MASTER_PORT", str(29500 + os.getpid() % 1000))
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda", 0))
    try:
        W = workloads.make_weight(N, K, 0.02, 9, outlier_frac=0.01, outlier_scale=20.0)
        X = workloads.make_activation(M, K, 10, outlier_frac=0.01, outlier_mode="set")
        layer = sharded.ShardedW4A16Linear.from_weight(W.cuda(), g, False, world=1, rank=0)
        Y = layer(X.cuda())
        torch.cuda.synchronize()
        Y64 = oracle.gemm_w4a16(workloads.bits(X), layer.packed.cpu().numpy(),
                                workloads.bits(layer.scales), workloads.bits(layer.zeros), g, False)
        assert_y_close(workloads.bits(Y), Y64, "sharded, one rank")
        Yg = sharded.gather_columns(torch.zeros(M, N, dtype=torch.bfloat16, device="cuda"), N, 1)
        assert tuple(Yg.shape) == (M, N)
    finally:
        dist.destroy_process_group()
