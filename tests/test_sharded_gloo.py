"""N-sharded W4A16 linear layer (weight_only_quantization_rtn_b200.sharded) on
CPU ranks with the gloo backend: each rank quantizes its rows of W and
multiplies them (here with the oracle standing in for the fused GPU kernel),
and one all-gather assembles Y.  Quantization groups run along K inside a row,
so sharding by output feature changes no code, scale or zero point: the gathered
Y equals the unsharded oracle result bit for bit, for even and uneven splits."""
import os
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _oracle_quantize(Wt, g, sym):
    import oracle
    import workloads
    P, S, Z = oracle.quantize(workloads.bits(Wt), g, sym)
    return torch.from_numpy(P), workloads.from_bits(S), workloads.from_bits(Z)


def _oracle_gemm(X, P, S, Z, g, sym):
    import oracle
    import workloads
    y64 = oracle.gemm_w4a16(workloads.bits(X), P.numpy(), workloads.bits(S), workloads.bits(Z), g, sym)
    return workloads.from_bits(oracle.bf16_from_f64(y64))


def _worker(rank, world, port, N, K, M, g, sym, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import workloads
    from weight_only_quantization_rtn_b200 import sharded
    dist.init_process_group("gloo", rank=rank, world_size=world)
    W = workloads.make_weight(N, K, 0.02, 5, outlier_frac=0.01, outlier_scale=20.0)
    X = workloads.make_activation(M, K, 6, outlier_frac=0.01, outlier_mode="set")
    layer = sharded.ShardedW4A16Linear.from_weight(W, g, sym, world, rank, quantize=_oracle_quantize,
                                                   local_gemm=_oracle_gemm)
    Y = layer(X)
    q.put((rank, layer.n0, layer.n1, workloads.bits(Y).tobytes(), tuple(Y.shape)))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("world,N,K,M,g,sym", [(2, 300, 512, 4, 128, False), (3, 1000, 256, 1, 64, True),
                                               (3, 2, 128, 3, 32, False)])
def test_sharded_equals_unsharded_oracle(world, N, K, M, g, sym):
    import oracle
    import workloads
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29400 + (os.getpid() + N) % 1000
    procs = [ctx.Process(target=_worker, args=(r, world, port, N, K, M, g, sym, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=300) for _ in range(world))
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    W = workloads.make_weight(N, K, 0.02, 5, outlier_frac=0.01, outlier_scale=20.0)
    X = workloads.make_activation(M, K, 6, outlier_frac=0.01, outlier_mode="set")
    P, S, Z = oracle.quantize(workloads.bits(W), g, sym)
    ref = oracle.bf16_from_f64(oracle.gemm_w4a16(workloads.bits(X), P, S, Z, g, sym))
    covered = []
    for rank, n0, n1, ybytes, shape in res:
        assert shape == (M, N)
        covered += list(range(n0, n1))
        assert np.array_equal(np.frombuffer(ybytes, dtype=np.uint16).reshape(M, N), ref), f"rank {rank}"
    assert covered == list(range(N))              # every row computed by exactly one rank


@pytest.mark.parametrize("N,world", [(28672, 8), (8192, 3), (1000, 7), (5, 8), (1, 2)])
def test_shard_rows_partition(N, world):
    from weight_only_quantization_rtn_b200.sharded import shard_rows
    per = -(-N // world)
    rows = []
    for r in range(world):
        n0, n1 = shard_rows(N, world, r)
        assert 0 <= n0 <= n1 <= N and n1 - n0 <= per
        rows += list(range(n0, n1))
    assert rows == list(range(N))
    with pytest.raises(ValueError):
        shard_rows(N, world, world)
