"""The decode GEMM entry point that allocates nothing (w4a16_gemm_decode_noalloc).

It keeps its split-K partial sums in a fixed device array inside the library
instead of a caller-supplied workspace.  Its output must match the ordinary
decode entry point (w4a16_gemm_ex, decode path) within the GEMM tolerance of
the parity tests, call after call, although every call reuses the same array
and finds the previous call's partial sums still in it.  This file is
collected last so that it also runs after every other test in one process."""
import ctypes

import numpy as np
import pytest
import torch

import workloads
import weight_only_quantization_rtn_b200 as w4
from weight_only_quantization_rtn_b200 import build as w4build
from helpers import MAX_REL, FRO_REL, bits_to_f64, y_errors

SCRATCH_BYTES = 8 << 20
EINVAL, EWORKSPACE = 1, 4
FAKE = 0x10000  # 16-byte aligned, never dereferenced: these calls fail validation first


@pytest.fixture(scope="module")
def lib():
    w4build.build()
    return w4.lib()


def _noalloc(lib, X, P, S, Z, g, sym, Y):
    st = lib.w4a16_gemm_decode_noalloc(
        ctypes.c_void_p(X.data_ptr()), X.shape[0], X.shape[1], ctypes.c_void_p(P.data_ptr()),
        ctypes.c_void_p(S.data_ptr()), None if sym else ctypes.c_void_p(Z.data_ptr()),
        P.shape[0], g, int(sym), ctypes.c_void_p(Y.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, lib.w4a16_status_string(st).decode()


def _case(M, N, K, g, sym, seed):
    W = workloads.make_weight(N, K, 0.02, seed, outlier_frac=0.01, outlier_scale=20.0)
    P, S, Z = w4.quantize(W.cuda(), g, sym)
    X = workloads.make_activation(M, K, seed + 1, outlier_frac=0.01, outlier_mode="set").cuda()
    return X, P, S, Z


# Every case splits row blocks between CTAs (the plan's split_tiles), so partial
# sums and ready flags pass through the scratch; the second call finds the first
# call's values still there.
CASES = [(1, 4096, 4096, 128, False, 101), (12, 11008, 4096, 64, True, 103),
         (3, 1000, 2304, 32, False, 105)]


@pytest.mark.gpu
def test_noalloc_matches_decode_entry_point(lib):
    prepared = []
    for (M, N, K, g, sym, seed) in CASES:
        p = w4.plan(M, N, K, g, sym, "decode")
        assert 0 < p["workspace_bytes"] <= SCRATCH_BYTES and p["split_tiles"] > 0
        X, P, S, Z = _case(M, N, K, g, sym, seed)
        Y_ref = w4.gemm(X, P, S, Z, g, sym, path="decode")
        prepared.append((X, P, S, Z, g, sym, Y_ref))
    torch.cuda.synchronize()
    for rep in range(2):
        outs = []
        for (X, P, S, Z, g, sym, _) in prepared:  # calls in a row, no sync between them
            Y = torch.full((X.shape[0], P.shape[0]), float("nan"), dtype=torch.bfloat16,
                           device=X.device)
            _noalloc(lib, X, P, S, Z, g, sym, Y)
            outs.append(Y)
        torch.cuda.synchronize()
        for (X, P, S, Z, g, sym, Y_ref), Y in zip(prepared, outs):
            yb, rb = workloads.bits(Y), workloads.bits(Y_ref)
            emax, efro = y_errors(yb, bits_to_f64(rb))
            what = f"rep {rep} M={X.shape[0]} N={P.shape[0]} g={g} sym={sym}"
            assert emax <= MAX_REL and efro <= FRO_REL, f"{what}: {emax:.3e} {efro:.3e}"
            # same kernel, same partition and reduction order: identical bits
            assert np.array_equal(yb, rb), what
    code = ctypes.c_int32(0)
    assert lib.w4a16_device_error(ctypes.byref(code)) == 0 and code.value == 0


@pytest.mark.gpu
def test_noalloc_binding_two_calls(lib):
    X, P, S, Z = _case(4, 4096, 4096, 128, False, 107)
    Y_ref = w4.gemm(X, P, S, Z, 128, False, path="decode")
    Y1 = w4.gemm_decode_noalloc(X, P, S, Z, 128, False)
    Y2 = w4.gemm_decode_noalloc(X, P, S, Z, 128, False)
    torch.cuda.synchronize()
    for Y in (Y1, Y2):
        assert np.array_equal(workloads.bits(Y), workloads.bits(Y_ref))


def test_noalloc_rejects_without_launching(lib):
    f = ctypes.c_void_p(FAKE)
    # more partial-sum scratch than the built-in array holds
    M, N, K, g = 16, 1 << 17, 4096, 128
    assert w4.plan(M, N, K, g, False, "decode")["workspace_bytes"] > SCRATCH_BYTES
    assert lib.w4a16_gemm_decode_noalloc(f, M, K, f, f, f, N, g, 0, f, None) == EWORKSPACE
    # beyond the decode path's row limit, and a missing zeros pointer
    assert lib.w4a16_gemm_decode_noalloc(f, 17, K, f, f, f, 256, g, 0, f, None) == EINVAL
    assert lib.w4a16_gemm_decode_noalloc(f, 1, K, f, f, None, 256, g, 0, f, None) == EINVAL
    assert lib.w4a16_gemm_decode_noalloc(f, 0, K, f, f, f, 256, g, 0, f, None) == 0


@pytest.mark.gpu
def test_noalloc_binding_rejects_mismatched_tensors(lib):
    """The binding checks shapes, dtypes and devices before the C call, so a
    mismatched tensor raises here and nothing is launched."""
    X, P, S, Z = _case(2, 256, 512, 128, False, 109)
    with pytest.raises(ValueError):
        w4.gemm_decode_noalloc(X[:, :256].contiguous(), P, S, Z, 128, False)   # K differs
    with pytest.raises(ValueError):
        w4.gemm_decode_noalloc(X, P, S, Z, 128, False,
                               out=torch.empty(2, 255, dtype=torch.bfloat16, device=X.device))
    with pytest.raises(TypeError):
        w4.gemm_decode_noalloc(X, P, S, Z, 128, False,
                               out=torch.empty(2, 256, dtype=torch.float32, device=X.device))
    with pytest.raises(ValueError):
        w4.gemm_decode_noalloc(X, P, S, Z, 128, False,
                               out=torch.empty(256, 2, dtype=torch.bfloat16, device=X.device).t())
