"""Host-side checks of the C ABI (no GPU needed, no kernel launched).

The library loads without a GPU; argument validation runs before any CUDA
call, so rejected calls return W4A16_EINVAL here as on a GPU machine."""
import ctypes
import os
import re
import subprocess

import pytest

import weight_only_quantization_rtn_b200 as w4
from weight_only_quantization_rtn_b200 import build as w4build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "w4a16.h")
EINVAL, EWORKSPACE = 1, 4


@pytest.fixture(scope="module")
def lib():
    w4build.build()
    return w4.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(w4a16_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_abi():
    names = declared_functions()
    for n in ("w4a16_quantize", "w4a16_dequantize", "w4a16_gemm", "w4a16_gemm_ex",
              "w4a16_gemm_workspace_size", "w4a16_gemm_plan", "w4a16_status_string",
              "w4a16_device_error", "w4a16_abi_version"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", w4.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\sT\s(w4a16_\w+)", out))
    for name in declared_functions():
        assert name in exported, f"{name} declared in w4a16.h but not exported"
        assert hasattr(lib, name)


def test_library_is_sm100a_only_and_links_no_cudart_dso(lib):
    out = subprocess.run(["ldd", w4.LIB_PATH], capture_output=True, text=True).stdout
    assert "libcudart" not in out          # runtime linked statically


def test_status_strings_and_version(lib):
    assert lib.w4a16_abi_version() == 1
    for s in range(6):
        assert lib.w4a16_status_string(s).startswith(b"W4A16")


FAKE = 0x10000          # 16-byte aligned, never dereferenced on the host


def _gemm(lib, M=1, K=128, N=64, g=128, sym=0, X=FAKE, P=FAKE, S=FAKE, Z=FAKE, Y=FAKE,
          path=0, split=0, ws=None, ws_bytes=0):
    return lib.w4a16_gemm_ex(X, M, K, P, S, Z, N, g, sym, Y, ws, ws_bytes, path, split, None)


@pytest.mark.parametrize("kw", [
    dict(g=48), dict(g=16), dict(g=256), dict(K=96), dict(K=0), dict(M=-1), dict(N=-2),
    dict(sym=2), dict(X=None), dict(P=None), dict(S=None), dict(Y=None), dict(Z=None),
    dict(X=FAKE + 8), dict(P=FAKE + 4), dict(Y=FAKE + 2), dict(S=FAKE + 2),
    dict(M=17, path=1), dict(path=3), dict(split=9), dict(split=2, path=2),
    dict(K=2 ** 31),
])
def test_gemm_rejects_invalid_arguments(lib, kw):
    assert _gemm(lib, **kw) == EINVAL


def test_gemm_sym_accepts_null_zeros_validation(lib):
    # with sym=1 a NULL zeros pointer passes validation; M=0 then returns before any launch
    assert _gemm(lib, M=0, sym=1, Z=None) == 0
    assert _gemm(lib, M=0) == 0 and _gemm(lib, N=0) == 0


def test_quantize_and_dequantize_reject_invalid(lib):
    q = lib.w4a16_quantize
    assert q(FAKE, 4, 96, 64, 0, FAKE, FAKE, FAKE, None) == EINVAL
    assert q(FAKE, 4, 128, 128, 0, FAKE, FAKE, None, None) == EINVAL     # asym needs zeros
    assert q(FAKE + 8, 4, 128, 128, 0, FAKE, FAKE, FAKE, None) == EINVAL
    assert q(FAKE, 4, 128, 100, 1, FAKE, FAKE, None, None) == EINVAL
    assert q(FAKE, 0, 128, 128, 1, FAKE, FAKE, None, None) == 0          # N = 0: nothing to do
    d = lib.w4a16_dequantize
    assert d(FAKE, FAKE, None, 4, 128, 128, 0, FAKE, None) == EINVAL
    assert d(FAKE, FAKE, FAKE, 4, 128, 32, 3, FAKE, None) == EINVAL
    assert d(FAKE, FAKE, FAKE, 4, 128, 32, 0, FAKE + 1, None) == EINVAL


def test_workspace_size_is_zero(lib):
    assert w4.workspace_size(1, 4096, 4096, 128) == 0
    assert w4.workspace_size(2048, 8192, 8192, 32) == 0


def test_dispatch_plans():
    assert w4.plan(1, 11008, 4096)["path"] == "decode"
    assert w4.plan(16, 4096, 11008)["path"] == "decode"
    assert w4.plan(17, 4096, 4096)["path"] == "tensorcore"
    p = w4.plan(2048, 8192, 8192)
    assert p["path"] == "tensorcore" and p["tile_m"] == 256 and p["grid"] == 64 * 8
    assert p["smem_bytes"] <= 232448
    for M, bm in ((17, 32), (32, 32), (33, 64), (64, 64), (65, 128), (128, 128), (129, 256)):
        assert w4.plan(M, 8192, 8192)["tile_m"] == bm
    for M in (1, 8):
        assert w4.plan(M, 4096, 4096)["tile_m"] == 8
    assert w4.plan(9, 4096, 4096)["tile_m"] == 16
    p = w4.plan(1, 4096, 11008, split_k=3)
    assert p["split_k"] == 3 and p["grid"] == 3 * 4096 // 32
    for N, K in ((11008, 4096), (4096, 11008), (28672, 8192), (8192, 28672), (256, 256)):
        p = w4.plan(1, N, K)
        assert 1 <= p["split_k"] <= 8
        assert p["grid"] % p["split_k"] == 0
        assert (K + 127) // 128 >= p["split_k"]
    with pytest.raises(w4.W4A16Error):
        w4.plan(17, 4096, 4096, path="decode")
