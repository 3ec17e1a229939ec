"""Host oracle for W4A16 weight-only RTN quantization — TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never calls it, and it
shares no code with the CUDA library.

The arithmetic lives in ``oracle.c`` (plain scalar C, binary32 quantizer,
binary64 matmul); this module compiles it with gcc and exposes it through
ctypes on numpy arrays.  bf16 tensors are passed as ``uint16`` bit patterns.

Parity status of each function (what pins it is in ``tests/test_oracle_pins.py``):
  bf16_from_f32 / bf16_from_f64 / f32_from_bf16 — pinned (torch conversion,
      exact rational brute force)
  quantize (asym, sym), pack/unpack, dequantize — pinned (hand-computed groups,
      nearest-grid-point brute force, error bounds, invariants)
  gemm_f64 / gemm_sampled — pinned (exact rational brute force, one-hot and
      all-ones special cases)
  group_asym8 / group_sym8 / quantize8 / dequantize8 / gemm_w8a16 /
      gemm_w8a16_sampled (W8A16: 8-bit codes, one per byte) — pinned
      (hand-computed 8-bit groups, brute force over all 256 codes, error
      bounds, on-grid recovery, invariants, one-hot activations)
  scale_activations / gemm_w4a16_act_scaled (per-K activation scale) — pinned
      (identity, exact power-of-two scaling, single rounding of the exact
      product, one-hot activations, the equivalent-scaling identity)
  quantize_act8 / gemm_w8a8 / gemm_w8a8_sampled / gemm_w8a8_from_bf16 (W8A8: per-token INT8
      activations × per-channel INT8 weights) — pinned (hand-computed rows with
      half-to-even ties, nearest-grid-point brute force, absmax to ±127,
      power-of-two scaling, sign symmetry, zero rows, exact rational brute
      force of the GEMM, numpy's float64 matmul of the dequantized operands,
      one-hot activations, the all-127 case)
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

CFLAGS = ["-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-fPIC", "-shared",
          "-std=c11", "-Wall"]


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so next to it (gcc, no fast-math).

    ``W4A16_ORACLE_LIB`` names an already-built library to load instead; the
    mutation tests use it to run the pins against deliberately broken copies.
    """
    override = os.environ.get("W4A16_ORACLE_LIB")
    if override:
        return override
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            i64, i32, vp = ctypes.c_int64, ctypes.c_int32, ctypes.c_void_p
            lib.oracle_bf16_to_f32.argtypes = [ctypes.c_uint16]
            lib.oracle_bf16_to_f32.restype = ctypes.c_float
            lib.oracle_f32_to_bf16_rn.argtypes = [ctypes.c_float]
            lib.oracle_f32_to_bf16_rn.restype = ctypes.c_uint16
            lib.oracle_f64_to_bf16_rn.argtypes = [ctypes.c_double]
            lib.oracle_f64_to_bf16_rn.restype = ctypes.c_uint16
            lib.oracle_group_asym.argtypes = [vp, i64, vp, vp, vp]
            lib.oracle_group_sym.argtypes = [vp, i64, vp, vp]
            lib.oracle_pack_codes.argtypes = [vp, i64, vp]
            lib.oracle_unpack_codes.argtypes = [vp, i64, i32, vp]
            lib.oracle_quantize.argtypes = [vp, i64, i64, i64, i32, vp, vp, vp]
            lib.oracle_quantize.restype = ctypes.c_int
            lib.oracle_dequantize.argtypes = [vp, vp, vp, i64, i64, i64, i32, vp]
            lib.oracle_dequantize.restype = ctypes.c_int
            lib.oracle_gemm_f64.argtypes = [vp, i64, i64, vp, i64, vp]
            lib.oracle_gemm_w4a16_sampled.argtypes = [vp, i64, i64, vp, vp, vp, i64, i64, i32,
                                                      vp, vp, i64, vp]
            lib.oracle_gemm_w4a16_sampled.restype = ctypes.c_int
            lib.oracle_group_asym8.argtypes = [vp, i64, vp, vp, vp]
            lib.oracle_group_sym8.argtypes = [vp, i64, vp, vp]
            lib.oracle_quantize8.argtypes = [vp, i64, i64, i64, i32, vp, vp, vp]
            lib.oracle_quantize8.restype = ctypes.c_int
            lib.oracle_dequantize8.argtypes = [vp, vp, vp, i64, i64, i64, i32, vp]
            lib.oracle_dequantize8.restype = ctypes.c_int
            lib.oracle_gemm_w8a16_sampled.argtypes = [vp, i64, i64, vp, vp, vp, i64, i64, i32,
                                                      vp, vp, i64, vp]
            lib.oracle_gemm_w8a16_sampled.restype = ctypes.c_int
            lib.oracle_scale_activations.argtypes = [vp, i64, i64, vp, vp]
            lib.oracle_quantize_act8.argtypes = [vp, i64, i64, vp, vp]
            lib.oracle_gemm_w8a8.argtypes = [vp, vp, vp, vp, i64, i64, i64, vp]
            lib.oracle_gemm_w8a8_sampled.argtypes = [vp, vp, vp, vp, i64, vp, vp, i64, vp]
            lib.oracle_round_to_bf16.argtypes = [vp, i64, vp]
            lib.oracle_f32_array_to_bf16.argtypes = [vp, i64, vp]
            lib.oracle_num_threads.restype = ctypes.c_int
            _lib = lib
    return _lib


def _ptr(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _u16(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    assert a.dtype == np.uint16, f"expected uint16 bf16 bit patterns, got {a.dtype}"
    return a


# ---------------------------------------------------------------- conversions
def f32_from_bf16(bits) -> np.ndarray:
    """bf16 bit patterns -> float32 values (exact)."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


def bf16_from_f32(x) -> np.ndarray:
    """float32 -> bf16 bits, round to nearest even (elementwise oracle call)."""
    lib = _load()
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, dtype=np.uint16)
    lib.oracle_f32_array_to_bf16(_ptr(x), x.size, _ptr(out))
    return out


def bf16_from_f64(y) -> np.ndarray:
    """float64 -> bf16 bits with a single round-to-nearest-even."""
    lib = _load()
    y = np.ascontiguousarray(y, dtype=np.float64)
    out = np.empty(y.shape, dtype=np.uint16)
    lib.oracle_round_to_bf16(_ptr(y), y.size, _ptr(out))
    return out


# ---------------------------------------------------------------- groups
def group_asym(x) -> tuple[int, int, np.ndarray]:
    """One asymmetric group -> (scale bf16 bits, zero point, codes)."""
    lib = _load()
    x = np.ascontiguousarray(x, dtype=np.float32)
    s = np.zeros(1, dtype=np.uint16)
    z = np.zeros(1, dtype=np.int32)
    q = np.zeros(x.size, dtype=np.int32)
    lib.oracle_group_asym(_ptr(x), x.size, _ptr(s), _ptr(z), _ptr(q))
    return int(s[0]), int(z[0]), q


def group_sym(x) -> tuple[int, np.ndarray]:
    """One symmetric group -> (scale bf16 bits, codes)."""
    lib = _load()
    x = np.ascontiguousarray(x, dtype=np.float32)
    s = np.zeros(1, dtype=np.uint16)
    q = np.zeros(x.size, dtype=np.int32)
    lib.oracle_group_sym(_ptr(x), x.size, _ptr(s), _ptr(q))
    return int(s[0]), q


def pack_codes(q) -> np.ndarray:
    lib = _load()
    q = np.ascontiguousarray(q, dtype=np.int32)
    out = np.zeros(q.size // 2, dtype=np.uint8)
    lib.oracle_pack_codes(_ptr(q), q.size, _ptr(out))
    return out


def unpack_codes(packed, n: int, sym: bool) -> np.ndarray:
    lib = _load()
    p = np.ascontiguousarray(packed, dtype=np.uint8)
    q = np.zeros(n, dtype=np.int32)
    lib.oracle_unpack_codes(_ptr(p), n, int(bool(sym)), _ptr(q))
    return q


# ---------------------------------------------------------------- matrices
def quantize(W_bits, g: int, sym: bool):
    """W[N, K] bf16 bits -> (packed u8[N, K/2], scales bf16[N, K/g], zeros bf16[N, K/g])."""
    lib = _load()
    W = _u16(W_bits)
    N, K = W.shape
    G = K // g
    packed = np.zeros((N, K // 2), dtype=np.uint8)
    scales = np.zeros((N, G), dtype=np.uint16)
    zeros = np.zeros((N, G), dtype=np.uint16)
    rc = lib.oracle_quantize(_ptr(W), N, K, g, int(bool(sym)), _ptr(packed), _ptr(scales),
                             _ptr(zeros))
    if rc != 0:
        raise ValueError(f"oracle_quantize rejected N={N} K={K} g={g}")
    return packed, scales, zeros


def dequantize(packed, scales, zeros, K: int, g: int, sym: bool) -> np.ndarray:
    lib = _load()
    p = np.ascontiguousarray(packed, dtype=np.uint8)
    s = _u16(scales)
    z = _u16(zeros) if zeros is not None else np.zeros_like(s)
    N = p.shape[0]
    out = np.zeros((N, K), dtype=np.uint16)
    rc = lib.oracle_dequantize(_ptr(p), _ptr(s), _ptr(z), N, K, g, int(bool(sym)), _ptr(out))
    if rc != 0:
        raise ValueError("oracle_dequantize rejected its arguments")
    return out


def gemm_f64(X_bits, W_hat_bits) -> np.ndarray:
    """Y64[M, N] = X[M, K] · W_hat[N, K]^T in binary64."""
    lib = _load()
    X, W = _u16(X_bits), _u16(W_hat_bits)
    M, K = X.shape
    N, K2 = W.shape
    assert K == K2
    Y = np.zeros((M, N), dtype=np.float64)
    lib.oracle_gemm_f64(_ptr(X), M, K, _ptr(W), N, _ptr(Y))
    return Y


def gemm_w4a16(X_bits, packed, scales, zeros, g: int, sym: bool) -> np.ndarray:
    """Full reference: dequantize, then binary64 matmul."""
    X = _u16(X_bits)
    W_hat = dequantize(packed, scales, zeros, X.shape[1], g, sym)
    return gemm_f64(X, W_hat)


def gemm_sampled(X_bits, packed, scales, zeros, g: int, sym: bool, ms, ns) -> np.ndarray:
    """Y64 at the listed (m, n) positions, dequantizing row n on the fly."""
    lib = _load()
    X = _u16(X_bits)
    M, K = X.shape
    p = np.ascontiguousarray(packed, dtype=np.uint8)
    s = _u16(scales)
    z = _u16(zeros) if zeros is not None else np.zeros_like(s)
    N = p.shape[0]
    ms = np.ascontiguousarray(ms, dtype=np.int64)
    ns = np.ascontiguousarray(ns, dtype=np.int64)
    out = np.zeros(ms.size, dtype=np.float64)
    rc = lib.oracle_gemm_w4a16_sampled(_ptr(X), M, K, _ptr(p), _ptr(s), _ptr(z), N, g,
                                       int(bool(sym)), _ptr(ms), _ptr(ns), ms.size, _ptr(out))
    if rc != 0:
        raise ValueError("oracle_gemm_w4a16_sampled rejected its arguments")
    return out


# ---------------------------------------------------------------- W8A16 (8-bit codes)
def group_asym8(x) -> tuple[int, int, np.ndarray]:
    """One asymmetric 8-bit group -> (scale bf16 bits, zero point, codes 0..255)."""
    lib = _load()
    x = np.ascontiguousarray(x, dtype=np.float32)
    s = np.zeros(1, dtype=np.uint16)
    z = np.zeros(1, dtype=np.int32)
    q = np.zeros(x.size, dtype=np.int32)
    lib.oracle_group_asym8(_ptr(x), x.size, _ptr(s), _ptr(z), _ptr(q))
    return int(s[0]), int(z[0]), q


def group_sym8(x) -> tuple[int, np.ndarray]:
    """One symmetric 8-bit group -> (scale bf16 bits, codes −128..127)."""
    lib = _load()
    x = np.ascontiguousarray(x, dtype=np.float32)
    s = np.zeros(1, dtype=np.uint16)
    q = np.zeros(x.size, dtype=np.int32)
    lib.oracle_group_sym8(_ptr(x), x.size, _ptr(s), _ptr(q))
    return int(s[0]), q


def quantize8(W_bits, g: int, sym: bool):
    """W[N, K] bf16 bits -> (codes u8[N, K], scales bf16[N, K/g], zeros bf16[N, K/g])."""
    lib = _load()
    W = _u16(W_bits)
    N, K = W.shape
    G = K // g
    codes = np.zeros((N, K), dtype=np.uint8)
    scales = np.zeros((N, G), dtype=np.uint16)
    zeros = np.zeros((N, G), dtype=np.uint16)
    rc = lib.oracle_quantize8(_ptr(W), N, K, g, int(bool(sym)), _ptr(codes), _ptr(scales),
                              _ptr(zeros))
    if rc != 0:
        raise ValueError(f"oracle_quantize8 rejected N={N} K={K} g={g}")
    return codes, scales, zeros


def dequantize8(codes, scales, zeros, g: int, sym: bool) -> np.ndarray:
    lib = _load()
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    s = _u16(scales)
    z = _u16(zeros) if zeros is not None else np.zeros_like(s)
    N, K = c.shape
    out = np.zeros((N, K), dtype=np.uint16)
    rc = lib.oracle_dequantize8(_ptr(c), _ptr(s), _ptr(z), N, K, g, int(bool(sym)), _ptr(out))
    if rc != 0:
        raise ValueError("oracle_dequantize8 rejected its arguments")
    return out


def gemm_w8a16(X_bits, codes, scales, zeros, g: int, sym: bool) -> np.ndarray:
    """Full W8A16 reference: dequantize the 8-bit codes, then binary64 matmul."""
    return gemm_f64(_u16(X_bits), dequantize8(codes, scales, zeros, g, sym))


def gemm_w8a16_sampled(X_bits, codes, scales, zeros, g: int, sym: bool, ms, ns) -> np.ndarray:
    lib = _load()
    X = _u16(X_bits)
    M, K = X.shape
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    s = _u16(scales)
    z = _u16(zeros) if zeros is not None else np.zeros_like(s)
    N = c.shape[0]
    ms = np.ascontiguousarray(ms, dtype=np.int64)
    ns = np.ascontiguousarray(ns, dtype=np.int64)
    out = np.zeros(ms.size, dtype=np.float64)
    rc = lib.oracle_gemm_w8a16_sampled(_ptr(X), M, K, _ptr(c), _ptr(s), _ptr(z), N, g,
                                       int(bool(sym)), _ptr(ms), _ptr(ns), ms.size, _ptr(out))
    if rc != 0:
        raise ValueError("oracle_gemm_w8a16_sampled rejected its arguments")
    return out


# ---------------------------------------------------------------- per-K activation scale
def scale_activations(X_bits, a_bits) -> np.ndarray:
    """X'[m, k] = bf16_rn(X[m, k]·a[k]) (bf16 bits in and out)."""
    lib = _load()
    X = _u16(X_bits)
    a = _u16(a_bits)
    M, K = X.shape
    assert a.shape == (K,)
    out = np.zeros((M, K), dtype=np.uint16)
    lib.oracle_scale_activations(_ptr(X), M, K, _ptr(a), _ptr(out))
    return out


def gemm_w4a16_act_scaled(X_bits, a_bits, packed, scales, zeros, g: int, sym: bool) -> np.ndarray:
    """Y64 = (X·diag(a))' · Ŵᵀ with the scaled activations rounded to bf16 first."""
    return gemm_w4a16(scale_activations(X_bits, a_bits), packed, scales, zeros, g, sym)


def quantize_act8(X_bits):
    """W8A8 activations: per-token (row) symmetric INT8, s_x = max|x|/127 in binary32.
    Returns (q int8 [M, K], s_x float32 [M])."""
    lib = _load()
    X = _u16(X_bits)
    M, K = X.shape
    q = np.zeros((M, K), dtype=np.int8)
    s = np.zeros(M, dtype=np.float32)
    lib.oracle_quantize_act8(_ptr(X), M, K, _ptr(q), _ptr(s))
    return q, s


def gemm_w8a8(qx, sx, qw, sw_bits) -> np.ndarray:
    """Y64[m, n] = s_x[m]·s_w[n]·Σ_k q_x[m, k]·q_w[n, k] (exact integer sum).
    qx int8 [M, K], sx float32 [M], qw int8 (or its uint8 bytes) [N, K], sw bf16 bits [N] or [N, 1]."""
    lib = _load()
    qx = np.ascontiguousarray(qx, dtype=np.int8)
    sx = np.ascontiguousarray(sx, dtype=np.float32)
    qw = np.ascontiguousarray(qw).view(np.int8)
    sw = _u16(np.ascontiguousarray(sw_bits).reshape(-1))
    M, K = qx.shape
    N, K2 = qw.shape
    assert K == K2 and sx.shape == (M,) and sw.shape == (N,)
    Y = np.zeros((M, N), dtype=np.float64)
    lib.oracle_gemm_w8a8(_ptr(qx), _ptr(sx), _ptr(qw), _ptr(sw), M, N, K, _ptr(Y))
    return Y


def gemm_w8a8_sampled(qx, sx, qw, sw_bits, ms, ns) -> np.ndarray:
    """gemm_w8a8 at the listed (m, n) positions only (for full-size checks)."""
    lib = _load()
    qx = np.ascontiguousarray(qx, dtype=np.int8)
    sx = np.ascontiguousarray(sx, dtype=np.float32)
    qw = np.ascontiguousarray(qw).view(np.int8)
    sw = _u16(np.ascontiguousarray(sw_bits).reshape(-1))
    ms = np.ascontiguousarray(ms, dtype=np.int64)
    ns = np.ascontiguousarray(ns, dtype=np.int64)
    assert qx.shape[1] == qw.shape[1] and ms.shape == ns.shape
    out = np.zeros(ms.shape[0], dtype=np.float64)
    lib.oracle_gemm_w8a8_sampled(_ptr(qx), _ptr(sx), _ptr(qw), _ptr(sw), qx.shape[1], _ptr(ms), _ptr(ns),
                                 ms.shape[0], _ptr(out))
    return out


def gemm_w8a8_from_bf16(X_bits, qw, sw_bits) -> np.ndarray:
    """The whole W8A8 product for bf16 activations: quantize X per token, then
    the integer GEMM with both scales."""
    qx, sx = quantize_act8(X_bits)
    return gemm_w8a8(qx, sx, qw, sw_bits)


def num_threads() -> int:
    return int(_load().oracle_num_threads())
