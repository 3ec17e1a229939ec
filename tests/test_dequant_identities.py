"""The arithmetic identities the GEMM kernels' dequantization relies on, proven
exhaustively on the host in IEEE binary32 (numpy) — independent of CUDA:

* INT4 (both GEMMs): a nibble OR'ed into the exponent pattern of 128.0 is the
  bf16 value 128 + q; subtracting 128 + z (bf16) is exact; the product with the
  bf16 scale s is exact in binary32, so the bf16 multiply rounds it once:
  bf16_mul(bf16_sub(128 + q, 128 + z), s) == bf16_rn((q − z)·s).
* 8-bit codes: a byte placed in the mantissa of 2^23 is 2^23 + q; subtracting
  2^23 + z and multiplying by s are exact in binary32, so one round to bf16
  gives bf16_rn((q − z)·s); symmetric codes XOR'ed with 0x80 and z = 128 give q.

Each is checked for every code, every zero point and a spread of bf16 scales
(subnormal and normal, up to 2^113, where 255·s stays finite in binary32),
against the exact product rounded once (the oracle's definition, R8)."""
import numpy as np
import pytest

import oracle


def _bf16_scales():
    # every bf16 significand at several exponents, plus subnormal and extreme ones
    sig = np.arange(128, dtype=np.uint32)
    exps = np.array([1, 20, 100, 120, 127, 130, 160, 200, 240], dtype=np.uint32)
    bits = ((exps[:, None] << 7) | sig[None, :]).ravel()
    return np.unique(np.concatenate([bits, np.arange(1, 128, dtype=np.uint32)])).astype(np.uint16)


def _f32(bits16):
    return (np.asarray(bits16, np.uint32) << 16).view(np.float32)


def _round_bf16_from_f32(x):
    """Round binary32 to bf16 (ties to even) — the bf16 result of a GPU bf16 op
    whose exact value is x (exact here because x is an exact product)."""
    return oracle.bf16_from_f32(np.asarray(x, np.float32))


def test_int4_magic_sequence_is_exact():
    S = _bf16_scales()
    s = _f32(S)
    for z in range(16):
        for q in range(16):
            a = np.float32(128 + q)                    # 0x4300 | q as bf16
            assert _round_bf16_from_f32(a)[()] == 0x4300 | q
            d = np.float32(a - np.float32(128 + z))    # bf16 sub: exact small integer
            assert d == q - z
            got = _round_bf16_from_f32(d * s)          # bf16 mul: exact product, one rounding
            exp = oracle.bf16_from_f64((q - z) * s.astype(np.float64))
            assert np.array_equal(got, exp), (q, z)


@pytest.mark.parametrize("sym", [False, True])
def test_byte_magic_sequence_is_exact(sym):
    S = _bf16_scales()
    s = _f32(S)
    zs = [128] if sym else range(256)
    for z in zs:
        zoff = np.float32(8388608.0 + z)
        assert zoff == 8388608.0 + z                  # 2^23 + z is exact (< 2^24)
        for b in range(256):
            stored = b ^ 0x80 if sym else b           # int8 code flipped to offset-128
            q = (b - 256 if b >= 128 else b) if sym else b
            m = np.array([0x4B000000 | stored], np.uint32).view(np.float32)[0]
            assert m == 8388608.0 + stored            # the byte in the mantissa of 2^23
            d = np.float32(m - zoff)
            assert d == q - (0 if sym else z)
            got = _round_bf16_from_f32(d * s)
            exp = oracle.bf16_from_f64((q - (0 if sym else z)) * s.astype(np.float64))
            assert np.array_equal(got, exp), (b, z)
