"""Pins for the host oracle: checks against what the pages and mathematics fix.

No expectation here is computed by re-typing the oracle's formulas.  The pins
are: hand-computed groups (tests/golden/hand_groups.json), a library routine
(torch's float32 -> bf16 conversion), exact rational brute force (fractions),
nearest-grid-point brute force over all 16 codes, closed-form constructions
(on-grid groups, exactly representable products, one-hot and all-ones
activations) and invariants (ranges, z = 0 in symmetric mode, power-of-two
scale invariance, error bounds).
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_groups.json")
CASES = json.load(open(GOLDEN))["cases"]


def _f32(vals):
    return np.array([float(v) for v in vals], dtype=np.float32)


# ------------------------------------------------------------------ golden groups
@pytest.mark.parametrize("case", CASES, ids=[c["name"] for c in CASES])
def test_hand_computed_group(case):
    x = _f32(case["x"])
    sym = case["mode"] == "sym"
    if sym:
        s_bits, q = oracle.group_sym(x)
        z = 0
    else:
        s_bits, z, q = oracle.group_asym(x)
    assert s_bits == int(case["s_bits"], 16)
    assert float(oracle.f32_from_bf16(np.array([s_bits], np.uint16))[0]) == float(case["s"])
    assert z == case["z"]
    assert list(q) == case["q"]
    packed = oracle.pack_codes(q)
    assert list(packed) == [int(b, 16) for b in case["packed"]]


@pytest.mark.parametrize("case", CASES, ids=[c["name"] for c in CASES])
def test_hand_computed_group_through_matrix_path(case):
    """Same groups through quantize/dequantize on a [3, 8] matrix (two groups per
    row, rows and groups permuted) to pin row/group/nibble indexing."""
    x = _f32(case["x"])
    sym = case["mode"] == "sym"
    other = _f32(CASES[0]["x"])                 # a different group beside it
    rows = [np.concatenate([x, other]), np.concatenate([other, x]), np.concatenate([x, x])]
    W = oracle.bf16_from_f32(np.stack(rows))
    P, S, Z = oracle.quantize(W, 4, sym)
    exp_bytes = [int(b, 16) for b in case["packed"]]
    for r, slot in ((0, 0), (1, 1), (2, 0), (2, 1)):
        assert list(P[r, 2 * slot:2 * slot + 2]) == exp_bytes
        assert S[r, slot] == int(case["s_bits"], 16)
        assert float(oracle.f32_from_bf16(Z[r, slot:slot + 1])[0]) == (0.0 if sym else case["z"])
    Wh = oracle.dequantize(P, S, Z, 8, 4, sym)
    xh = oracle.f32_from_bf16(Wh)
    exp = [float(v) for v in case["x_hat"]]
    assert list(xh[0, :4]) == exp and list(xh[1, 4:]) == exp and list(xh[2, 4:]) == exp


# ------------------------------------------------------------------ bf16 conversions
def _interesting_floats(n=20000, seed=0):
    rng = np.random.default_rng(seed)
    a = rng.standard_normal(n).astype(np.float32) * np.float32(3.0)
    b = (rng.integers(0, 2**32, n, dtype=np.uint64).astype(np.uint32)).view(np.float32)
    b = b[np.isfinite(b)]
    # exact ties: upper 16 bits arbitrary, lower 16 bits = 0x8000
    t = ((rng.integers(0, 2**16, 4000, dtype=np.uint64).astype(np.uint32) << 16) | 0x8000)
    t = t.view(np.float32)
    t = t[np.isfinite(t)]
    special = np.array([0.0, -0.0, 1e-45, -1e-45, 1e-39, 3.3895313e38, 3.4e38, -3.4e38,
                        np.inf, -np.inf], dtype=np.float32)
    return np.concatenate([a, b, t, special]).astype(np.float32)


def test_f32_to_bf16_matches_torch():
    x = _interesting_floats()
    ours = oracle.bf16_from_f32(x)
    ref = workloads.bits(torch.from_numpy(x).to(torch.bfloat16))
    assert np.array_equal(ours, ref)


def test_bf16_to_f32_is_exact_upper_half():
    b = np.arange(0, 2**16, dtype=np.uint32).astype(np.uint16)
    f = oracle.f32_from_bf16(b)
    t = workloads.from_bits(b).to(torch.float32).numpy()
    fin = np.isfinite(t)
    assert np.array_equal(f[fin], t[fin])


def _bf16_value(bits16):
    f = oracle.f32_from_bf16(np.array([bits16], np.uint16))[0]
    return Fraction(float(f))


def _bf16_rne_bruteforce(d: float) -> int:
    """Nearest bf16 to the exact value of d, ties to even mantissa (pure Python)."""
    exact = Fraction(d)
    if d == 0:
        return 0x8000 if np.signbit(d) else 0
    c = int(np.array([np.float32(d)]).view(np.uint32)[0] >> 16)
    best = None
    for cand in range(max(c - 2, 0), min(c + 3, 0xFFFF) + 1):
        if (cand & 0x7F80) == 0x7F80:
            continue
        if (cand >> 15) != (1 if d < 0 else 0):
            continue
        dist = abs(_bf16_value(cand) - exact)
        key = (dist, cand & 1)
        if best is None or key < best[0]:
            best = (key, cand)
    return best[1]


def test_f64_to_bf16_single_rounding_bruteforce():
    rng = np.random.default_rng(1)
    vals = list(rng.standard_normal(3000) * 10.0)
    # doubles just beside bf16 ties: a binary32-then-bf16 double rounding would break these
    for _ in range(500):
        hi = int(rng.integers(0x3C00, 0x4400))
        base = float(Fraction(float(oracle.f32_from_bf16(np.array([hi], np.uint16))[0])))
        ulp = float(_bf16_value(hi + 1) - _bf16_value(hi))
        mid = base + ulp / 2
        vals += [mid, np.nextafter(mid, np.inf), np.nextafter(mid, -np.inf),
                 mid + ulp * 2.0**-20, mid - ulp * 2.0**-20]
    vals = np.array(vals, dtype=np.float64)
    ours = oracle.bf16_from_f64(vals)
    for v, o in zip(vals, ours):
        assert int(o) == _bf16_rne_bruteforce(float(v)), (v, hex(o))


# ------------------------------------------------------------------ packing
@pytest.mark.parametrize("sym", [False, True])
def test_unpack_pack_all_256_bytes(sym):
    allb = np.arange(256, dtype=np.uint8)
    q = oracle.unpack_codes(allb, 512, sym)
    assert np.array_equal(oracle.pack_codes(q), allb)
    lo, hi = q[0::2], q[1::2]
    if sym:
        assert lo.min() == -8 and lo.max() == 7
        assert np.array_equal(lo, ((allb & 0xF).astype(np.int32) ^ 8) - 8)
    else:
        assert np.array_equal(lo, allb & 0xF) and np.array_equal(hi, allb >> 4)


@pytest.mark.parametrize("sym", [False, True])
def test_pack_unpack_all_code_pairs(sym):
    r = np.arange(-8, 8) if sym else np.arange(16)
    a, b = np.meshgrid(r, r, indexing="ij")
    q = np.stack([a.ravel(), b.ravel()], 1).ravel().astype(np.int32)
    assert np.array_equal(oracle.unpack_codes(oracle.pack_codes(q), q.size, sym), q)


# ------------------------------------------------------------------ quantizer properties
def _groups(seed, g, n):
    """Random groups of assorted shapes: Gaussian, outlier-laden, one-sided, tiny, huge."""
    rng = np.random.default_rng(seed)
    out = []
    for i in range(n):
        kind = i % 6
        x = rng.standard_normal(g)
        if kind == 1:
            x[rng.integers(0, g)] *= 50.0
        elif kind == 2:
            x = np.abs(x) + 0.1
        elif kind == 3:
            x = -np.abs(x) - 0.1
        elif kind == 4:
            x *= 2.0**-60
        elif kind == 5:
            x *= 2.0**40
        out.append(oracle.f32_from_bf16(oracle.bf16_from_f32(x.astype(np.float32))))
    return out


@pytest.mark.parametrize("g", [4, 32, 64, 128])
def test_asym_codes_are_nearest_grid_points(g):
    """Brute force over all 16 codes: the chosen code minimises |x − (c − z)s|,
    up to the rounding of the binary32 quotient x/s next to a tie."""
    for x in _groups(10 + g, g, 240):
        s_bits, z, q = oracle.group_asym(x)
        s = float(oracle.f32_from_bf16(np.array([s_bits], np.uint16))[0])
        assert 0 <= z <= 15 and np.all((q >= 0) & (q <= 15))
        if s == 0.0:
            assert np.all(q == 0) and z == 0
            continue
        xs = x.astype(np.float64)
        grid = (np.arange(16)[None, :] - z) * s               # exact in binary64
        dist = np.abs(xs[:, None] - grid)
        chosen = dist[np.arange(g), q]
        slack = np.abs(xs) * 2.0**-22 + s * 2.0**-20
        assert np.all(chosen <= dist.min(1) + slack)


@pytest.mark.parametrize("g", [4, 32, 128])
def test_sym_codes_are_nearest_grid_points(g):
    for x in _groups(20 + g, g, 240):
        s_bits, q = oracle.group_sym(x)
        s = float(oracle.f32_from_bf16(np.array([s_bits], np.uint16))[0])
        assert np.all((q >= -7) & (q <= 7)), "absmax/7 never reaches -8"
        if s == 0.0:
            assert np.all(q == 0)
            continue
        xs = x.astype(np.float64)
        grid = np.arange(-8, 8)[None, :] * s
        dist = np.abs(xs[:, None] - grid)
        chosen = dist[np.arange(g), q + 8]
        slack = np.abs(xs) * 2.0**-22 + s * 2.0**-20
        assert np.all(chosen <= dist.min(1) + slack)


@pytest.mark.parametrize("g", [32, 128])
def test_error_bound_half_step(g):
    """|x − (q − z)s| ≤ s/2 for unclamped codes; clamped codes can exceed it only
    by the bf16 rounding of s: ≤ s/2 + 15·2^-8·s."""
    for x in _groups(30 + g, g, 240):
        s_bits, z, q = oracle.group_asym(x)
        s = float(oracle.f32_from_bf16(np.array([s_bits], np.uint16))[0])
        if s == 0.0:
            continue
        err = np.abs(x.astype(np.float64) - (q - z) * s)
        inner = (q > 0) & (q < 15)
        assert np.all(err[inner] <= s / 2 * (1 + 2.0**-20))
        assert np.all(err <= s / 2 + 15 * 2.0**-8 * s)
        # the group minimum maps to code 0 (rint is odd-symmetric); the maximum to 14 or 15
        lo, hi = np.argmin(x), np.argmax(x)
        if x[lo] < 0:
            assert q[lo] == 0
        if x[hi] > 0:
            assert q[hi] >= 14


def test_sym_zero_points_are_zero_and_error_bound():
    W = workloads.bits(workloads.make_weight(37, 256, 0.02, seed=5, outlier_frac=0.05,
                                             outlier_scale=20.0))
    P, S, Z = oracle.quantize(W, 64, sym=True)
    assert np.all(Z == 0)
    q = oracle.unpack_codes(P.reshape(-1), P.size * 2, True).reshape(37, 256)
    s = np.repeat(oracle.f32_from_bf16(S).astype(np.float64), 64, axis=1)
    x = oracle.f32_from_bf16(W).astype(np.float64)
    assert np.all(np.abs(x - q * s) <= s / 2 * (1 + 2.0**-20) + 0.0)


@pytest.mark.parametrize("sym", [False, True])
@pytest.mark.parametrize("e", [-7, 5])
def test_power_of_two_scale_invariance(sym, e):
    W = workloads.make_weight(16, 256, 0.02, seed=7, outlier_frac=0.02, outlier_scale=20.0)
    W2 = (W.to(torch.float32) * 2.0**e).to(torch.bfloat16)     # exact scaling
    P1, S1, Z1 = oracle.quantize(workloads.bits(W), 32, sym)
    P2, S2, Z2 = oracle.quantize(workloads.bits(W2), 32, sym)
    assert np.array_equal(P1, P2) and np.array_equal(Z1, Z2)
    assert np.array_equal(oracle.f32_from_bf16(S1) * np.float32(2.0**e), oracle.f32_from_bf16(S2))


@pytest.mark.parametrize("g", [32, 64, 128])
def test_on_grid_matrix_is_recovered_exactly(g):
    """Closed form: W = (q − z)·s with s of ≤ 4 significant bits and each group
    using codes 0 and 15 re-quantizes to exactly (s, z, q), and dequantizes to W."""
    rng = np.random.default_rng(g)
    N, K = 6, 4 * g
    G = K // g
    q = rng.integers(0, 16, size=(N, K))
    q[:, ::g] = 0
    q[:, 1::g] = 15
    z = rng.integers(0, 16, size=(N, G))
    mant = rng.choice([8, 9, 10, 11, 12, 13, 14, 15], size=(N, G))   # 4 significant bits
    s = mant * 2.0 ** rng.integers(-14, -6, size=(N, G)).astype(np.float64)
    x = (q - np.repeat(z, g, 1)) * np.repeat(s, g, 1)
    Wb = oracle.bf16_from_f32(x.astype(np.float32))
    assert np.array_equal(oracle.f32_from_bf16(Wb).astype(np.float64), x)
    P, S, Z = oracle.quantize(Wb, g, sym=False)
    assert np.array_equal(oracle.f32_from_bf16(S).astype(np.float64), s)
    assert np.array_equal(oracle.f32_from_bf16(Z).astype(np.int64), z)
    qq = oracle.unpack_codes(P.reshape(-1), N * K, False).reshape(N, K)
    assert np.array_equal(qq, q)
    Wh = oracle.dequantize(P, S, Z, K, g, False)
    assert np.array_equal(Wh, Wb)


# ------------------------------------------------------------------ per-channel (g = K)
@pytest.mark.parametrize("sym", [False, True])
def test_hand_computed_rows_per_channel(sym):
    """Per-channel granularity (one scale per output row; "量化实战深入（GPTQ / AWQ / SmoothQuant / KV 量化）",
    量化粒度 table; "推理优化中“用精度换性能“的核心技术：量化", §3.4) is g = K: each row of a [rows, 4] matrix is one of
    the hand-computed groups and must get that group's s, z, codes and x̂."""
    cases = [c for c in CASES if (c["mode"] == "sym") == sym]
    assert cases
    W = oracle.bf16_from_f32(np.stack([_f32(c["x"]) for c in cases]))
    P, S, Z = oracle.quantize(W, 4, sym)
    assert S.shape == (len(cases), 1) and Z.shape == (len(cases), 1)
    Wh = oracle.f32_from_bf16(oracle.dequantize(P, S, Z, 4, 4, sym))
    for r, c in enumerate(cases):
        assert S[r, 0] == int(c["s_bits"], 16)
        assert float(oracle.f32_from_bf16(Z[r, :1])[0]) == (0.0 if sym else c["z"])
        assert list(P[r]) == [int(b, 16) for b in c["packed"]]
        assert list(Wh[r]) == [float(v) for v in c["x_hat"]]


def test_on_grid_rows_per_channel_recovered_exactly():
    """Closed form at g = K: rows (q − z)·s with one s and z per row, each row
    using codes 0 and 15, re-quantize to exactly (s, z, q) and dequantize to W."""
    rng = np.random.default_rng(17)
    N, K = 7, 416
    q = rng.integers(0, 16, size=(N, K))
    q[:, 3] = 0
    q[:, K - 2] = 15
    z = rng.integers(0, 16, size=(N, 1))
    s = rng.choice([8, 9, 11, 13, 15], size=(N, 1)) * 2.0 ** rng.integers(-14, -6, size=(N, 1))
    x = (q - z) * s
    Wb = oracle.bf16_from_f32(x.astype(np.float32))
    assert np.array_equal(oracle.f32_from_bf16(Wb).astype(np.float64), x)
    P, S, Z = oracle.quantize(Wb, K, sym=False)
    assert np.array_equal(oracle.f32_from_bf16(S).astype(np.float64), s)
    assert np.array_equal(oracle.f32_from_bf16(Z).astype(np.int64), z)
    assert np.array_equal(oracle.unpack_codes(P.reshape(-1), N * K, False).reshape(N, K), q)
    assert np.array_equal(oracle.dequantize(P, S, Z, K, K, False), Wb)


def test_per_channel_equals_groups_with_equal_ranges():
    """Invariant: when every 32-wide group of a row holds the row's minimum and
    maximum (hence also its max|x|), grouped (g = 32) and per-channel (g = K)
    quantization give the same codes, and the grouped scales and zeros are the
    per-channel ones repeated."""
    rng = np.random.default_rng(23)
    N, K = 5, 256
    x = rng.standard_normal((N, K)) * 0.02
    lo, hi = x.min(1, keepdims=True) - 0.01, x.max(1, keepdims=True) + 0.01
    x[:, 0::32], x[:, 1::32] = lo, hi
    Wb = oracle.bf16_from_f32(x.astype(np.float32))
    for sym in (False, True):
        Pg, Sg, Zg = oracle.quantize(Wb, 32, sym)
        Pc, Sc, Zc = oracle.quantize(Wb, K, sym)
        assert np.array_equal(Pg, Pc)
        assert np.array_equal(Sg, np.repeat(Sc, K // 32, 1))
        assert np.array_equal(Zg, np.repeat(Zc, K // 32, 1))


@pytest.mark.parametrize("sym", [False, True])
def test_dequantize_closed_form_indexing(sym):
    """Hand-built packed/scales/zeros whose products (q − z)·s are exact in bf16:
    dequantize must place each value at its (row, k)."""
    rng = np.random.default_rng(3 + sym)
    N, K, g = 5, 192, 64
    G = K // g
    q = rng.integers(-8, 8, size=(N, K)) if sym else rng.integers(0, 16, size=(N, K))
    z = np.zeros((N, G), np.int64) if sym else rng.integers(0, 16, size=(N, G))
    s = rng.choice([8, 10, 12, 14], size=(N, G)) * 2.0 ** rng.integers(-12, 0, size=(N, G))
    packed = oracle.pack_codes(q.reshape(-1)).reshape(N, K // 2)
    # scales and zeros are exact in bf16 by construction (≤ 4 significant bits, small ints)
    S = oracle.bf16_from_f32(s.astype(np.float32))
    Z = oracle.bf16_from_f32(z.astype(np.float32))
    Wh = oracle.f32_from_bf16(oracle.dequantize(packed, S, Z, K, g, sym)).astype(np.float64)
    expect = (q - np.repeat(z, g, 1)) * np.repeat(s, g, 1)      # ≤ 8 significant bits: exact
    assert np.array_equal(Wh, expect)


# ------------------------------------------------------------------ reference matmul
def _bounded_bf16(rng, shape, emin=-6, emax=6):
    mant = rng.integers(128, 256, size=shape)                  # 8 significant bits
    e = rng.integers(emin, emax + 1, size=shape)
    sign = rng.choice([-1, 1], size=shape)
    v = sign * mant * 2.0 ** (e - 7)
    return oracle.bf16_from_f32(v.astype(np.float32))


@pytest.mark.parametrize("M,N,K", [(1, 1, 1), (3, 5, 7), (4, 16, 16), (7, 3, 33)])
def test_gemm_f64_exact_rational_bruteforce(M, N, K):
    rng = np.random.default_rng(M * 100 + N * 10 + K)
    X = _bounded_bf16(rng, (M, K))
    W = _bounded_bf16(rng, (N, K))
    Y = oracle.gemm_f64(X, W)
    xf, wf = oracle.f32_from_bf16(X), oracle.f32_from_bf16(W)
    for m in range(M):
        for n in range(N):
            exact = sum(Fraction(float(xf[m, k])) * Fraction(float(wf[n, k])) for k in range(K))
            assert Y[m, n] == float(exact)         # exact: bounded exponents fit binary64


def test_gemm_one_hot_reduces_to_dequantize():
    W = workloads.bits(workloads.make_weight(24, 256, 0.02, seed=9))
    for sym in (False, True):
        P, S, Z = oracle.quantize(W, 128, sym)
        Wh = oracle.dequantize(P, S, Z, 256, 128, sym)
        ks = np.array([0, 1, 127, 128, 200, 255])
        X = np.zeros((ks.size, 256), np.float32)
        X[np.arange(ks.size), ks] = 1.0
        Y = oracle.gemm_w4a16(oracle.bf16_from_f32(X), P, S, Z, 128, sym)
        assert np.array_equal(oracle.bf16_from_f64(Y), Wh[:, ks].T)


def test_gemm_all_ones_gives_row_sums():
    W = workloads.bits(workloads.make_weight(9, 128, 0.02, seed=4))
    P, S, Z = oracle.quantize(W, 32, False)
    Wh = oracle.f32_from_bf16(oracle.dequantize(P, S, Z, 128, 32, False))
    X = oracle.bf16_from_f32(np.ones((2, 128), np.float32))
    Y = oracle.gemm_w4a16(X, P, S, Z, 32, False)
    for n in range(9):
        exact = sum(Fraction(float(v)) for v in Wh[n])
        assert Y[0, n] == float(exact) and Y[1, n] == float(exact)


def test_gemm_sampled_equals_full():
    W = workloads.bits(workloads.make_weight(40, 384, 0.02, seed=2))
    X = workloads.bits(workloads.make_activation(5, 384, seed=3, outlier_frac=0.02,
                                                 outlier_mode="set"))
    for sym in (False, True):
        P, S, Z = oracle.quantize(W, 64, sym)
        full = oracle.gemm_w4a16(X, P, S, Z, 64, sym)
        ms = np.array([0, 4, 2, 3, 1, 4])
        ns = np.array([0, 39, 17, 5, 38, 1])
        assert np.array_equal(oracle.gemm_sampled(X, P, S, Z, 64, sym, ms, ns), full[ms, ns])


def test_quantize_rejects_bad_shapes():
    W = np.zeros((2, 96), np.uint16)
    with pytest.raises(ValueError):
        oracle.quantize(W, 64, False)           # K % g != 0


# ------------------------------------------------------------------ W8A16 (8-bit codes)
GOLDEN_W8 = os.path.join(os.path.dirname(__file__), "golden", "hand_groups_w8.json")
CASES_W8 = json.load(open(GOLDEN_W8))["cases"]


@pytest.mark.parametrize("case", CASES_W8, ids=[c["name"] for c in CASES_W8])
def test_hand_computed_group_w8(case):
    """8-bit groups worked by hand (INT8 form of "推理优化中“用精度换性能“的核心技术：量化", §3.3;
    "量化实战深入（GPTQ / AWQ / SmoothQuant / KV 量化）",
    §二 absmax with b = 8): scale bits, zero point and codes."""
    x = _f32(case["x"])
    if case["mode"] == "sym":
        s_bits, q = oracle.group_sym8(x)
        z = 0
    else:
        s_bits, z, q = oracle.group_asym8(x)
    assert s_bits == int(case["s_bits"], 16)
    assert float(oracle.f32_from_bf16(np.array([s_bits], np.uint16))[0]) == float(case["s"])
    assert z == case["z"]
    assert list(q) == case["q"]


@pytest.mark.parametrize("case", CASES_W8, ids=[c["name"] for c in CASES_W8])
def test_hand_computed_group_w8_through_matrix_path(case):
    """The same groups through quantize8/dequantize8 on a [3, 2g] matrix (two
    groups per row, in both orders): code bytes, scale and zero slots, x̂."""
    x = _f32(case["x"])
    g = x.size
    sym = case["mode"] == "sym"
    other = np.linspace(-3.0, 1.0, g).astype(np.float32)
    rows = [np.concatenate([x, other]), np.concatenate([other, x]), np.concatenate([x, x])]
    W = oracle.bf16_from_f32(np.stack(rows))
    C, S, Z = oracle.quantize8(W, g, sym)
    assert C.shape == (3, 2 * g) and S.shape == (3, 2)
    exp_codes = [int(b, 16) for b in case["codes"]]
    for r, slot in ((0, 0), (1, 1), (2, 0), (2, 1)):
        assert list(C[r, slot * g:(slot + 1) * g]) == exp_codes
        assert S[r, slot] == int(case["s_bits"], 16)
        assert float(oracle.f32_from_bf16(Z[r, slot:slot + 1])[0]) == (0.0 if sym else case["z"])
    xh = oracle.f32_from_bf16(oracle.dequantize8(C, S, Z, g, sym))
    exp = [float(v) for v in case["x_hat"]]
    assert list(xh[0, :g]) == exp and list(xh[1, g:]) == exp and list(xh[2, g:]) == exp


@pytest.mark.parametrize("g", [4, 32, 128])
def test_asym8_codes_are_nearest_grid_points(g):
    """Brute force over all 256 codes: the chosen code minimises |x − (c − z)s|,
    up to the rounding of the binary32 quotient next to a tie."""
    for x in _groups(50 + g, g, 240):
        s_bits, z, q = oracle.group_asym8(x)
        s = float(oracle.f32_from_bf16(np.array([s_bits], np.uint16))[0])
        assert 0 <= z <= 255 and np.all((q >= 0) & (q <= 255))
        if s == 0.0:
            assert np.all(q == 0) and z == 0
            continue
        xs = x.astype(np.float64)
        grid = (np.arange(256)[None, :] - z) * s
        dist = np.abs(xs[:, None] - grid)
        chosen = dist[np.arange(g), q]
        slack = np.abs(xs) * 2.0**-22 + s * 2.0**-20
        assert np.all(chosen <= dist.min(1) + slack)


@pytest.mark.parametrize("g", [4, 32, 128])
def test_sym8_codes_are_nearest_grid_points(g):
    for x in _groups(60 + g, g, 240):
        s_bits, q = oracle.group_sym8(x)
        s = float(oracle.f32_from_bf16(np.array([s_bits], np.uint16))[0])
        assert np.all((q >= -127) & (q <= 127)), "absmax/127 never reaches -128"
        if s == 0.0:
            assert np.all(q == 0)
            continue
        xs = x.astype(np.float64)
        grid = np.arange(-128, 128)[None, :] * s
        dist = np.abs(xs[:, None] - grid)
        chosen = dist[np.arange(g), q + 128]
        slack = np.abs(xs) * 2.0**-22 + s * 2.0**-20
        assert np.all(chosen <= dist.min(1) + slack)


@pytest.mark.parametrize("g", [32, 128])
def test_error_bound_half_step_w8(g):
    """|x − (q − z)s| ≤ s/2 for unclamped codes; clamped codes exceed it only by
    the bf16 rounding of s: ≤ s/2 + 255·2^-8·s.  The group minimum maps to code
    0 and the maximum to 254 or 255."""
    for x in _groups(70 + g, g, 240):
        s_bits, z, q = oracle.group_asym8(x)
        s = float(oracle.f32_from_bf16(np.array([s_bits], np.uint16))[0])
        if s == 0.0:
            continue
        err = np.abs(x.astype(np.float64) - (q - z) * s)
        inner = (q > 0) & (q < 255)
        assert np.all(err[inner] <= s / 2 * (1 + 2.0**-20))
        assert np.all(err <= s / 2 + 255 * 2.0**-8 * s)
        lo, hi = np.argmin(x), np.argmax(x)
        if x[lo] < 0:
            assert q[lo] == 0
        if x[hi] > 0:
            assert q[hi] >= 254


def test_w8_sym_zeros_and_int8_storage():
    W = workloads.bits(workloads.make_weight(37, 256, 0.02, seed=15, outlier_frac=0.05,
                                             outlier_scale=20.0))
    C, S, Z = oracle.quantize8(W, 64, sym=True)
    assert np.all(Z == 0)
    q = C.view(np.int8).astype(np.int64)               # int8 two's complement
    s = np.repeat(oracle.f32_from_bf16(S).astype(np.float64), 64, axis=1)
    x = oracle.f32_from_bf16(W).astype(np.float64)
    assert np.all(np.abs(x - q * s) <= s / 2 * (1 + 2.0**-20))
    assert q.min() >= -127


@pytest.mark.parametrize("sym", [False, True])
@pytest.mark.parametrize("e", [-9, 6])
def test_w8_power_of_two_scale_invariance(sym, e):
    W = workloads.make_weight(16, 256, 0.02, seed=8, outlier_frac=0.02, outlier_scale=20.0)
    W2 = (W.to(torch.float32) * 2.0**e).to(torch.bfloat16)     # exact scaling
    C1, S1, Z1 = oracle.quantize8(workloads.bits(W), 32, sym)
    C2, S2, Z2 = oracle.quantize8(workloads.bits(W2), 32, sym)
    assert np.array_equal(C1, C2) and np.array_equal(Z1, Z2)
    assert np.array_equal(oracle.f32_from_bf16(S1) * np.float32(2.0**e), oracle.f32_from_bf16(S2))


@pytest.mark.parametrize("g", [32, 128, 512])       # 512 = K: per-channel
def test_w8_on_grid_matrix_is_recovered_exactly(g):
    """Closed form: W = (q − z)·s with s a power of two (|q − z| ≤ 255 already
    takes bf16's 8 significant bits) and each group using codes 0 and 255
    re-quantizes to exactly (s, z, q) and dequantizes to W."""
    rng = np.random.default_rng(100 + g)
    N, K = 6, 512
    G = K // g
    q = rng.integers(0, 256, size=(N, K))
    q[:, 1::g] = 0
    q[:, 2::g] = 255
    z = rng.integers(0, 256, size=(N, G))
    s = 2.0 ** rng.integers(-18, -6, size=(N, G)).astype(np.float64)
    x = (q - np.repeat(z, g, 1)) * np.repeat(s, g, 1)
    Wb = oracle.bf16_from_f32(x.astype(np.float32))
    assert np.array_equal(oracle.f32_from_bf16(Wb).astype(np.float64), x)
    C, S, Z = oracle.quantize8(Wb, g, sym=False)
    assert np.array_equal(oracle.f32_from_bf16(S).astype(np.float64), s)
    assert np.array_equal(oracle.f32_from_bf16(Z).astype(np.int64), z)
    assert np.array_equal(C.astype(np.int64), q)
    assert np.array_equal(oracle.dequantize8(C, S, Z, g, False), Wb)


@pytest.mark.parametrize("sym", [False, True])
def test_dequantize8_closed_form_indexing(sym):
    """Hand-built codes/scales/zeros whose products (q − z)·s are exact in bf16:
    dequantize8 must place each value at its (row, k)."""
    rng = np.random.default_rng(31 + sym)
    N, K, g = 5, 192, 64
    G = K // g
    q = rng.integers(-128, 128, size=(N, K)) if sym else rng.integers(0, 256, size=(N, K))
    z = np.zeros((N, G), np.int64) if sym else rng.integers(0, 256, size=(N, G))
    s = 2.0 ** rng.integers(-12, 0, size=(N, G)).astype(np.float64)      # powers of two
    codes = (q & 0xFF).astype(np.uint8)
    S = oracle.bf16_from_f32(s.astype(np.float32))
    Z = oracle.bf16_from_f32(z.astype(np.float32))
    Wh = oracle.f32_from_bf16(oracle.dequantize8(codes, S, Z, g, sym)).astype(np.float64)
    exp = (q - np.repeat(z, g, 1)) * np.repeat(s, g, 1)     # |q − z| ≤ 255 times a power of two
    exp_b = oracle.f32_from_bf16(oracle.bf16_from_f32(exp.astype(np.float32))).astype(np.float64)
    assert np.array_equal(exp, exp_b), "construction: (q − z)·s exact in bf16"
    assert np.array_equal(Wh, exp)


def test_w8_gemm_one_hot_and_sampled():
    W = workloads.bits(workloads.make_weight(24, 256, 0.02, seed=19))
    for sym in (False, True):
        C, S, Z = oracle.quantize8(W, 128, sym)
        Wh = oracle.dequantize8(C, S, Z, 128, sym)
        ks = np.array([0, 1, 127, 128, 200, 255])
        X = np.zeros((ks.size, 256), np.float32)
        X[np.arange(ks.size), ks] = 1.0
        Y = oracle.gemm_w8a16(oracle.bf16_from_f32(X), C, S, Z, 128, sym)
        assert np.array_equal(oracle.bf16_from_f64(Y), Wh[:, ks].T)
        Xr = workloads.bits(workloads.make_activation(3, 256, 20))
        Yf = oracle.gemm_w8a16(Xr, C, S, Z, 128, sym)
        ms, ns = np.array([0, 2, 1, 2]), np.array([0, 23, 7, 11])
        assert np.array_equal(oracle.gemm_w8a16_sampled(Xr, C, S, Z, 128, sym, ms, ns), Yf[ms, ns])


# ------------------------------------------------------------------ per-K activation scale
def _rand_bf16(shape, seed, scale=1.0):
    x = np.random.default_rng(seed).standard_normal(shape).astype(np.float32) * np.float32(scale)
    return oracle.bf16_from_f32(x)


def test_activation_scale_by_one_is_identity():
    X = _rand_bf16((5, 96), 1)
    a = oracle.bf16_from_f32(np.ones(96, np.float32))
    assert np.array_equal(oracle.scale_activations(X, a), X)


def test_activation_scale_by_powers_of_two_is_exact():
    X = _rand_bf16((7, 128), 2)
    e = np.random.default_rng(3).integers(-20, 21, 128)
    a = oracle.bf16_from_f32((2.0 ** e).astype(np.float32))
    got = oracle.f32_from_bf16(oracle.scale_activations(X, a)).astype(np.float64)
    exp = oracle.f32_from_bf16(X).astype(np.float64) * 2.0 ** e      # exact
    assert np.array_equal(got, exp)


def test_activation_scale_rounds_the_exact_product_once():
    """x·a of two bf16 values is exact in binary64; the result must be that
    product rounded once to bf16 (not a double rounding, not a truncation)."""
    X = _rand_bf16((16, 512), 4)
    a = _rand_bf16((512,), 5, 3.0)
    exact = oracle.f32_from_bf16(X).astype(np.float64) * oracle.f32_from_bf16(a).astype(np.float64)
    assert np.array_equal(oracle.scale_activations(X, a), oracle.bf16_from_f64(exact))


def test_act_scaled_gemm_one_hot():
    """One-hot rows of X select a[k]·x̂[n, k], exact in binary64."""
    W = workloads.bits(workloads.make_weight(24, 256, 0.02, seed=21))
    P, S, Z = oracle.quantize(W, 64, False)
    Wh = oracle.f32_from_bf16(oracle.dequantize(P, S, Z, 256, 64, False)).astype(np.float64)
    a = _rand_bf16((256,), 6, 2.0)
    ks = np.array([0, 3, 63, 64, 200, 255])
    X = np.zeros((ks.size, 256), np.float32)
    X[np.arange(ks.size), ks] = 1.0
    Y = oracle.gemm_w4a16_act_scaled(oracle.bf16_from_f32(X), a, P, S, Z, 64, False)
    af = oracle.f32_from_bf16(a).astype(np.float64)
    assert np.array_equal(Y, (Wh[:, ks] * af[ks]).T)


@pytest.mark.parametrize("sym", [False, True])
def test_equivalent_scaling_identity(sym):
    """The identity the activation scale serves ((X/s)·(s·W) = X·W): with s a
    power of two constant over each weight group, quantizing s·W gives the same
    codes and scales multiplied by s, so X·diag(1/s) against them reproduces
    the unscaled result exactly."""
    N, K, g = 12, 256, 32
    W = workloads.make_weight(N, K, 0.02, seed=22, outlier_frac=0.02, outlier_scale=20.0)
    e = np.repeat(np.random.default_rng(7).integers(-6, 7, K // g), g)
    Ws = (W.to(torch.float32) * torch.tensor(2.0 ** e, dtype=torch.float32)).to(torch.bfloat16)
    X = workloads.bits(workloads.make_activation(3, K, 8))
    a = oracle.bf16_from_f32((2.0 ** -e).astype(np.float32))
    P, S, Z = oracle.quantize(workloads.bits(W), g, sym)
    Ps, Ss, Zs = oracle.quantize(workloads.bits(Ws), g, sym)
    Y = oracle.gemm_w4a16(X, P, S, Z, g, sym)
    Ysc = oracle.gemm_w4a16_act_scaled(X, a, Ps, Ss, Zs, g, sym)
    assert np.array_equal(Y, Ysc)


# ---------------------------------------------------------------------------- W8A8
# Per-token INT8 activations × per-channel INT8 weights (oracle.quantize_act8,
# oracle.gemm_w8a8): pinned to hand-computed rows, nearest-grid-point brute
# force, invariants, and exact rational / independent library evaluations of
# the integer GEMM.

W8A8_ROWS = json.load(open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden",
                                        "hand_rows_w8a8.json")))["rows"]


def _bf16_bits_of(values):
    return torch.tensor([float(v) for v in values], dtype=torch.float32).to(
        torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("row", W8A8_ROWS, ids=[r["name"] for r in W8A8_ROWS])
def test_w8a8_hand_computed_rows(row):
    X = _bf16_bits_of(row["x"]).reshape(1, -1)
    q, s = oracle.quantize_act8(X)
    assert float(s[0]) == float(row["s"])
    assert q[0].tolist() == row["q"]


def test_w8a8_rows_are_independent():
    """Each token gets its own scale: the hand rows quantized together, zero-padded
    to one width, give each row's own hand result."""
    width = max(len(r["x"]) for r in W8A8_ROWS)
    X = np.stack([np.pad(_bf16_bits_of(r["x"]), (0, width - len(r["x"]))) for r in W8A8_ROWS])
    q, s = oracle.quantize_act8(X)
    for i, r in enumerate(W8A8_ROWS):
        assert float(s[i]) == float(r["s"])
        assert q[i, :len(r["q"])].tolist() == r["q"] and not q[i, len(r["q"]):].any()


def _act_rows(seed, M=6, K=97):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((M, K)) * np.exp(rng.uniform(-6, 6, (M, 1)))
    x[1, 7] *= 300.0                                   # an outlier channel in one token
    x[2] = 0.0                                         # an all-zero token
    return torch.tensor(x, dtype=torch.float32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("seed", [1, 2, 3])
def test_w8a8_codes_are_the_nearest_grid_point(seed):
    """Brute force over all 256 codes with exact rationals: q minimizes |x − s·q|
    (ties to the even code); the binary32 quotient may decide a near-tie either
    way, so within 2^-18 of a tie both neighbours are accepted."""
    X = _act_rows(seed)
    q, s = oracle.quantize_act8(X)
    xs = oracle.f32_from_bf16(X)
    for m in range(X.shape[0]):
        S = Fraction(float(s[m]))
        if S == 0:
            assert not q[m].any()
            continue
        for k in range(X.shape[1]):
            x = Fraction(float(xs[m, k]))
            best = min(range(-128, 128), key=lambda c: (abs(x - S * c), c % 2))
            r = x / S
            near_tie = abs(r - (r.numerator // r.denominator) - Fraction(1, 2)) < Fraction(1, 2 ** 18)
            assert q[m, k] == best or (near_tie and abs(int(q[m, k]) - best) == 1), (m, k)


def test_w8a8_absmax_maps_to_127_and_errors_are_bounded():
    X = _act_rows(4)
    q, s = oracle.quantize_act8(X)
    xs = oracle.f32_from_bf16(X).astype(np.float64)
    for m in range(X.shape[0]):
        if s[m] == 0:
            continue
        k = int(np.argmax(np.abs(xs[m])))
        assert abs(int(q[m, k])) == 127 and np.sign(q[m, k]) == np.sign(xs[m, k])
        err = np.abs(xs[m] - float(s[m]) * q[m].astype(np.float64))
        assert np.all(err <= 0.5 * float(s[m]) * (1 + 2 ** -20))


def test_w8a8_power_of_two_scaling_and_sign_symmetry():
    X = _act_rows(5)
    q, s = oracle.quantize_act8(X)
    xs = oracle.f32_from_bf16(X)
    for k in (-3, 5):
        X2 = torch.tensor(xs * 2.0 ** k).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        q2, s2 = oracle.quantize_act8(X2)
        assert np.array_equal(q2, q) and np.array_equal(s2, s * np.float32(2.0 ** k))
    Xn = torch.tensor(-xs).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    qn, sn = oracle.quantize_act8(Xn)
    assert np.array_equal(qn, -q) and np.array_equal(sn, s)


def test_w8a8_gemm_exact_rational_bruteforce():
    rng = np.random.default_rng(6)
    M, N, K = 3, 5, 9
    qx = rng.integers(-128, 128, (M, K)).astype(np.int8)
    qw = rng.integers(-128, 128, (N, K)).astype(np.int8)
    sx = (rng.standard_normal(M) * 0.01).astype(np.float32)
    sw = _bf16_bits_of(rng.standard_normal(N) * 0.003)
    Y = oracle.gemm_w8a8(qx, sx, qw, sw)
    swv = oracle.f32_from_bf16(sw)
    for m in range(M):
        for n in range(N):
            exact = Fraction(float(sx[m])) * Fraction(float(swv[n])) * sum(
                int(qx[m, k]) * int(qw[n, k]) for k in range(K))
            assert abs(Fraction(Y[m, n]) - exact) <= abs(exact) * Fraction(1, 2 ** 50)


def test_w8a8_gemm_matches_numpy_on_dequantized_operands():
    """numpy's float64 matmul of (s_x·q_x) and (s_w·q_w) — every product exact in
    binary64 — against the oracle's exact integer sum times the scales."""
    rng = np.random.default_rng(7)
    M, N, K = 7, 33, 256
    X = torch.tensor(rng.standard_normal((M, K)), dtype=torch.float32).to(torch.bfloat16)
    W = torch.tensor(rng.standard_normal((N, K)) * 0.02, dtype=torch.float32).to(torch.bfloat16)
    Xb = X.view(torch.int16).numpy().view(np.uint16)
    Wb = W.view(torch.int16).numpy().view(np.uint16)
    qw, sw, _ = oracle.quantize8(Wb, K, True)
    qw = qw.view(np.int8)
    qx, sx = oracle.quantize_act8(Xb)
    Y = oracle.gemm_w8a8(qx, sx, qw, sw)
    ref = (sx[:, None].astype(np.float64) * qx) @ (oracle.f32_from_bf16(sw).reshape(-1, 1).astype(np.float64) * qw).T
    assert np.allclose(Y, ref, rtol=1e-12, atol=1e-12 * np.max(np.abs(ref)))
    assert np.allclose(oracle.gemm_w8a8_from_bf16(Xb, qw, sw), Y, rtol=0, atol=0)


def test_w8a8_gemm_one_hot_and_saturated_cases():
    K, N = 64, 4
    rng = np.random.default_rng(8)
    qw = rng.integers(-128, 128, (N, K)).astype(np.int8)
    sw = _bf16_bits_of([0.5, 0.25, 2.0, 1.0])
    # one-hot token: x = c at k0 -> s_x = |c|/127, q = ±127 there
    X = np.zeros((1, K), dtype=np.float32)
    X[0, 11] = -3.0
    Xb = torch.tensor(X).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    Y = oracle.gemm_w8a8_from_bf16(Xb, qw, sw)
    sx = np.float32(3.0) / np.float32(127.0)
    want = [float(sx) * w * (-127) * int(qw[n, 11]) for n, w in enumerate([0.5, 0.25, 2.0, 1.0])]
    assert np.allclose(Y[0], want, rtol=1e-15, atol=0)
    # every code 127: the integer sum is 127²·K exactly
    big = np.full((1, 4096), 127, dtype=np.int8)
    Y2 = oracle.gemm_w8a8(big, np.ones(1, np.float32), big, _bf16_bits_of([1.0]))
    assert Y2[0, 0] == 127 * 127 * 4096


def test_w8a8_sampled_equals_full_product():
    rng = np.random.default_rng(9)
    M, N, K = 5, 7, 160
    qx = rng.integers(-128, 128, (M, K)).astype(np.int8)
    qw = rng.integers(-128, 128, (N, K)).astype(np.int8)
    sx = (rng.standard_normal(M) * 0.01).astype(np.float32)
    sw = _bf16_bits_of(rng.standard_normal(N) * 0.003)
    Y = oracle.gemm_w8a8(qx, sx, qw, sw)
    ms, ns = np.meshgrid(np.arange(M), np.arange(N), indexing="ij")
    Ys = oracle.gemm_w8a8_sampled(qx, sx, qw, sw, ms.ravel(), ns.ravel())
    assert np.array_equal(Ys, Y.ravel())
