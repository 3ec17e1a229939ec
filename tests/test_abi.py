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
    return sorted(set(re.findall(r"\b(w(?:[48]a16|8a8)_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_abi():
    names = declared_functions()
    for n in ("w4a16_quantize", "w4a16_dequantize", "w4a16_gemm", "w4a16_gemm_ex",
              "w4a16_gemm_workspace_size", "w4a16_gemm_plan", "w4a16_status_string",
              "w4a16_device_error", "w4a16_abi_version", "w8a16_quantize", "w8a16_dequantize",
              "w8a16_gemm", "w8a16_gemm_plan", "w8a16_gemm_ex", "w8a8_quantize_activations",
              "w8a8_gemm"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", w4.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\sT\s(w(?:[48]a16|8a8)_\w+)", out))
    for name in declared_functions():
        assert name in exported, f"{name} declared in w4a16.h but not exported"
        assert hasattr(lib, name)


def test_library_is_sm100a_only_and_links_no_cudart_dso(lib):
    out = subprocess.run(["ldd", w4.LIB_PATH], capture_output=True, text=True).stdout
    assert "libcudart" not in out          # runtime linked statically


def test_status_strings_and_version(lib):
    assert lib.w4a16_abi_version() == 5
    for s in range(6):
        assert lib.w4a16_status_string(s).startswith(b"W4A16")


FAKE = 0x10000          # 16-byte aligned, never dereferenced on the host


def _gemm(lib, M=1, K=128, N=64, g=128, sym=0, X=FAKE, P=FAKE, S=FAKE, Z=FAKE, Y=FAKE,
          path=0, ctas=0, ws=FAKE, ws_bytes=1 << 30):
    return lib.w4a16_gemm_ex(X, M, K, P, S, Z, N, g, sym, Y, ws, ws_bytes, path, ctas, None)


@pytest.mark.parametrize("kw", [
    dict(g=48), dict(g=16), dict(g=256), dict(K=96), dict(K=0), dict(M=-1), dict(N=-2),
    dict(sym=2), dict(X=None), dict(P=None), dict(S=None), dict(Y=None), dict(Z=None),
    dict(X=FAKE + 8), dict(P=FAKE + 4), dict(Y=FAKE + 2), dict(S=FAKE + 2),
    dict(M=17, path=1), dict(path=3), dict(ctas=-1), dict(ctas=70000), dict(ctas=2, path=2),
    dict(K=2 ** 31),
])
def test_gemm_rejects_invalid_arguments(lib, kw):
    assert _gemm(lib, **kw) == EINVAL


def _gemm_host(lib, M=1, K=128, N=64, g=128, sym=0, Xh=FAKE, P=FAKE, S=FAKE, Z=FAKE, Yh=FAKE,
               Xd=FAKE, Yd=FAKE, ws=FAKE, ws_bytes=1 << 30, flags=0):
    return lib.w4a16_gemm_host(Xh, M, K, P, S, Z, N, g, sym, Yh, Xd, Yd, ws, ws_bytes, flags, None)


@pytest.mark.parametrize("kw", [
    dict(g=48), dict(K=96), dict(M=-1), dict(sym=2), dict(Xh=None), dict(Yh=None), dict(Xd=None),
    dict(Yd=None), dict(Xd=FAKE + 8), dict(Yd=FAKE + 2), dict(P=None), dict(S=None), dict(Z=None),
    dict(P=FAKE + 4), dict(M=17, flags=1), dict(flags=3),
])
def test_gemm_host_rejects_invalid_arguments(lib, kw):
    """The host-buffer GEMM checks everything before it queues its first copy."""
    assert _gemm_host(lib, **kw) == EINVAL


def test_gemm_host_empty_and_workspace(lib):
    assert _gemm_host(lib, M=0) == 0 and _gemm_host(lib, N=0) == 0
    # a split shape needs its workspace: too small is reported before any copy
    assert _gemm_host(lib, M=17, K=8192, N=8192, g=32, ws_bytes=16) == EWORKSPACE


@pytest.mark.parametrize("K,g,ok", [
    (4096, 4096, True), (11008, 11008, True), (96, 96, True), (512, 512, True),   # g = K
    (128, 128, True), (4096, 128, True),                                          # grouped
    (48, 48, False), (200, 200, False),          # per-channel needs K a multiple of 32
    (4096, 2048, False), (512, 256, False),      # other group sizes are not supported
])
def test_per_channel_shape_rules(lib, K, g, ok):
    """g = K selects per-channel granularity (one scale and zero per row)."""
    assert (_gemm(lib, M=0, K=K, g=g) == 0) == ok
    assert (lib.w4a16_quantize(FAKE, 0, K, g, 0, FAKE, FAKE, FAKE, None) == 0) == ok
    assert (lib.w4a16_dequantize(FAKE, FAKE, FAKE, 0, K, g, 0, FAKE, None) == 0) == ok


def test_per_channel_plans():
    """Per-channel plans cover the same units as grouped ones; the decode stage
    carries one scale/zero pair per row, so it fits at least as many stages."""
    for M, N, K in ((1, 11008, 4096), (1, 4096, 11008), (8, 8192, 28672), (16, 4096, 4096)):
        pc, gr = w4.plan(M, N, K, K), w4.plan(M, N, K, 128)
        assert pc["path"] == gr["path"] == "decode"
        assert pc["grid"] == gr["grid"] and pc["kernels"] == gr["kernels"]
        assert pc["workspace_bytes"] == gr["workspace_bytes"]
        assert pc["stages"] >= gr["stages"]
    for M, N, K in ((48, 1000, 4352), (300, 10240, 2048), (2048, 8192, 8192)):
        head, tail, splits, bm = _tc_schedule(M, N, K, K)
        p = w4.plan(M, N, K, K)
        assert p["path"] == "tensorcore" and p["grid"] == head + tail * splits


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


def test_workspace_sizes(lib):
    # tensor-core path: none with enough output tiles to fill the SMs, else S fp32
    # partial M x N results (split-K); decode: partial row blocks
    assert w4.workspace_size(4096, 8192, 8192, 32) == 0          # 1024 tiles: last wave 92% full
    p17 = w4.plan(17, 8192, 8192, 32)
    splits = p17["grid"] // ((8192 // 128) * 1)
    # 64 tiles, 2 x 148 resident slots (two CTAs per SM at 32 activation rows): 4 splits
    assert splits == 4 and p17["kernels"] == 2
    # tile-local parts: [split][tile][32 activation rows][128 weight rows] fp32
    assert w4.workspace_size(17, 8192, 8192, 32) == splits * 64 * 32 * 128 * 4
    # decode: per slot (row blocks + CTAs) 16 ready flags (rounded to 256 bytes in
    # all) and 16 warps x 32 lanes x 4·mb fp32 partial sums
    rb = 4096 // 256
    for M, mb in ((1, 1), (16, 2)):
        p = w4.plan(M, 4096, 4096, 128)
        slots = rb + p["grid"]
        assert p["workspace_bytes"] == -(-slots * 16 * 4 // 256) * 256 + slots * 16 * 32 * 16 * mb
    assert w4.workspace_size(1, 4096, 4096, 128) == w4.plan(1, 4096, 4096, 128)["workspace_bytes"]


def test_static_weights_flag_is_accepted_only_as_a_flag(lib):
    """W4A16_STATIC_WEIGHTS (0x100) may be OR'ed into the path; other high bits
    are rejected before anything is launched."""
    f = ctypes.c_void_p(FAKE)
    assert w4.plan(1, 4096, 4096, path=w4.PATH_AUTO | w4.STATIC_WEIGHTS) == w4.plan(1, 4096, 4096)
    assert lib.w4a16_gemm_ex(f, 1, 256, f, f, f, 256, 128, 0, f, f, 1 << 30, 0x200, 0, None) == EINVAL
    assert lib.w4a16_gemm_ex(f, 1, 256, f, f, f, 256, 128, 0, f, f, 1 << 30, 0x103, 0, None) == EINVAL


def test_w8a8_rejects_without_launching(lib):
    f = ctypes.c_void_p(FAKE)
    q = lib.w8a8_quantize_activations
    assert q(f, 4, 48, f, f, None) == EINVAL                  # K not a multiple of 32
    assert q(f, -1, 64, f, f, None) == EINVAL
    assert q(ctypes.c_void_p(FAKE + 2), 4, 64, f, f, None) == EINVAL
    assert q(f, 0, 64, f, f, None) == 0                       # empty: nothing launched
    gm = lib.w8a8_gemm
    assert gm(f, f, 4, 48, f, f, 16, f, None) == EINVAL
    assert gm(f, f, 4, 64, f, None, 16, f, None) == EINVAL     # missing weight scales
    assert gm(f, f, 4, 64, f, f, 16, ctypes.c_void_p(FAKE + 8), None) == EINVAL
    assert gm(f, f, 0, 64, f, f, 16, f, None) == 0
    assert gm(f, f, 4, 64, f, f, 0, f, None) == 0


def test_act_scaled_rejects_without_launching(lib):
    f = ctypes.c_void_p(FAKE)
    g = lib.w4a16_gemm_act_scaled
    assert g(f, 1, 256, None, f, f, f, 256, 128, 0, f, f, 1 << 30, None) == EINVAL     # no scale
    assert g(f, 1, 256, ctypes.c_void_p(FAKE + 2), f, f, f, 256, 128, 0, f, f, 1 << 30, None) == EINVAL
    assert g(f, 1, 250, f, f, f, f, 256, 128, 0, f, f, 1 << 30, None) == EINVAL        # K % g
    assert g(f, 0, 256, None, f, f, f, 256, 128, 0, f, f, 0, None) == 0                # M = 0


def test_act_scaled_workspace_sizes(lib):
    """Decode path: the plan's workspace (the kernel scales X itself); tensor-core
    path: that rounded up to 256 bytes plus M·K bf16 for the scaled activations."""
    f = lib.w4a16_gemm_act_scaled_workspace_size
    f.argtypes = [ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int32]
    f.restype = ctypes.c_size_t
    assert f(1, 28672, 8192, 128) == w4.workspace_size(1, 28672, 8192, 128)
    for M, N, K in ((2048, 8192, 8192), (17, 300, 1024), (4096, 8192, 8192)):
        base = w4.workspace_size(M, N, K, 128)
        assert f(M, N, K, 128) == -(-base // 256) * 256 + M * K * 2
    assert f(17, 300, 1000, 128) == 0                       # rejected shape


def test_decode_rejects_small_workspace(lib):
    need = w4.plan(1, 64, 128, 128)["workspace_bytes"]
    assert need > 0
    assert _gemm(lib, ws_bytes=need - 1) == EWORKSPACE
    assert _gemm(lib, ws=None) == EINVAL
    assert _gemm(lib, ws=FAKE + 8) == EINVAL


def test_dispatch_plans():
    assert w4.plan(1, 11008, 4096)["path"] == "decode"
    assert w4.plan(16, 4096, 11008)["path"] == "decode"
    assert w4.plan(17, 4096, 4096)["path"] == "tensorcore"
    p = w4.plan(2048, 8192, 8192)
    # 512 tiles on 148 SMs: three full waves unsplit, the 68-tile last wave split in two
    assert p["path"] == "tensorcore" and p["tile_m"] == 256 and p["grid"] == 444 + 68 * 2
    assert p["smem_bytes"] <= 232448 and p["kernels"] == 3
    assert p["workspace_bytes"] == 2 * 68 * 256 * 128 * 4
    for M, bm in ((17, 32), (32, 32), (33, 64), (64, 64), (65, 128), (128, 128), (129, 256)):
        assert w4.plan(M, 8192, 8192)["tile_m"] == bm
    for M in (1, 8):
        assert w4.plan(M, 4096, 4096)["tile_m"] == 8
    assert w4.plan(9, 4096, 4096)["tile_m"] == 16


def _tc_schedule(M, N, K, g, sm_count=148):
    """Mirror of the tensor-core launch schedule: (head tiles, tail tiles, splits)."""
    bm = 32 if M <= 32 else 64 if M <= 64 else 128 if M <= 128 else 256
    sms = sm_count * (2 if bm <= 64 else 1)            # resident CTA slots
    tiles = -(-N // 128) * -(-M // bm)
    num_kb = -(-K // 64)
    tail = tiles if tiles < sms else (tiles % sms if 0 < tiles % sms <= sms // 2 else 0)
    s = max(1, min(sms // tail, 8, num_kb // 4)) if tail else 1
    slab = g // 8 if (K // g) % 8 == 0 else 1
    kbs = -(-(-(-num_kb // s)) // slab) * slab
    splits = -(-num_kb // kbs)
    if splits < 2:
        return tiles, 0, 1, bm
    return tiles - tail, tail, splits, bm


@pytest.mark.parametrize("M,N,K,g", [(17, 8192, 8192, 32), (64, 4096, 4096, 128), (256, 11008, 4096, 64),
                                     (2048, 8192, 8192, 128), (4096, 8192, 8192, 128),
                                     (1024, 28672, 8192, 128), (20, 37, 96, 32), (200, 4096, 1152, 32)])
def test_tensorcore_schedule(M, N, K, g):
    head, tail, splits, bm = _tc_schedule(M, N, K, g)
    p = w4.plan(M, N, K, g, path="tensorcore")
    assert p["tile_m"] == bm
    assert p["grid"] == head + tail * splits
    assert p["kernels"] == (1 if head else 0) + (2 if tail else 0)
    assert p["workspace_bytes"] == (splits * tail * bm * 128 * 4 if tail else 0)


def test_decode_persistent_grid_and_smem():
    for M, N, K in ((1, 11008, 4096), (1, 4096, 11008), (1, 28672, 8192), (8, 8192, 28672),
                    (16, 8192, 8192), (1, 256, 256)):
        p = w4.plan(M, N, K)
        units = -(-N // 256) * -(-K // 256)
        assert p["grid"] == min(units, 148)                    # one CTA per SM
        assert p["smem_bytes"] <= 232448 and p["stages"] >= 2 and p["kernels"] == 1
        assert p["threads"] == 576 and p["tile_n"] == 256
    # the M=1 workloads keep at least five stages of 32 KB in flight per SM
    assert w4.plan(1, 28672, 8192)["stages"] >= 5 and w4.plan(1, 28672, 8192)["grid"] == 148
    # forced grid sizes: any positive count, capped at the units and at one resident wave
    assert w4.plan(1, 4096, 11008, ctas=7)["grid"] == 7
    assert w4.plan(1, 64, 1024, ctas=50)["grid"] == 4          # 1 row block x 4 K blocks
    assert w4.plan(1, 28672, 8192, ctas=5000)["grid"] == 148
    with pytest.raises(w4.W4A16Error):
        w4.plan(17, 4096, 4096, path="decode")
    with pytest.raises(w4.W4A16Error):
        w4.plan(64, 4096, 4096, path="tensorcore", ctas=4)


@pytest.mark.parametrize("M", list(range(1, 17)))
def test_decode_stage_layout_is_valid_for_every_shape(M):
    """The library refuses (W4A16_EUNSUPPORTED) a decode plan whose stage layout
    breaks its invariants — TMA destinations 128-byte aligned, the codes tile
    1024-byte aligned, the ring within one CTA's shared memory — so planning
    every M, g and a spread of K and N here checks the layout arithmetic."""
    for K in (32, 64, 96, 128, 160, 256, 384, 1024, 1056, 2304, 4096, 4352, 5376, 11008, 28672):
        for g in (32, 64, 128, K):
            if K % g:
                continue
            for N in (1, 128, 1000, 28672):
                p = w4.plan(M, N, K, g, False, "decode")
                assert p["stages"] >= 2 and p["smem_bytes"] <= 232448


@pytest.mark.parametrize("M", list(range(1, 17)))
def test_w8_decode_stage_layout_is_valid_for_every_shape(M):
    """The same layout checks for the decode kernel with 8-bit codes (units of
    256 rows x 128 K, X rows of 256 bytes, the pair-copy mode for one scale group
    per unit): every M, g and a spread of K and N plans without EUNSUPPORTED."""
    for K in (32, 64, 96, 128, 160, 256, 384, 1024, 1056, 2304, 4096, 4352, 5376, 11008, 28672):
        for g in (32, 64, 128, K):
            if K % g:
                continue
            for N in (1, 128, 1000, 28672):
                p = w4.plan8(M, N, K, g, False)
                assert p == w4.plan8(M, N, K, g, False, path="decode")
                assert p["path"] == "decode" and p["stages"] >= 2 and p["smem_bytes"] <= 232448
                assert p["threads"] == 576 and p["grid"] == min(148, -(-N // 256) * -(-K // 128))
    assert w4.plan8(17, 4096, 4096)["path"] == "tensorcore"


def _owner(u, U, C):
    return ((u + 1) * C - 1) // U


@pytest.mark.parametrize("U,C", [(10, 3), (1376, 296), (1408, 296), (7, 7), (5, 1), (100, 99)])
def test_stream_k_partition_arithmetic(U, C):
    """The kernel's split u_c = floor(c·U/C) and its inverse owner(u): every
    unit has exactly one owner, owners are contiguous and non-decreasing, and
    the partial-sum slot rb + c of a split row block never collides."""
    starts = [c * U // C for c in range(C + 1)]
    for c in range(C):
        for u in range(starts[c], starts[c + 1]):
            assert _owner(u, U, C) == c
    for kbn in (1, 3, 4, 11):
        if U % kbn:
            continue
        rbs = U // kbn
        used = set()
        for rb in range(rbs):
            cf, cl = _owner(rb * kbn, U, C), _owner(rb * kbn + kbn - 1, U, C)
            for c in range(cf, cl + 1):
                slot = rb + c
                assert slot not in used and slot < rbs + C
                used.add(slot)


def _walk(u0, u1, kbn):
    """Mirror of the decode kernel's unit visiting order (UnitWalk)."""
    rb_first = u0 // kbn
    rb, kb = rb_first, u0 - rb_first * kbn
    rb_last = (u1 - 1) // kbn
    kb_last_end = (u1 - 1) - rb_last * kbn + 1
    two, phase, out = rb_last != rb_first, 0, []
    for i in range(u1 - u0):
        if i > 0:
            if phase == 0 and two and kb == kbn - 1:
                phase, rb, kb = 1, rb_last, 0
            elif phase == 1 and kb == kb_last_end - 1:
                phase, rb, kb = 2, rb_first + 1, 0
            elif phase == 2 and kb == kbn - 1:
                rb, kb = rb + 1, 0
            else:
                kb += 1
        if phase == 0:
            end = (kb == kbn - 1) if two else (kb == kb_last_end - 1)
        elif phase == 1:
            end = kb == kb_last_end - 1
        else:
            end = kb == kbn - 1
        out.append((rb, kb, end))
    return out


@pytest.mark.parametrize("kbn", [1, 2, 3, 4, 8, 11, 28])
def test_stream_k_unit_walk(kbn):
    """Each CTA visits its units exactly once, each row block contiguously,
    and marks the end of every row block it touches exactly once (after its
    last unit there): the split first and last segments come first."""
    for rbs in (1, 2, 3, 7, 20):
        U = rbs * kbn
        for C in range(1, min(U, 40) + 1):
            for c in range(C):
                u0, u1 = c * U // C, (c + 1) * U // C
                w = _walk(u0, u1, kbn)
                assert sorted(rb * kbn + kb for rb, kb, _ in w) == list(range(u0, u1))
                for rb in set(r for r, _, _ in w):
                    idx = [i for i, (r, _, _) in enumerate(w) if r == rb]
                    assert idx == list(range(idx[0], idx[-1] + 1))
                    assert [i for i in idx if w[i][2]] == [idx[-1]]


def _decode_events(U, C, kbn):
    """Per CTA, in visiting order, what it does at each row-block end: 'store'
    (whole row block), 'publish' (its part of a split row block, for the first
    owner) or 'finish' (first owner: wait for the other parts, add, store)."""
    ev = {}
    for c in range(C):
        u0, u1 = c * U // C, (c + 1) * U // C
        out = []
        for rb, kb, end in _walk(u0, u1, kbn):
            if not end:
                continue
            first = rb * kbn
            if first >= u0 and first + kbn <= u1:
                out.append(("store", rb))
            elif _owner(first, U, C) == c:
                out.append(("finish", rb))
            else:
                out.append(("publish", rb))
        ev[c] = out
    return ev


@pytest.mark.parametrize("kbn", [1, 2, 4, 11, 16, 32, 43])
def test_decode_split_row_blocks_finish_once_and_never_deadlock(kbn):
    """Every row block is stored exactly once; a split row block is finished by
    its first owner after every other owner publishes a part; and every CTA
    publishes all its parts before it waits for any, so with all CTAs resident
    every wait ends (the waited-for CTAs never wait first)."""
    for rbs in (1, 2, 3, 7, 20, 33):
        U = rbs * kbn
        for C in sorted({1, 2, 3, 5, 7, 13, 40, 97, 296, U} & set(range(1, U + 1))):
            ev = _decode_events(U, C, kbn)
            stored = [rb for c in range(C) for kind, rb in ev[c] if kind in ("store", "finish")]
            assert sorted(stored) == list(range(rbs))
            for rb in range(rbs):
                cf, cl = _owner(rb * kbn, U, C), _owner(rb * kbn + kbn - 1, U, C)
                pubs = sorted(c for c in range(C) for kind, r in ev[c] if kind == "publish" and r == rb)
                assert pubs == list(range(cf + 1, cl + 1))
            for c in range(C):
                kinds = [k for k, _ in ev[c]]
                if "finish" in kinds and "publish" in kinds:
                    assert max(i for i, k in enumerate(kinds) if k == "publish") < kinds.index("finish")


def test_decode_plan_reports_split_row_blocks():
    U_rows, kbn = -(-4096 // 256), -(-4096 // 256)
    p = w4.plan(1, 4096, 4096, 128)
    U, C = U_rows * kbn, p["grid"]
    cut = {(b * U // C) // kbn for b in range(1, C) if (b * U // C) % kbn}
    assert p["split_tiles"] == len(cut) > 0
    assert w4.plan(1, 4096, 4096, 128, ctas=U_rows)["split_tiles"] == 0   # one row block per CTA
    assert w4.plan(2048, 8192, 8192)["split_tiles"] == 68                  # the tensor-core tail


# ------------------------------------------------------------------ W8A16 entry points
def test_w8a16_entry_points_reject_invalid(lib):
    q, d, gm = lib.w8a16_quantize, lib.w8a16_dequantize, lib.w8a16_gemm
    assert q(FAKE, 4, 128, 48, 0, FAKE, FAKE, FAKE, None) == EINVAL          # g not supported
    assert q(FAKE, 4, 200, 200, 0, FAKE, FAKE, FAKE, None) == EINVAL         # per-channel K % 32
    assert q(FAKE, 4, 128, 128, 0, FAKE, FAKE, None, None) == EINVAL         # asym needs zeros
    assert q(FAKE + 8, 4, 128, 128, 1, FAKE, FAKE, None, None) == EINVAL     # misaligned W
    assert q(FAKE, 4, 128, 128, 2, FAKE, FAKE, FAKE, None) == EINVAL         # bad mode
    assert q(FAKE, 0, 128, 128, 0, FAKE, FAKE, FAKE, None) == 0              # N = 0: nothing to do
    assert q(FAKE, 0, 4096, 4096, 0, FAKE, FAKE, FAKE, None) == 0            # per-channel accepted
    assert d(FAKE, FAKE, None, 4, 128, 128, 0, FAKE, None) == EINVAL
    assert d(FAKE, FAKE, FAKE, 4, 128, 32, 0, FAKE + 2, None) == EINVAL
    assert d(FAKE, FAKE, FAKE, 0, 96, 96, 0, FAKE, None) == 0
    X = S = Z = Y = FAKE
    big = 1 << 30
    assert gm(X, -1, 128, FAKE, S, Z, 64, 128, 0, Y, FAKE, big, None) == EINVAL
    assert gm(X, 1, 96, FAKE, S, Z, 64, 128, 0, Y, FAKE, big, None) == EINVAL      # K % g
    assert gm(X + 8, 1, 128, FAKE, S, Z, 64, 128, 0, Y, FAKE, big, None) == EINVAL
    assert gm(X, 1, 128, FAKE, S, None, 64, 128, 0, Y, FAKE, big, None) == EINVAL
    assert gm(X, 0, 128, FAKE, S, Z, 64, 128, 0, Y, FAKE, big, None) == 0         # empty: no launch
    assert gm(X, 4, 128, FAKE, S, Z, 0, 128, 0, Y, FAKE, big, None) == 0
    ws = lib.w8a16_gemm_workspace_size
    # M ≤ 16: the decode kernel with 8-bit codes; its workspace depends on the row
    # blocks and the grid only, so it equals the INT4 one when both grids are full
    assert ws(16, 4096, 4096, 128) == w4.workspace_size(16, 4096, 4096, 128) > 0
    assert ws(17, 8192, 8192, 32) == w4.workspace_size(17, 8192, 8192, 32) > 0
    assert ws(2048, 8192, 8192, 128) == w4.workspace_size(2048, 8192, 8192, 128)


@pytest.mark.parametrize("compiler,std", [("gcc", "-std=c99"), ("g++", "-std=c++11")])
def test_header_compiles_as_plain_c_and_cpp(tmp_path, compiler, std):
    """The public header is a C ABI: it must compile as strict C99 (no C++
    constructs leaking in) as well as C++, and every declared entry point must be
    callable through it."""
    calls = "\n".join(f"    (void){n};" for n in declared_functions())
    src = tmp_path / ("use.c" if compiler == "gcc" else "use.cpp")
    src.write_text('#include "w4a16.h"\nint main(void) {\n' + calls + "\n    return 0;\n}\n")
    r = subprocess.run([compiler, std, "-Wall", "-Werror", "-pedantic", "-fsyntax-only",
                        "-I", os.path.dirname(HEADER), str(src)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


def test_plain_c_program_links_and_plans(tmp_path):
    """A C program linked against the library (no Python, no torch) can call the
    host-only entry points: version, status strings, plans and workspace sizes."""
    src = tmp_path / "plan.c"
    src.write_text(r'''
#include <stdio.h>
#include "w4a16.h"
int main(void) {
    w4a16_plan p;
    if (w4a16_abi_version() != W4A16_ABI_VERSION) return 1;
    if (w4a16_gemm_plan(1, 11008, 4096, 128, 0, W4A16_PATH_AUTO, 0, &p) != W4A16_OK) return 2;
    printf("%d %lld %d %lld\n", p.path, (long long)p.grid, p.kernels, (long long)p.workspace_bytes);
    if (w4a16_gemm_plan(17, 4096, 4096, 48, 0, W4A16_PATH_AUTO, 0, &p) != W4A16_EINVAL) return 3;
    printf("%zu %zu\n", w4a16_gemm_workspace_size(2048, 8192, 8192, 128),
           w8a16_gemm_workspace_size(2048, 8192, 8192, 128));
    printf("%s\n", w4a16_status_string(W4A16_EWORKSPACE));
    return 0;
}
''')
    exe = tmp_path / "plan"
    libdir = os.path.dirname(w4.LIB_PATH)
    subprocess.run(["gcc", "-std=c99", "-I", os.path.dirname(HEADER), str(src), "-o", str(exe),
                    "-L", libdir, "-lw4a16", f"-Wl,-rpath,{libdir}"], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0, (out.returncode, out.stderr)
    lines = out.stdout.split("\n")
    path, grid, kernels, ws = map(int, lines[0].split())
    p = w4.plan(1, 11008, 4096, 128)
    assert (path, grid, kernels, ws) == (1, p["grid"], p["kernels"], p["workspace_bytes"])
    a, b = map(int, lines[1].split())
    assert a == b == w4.workspace_size(2048, 8192, 8192, 128)
    assert lines[2].startswith("W4A16_EWORKSPACE")
