"""W4A16 weight-only RTN quantization and fused INT4 x bf16 GEMM for B200 (sm_100a).

A thin binding over the C ABI in ``include/w4a16.h`` (``libw4a16.so``, built
in-tree by ``python -m weight_only_quantization_rtn_b200.build``).  PyTorch is
used only for device memory and the current CUDA stream; every step of the
computation runs in the library's CUDA kernels.  There is no CPU fallback:
the first call raises ImportError if the library is missing.

    packed, scales, zeros = quantize(W, g=128, sym=False)   # W: bf16 [N, K] on cuda
    Y = gemm(X, packed, scales, zeros, g=128, sym=False)      # X: bf16 [M, K] -> Y [M, N]
    W_hat = dequantize(packed, scales, zeros, g=128, sym=False)
"""
from __future__ import annotations

import contextlib
import ctypes
import os

import torch

__all__ = ["lib", "quantize", "dequantize", "gemm", "gemm_decode_noalloc", "plan", "plan8",
           "quantize8", "dequantize8", "gemm8", "quantize_act8", "gemm_w8a8", "linear_w8a8",
           "workspace_size", "device_error", "W4A16Error", "PATH_AUTO", "PATH_DECODE", "PATH_TENSORCORE", "STATIC_WEIGHTS", "LIB_PATH"]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libw4a16.so")

# W4A16_ABI_VERSION in include/w4a16.h that the argument lists below follow
ABI_VERSION = 5
PATH_AUTO, PATH_DECODE, PATH_TENSORCORE = 0, 1, 2
STATIC_WEIGHTS = 0x100   # W4A16_STATIC_WEIGHTS, OR'ed into the path argument
_PATHS = {"auto": PATH_AUTO, "decode": PATH_DECODE, "tensorcore": PATH_TENSORCORE}
_STATUS = {0: "OK", 1: "EINVAL", 2: "EUNSUPPORTED", 3: "ECUDA", 4: "EWORKSPACE", 5: "EDEVICE"}


class W4A16Error(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {lib().w4a16_status_string(status).decode()}")


class Plan(ctypes.Structure):
    _fields_ = [("path", ctypes.c_int32), ("tile_m", ctypes.c_int32),
                ("tile_n", ctypes.c_int32), ("threads", ctypes.c_int32),
                ("grid", ctypes.c_int64), ("smem_bytes", ctypes.c_int32),
                ("stages", ctypes.c_int32), ("kernels", ctypes.c_int32),
                ("workspace_bytes", ctypes.c_int64), ("split_tiles", ctypes.c_int64)]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"W4A16 CUDA library not built: {LIB_PATH} is missing "
                          "(run `python -m weight_only_quantization_rtn_b200.build`)")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_size_t
    lib.w4a16_quantize.argtypes = [vp, i64, i64, i32, i32, vp, vp, vp, vp]
    lib.w4a16_dequantize.argtypes = [vp, vp, vp, i64, i64, i32, i32, vp, vp]
    lib.w4a16_gemm_workspace_size.argtypes = [i64, i64, i64, i32]
    lib.w4a16_gemm_workspace_size.restype = sz
    lib.w4a16_gemm.argtypes = [vp, i64, i64, vp, vp, vp, i64, i32, i32, vp, vp, sz, vp]
    lib.w4a16_gemm_ex.argtypes = [vp, i64, i64, vp, vp, vp, i64, i32, i32, vp, vp, sz, i32, i32,
                                  vp]
    lib.w4a16_gemm_plan.argtypes = [i64, i64, i64, i32, i32, i32, i32, ctypes.POINTER(Plan)]
    lib.w4a16_gemm_act_scaled.argtypes = [vp, i64, i64, vp, vp, vp, vp, i64, i32, i32, vp, vp, sz,
                                          vp]
    lib.w4a16_gemm_act_scaled_workspace_size.argtypes = [i64, i64, i64, i32]
    lib.w4a16_gemm_act_scaled_workspace_size.restype = sz
    lib.w4a16_gemm_host.argtypes = [vp, i64, i64, vp, vp, vp, i64, i32, i32, vp, vp, vp, vp, sz,
                                    i32, vp]
    lib.w4a16_gemm_host.restype = ctypes.c_int
    lib.w4a16_gemm_decode_noalloc.argtypes = [vp, i64, i64, vp, vp, vp, i64, i32, i32, vp, vp]
    lib.w4a16_gemm_decode_noalloc.restype = ctypes.c_int
    lib.w4a16_device_error.argtypes = [ctypes.POINTER(ctypes.c_int32)]
    lib.w4a16_status_string.argtypes = [ctypes.c_int]
    lib.w4a16_status_string.restype = ctypes.c_char_p
    lib.w4a16_abi_version.restype = ctypes.c_int32
    lib.w8a16_quantize.argtypes = [vp, i64, i64, i32, i32, vp, vp, vp, vp]
    lib.w8a16_dequantize.argtypes = [vp, vp, vp, i64, i64, i32, i32, vp, vp]
    lib.w8a16_gemm.argtypes = [vp, i64, i64, vp, vp, vp, i64, i32, i32, vp, vp, sz, vp]
    lib.w8a16_gemm_workspace_size.argtypes = [i64, i64, i64, i32]
    lib.w8a16_gemm_plan.argtypes = [i64, i64, i64, i32, i32, i32, ctypes.POINTER(Plan)]
    lib.w8a16_gemm_ex.argtypes = [vp, i64, i64, vp, vp, vp, i64, i32, i32, vp, vp, sz, i32, vp]
    lib.w8a8_quantize_activations.argtypes = [vp, i64, i64, vp, vp, vp]
    lib.w8a8_gemm.argtypes = [vp, vp, i64, i64, vp, vp, i64, vp, vp]
    lib.w8a16_gemm_workspace_size.restype = sz
    for name in ("w4a16_quantize", "w4a16_dequantize", "w4a16_gemm", "w4a16_gemm_ex",
                 "w4a16_gemm_act_scaled",
                 "w4a16_gemm_plan", "w4a16_device_error", "w8a16_quantize", "w8a16_dequantize",
                 "w8a16_gemm", "w8a16_gemm_plan", "w8a16_gemm_ex",
                 "w8a8_quantize_activations", "w8a8_gemm"):
        getattr(lib, name).restype = ctypes.c_int
    if lib.w4a16_abi_version() != ABI_VERSION:
        raise ImportError(f"{LIB_PATH} has ABI version {lib.w4a16_abi_version()}, this binding "
                          f"expects {ABI_VERSION}: rebuild it")
    return lib


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded C library; raises ImportError if it has not been built."""
    global _lib
    if _lib is None:
        _lib = _load()
    return _lib


_NO_CONTEXT = contextlib.nullcontext()     # reusable: holds no state


def _check(status: int, what: str) -> None:
    if status != 0:
        raise W4A16Error(status, what)


def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(dev: torch.device):
    return ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)


def _need(t: torch.Tensor, dtype: torch.dtype, name: str, ndim: int = 2) -> None:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != ndim:
        raise ValueError(f"{name} must be {ndim}-D, got shape {tuple(t.shape)}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be on a CUDA device")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _same_device(dev: torch.device, **tensors) -> None:
    for name, t in tensors.items():
        if t is not None and t.device != dev:
            raise ValueError(f"{name} is on {t.device}, the weights are on {dev}")


def quantize(W: torch.Tensor, g: int = 128, sym: bool = False):
    """Group-wise RTN quantization of W[N, K] (bf16, cuda); g = K quantizes per
    channel (one scale and zero per row).

    Returns (packed uint8 [N, K/2], scales bf16 [N, K/g], zeros bf16 [N, K/g]);
    zeros are all 0 when ``sym``."""
    _need(W, torch.bfloat16, "W")
    N, K = W.shape
    if g <= 0 or K % g:
        raise ValueError(f"K={K} must be a multiple of g={g}")
    packed = torch.empty((N, K // 2), dtype=torch.uint8, device=W.device)
    scales = torch.empty((N, K // g), dtype=torch.bfloat16, device=W.device)
    zeros = torch.empty((N, K // g), dtype=torch.bfloat16, device=W.device)
    with torch.cuda.device(W.device):
        _check(lib().w4a16_quantize(_ptr(W), N, K, g, int(bool(sym)), _ptr(packed), _ptr(scales),
                                   _ptr(zeros), _stream(W.device)), "w4a16_quantize")
    return packed, scales, zeros


def dequantize(packed: torch.Tensor, scales: torch.Tensor, zeros: torch.Tensor | None,
               g: int = 128, sym: bool = False, out: torch.Tensor | None = None) -> torch.Tensor:
    """Ŵ[N, K] = bf16_rn((q − z)·s), materialised (the unfused form)."""
    _need(packed, torch.uint8, "packed")
    _need(scales, torch.bfloat16, "scales")
    if not sym:
        _need(zeros, torch.bfloat16, "zeros")
    N, K = packed.shape[0], packed.shape[1] * 2
    if out is None:
        W_hat = torch.empty((N, K), dtype=torch.bfloat16, device=packed.device)
    else:
        _need(out, torch.bfloat16, "out")
        if tuple(out.shape) != (N, K):
            raise ValueError("out has the wrong shape")
        W_hat = out
    with torch.cuda.device(packed.device):
        _check(lib().w4a16_dequantize(_ptr(packed), _ptr(scales), _ptr(zeros if not sym else None),
                                     N, K, g, int(bool(sym)), _ptr(W_hat),
                                     _stream(packed.device)), "w4a16_dequantize")
    return W_hat


def workspace_size(M: int, N: int, K: int, g: int) -> int:
    return int(lib().w4a16_gemm_workspace_size(M, N, K, g))


def _plan_dict(p) -> dict:
    return {"path": {v: k for k, v in _PATHS.items()}[p.path], "tile_m": p.tile_m,
            "tile_n": p.tile_n, "grid": p.grid, "threads": p.threads,
            "smem_bytes": p.smem_bytes, "stages": p.stages, "kernels": p.kernels,
            "workspace_bytes": p.workspace_bytes, "split_tiles": p.split_tiles}


def plan(M: int, N: int, K: int, g: int = 128, sym: bool = False, path: str | int = "auto",
         ctas: int = 0) -> dict:
    """The launch w4a16_gemm would make for this shape (host only)."""
    p = Plan()
    pid = _PATHS[path] if isinstance(path, str) else int(path)
    _check(lib().w4a16_gemm_plan(M, N, K, g, int(bool(sym)), pid, ctas, ctypes.byref(p)),
           "w4a16_gemm_plan")
    return _plan_dict(p)


def plan8(M: int, N: int, K: int, g: int = 128, sym: bool = False,
          path: str | int = "auto") -> dict:
    """The launch w8a16_gemm_ex would make for this shape and path (host only)."""
    p = Plan()
    pid = _PATHS[path] if isinstance(path, str) else int(path)
    _check(lib().w8a16_gemm_plan(M, N, K, g, int(bool(sym)), pid, ctypes.byref(p)),
           "w8a16_gemm_plan")
    return _plan_dict(p)


_workspaces: dict = {}
_plan_bytes: dict = {}


def _workspace_bytes(dev: torch.device, M, N, K, g, sym, pid, ctas) -> int:
    """Workspace of the plan for this shape on this device, asked of the library
    once per distinct call shape (plans depend only on the shape, the forced
    kernel and grid, and the device's SM count)."""
    key = (dev.index, M, N, K, g, bool(sym), pid, ctas)
    nbytes = _plan_bytes.get(key)
    if nbytes is None:
        nbytes = plan(M, N, K, g, sym, pid, ctas)["workspace_bytes"] if M and N else 0
        _plan_bytes[key] = nbytes
    return nbytes


def _workspace(dev: torch.device, nbytes: int, sid: int | None = None):
    """A scratch buffer per (device, stream), grown on demand; calls on one
    stream never overlap, so they can share it.  ``sid``: the current stream's
    handle when the caller has it already."""
    if nbytes == 0:
        return None
    key = (dev, torch.cuda.current_stream(dev).cuda_stream if sid is None else sid)
    ws = _workspaces.get(key)
    if ws is None or ws.numel() < nbytes:
        ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)
        _workspaces[key] = ws
    return ws


_dev_bufs: dict = {}


def _device_buffer(dev: torch.device, M: int, N: int, sid: int, tag: str = "y") -> torch.Tensor:
    """A device bf16 [M, N] buffer per (device, stream, shape, role) for calls
    whose operands live in host memory (``tag`` "x": the copied activations, "y":
    the result); calls on one stream are ordered, so they can share it."""
    key = (dev, sid, M, N, tag)
    buf = _dev_bufs.get(key)
    if buf is None:
        buf = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        _dev_bufs[key] = buf
    return buf


def gemm(X: torch.Tensor, packed: torch.Tensor, scales: torch.Tensor,
         zeros: torch.Tensor | None, g: int = 128, sym: bool = False, path: str | int = "auto",
         ctas: int = 0, out: torch.Tensor | None = None, sync: bool = True,
         act_scale: torch.Tensor | None = None, static_weights: bool = False) -> torch.Tensor:
    """Fused W4A16 GEMM: Y[M, N] = X[M, K] · Ŵ[N, K]ᵀ (bf16 in/out, fp32 accumulation).

    ``static_weights``: the kernel before this call on the stream does not write
    ``packed``, ``scales`` or ``zeros`` (inference with fixed weights), so the
    decode kernel may start streaming them while that kernel drains
    (W4A16_STATIC_WEIGHTS).  Not for a call right after quantizing on the same
    stream.

    ``act_scale`` (bf16 [K] on the weights' device): multiply each activation
    by its input channel's scale as it is loaded, X'[m, k] = bf16_rn(X[m, k]·a[k])
    (w4a16_gemm_act_scaled; the automatic kernel choice only).

    If X lives in host memory (ideally pinned) it is copied to the weights'
    device and Y is copied back into host memory — ``out`` when given (a pinned
    bf16 [M, N] host tensor), else new pinned memory: the end-to-end form of the
    call.  With ``sync`` (the default) the call waits for that copy; with
    ``sync=False`` it returns at once and the caller synchronizes the current
    stream before reading Y (e.g. once per step of several calls)."""
    host_in = not X.is_cuda
    dev = packed.device
    if (host_in and act_scale is None and not ctas and X.is_pinned()
            and (out is None or out.is_pinned())):
        return _gemm_host(X, packed, scales, zeros, g, sym, path, out, sync, static_weights)
    Xd = X.to(dev, non_blocking=True) if host_in else X
    _need(Xd, torch.bfloat16, "X")
    _need(packed, torch.uint8, "packed")
    _need(scales, torch.bfloat16, "scales")
    if not sym:
        _need(zeros, torch.bfloat16, "zeros")
    M, K = Xd.shape
    N = packed.shape[0]
    if packed.shape[1] * 2 != K:
        raise ValueError(f"packed has K={packed.shape[1] * 2}, X has K={K}")
    _same_device(dev, X=Xd, scales=scales, zeros=None if sym else zeros)
    stream = torch.cuda.current_stream(dev)      # looked up once per call: host overhead
    sid = stream.cuda_stream
    host_out = None
    if host_in:
        if out is not None:
            if out.is_cuda or out.dtype != torch.bfloat16 or tuple(out.shape) != (M, N) \
                    or not out.is_contiguous():
                raise ValueError("out must be a contiguous bf16 [M, N] host tensor when X is on the host")
            host_out = out
        out = _device_buffer(dev, M, N, sid)
    elif out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    else:
        _need(out, torch.bfloat16, "out")
        if tuple(out.shape) != (M, N):
            raise ValueError("out has the wrong shape")
        _same_device(dev, out=out)
    pid = _PATHS[path] if isinstance(path, str) else int(path)
    if act_scale is not None:
        _need(act_scale, torch.bfloat16, "act_scale", ndim=1)
        if act_scale.shape[0] != K:
            raise ValueError(f"act_scale has {act_scale.shape[0]} entries, X has K={K}")
        _same_device(dev, act_scale=act_scale)
        if pid != PATH_AUTO or ctas:
            raise ValueError("act_scale uses the automatic kernel choice")
    with (torch.cuda.device(dev) if dev.index != torch.cuda.current_device() else _NO_CONTEXT):
        if act_scale is None:
            ws_bytes = _workspace_bytes(dev, M, N, K, g, sym, pid, ctas)
        else:
            key = ("act", dev.index, M, N, K, g)
            ws_bytes = _plan_bytes.get(key)
            if ws_bytes is None:
                ws_bytes = int(lib().w4a16_gemm_act_scaled_workspace_size(M, N, K, g)) if M and N else 0
                _plan_bytes[key] = ws_bytes
        ws = _workspace(dev, ws_bytes, sid)
        if act_scale is None:
            _check(lib().w4a16_gemm_ex(_ptr(Xd), M, K, _ptr(packed), _ptr(scales),
                                       _ptr(zeros if not sym else None), N, g, int(bool(sym)),
                                       _ptr(out), _ptr(ws), ws_bytes,
                                       pid | (STATIC_WEIGHTS if static_weights else 0), ctas,
                                       ctypes.c_void_p(sid)),
                   "w4a16_gemm")
        else:
            _check(lib().w4a16_gemm_act_scaled(_ptr(Xd), M, K, _ptr(act_scale), _ptr(packed),
                                               _ptr(scales), _ptr(zeros if not sym else None), N, g,
                                               int(bool(sym)), _ptr(out), _ptr(ws), ws_bytes,
                                               ctypes.c_void_p(sid)),
                   "w4a16_gemm_act_scaled")
    if host_in:
        if host_out is None:
            host_out = torch.empty((M, N), dtype=torch.bfloat16, pin_memory=True)
        host_out.copy_(out, non_blocking=True)
        if sync:
            stream.synchronize()
        return host_out
    return out


def _gemm_host(X, packed, scales, zeros, g, sym, path, out, sync, static_weights):
    """gemm() with X (and Y) in page-locked host memory: one w4a16_gemm_host call
    copies X in, multiplies and copies Y out on the current stream."""
    dev = packed.device
    if X.dtype != torch.bfloat16 or X.dim() != 2 or not X.is_contiguous():
        raise ValueError("X must be a contiguous bf16 [M, K] tensor")
    _need(packed, torch.uint8, "packed")
    _need(scales, torch.bfloat16, "scales")
    if not sym:
        _need(zeros, torch.bfloat16, "zeros")
    M, K = X.shape
    N = packed.shape[0]
    if packed.shape[1] * 2 != K:
        raise ValueError(f"packed has K={packed.shape[1] * 2}, X has K={K}")
    _same_device(dev, scales=scales, zeros=None if sym else zeros)
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, pin_memory=True)
    elif out.dtype != torch.bfloat16 or tuple(out.shape) != (M, N) or not out.is_contiguous():
        raise ValueError("out must be a contiguous bf16 [M, N] host tensor when X is on the host")
    stream = torch.cuda.current_stream(dev)
    sid = stream.cuda_stream
    pid = _PATHS[path] if isinstance(path, str) else int(path)
    with (torch.cuda.device(dev) if dev.index != torch.cuda.current_device() else _NO_CONTEXT):
        ws_bytes = _workspace_bytes(dev, M, N, K, g, sym, pid, 0)
        ws = _workspace(dev, ws_bytes, sid)
        xd = _device_buffer(dev, M, K, sid, "x")
        yd = _device_buffer(dev, M, N, sid, "y")
        _check(lib().w4a16_gemm_host(X.data_ptr(), M, K, packed.data_ptr(), scales.data_ptr(),
                                     None if sym else zeros.data_ptr(), N, g, int(bool(sym)),
                                     out.data_ptr(), xd.data_ptr(), yd.data_ptr(),
                                     None if ws is None else ws.data_ptr(), ws_bytes,
                                     pid | (STATIC_WEIGHTS if static_weights else 0), sid),
               "w4a16_gemm_host")
    if sync:
        stream.synchronize()
    return out


def gemm_decode_noalloc(X: torch.Tensor, packed: torch.Tensor, scales: torch.Tensor,
                        zeros: torch.Tensor | None, g: int = 128, sym: bool = False,
                        out: torch.Tensor | None = None) -> torch.Tensor:
    """Decode-path GEMM (M ≤ 16, device tensors) through the entry point that
    allocates no device memory of its own: its split-K scratch is a fixed
    array inside the library, shared by every call, so calls must not overlap
    on the GPU.  Only ``out`` is allocated here, and only when it is None."""
    _need(X, torch.bfloat16, "X")
    _need(packed, torch.uint8, "packed")
    _need(scales, torch.bfloat16, "scales")
    if not sym:
        _need(zeros, torch.bfloat16, "zeros")
    M, K = X.shape
    N = packed.shape[0]
    dev = packed.device
    if packed.shape[1] * 2 != K:
        raise ValueError(f"packed has K={packed.shape[1] * 2}, X has K={K}")
    _same_device(dev, X=X, scales=scales, zeros=None if sym else zeros)
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    else:
        _need(out, torch.bfloat16, "out")
        if tuple(out.shape) != (M, N):
            raise ValueError("out has the wrong shape")
        _same_device(dev, out=out)
    with torch.cuda.device(dev):
        _check(lib().w4a16_gemm_decode_noalloc(_ptr(X), M, K, _ptr(packed), _ptr(scales),
                                               _ptr(zeros if not sym else None), N, g,
                                               int(bool(sym)), _ptr(out), _stream(dev)),
               "w4a16_gemm_decode_noalloc")
    return out


# ---------------------------------------------------------------- W8A16 (8-bit codes)
def quantize8(W: torch.Tensor, g: int = 128, sym: bool = False):
    """RTN quantization of W[N, K] (bf16, cuda) to 8-bit codes, one per byte;
    g = K quantizes per channel.

    Returns (codes uint8 [N, K], scales bf16 [N, K/g], zeros bf16 [N, K/g]);
    symmetric codes are int8 two's complement and zeros are all 0."""
    _need(W, torch.bfloat16, "W")
    N, K = W.shape
    if g <= 0 or K % g:
        raise ValueError(f"K={K} must be a multiple of g={g}")
    codes = torch.empty((N, K), dtype=torch.uint8, device=W.device)
    scales = torch.empty((N, K // g), dtype=torch.bfloat16, device=W.device)
    zeros = torch.empty((N, K // g), dtype=torch.bfloat16, device=W.device)
    with torch.cuda.device(W.device):
        _check(lib().w8a16_quantize(_ptr(W), N, K, g, int(bool(sym)), _ptr(codes), _ptr(scales),
                                   _ptr(zeros), _stream(W.device)), "w8a16_quantize")
    return codes, scales, zeros


def dequantize8(codes: torch.Tensor, scales: torch.Tensor, zeros: torch.Tensor | None,
                g: int = 128, sym: bool = False, out: torch.Tensor | None = None) -> torch.Tensor:
    """Ŵ[N, K] = bf16_rn((q − z)·s) from 8-bit codes, materialised."""
    _need(codes, torch.uint8, "codes")
    _need(scales, torch.bfloat16, "scales")
    if not sym:
        _need(zeros, torch.bfloat16, "zeros")
    N, K = codes.shape
    if out is None:
        out = torch.empty((N, K), dtype=torch.bfloat16, device=codes.device)
    else:
        _need(out, torch.bfloat16, "out")
        if tuple(out.shape) != (N, K):
            raise ValueError("out has the wrong shape")
    with torch.cuda.device(codes.device):
        _check(lib().w8a16_dequantize(_ptr(codes), _ptr(scales), _ptr(zeros if not sym else None),
                                     N, K, g, int(bool(sym)), _ptr(out), _stream(codes.device)),
               "w8a16_dequantize")
    return out


def gemm8(X: torch.Tensor, codes: torch.Tensor, scales: torch.Tensor,
          zeros: torch.Tensor | None, g: int = 128, sym: bool = False,
          out: torch.Tensor | None = None, path: str | int = "auto",
          static_weights: bool = False) -> torch.Tensor:
    """Fused W8A16 GEMM: Y[M, N] = X[M, K] · Ŵ[N, K]ᵀ (bf16 in/out, fp32
    accumulation), device tensors.  M ≤ 16 runs the decode kernel with 8-bit
    codes, larger M the tensor-core kernel with 8-bit codes (each with the
    workspace the library asks for)."""
    _need(X, torch.bfloat16, "X")
    _need(codes, torch.uint8, "codes")
    _need(scales, torch.bfloat16, "scales")
    if not sym:
        _need(zeros, torch.bfloat16, "zeros")
    M, K = X.shape
    N = codes.shape[0]
    if codes.shape[1] != K:
        raise ValueError(f"codes have K={codes.shape[1]}, X has K={K}")
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=codes.device)
    dev = codes.device
    with torch.cuda.device(dev):
        pid = _PATHS[path] if isinstance(path, str) else int(path)
        key = ("w8", dev.index, M, N, K, g, pid)
        ws_bytes = _plan_bytes.get(key)
        if ws_bytes is None:
            ws_bytes = plan8(M, N, K, g, sym, pid)["workspace_bytes"] if M and N else 0
            _plan_bytes[key] = ws_bytes
        ws = _workspace(dev, ws_bytes)
        _check(lib().w8a16_gemm_ex(_ptr(X), M, K, _ptr(codes), _ptr(scales),
                                   _ptr(zeros if not sym else None), N, g, int(bool(sym)),
                                   _ptr(out), _ptr(ws), ws_bytes,
                                   pid | (STATIC_WEIGHTS if static_weights else 0), _stream(dev)),
               "w8a16_gemm")
    return out


def quantize_act8(X: torch.Tensor, out: tuple | None = None):
    """W8A8 activations: per-token INT8 (w8a8_quantize_activations).  X bf16 [M, K]
    on a device -> (q int8 [M, K], s float32 [M])."""
    _need(X, torch.bfloat16, "X")
    M, K = X.shape
    if out is None:
        q = torch.empty((M, K), dtype=torch.int8, device=X.device)
        s = torch.empty((M,), dtype=torch.float32, device=X.device)
    else:
        q, s = out
    with torch.cuda.device(X.device):
        _check(lib().w8a8_quantize_activations(_ptr(X), M, K, _ptr(q), _ptr(s), _stream(X.device)),
               "w8a8_quantize_activations")
    return q, s


def gemm_w8a8(qx: torch.Tensor, sx: torch.Tensor, qw: torch.Tensor, sw: torch.Tensor,
              out: torch.Tensor | None = None) -> torch.Tensor:
    """W8A8 GEMM on the INT8 tensor cores: Y = s_x·s_w·(q_x·q_wᵀ) (w8a8_gemm).
    qx int8 [M, K], sx float32 [M]; qw int8 (or uint8 bytes) [N, K] and sw bf16 [N]
    or [N, 1] from quantize8(W, g=K, sym=True); Y bf16 [M, N]."""
    if qx.dtype != torch.int8 or sx.dtype != torch.float32:
        raise TypeError("qx must be int8 and sx float32")
    if qw.dtype not in (torch.int8, torch.uint8) or sw.dtype != torch.bfloat16:
        raise TypeError("qw must be int8/uint8 codes and sw bf16 scales")
    M, K = qx.shape
    N = qw.shape[0]
    if qw.shape[1] != K or sx.numel() != M or sw.numel() != N:
        raise ValueError("W8A8 operand shapes disagree")
    for t in (qx, sx, qw, sw):
        if not t.is_contiguous() or t.device != qx.device:
            raise ValueError("W8A8 operands must be contiguous and on one device")
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=qx.device)
    with torch.cuda.device(qx.device):
        _check(lib().w8a8_gemm(_ptr(qx), _ptr(sx), M, K, _ptr(qw), _ptr(sw), N, _ptr(out),
                               _stream(qx.device)), "w8a8_gemm")
    return out


def linear_w8a8(X: torch.Tensor, qw: torch.Tensor, sw: torch.Tensor,
                out: torch.Tensor | None = None) -> torch.Tensor:
    """Quantize X per token, then the W8A8 GEMM (two kernels)."""
    qx, sx = quantize_act8(X)
    return gemm_w8a8(qx, sx, qw, sw, out=out)


def device_error() -> int:
    """Read and clear the device error word (0 = no kernel gave up a wait)."""
    code = ctypes.c_int32(0)
    _check(lib().w4a16_device_error(ctypes.byref(code)), "w4a16_device_error")
    return int(code.value)
