"""Thin ctypes binding of libw4a16 (argument marshalling only).

The functions carry the C ABI's names.  Tensors are PyTorch tensors (PyTorch supplies device
memory and streams); every step of the computation runs in the library's CUDA kernels.  There is
no fallback: if libw4a16.so is missing or fails to load, every call raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libw4a16.so")

W4_OK = 0
STATUS_NAMES = {
    0: "W4_OK", 1: "W4_ERR_NULL", 2: "W4_ERR_SHAPE", 3: "W4_ERR_ALIGN", 4: "W4_ERR_UNSUPPORTED",
    5: "W4_ERR_WORKSPACE", 6: "W4_ERR_CUDA", 7: "W4_ERR_DEVICE_TIMEOUT", 8: "W4_ERR_RANGE",
}
VARIANT_AUTO, VARIANT_SKINNY, VARIANT_TC, VARIANT_GEMV, VARIANT_GEMV_TC = 0, 1, 2, 3, 4
FLAG_WEIGHTS_STATIC = 0x100

# Entry points declared in include/w4a16.h: (name, restype, argtypes)
_P, _I64, _I32, _SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
SIGNATURES = {
    "w4_quantize_pack": (_I32, [_P, _I64, _I64, _I32, _P, _P, _P, _P, _P]),
    "w4_gemm_workspace_size": (_I32, [_I64, _I64, _I64, _I32, ctypes.POINTER(_SZ)]),
    "w4_gemm": (_I32, [_P, _I64, _I64, _I64, _P, _P, _P, _I32, _P, _P, _SZ, _P]),
    "w4_gemm_ex": (_I32, [_P, _I64, _I64, _I64, _P, _P, _P, _I32, _P, _P, _SZ, _I32, _P]),
    "w4_gemm_host": (_I32, [_P, _I64, _I64, _I64, _P, _P, _P, _I32, _P, _P, _P, _P, _SZ, _I32, _P]),
    "w4_gemm_host_batch": (_I32, [_P, _I32, _I32, _P, _P, _SZ, _P, _P, _SZ, _P, _SZ, _I32, _P]),
    "w4_gemm_plan": (_I32, [_I64, _I64, _I64, _I32, _I32, _P, _P, ctypes.POINTER(ctypes.c_int),
                            ctypes.POINTER(ctypes.c_int)]),
    "awq_workspace_size": (_I32, [_I64, _I64, _I64, _I32, _I32, ctypes.POINTER(_SZ)]),
    "awq_scale_search": (_I32, [_P, _I64, _P, _I64, _I64, _I32, _I32, _P, _P, _P, _P, _SZ, _P]),
    "awq_scale_search_noalloc": (_I32, [_P, _I64, _P, _I64, _I64, _I32, _I32, _P, _P, _P, _P]),
    "awq_gram_workspace_size": (_I32, [_I64, _I64, _I64, _I32, _I32, ctypes.POINTER(_SZ)]),
    "awq_scale_search_gram": (_I32, [_P, _I64, _P, _I64, _I64, _I32, _I32, _P, _P, _P, _P, _SZ, _P]),
    "gptq_workspace_size": (_I32, [_I64, _I64, _I64, _I32, ctypes.POINTER(_SZ)]),
    "gptq_quantize": (_I32, [_P, _I64, _P, _I64, _I64, _I32, ctypes.c_double, _P, _P, _P, _P, _SZ, _P]),
    "gptq_quantize_ex": (_I32, [_P, _I64, _P, _I64, _I64, _I32, _I32, ctypes.c_double, _I32, _P, _P, _P, _P, _P,
                                _P, _SZ, _P]),
    "w4_quantize_pack_bits": (_I32, [_P, _I64, _I64, _I32, _I32, _P, _P, _P, _P, _P]),
    "wb_gemm_workspace_size": (_I32, [_I64, _I64, _I64, _I32, _I32, ctypes.POINTER(_SZ)]),
    "wb_gemm": (_I32, [_P, _I64, _I64, _I64, _P, _P, _P, _I32, _I32, _P, _P, _SZ, _P]),
    "w4_act_prepare": (_I32, [_P, _I64, _I64, _P, _P, _P, _P]),
    "awq_colsum": (_I32, [_P, _I64, _I64, _P, _P]),
    "awq_scales_from_colsum": (_I32, [_P, _I64, _I64, _I32, _P, _P]),
    "awq_sse_workspace_size": (_I32, [_I64, _I64, _I64, _I32, _I32, ctypes.POINTER(_SZ)]),
    "awq_sse": (_I32, [_P, _I64, _P, _I64, _I64, _I32, _I32, _P, _P, _P, _SZ, _P]),
    "awq_select": (_I32, [_P, _I32, _I32, _I64, _I64, _P, _I64, _P, _P, _P, _P]),
    "w4_selftest_bounded_wait": (_I32, [ctypes.c_uint64, _P]),
    "awq_clip_workspace_size": (_I32, [_I64, _I64, _I64, _I32, _I32, ctypes.POINTER(_SZ)]),
    "awq_clip_search": (_I32, [_P, _I64, _P, _I64, _I64, _I32, _I32, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "w4_check_device_status": (_I32, [_P]),
    "w4_status_string": (ctypes.c_char_p, [_I32]),
}

_lib = None


class W4Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}")


def lib() -> ctypes.CDLL:
    """The loaded libw4a16 (raises if it has not been built or cannot be loaded)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libw4a16.so not built ({LIB_PATH}); run "
                               "`python -m weight_only_int4_06_b200.build_lib`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _check(st: int, where: str):
    if st != W4_OK:
        raise W4Error(st, where)


def _stream(stream):
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(stream)


def _dev(t: torch.Tensor, dtype, name):
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def w4_quantize_pack(W: torch.Tensor, act_scale: torch.Tensor | None = None, group: int = 128,
                     stream=None):
    """Returns (packed [N, K/8] int32 (uint32 bits), scales [N, K/group] fp16, zeros [N, K/group] uint8)."""
    N, K = W.shape
    G = K // group if group else 0
    packed = torch.empty((N, K // 8), dtype=torch.int32, device=W.device)
    scales = torch.empty((N, G), dtype=torch.float16, device=W.device)
    zeros = torch.empty((N, G), dtype=torch.uint8, device=W.device)
    a = _dev(act_scale, torch.float32, "act_scale") if act_scale is not None else None
    st = lib().w4_quantize_pack(_dev(W, torch.float16, "W"), N, K, group, a,
                                ctypes.c_void_p(packed.data_ptr()), ctypes.c_void_p(scales.data_ptr()),
                                ctypes.c_void_p(zeros.data_ptr()), _stream(stream))
    _check(st, "w4_quantize_pack")
    return packed, scales, zeros


def w4_gemm_workspace_size(M: int, N: int, K: int, group: int = 128) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().w4_gemm_workspace_size(M, N, K, group, ctypes.byref(n)), "w4_gemm_workspace_size")
    return n.value


def w4_gemm_plan(M: int, N: int, K: int, group: int = 128, variant: int = VARIANT_AUTO, scales=None,
                 zeros=None) -> tuple[int, int]:
    """(kernel family, kernel launches) of a w4_gemm call with these arguments (no device work).
    scales / zeros: the metadata tensors the call will use (their alignment matters), or None."""
    fam, n = ctypes.c_int(0), ctypes.c_int(0)
    sp = ctypes.c_void_p(scales.data_ptr()) if scales is not None else None
    zp = ctypes.c_void_p(zeros.data_ptr()) if zeros is not None else None
    _check(lib().w4_gemm_plan(M, N, K, group, variant, sp, zp, ctypes.byref(fam), ctypes.byref(n)), "w4_gemm_plan")
    return fam.value, n.value


def w4_gemm(X: torch.Tensor, packed: torch.Tensor, scales: torch.Tensor, zeros: torch.Tensor,
            group: int = 128, out: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
            variant: int = VARIANT_AUTO, stream=None) -> torch.Tensor:
    """Y = X . dequant(W)^T.

    Device X: Y is written to `out` (or a new device tensor) on `stream`; nothing synchronises.
    Host X (ideally pinned): X is copied to the device on `stream`.  If `out` is a pinned host
    tensor, Y is copied into it asynchronously on `stream` and the call returns at once (`out` is
    valid after the stream synchronises); otherwise the call synchronises and returns Y on the host.
    """
    host = not X.is_cuda
    dev = packed.device
    M, K = X.shape
    N = packed.shape[0]
    if stream is None:
        tstream = torch.cuda.current_stream(dev)
    elif isinstance(stream, torch.cuda.Stream):
        tstream = stream
    else:
        tstream = torch.cuda.ExternalStream(stream, device=dev)
    host_out = out is not None and not out.is_cuda
    if host_out and (not host or not out.is_pinned()):
        raise ValueError("a host `out` must be pinned and needs a host X")
    with torch.cuda.stream(tstream):
        Xd = X.to(dev, non_blocking=True) if host else X
        Yd = out if (out is not None and not host_out) else torch.empty((M, N), dtype=torch.float16,
                                                                          device=dev)
        need = _ws_size(M, N, K, group)
        if need and (workspace is None or workspace.numel() * workspace.element_size() < need):
            workspace = torch.empty(need, dtype=torch.uint8, device=dev)
        ws_ptr = ctypes.c_void_p(workspace.data_ptr()) if workspace is not None else None
        ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
        st = lib().w4_gemm_ex(_dev(Xd, torch.float16, "X"), M, N, K, _dev(packed, torch.int32, "packed"),
                              _dev(scales, torch.float16, "scales"), _dev(zeros, torch.uint8, "zeros"),
                              group, _dev(Yd, torch.float16, "Y"), ws_ptr, ws_bytes, variant,
                              ctypes.c_void_p(tstream.cuda_stream))
        _check(st, "w4_gemm")
        if host_out:
            if out.dtype != torch.float16 or tuple(out.shape) != (M, N):
                raise ValueError("out must be float16 [M, N]")
            out.copy_(Yd, non_blocking=True)
            return out
        if host:
            return Yd.to("cpu", non_blocking=False)
    return Yd


def w4_gemm_host(X_host: torch.Tensor, packed: torch.Tensor, scales: torch.Tensor, zeros: torch.Tensor,
                 out_host: torch.Tensor, x_dev: torch.Tensor, y_dev: torch.Tensor, group: int = 128,
                 workspace: torch.Tensor | None = None, variant: int = VARIANT_AUTO, stream=None) -> torch.Tensor:
    """One C-ABI call: copy X_host to x_dev, GEMM into y_dev, copy y_dev to out_host, all enqueued on
    `stream` (no synchronisation; out_host is valid once the stream has drained).  Host tensors
    should be pinned; x_dev / y_dev are caller-owned device staging buffers."""
    M, K = X_host.shape
    N = packed.shape[0]
    for t, name, shape in ((X_host, "X_host", (M, K)), (out_host, "out_host", (M, N))):
        if t.is_cuda or t.dtype != torch.float16 or not t.is_contiguous() or tuple(t.shape) != shape:
            raise ValueError(f"{name} must be a contiguous float16 host tensor of shape {shape}")
    if x_dev.numel() < M * K or y_dev.numel() < M * N:
        raise ValueError("x_dev / y_dev too small")
    need = _ws_size(M, N, K, group)
    if need and (workspace is None or workspace.numel() * workspace.element_size() < need):
        raise ValueError("workspace too small: see w4_gemm_workspace_size")
    ws_ptr = workspace.data_ptr() if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = lib().w4_gemm_host(X_host.data_ptr(), M, N, K, _dev(packed, torch.int32, "packed"),
                            _dev(scales, torch.float16, "scales"), _dev(zeros, torch.uint8, "zeros"), group,
                            out_host.data_ptr(), _dev(x_dev, torch.float16, "x_dev"),
                            _dev(y_dev, torch.float16, "y_dev"), ws_ptr, ws_bytes, variant, _stream(stream))
    _check(st, "w4_gemm_host")
    return out_host


class HostGemmCall:
    """A w4_gemm_host call whose arguments are checked and marshalled once, for loops that reuse
    the same buffers (a serving loop refills X_host and reads out_host between runs).

    run() makes the one C call -- copy X_host to x_dev, GEMM into y_dev, copy y_dev to out_host,
    enqueued on the stream chosen at construction, no synchronisation -- without re-validating or
    re-converting the arguments.  The tensors are kept alive by this object; they must keep their
    storage (no resize) for as long as it is used."""

    def __init__(self, X_host: torch.Tensor, packed: torch.Tensor, scales: torch.Tensor, zeros: torch.Tensor,
                 out_host: torch.Tensor, x_dev: torch.Tensor, y_dev: torch.Tensor, group: int = 128,
                 workspace: torch.Tensor | None = None, variant: int = VARIANT_AUTO, stream=None):
        M, K = X_host.shape
        N = packed.shape[0]
        for t, name, shape in ((X_host, "X_host", (M, K)), (out_host, "out_host", (M, N))):
            if t.is_cuda or t.dtype != torch.float16 or not t.is_contiguous() or tuple(t.shape) != shape:
                raise ValueError(f"{name} must be a contiguous float16 host tensor of shape {shape}")
        if x_dev.numel() < M * K or y_dev.numel() < M * N:
            raise ValueError("x_dev / y_dev too small")
        need = _ws_size(M, N, K, group)
        if need and (workspace is None or workspace.numel() * workspace.element_size() < need):
            raise ValueError("workspace too small: see w4_gemm_workspace_size")
        ws_ptr = ctypes.c_void_p(workspace.data_ptr()) if workspace is not None else None
        ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
        self._fn = lib().w4_gemm_host
        self._args = (ctypes.c_void_p(X_host.data_ptr()), ctypes.c_int64(M), ctypes.c_int64(N), ctypes.c_int64(K),
                      _dev(packed, torch.int32, "packed"), _dev(scales, torch.float16, "scales"),
                      _dev(zeros, torch.uint8, "zeros"), ctypes.c_int32(group), ctypes.c_void_p(out_host.data_ptr()),
                      _dev(x_dev, torch.float16, "x_dev"), _dev(y_dev, torch.float16, "y_dev"), ws_ptr,
                      ctypes.c_size_t(ws_bytes), ctypes.c_int32(variant), _stream(stream))
        self._keep = (X_host, packed, scales, zeros, out_host, x_dev, y_dev, workspace)
        self.out_host = out_host

    def run(self) -> torch.Tensor:
        st = self._fn(*self._args)
        if st != W4_OK:
            raise W4Error(st, "w4_gemm_host")
        return self.out_host


class GemmLayer(ctypes.Structure):
    """One layer of w4_gemm_host_batch (the C struct w4_gemm_layer)."""
    _fields_ = [("M", ctypes.c_int64), ("N", ctypes.c_int64), ("K", ctypes.c_int64),
                ("packed", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("zeros", ctypes.c_void_p),
                ("x_offset", ctypes.c_int64), ("y_offset", ctypes.c_int64)]


def _align16(n: int) -> int:
    return (n + 15) // 16 * 16


class HostGemmBatch:
    """w4_gemm_host_batch over fixed buffers: every layer's X is packed into one pinned host buffer
    (x_host, 16-byte aligned regions in layer order) and every Y into another (y_host); run() makes
    the one C call: one host-to-device copy, the layers' GEMMs, one device-to-host copy, enqueued
    on the stream chosen at construction, no synchronisation.

    weights: [(packed, scales, zeros)] device tensors per layer; shapes: [(M, K, N)] per layer.
    x(i) / y(i) are views of layer i's input and result inside the host buffers."""

    def __init__(self, weights, shapes, group: int = 128, workspace: torch.Tensor | None = None,
                 variant: int = VARIANT_AUTO, stream=None):
        if len(weights) != len(shapes) or not shapes:
            raise ValueError("one (packed, scales, zeros) per layer shape")
        self.shapes = [tuple(int(v) for v in sh) for sh in shapes]
        self.x_off, self.y_off, xo, yo = [], [], 0, 0
        for (M, K, N) in self.shapes:
            self.x_off.append(xo)
            self.y_off.append(yo)
            xo += _align16(2 * M * K)
            yo += _align16(2 * M * N)
        self.x_bytes, self.y_bytes = xo, yo
        self.x_host = torch.empty(max(xo, 16), dtype=torch.uint8).pin_memory()
        self.y_host = torch.empty(max(yo, 16), dtype=torch.uint8).pin_memory()
        self.x_dev = torch.empty(max(xo, 16), dtype=torch.uint8, device="cuda")
        self.y_dev = torch.empty(max(yo, 16), dtype=torch.uint8, device="cuda")
        arr = (GemmLayer * len(self.shapes))()
        for i, ((p, sc, z), (M, K, N)) in enumerate(zip(weights, self.shapes)):
            if tuple(p.shape) != (N, K // 8) or tuple(sc.shape) != (N, K // group):
                raise ValueError(f"layer {i}: weights do not match shape (M={M}, K={K}, N={N})")
            arr[i] = GemmLayer(M, N, K, _dev(p, torch.int32, "packed").value, _dev(sc, torch.float16, "scales").value,
                               _dev(z, torch.uint8, "zeros").value, self.x_off[i], self.y_off[i])
        need = max(_ws_size(M, N, K, group) for (M, K, N) in self.shapes)
        if need and workspace is None:  # the largest layer's partial tiles (held by this object)
            workspace = torch.empty(need, dtype=torch.uint8, device="cuda")
        if need and workspace.numel() * workspace.element_size() < need:
            raise ValueError("workspace too small: see w4_gemm_workspace_size")
        ws_ptr = ctypes.c_void_p(workspace.data_ptr()) if workspace is not None else None
        ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
        self._fn = lib().w4_gemm_host_batch
        self._args = (ctypes.cast(arr, ctypes.c_void_p), ctypes.c_int32(len(self.shapes)), ctypes.c_int32(group),
                      ctypes.c_void_p(self.x_host.data_ptr()), ctypes.c_void_p(self.x_dev.data_ptr()),
                      ctypes.c_size_t(self.x_bytes), ctypes.c_void_p(self.y_host.data_ptr()),
                      ctypes.c_void_p(self.y_dev.data_ptr()), ctypes.c_size_t(self.y_bytes), ws_ptr,
                      ctypes.c_size_t(ws_bytes), ctypes.c_int32(variant), _stream(stream))
        self._keep = (arr, weights, workspace)

    def x(self, i: int) -> torch.Tensor:
        M, K, _ = self.shapes[i]
        return self.x_host[self.x_off[i]:self.x_off[i] + 2 * M * K].view(torch.float16).view(M, K)

    def y(self, i: int) -> torch.Tensor:
        M, _, N = self.shapes[i]
        return self.y_host[self.y_off[i]:self.y_off[i] + 2 * M * N].view(torch.float16).view(M, N)

    def run(self):
        st = self._fn(*self._args)
        if st != W4_OK:
            raise W4Error(st, "w4_gemm_host_batch")

    def capture(self) -> "torch.cuda.CUDAGraph":
        """The batch call (both copies and every GEMM) captured once into a CUDA graph; replay() on
        the current stream then enqueues all of it with one launch.  The graph reads x_host and
        writes y_host in place, so refill x(i) and read y(i) around each replay as with run().
        Capture the graph on the stream the batch was built for (the default: the current one)."""
        self.run()  # one direct call first: kernel set-up happens outside the capture
        torch.cuda.current_stream().synchronize()
        g = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            with torch.cuda.graph(g, stream=side):
                st = lib().w4_gemm_host_batch(*self._args[:-1], ctypes.c_void_p(side.cuda_stream))
        torch.cuda.current_stream().wait_stream(side)
        if st != W4_OK:
            raise W4Error(st, "w4_gemm_host_batch (capture)")
        return g


_ws_cache: dict = {}


def _ws_size(M: int, N: int, K: int, group: int) -> int:
    key = (M, N, K, group)
    if key not in _ws_cache:
        _ws_cache[key] = w4_gemm_workspace_size(M, N, K, group)
    return _ws_cache[key]


def awq_workspace_size(T: int, N: int, K: int, group: int = 128, n_alpha: int = 20) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().awq_workspace_size(T, N, K, group, n_alpha, ctypes.byref(n)), "awq_workspace_size")
    return n.value


def awq_scale_search(X: torch.Tensor, W: torch.Tensor, n_alpha: int = 20, group: int = 128,
                     workspace: torch.Tensor | None = None, stream=None):
    """Returns (mse [n_alpha] fp64, best_idx [1] int32, best_s [K] fp32), all on the device."""
    T, K = X.shape
    N = W.shape[0]
    need = awq_workspace_size(T, N, K, group, n_alpha)
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=X.device)
    mse = torch.empty(n_alpha, dtype=torch.float64, device=X.device)
    best = torch.empty(1, dtype=torch.int32, device=X.device)
    best_s = torch.empty(K, dtype=torch.float32, device=X.device)
    st = lib().awq_scale_search(_dev(X, torch.float16, "X"), T, _dev(W, torch.float16, "W"), N, K,
                                group, n_alpha, ctypes.c_void_p(mse.data_ptr()),
                                ctypes.c_void_p(best.data_ptr()), ctypes.c_void_p(best_s.data_ptr()),
                                ctypes.c_void_p(workspace.data_ptr()),
                                workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "awq_scale_search")
    return mse, best, best_s


def awq_gram_workspace_size(T: int, N: int, K: int, group: int = 128, n_alpha: int = 20) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().awq_gram_workspace_size(T, N, K, group, n_alpha, ctypes.byref(n)), "awq_gram_workspace_size")
    return n.value


def awq_scale_search_gram(X: torch.Tensor, W: torch.Tensor, n_alpha: int = 20, group: int = 128,
                          workspace: torch.Tensor | None = None, stream=None):
    """awq_scale_search through the Gram matrix of X.  Returns (mse, best_idx, best_s) on the device."""
    T, K = X.shape
    N = W.shape[0]
    need = awq_gram_workspace_size(T, N, K, group, n_alpha)
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=X.device)
    mse = torch.empty(n_alpha, dtype=torch.float64, device=X.device)
    best = torch.empty(1, dtype=torch.int32, device=X.device)
    best_s = torch.empty(K, dtype=torch.float32, device=X.device)
    st = lib().awq_scale_search_gram(_dev(X, torch.float16, "X"), T, _dev(W, torch.float16, "W"), N, K,
                                     group, n_alpha, ctypes.c_void_p(mse.data_ptr()),
                                     ctypes.c_void_p(best.data_ptr()), ctypes.c_void_p(best_s.data_ptr()),
                                     ctypes.c_void_p(workspace.data_ptr()),
                                     workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "awq_scale_search_gram")
    return mse, best, best_s


def gptq_workspace_size(T: int, N: int, K: int, group: int = 128) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().gptq_workspace_size(T, N, K, group, ctypes.byref(n)), "gptq_workspace_size")
    return n.value


def gptq_quantize(X: torch.Tensor, W: torch.Tensor, damp: float = 0.01, group: int = 128,
                  workspace: torch.Tensor | None = None, stream=None):
    """GPTQ on one layer.  Returns (packed [N, K/8] int32 view of uint32, scales [N, K/128] fp16,
    zeros [N, K/128] uint8) on the device, in w4_quantize_pack's format."""
    T, K = X.shape
    N = W.shape[0]
    need = gptq_workspace_size(T, N, K, group)
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=X.device)
    packed = torch.empty(N, K // 8, dtype=torch.int32, device=X.device)
    scales = torch.empty(N, K // group, dtype=torch.float16, device=X.device)
    zeros = torch.empty(N, K // group, dtype=torch.uint8, device=X.device)
    st = lib().gptq_quantize(_dev(X, torch.float16, "X"), T, _dev(W, torch.float16, "W"), N, K, group,
                             float(damp), ctypes.c_void_p(packed.data_ptr()), ctypes.c_void_p(scales.data_ptr()),
                             ctypes.c_void_p(zeros.data_ptr()), ctypes.c_void_p(workspace.data_ptr()),
                             workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "gptq_quantize")
    return packed, scales, zeros


def gptq_quantize_ex(X: torch.Tensor, W: torch.Tensor, bits: int = 4, group: int = 128, damp: float = 0.01,
                     act_order: bool = False, act_scale: torch.Tensor | None = None,
                     workspace: torch.Tensor | None = None, stream=None):
    """GPTQ at `bits` in {2, 3, 4, 8}, group 64 or 128, natural or act-order.  Returns (packed
    [N, K*bits/32] int32 (uint32 bits), scales, zeros, perm [K] int32 or None), outputs in
    processing order."""
    T, K = X.shape
    N = W.shape[0]
    need = gptq_workspace_size(T, N, K, group)
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=X.device)
    packed = torch.empty(N, K * bits // 32, dtype=torch.int32, device=X.device)
    scales = torch.empty(N, K // group, dtype=torch.float16, device=X.device)
    zeros = torch.empty(N, K // group, dtype=torch.uint8, device=X.device)
    perm = torch.empty(K, dtype=torch.int32, device=X.device) if act_order else None
    st = lib().gptq_quantize_ex(_dev(X, torch.float16, "X"), T, _dev(W, torch.float16, "W"), N, K, bits, group,
                                float(damp), 1 if act_order else 0,
                                _dev(act_scale, torch.float32, "act_scale") if act_scale is not None else None,
                                ctypes.c_void_p(packed.data_ptr()),
                                ctypes.c_void_p(scales.data_ptr()), ctypes.c_void_p(zeros.data_ptr()),
                                ctypes.c_void_p(perm.data_ptr()) if perm is not None else None,
                                ctypes.c_void_p(workspace.data_ptr()), workspace.numel() * workspace.element_size(),
                                _stream(stream))
    _check(st, "gptq_quantize_ex")
    return packed, scales, zeros, perm


def w4_quantize_pack_bits(W: torch.Tensor, bits: int, group: int = 128, act_scale: torch.Tensor | None = None,
                          stream=None):
    """Returns (packed [N, K*bits/32] int32 (uint32 bits), scales [N, K/group] fp16, zeros uint8)."""
    N, K = W.shape
    packed = torch.empty((N, K * bits // 32), dtype=torch.int32, device=W.device)
    scales = torch.empty((N, K // group), dtype=torch.float16, device=W.device)
    zeros = torch.empty((N, K // group), dtype=torch.uint8, device=W.device)
    a = _dev(act_scale, torch.float32, "act_scale") if act_scale is not None else None
    st = lib().w4_quantize_pack_bits(_dev(W, torch.float16, "W"), N, K, bits, group, a,
                                     ctypes.c_void_p(packed.data_ptr()), ctypes.c_void_p(scales.data_ptr()),
                                     ctypes.c_void_p(zeros.data_ptr()), _stream(stream))
    _check(st, "w4_quantize_pack_bits")
    return packed, scales, zeros


def wb_gemm(X: torch.Tensor, packed: torch.Tensor, scales: torch.Tensor, zeros: torch.Tensor, bits: int,
            group: int = 128, workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Y = X dequant(W)^T for b-bit weights (dequantise to fp16, then the tcgen05 GEMM)."""
    M, K = X.shape
    N = scales.shape[0]
    n = ctypes.c_size_t(0)
    _check(lib().wb_gemm_workspace_size(M, N, K, bits, group, ctypes.byref(n)), "wb_gemm_workspace_size")
    if workspace is None or workspace.numel() * workspace.element_size() < n.value:
        workspace = torch.empty(max(n.value, 1), dtype=torch.uint8, device=X.device)
    Y = torch.empty((M, N), dtype=torch.float16, device=X.device)
    st = lib().wb_gemm(_dev(X, torch.float16, "X"), M, N, K, ctypes.c_void_p(packed.data_ptr()),
                       ctypes.c_void_p(scales.data_ptr()), ctypes.c_void_p(zeros.data_ptr()), bits, group,
                       ctypes.c_void_p(Y.data_ptr()), ctypes.c_void_p(workspace.data_ptr()),
                       workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "wb_gemm")
    return Y


def w4_act_prepare(X: torch.Tensor, perm: torch.Tensor | None = None, s: torch.Tensor | None = None,
                   stream=None) -> torch.Tensor:
    """X_out[m, i] = X[m, perm[i]] (optionally / s[perm[i]]) in fp16."""
    M, K = X.shape
    out = torch.empty_like(X)
    p = _dev(perm, torch.int32, "perm") if perm is not None else None
    sc = _dev(s, torch.float32, "s") if s is not None else None
    st = lib().w4_act_prepare(_dev(X, torch.float16, "X"), M, K, p, sc, ctypes.c_void_p(out.data_ptr()),
                              _stream(stream))
    _check(st, "w4_act_prepare")
    return out


def awq_colsum(X: torch.Tensor, stream=None) -> torch.Tensor:
    """[K] int64 (uint64 bits) exact column sums of |X| in units of 2^-24."""
    T, K = X.shape
    out = torch.empty(K, dtype=torch.int64, device=X.device)
    _check(lib().awq_colsum(_dev(X, torch.float16, "X"), T, K, ctypes.c_void_p(out.data_ptr()), _stream(stream)),
           "awq_colsum")
    return out


def awq_scales_from_colsum(colsum: torch.Tensor, T_total: int, n_alpha: int = 20, stream=None) -> torch.Tensor:
    """[n_alpha, K] fp32 scales from the (all-part) column sums and total row count."""
    K = colsum.shape[0]
    s_all = torch.empty(n_alpha, K, dtype=torch.float32, device=colsum.device)
    _check(lib().awq_scales_from_colsum(_dev(colsum, torch.int64, "colsum"), T_total, K, n_alpha,
                                        ctypes.c_void_p(s_all.data_ptr()), _stream(stream)), "awq_scales_from_colsum")
    return s_all


def awq_sse(X: torch.Tensor, W: torch.Tensor, s_all: torch.Tensor, group: int = 128,
            workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """[n_alpha] fp64 sums of squared output errors over this part's rows."""
    T, K = X.shape
    N = W.shape[0]
    n_alpha = s_all.shape[0]
    n = ctypes.c_size_t(0)
    _check(lib().awq_sse_workspace_size(T, N, K, group, n_alpha, ctypes.byref(n)), "awq_sse_workspace_size")
    if workspace is None or workspace.numel() * workspace.element_size() < n.value:
        workspace = torch.empty(max(n.value, 1), dtype=torch.uint8, device=X.device)
    sse = torch.empty(n_alpha, dtype=torch.float64, device=X.device)
    _check(lib().awq_sse(_dev(X, torch.float16, "X"), T, _dev(W, torch.float16, "W"), N, K, group, n_alpha,
                         _dev(s_all, torch.float32, "s_all"), ctypes.c_void_p(sse.data_ptr()),
                         ctypes.c_void_p(workspace.data_ptr()), workspace.numel() * workspace.element_size(),
                         _stream(stream)), "awq_sse")
    return sse


def awq_select(sse_by_part: torch.Tensor, T_total: int, N: int, s_all: torch.Tensor, stream=None):
    """sse_by_part [n_parts, n_alpha] fp64 -> (mse [n_alpha] fp64, best [1] int32, best_s [K] fp32)."""
    n_parts, n_alpha = sse_by_part.shape
    K = s_all.shape[1]
    mse = torch.empty(n_alpha, dtype=torch.float64, device=s_all.device)
    best = torch.empty(1, dtype=torch.int32, device=s_all.device)
    best_s = torch.empty(K, dtype=torch.float32, device=s_all.device)
    _check(lib().awq_select(_dev(sse_by_part, torch.float64, "sse_by_part"), n_parts, n_alpha, T_total, N,
                            _dev(s_all, torch.float32, "s_all"), K, ctypes.c_void_p(mse.data_ptr()),
                            ctypes.c_void_p(best.data_ptr()), ctypes.c_void_p(best_s.data_ptr()), _stream(stream)),
           "awq_select")
    return mse, best, best_s


def awq_scale_search_noalloc(X: torch.Tensor, W: torch.Tensor, n_alpha: int = 20, group: int = 128,
                             stream=None):
    """awq_scale_search without a workspace: the library's built-in scratch array is used instead
    (for callers that cannot allocate device memory).  The outputs are allocated here only for
    convenience; a caller that cannot allocate passes its own buffers to the C entry point."""
    T, K = X.shape
    N = W.shape[0]
    mse = torch.empty(n_alpha, dtype=torch.float64, device=X.device)
    best = torch.empty(1, dtype=torch.int32, device=X.device)
    best_s = torch.empty(K, dtype=torch.float32, device=X.device)
    st = lib().awq_scale_search_noalloc(_dev(X, torch.float16, "X"), T, _dev(W, torch.float16, "W"), N, K,
                                        group, n_alpha, ctypes.c_void_p(mse.data_ptr()),
                                        ctypes.c_void_p(best.data_ptr()), ctypes.c_void_p(best_s.data_ptr()),
                                        _stream(stream))
    _check(st, "awq_scale_search_noalloc")
    return mse, best, best_s


def awq_clip_workspace_size(T: int, N: int, K: int, group: int = 128, n_ratios: int = 10) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().awq_clip_workspace_size(T, N, K, group, n_ratios, ctypes.byref(n)), "awq_clip_workspace_size")
    return n.value


def awq_clip_search(X: torch.Tensor, W: torch.Tensor, act_scale: torch.Tensor | None = None,
                    n_ratios: int = 10, group: int = 128, with_err: bool = False, workspace=None, stream=None):
    """AWQ clip search.  Returns (best_idx [N, G] uint8, err [N, G, R] fp32 or None, packed, scales,
    zeros), all on X's device."""
    T, K = X.shape
    N = W.shape[0]
    G = K // group
    dev = X.device
    need = awq_clip_workspace_size(T, N, K, group, n_ratios)
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    best = torch.empty((N, G), dtype=torch.uint8, device=dev)
    err = torch.empty((N, G, n_ratios), dtype=torch.float32, device=dev) if with_err else None
    packed = torch.empty((N, K // 8), dtype=torch.int32, device=dev)
    scales = torch.empty((N, G), dtype=torch.float16, device=dev)
    zeros = torch.empty((N, G), dtype=torch.uint8, device=dev)
    a = _dev(act_scale, torch.float32, "act_scale") if act_scale is not None else None
    st = lib().awq_clip_search(_dev(X, torch.float16, "X"), T, _dev(W, torch.float16, "W"), N, K, group,
                               n_ratios, a, ctypes.c_void_p(best.data_ptr()),
                               ctypes.c_void_p(err.data_ptr()) if err is not None else None,
                               ctypes.c_void_p(packed.data_ptr()), ctypes.c_void_p(scales.data_ptr()),
                               ctypes.c_void_p(zeros.data_ptr()), ctypes.c_void_p(workspace.data_ptr()),
                               workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "awq_clip_search")
    return best, err, packed, scales, zeros


def w4_check_device_status(stream=None) -> int:
    return lib().w4_check_device_status(_stream(stream))


def w4_selftest_bounded_wait(limit_ns: int = 200_000_000, stream=None) -> None:
    """Launch the bounded-wait self-test (a wait that must time out after limit_ns)."""
    _check(lib().w4_selftest_bounded_wait(limit_ns, _stream(stream)), "w4_selftest_bounded_wait")


def w4_status_string(status: int) -> str:
    return lib().w4_status_string(status).decode()
