"""Python binding of libbsa, the B200 block-sparse video attention library.

Argument marshalling only: every step of the path runs in the library's CUDA kernels.
PyTorch supplies device memory and the current stream. There is no CPU fallback: if
libbsa.so is missing or the device is not a B200, the calls raise.

Entry points (same names as the C ABI in include/bsa.h):
    reorder(g, x)                   raster [B,N,H,d] -> tile-major [B,H,NT,64,d]
    reorder_pool(g, x)              the same, plus the per-tile means fp32 [B,H,NT,d]
    unreorder(g, xt)                the inverse
    build_mask(g, p, qt, kt, difficulty)     -> (mask uint32 [B,H,NQT,W], kv_count int32)
    build_mask_pooled(g, p, qbar, kbar, difficulty)   the same from the per-tile means
    sparse_attn_fwd(g, qt, kt, vt, mask, kv_count)  -> (out bf16 [B,N,H,d], lse fp32 [B,H,N])
    sparse_attn_fwd_token(g, qt, kt, vt, mask, kv_count, dense, token_radius)
                                    the same under a token-level circular support
    forward(g, p, q, k, v, difficulty)       the whole path, raster in, raster out
"""
from __future__ import annotations

import ctypes
import math
import os
import threading
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libbsa.so")

BSA_OK = 0
STATUS_NAMES = {0: "BSA_OK", 1: "BSA_ERR_INVALID_ARG", 2: "BSA_ERR_WORKSPACE",
                3: "BSA_ERR_UNSUPPORTED_DEVICE", 4: "BSA_ERR_CUDA"}
KERR_WAIT_TIMEOUT, KERR_BAD_UNIT, KERR_BAD_MASK = 1, 2, 4


class bsa_geom(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("d", ctypes.c_int),
                ("T", ctypes.c_int), ("Hs", ctypes.c_int), ("Ws", ctypes.c_int)]


class bsa_mask_params(ctypes.Structure):
    _fields_ = [("window_kind", ctypes.c_int), ("radius", ctypes.c_int), ("topk", ctypes.c_int),
                ("dense_fraction", ctypes.c_float), ("budget_mode", ctypes.c_int),
                ("budget_target", ctypes.c_float)]


class BsaError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {STATUS_NAMES.get(status, status)}")
        self.status = status


_lib = None
_lib_lock = threading.Lock()


def load_library(path: str | None = None) -> ctypes.CDLL:
    """Load libbsa.so (built in-tree by _build.py); raises if it is missing."""
    global _lib
    with _lib_lock:
        if _lib is not None and path is None:
            return _lib
        p = path or LIB_PATH
        if not os.path.exists(p):
            raise RuntimeError(f"libbsa.so not found at {p}: run `python -m "
                               "block_sparse_attention_major_b200._build` first")
        lib = ctypes.CDLL(p)
        vp, sz = ctypes.c_void_p, ctypes.c_size_t
        G, P = ctypes.POINTER(bsa_geom), ctypes.POINTER(bsa_mask_params)
        lib.bsa_status_string.restype = ctypes.c_char_p
        lib.bsa_status_string.argtypes = [ctypes.c_int]
        lib.bsa_tile_grid.restype = ctypes.c_int
        lib.bsa_tile_grid.argtypes = [G] + [ctypes.POINTER(ctypes.c_int)] * 4
        lib.bsa_workspace_bytes.restype = sz
        lib.bsa_workspace_bytes.argtypes = [G, P]
        lib.bsa_clear_error.restype = ctypes.c_int
        lib.bsa_clear_error.argtypes = [vp, vp]
        lib.bsa_reorder.restype = ctypes.c_int
        lib.bsa_reorder.argtypes = [G, vp, vp, vp]
        lib.bsa_unreorder.restype = ctypes.c_int
        lib.bsa_unreorder.argtypes = [G, vp, vp, vp]
        lib.bsa_reorder_pool.restype = ctypes.c_int
        lib.bsa_reorder_pool.argtypes = [G, vp, vp, vp, vp]
        lib.bsa_build_mask_pooled.restype = ctypes.c_int
        lib.bsa_build_mask_pooled.argtypes = [G, P, vp, vp, vp, vp, vp, vp, sz, vp]
        lib.bsa_build_mask.restype = ctypes.c_int
        lib.bsa_build_mask.argtypes = [G, P, vp, vp, vp, vp, vp, vp, sz, vp]
        lib.bsa_sparse_attn_fwd.restype = ctypes.c_int
        lib.bsa_sparse_attn_fwd.argtypes = [G, vp, vp, vp, vp, vp, ctypes.c_float, vp, vp, vp, sz, vp]
        lib.bsa_sparse_attn_fwd_token.restype = ctypes.c_int
        lib.bsa_sparse_attn_fwd_token.argtypes = [G, vp, vp, vp, vp, vp, vp, ctypes.c_int, ctypes.c_float, vp,
                                                  vp, vp, sz, vp]
        lib.bsa_route_flags_offset.restype = sz
        lib.bsa_route_flags_offset.argtypes = [G]
        lib.bsa_sparse_attn_fwd_fixed_scratch.restype = ctypes.c_int
        lib.bsa_sparse_attn_fwd_fixed_scratch.argtypes = [G, vp, vp, vp, vp, vp, ctypes.c_float, vp, vp,
                                                          vp, vp]
        lib.bsa_launch_count.restype = ctypes.c_uint64
        lib.bsa_launch_count.argtypes = []
        lib.bsa_selftest_bounded_wait.restype = ctypes.c_int
        lib.bsa_selftest_bounded_wait.argtypes = [ctypes.c_longlong, vp, vp]
        if path is None:
            _lib = lib
        return lib


@dataclass(frozen=True)
class Geometry:
    B: int
    H: int
    d: int
    T: int
    Hs: int
    Ws: int

    @property
    def N(self) -> int:
        return self.T * self.Hs * self.Ws

    @property
    def tiles(self) -> tuple[int, int, int]:
        return (-(-self.T // 4), -(-self.Hs // 4), -(-self.Ws // 4))

    @property
    def NT(self) -> int:
        a, b, c = self.tiles
        return a * b * c

    @property
    def NW(self) -> int:
        return -(-self.NT // 32)

    def c(self) -> bsa_geom:
        return bsa_geom(self.B, self.H, self.d, self.T, self.Hs, self.Ws)


@dataclass(frozen=True)
class MaskParams:
    window_kind: int = 0
    radius: int = 1
    topk: int = 0
    dense_fraction: float = 0.0
    budget_mode: int = 0
    budget_target: float = 0.0

    def c(self) -> bsa_mask_params:
        return bsa_mask_params(self.window_kind, self.radius, self.topk, self.dense_fraction,
                               self.budget_mode, self.budget_target)


def _stream(stream, device: torch.device) -> ctypes.c_void_p:
    s = torch.cuda.current_stream(device) if stream is None else stream
    if s.device != device:
        raise ValueError(f"stream is on {s.device}, the tensors on {device}")
    return ctypes.c_void_p(s.cuda_stream)


def _device_of(*tensors: torch.Tensor | None) -> torch.device:
    """The one device of the given tensors (None entries skipped). The library launches on
    the current device with the pointers it is given, so tensors of two devices, or of a
    device other than the one the call runs on, are refused here."""
    devs = [t.device for t in tensors if t is not None]
    if not devs or any(d != devs[0] for d in devs):
        raise ValueError(f"tensors of one call must share one device, got {sorted(set(map(str, devs)))}")
    return devs[0]


def _run(what: str, device: torch.device, stream, call) -> None:
    """call(stream_handle) with `device` current, so that the library's launches, its
    device queries and the stream all refer to the device that holds the tensors."""
    with torch.cuda.device(device):
        _check(call(_stream(stream, device)), what)


def _ptr(t: torch.Tensor | None) -> ctypes.c_void_p:
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _need(t: torch.Tensor, dtype, shape, name: str) -> None:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _need_ws(ws: torch.Tensor) -> None:
    if (not isinstance(ws, torch.Tensor) or not ws.is_cuda or ws.dtype != torch.uint8 or ws.dim() != 1
            or not ws.is_contiguous()):
        raise ValueError("ws must be a contiguous 1-D uint8 CUDA tensor (see alloc_workspace)")


def _check(status: int, what: str) -> None:
    if status != BSA_OK:
        raise BsaError(status, what)


def workspace_bytes(g: Geometry, p: MaskParams | None = None) -> int:
    pc = p.c() if p is not None else None
    return int(load_library().bsa_workspace_bytes(ctypes.byref(g.c()),
                                                  ctypes.byref(pc) if pc is not None else None))


def alloc_workspace(g: Geometry, device=None) -> torch.Tensor:
    """A zeroed device workspace (byte 0 = kernel error word)."""
    n = workspace_bytes(g)
    if n == 0:
        raise ValueError("invalid geometry")
    return torch.zeros(n, dtype=torch.uint8, device=device or "cuda")


def read_error(ws: torch.Tensor) -> int:
    """The kernel error word (synchronises the current stream)."""
    return int(ws[:4].view(torch.int32).item()) & 0xFFFFFFFF


def clear_error(ws: torch.Tensor, stream=None) -> None:
    _need_ws(ws)
    _run("bsa_clear_error", ws.device, stream, lambda s: load_library().bsa_clear_error(_ptr(ws), s))


def launch_count() -> int:
    return int(load_library().bsa_launch_count())


def selftest_bounded_wait(err: torch.Tensor, limit_cycles: int = 20_000_000, stream=None) -> None:
    """Run the bounded-wait self-test: a wait that nothing completes gives up after
    limit_cycles SM cycles and sets BSA_KERR_WAIT_TIMEOUT in err (int32 [1], device)."""
    _need(err, torch.int32, (1,), "err")
    _run("bsa_selftest_bounded_wait", err.device, stream,
         lambda s: load_library().bsa_selftest_bounded_wait(ctypes.c_longlong(limit_cycles), _ptr(err), s))


def reorder(g: Geometry, x: torch.Tensor, xt: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    _need(x, torch.bfloat16, (g.B, g.N, g.H, g.d), "x")
    if xt is None:
        xt = torch.empty((g.B, g.H, g.NT, 64, g.d), dtype=torch.bfloat16, device=x.device)
    _need(xt, torch.bfloat16, (g.B, g.H, g.NT, 64, g.d), "xt")
    _run("bsa_reorder", _device_of(x, xt), stream,
         lambda s: load_library().bsa_reorder(ctypes.byref(g.c()), _ptr(x), _ptr(xt), s))
    return xt


def reorder_pool(g: Geometry, x: torch.Tensor, xt: torch.Tensor | None = None,
                 xbar: torch.Tensor | None = None, stream=None) -> tuple[torch.Tensor, torch.Tensor]:
    """Tile-major reorder and the per-tile means of the valid tokens, in one pass."""
    _need(x, torch.bfloat16, (g.B, g.N, g.H, g.d), "x")
    if xt is None:
        xt = torch.empty((g.B, g.H, g.NT, 64, g.d), dtype=torch.bfloat16, device=x.device)
    if xbar is None:
        xbar = torch.empty((g.B, g.H, g.NT, g.d), dtype=torch.float32, device=x.device)
    _need(xt, torch.bfloat16, (g.B, g.H, g.NT, 64, g.d), "xt")
    _need(xbar, torch.float32, (g.B, g.H, g.NT, g.d), "xbar")
    _run("bsa_reorder_pool", _device_of(x, xt, xbar), stream,
         lambda s: load_library().bsa_reorder_pool(ctypes.byref(g.c()), _ptr(x), _ptr(xt), _ptr(xbar), s))
    return xt, xbar


def unreorder(g: Geometry, xt: torch.Tensor, x: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    _need(xt, torch.bfloat16, (g.B, g.H, g.NT, 64, g.d), "xt")
    if x is None:
        x = torch.empty((g.B, g.N, g.H, g.d), dtype=torch.bfloat16, device=xt.device)
    _need(x, torch.bfloat16, (g.B, g.N, g.H, g.d), "x")
    _run("bsa_unreorder", _device_of(xt, x), stream,
         lambda s: load_library().bsa_unreorder(ctypes.byref(g.c()), _ptr(xt), _ptr(x), s))
    return x


def build_mask(g: Geometry, p: MaskParams, qt: torch.Tensor, kt: torch.Tensor,
               difficulty: torch.Tensor, mask: torch.Tensor | None = None,
               kv_count: torch.Tensor | None = None, ws: torch.Tensor | None = None,
               stream=None) -> tuple[torch.Tensor, torch.Tensor]:
    _need(qt, torch.bfloat16, (g.B, g.H, g.NT, 64, g.d), "qt")
    _need(kt, torch.bfloat16, (g.B, g.H, g.NT, 64, g.d), "kt")
    _need(difficulty, torch.float32, (g.B, g.NT), "difficulty")
    dev = qt.device
    if mask is None:
        mask = torch.empty((g.B, g.H, g.NT, g.NW), dtype=torch.int32, device=dev)
    if kv_count is None:
        kv_count = torch.empty((g.B, g.H, g.NT), dtype=torch.int32, device=dev)
    _need(mask, torch.int32, (g.B, g.H, g.NT, g.NW), "mask")
    _need(kv_count, torch.int32, (g.B, g.H, g.NT), "kv_count")
    if ws is None:
        ws = alloc_workspace(g, dev)
    _need_ws(ws)
    pc = p.c()
    _run("bsa_build_mask", _device_of(qt, kt, difficulty, mask, kv_count, ws), stream,
         lambda s: load_library().bsa_build_mask(ctypes.byref(g.c()), ctypes.byref(pc), _ptr(qt), _ptr(kt),
                                                 _ptr(difficulty), _ptr(mask), _ptr(kv_count), _ptr(ws),
                                                 ctypes.c_size_t(ws.numel()), s))
    return mask, kv_count


def build_mask_pooled(g: Geometry, p: MaskParams, qbar: torch.Tensor, kbar: torch.Tensor,
                      difficulty: torch.Tensor, mask: torch.Tensor | None = None,
                      kv_count: torch.Tensor | None = None, ws: torch.Tensor | None = None,
                      stream=None) -> tuple[torch.Tensor, torch.Tensor]:
    """build_mask from the per-tile means that reorder_pool wrote."""
    _need(qbar, torch.float32, (g.B, g.H, g.NT, g.d), "qbar")
    _need(kbar, torch.float32, (g.B, g.H, g.NT, g.d), "kbar")
    _need(difficulty, torch.float32, (g.B, g.NT), "difficulty")
    dev = qbar.device
    if mask is None:
        mask = torch.empty((g.B, g.H, g.NT, g.NW), dtype=torch.int32, device=dev)
    if kv_count is None:
        kv_count = torch.empty((g.B, g.H, g.NT), dtype=torch.int32, device=dev)
    _need(mask, torch.int32, (g.B, g.H, g.NT, g.NW), "mask")
    _need(kv_count, torch.int32, (g.B, g.H, g.NT), "kv_count")
    if ws is None:
        ws = alloc_workspace(g, dev)
    _need_ws(ws)
    pc = p.c()
    _run("bsa_build_mask_pooled", _device_of(qbar, kbar, difficulty, mask, kv_count, ws), stream,
         lambda s: load_library().bsa_build_mask_pooled(ctypes.byref(g.c()), ctypes.byref(pc), _ptr(qbar),
                                                        _ptr(kbar), _ptr(difficulty), _ptr(mask),
                                                        _ptr(kv_count), _ptr(ws), ctypes.c_size_t(ws.numel()),
                                                        s))
    return mask, kv_count


def sparse_attn_fwd(g: Geometry, qt: torch.Tensor, kt: torch.Tensor, vt: torch.Tensor,
                    mask: torch.Tensor, kv_count: torch.Tensor, scale: float | None = None,
                    out: torch.Tensor | None = None, lse: torch.Tensor | None = None,
                    ws: torch.Tensor | None = None, want_lse: bool = True,
                    stream=None) -> tuple[torch.Tensor, torch.Tensor | None]:
    for name, t in (("qt", qt), ("kt", kt), ("vt", vt)):
        _need(t, torch.bfloat16, (g.B, g.H, g.NT, 64, g.d), name)
    _need(mask, torch.int32, (g.B, g.H, g.NT, g.NW), "mask")
    _need(kv_count, torch.int32, (g.B, g.H, g.NT), "kv_count")
    dev = qt.device
    if out is None:
        out = torch.empty((g.B, g.N, g.H, g.d), dtype=torch.bfloat16, device=dev)
    _need(out, torch.bfloat16, (g.B, g.N, g.H, g.d), "out")
    if want_lse and lse is None:
        lse = torch.empty((g.B, g.H, g.N), dtype=torch.float32, device=dev)
    if lse is not None:
        _need(lse, torch.float32, (g.B, g.H, g.N), "lse")
    if ws is None:
        ws = alloc_workspace(g, dev)
    _need_ws(ws)
    sc = 1.0 / math.sqrt(g.d) if scale is None else float(scale)
    _run("bsa_sparse_attn_fwd", _device_of(qt, kt, vt, mask, kv_count, out, lse, ws), stream,
         lambda s: load_library().bsa_sparse_attn_fwd(ctypes.byref(g.c()), _ptr(qt), _ptr(kt), _ptr(vt),
                                                      _ptr(mask), _ptr(kv_count), ctypes.c_float(sc),
                                                      _ptr(out), _ptr(lse), _ptr(ws),
                                                      ctypes.c_size_t(ws.numel()), s))
    return out, lse


def route_flags(g: Geometry, ws: torch.Tensor) -> torch.Tensor:
    """The route flags (uint8 [B, NQT], 1 = dense row) that build_mask left in `ws`: a view
    into the workspace, valid until the workspace is given to another build_mask."""
    _need_ws(ws)
    off = int(load_library().bsa_route_flags_offset(ctypes.byref(g.c())))
    if off == 0:
        raise ValueError("invalid geometry")
    return ws[off:off + g.B * g.NT].view(g.B, g.NT)


def sparse_attn_fwd_token(g: Geometry, qt: torch.Tensor, kt: torch.Tensor, vt: torch.Tensor,
                          mask: torch.Tensor, kv_count: torch.Tensor, dense: torch.Tensor,
                          token_radius: int, scale: float | None = None, out: torch.Tensor | None = None,
                          lse: torch.Tensor | None = None, ws: torch.Tensor | None = None,
                          want_lse: bool = True, stream=None) -> tuple[torch.Tensor, torch.Tensor | None]:
    """Block-sparse attention under a token-level circular support of radius token_radius
    (tokens): local rows (dense == 0) see their window tiles token by token, as
    bsa_sparse_attn_fwd_token in include/bsa.h describes."""
    for name, t in (("qt", qt), ("kt", kt), ("vt", vt)):
        _need(t, torch.bfloat16, (g.B, g.H, g.NT, 64, g.d), name)
    _need(mask, torch.int32, (g.B, g.H, g.NT, g.NW), "mask")
    _need(kv_count, torch.int32, (g.B, g.H, g.NT), "kv_count")
    _need(dense, torch.uint8, (g.B, g.NT), "dense")
    dev = qt.device
    if out is None:
        out = torch.empty((g.B, g.N, g.H, g.d), dtype=torch.bfloat16, device=dev)
    _need(out, torch.bfloat16, (g.B, g.N, g.H, g.d), "out")
    if want_lse and lse is None:
        lse = torch.empty((g.B, g.H, g.N), dtype=torch.float32, device=dev)
    if lse is not None:
        _need(lse, torch.float32, (g.B, g.H, g.N), "lse")
    if ws is None:
        ws = alloc_workspace(g, dev)
    _need_ws(ws)
    sc = 1.0 / math.sqrt(g.d) if scale is None else float(scale)
    _run("bsa_sparse_attn_fwd_token", _device_of(qt, kt, vt, mask, kv_count, dense, out, lse, ws), stream,
         lambda s: load_library().bsa_sparse_attn_fwd_token(
             ctypes.byref(g.c()), _ptr(qt), _ptr(kt), _ptr(vt), _ptr(mask), _ptr(kv_count), _ptr(dense),
             ctypes.c_int(int(token_radius)), ctypes.c_float(sc), _ptr(out), _ptr(lse), _ptr(ws),
             ctypes.c_size_t(ws.numel()), s))
    return out, lse


def sparse_attn_fwd_fixed_scratch(g: Geometry, qt: torch.Tensor, kt: torch.Tensor, vt: torch.Tensor,
                                  mask: torch.Tensor, kv_count: torch.Tensor,
                                  scale: float | None = None, out: torch.Tensor | None = None,
                                  lse: torch.Tensor | None = None,
                                  kernel_errors: torch.Tensor | None = None,
                                  want_lse: bool = True,
                                  stream=None) -> tuple[torch.Tensor, torch.Tensor | None]:
    """Block-sparse attention whose scratch is the library's own fixed device array.

    For callers that cannot allocate device memory (a plug-in that receives tensors from a
    host application which owns all device memory, or a serving loop that forbids
    allocation after start-up): pass preallocated `out` / `lse` and nothing is allocated
    here or in the library. Limits and sharing rules are those of
    bsa_sparse_attn_fwd_fixed_scratch in include/bsa.h: one call at a time per device, and
    the first call on a device should come before any stream capture.
    `kernel_errors`, if given, is a 1-element int32 device tensor that receives the call's
    kernel error word.
    """
    for name, t in (("qt", qt), ("kt", kt), ("vt", vt)):
        _need(t, torch.bfloat16, (g.B, g.H, g.NT, 64, g.d), name)
    _need(mask, torch.int32, (g.B, g.H, g.NT, g.NW), "mask")
    _need(kv_count, torch.int32, (g.B, g.H, g.NT), "kv_count")
    dev = qt.device
    if out is None:
        out = torch.empty((g.B, g.N, g.H, g.d), dtype=torch.bfloat16, device=dev)
    _need(out, torch.bfloat16, (g.B, g.N, g.H, g.d), "out")
    if want_lse and lse is None:
        lse = torch.empty((g.B, g.H, g.N), dtype=torch.float32, device=dev)
    if lse is not None:
        _need(lse, torch.float32, (g.B, g.H, g.N), "lse")
    if kernel_errors is not None:
        _need(kernel_errors, torch.int32, (1,), "kernel_errors")
    sc = 1.0 / math.sqrt(g.d) if scale is None else float(scale)
    _run("bsa_sparse_attn_fwd_fixed_scratch", _device_of(qt, kt, vt, mask, kv_count, out, lse, kernel_errors),
         stream,
         lambda s: load_library().bsa_sparse_attn_fwd_fixed_scratch(
             ctypes.byref(g.c()), _ptr(qt), _ptr(kt), _ptr(vt), _ptr(mask), _ptr(kv_count),
             ctypes.c_float(sc), _ptr(out), _ptr(lse), _ptr(kernel_errors), s))
    return out, lse


class Buffers:
    """Device buffers of one attention call, allocated once and reused across calls."""

    def __init__(self, g: Geometry, device=None):
        dev = device or "cuda"
        tiled = (g.B, g.H, g.NT, 64, g.d)
        self.qt = torch.empty(tiled, dtype=torch.bfloat16, device=dev)
        self.kt = torch.empty(tiled, dtype=torch.bfloat16, device=dev)
        self.vt = torch.empty(tiled, dtype=torch.bfloat16, device=dev)
        self.qbar = torch.empty((g.B, g.H, g.NT, g.d), dtype=torch.float32, device=dev)
        self.kbar = torch.empty((g.B, g.H, g.NT, g.d), dtype=torch.float32, device=dev)
        self.mask = torch.empty((g.B, g.H, g.NT, g.NW), dtype=torch.int32, device=dev)
        self.kv_count = torch.empty((g.B, g.H, g.NT), dtype=torch.int32, device=dev)
        self.out = torch.empty((g.B, g.N, g.H, g.d), dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty((g.B, g.H, g.N), dtype=torch.float32, device=dev)
        self.ws = alloc_workspace(g, dev)


def forward(g: Geometry, p: MaskParams, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
            difficulty: torch.Tensor, bufs: Buffers | None = None, scale: float | None = None,
            stream=None, rebuild_mask: bool = True) -> Buffers:
    """The whole path: reorder Q, K, V; build the mask; block-sparse attention.

    Returns the buffers; out / lse hold the attention output and LSE in raster order.
    rebuild_mask=False skips the mask build and attends through the mask (and counts) that
    an earlier call left in `bufs`: the reuse of a previous step's routing and sparsity
    (HetA-DiT reuses the preceding denoising step's estimates; MOD-DiT keeps historical
    sparsity). How often to rebuild is the caller's choice.
    With window kind 2 (token-level circular support, radius p.radius in tokens) the
    attention masks the tokens outside each query token's support inside window tiles,
    with the route flags the mask build left in the workspace.
    """
    if not rebuild_mask and bufs is None:
        raise ValueError("rebuild_mask=False attends through the mask held in bufs: pass the "
                         "Buffers of an earlier call")
    b = bufs or Buffers(g, q.device)
    if rebuild_mask:
        reorder_pool(g, q, b.qt, b.qbar, stream)
        reorder_pool(g, k, b.kt, b.kbar, stream)
    else:
        reorder(g, q, b.qt, stream)
        reorder(g, k, b.kt, stream)
    reorder(g, v, b.vt, stream)
    if rebuild_mask:
        build_mask_pooled(g, p, b.qbar, b.kbar, difficulty, b.mask, b.kv_count, b.ws, stream)
    if p.window_kind == 2:
        sparse_attn_fwd_token(g, b.qt, b.kt, b.vt, b.mask, b.kv_count, route_flags(g, b.ws), p.radius,
                              scale, b.out, b.lse, b.ws, stream=stream)
    else:
        sparse_attn_fwd(g, b.qt, b.kt, b.vt, b.mask, b.kv_count, scale, b.out, b.lse, b.ws,
                        stream=stream)
    return b


# kernels launched by forward(): 3 reorders (Q and K fused with their pooling when the
# mask is rebuilt); route, score and select (plus entropy and budget in budget mode) unless
# the mask is reused; 3 scheduler kernels and the attention kernel
def launches_per_forward(p: MaskParams, rebuild_mask: bool = True) -> int:
    return 3 + ((3 + (2 if p.budget_mode == 1 else 0)) if rebuild_mask else 0) + 4
