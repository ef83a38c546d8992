"""Python binding of libsvdq, the SVDQuant W4A4 linear layer (svdq_w4a4) for one
NVIDIA B200 (sm_100a).

Argument marshalling only: every step of the layer runs in the CUDA library
(include/svdq.h).  torch is used for device memory and streams.  There is no
CPU fallback: if libsvdq.so is missing or cannot be loaded, every call raises.

Entry points keep the C names (svdq_prepare, svdq_pack, svdq_layer_create,
svdq_forward, ..., and svdq_awq_* for the awq_w4a16 layer).  `SvdqLinear` and
`AwqLinear` bundle them for nn.Linear-style use.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
# SVDQ_LIBRARY=debug selects the bounds-checked debug variant (libsvdq_debug.so,
# built by build.build(debug=True)); the default is the release library.
LIB_PATH = os.path.join(_HERE, "libsvdq_debug.so" if os.environ.get("SVDQ_LIBRARY") == "debug" else "libsvdq.so")

SVDQ_OK = 0
SVDQ_ERR_INVALID_ARG = 1
SVDQ_ERR_UNSUPPORTED_DEVICE = 2
SVDQ_ERR_OOM = 3
SVDQ_ERR_CUDA = 4
SVDQ_ERR_NUMERIC = 5
SVDQ_ERR_TIMEOUT = 6
SVDQ_ERR_BOUNDS = 7
SVDQ_INT4_G64 = 1
SVDQ_NVFP4_G16 = 2
FORMATS = {"int4": SVDQ_INT4_G64, "nvfp4": SVDQ_NVFP4_G16, SVDQ_INT4_G64: SVDQ_INT4_G64,
           SVDQ_NVFP4_G16: SVDQ_NVFP4_G16}


def _fmt(f) -> int:
    """Format name or code -> code (unknown integers pass through for the library to reject)."""
    return int(f) if isinstance(f, (int, np.integer)) else FORMATS[f]


class SvdqError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {svdq_status_string(status)}")


class svdq_canonical(ctypes.Structure):
    _fields_ = [("N", ctypes.c_int64), ("K", ctypes.c_int64), ("rank", ctypes.c_int32), ("fmt", ctypes.c_int32),
                ("alpha", ctypes.c_float), ("g_x", ctypes.c_float), ("g_w", ctypes.c_float),
                ("reserved", ctypes.c_float), ("lambda_", ctypes.c_void_p), ("inv_lambda", ctypes.c_void_p),
                ("L1", ctypes.c_void_p), ("L2", ctypes.c_void_p), ("wcodes", ctypes.c_void_p),
                ("wscales", ctypes.c_void_p), ("bias", ctypes.c_void_p)]


class svdq_awq_canonical(ctypes.Structure):
    _fields_ = [("N", ctypes.c_int64), ("K", ctypes.c_int64), ("alpha", ctypes.c_float), ("reserved", ctypes.c_float),
                ("s", ctypes.c_void_p), ("inv_s", ctypes.c_void_p), ("wcodes", ctypes.c_void_p),
                ("wscales", ctypes.c_void_p), ("bias", ctypes.c_void_p)]


_lib = None
_EXPORTS = {
    # name: (restype, argtypes)
    "svdq_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "svdq_abi_version": (ctypes.c_int, []),
    "svdq_debug_build": (ctypes.c_int, []),
    "svdq_canonical_sizes": (ctypes.c_int, [ctypes.c_int64, ctypes.c_int64, ctypes.c_int, ctypes.c_int,
                                            ctypes.POINTER(ctypes.c_size_t)]),
    "svdq_prepare": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_float,
                                    ctypes.POINTER(svdq_canonical)]),
    "svdq_packed_size": (ctypes.c_int, [ctypes.c_int64, ctypes.c_int64, ctypes.c_int, ctypes.c_int,
                                        ctypes.POINTER(ctypes.c_size_t)]),
    "svdq_pack": (ctypes.c_int, [ctypes.POINTER(svdq_canonical), ctypes.c_void_p, ctypes.c_size_t]),
    "svdq_device_check": (ctypes.c_int, [ctypes.c_int]),
    "svdq_layer_create": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int64, ctypes.c_int64,
                                         ctypes.c_int, ctypes.c_int, ctypes.c_float, ctypes.c_float,
                                         ctypes.POINTER(ctypes.c_void_p)]),
    "svdq_layer_destroy": (None, [ctypes.c_void_p]),
    "svdq_workspace_size": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64, ctypes.POINTER(ctypes.c_size_t)]),
    "svdq_workspace_layout": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64, ctypes.POINTER(ctypes.c_size_t),
                                             ctypes.POINTER(ctypes.c_size_t)]),
    "svdq_workspace_init": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_size_t,
                                           ctypes.c_void_p]),
    "svdq_forward": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p,
                                    ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "svdq_quantize_act": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p,
                                         ctypes.c_size_t, ctypes.c_void_p]),
    "svdq_gemm": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p,
                                 ctypes.c_size_t, ctypes.c_void_p]),
    "svdq_int4_group_acc": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_size_t,
                                           ctypes.c_void_p, ctypes.c_void_p]),
    "svdq_read_status": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_size_t,
                                        ctypes.POINTER(ctypes.c_int)]),
    "svdq_set_wait_limit": (ctypes.c_int, [ctypes.c_uint64]),
    "svdq_forward_noalloc": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p,
                                            ctypes.c_void_p]),
    "svdq_mlp_fusable": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p]),
    "svdq_gemm_gelu_quantize": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p,
                                               ctypes.c_size_t, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p,
                                               ctypes.c_void_p]),
    "svdq_mlp_forward": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
                                        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p,
                                        ctypes.c_size_t, ctypes.c_void_p]),
    "svdq_awq_canonical_sizes": (ctypes.c_int, [ctypes.c_int64, ctypes.c_int64, ctypes.POINTER(ctypes.c_size_t)]),
    "svdq_awq_prepare": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
                                        ctypes.POINTER(svdq_awq_canonical)]),
    "svdq_awq_packed_size": (ctypes.c_int, [ctypes.c_int64, ctypes.c_int64, ctypes.POINTER(ctypes.c_size_t)]),
    "svdq_awq_pack": (ctypes.c_int, [ctypes.POINTER(svdq_awq_canonical), ctypes.c_void_p, ctypes.c_size_t]),
    "svdq_awq_layer_create": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int64, ctypes.c_int64,
                                             ctypes.POINTER(ctypes.c_void_p)]),
    "svdq_awq_layer_destroy": (None, [ctypes.c_void_p]),
    "svdq_awq_read_status": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p]),
    "svdq_awq_forward": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p,
                                        ctypes.c_void_p]),
    "svdq_w8a8_prepare": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p,
                                         ctypes.POINTER(ctypes.c_float)]),
    "svdq_w8a8_packed_size": (ctypes.c_int, [ctypes.c_int64, ctypes.c_int64, ctypes.POINTER(ctypes.c_size_t)]),
    "svdq_w8a8_pack": (ctypes.c_int, [ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p,
                                      ctypes.c_void_p, ctypes.c_size_t]),
    "svdq_w8a8_layer_create": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int64, ctypes.c_int64,
                                              ctypes.c_float, ctypes.POINTER(ctypes.c_void_p)]),
    "svdq_w8a8_layer_destroy": (None, [ctypes.c_void_p]),
    "svdq_w8a8_workspace_size": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64, ctypes.POINTER(ctypes.c_size_t)]),
    "svdq_w8a8_quantize_act": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p,
                                              ctypes.c_size_t, ctypes.c_void_p]),
    "svdq_w8a8_gemm": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p,
                                      ctypes.c_size_t, ctypes.c_void_p]),
    "svdq_w8a8_forward": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p,
                                         ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "svdq_w8a8_read_status": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_size_t,
                                             ctypes.POINTER(ctypes.c_int)]),
}


def lib() -> ctypes.CDLL:
    """The loaded libsvdq.so; raises if it was not built (no fallback)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{os.path.basename(LIB_PATH)} not found at {LIB_PATH}: build it with "
                               "`python -m diffusion_transformer_w4a4_b200.build` (there is no CPU fallback)")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _EXPORTS.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _check(status: int, where: str):
    if status != SVDQ_OK:
        raise SvdqError(status, where)


def _ptr(a) -> int | None:
    if a is None:
        return None
    if isinstance(a, np.ndarray):
        assert a.flags["C_CONTIGUOUS"]
        return a.ctypes.data
    return a.data_ptr()  # torch tensor


def _stream(stream) -> int | None:
    if stream is None:
        import torch

        return torch.cuda.current_stream().cuda_stream
    return int(getattr(stream, "cuda_stream", stream))


# ----------------------------------------------------------------------------- C names
def svdq_status_string(status: int) -> str:
    return lib().svdq_status_string(int(status)).decode()


def svdq_debug_build() -> int:
    """1 when the loaded library is the bounds-checked debug variant."""
    return int(lib().svdq_debug_build())


def svdq_abi_version() -> int:
    return int(lib().svdq_abi_version())


def svdq_canonical_sizes(N: int, K: int, rank: int, fmt) -> list[int]:
    sizes = (ctypes.c_size_t * 7)()
    _check(lib().svdq_canonical_sizes(N, K, rank, _fmt(fmt), sizes), "svdq_canonical_sizes")
    return list(sizes)


def _canonical_arrays(N, K, rank, fmt):
    fmt = _fmt(fmt)
    return dict(
        N=N, K=K, rank=rank, fmt=fmt,
        lambda_=np.zeros(K, np.float32), inv_lambda=np.zeros(K, np.float32),
        L1=np.zeros((K, rank), np.uint16), L2=np.zeros((rank, N), np.uint16),
        wcodes=np.zeros((N, K // 2), np.uint8),
        wscales=np.zeros((N, K // 64), np.uint16) if fmt == SVDQ_INT4_G64 else np.zeros((N, K // 16), np.uint8),
        bias=np.zeros(N, np.uint16), g_x=1.0, g_w=1.0, alpha=0.5)


def _to_struct(c: dict) -> svdq_canonical:
    s = svdq_canonical()
    s.N, s.K, s.rank, s.fmt = int(c["N"]), int(c["K"]), int(c["rank"]), _fmt(c["fmt"])
    s.alpha, s.g_x, s.g_w = float(c.get("alpha", 0.5)), float(c.get("g_x", 1.0)), float(c.get("g_w", 1.0))
    for f in ("lambda_", "inv_lambda", "L1", "L2", "wcodes", "wscales", "bias"):
        arr = c.get(f)
        setattr(s, f, None if arr is None or arr.size == 0 else arr.ctypes.data)
    return s


def svdq_prepare(W: np.ndarray, bias, act_absmax: np.ndarray, alpha: float, rank: int, fmt) -> dict:
    """Host-side preparation (smoothing, truncated SVD, residual quantize).
    W: bf16 bits [N,K] uint16; bias: bf16 bits [N] or None; act_absmax: float32 [K]."""
    W = np.ascontiguousarray(W, np.uint16)
    N, K = W.shape
    c = _canonical_arrays(N, K, rank, fmt)
    s = _to_struct(c)
    b = None if bias is None else np.ascontiguousarray(bias, np.uint16)
    am = np.ascontiguousarray(act_absmax, np.float32)
    _check(lib().svdq_prepare(W.ctypes.data, None if b is None else b.ctypes.data, am.ctypes.data,
                              float(alpha), ctypes.byref(s)), "svdq_prepare")
    c["g_x"], c["g_w"], c["alpha"] = float(s.g_x), float(s.g_w), float(s.alpha)
    return c


def svdq_packed_size(N: int, K: int, rank: int, fmt) -> int:
    n = ctypes.c_size_t()
    _check(lib().svdq_packed_size(N, K, rank, _fmt(fmt), ctypes.byref(n)), "svdq_packed_size")
    return n.value


def svdq_pack(c: dict) -> np.ndarray:
    """Canonical prepared weights (dict of host arrays) -> device-layout blob (host bytes)."""
    c = dict(c)
    for f, dt in (("lambda_", np.float32), ("inv_lambda", np.float32), ("L1", np.uint16), ("L2", np.uint16),
                  ("wcodes", np.uint8), ("bias", np.uint16)):
        if c.get(f) is not None:
            c[f] = np.ascontiguousarray(c[f], dt)
    c["wscales"] = np.ascontiguousarray(c["wscales"])
    size = svdq_packed_size(c["N"], c["K"], c["rank"], c["fmt"])
    blob = np.zeros(size, np.uint8)
    s = _to_struct(c)
    _check(lib().svdq_pack(ctypes.byref(s), blob.ctypes.data, size), "svdq_pack")
    return blob


def svdq_device_check(device: int = 0) -> int:
    return int(lib().svdq_device_check(int(device)))


def svdq_layer_create(dev_blob, blob_bytes: int, N: int, K: int, rank: int, fmt, g_x: float, g_w: float):
    h = ctypes.c_void_p()
    _check(lib().svdq_layer_create(_ptr(dev_blob), blob_bytes, N, K, rank, _fmt(fmt), float(g_x), float(g_w),
                                   ctypes.byref(h)), "svdq_layer_create")
    return h


def svdq_layer_destroy(h) -> None:
    lib().svdq_layer_destroy(h)


def svdq_workspace_size(h, M: int) -> int:
    n = ctypes.c_size_t()
    _check(lib().svdq_workspace_size(h, M, ctypes.byref(n)), "svdq_workspace_size")
    return n.value


def svdq_workspace_layout(h, M: int):
    off = (ctypes.c_size_t * 4)()
    sz = (ctypes.c_size_t * 4)()
    _check(lib().svdq_workspace_layout(h, M, off, sz), "svdq_workspace_layout")
    return list(off), list(sz)


def svdq_workspace_init(h, M: int, ws, stream=None) -> None:
    _check(lib().svdq_workspace_init(h, M, _ptr(ws), ws.numel(), _stream(stream)), "svdq_workspace_init")


def svdq_forward(h, X, M: int, Y, ws, stream=None) -> None:
    _check(lib().svdq_forward(h, _ptr(X), M, _ptr(Y), _ptr(ws), ws.numel(), _stream(stream)), "svdq_forward")


def svdq_quantize_act(h, X, M: int, ws, stream=None) -> None:
    _check(lib().svdq_quantize_act(h, _ptr(X), M, _ptr(ws), ws.numel(), _stream(stream)), "svdq_quantize_act")


def svdq_gemm(h, M: int, Y, ws, stream=None) -> None:
    _check(lib().svdq_gemm(h, M, _ptr(Y), _ptr(ws), ws.numel(), _stream(stream)), "svdq_gemm")


def svdq_int4_group_acc(h, M: int, ws, acc, stream=None) -> None:
    _check(lib().svdq_int4_group_acc(h, M, _ptr(ws), ws.numel(), _ptr(acc), _stream(stream)), "svdq_int4_group_acc")


def svdq_read_status(h, M: int, ws) -> int:
    """Status word of a caller workspace, or (ws=None) of the last
    svdq_forward_noalloc call for M tokens on the current device."""
    v = ctypes.c_int()
    nbytes = ws.numel() if ws is not None else 0
    _check(lib().svdq_read_status(h, M, _ptr(ws), nbytes, ctypes.byref(v)), "svdq_read_status")
    return int(v.value)


def svdq_forward_noalloc(h, X, M: int, Y, stream=None) -> None:
    """Forward without a caller workspace (library-owned 32 MiB scratch per GPU)."""
    _check(lib().svdq_forward_noalloc(h, _ptr(X), M, _ptr(Y), _stream(stream)), "svdq_forward_noalloc")


def svdq_mlp_fusable(up, down) -> int:
    """SVDQ_OK when the pair (up, down) can run as one fused MLP (see svdq_mlp_forward)."""
    return int(lib().svdq_mlp_fusable(up, down))


def svdq_gemm_gelu_quantize(up, down, M: int, ws_up, ws_dn, H=None, stream=None) -> None:
    """The up layer's GEMM with GELU and the down layer's quantizer in its epilogue."""
    _check(lib().svdq_gemm_gelu_quantize(up, down, M, _ptr(ws_up), ws_up.numel(), _ptr(ws_dn), ws_dn.numel(),
                                         _ptr(H), _stream(stream)), "svdq_gemm_gelu_quantize")


def svdq_mlp_forward(up, down, X, M: int, Y, ws_up, ws_dn, stream=None) -> None:
    """Y = down(GELU(up(X))) with the cross-layer fused GEMM in the middle."""
    _check(lib().svdq_mlp_forward(up, down, _ptr(X), M, _ptr(Y), _ptr(ws_up), ws_up.numel(), _ptr(ws_dn),
                                  ws_dn.numel(), _stream(stream)), "svdq_mlp_forward")


def svdq_set_wait_limit(cycles: int) -> None:
    _check(lib().svdq_set_wait_limit(int(cycles)), "svdq_set_wait_limit")


# ----------------------------------------------------------------------------- convenience
def _layer_device(device):
    """The CUDA device a layer lives on, always with its index."""
    import torch

    d = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
    if d.type != "cuda":
        raise ValueError(f"a layer lives on a CUDA device, not {d}")
    return d if d.index is not None else torch.device("cuda", torch.cuda.current_device())


def _check_input(x, K: int, device):
    import torch

    if not (x.dtype == torch.bfloat16 and x.is_cuda and x.is_contiguous() and x.shape[-1] == K):
        raise ValueError(f"expected a contiguous bf16 CUDA tensor [..., {K}], got {x.dtype} {tuple(x.shape)}")
    if x.device != device:
        raise ValueError(f"input on {x.device}, layer on {device}")


class SvdqLinear:
    """One svdq_w4a4 layer resident on `device` (default: the current CUDA device).

    Built from canonical prepared weights (svdq_prepare output, or any dict with
    the same arrays); `forward(x)` takes a bf16 CUDA tensor [M, K] on that device
    and returns bf16 [M, N].  Workspaces are cached per token count.  The handle
    is created, and every call that enqueues work is made, with the layer's
    device current (the library refuses a call from another device)."""

    def __init__(self, canonical: dict, device=None):
        import torch

        self.N, self.K, self.rank = int(canonical["N"]), int(canonical["K"]), int(canonical["rank"])
        self.fmt = _fmt(canonical["fmt"])
        self.g_x, self.g_w = float(canonical.get("g_x", 1.0)), float(canonical.get("g_w", 1.0))
        self.device = _layer_device(device)
        blob = svdq_pack(canonical)
        self.blob = torch.from_numpy(blob).to(self.device)
        with torch.cuda.device(self.device):
            self.handle = svdq_layer_create(self.blob, self.blob.numel(), self.N, self.K, self.rank, self.fmt,
                                            self.g_x, self.g_w)
        self._ws = {}

    def workspace(self, M: int):
        import torch

        ws = self._ws.get(M)
        if ws is None:
            ws = torch.empty(max(svdq_workspace_size(self.handle, M), 1024), dtype=torch.uint8, device=self.device)
            with torch.cuda.device(self.device):
                svdq_workspace_init(self.handle, M, ws)
            self._ws[M] = ws
        return ws

    def forward(self, x, out=None, stream=None):
        import torch

        _check_input(x, self.K, self.device)
        M = x.numel() // self.K
        y = out if out is not None else torch.empty(M, self.N, dtype=torch.bfloat16, device=x.device)
        ws = self.workspace(M)
        with torch.cuda.device(self.device):
            svdq_forward(self.handle, x, M, y, ws, stream)
        return y

    __call__ = forward

    def status(self, M: int) -> int:
        return svdq_read_status(self.handle, M, self.workspace(M))

    def __del__(self):
        h = getattr(self, "handle", None)
        if h is not None and _lib is not None:
            _lib.svdq_layer_destroy(h)
            self.handle = None


# ----------------------------------------------------------------------------- awq_w4a16
def svdq_awq_canonical_sizes(N: int, K: int) -> list[int]:
    sizes = (ctypes.c_size_t * 5)()
    _check(lib().svdq_awq_canonical_sizes(N, K, sizes), "svdq_awq_canonical_sizes")
    return list(sizes)


def _awq_arrays(N, K):
    return dict(N=N, K=K, alpha=0.0, s=np.zeros(K, np.float32), inv_s=np.zeros(K, np.float32),
                wcodes=np.zeros((N, K // 2), np.uint8), wscales=np.zeros((N, K // 64), np.uint16),
                bias=np.zeros(N, np.uint16))


def _awq_struct(c: dict) -> svdq_awq_canonical:
    st = svdq_awq_canonical()
    st.N, st.K, st.alpha = int(c["N"]), int(c["K"]), float(c.get("alpha", 0.0))
    for f in ("s", "inv_s", "wcodes", "wscales", "bias"):
        arr = c.get(f)
        setattr(st, f, None if arr is None else arr.ctypes.data)
    return st


def svdq_awq_prepare(W: np.ndarray, bias, X_calib: np.ndarray) -> dict:
    """Host-side activation-aware preparation of an awq_w4a16 layer.
    W: bf16 bits [N,K]; bias: bf16 bits [N] or None; X_calib: bf16 bits [M_calib, K]."""
    W = np.ascontiguousarray(W, np.uint16)
    X = np.ascontiguousarray(X_calib, np.uint16)
    N, K = W.shape
    c = _awq_arrays(N, K)
    st = _awq_struct(c)
    b = None if bias is None else np.ascontiguousarray(bias, np.uint16)
    _check(lib().svdq_awq_prepare(W.ctypes.data, None if b is None else b.ctypes.data, X.ctypes.data, X.shape[0],
                                  ctypes.byref(st)), "svdq_awq_prepare")
    c["alpha"] = float(st.alpha)
    return c


def svdq_awq_packed_size(N: int, K: int) -> int:
    n = ctypes.c_size_t()
    _check(lib().svdq_awq_packed_size(N, K, ctypes.byref(n)), "svdq_awq_packed_size")
    return n.value


def svdq_awq_pack(c: dict) -> np.ndarray:
    c = dict(c)
    for f, dt in (("s", np.float32), ("inv_s", np.float32), ("wcodes", np.uint8), ("wscales", np.uint16),
                  ("bias", np.uint16)):
        if c.get(f) is not None:
            c[f] = np.ascontiguousarray(c[f], dt)
    size = svdq_awq_packed_size(c["N"], c["K"])
    blob = np.zeros(size, np.uint8)
    _check(lib().svdq_awq_pack(ctypes.byref(_awq_struct(c)), blob.ctypes.data, size), "svdq_awq_pack")
    return blob


def svdq_awq_layer_create(dev_blob, blob_bytes: int, N: int, K: int):
    h = ctypes.c_void_p()
    _check(lib().svdq_awq_layer_create(_ptr(dev_blob), blob_bytes, N, K, ctypes.byref(h)), "svdq_awq_layer_create")
    return h


def svdq_awq_layer_destroy(h) -> None:
    lib().svdq_awq_layer_destroy(h)


def svdq_awq_read_status(h) -> int:
    v = ctypes.c_int()
    _check(lib().svdq_awq_read_status(h, ctypes.byref(v)), "svdq_awq_read_status")
    return v.value


def svdq_awq_forward(h, X, M: int, Y, stream=None) -> None:
    _check(lib().svdq_awq_forward(h, _ptr(X), M, _ptr(Y), _stream(stream)), "svdq_awq_forward")


class AwqLinear:
    """One awq_w4a16 layer (4-bit weights, bf16 activations) on `device` (default:
    the current CUDA device), built from canonical prepared weights
    (svdq_awq_prepare output or a dict with the same arrays); `forward(x)` maps
    bf16 [M, K] to bf16 [M, N], enqueued with the layer's device current."""

    def __init__(self, canonical: dict, device=None):
        import torch

        self.N, self.K = int(canonical["N"]), int(canonical["K"])
        self.device = _layer_device(device)
        self.blob = torch.from_numpy(svdq_awq_pack(canonical)).to(self.device)
        with torch.cuda.device(self.device):
            self.handle = svdq_awq_layer_create(self.blob, self.blob.numel(), self.N, self.K)

    def forward(self, x, out=None, stream=None):
        import torch

        _check_input(x, self.K, self.device)
        M = x.numel() // self.K
        y = out if out is not None else torch.empty(M, self.N, dtype=torch.bfloat16, device=x.device)
        with torch.cuda.device(self.device):
            svdq_awq_forward(self.handle, x, M, y, stream)
        return y

    __call__ = forward

    def status(self) -> int:
        return svdq_awq_read_status(self.handle)

    def __del__(self):
        h = getattr(self, "handle", None)
        if h is not None and _lib is not None:
            _lib.svdq_awq_layer_destroy(h)
            self.handle = None


# ----------------------------------------------------------------------------- int8 tensorwise W8A8
def svdq_w8a8_prepare(W):
    """Host: W [N,K] bf16 bits -> (int8 codes [N,K], s_w)."""
    W = np.ascontiguousarray(W, np.uint16)
    N, K = W.shape
    codes = np.empty((N, K), np.int8)
    s = ctypes.c_float()
    _check(lib().svdq_w8a8_prepare(W.ctypes.data, N, K, codes.ctypes.data, ctypes.byref(s)), "svdq_w8a8_prepare")
    return codes, float(s.value)


def svdq_w8a8_packed_size(N: int, K: int) -> int:
    v = ctypes.c_size_t()
    _check(lib().svdq_w8a8_packed_size(N, K, ctypes.byref(v)), "svdq_w8a8_packed_size")
    return v.value


def svdq_w8a8_pack(wcodes, bias=None) -> np.ndarray:
    wcodes = np.ascontiguousarray(wcodes, np.int8)
    N, K = wcodes.shape
    size = svdq_w8a8_packed_size(N, K)
    blob = np.zeros(size, np.uint8)
    b = None if bias is None else np.ascontiguousarray(bias, np.uint16)
    _check(lib().svdq_w8a8_pack(N, K, wcodes.ctypes.data, None if b is None else b.ctypes.data, blob.ctypes.data,
                                size), "svdq_w8a8_pack")
    return blob


def svdq_w8a8_layer_create(dev_blob, blob_bytes: int, N: int, K: int, s_w: float):
    h = ctypes.c_void_p()
    _check(lib().svdq_w8a8_layer_create(_ptr(dev_blob), blob_bytes, N, K, s_w, ctypes.byref(h)),
           "svdq_w8a8_layer_create")
    return h


def svdq_w8a8_layer_destroy(h) -> None:
    lib().svdq_w8a8_layer_destroy(h)


def svdq_w8a8_workspace_size(h, M: int) -> int:
    v = ctypes.c_size_t()
    _check(lib().svdq_w8a8_workspace_size(h, M, ctypes.byref(v)), "svdq_w8a8_workspace_size")
    return v.value


def svdq_w8a8_quantize_act(h, X, M: int, ws, stream=None) -> None:
    _check(lib().svdq_w8a8_quantize_act(h, _ptr(X), M, _ptr(ws), ws.numel(), _stream(stream)),
           "svdq_w8a8_quantize_act")


def svdq_w8a8_gemm(h, M: int, Y, ws, stream=None) -> None:
    _check(lib().svdq_w8a8_gemm(h, M, _ptr(Y), _ptr(ws), ws.numel(), _stream(stream)), "svdq_w8a8_gemm")


def svdq_w8a8_forward(h, X, M: int, Y, ws, stream=None) -> None:
    _check(lib().svdq_w8a8_forward(h, _ptr(X), M, _ptr(Y), _ptr(ws), ws.numel(), _stream(stream)),
           "svdq_w8a8_forward")


def svdq_w8a8_read_status(h, M: int, ws) -> int:
    v = ctypes.c_int()
    _check(lib().svdq_w8a8_read_status(h, M, _ptr(ws), ws.numel(), ctypes.byref(v)), "svdq_w8a8_read_status")
    return v.value


class W8A8Linear:
    """One INT8 tensorwise W8A8 layer on `device` (default: the current CUDA
    device), from prepared int8 weight codes [N,K], the weight scale s_w and an
    optional bf16 bias; `forward(x)` maps bf16 [M, K] to bf16 [M, N], enqueued
    with the layer's device current."""

    def __init__(self, wcodes, s_w: float, bias=None, device=None):
        import torch

        self.N, self.K = int(wcodes.shape[0]), int(wcodes.shape[1])
        self.s_w = float(s_w)
        self.device = _layer_device(device)
        self.blob = torch.from_numpy(svdq_w8a8_pack(wcodes, bias)).to(self.device)
        with torch.cuda.device(self.device):
            self.handle = svdq_w8a8_layer_create(self.blob, self.blob.numel(), self.N, self.K, self.s_w)
        self._ws = {}

    def workspace_size(self, M: int) -> int:
        return svdq_w8a8_workspace_size(self.handle, M)

    def workspace(self, M: int):
        import torch

        if M not in self._ws:
            self._ws[M] = torch.empty(self.workspace_size(M), dtype=torch.uint8, device=self.device)
        return self._ws[M]

    def quantize_act(self, x, M: int, stream=None):
        import torch

        ws = self.workspace(M)
        with torch.cuda.device(self.device):
            svdq_w8a8_quantize_act(self.handle, x, M, ws, stream)

    def gemm(self, M: int, y, stream=None):
        import torch

        ws = self.workspace(M)
        with torch.cuda.device(self.device):
            svdq_w8a8_gemm(self.handle, M, y, ws, stream)

    def forward(self, x, out=None, stream=None):
        import torch

        _check_input(x, self.K, self.device)
        M = x.numel() // self.K
        y = out if out is not None else torch.empty(M, self.N, dtype=torch.bfloat16, device=x.device)
        ws = self.workspace(M)
        with torch.cuda.device(self.device):
            svdq_w8a8_forward(self.handle, x, M, y, ws, stream)
        return y

    __call__ = forward

    def status(self, M: int) -> int:
        return svdq_w8a8_read_status(self.handle, M, self.workspace(M))

    def read_act(self, M: int):
        """Activation codes int8 [M, K] and s_x from the workspace (after quantize_act)."""
        ws = self.workspace(M).cpu().numpy()
        ctrl = (M * self.K + 1023) // 1024 * 1024
        return dict(codes=ws[:M * self.K].view(np.int8).reshape(M, self.K).copy(),
                    s_x=np.float32(ws[ctrl + 4:ctrl + 8].view(np.float32)[0]))

    def __del__(self):
        h = getattr(self, "handle", None)
        if h is not None and _lib is not None:
            _lib.svdq_w8a8_layer_destroy(h)
            self.handle = None
