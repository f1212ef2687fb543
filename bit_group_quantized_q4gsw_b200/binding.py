"""ctypes binding of the q4gsw C ABI (include/q4gsw.h).

Argument marshalling only: every entry point takes torch tensors, checks their
dtype / device / contiguity, and passes raw device pointers and the current
CUDA stream to the library.  Results are computed by the library's CUDA
kernels; nothing here touches the numbers.  When ``libq4gsw.so`` is missing the
first call raises: there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os

import torch

from . import build as _build

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libq4gsw.so")

Q4GSW_OK = 0
STATUS_NAMES = {0: "Q4GSW_OK", 1: "Q4GSW_ERR_NULL", 2: "Q4GSW_ERR_SHAPE", 3: "Q4GSW_ERR_ALIGN",
                4: "Q4GSW_ERR_UNSUPPORTED", 5: "Q4GSW_ERR_CODE_RANGE", 6: "Q4GSW_ERR_CUDA",
                7: "Q4GSW_ERR_SIZE", 8: "Q4GSW_ERR_TIMEOUT", 9: "Q4GSW_ERR_INDEX"}

# (name, restype, argtypes) of every function declared in include/q4gsw.h
_VP, _I, _SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
SIGNATURES = [
    ("q4gsw_layout_version", _I, []),
    ("q4gsw_packed_bytes", _SZ, [_I, _I, _I]),
    ("q4gsw_prepack", _I, [_VP, _VP, _I, _I, _I, _VP, _SZ, _VP]),
    ("q4gsw_linear_fwd", _I, [_VP, _I, _I, _I, _VP, _I, _VP, _VP]),
    ("q4gsw_linear_bwd_input", _I, [_VP, _I, _I, _I, _VP, _I, _VP, _VP]),
    ("q4gsw_qkv_fwd", _I, [_VP, _I, _I, _I, _I, _I, _VP, _I, _VP, _VP, _VP, _VP]),
    ("q4gsw_embedding", _I, [_VP, _I, _I, _I, _VP, _I, _VP, _VP]),
    ("q4gsw_device_error_check", _I, [_VP]),
    ("q4gsw_unpack", _I, [_VP, _I, _I, _I, _VP, _VP]),
    ("q4gsw_dequant", _I, [_VP, _I, _I, _I, _VP, _VP, _VP]),
    ("q4gsw_packed_bytes_f32s", _SZ, [_I, _I, _I]),
    ("q4gsw_prepack_f32s", _I, [_VP, _VP, _I, _I, _I, _VP, _SZ, _VP]),
    ("q4gsw_linear_fwd_f32s", _I, [_VP, _I, _I, _I, _VP, _I, _VP, _VP]),
    ("q4gsw_linear_bwd_input_f32s", _I, [_VP, _I, _I, _I, _VP, _I, _VP, _VP]),
    ("q4gsw_qkv_fwd_f32s", _I, [_VP, _I, _I, _I, _I, _I, _VP, _I, _VP, _VP, _VP, _VP]),
    ("q4gsw_embedding_f32s", _I, [_VP, _I, _I, _I, _VP, _I, _VP, _VP]),
    ("q4gsw_dequant_f32s", _I, [_VP, _I, _I, _I, _VP, _VP, _VP]),
    ("q4gsw_adapter_workspace_bytes", _SZ, [_I, _I]),
    ("q4gsw_adapter_fwd", _I, [_VP, _I, _I, _I, _VP, _VP, _I, _VP, _I, _VP, _VP, _SZ, _VP]),
    ("q4gsw_adapter_bwd_input", _I, [_VP, _I, _I, _I, _VP, _VP, _I, _VP, _I, _VP, _VP, _SZ, _VP]),
    ("q4gsw_adapter_fwd_noalloc", _I, [_VP, _I, _I, _I, _VP, _VP, _I, _VP, _I, _VP, _VP]),
    ("q4gsw_dq8ca_workspace_bytes", _SZ, [_I, _I]),
    ("q4gsw_linear_dq8ca_fwd", _I, [_VP, _I, _I, _I, _VP, _I, _VP, _VP, _SZ, _VP]),
    ("q4gsw_dq8ca_quantize", _I, [_VP, _I, _I, _VP, _SZ, _VP]),
    ("q4gsw_debug_pin_routes", _I, [_I, _I]),
    ("q4gsw_debug_wait_timeout", _I, [ctypes.c_uint, _VP]),
    ("q4gsw_last_route", ctypes.c_char_p, []),
    ("q4gsw_status_str", ctypes.c_char_p, [_I]),
]

_lib = None


class Q4gswError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        self.status_name = STATUS_NAMES.get(status, str(status))
        msg = library().q4gsw_status_str(status).decode()
        super().__init__(f"{fn} failed: {self.status_name} ({msg})")


def library(path: str | None = None) -> ctypes.CDLL:
    """Load libq4gsw.so (building it first when nvcc is present and it is stale)."""
    global _lib
    if _lib is not None:
        return _lib
    path = path or LIB_PATH
    if path == LIB_PATH and not _build.up_to_date():
        try:
            _build.build()
        except RuntimeError:
            if not os.path.exists(LIB_PATH):
                raise
    if not os.path.exists(path):
        raise ImportError(f"q4gsw CUDA library not found at {path}; run `python -m bit_group_quantized_q4gsw_b200.build`")
    lib = ctypes.CDLL(path)
    for name, res, args in SIGNATURES:
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _check(fn: str, status: int):
    if status != Q4GSW_OK:
        raise Q4gswError(fn, status)


def _stream(t: torch.Tensor) -> int:
    return torch.cuda.current_stream(t.device).cuda_stream


def _dev(t: torch.Tensor, dtype, name: str, ndim: int | None = None) -> int:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be a CUDA tensor (got {t.device})")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype} (got {t.dtype})")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims (got {t.dim()})")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


# ---------------------------------------------------------------------------- public names = C names
def q4gsw_layout_version() -> int:
    return library().q4gsw_layout_version()


def q4gsw_packed_bytes(N: int, K: int, group_size: int) -> int:
    return int(library().q4gsw_packed_bytes(N, K, group_size))


def q4gsw_last_route() -> str:
    return library().q4gsw_last_route().decode()


def q4gsw_status_str(status: int) -> str:
    return library().q4gsw_status_str(status).decode()


def q4gsw_prepack(codes: torch.Tensor, scales: torch.Tensor, group_size: int,
                  packed: torch.Tensor | None = None) -> torch.Tensor:
    """codes uint8 [N, K] (0..15), scales fp16 [K/gs, N] -> packed uint8 blob.

    fp32 scales select the fp32-scale packer (layout version 2, q4gsw_prepack_f32s);
    its blob goes to the *_f32s compute functions."""
    lib = library()
    N, K = codes.shape
    f32s = scales.dtype == torch.float32
    nbytes = (lib.q4gsw_packed_bytes_f32s if f32s else lib.q4gsw_packed_bytes)(N, K, group_size)
    if packed is None:
        packed = torch.empty(max(int(nbytes), 1), dtype=torch.uint8, device=codes.device)
    fn, name = (lib.q4gsw_prepack_f32s, "q4gsw_prepack_f32s") if f32s else (lib.q4gsw_prepack, "q4gsw_prepack")
    st = fn(_dev(codes, torch.uint8, "codes", 2), _dev(scales, torch.float32 if f32s else torch.float16, "scales", 2),
            N, K, group_size, _dev(packed, torch.uint8, "packed"), packed.numel(), _stream(codes))
    _check(name, st)
    return packed


def q4gsw_prepack_f32s(codes: torch.Tensor, scales: torch.Tensor, group_size: int,
                       packed: torch.Tensor | None = None) -> torch.Tensor:
    """codes uint8 [N, K] (0..15), scales fp32 [K/gs, N] -> layout-version-2 blob."""
    if scales.dtype != torch.float32:
        raise TypeError("q4gsw_prepack_f32s takes fp32 scales")
    return q4gsw_prepack(codes, scales, group_size, packed)


def q4gsw_linear_fwd(packed: torch.Tensor, N: int, K: int, group_size: int, x: torch.Tensor,
                     y: torch.Tensor | None = None, f32s: bool = False) -> torch.Tensor:
    """y[M, N] = x[M, K] @ dequant(W)[N, K]^T in fp32 (f32s: a layout-version-2 blob)."""
    M = x.shape[0]
    if y is None:
        y = torch.empty((M, N), dtype=torch.float32, device=x.device)
    name = "q4gsw_linear_fwd_f32s" if f32s else "q4gsw_linear_fwd"
    st = getattr(library(), name)(_dev(packed, torch.uint8, "packed"), N, K, group_size,
                                  _dev(x, torch.float16, "x", 2), M, _dev(y, torch.float32, "y", 2), _stream(x))
    _check(name, st)
    return y


def q4gsw_linear_bwd_input(packed: torch.Tensor, N: int, K: int, group_size: int, d_out: torch.Tensor,
                           d_x: torch.Tensor | None = None, f32s: bool = False) -> torch.Tensor:
    """d_x[M, K] = d_out[M, N] @ dequant(W)[N, K] in fp32 (f32s: a layout-version-2 blob)."""
    M = d_out.shape[0]
    if d_x is None:
        d_x = torch.empty((M, K), dtype=torch.float32, device=d_out.device)
    name = "q4gsw_linear_bwd_input_f32s" if f32s else "q4gsw_linear_bwd_input"
    st = getattr(library(), name)(_dev(packed, torch.uint8, "packed"), N, K, group_size,
                                  _dev(d_out, torch.float16, "d_out", 2), M,
                                  _dev(d_x, torch.float32, "d_x", 2), _stream(d_out))
    _check(name, st)
    return d_x


def q4gsw_qkv_fwd(packed_qkv: torch.Tensor, Nq: int, Nk: int, Nv: int, K: int, group_size: int,
                  x: torch.Tensor, outs=None, f32s: bool = False):
    """Three projections of x from one packed [Nq+Nk+Nv, K] weight -> (y_q, y_k, y_v)."""
    M = x.shape[0]
    if outs is None:
        outs = tuple(torch.empty((M, n), dtype=torch.float32, device=x.device) for n in (Nq, Nk, Nv))
    yq, yk, yv = outs
    name = "q4gsw_qkv_fwd_f32s" if f32s else "q4gsw_qkv_fwd"
    st = getattr(library(), name)(_dev(packed_qkv, torch.uint8, "packed_qkv"), Nq, Nk, Nv, K, group_size,
                                  _dev(x, torch.float16, "x", 2), M, _dev(yq, torch.float32, "y_q", 2),
                                  _dev(yk, torch.float32, "y_k", 2), _dev(yv, torch.float32, "y_v", 2), _stream(x))
    _check(name, st)
    return yq, yk, yv


def q4gsw_embedding(packed: torch.Tensor, N: int, K: int, group_size: int, indices: torch.Tensor,
                    out: torch.Tensor | None = None, f32s: bool = False) -> torch.Tensor:
    """out[T, K] = dequant(W)[indices] in fp32 (indices int32 [T] on the device, each in [0, N))."""
    T = indices.shape[0]
    if out is None:
        out = torch.empty((T, K), dtype=torch.float32, device=indices.device)
    name = "q4gsw_embedding_f32s" if f32s else "q4gsw_embedding"
    st = getattr(library(), name)(_dev(packed, torch.uint8, "packed"), N, K, group_size,
                                  _dev(indices, torch.int32, "indices", 1), T,
                                  _dev(out, torch.float32, "out", 2), _stream(indices))
    _check(name, st)
    return out


def q4gsw_device_error_check(device=None) -> None:
    """Raise Q4gswError if a kernel wait ran out (Q4GSW_ERR_TIMEOUT) or an embedding
    index was out of range (Q4GSW_ERR_INDEX) since the last check."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    st = library().q4gsw_device_error_check(torch.cuda.current_stream(dev).cuda_stream)
    _check("q4gsw_device_error_check", st)


def _adapter(name, packed, N, K, group_size, a, b, act, out, workspace, out_cols):
    lib = library()
    r = a.shape[0]
    M = act.shape[0]
    if out is None:
        out = torch.empty((M, out_cols), dtype=torch.float32, device=act.device)
    if workspace is None:
        workspace = torch.empty(max(int(lib.q4gsw_adapter_workspace_bytes(M, r)), 16), dtype=torch.uint8,
                                device=act.device)
    st = getattr(lib, name)(_dev(packed, torch.uint8, "packed"), N, K, group_size, _dev(a, torch.float16, "a", 2),
                            _dev(b, torch.float16, "b", 2), r, _dev(act, torch.float16, "act", 2), M,
                            _dev(out, torch.float32, "out", 2), _dev(workspace, torch.uint8, "workspace"),
                            workspace.numel(), _stream(act))
    _check(name, st)
    return out


def q4gsw_adapter_fwd(packed, N: int, K: int, group_size: int, a, b, x, y=None, workspace=None):
    """y = x dequant(W)^T + (x a^T) b^T with a fp16 [r, K], b fp16 [N, r] (frozen-base adapter)."""
    return _adapter("q4gsw_adapter_fwd", packed, N, K, group_size, a, b, x, y, workspace, N)


def q4gsw_adapter_bwd_input(packed, N: int, K: int, group_size: int, a, b, d_out, d_x=None, workspace=None):
    """d_x = d_out dequant(W) + (d_out b) a (input gradient of the adapter forward)."""
    return _adapter("q4gsw_adapter_bwd_input", packed, N, K, group_size, a, b, d_out, d_x, workspace, K)


def q4gsw_linear_dq8ca_fwd(packed, N: int, K: int, group_size: int, x, y=None, workspace=None):
    """y from int8 dynamically quantised x (per token, asymmetric) and the q4gsw weight."""
    lib = library()
    M = x.shape[0]
    if y is None:
        y = torch.empty((M, N), dtype=torch.float32, device=x.device)
    if workspace is None:
        workspace = torch.empty(max(int(lib.q4gsw_dq8ca_workspace_bytes(M, K)), 16), dtype=torch.uint8,
                                device=x.device)
    st = lib.q4gsw_linear_dq8ca_fwd(_dev(packed, torch.uint8, "packed"), N, K, group_size,
                                    _dev(x, torch.float16, "x", 2), M, _dev(y, torch.float32, "y", 2),
                                    _dev(workspace, torch.uint8, "workspace"), workspace.numel(), _stream(x))
    _check("q4gsw_linear_dq8ca_fwd", st)
    return y


def q4gsw_dq8ca_quantize(x, workspace=None):
    """The quantised activations of x: returns the workspace (see include/q4gsw.h for its map)."""
    lib = library()
    M, K = x.shape
    if workspace is None:
        workspace = torch.empty(max(int(lib.q4gsw_dq8ca_workspace_bytes(M, K)), 16), dtype=torch.uint8,
                                device=x.device)
    st = lib.q4gsw_dq8ca_quantize(_dev(x, torch.float16, "x", 2), M, K, _dev(workspace, torch.uint8, "workspace"),
                                  workspace.numel(), _stream(x))
    _check("q4gsw_dq8ca_quantize", st)
    return workspace


GEMV_ROUTES = {"auto": 0, "reg": 1, "tma": 2, "tma_xs": 3}
GEMM_ROUTES = {"auto": 0, "ts": 1, "ss": 2, "ss1": 3, "ss2": 4}


def q4gsw_debug_pin_routes(gemv: str = "auto", gemm: str = "auto") -> None:
    """Pin the kernel routes of this thread's later calls (debug export; see include/q4gsw.h)."""
    st = library().q4gsw_debug_pin_routes(GEMV_ROUTES[gemv], GEMM_ROUTES[gemm])
    _check("q4gsw_debug_pin_routes", st)


def q4gsw_debug_wait_timeout(limit_us: int, device=None) -> None:
    """Enqueue the bounded-wait probe: one wait that runs out after limit_us microseconds."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    st = library().q4gsw_debug_wait_timeout(limit_us, torch.cuda.current_stream(dev).cuda_stream)
    _check("q4gsw_debug_wait_timeout", st)


def q4gsw_unpack(packed: torch.Tensor, N: int, K: int, group_size: int) -> torch.Tensor:
    codes = torch.empty((N, K), dtype=torch.uint8, device=packed.device)
    st = library().q4gsw_unpack(_dev(packed, torch.uint8, "packed"), N, K, group_size,
                                _dev(codes, torch.uint8, "codes", 2), _stream(packed))
    _check("q4gsw_unpack", st)
    return codes


def q4gsw_dequant(packed: torch.Tensor, N: int, K: int, group_size: int, want_w32: bool = True,
                  want_w16: bool = True, f32s: bool = False):
    """(w32 fp32 [N, K], w16 fp16 [N, K] tensor-core operand); either may be None."""
    w32 = torch.empty((N, K), dtype=torch.float32, device=packed.device) if want_w32 else None
    w16 = torch.empty((N, K), dtype=torch.float16, device=packed.device) if want_w16 else None
    name = "q4gsw_dequant_f32s" if f32s else "q4gsw_dequant"
    st = getattr(library(), name)(_dev(packed, torch.uint8, "packed"), N, K, group_size,
                                  None if w32 is None else w32.data_ptr(),
                                  None if w16 is None else w16.data_ptr(), _stream(packed))
    _check(name, st)
    return w32, w16
