"""Mamba-2 SSD selective scan on NVIDIA B200: Python binding of libssd_b200.so.

The functions here carry the names of the C ABI in include/ssd.h and only
marshal arguments: they read shapes and device pointers off torch tensors,
allocate outputs/workspace with torch when the caller does not pass them, and
call the library on the current torch CUDA stream.  Every step of the scan runs
in the library's CUDA kernels; there is no CPU fallback, and a missing library
raises immediately.
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "SsdError", "ssd_fwd", "ssd_fwd_workspace_size", "ssd_fwd_check_status", "ssd_fwd_no_alloc",
    "ssd_fwd_no_alloc_check_status", "ssd_fwd_no_alloc_scratch_bytes", "ssd_debug_set_withhold",
    "SSD_DEBUG_CONV_TILE", "SSD_DEBUG_FWD_CARRY", "SSD_DEBUG_SCAN_DECAYS",
    "ssd_fwd_tensor_core_steps", "tensor_core_steps", "ssd_chunk_cumsum", "ssd_chunk_state",
    "ssd_state_passing", "ssd_chunk_scan", "ssd_state_passing_hilo", "ssd_chunk_scan_hilo",
    "ssd_state_update", "ssd_status_string",
    "ssd_version", "lib_path", "load_library", "SSD_FLAG_CUDA_CORES", "SSD_FLAG_WHOLE_GROUPS",
    "SSD_FLAG_SPLIT_STEPS", "SSD_FLAG_BF16_STATES", "SSD_FLAG_SINGLE_PASS", "SSD_TC_CHUNK_STATE",
    "SSD_TC_CHUNK_SCAN",
    "SSD_TC_FUSED",
    "ssd_causal_conv1d", "ssd_conv1d_update", "ssd_conv1d_check_status",
    "ssd_bwd", "ssd_bwd_workspace_size", "ssd_selective_scan", "ssd_selective_scan_workspace_size",
    "ssd_selective_state_update", "ssd_gated_rmsnorm",
]

_PKG = os.path.dirname(os.path.abspath(__file__))
_LIB_FILE = os.path.join(_PKG, "libssd_b200.so")

SSD_OK, SSD_ERR_INVALID_ARG, SSD_ERR_UNSUPPORTED, SSD_ERR_CUDA, SSD_ERR_TIMEOUT = range(5)
SSD_F32, SSD_BF16 = 0, 1
SSD_FLAG_CUDA_CORES = 1
SSD_FLAG_WHOLE_GROUPS = 2
SSD_FLAG_SPLIT_STEPS = 4
SSD_FLAG_BF16_STATES = 8
SSD_FLAG_SINGLE_PASS = 16
SSD_TC_CHUNK_STATE, SSD_TC_CHUNK_SCAN, SSD_TC_FUSED = 1, 2, 4

_i64, _i32, _vp, _sz = ctypes.c_int64, ctypes.c_int32, ctypes.c_void_p, ctypes.c_size_t


class SsdFwdArgs(ctypes.Structure):
    """Mirror of ssd_fwd_args."""
    _fields_ = [("batch", _i64), ("seqlen", _i64), ("nheads", _i64), ("headdim", _i64),
                ("dstate", _i64), ("ngroups", _i64), ("chunk", _i64), ("dtype", _i32),
                ("flags", _i32), ("x", _vp), ("dt", _vp), ("A", _vp), ("B", _vp), ("C", _vp),
                ("D", _vp), ("dt_bias", _vp), ("init_state", _vp), ("y", _vp),
                ("final_state", _vp), ("workspace", _vp), ("workspace_bytes", _sz),
                ("z", _vp)]


class SsdBwdArgs(ctypes.Structure):
    """Mirror of ssd_bwd_args."""
    _fields_ = [("batch", _i64), ("seqlen", _i64), ("nheads", _i64), ("headdim", _i64),
                ("dstate", _i64), ("ngroups", _i64), ("chunk", _i64), ("dtype", _i32),
                ("flags", _i32), ("x", _vp), ("dt", _vp), ("A", _vp), ("B", _vp), ("C", _vp),
                ("D", _vp), ("dt_bias", _vp), ("init_state", _vp), ("dy", _vp),
                ("d_final", _vp), ("dx", _vp), ("ddt", _vp), ("dA", _vp), ("dB", _vp),
                ("dC", _vp), ("dD", _vp), ("ddt_bias", _vp), ("d_init", _vp),
                ("workspace", _vp), ("workspace_bytes", _sz)]


class SsdSelectiveScanArgs(ctypes.Structure):
    """Mirror of ssd_selective_scan_args."""
    _fields_ = [("batch", _i64), ("seqlen", _i64), ("channels", _i64), ("dstate", _i64),
                ("chunk", _i64), ("dtype", _i32), ("flags", _i32), ("x", _vp), ("dt", _vp),
                ("A", _vp), ("B", _vp), ("C", _vp), ("D", _vp), ("dt_bias", _vp),
                ("init_state", _vp), ("y", _vp), ("final_state", _vp), ("workspace", _vp),
                ("workspace_bytes", _sz)]


class SsdSelectiveStateUpdateArgs(ctypes.Structure):
    """Mirror of ssd_selective_state_update_args."""
    _fields_ = [("batch", _i64), ("channels", _i64), ("dstate", _i64), ("dtype", _i32),
                ("flags", _i32), ("state", _vp), ("x", _vp), ("dt", _vp), ("A", _vp),
                ("B", _vp), ("C", _vp), ("D", _vp), ("dt_bias", _vp), ("y", _vp)]


class SsdStateUpdateArgs(ctypes.Structure):
    """Mirror of ssd_state_update_args."""
    _fields_ = [("batch", _i64), ("nheads", _i64), ("headdim", _i64), ("dstate", _i64),
                ("ngroups", _i64), ("dtype", _i32), ("flags", _i32), ("state", _vp),
                ("x", _vp), ("dt", _vp), ("A", _vp), ("B", _vp), ("C", _vp), ("D", _vp),
                ("dt_bias", _vp), ("y", _vp), ("z", _vp)]


class SsdConv1dArgs(ctypes.Structure):
    """Mirror of ssd_conv1d_args."""
    _fields_ = [("batch", _i64), ("seqlen", _i64), ("channels", _i64), ("width", _i64),
                ("dtype", _i32), ("activation", _i32), ("x", _vp), ("weight", _vp),
                ("bias", _vp), ("init_state", _vp), ("y", _vp), ("final_state", _vp)]


class SsdConv1dUpdateArgs(ctypes.Structure):
    """Mirror of ssd_conv1d_update_args."""
    _fields_ = [("batch", _i64), ("channels", _i64), ("width", _i64), ("dtype", _i32),
                ("activation", _i32), ("state", _vp), ("x", _vp), ("weight", _vp),
                ("bias", _vp), ("y", _vp)]


class SsdGatedRmsnormArgs(ctypes.Structure):
    """Mirror of ssd_gated_rmsnorm_args."""
    _fields_ = [("rows", _i64), ("channels", _i64), ("group", _i64), ("dtype", _i32),
                ("eps", ctypes.c_float), ("y", _vp), ("z", _vp), ("weight", _vp), ("out", _vp)]


class SsdError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = f"{where}: {ssd_status_string(status)}"
        if status == SSD_ERR_CUDA:
            msg += f" ({load_library().ssd_last_cuda_error().decode()})"
        super().__init__(msg)


_lib = None


def lib_path() -> str:
    return _LIB_FILE


def load_library():
    """Load libssd_b200.so (built by mamba_ssd_scan_b200.build); raises if absent."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_FILE):
        raise RuntimeError(f"{_LIB_FILE} is missing: run `python -m mamba_ssd_scan_b200.build`")
    lib = ctypes.CDLL(_LIB_FILE)
    F = ctypes.POINTER(SsdFwdArgs)
    lib.ssd_fwd_workspace_size.restype = _sz
    lib.ssd_fwd_workspace_size.argtypes = [F]
    lib.ssd_fwd.restype = ctypes.c_int
    lib.ssd_fwd.argtypes = [F, _vp]
    lib.ssd_fwd_tensor_core_steps.restype = ctypes.c_int
    lib.ssd_fwd_tensor_core_steps.argtypes = [F]
    lib.ssd_fwd_no_alloc.restype = ctypes.c_int
    lib.ssd_fwd_no_alloc.argtypes = [F, _vp]
    lib.ssd_fwd_check_status.restype = ctypes.c_int
    lib.ssd_fwd_check_status.argtypes = [F, _vp]
    lib.ssd_fwd_no_alloc_check_status.restype = ctypes.c_int
    lib.ssd_fwd_no_alloc_check_status.argtypes = [F, _vp]
    lib.ssd_fwd_no_alloc_scratch_bytes.restype = _sz
    lib.ssd_fwd_no_alloc_scratch_bytes.argtypes = []
    lib.ssd_debug_set_withhold.restype = None
    lib.ssd_debug_set_withhold.argtypes = [ctypes.c_int, ctypes.c_int64]
    lib.ssd_chunk_cumsum.restype = ctypes.c_int
    lib.ssd_chunk_cumsum.argtypes = [F, _vp, _vp, _vp]
    lib.ssd_chunk_state.restype = ctypes.c_int
    lib.ssd_chunk_state.argtypes = [F, _vp, _vp, _vp, _vp]
    lib.ssd_state_passing.restype = ctypes.c_int
    lib.ssd_state_passing.argtypes = [F, _vp, _vp, _vp]
    lib.ssd_chunk_scan.restype = ctypes.c_int
    lib.ssd_chunk_scan.argtypes = [F, _vp, _vp, _vp, _vp]
    lib.ssd_state_passing_hilo.restype = ctypes.c_int
    lib.ssd_state_passing_hilo.argtypes = [F, _vp, _vp, _vp, _vp]
    lib.ssd_chunk_scan_hilo.restype = ctypes.c_int
    lib.ssd_chunk_scan_hilo.argtypes = [F, _vp, _vp, _vp, _vp]
    lib.ssd_state_update.restype = ctypes.c_int
    lib.ssd_state_update.argtypes = [ctypes.POINTER(SsdStateUpdateArgs), _vp]
    BW = ctypes.POINTER(SsdBwdArgs)
    lib.ssd_bwd_workspace_size.restype = _sz
    lib.ssd_bwd_workspace_size.argtypes = [BW]
    lib.ssd_bwd.restype = ctypes.c_int
    lib.ssd_bwd.argtypes = [BW, _vp]
    lib.ssd_bwd_check_status.restype = ctypes.c_int
    lib.ssd_bwd_check_status.argtypes = [BW, _vp]
    SA = ctypes.POINTER(SsdSelectiveScanArgs)
    lib.ssd_selective_scan_workspace_size.restype = _sz
    lib.ssd_selective_scan_workspace_size.argtypes = [SA]
    lib.ssd_selective_scan.restype = ctypes.c_int
    lib.ssd_selective_scan.argtypes = [SA, _vp]
    lib.ssd_selective_state_update.restype = ctypes.c_int
    lib.ssd_selective_state_update.argtypes = [ctypes.POINTER(SsdSelectiveStateUpdateArgs), _vp]
    lib.ssd_causal_conv1d.restype = ctypes.c_int
    lib.ssd_causal_conv1d.argtypes = [ctypes.POINTER(SsdConv1dArgs), _vp]
    lib.ssd_conv1d_update.restype = ctypes.c_int
    lib.ssd_conv1d_update.argtypes = [ctypes.POINTER(SsdConv1dUpdateArgs), _vp]
    lib.ssd_gated_rmsnorm.restype = ctypes.c_int
    lib.ssd_gated_rmsnorm.argtypes = [ctypes.POINTER(SsdGatedRmsnormArgs), _vp]
    lib.ssd_conv1d_check_status.restype = ctypes.c_int
    lib.ssd_conv1d_check_status.argtypes = [_vp]
    lib.ssd_status_string.restype = ctypes.c_char_p
    lib.ssd_status_string.argtypes = [ctypes.c_int]
    lib.ssd_last_cuda_error.restype = ctypes.c_char_p
    lib.ssd_last_cuda_error.argtypes = []
    lib.ssd_version.restype = ctypes.c_char_p
    lib.ssd_version.argtypes = []
    _lib = lib
    return lib


def ssd_status_string(status: int) -> str:
    return load_library().ssd_status_string(int(status)).decode()


def ssd_version() -> str:
    return load_library().ssd_version().decode()


# ---------------------------------------------------------------------------
def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return SSD_F32
    if t.dtype == torch.bfloat16:
        return SSD_BF16
    raise TypeError(f"unsupported dtype {t.dtype} (float32 or bfloat16)")


def _ptr(t) -> int | None:
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return t.data_ptr()


def _stream_ptr(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _check(status: int, where: str):
    if status != SSD_OK:
        raise SsdError(status, where)


def _fwd_args(x, dt, A, B, C, D, dt_bias, chunk, init_state, y, final_state, flags, z=None):
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    a = SsdFwdArgs()
    a.batch, a.seqlen, a.nheads, a.headdim, a.dstate, a.ngroups, a.chunk = b, L, H, P, N, G, chunk
    a.dtype = _dtype_code(x)
    a.flags = int(flags)
    for name, t in (("dt", dt), ("B", B), ("C", C), ("z", z)):
        if t is not None and t.dtype != x.dtype:
            raise TypeError(f"{name} must have x's dtype {x.dtype}")
    if z is not None and tuple(z.shape) != tuple(x.shape):
        raise ValueError("z must have x's shape")
    for name, t in (("A", A), ("D", D), ("dt_bias", dt_bias), ("init_state", init_state)):
        if t is not None and t.dtype != torch.float32:
            raise TypeError(f"{name} must be float32")
    a.x, a.dt, a.A, a.B, a.C = _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C)
    a.D, a.dt_bias, a.init_state = _ptr(D), _ptr(dt_bias), _ptr(init_state)
    a.y, a.final_state = _ptr(y), _ptr(final_state)
    a.z = _ptr(z)
    return a


def ssd_fwd_workspace_size(batch, seqlen, nheads, headdim, dstate, ngroups, chunk,
                           dtype=torch.bfloat16, flags: int = 0) -> int:
    a = SsdFwdArgs()
    a.batch, a.seqlen, a.nheads, a.headdim, a.dstate, a.ngroups, a.chunk = (
        batch, seqlen, nheads, headdim, dstate, ngroups, chunk)
    a.dtype = SSD_BF16 if dtype == torch.bfloat16 else SSD_F32
    a.flags = flags
    return int(load_library().ssd_fwd_workspace_size(ctypes.byref(a)))


def ssd_fwd_tensor_core_steps(batch, seqlen, nheads, headdim, dstate, ngroups, chunk,
                              dtype=torch.bfloat16, flags: int = 0) -> int:
    """Bitmask of the ssd_fwd steps that run on the tensor cores for these sizes
    (1 = chunk_state, 2 = chunk_scan, 4 = the whole forward as one kernel, with
    SSD_FLAG_SINGLE_PASS)."""
    a = SsdFwdArgs()
    a.batch, a.seqlen, a.nheads, a.headdim, a.dstate, a.ngroups, a.chunk = (
        batch, seqlen, nheads, headdim, dstate, ngroups, chunk)
    a.dtype = SSD_BF16 if dtype == torch.bfloat16 else SSD_F32
    a.flags = flags
    return int(load_library().ssd_fwd_tensor_core_steps(ctypes.byref(a)))


def tensor_core_steps(batch, seqlen, nheads, headdim, dstate, ngroups, chunk,
                      dtype=torch.bfloat16, flags: int = 0) -> set:
    """Names of the ssd_fwd steps that run on the tensor cores for these sizes."""
    m = ssd_fwd_tensor_core_steps(batch, seqlen, nheads, headdim, dstate, ngroups, chunk,
                                  dtype, flags)
    return {n for bit, n in ((1, "chunk_state"), (2, "chunk_scan"), (4, "fused")) if m & bit}


def ssd_fwd(x, dt, A, B, C, D=None, dt_bias=None, chunk: int = 256, init_state=None, *,
            return_final_state: bool = False, y=None, final_state=None, workspace=None,
            flags: int = 0, stream=None, z=None):
    """The SSD scan forward.  x [b,L,H,P], dt [b,L,H] (raw), B/C [b,L,G,N] in one
    dtype (float32 or bfloat16); A, D, dt_bias [H] and init_state [b,H,P,N]
    float32; z (optional output gate, x's shape and dtype): y *= silu(z).
    Returns y (and the final fp32 state when asked)."""
    lib = load_library()
    if y is None:
        y = torch.empty_like(x)
    if final_state is None and return_final_state:
        final_state = torch.empty((x.shape[0], x.shape[2], x.shape[3], B.shape[3]),
                                  dtype=torch.float32, device=x.device)
    a = _fwd_args(x, dt, A, B, C, D, dt_bias, chunk, init_state, y, final_state, flags, z)
    need = int(lib.ssd_fwd_workspace_size(ctypes.byref(a)))
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=x.device)
    a.workspace = workspace.data_ptr()
    a.workspace_bytes = workspace.numel() * workspace.element_size()
    _check(lib.ssd_fwd(ctypes.byref(a), _stream_ptr(stream)), "ssd_fwd")
    if final_state is not None:
        return y, final_state
    return y


def _bwd_args(x, dt, A, B, C, D, dt_bias, chunk, init_state, flags):
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    a = SsdBwdArgs()
    a.batch, a.seqlen, a.nheads, a.headdim, a.dstate, a.ngroups, a.chunk = b, L, H, P, N, G, chunk
    a.dtype = _dtype_code(x)
    a.flags = int(flags)
    for name, t in (("dt", dt), ("B", B), ("C", C)):
        if t.dtype != x.dtype:
            raise TypeError(f"{name} must have x's dtype {x.dtype}")
    for name, t in (("A", A), ("D", D), ("dt_bias", dt_bias), ("init_state", init_state)):
        if t is not None and t.dtype != torch.float32:
            raise TypeError(f"{name} must be float32")
    a.x, a.dt, a.A, a.B, a.C = _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C)
    a.D, a.dt_bias, a.init_state = _ptr(D), _ptr(dt_bias), _ptr(init_state)
    return a


def ssd_bwd_workspace_size(batch, seqlen, nheads, headdim, dstate, ngroups, chunk,
                           dtype=torch.bfloat16, flags: int = 0) -> int:
    a = SsdBwdArgs()
    a.batch, a.seqlen, a.nheads, a.headdim, a.dstate, a.ngroups, a.chunk = (
        batch, seqlen, nheads, headdim, dstate, ngroups, chunk)
    a.dtype = SSD_BF16 if dtype == torch.bfloat16 else SSD_F32
    a.flags = flags
    return int(load_library().ssd_bwd_workspace_size(ctypes.byref(a)))


def ssd_bwd(x, dt, A, B, C, dy, D=None, dt_bias=None, chunk: int = 256, init_state=None,
            d_final=None, *, out=None, workspace=None, flags: int = 0, stream=None) -> dict:
    """The backward pass of ssd_fwd (no output gate): gradients of
    sum(dy * y) + sum(d_final * final_state) with respect to every input.
    dy has x's shape and dtype; d_final [b,H,P,N] float32 or None.  Returns a
    dict dx, ddt (of the raw dt), dB, dC (input dtype), dA, dD, ddt_bias [H]
    and d_init [b,H,P,N] (float32); ``out`` may hold preallocated tensors under
    the same keys."""
    lib = load_library()
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    if dy.dtype != x.dtype or tuple(dy.shape) != tuple(x.shape):
        raise TypeError("dy must have x's shape and dtype")
    if d_final is not None and d_final.dtype != torch.float32:
        raise TypeError("d_final must be float32")
    o = dict(out or {})
    o.setdefault("dx", torch.empty_like(x))
    o.setdefault("ddt", torch.empty_like(dt))
    o.setdefault("dB", torch.empty_like(B))
    o.setdefault("dC", torch.empty_like(C))
    o.setdefault("dA", torch.empty(H, dtype=torch.float32, device=x.device))
    o.setdefault("dD", torch.empty(H, dtype=torch.float32, device=x.device))
    o.setdefault("ddt_bias", torch.empty(H, dtype=torch.float32, device=x.device))
    o.setdefault("d_init", torch.empty((b, H, P, N), dtype=torch.float32, device=x.device))
    a = _bwd_args(x, dt, A, B, C, D, dt_bias, chunk, init_state, flags)
    a.dy, a.d_final = _ptr(dy), _ptr(d_final)
    a.dx, a.ddt, a.dA, a.dB, a.dC = (_ptr(o["dx"]), _ptr(o["ddt"]), _ptr(o["dA"]), _ptr(o["dB"]),
                                     _ptr(o["dC"]))
    a.dD, a.ddt_bias, a.d_init = _ptr(o["dD"]), _ptr(o["ddt_bias"]), _ptr(o["d_init"])
    need = int(lib.ssd_bwd_workspace_size(ctypes.byref(a)))
    if need == 0:
        raise SsdError(SSD_ERR_UNSUPPORTED, "ssd_bwd (sizes)")
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    a.workspace = workspace.data_ptr()
    a.workspace_bytes = workspace.numel() * workspace.element_size()
    _check(lib.ssd_bwd(ctypes.byref(a), _stream_ptr(stream)), "ssd_bwd")
    return o


SSD_DEBUG_CONV_TILE = 0
SSD_DEBUG_FWD_CARRY = 1
SSD_DEBUG_SCAN_DECAYS = 2


def ssd_debug_set_withhold(what: int, index: int) -> None:
    """Test hook (include/ssd.h): make one producer withhold one hand-off so
    the consumers' bounded waits run out; index < 0 turns it off."""
    load_library().ssd_debug_set_withhold(int(what), int(index))


def ssd_fwd_no_alloc_scratch_bytes() -> int:
    """The size of the library's built-in scratch buffer (bytes)."""
    return int(load_library().ssd_fwd_no_alloc_scratch_bytes())


def ssd_fwd_no_alloc(x, dt, A, B, C, D=None, dt_bias=None, chunk: int = 256, init_state=None,
                     *, y, final_state=None, flags: int = 0, stream=None, z=None):
    """ssd_fwd without a workspace, for callers that cannot allocate: the
    scratch comes from a fixed buffer inside the library (see ssd_fwd_no_alloc
    in include/ssd.h).  ``y`` (and ``final_state``, if wanted) are caller-owned
    outputs; calls that can overlap on the GPU race and must be serialised.
    Sizes beyond the buffer are rejected by the library (SsdError,
    SSD_ERR_UNSUPPORTED) before anything is launched."""
    lib = load_library()
    a = _fwd_args(x, dt, A, B, C, D, dt_bias, chunk, init_state, y, final_state, flags, z)
    _check(lib.ssd_fwd_no_alloc(ctypes.byref(a), _stream_ptr(stream)), "ssd_fwd_no_alloc")
    return y


def ssd_fwd_no_alloc_check_status(x, B, chunk: int, flags: int = 0, stream=None) -> int:
    """Synchronise and return the device status of the last ssd_fwd_no_alloc
    call on the current device with these sizes (SSD_OK = 0,
    SSD_ERR_TIMEOUT = 4)."""
    b, L, H, P = x.shape
    a = SsdFwdArgs()
    a.batch, a.seqlen, a.nheads, a.headdim, a.dstate, a.ngroups, a.chunk = (
        b, L, H, P, B.shape[3], B.shape[2], chunk)
    a.dtype = _dtype_code(x)
    a.flags = flags
    return int(load_library().ssd_fwd_no_alloc_check_status(ctypes.byref(a),
                                                            _stream_ptr(stream)))


def ssd_fwd_check_status(x, B, chunk: int, workspace, flags: int = 0, stream=None) -> int:
    """Synchronise and return the device status of the last ssd_fwd call that
    used ``workspace`` (SSD_OK = 0, SSD_ERR_TIMEOUT = 4)."""
    b, L, H, P = x.shape
    a = SsdFwdArgs()
    a.batch, a.seqlen, a.nheads, a.headdim, a.dstate, a.ngroups, a.chunk = (
        b, L, H, P, B.shape[3], B.shape[2], chunk)
    a.dtype = _dtype_code(x)
    a.flags = flags
    a.workspace = workspace.data_ptr()
    a.workspace_bytes = workspace.numel() * workspace.element_size()
    return int(load_library().ssd_fwd_check_status(ctypes.byref(a), _stream_ptr(stream)))


def _intermediate_shapes(x, B, chunk):
    b, L, H, P = x.shape
    N = B.shape[3]
    nc = (L + chunk - 1) // chunk
    return (b, H, nc, chunk), (b, nc, H, P, N)


def _states_dtype(x, flags):
    """The chunk states are fp32, except bf16 inputs in the bf16-states mode."""
    if x.dtype == torch.bfloat16 and flags & SSD_FLAG_BF16_STATES:
        return torch.bfloat16
    return torch.float32


def ssd_chunk_cumsum(x, dt, A, B, C, dt_bias=None, chunk: int = 256, *, dt_out=None,
                     cumA_out=None, stream=None):
    """Step 1: returns (dt, cumA), each [b, H, nc, chunk] float32."""
    lib = load_library()
    vshape, _ = _intermediate_shapes(x, B, chunk)
    dt_out = dt_out if dt_out is not None else torch.empty(vshape, dtype=torch.float32,
                                                           device=x.device)
    cumA_out = cumA_out if cumA_out is not None else torch.empty_like(dt_out)
    a = _fwd_args(x, dt, A, B, C, None, dt_bias, chunk, None, None, None, 0)
    _check(lib.ssd_chunk_cumsum(ctypes.byref(a), _ptr(dt_out), _ptr(cumA_out),
                                _stream_ptr(stream)), "ssd_chunk_cumsum")
    return dt_out, cumA_out


def ssd_chunk_state(x, dt, A, B, C, dt_sp, cumA, chunk: int = 256, *, states=None,
                    stream=None, flags: int = 0):
    """Step 2: returns the chunk-local states [b, nc, H, P, N], fp32 (bf16 for
    bf16 inputs with SSD_FLAG_BF16_STATES).  ``dt_sp``/``cumA`` are step 1's
    outputs."""
    lib = load_library()
    _, sshape = _intermediate_shapes(x, B, chunk)
    states = states if states is not None else torch.empty(
        sshape, dtype=_states_dtype(x, flags), device=x.device)
    a = _fwd_args(x, dt, A, B, C, None, None, chunk, None, None, None, flags)
    _check(lib.ssd_chunk_state(ctypes.byref(a), _ptr(dt_sp), _ptr(cumA), _ptr(states),
                               _stream_ptr(stream)), "ssd_chunk_state")
    return states


def ssd_state_passing(x, dt, A, B, C, cumA, states, chunk: int = 256, init_state=None,
                      final_state=None, stream=None, flags: int = 0):
    """Step 3, in place: ``states`` goes from chunk-local states to the states
    entering each chunk.  Writes ``final_state`` if given.  Returns states."""
    lib = load_library()
    a = _fwd_args(x, dt, A, B, C, None, None, chunk, init_state, None, final_state, flags)
    _check(lib.ssd_state_passing(ctypes.byref(a), _ptr(cumA), _ptr(states),
                                 _stream_ptr(stream)), "ssd_state_passing")
    return states


def ssd_chunk_scan(x, dt, A, B, C, dt_sp, cumA, states, D=None, chunk: int = 256, *, y=None,
                   stream=None, z=None, flags: int = 0):
    """Step 4: y from the chunk's tokens and the states entering each chunk
    (times silu(z) when the gate z is given)."""
    lib = load_library()
    y = y if y is not None else torch.empty_like(x)
    a = _fwd_args(x, dt, A, B, C, D, None, chunk, None, y, None, flags, z)
    _check(lib.ssd_chunk_scan(ctypes.byref(a), _ptr(dt_sp), _ptr(cumA), _ptr(states),
                              _stream_ptr(stream)), "ssd_chunk_scan")
    return y


def ssd_state_passing_hilo(x, dt, A, B, C, cumA, states, chunk: int = 256, init_state=None,
                           final_state=None, *, states_hl=None, stream=None, flags: int = 0):
    """Step 3 as ssd_fwd runs it for bf16 on the tensor cores: the fp32 local
    ``states`` (not modified) -> the states entering each chunk as hi / lo bf16
    halves, returned as ``states_hl`` [2, b, nc, H, P, N] (hi, then lo).
    Writes ``final_state`` if given."""
    lib = load_library()
    _, sshape = _intermediate_shapes(x, B, chunk)
    states_hl = states_hl if states_hl is not None else torch.empty(
        (2,) + sshape, dtype=torch.bfloat16, device=x.device)
    a = _fwd_args(x, dt, A, B, C, None, None, chunk, init_state, None, final_state, flags)
    _check(lib.ssd_state_passing_hilo(ctypes.byref(a), _ptr(cumA), _ptr(states), _ptr(states_hl),
                                      _stream_ptr(stream)), "ssd_state_passing_hilo")
    return states_hl


def ssd_chunk_scan_hilo(x, dt, A, B, C, dt_sp, cumA, states_hl, D=None, chunk: int = 256, *,
                        y=None, stream=None, z=None, flags: int = 0):
    """Step 4 on the tensor cores from the hi / lo entering states of
    ssd_state_passing_hilo (times silu(z) when the gate z is given)."""
    lib = load_library()
    y = y if y is not None else torch.empty_like(x)
    a = _fwd_args(x, dt, A, B, C, D, None, chunk, None, y, None, flags, z)
    _check(lib.ssd_chunk_scan_hilo(ctypes.byref(a), _ptr(dt_sp), _ptr(cumA), _ptr(states_hl),
                                   _stream_ptr(stream)), "ssd_chunk_scan_hilo")
    return y


def ssd_state_update(state, x, dt, A, B, C, D=None, dt_bias=None, *, y=None, stream=None,
                     z=None):
    """One decode step, in place on ``state`` [b,H,P,N] float32.  x [b,H,P],
    dt [b,H], B/C [b,G,N] in one dtype; z (optional output gate, x's shape and
    dtype).  Returns y [b,H,P] in x's dtype."""
    lib = load_library()
    b, H, P, N = state.shape
    G = B.shape[1]
    if state.dtype != torch.float32:
        raise TypeError("state must be float32")
    y = y if y is not None else torch.empty_like(x)
    a = SsdStateUpdateArgs()
    a.batch, a.nheads, a.headdim, a.dstate, a.ngroups = b, H, P, N, G
    a.dtype = _dtype_code(x)
    a.flags = 0
    a.state, a.x, a.dt, a.A, a.B, a.C = (_ptr(state), _ptr(x), _ptr(dt), _ptr(A), _ptr(B),
                                         _ptr(C))
    if z is not None and (z.dtype != x.dtype or tuple(z.shape) != tuple(x.shape)):
        raise TypeError("z must have x's shape and dtype")
    a.D, a.dt_bias, a.y, a.z = _ptr(D), _ptr(dt_bias), _ptr(y), _ptr(z)
    _check(lib.ssd_state_update(ctypes.byref(a), _stream_ptr(stream)), "ssd_state_update")
    return y


def ssd_causal_conv1d(x, weight, bias=None, init_state=None, *, activation: bool = True,
                      y=None, final_state=None, return_final_state: bool = False, stream=None):
    """Causal depthwise conv1d (+ SiLU) in front of the scan.  x [b,L,C] float32
    or bfloat16; weight [C,K] float32; bias [C] float32 or None; init_state
    [b,C,K-1] float32 or None.  Returns y (and the final [b,C,K-1] state when
    asked)."""
    lib = load_library()
    b, L, Cn = x.shape
    K = weight.shape[1]
    for name, t in (("weight", weight), ("bias", bias), ("init_state", init_state),
                    ("final_state", final_state)):
        if t is not None and t.dtype != torch.float32:
            raise TypeError(f"{name} must be float32")
    y = y if y is not None else torch.empty_like(x)
    if final_state is None and return_final_state and K > 1:
        final_state = torch.empty((b, Cn, K - 1), dtype=torch.float32, device=x.device)
    a = SsdConv1dArgs()
    a.batch, a.seqlen, a.channels, a.width = b, L, Cn, K
    a.dtype = _dtype_code(x)
    a.activation = 1 if activation else 0
    a.x, a.weight, a.bias, a.init_state = _ptr(x), _ptr(weight), _ptr(bias), _ptr(init_state)
    a.y, a.final_state = _ptr(y), _ptr(final_state)
    _check(lib.ssd_causal_conv1d(ctypes.byref(a), _stream_ptr(stream)), "ssd_causal_conv1d")
    if return_final_state:
        return y, final_state
    return y


def _sel_args(x, dt, A, B, C, D, dt_bias, chunk, init_state, y, final_state):
    b, L, Dc = x.shape
    N = A.shape[1]
    for name, t in (("dt", dt), ("B", B), ("C", C)):
        if t.dtype != x.dtype:
            raise TypeError(f"{name} must have x's dtype {x.dtype}")
    for name, t in (("A", A), ("D", D), ("dt_bias", dt_bias), ("init_state", init_state),
                    ("final_state", final_state)):
        if t is not None and t.dtype != torch.float32:
            raise TypeError(f"{name} must be float32")
    a = SsdSelectiveScanArgs()
    a.batch, a.seqlen, a.channels, a.dstate, a.chunk = b, L, Dc, N, chunk
    a.dtype = _dtype_code(x)
    a.flags = 0
    a.x, a.dt, a.A, a.B, a.C = _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C)
    a.D, a.dt_bias, a.init_state = _ptr(D), _ptr(dt_bias), _ptr(init_state)
    a.y, a.final_state = _ptr(y), _ptr(final_state)
    return a


def ssd_selective_scan(x, dt, A, B, C, D=None, dt_bias=None, chunk: int = 64, init_state=None,
                       *, y=None, final_state=None, return_final_state: bool = False,
                       workspace=None, stream=None):
    """The diagonal-A (Mamba-1 form) selective scan.  x, dt [b,L,Dc] and B, C
    [b,L,N] in one dtype; A [Dc,N], D, dt_bias [Dc], init_state [b,Dc,N] fp32.
    Returns y (and the final fp32 state when asked)."""
    lib = load_library()
    b, L, Dc = x.shape
    N = A.shape[1]
    y = y if y is not None else torch.empty_like(x)
    if final_state is None and return_final_state:
        final_state = torch.empty((b, Dc, N), dtype=torch.float32, device=x.device)
    a = _sel_args(x, dt, A, B, C, D, dt_bias, chunk, init_state, y, final_state)
    need = int(lib.ssd_selective_scan_workspace_size(ctypes.byref(a)))
    if need == 0:
        raise SsdError(SSD_ERR_UNSUPPORTED, "ssd_selective_scan (sizes)")
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    a.workspace = workspace.data_ptr()
    a.workspace_bytes = workspace.numel() * workspace.element_size()
    _check(lib.ssd_selective_scan(ctypes.byref(a), _stream_ptr(stream)), "ssd_selective_scan")
    if final_state is not None:
        return y, final_state
    return y


def ssd_selective_scan_workspace_size(batch, seqlen, channels, dstate, chunk,
                                      dtype=torch.bfloat16) -> int:
    a = SsdSelectiveScanArgs()
    a.batch, a.seqlen, a.channels, a.dstate, a.chunk = batch, seqlen, channels, dstate, chunk
    a.dtype = SSD_BF16 if dtype == torch.bfloat16 else SSD_F32
    return int(load_library().ssd_selective_scan_workspace_size(ctypes.byref(a)))


def ssd_selective_state_update(state, x, dt, A, B, C, D=None, dt_bias=None, *, y=None,
                               stream=None):
    """One decode step of the diagonal-A scan, in place on state [b,Dc,N] fp32;
    x, dt [b,Dc] and B, C [b,N] in one dtype.  Returns y [b,Dc]."""
    lib = load_library()
    b, Dc = x.shape
    N = A.shape[1]
    if state.dtype != torch.float32:
        raise TypeError("state must be float32")
    y = y if y is not None else torch.empty_like(x)
    a = SsdSelectiveStateUpdateArgs()
    a.batch, a.channels, a.dstate = b, Dc, N
    a.dtype = _dtype_code(x)
    a.flags = 0
    a.state, a.x, a.dt, a.A, a.B, a.C = (_ptr(state), _ptr(x), _ptr(dt), _ptr(A), _ptr(B),
                                         _ptr(C))
    a.D, a.dt_bias, a.y = _ptr(D), _ptr(dt_bias), _ptr(y)
    _check(lib.ssd_selective_state_update(ctypes.byref(a), _stream_ptr(stream)),
           "ssd_selective_state_update")
    return y


def ssd_conv1d_check_status(stream=None) -> int:
    """Synchronises the stream; SSD_ERR_TIMEOUT if a forward convolution on
    this device gave up on an internal wait since the last check, else 0."""
    return int(load_library().ssd_conv1d_check_status(_stream_ptr(stream)))


def ssd_conv1d_update(state, x, weight, bias=None, *, activation: bool = True, y=None,
                      stream=None):
    """One decode step of the convolution, in place on ``state`` [b,C,K-1]
    float32.  x [b,C].  Returns y [b,C] in x's dtype."""
    lib = load_library()
    b, Cn = x.shape
    K = weight.shape[1]
    if state is not None and state.dtype != torch.float32:
        raise TypeError("state must be float32")
    y = y if y is not None else torch.empty_like(x)
    a = SsdConv1dUpdateArgs()
    a.batch, a.channels, a.width = b, Cn, K
    a.dtype = _dtype_code(x)
    a.activation = 1 if activation else 0
    a.state, a.x, a.weight, a.bias, a.y = _ptr(state), _ptr(x), _ptr(weight), _ptr(bias), _ptr(y)
    _check(lib.ssd_conv1d_update(ctypes.byref(a), _stream_ptr(stream)), "ssd_conv1d_update")
    return y


def ssd_gated_rmsnorm(y, z, weight, *, group: int | None = None, eps: float = 1e-5, out=None,
                      stream=None):
    """RMSNorm of g = y * silu(z) (g = y when z is None) over each group of
    ``group`` consecutive channels of the last axis (default: the whole last
    axis), times weight [channels] float32.  y, z: [..., channels] in one
    dtype.  ``out`` may be ``y`` (in place).  Returns out."""
    lib = load_library()
    channels = y.shape[-1]
    rows = y.numel() // channels
    if z is not None and (z.dtype != y.dtype or z.shape != y.shape):
        raise TypeError("z must match y in dtype and shape")
    if weight.dtype != torch.float32 or weight.numel() != channels:
        raise TypeError("weight must be float32 with one entry per channel")
    out = out if out is not None else torch.empty_like(y)
    a = SsdGatedRmsnormArgs()
    a.rows, a.channels, a.group = rows, channels, int(group if group is not None else channels)
    a.dtype = _dtype_code(y)
    a.eps = float(eps)
    a.y, a.z, a.weight, a.out = _ptr(y), _ptr(z), _ptr(weight), _ptr(out)
    _check(lib.ssd_gated_rmsnorm(ctypes.byref(a), _stream_ptr(stream)), "ssd_gated_rmsnorm")
    return out
