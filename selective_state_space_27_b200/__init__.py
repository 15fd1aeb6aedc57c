"""B200 (sm_100a) selective scan (S6): Python binding of the C ABI in include/mambascan.h.

Two operations of the Mamba selective state-space layer ("Notas sobre Mamba",
section "O mecanismo de seleção (S6)"; "Mamba-2 e State Space Duality (SSD)",
section "Como o Mamba-1 alcançou complexidade linear"):

* :func:`scan_fwd` -- the fused selective scan over a sequence: y and the final
  state, with delta = softplus(delta_raw + delta_bias), Abar = exp(delta A),
  Bbar = delta B, h_t = Abar_t h_{t-1} + Bbar_t u_t, y_t = C_t h_t + D u_t,
  optionally times silu(z_t).
* :func:`state_update` -- the same recurrence for one token, on a state
  updated in place (decode).

This module only marshals arguments: PyTorch supplies device memory and the
current CUDA stream, and every step of the computation runs in the CUDA
kernels of ``libmambascan.so``. There is no CPU fallback: if the library is
missing or cannot be loaded, every call raises.
"""
from __future__ import annotations

import ctypes
import os

__all__ = [
    "scan_fwd", "state_update", "scan_workspace_size", "scan_plan", "scan_configs", "library_path",
    "load_library", "MambaScanError", "ScanArgs", "UpdateArgs", "ScanPlan", "MS_F32", "MS_BF16",
    "Conv1dArgs", "conv_scan_fwd", "conv_state_update", "build_conv_args", "trap_scan_fwd",
    "ScanBwdArgs", "scan_bwd", "SsdArgs", "build_ssd_args", "ssd_fwd", "ssd_check", "SSD_WORKSPACE_BYTES",
    "MAX_DSTATE", "probe_unit_throughput", "PROBE_UNITS", "plan_workspace_size", "scan_status",
]

_PKG = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_PKG, "libmambascan.so")
_lib = None

MS_F32, MS_BF16 = 0, 1
MAX_DSTATE = 16
SSD_HEADDIM, SSD_DSTATE, SSD_WORKSPACE_BYTES = 64, 128, 256
STATUS = {0: "MS_OK", 1: "MS_ERR_INVALID_ARG", 2: "MS_ERR_UNSUPPORTED", 3: "MS_ERR_ALIGNMENT",
          4: "MS_ERR_CUDA", 5: "MS_ERR_TIMEOUT", 6: "MS_ERR_WORKSPACE"}

_i64 = ctypes.c_int64
_i32 = ctypes.c_int32
_vp = ctypes.c_void_p


class ScanArgs(ctypes.Structure):
    """Mirror of ``ms_scan_args``."""
    _fields_ = [
        ("batch", _i64), ("dim", _i64), ("dstate", _i64), ("seqlen", _i64),
        ("in_dtype", _i32), ("delta_softplus", _i32),
        ("u", _vp), ("u_batch_stride", _i64), ("u_dim_stride", _i64),
        ("delta", _vp), ("delta_batch_stride", _i64), ("delta_dim_stride", _i64),
        ("B", _vp), ("B_batch_stride", _i64), ("B_state_stride", _i64),
        ("C", _vp), ("C_batch_stride", _i64), ("C_state_stride", _i64),
        ("z", _vp), ("z_batch_stride", _i64), ("z_dim_stride", _i64),
        ("y", _vp), ("y_batch_stride", _i64), ("y_dim_stride", _i64),
        ("A", _vp), ("D", _vp), ("delta_bias", _vp), ("initial_state", _vp), ("final_state", _vp),
        ("force_segments", _i32), ("reserved", _i32),
    ]


class UpdateArgs(ctypes.Structure):
    """Mirror of ``ms_update_args``."""
    _fields_ = [
        ("batch", _i64), ("dim", _i64), ("dstate", _i64),
        ("in_dtype", _i32), ("delta_softplus", _i32),
        ("state", _vp), ("state_batch_stride", _i64), ("state_dim_stride", _i64),
        ("x", _vp), ("x_batch_stride", _i64),
        ("delta", _vp), ("delta_batch_stride", _i64),
        ("B", _vp), ("B_batch_stride", _i64),
        ("C", _vp), ("C_batch_stride", _i64),
        ("z", _vp), ("z_batch_stride", _i64),
        ("y", _vp), ("y_batch_stride", _i64),
        ("A", _vp), ("D", _vp), ("delta_bias", _vp),
    ]


class Conv1dArgs(ctypes.Structure):
    """Mirror of ``ms_conv1d_args``."""
    _fields_ = [("weight", _vp), ("bias", _vp), ("width", _i32), ("silu", _i32)]


class ScanBwdArgs(ctypes.Structure):
    """Mirror of ``ms_scan_bwd_args``."""
    _fields_ = [
        ("dy", _vp), ("dy_batch_stride", _i64), ("dy_dim_stride", _i64),
        ("dfinal_state", _vp),
        ("du", _vp), ("du_batch_stride", _i64), ("du_dim_stride", _i64),
        ("ddelta", _vp), ("ddelta_batch_stride", _i64), ("ddelta_dim_stride", _i64),
        ("dz", _vp), ("dz_batch_stride", _i64), ("dz_dim_stride", _i64),
        ("dA", _vp), ("dB", _vp), ("dC", _vp), ("dD", _vp), ("ddelta_bias", _vp), ("dinitial_state", _vp),
    ]


class SsdArgs(ctypes.Structure):
    """Mirror of ``ms_ssd_args``."""
    _fields_ = [
        ("batch", _i64), ("seqlen", _i64), ("nheads", _i64), ("ngroups", _i64),
        ("in_dtype", _i32), ("dt_softplus", _i32),
        ("x", _vp), ("x_batch_stride", _i64), ("x_token_stride", _i64),
        ("dt", _vp), ("dt_batch_stride", _i64), ("dt_token_stride", _i64),
        ("B", _vp), ("B_batch_stride", _i64), ("B_token_stride", _i64),
        ("C", _vp), ("C_batch_stride", _i64), ("C_token_stride", _i64),
        ("z", _vp), ("z_batch_stride", _i64), ("z_token_stride", _i64),
        ("y", _vp), ("y_batch_stride", _i64), ("y_token_stride", _i64),
        ("A", _vp), ("D", _vp), ("dt_bias", _vp), ("initial_state", _vp), ("final_state", _vp),
        ("wait_limit_us", ctypes.c_uint32), ("withhold_block", _i32),
    ]


class ScanPlan(ctypes.Structure):
    """Mirror of ``ms_scan_plan``."""
    _fields_ = [
        ("config", _i32), ("warps_per_cta", _i32), ("segments", _i32), ("lanes", _i32),
        ("segment_len", _i64), ("workspace_bytes", ctypes.c_uint64), ("ctas", _i32), ("reserved", _i32),
    ]


class MambaScanError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS.get(status, status)}: {message}")
        self.status = status


def library_path() -> str:
    return _LIB_PATH


def load_library():
    """Load libmambascan.so (built by ``python -m selective_state_space_27_b200.build``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(f"CUDA library not built: {_LIB_PATH} is missing "
                               "(run python -m selective_state_space_27_b200.build)")
        lib = ctypes.CDLL(_LIB_PATH)
        lib.mamba_status_string.restype = ctypes.c_char_p
        lib.mamba_status_string.argtypes = [ctypes.c_int]
        lib.mamba_last_error.restype = ctypes.c_char_p
        lib.mamba_last_error.argtypes = []
        lib.mamba_abi_version.restype = ctypes.c_int
        lib.mamba_abi_version.argtypes = []
        lib.mamba_scan_workspace_size.restype = ctypes.c_int
        lib.mamba_scan_workspace_size.argtypes = [ctypes.POINTER(ScanArgs), ctypes.POINTER(ctypes.c_size_t)]
        lib.mamba_scan_fwd.restype = ctypes.c_int
        lib.mamba_scan_fwd.argtypes = [ctypes.POINTER(ScanArgs), _vp, ctypes.c_size_t, _vp]
        lib.mamba_state_update.restype = ctypes.c_int
        lib.mamba_state_update.argtypes = [ctypes.POINTER(UpdateArgs), _vp]
        lib.mamba_scan_num_configs.restype = ctypes.c_int
        lib.mamba_scan_num_configs.argtypes = []
        lib.mamba_scan_config_info.restype = ctypes.c_int
        lib.mamba_scan_config_info.argtypes = [ctypes.c_int, ctypes.POINTER(ctypes.c_int),
                                               ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_int)]
        lib.mamba_conv_scan_fwd.restype = ctypes.c_int
        lib.mamba_conv_scan_fwd.argtypes = [ctypes.POINTER(ScanArgs), ctypes.POINTER(Conv1dArgs),
                                            ctypes.POINTER(ScanPlan), _vp]
        lib.mamba_conv_state_update.restype = ctypes.c_int
        lib.mamba_conv_state_update.argtypes = [ctypes.POINTER(UpdateArgs), ctypes.POINTER(Conv1dArgs), _vp,
                                                ctypes.c_int64, ctypes.c_int64, _vp]
        lib.mamba_trap_scan_fwd.restype = ctypes.c_int
        lib.mamba_trap_scan_fwd.argtypes = [ctypes.POINTER(ScanArgs), _vp, ctypes.c_int64, ctypes.c_int64,
                                            ctypes.POINTER(ScanPlan), _vp]
        lib.mamba_scan_bwd_workspace_size.restype = ctypes.c_int
        lib.mamba_scan_bwd_workspace_size.argtypes = [ctypes.POINTER(ScanArgs), ctypes.POINTER(ctypes.c_size_t)]
        lib.mamba_conv_scan_workspace_size.restype = ctypes.c_int
        lib.mamba_conv_scan_workspace_size.argtypes = [ctypes.POINTER(ScanArgs), ctypes.POINTER(Conv1dArgs),
                                                       ctypes.POINTER(ScanPlan), ctypes.POINTER(ctypes.c_size_t)]
        lib.mamba_conv_scan_fwd_ws.restype = ctypes.c_int
        lib.mamba_conv_scan_fwd_ws.argtypes = [ctypes.POINTER(ScanArgs), ctypes.POINTER(Conv1dArgs),
                                               ctypes.POINTER(ScanPlan), _vp, ctypes.c_size_t, _vp]
        lib.mamba_trap_scan_workspace_size.restype = ctypes.c_int
        lib.mamba_trap_scan_workspace_size.argtypes = [ctypes.POINTER(ScanArgs), _vp, ctypes.c_int64, ctypes.c_int64,
                                                       ctypes.POINTER(ScanPlan), ctypes.POINTER(ctypes.c_size_t)]
        lib.mamba_trap_scan_fwd_ws.restype = ctypes.c_int
        lib.mamba_trap_scan_fwd_ws.argtypes = [ctypes.POINTER(ScanArgs), _vp, ctypes.c_int64, ctypes.c_int64,
                                               ctypes.POINTER(ScanPlan), _vp, ctypes.c_size_t, _vp]
        lib.mamba_scan_fwd_checkpointed.restype = ctypes.c_int
        lib.mamba_scan_fwd_checkpointed.argtypes = [ctypes.POINTER(ScanArgs), _vp, ctypes.c_size_t, _vp,
                                                    ctypes.c_size_t, _vp]
        lib.mamba_scan_bwd_checkpointed.restype = ctypes.c_int
        lib.mamba_scan_bwd_checkpointed.argtypes = [ctypes.POINTER(ScanArgs), ctypes.POINTER(ScanBwdArgs), _vp,
                                                    ctypes.c_size_t, _vp]
        lib.mamba_scan_bwd.restype = ctypes.c_int
        lib.mamba_scan_bwd.argtypes = [ctypes.POINTER(ScanArgs), ctypes.POINTER(ScanBwdArgs), _vp, ctypes.c_size_t,
                                       _vp]
        lib.mamba_scan_config_kind.restype = ctypes.c_int
        lib.mamba_scan_config_kind.argtypes = [ctypes.c_int, ctypes.POINTER(ctypes.c_int)]
        lib.mamba_scan_plan_query.restype = ctypes.c_int
        lib.mamba_scan_plan_query.argtypes = [ctypes.POINTER(ScanArgs), ctypes.POINTER(ScanPlan)]
        lib.mamba_scan_plan_workspace_size.restype = ctypes.c_int
        lib.mamba_scan_plan_workspace_size.argtypes = [ctypes.POINTER(ScanArgs), ctypes.POINTER(ScanPlan),
                                                       ctypes.POINTER(ctypes.c_size_t)]
        lib.mamba_scan_fwd_with_plan.restype = ctypes.c_int
        lib.mamba_scan_fwd_with_plan.argtypes = [ctypes.POINTER(ScanArgs), ctypes.POINTER(ScanPlan), _vp,
                                                 ctypes.c_size_t, _vp]
        lib.mamba_ssd_fwd.restype = ctypes.c_int
        lib.mamba_ssd_fwd.argtypes = [ctypes.POINTER(SsdArgs), _vp, ctypes.c_size_t, _vp]
        lib.mamba_ssd_workspace_size.restype = ctypes.c_int
        lib.mamba_ssd_workspace_size.argtypes = [ctypes.POINTER(SsdArgs), ctypes.POINTER(ctypes.c_size_t)]
        lib.mamba_probe_unit_throughput.restype = ctypes.c_int
        lib.mamba_probe_unit_throughput.argtypes = [ctypes.c_int, _vp, ctypes.POINTER(ctypes.c_double),
                                                    ctypes.POINTER(ctypes.c_double), _vp]
        if lib.mamba_abi_version() != 2:
            raise RuntimeError("libmambascan.so ABI version mismatch")
        _lib = lib
    return _lib


def _check(status: int):
    if status != 0:
        msg = load_library().mamba_last_error().decode(errors="replace")
        raise MambaScanError(status, msg)


# ----------------------------------------------------------------------------
# torch marshalling

def _torch():
    import torch
    return torch


def _dtype_code(t) -> int:
    torch = _torch()
    if t.dtype == torch.float32:
        return MS_F32
    if t.dtype == torch.bfloat16:
        return MS_BF16
    raise TypeError(f"unsupported dtype {t.dtype} (float32 or bfloat16)")


def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream_ptr(stream):
    torch = _torch()
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _keep_until_done(t, stream):
    """A scratch tensor allocated here on the current stream but used by a
    launch on ``stream``: tell the caching allocator not to hand its memory to
    other work before that stream has finished with it."""
    if stream is not None:
        t.record_stream(stream)


def _need_cuda(name, t, dtype=None, ndim=None):
    if t is None:
        return
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dimensions")
    if t.dim() > 0 and t.stride(-1) != 1 and t.shape[-1] > 1:
        raise ValueError(f"{name} must be contiguous in its last dimension")


def build_scan_args(u, delta, A, B, C, y, *, D=None, z=None, delta_bias=None,
                    delta_softplus=True, initial_state=None, final_state=None,
                    force_segments=0) -> ScanArgs:
    """Fill an ``ms_scan_args`` from torch tensors (no checks beyond dtype/layout)."""
    torch = _torch()
    batch, dim, L = u.shape
    dstate = B.shape[1]
    f32 = torch.float32
    dt = u.dtype
    for name, t in (("u", u), ("delta", delta), ("z", z), ("y", y)):
        _need_cuda(name, t, dt, 3)
        if t is not None and tuple(t.shape) != (batch, dim, L):
            raise ValueError(f"{name} must have shape {(batch, dim, L)}, got {tuple(t.shape)}")
    for name, t in (("B", B), ("C", C)):
        _need_cuda(name, t, dt, 3)
        if tuple(t.shape) != (batch, dstate, L):
            raise ValueError(f"{name} must have shape {(batch, dstate, L)}, got {tuple(t.shape)}")
    _need_cuda("A", A, f32, 2)
    if tuple(A.shape) != (dim, dstate) or not A.is_contiguous():
        raise ValueError("A must be a contiguous (dim, dstate) float32 tensor")
    for name, t in (("D", D), ("delta_bias", delta_bias)):
        _need_cuda(name, t, f32, 1)
        if t is not None and (tuple(t.shape) != (dim,) or not t.is_contiguous()):
            raise ValueError(f"{name} must be a contiguous ({dim},) float32 tensor")
    for name, t in (("initial_state", initial_state), ("final_state", final_state)):
        _need_cuda(name, t, f32, 3)
        if t is not None and (tuple(t.shape) != (batch, dim, dstate) or not t.is_contiguous()):
            raise ValueError(f"{name} must be a contiguous {(batch, dim, dstate)} float32 tensor")
    a = ScanArgs()
    a.batch, a.dim, a.dstate, a.seqlen = batch, dim, dstate, L
    a.in_dtype = _dtype_code(u)
    a.delta_softplus = 1 if delta_softplus else 0
    a.u, a.u_batch_stride, a.u_dim_stride = _ptr(u), u.stride(0), u.stride(1)
    a.delta, a.delta_batch_stride, a.delta_dim_stride = _ptr(delta), delta.stride(0), delta.stride(1)
    a.B, a.B_batch_stride, a.B_state_stride = _ptr(B), B.stride(0), B.stride(1)
    a.C, a.C_batch_stride, a.C_state_stride = _ptr(C), C.stride(0), C.stride(1)
    if z is not None:
        a.z, a.z_batch_stride, a.z_dim_stride = _ptr(z), z.stride(0), z.stride(1)
    a.y, a.y_batch_stride, a.y_dim_stride = _ptr(y), y.stride(0), y.stride(1)
    a.A, a.D, a.delta_bias = _ptr(A), _ptr(D), _ptr(delta_bias)
    a.initial_state, a.final_state = _ptr(initial_state), _ptr(final_state)
    a.force_segments = int(force_segments)
    a.reserved = 0
    return a


def scan_workspace_size(args: ScanArgs) -> int:
    n = ctypes.c_size_t(0)
    _check(load_library().mamba_scan_workspace_size(ctypes.byref(args), ctypes.byref(n)))
    return int(n.value)


def plan_workspace_size(args: ScanArgs, plan: ScanPlan) -> int:
    """Workspace bytes that ``plan`` needs for these arguments."""
    n = ctypes.c_size_t(0)
    _check(load_library().mamba_scan_plan_workspace_size(ctypes.byref(args), ctypes.byref(plan), ctypes.byref(n)))
    return int(n.value)


def scan_status(workspace) -> int:
    """The status word a persistent-schedule scan leaves at the start of its
    workspace (0, or MS_ERR_TIMEOUT = 5). Synchronizes the device."""
    torch = _torch()
    torch.cuda.synchronize(workspace.device)
    return int(workspace[:4].view(torch.int32)[0].item())


def scan_configs():
    """[(index, lanes, states_per_pass, max_warps, kind)] of the compiled scan
    kernels; kind 0 = chunked (lanes per row pair), 1 = sequential (lanes per
    row, fixed CTA of max_warps warps, one segment)."""
    lib = load_library()
    out = []
    for i in range(lib.mamba_scan_num_configs()):
        a, b, c, k = ctypes.c_int(), ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
        _check(lib.mamba_scan_config_info(i, ctypes.byref(a), ctypes.byref(b), ctypes.byref(c)))
        _check(lib.mamba_scan_config_kind(i, ctypes.byref(k)))
        out.append((i, a.value, b.value, c.value, k.value))
    return out


def scan_plan(args: ScanArgs) -> ScanPlan:
    """The launch plan mamba_scan_fwd would use for these arguments."""
    plan = ScanPlan()
    _check(load_library().mamba_scan_plan_query(ctypes.byref(args), ctypes.byref(plan)))
    return plan


def scan_fwd(u, delta, A, B, C, D=None, z=None, delta_bias=None, delta_softplus=True,
             initial_state=None, return_last_state=True, out=None, force_segments=0,
             workspace=None, stream=None, plan=None, checkpoints=None):
    """Selective scan forward on the current (or given) CUDA stream.

    u, delta, z: (batch, dim, L); B, C: (batch, dstate, L) -- all float32 or
    all bfloat16, contiguous along L. A: (dim, dstate) float32 (normally
    -exp(A_log)); D, delta_bias: (dim,) float32. Returns y (u's dtype), and
    the final float32 state (batch, dim, dstate) when ``return_last_state``.
    ``workspace``: optional uint8 CUDA tensor reused for the multi-block carry
    (allocated here when needed and not given). ``checkpoints``: optional
    float32 CUDA tensor of at least :func:`checkpoint_numel` elements that
    receives the state after every 8th step, for :func:`scan_bwd` (automatic
    plan only).
    """
    torch = _torch()
    y = torch.empty_like(u) if out is None else out
    hT = None
    if return_last_state:
        hT = torch.empty((u.shape[0], u.shape[1], B.shape[1]), device=u.device, dtype=torch.float32)
    args = build_scan_args(u, delta, A, B, C, y, D=D, z=z, delta_bias=delta_bias,
                           delta_softplus=delta_softplus, initial_state=initial_state,
                           final_state=hT, force_segments=force_segments)
    lib = load_library()
    with torch.cuda.device(u.device):
        if plan is None:
            need = scan_workspace_size(args)
        else:
            need = plan_workspace_size(args, plan)
        ws_ptr, ws_bytes, own_ws = None, 0, False
        if need:
            if workspace is None or workspace.numel() < need:
                workspace = torch.empty(need, dtype=torch.uint8, device=u.device)
                own_ws = True
            ws_ptr, ws_bytes = workspace.data_ptr(), workspace.numel()
        if checkpoints is not None:
            if plan is not None:
                raise ValueError("checkpoints are written with the automatic plan only")
            _need_cuda("checkpoints", checkpoints, torch.float32, None)
            if not checkpoints.is_contiguous():
                raise ValueError("checkpoints must be contiguous")
            _check(lib.mamba_scan_fwd_checkpointed(ctypes.byref(args), checkpoints.data_ptr(),
                                                   checkpoints.numel() * 4, ws_ptr, ws_bytes, _stream_ptr(stream)))
        elif plan is None:
            _check(lib.mamba_scan_fwd(ctypes.byref(args), ws_ptr, ws_bytes, _stream_ptr(stream)))
        else:
            _check(lib.mamba_scan_fwd_with_plan(ctypes.byref(args), ctypes.byref(plan), ws_ptr, ws_bytes,
                                                _stream_ptr(stream)))
        if own_ws:
            _keep_until_done(workspace, stream)
    return (y, hT) if return_last_state else y


def build_update_args(state, x, delta, A, B, C, y, *, D=None, z=None, delta_bias=None,
                      delta_softplus=True) -> UpdateArgs:
    torch = _torch()
    batch, dim = x.shape
    dstate = B.shape[1]
    dt = x.dtype
    _need_cuda("state", state, torch.float32, 3)
    if tuple(state.shape) != (batch, dim, dstate):
        raise ValueError(f"state must have shape {(batch, dim, dstate)}")
    for name, t in (("x", x), ("delta", delta), ("z", z), ("y", y)):
        _need_cuda(name, t, dt, 2)
        if t is not None and tuple(t.shape) != (batch, dim):
            raise ValueError(f"{name} must have shape {(batch, dim)}")
    for name, t in (("B", B), ("C", C)):
        _need_cuda(name, t, dt, 2)
        if tuple(t.shape) != (batch, dstate):
            raise ValueError(f"{name} must have shape {(batch, dstate)}")
    _need_cuda("A", A, torch.float32, 2)
    if tuple(A.shape) != (dim, dstate) or not A.is_contiguous():
        raise ValueError("A must be a contiguous (dim, dstate) float32 tensor")
    for name, t in (("D", D), ("delta_bias", delta_bias)):
        _need_cuda(name, t, torch.float32, 1)
        if t is not None and (tuple(t.shape) != (dim,) or not t.is_contiguous()):
            raise ValueError(f"{name} must be a contiguous ({dim},) float32 tensor")
    a = UpdateArgs()
    a.batch, a.dim, a.dstate = batch, dim, dstate
    a.in_dtype = _dtype_code(x)
    a.delta_softplus = 1 if delta_softplus else 0
    a.state, a.state_batch_stride, a.state_dim_stride = _ptr(state), state.stride(0), state.stride(1)
    a.x, a.x_batch_stride = _ptr(x), x.stride(0)
    a.delta, a.delta_batch_stride = _ptr(delta), delta.stride(0)
    a.B, a.B_batch_stride = _ptr(B), B.stride(0)
    a.C, a.C_batch_stride = _ptr(C), C.stride(0)
    if z is not None:
        a.z, a.z_batch_stride = _ptr(z), z.stride(0)
    a.y, a.y_batch_stride = _ptr(y), y.stride(0)
    a.A, a.D, a.delta_bias = _ptr(A), _ptr(D), _ptr(delta_bias)
    return a


def state_update(state, x, delta, A, B, C, D=None, z=None, delta_bias=None, delta_softplus=True,
                 out=None, stream=None):
    """One decode step: updates ``state`` (batch, dim, dstate) float32 in place; returns y (batch, dim)."""
    torch = _torch()
    y = torch.empty_like(x) if out is None else out
    args = build_update_args(state, x, delta, A, B, C, y, D=D, z=z, delta_bias=delta_bias,
                             delta_softplus=delta_softplus)
    with torch.cuda.device(x.device):
        _check(load_library().mamba_state_update(ctypes.byref(args), _stream_ptr(stream)))
    return y


def build_conv_args(weight, bias=None, silu=True) -> Conv1dArgs:
    """Fill an ``ms_conv1d_args`` from a (dim, width) float32 weight and an
    optional (dim,) float32 bias."""
    torch = _torch()
    _need_cuda("conv weight", weight, torch.float32, 2)
    if not weight.is_contiguous():
        raise ValueError("conv weight must be contiguous (dim, width)")
    _need_cuda("conv bias", bias, torch.float32, 1)
    if bias is not None and (tuple(bias.shape) != (weight.shape[0],) or not bias.is_contiguous()):
        raise ValueError("conv bias must be a contiguous (dim,) float32 tensor")
    c = Conv1dArgs()
    c.weight, c.bias, c.width, c.silu = _ptr(weight), _ptr(bias), weight.shape[1], 1 if silu else 0
    return c


def conv_scan_fwd(x, conv_weight, delta, A, B, C, D=None, z=None, delta_bias=None, conv_bias=None,
                  conv_silu=True, delta_softplus=True, initial_state=None, return_last_state=True, out=None,
                  stream=None, plan=None):
    """Causal depthwise convolution + SiLU prologue fused into the selective
    scan: ``x`` (batch, dim, L) is the convolution input, ``conv_weight``
    (dim, width) and ``conv_bias`` (dim,) float32; the scan input is
    u = silu(conv(x)). Other arguments as :func:`scan_fwd` (no segments);
    ``plan`` may ask for the persistent schedule (ctas > 0), whose workspace
    is allocated here."""
    torch = _torch()
    y = torch.empty_like(x) if out is None else out
    hT = None
    if return_last_state:
        hT = torch.empty((x.shape[0], x.shape[1], B.shape[1]), device=x.device, dtype=torch.float32)
    args = build_scan_args(x, delta, A, B, C, y, D=D, z=z, delta_bias=delta_bias, delta_softplus=delta_softplus,
                           initial_state=initial_state, final_state=hT)
    conv = build_conv_args(conv_weight, conv_bias, conv_silu)
    if conv_weight.shape[0] != x.shape[1]:
        raise ValueError("conv weight must have one row per channel")
    lib = load_library()
    plan_ref = None if plan is None else ctypes.byref(plan)
    with torch.cuda.device(x.device):
        n = ctypes.c_size_t(0)
        _check(lib.mamba_conv_scan_workspace_size(ctypes.byref(args), ctypes.byref(conv), plan_ref, ctypes.byref(n)))
        workspace = torch.empty(n.value, dtype=torch.uint8, device=x.device) if n.value else None
        _check(lib.mamba_conv_scan_fwd_ws(ctypes.byref(args), ctypes.byref(conv), plan_ref,
                                          None if workspace is None else workspace.data_ptr(), n.value,
                                          _stream_ptr(stream)))
        if workspace is not None:
            _keep_until_done(workspace, stream)
    return (y, hT) if return_last_state else y


def conv_state_update(state, conv_state, x, conv_weight, delta, A, B, C, D=None, z=None, delta_bias=None,
                      conv_bias=None, conv_silu=True, delta_softplus=True, out=None, stream=None):
    """One decode step with the convolution prologue: ``conv_state`` (batch,
    dim, width) in x's dtype holds the last ``width`` inputs (oldest first) and
    is updated in place with ``x``; ``state`` as :func:`state_update`."""
    torch = _torch()
    y = torch.empty_like(x) if out is None else out
    args = build_update_args(state, x, delta, A, B, C, y, D=D, z=z, delta_bias=delta_bias,
                             delta_softplus=delta_softplus)
    conv = build_conv_args(conv_weight, conv_bias, conv_silu)
    _need_cuda("conv_state", conv_state, x.dtype, 3)
    if tuple(conv_state.shape) != (x.shape[0], x.shape[1], conv_weight.shape[1]) or conv_state.stride(2) != 1:
        raise ValueError("conv_state must be (batch, dim, width) with a contiguous width axis")
    with torch.cuda.device(x.device):
        _check(load_library().mamba_conv_state_update(ctypes.byref(args), ctypes.byref(conv), _ptr(conv_state),
                                                      conv_state.stride(0), conv_state.stride(1),
                                                      _stream_ptr(stream)))
    return y


def trap_scan_fwd(u, delta, lambda_raw, A, B, C, D=None, z=None, delta_bias=None, delta_softplus=True,
                  initial_state=None, return_last_state=True, out=None, stream=None, plan=None):
    """Exponential-trapezoidal selective scan (Mamba-3): as :func:`scan_fwd`
    plus ``lambda_raw`` (batch, dim, L) in u's dtype, lambda = sigmoid(lambda_raw)
    mixing the previous and the current input (no segments); ``plan`` may ask
    for the persistent schedule (ctas > 0), whose workspace is allocated here."""
    torch = _torch()
    _need_cuda("lambda_raw", lambda_raw, u.dtype, 3)
    if tuple(lambda_raw.shape) != tuple(u.shape):
        raise ValueError("lambda_raw must have u's shape")
    y = torch.empty_like(u) if out is None else out
    hT = None
    if return_last_state:
        hT = torch.empty((u.shape[0], u.shape[1], B.shape[1]), device=u.device, dtype=torch.float32)
    args = build_scan_args(u, delta, A, B, C, y, D=D, z=z, delta_bias=delta_bias, delta_softplus=delta_softplus,
                           initial_state=initial_state, final_state=hT)
    lib = load_library()
    plan_ref = None if plan is None else ctypes.byref(plan)
    lam = (_ptr(lambda_raw), lambda_raw.stride(0), lambda_raw.stride(1))
    with torch.cuda.device(u.device):
        n = ctypes.c_size_t(0)
        _check(lib.mamba_trap_scan_workspace_size(ctypes.byref(args), *lam, plan_ref, ctypes.byref(n)))
        workspace = torch.empty(n.value, dtype=torch.uint8, device=u.device) if n.value else None
        _check(lib.mamba_trap_scan_fwd_ws(ctypes.byref(args), *lam, plan_ref,
                                          None if workspace is None else workspace.data_ptr(), n.value,
                                          _stream_ptr(stream)))
        if workspace is not None:
            _keep_until_done(workspace, stream)
    return (y, hT) if return_last_state else y


def checkpoint_numel(u, B):
    """float32 elements of the checkpoint buffer of :func:`scan_fwd` /
    :func:`scan_bwd` for u (batch, dim, L) and B (batch, dstate, L)."""
    batch, dim, L = u.shape
    return batch * dim * ((L + 7) // 8) * 16


def scan_bwd(u, delta, A, B, C, dy, D=None, z=None, delta_bias=None, delta_softplus=True, initial_state=None,
             dfinal_state=None, workspace=None, stream=None, checkpoints=None):
    """Gradients of :func:`scan_fwd` for the loss sum(y * dy) + sum(h_T * dfinal_state).

    Forward inputs as :func:`scan_fwd`; ``dy`` (batch, dim, L) in u's dtype;
    ``dfinal_state`` (batch, dim, dstate) float32 or None. Returns a dict:
    du, ddelta (w.r.t. the raw delta), dz (None without z) in u's dtype; dA
    (dim, dstate), dB, dC (batch, dstate, L), dD, ddelta_bias (dim,) (None
    when the input is None) and dinitial_state (batch, dim, dstate), float32.
    ``checkpoints``: the tensor a :func:`scan_fwd` call on the same inputs
    filled; the backward then recomputes from it instead of sweeping the
    sequence forward first.
    """
    torch = _torch()
    batch, dim, L = u.shape
    N = B.shape[1]
    # the forward's arguments; its output pointer is not used by the backward (u stands in for it)
    args = build_scan_args(u, delta, A, B, C, u, D=D, z=z, delta_bias=delta_bias, delta_softplus=delta_softplus,
                           initial_state=initial_state)
    _need_cuda("dy", dy, u.dtype, 3)
    if tuple(dy.shape) != tuple(u.shape):
        raise ValueError("dy must have u's shape")
    if dfinal_state is not None:
        _need_cuda("dfinal_state", dfinal_state, torch.float32, 3)
        if tuple(dfinal_state.shape) != (batch, dim, N) or not dfinal_state.is_contiguous():
            raise ValueError("dfinal_state must be a contiguous (batch, dim, dstate) float32 tensor")
    f32 = dict(device=u.device, dtype=torch.float32)
    out = {"du": torch.empty_like(u), "ddelta": torch.empty_like(u), "dz": torch.empty_like(u) if z is not None else None,
           "dA": torch.empty((dim, N), **f32), "dB": torch.empty((batch, N, L), **f32),
           "dC": torch.empty((batch, N, L), **f32), "dD": torch.empty(dim, **f32) if D is not None else None,
           "ddelta_bias": torch.empty(dim, **f32) if delta_bias is not None else None,
           "dinitial_state": torch.empty((batch, dim, N), **f32)}
    g = ScanBwdArgs()
    g.dy, g.dy_batch_stride, g.dy_dim_stride = _ptr(dy), dy.stride(0), dy.stride(1)
    g.dfinal_state = _ptr(dfinal_state)
    for k in ("du", "ddelta", "dz"):
        t = out[k]
        if t is not None:
            setattr(g, k, _ptr(t))
            setattr(g, f"{k}_batch_stride", t.stride(0))
            setattr(g, f"{k}_dim_stride", t.stride(1))
    for k in ("dA", "dB", "dC", "dD", "ddelta_bias", "dinitial_state"):
        setattr(g, k, _ptr(out[k]))
    lib = load_library()
    with torch.cuda.device(u.device):
        if checkpoints is not None:
            _need_cuda("checkpoints", checkpoints, torch.float32, None)
            if not checkpoints.is_contiguous():
                raise ValueError("checkpoints must be contiguous")
            _check(lib.mamba_scan_bwd_checkpointed(ctypes.byref(args), ctypes.byref(g), checkpoints.data_ptr(),
                                                   checkpoints.numel() * 4, _stream_ptr(stream)))
            return out
        n = ctypes.c_size_t(0)
        _check(lib.mamba_scan_bwd_workspace_size(ctypes.byref(args), ctypes.byref(n)))
        own_ws = workspace is None or workspace.numel() < n.value
        if own_ws:
            workspace = torch.empty(max(n.value, 1), dtype=torch.uint8, device=u.device)
        _check(lib.mamba_scan_bwd(ctypes.byref(args), ctypes.byref(g), workspace.data_ptr(), workspace.numel(),
                                  _stream_ptr(stream)))
        if own_ws:
            _keep_until_done(workspace, stream)
    return out


def build_ssd_args(x, dt, A, B, C, y, *, D=None, z=None, dt_bias=None, dt_softplus=True, initial_state=None,
                   final_state=None) -> SsdArgs:
    """Fill an ``ms_ssd_args`` from torch tensors: x, z, y (batch, L, nheads,
    64), dt (batch, L, nheads), B, C (batch, L, ngroups, 128), all bf16 with
    the inner axes contiguous; A, D, dt_bias (nheads,) float32; states
    (batch, nheads, 64, 128) float32 contiguous."""
    torch = _torch()
    for name, t in (("x", x), ("y", y), ("z", z)):
        _need_cuda(name, t, None, 4)
        if t is not None and (t.shape[3] != SSD_HEADDIM or (t.shape[2] > 1 and t.stride(2) != SSD_HEADDIM)):
            raise ValueError(f"{name} must be (batch, L, nheads, 64) with the last two axes contiguous")
    batch, L, nheads, _ = x.shape
    for name, t in (("y", y), ("z", z)):
        if t is not None and tuple(t.shape) != tuple(x.shape):
            raise ValueError(f"{name} must have x's shape")
    _need_cuda("dt", dt, None, 3)
    if tuple(dt.shape) != (batch, L, nheads):
        raise ValueError("dt must be (batch, L, nheads)")
    for name, t in (("B", B), ("C", C)):
        _need_cuda(name, t, None, 4)
        if (t.shape[0] != batch or t.shape[1] != L or t.shape[3] != SSD_DSTATE
                or (t.shape[2] > 1 and t.stride(2) != SSD_DSTATE)):
            raise ValueError(f"{name} must be (batch, L, ngroups, 128) with the last two axes contiguous")
    if tuple(C.shape) != tuple(B.shape):
        raise ValueError("B and C must have one shape")
    for name, t in (("A", A), ("D", D), ("dt_bias", dt_bias)):
        _need_cuda(name, t, torch.float32, 1)
        if t is not None and (tuple(t.shape) != (nheads,) or not t.is_contiguous()):
            raise ValueError(f"{name} must be a contiguous ({nheads},) float32 tensor")
    for name, t in (("initial_state", initial_state), ("final_state", final_state)):
        _need_cuda(name, t, torch.float32, 4)
        if t is not None and (tuple(t.shape) != (batch, nheads, SSD_HEADDIM, SSD_DSTATE) or not t.is_contiguous()):
            raise ValueError(f"{name} must be a contiguous (batch, nheads, 64, 128) float32 tensor")
    a = SsdArgs()
    a.batch, a.seqlen, a.nheads, a.ngroups = batch, L, nheads, B.shape[2]
    a.in_dtype = _dtype_code(x)
    a.dt_softplus = 1 if dt_softplus else 0
    for name, t in (("x", x), ("dt", dt), ("B", B), ("C", C), ("z", z), ("y", y)):
        if t is not None:
            setattr(a, name, _ptr(t))
            setattr(a, f"{name}_batch_stride", t.stride(0))
            setattr(a, f"{name}_token_stride", t.stride(1))
    a.A, a.D, a.dt_bias = _ptr(A), _ptr(D), _ptr(dt_bias)
    a.initial_state, a.final_state = _ptr(initial_state), _ptr(final_state)
    return a


def ssd_check(workspace, stream=None):
    """Synchronize ``stream`` and raise :class:`MambaScanError` if the SSD
    kernel that used ``workspace`` reported a failed internal wait."""
    torch = _torch()
    (stream or torch.cuda.current_stream(workspace.device)).synchronize()
    code = int(workspace[:4].view(torch.int32)[0].item())
    if code != 0:
        raise MambaScanError(code, "the SSD kernel reported a failure in its status word")


def ssd_fwd(x, dt, A, B, C, D=None, z=None, dt_bias=None, dt_softplus=True, initial_state=None,
            return_final_state=True, out=None, workspace=None, check=True, stream=None, wait_limit_us=0,
            withhold_block=0):
    """Mamba-2 scalar-decay SSM forward (chunked SSD on the tensor cores).

    Shapes as :func:`build_ssd_args`. Returns ``(y, final_state)``
    (final_state None when not asked for). ``workspace``: a uint8 CUDA tensor
    of at least ``SSD_WORKSPACE_BYTES`` bytes holding the status word; when
    None, one of ``mamba_ssd_workspace_size`` bytes is allocated, which lets
    the call take the persistent schedule. With ``check`` the call synchronizes the stream and
    raises if the kernel reported a failed wait; without it, call
    :func:`ssd_check` on the workspace later. ``wait_limit_us`` bounds each
    of the kernel's pipeline waits (0: about one second); ``withhold_block``
    is the fault-injection hook of ``ms_ssd_args`` (tests only).
    """
    torch = _torch()
    y = torch.empty_like(x) if out is None else out
    hT = None
    if return_final_state:
        hT = torch.empty((x.shape[0], x.shape[2], SSD_HEADDIM, SSD_DSTATE), device=x.device, dtype=torch.float32)
    args = build_ssd_args(x, dt, A, B, C, y, D=D, z=z, dt_bias=dt_bias, dt_softplus=dt_softplus,
                          initial_state=initial_state, final_state=hT)
    args.wait_limit_us = int(wait_limit_us)
    args.withhold_block = int(withhold_block)
    own_ws = workspace is None
    lib = load_library()
    with torch.cuda.device(x.device):
        if own_ws:
            n = ctypes.c_size_t(0)
            _check(lib.mamba_ssd_workspace_size(ctypes.byref(args), ctypes.byref(n)))
            workspace = torch.empty(n.value, dtype=torch.uint8, device=x.device)
        _check(lib.mamba_ssd_fwd(ctypes.byref(args), workspace.data_ptr(), workspace.numel(), _stream_ptr(stream)))
        if own_ws:
            _keep_until_done(workspace, stream)
    if check:
        ssd_check(workspace, stream)
    return y, hT


PROBE_UNITS = {"ex2": 0, "tanh": 1, "ffma": 2, "ffma2": 3}


def probe_unit_throughput(unit: str, device=None, stream=None):
    """Measured throughput of one arithmetic unit on ``device`` (see
    ``mamba_probe_unit_throughput``): returns (results per second, results per
    clock per SM). ``unit``: "ex2", "tanh", "ffma" or "ffma2". Synchronous."""
    torch = _torch()
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    with torch.cuda.device(dev):
        scratch = torch.empty(256, dtype=torch.uint8, device=dev)
        per_s, per_clk = ctypes.c_double(0.0), ctypes.c_double(0.0)
        _check(load_library().mamba_probe_unit_throughput(PROBE_UNITS[unit], scratch.data_ptr(),
                                                          ctypes.byref(per_s), ctypes.byref(per_clk),
                                                          _stream_ptr(stream)))
    return per_s.value, per_clk.value
