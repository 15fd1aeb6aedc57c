"""fp64 CPU oracle for the selective scan (S6) and its decode state update.

TEST INFRASTRUCTURE ONLY: imported by the tests, by the smoke check and by the
benchmark's CPU-baseline leg. The product (the CUDA library and its binding)
never imports it. The arithmetic lives in ``s6_oracle.c`` (the selective scan,
its decode step, convolution prologue, trapezoidal variant and gradients) and
``ssd_oracle.c`` (the Mamba-2 scalar-decay SSM in recurrent form): plain C,
double precision, OpenMP across independent rows. This module compiles them
with gcc on first use and marshals numpy arrays into them.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRCS = [os.path.join(_HERE, "s6_oracle.c"), os.path.join(_HERE, "ssd_oracle.c")]
_LIB = os.path.join(_HERE, "_build", "libs6oracle.so")
_lock = threading.Lock()
_lib = None

F32, BF16 = 0, 1
_DTYPES = {"f32": F32, "bf16": BF16}


def build(force: bool = False) -> str:
    """Compile the oracle (gcc -O2, no fast-math, OpenMP) and return the .so path."""
    with _lock:
        if (not force and os.path.exists(_LIB)
                and os.path.getmtime(_LIB) >= max(os.path.getmtime(s) for s in _SRCS)):
            return _LIB
        os.makedirs(os.path.dirname(_LIB), exist_ok=True)
        tmp = _LIB + f".{os.getpid()}.tmp"
        subprocess.check_call(["gcc", "-O2", "-fno-fast-math", "-fopenmp", "-fPIC", "-shared",
                               "-std=c11", "-Wall", "-Werror", *_SRCS, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
        return _LIB


def _bind(path: str):
    lib = ctypes.CDLL(path)
    i64, ip, vp = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p
    lib.s6_oracle_scan.restype = ip
    lib.s6_oracle_scan.argtypes = [i64, i64, i64, i64, ip, vp, vp, vp, vp, vp, vp, vp, vp,
                                   ip, vp, i64, vp, vp, vp, ip]
    lib.s6_oracle_state_update.restype = ip
    lib.s6_oracle_state_update.argtypes = [i64, i64, i64, ip, vp, vp, vp, vp, vp, vp, vp, vp,
                                           vp, ip, vp, i64, vp, ip]
    lib.s6_oracle_conv_scan.restype = ip
    lib.s6_oracle_conv_scan.argtypes = [i64, i64, i64, i64, ip, vp, vp, vp, ip, ip, vp, vp, vp, vp,
                                        vp, vp, vp, ip, vp, i64, vp, vp, vp, vp, ip]
    lib.s6_oracle_conv_state_update.restype = ip
    lib.s6_oracle_conv_state_update.argtypes = [i64, i64, i64, ip, vp, vp, vp, vp, vp, ip, ip, vp, vp,
                                                vp, vp, vp, vp, vp, ip, vp, i64, vp, ip]
    lib.s6_oracle_trap_scan.restype = ip
    lib.s6_oracle_trap_scan.argtypes = [i64, i64, i64, i64, ip, vp, vp, vp, vp, vp, vp, vp, vp, vp, ip, vp,
                                        i64, vp, vp, vp, ip]
    lib.s6_oracle_scan_d.restype = ip
    lib.s6_oracle_scan_d.argtypes = [i64, i64, i64, i64] + [vp] * 8 + [ip, vp, vp, vp]
    lib.s6_oracle_scan_bwd.restype = ip
    lib.s6_oracle_scan_bwd.argtypes = [i64, i64, i64, i64] + [vp] * 8 + [ip] + [vp] * 12
    lib.ssd_oracle_rec_d.restype = ip
    lib.ssd_oracle_rec_d.argtypes = [i64, i64, i64] + [vp] * 6
    lib.ssd_oracle_scan.restype = ip
    lib.ssd_oracle_scan.argtypes = [i64] * 6 + [ip] + [vp] * 8 + [ip, vp, i64, vp, vp, vp, ip]
    lib.s6_oracle_max_threads.restype = ip
    lib.s6_oracle_max_threads.argtypes = []
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = _bind(build())
    return _lib


def max_threads() -> int:
    return int(_load().s6_oracle_max_threads())


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _in(a, dtype: int):
    if a is None:
        return None
    want = np.float32 if dtype == F32 else np.uint16
    a = np.ascontiguousarray(a)
    if a.dtype != want:
        raise TypeError(f"oracle input has dtype {a.dtype}, expected {np.dtype(want)}")
    return a


def _f32(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.float32)


def scan(*, u, delta, A, B, C, D=None, z=None, delta_bias=None, delta_softplus=True,
         dtype="f32", rows=None, h0=None, threads: int = 0, _lib_override=None):
    """Selective scan forward in fp64.

    ``u, delta, z``: (batch, dim, L); ``B, C``: (batch, dstate, L), float32
    arrays or uint16 bf16 bits according to ``dtype``. ``A`` (dim, dstate),
    ``D`` and ``delta_bias`` (dim,) float32. ``rows``: optional list of row
    indices ``b*dim + d`` to compute (default: all rows in order). ``h0``:
    optional initial state (n_rows, dstate).

    Returns ``(y, h)``: y (batch, dim, L) float64 (or (n_rows, L) with
    ``rows``) and the final state (batch, dim, dstate) (or (n_rows, dstate)).
    """
    dt = _DTYPES[dtype]
    u, delta, B, C, z = (_in(a, dt) for a in (u, delta, B, C, z))
    A, D, delta_bias = _f32(A), _f32(D), _f32(delta_bias)
    batch, dim, L = u.shape
    dstate = B.shape[1]
    if delta.shape != u.shape or (z is not None and z.shape != u.shape):
        raise ValueError("u, delta and z must share one (batch, dim, L) shape")
    if B.shape != (batch, dstate, L) or C.shape != B.shape or A.shape != (dim, dstate):
        raise ValueError("B, C must be (batch, dstate, L) and A (dim, dstate)")
    if rows is None:
        n_rows, rows_arr = batch * dim, None
    else:
        rows_arr = np.ascontiguousarray(rows, dtype=np.int64)
        n_rows = rows_arr.size
    h0_arr = None if h0 is None else np.ascontiguousarray(h0, dtype=np.float64).reshape(n_rows, dstate)
    y = np.empty((n_rows, L), np.float64)
    h = np.empty((n_rows, dstate), np.float64)
    lib = _lib_override or _load()
    rc = lib.s6_oracle_scan(batch, dim, dstate, L, dt, _ptr(u), _ptr(delta), _ptr(A), _ptr(B),
                                _ptr(C), _ptr(D), _ptr(z), _ptr(delta_bias), int(bool(delta_softplus)),
                                _ptr(rows_arr), n_rows, _ptr(h0_arr), _ptr(y), _ptr(h), int(threads))
    if rc != 0:
        raise ValueError("oracle rejected its arguments")
    if rows is None:
        return y.reshape(batch, dim, L), h.reshape(batch, dim, dstate)
    return y, h


def state_update(*, state, x, delta, A, B, C, D=None, z=None, delta_bias=None,
                 delta_softplus=True, dtype="f32", rows=None, threads: int = 0,
                 _lib_override=None):
    """One decode step in fp64.

    ``state``: float64 (batch, dim, dstate) (or (n_rows, dstate) with
    ``rows``), updated in place. ``x, delta, z``: (batch, dim); ``B, C``:
    (batch, dstate). Returns y (batch, dim) float64 (or (n_rows,)).
    """
    dt = _DTYPES[dtype]
    x, delta, B, C, z = (_in(a, dt) for a in (x, delta, B, C, z))
    A, D, delta_bias = _f32(A), _f32(D), _f32(delta_bias)
    batch, dim = x.shape
    dstate = B.shape[1]
    if not (isinstance(state, np.ndarray) and state.dtype == np.float64 and state.flags.c_contiguous):
        raise TypeError("state must be a C-contiguous float64 array (updated in place)")
    if rows is None:
        n_rows, rows_arr = batch * dim, None
    else:
        rows_arr = np.ascontiguousarray(rows, dtype=np.int64)
        n_rows = rows_arr.size
    if state.size != n_rows * dstate:
        raise ValueError("state has the wrong size")
    y = np.empty(n_rows, np.float64)
    lib = _lib_override or _load()
    rc = lib.s6_oracle_state_update(batch, dim, dstate, dt, _ptr(state), _ptr(x), _ptr(delta),
                                        _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z),
                                        _ptr(delta_bias), int(bool(delta_softplus)),
                                        _ptr(rows_arr), n_rows, _ptr(y), int(threads))
    if rc != 0:
        raise ValueError("oracle rejected its arguments")
    return y.reshape(batch, dim) if rows is None else y


def conv_scan(*, x, conv_w, conv_b=None, conv_silu=True, delta, A, B, C, D=None, z=None,
              delta_bias=None, delta_softplus=True, dtype="f32", rows=None, h0=None,
              return_u=False, threads: int = 0, _lib_override=None):
    """Causal depthwise convolution prologue + selective scan, in fp64.

    ``x`` (batch, dim, L) is the convolution input (float32 or bf16 bits);
    ``conv_w`` (dim, width) and ``conv_b`` (dim,) float32. The scan input is
    u = silu(conv(x)) (or conv(x) with ``conv_silu=False``). Other arguments as
    :func:`scan`. Returns ``(y, h)``, or ``(y, h, u)`` with ``return_u``.
    """
    dt = _DTYPES[dtype]
    x, delta, B, C, z = (_in(a, dt) for a in (x, delta, B, C, z))
    A, D, delta_bias, conv_w, conv_b = _f32(A), _f32(D), _f32(delta_bias), _f32(conv_w), _f32(conv_b)
    batch, dim, L = x.shape
    dstate = B.shape[1]
    width = conv_w.shape[1]
    if conv_w.shape != (dim, width) or (conv_b is not None and conv_b.shape != (dim,)):
        raise ValueError("conv_w must be (dim, width) and conv_b (dim,)")
    if delta.shape != x.shape or (z is not None and z.shape != x.shape):
        raise ValueError("x, delta and z must share one (batch, dim, L) shape")
    if B.shape != (batch, dstate, L) or C.shape != B.shape or A.shape != (dim, dstate):
        raise ValueError("B, C must be (batch, dstate, L) and A (dim, dstate)")
    if rows is None:
        n_rows, rows_arr = batch * dim, None
    else:
        rows_arr = np.ascontiguousarray(rows, dtype=np.int64)
        n_rows = rows_arr.size
    h0_arr = None if h0 is None else np.ascontiguousarray(h0, dtype=np.float64).reshape(n_rows, dstate)
    y = np.empty((n_rows, L), np.float64)
    h = np.empty((n_rows, dstate), np.float64)
    u = np.empty((n_rows, L), np.float64) if return_u else None
    lib = _lib_override or _load()
    rc = lib.s6_oracle_conv_scan(batch, dim, dstate, L, dt, _ptr(x), _ptr(conv_w), _ptr(conv_b), width,
                                 int(bool(conv_silu)), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D),
                                 _ptr(z), _ptr(delta_bias), int(bool(delta_softplus)), _ptr(rows_arr),
                                 n_rows, _ptr(h0_arr), _ptr(y), _ptr(h), _ptr(u), int(threads))
    if rc != 0:
        raise ValueError("oracle rejected its arguments")
    if rows is None:
        out = (y.reshape(batch, dim, L), h.reshape(batch, dim, dstate))
        return out + (u.reshape(batch, dim, L),) if return_u else out
    return (y, h, u) if return_u else (y, h)


def conv_state_update(*, state, conv_state, x, conv_w, conv_b=None, conv_silu=True, delta, A, B, C,
                      D=None, z=None, delta_bias=None, delta_softplus=True, dtype="f32", rows=None,
                      threads: int = 0, _lib_override=None):
    """One decode step with the convolution prologue, in fp64.

    ``conv_state``: float64 (batch, dim, width) (or (n_rows, width)), the last
    ``width`` convolution inputs oldest first, updated in place; ``state`` as
    :func:`state_update`. Returns y (batch, dim) float64 (or (n_rows,)).
    """
    dt = _DTYPES[dtype]
    x, delta, B, C, z = (_in(a, dt) for a in (x, delta, B, C, z))
    A, D, delta_bias, conv_w, conv_b = _f32(A), _f32(D), _f32(delta_bias), _f32(conv_w), _f32(conv_b)
    batch, dim = x.shape
    dstate = B.shape[1]
    width = conv_w.shape[1]
    for a in (state, conv_state):
        if not (isinstance(a, np.ndarray) and a.dtype == np.float64 and a.flags.c_contiguous):
            raise TypeError("state and conv_state must be C-contiguous float64 arrays (updated in place)")
    if rows is None:
        n_rows, rows_arr = batch * dim, None
    else:
        rows_arr = np.ascontiguousarray(rows, dtype=np.int64)
        n_rows = rows_arr.size
    if state.size != n_rows * dstate or conv_state.size != n_rows * width:
        raise ValueError("state or conv_state has the wrong size")
    y = np.empty(n_rows, np.float64)
    lib = _lib_override or _load()
    rc = lib.s6_oracle_conv_state_update(batch, dim, dstate, dt, _ptr(state), _ptr(conv_state), _ptr(x),
                                         _ptr(conv_w), _ptr(conv_b), width, int(bool(conv_silu)),
                                         _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z),
                                         _ptr(delta_bias), int(bool(delta_softplus)), _ptr(rows_arr),
                                         n_rows, _ptr(y), int(threads))
    if rc != 0:
        raise ValueError("oracle rejected its arguments")
    return y.reshape(batch, dim) if rows is None else y


def trap_scan(*, u, delta, lambda_raw, A, B, C, D=None, z=None, delta_bias=None, delta_softplus=True,
              dtype="f32", rows=None, h0=None, threads: int = 0, _lib_override=None):
    """Exponential-trapezoidal selective scan (Mamba-3) in fp64: as :func:`scan`
    plus ``lambda_raw`` (batch, dim, L), the pre-activation of the gate
    lambda = sigmoid(lambda_raw). Returns ``(y, h)``."""
    dt = _DTYPES[dtype]
    u, delta, lambda_raw, B, C, z = (_in(a, dt) for a in (u, delta, lambda_raw, B, C, z))
    A, D, delta_bias = _f32(A), _f32(D), _f32(delta_bias)
    batch, dim, L = u.shape
    dstate = B.shape[1]
    if delta.shape != u.shape or lambda_raw.shape != u.shape or (z is not None and z.shape != u.shape):
        raise ValueError("u, delta, lambda_raw and z must share one (batch, dim, L) shape")
    if B.shape != (batch, dstate, L) or C.shape != B.shape or A.shape != (dim, dstate):
        raise ValueError("B, C must be (batch, dstate, L) and A (dim, dstate)")
    if rows is None:
        n_rows, rows_arr = batch * dim, None
    else:
        rows_arr = np.ascontiguousarray(rows, dtype=np.int64)
        n_rows = rows_arr.size
    h0_arr = None if h0 is None else np.ascontiguousarray(h0, dtype=np.float64).reshape(n_rows, dstate)
    y = np.empty((n_rows, L), np.float64)
    h = np.empty((n_rows, dstate), np.float64)
    lib = _lib_override or _load()
    rc = lib.s6_oracle_trap_scan(batch, dim, dstate, L, dt, _ptr(u), _ptr(delta), _ptr(lambda_raw), _ptr(A),
                                 _ptr(B), _ptr(C), _ptr(D), _ptr(z), _ptr(delta_bias), int(bool(delta_softplus)),
                                 _ptr(rows_arr), n_rows, _ptr(h0_arr), _ptr(y), _ptr(h), int(threads))
    if rc != 0:
        raise ValueError("oracle rejected its arguments")
    if rows is None:
        return y.reshape(batch, dim, L), h.reshape(batch, dim, dstate)
    return y, h


def as_f64(a, dtype=None):
    """Values of an oracle input as float64: float32 arrays, bf16 bit patterns
    (uint16, widened exactly) or float64 arrays."""
    if a is None:
        return None
    a = np.asarray(a)
    if a.dtype == np.uint16:
        return np.ascontiguousarray((a.astype(np.uint32) << 16).view(np.float32).astype(np.float64))
    return np.ascontiguousarray(a, dtype=np.float64)


def scan_d(*, u, delta, A, B, C, D=None, z=None, delta_bias=None, delta_softplus=True, h0=None,
           _lib_override=None):
    """The forward scan with every input in float64 (the backward's reference
    forward; used by the finite-difference pins). Returns ``(y, h)``."""
    u, delta, A, B, C, D, z, delta_bias, h0 = (as_f64(a) for a in (u, delta, A, B, C, D, z, delta_bias, h0))
    batch, dim, L = u.shape
    N = B.shape[1]
    y = np.empty((batch, dim, L))
    h = np.empty((batch, dim, N))
    lib = _lib_override or _load()
    rc = lib.s6_oracle_scan_d(batch, dim, N, L, _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z),
                              _ptr(delta_bias), int(bool(delta_softplus)), _ptr(h0), _ptr(y), _ptr(h))
    if rc != 0:
        raise ValueError("oracle rejected its arguments")
    return y, h


def scan_bwd(*, u, delta, A, B, C, dy, D=None, z=None, delta_bias=None, delta_softplus=True, h0=None, dhT=None,
             _lib_override=None):
    """Gradients of the scan in float64 for the loss sum(y * dy) + sum(hT * dhT).

    Inputs as :func:`scan` (float32, bf16 bits or float64 arrays), ``dy``
    (batch, dim, L), ``dhT`` (batch, dim, N). Returns a dict with du, ddelta
    (w.r.t. delta_raw), dz, dA, dB, dC, dD, ddelta_bias, dh0 (float64; dz is
    None without z)."""
    u, delta, A, B, C, D, z, delta_bias, h0, dy, dhT = (
        as_f64(a) for a in (u, delta, A, B, C, D, z, delta_bias, h0, dy, dhT))
    batch, dim, L = u.shape
    N = B.shape[1]
    out = {"du": np.empty((batch, dim, L)), "ddelta": np.empty((batch, dim, L)),
           "dz": np.empty((batch, dim, L)) if z is not None else None, "dA": np.empty((dim, N)),
           "dB": np.empty((batch, N, L)), "dC": np.empty((batch, N, L)), "dD": np.empty(dim),
           "ddelta_bias": np.empty(dim), "dh0": np.empty((batch, dim, N))}
    lib = _lib_override or _load()
    rc = lib.s6_oracle_scan_bwd(batch, dim, N, L, _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D),
                                _ptr(z), _ptr(delta_bias), int(bool(delta_softplus)), _ptr(h0), _ptr(dy), _ptr(dhT),
                                _ptr(out["du"]), _ptr(out["ddelta"]), _ptr(out["dz"]), _ptr(out["dA"]),
                                _ptr(out["dB"]), _ptr(out["dC"]), _ptr(out["dD"]), _ptr(out["ddelta_bias"]),
                                _ptr(out["dh0"]))
    if rc != 0:
        raise ValueError("oracle rejected its arguments")
    return out


def ssd_rec(*, a, B, C, X, H0=None, _lib_override=None):
    """Recurrent form of one head in the page's parametrisation, in fp64:
    H = a[t] H + X[t] B[t]^T, Y[t] = H C[t]. ``a`` (L,), ``B, C`` (L, N), ``X``
    (L, P); ``H0`` optional (P, N). Returns ``(Y (L, P), H (P, N))``."""
    a, B, C, X = (np.ascontiguousarray(v, dtype=np.float64) for v in (a, B, C, X))
    L, P = X.shape
    N = B.shape[1]
    if a.shape != (L,) or B.shape != (L, N) or C.shape != (L, N):
        raise ValueError("a must be (L,), B and C (L, N), X (L, P)")
    H = np.zeros((P, N)) if H0 is None else np.array(H0, dtype=np.float64, order="C").reshape(P, N)
    Y = np.empty((L, P))
    lib = _lib_override or _load()
    if lib.ssd_oracle_rec_d(L, P, N, _ptr(a), _ptr(B), _ptr(C), _ptr(X), _ptr(H), _ptr(Y)) != 0:
        raise ValueError("oracle rejected its arguments")
    return Y, H


def ssd_scan(*, x, dt, A, B, C, D=None, z=None, dt_bias=None, dt_softplus=True, dtype="f32",
             pairs=None, h0=None, threads: int = 0, _lib_override=None):
    """Mamba-2 scalar-decay SSM forward in fp64 (recurrent form).

    ``x, z``: (batch, L, nheads, headdim); ``dt``: (batch, L, nheads); ``B, C``:
    (batch, L, ngroups, dstate) -- float32 arrays or uint16 bf16 bits according
    to ``dtype``. ``A`` (nheads,), ``D`` and ``dt_bias`` (nheads,) float32.
    ``pairs``: optional list of ``b*nheads + h`` to compute (default: all, in
    order). ``h0``: optional initial state (n_pairs, headdim, dstate).

    Returns ``(y, h)``: y (batch, L, nheads, headdim) float64 and the final
    state (batch, nheads, headdim, dstate); with ``pairs``, y is
    (n_pairs, L, headdim) and h (n_pairs, headdim, dstate).
    """
    dtc = _DTYPES[dtype]
    x, dt, B, C, z = (_in(v, dtc) for v in (x, dt, B, C, z))
    A, D, dt_bias = _f32(A), _f32(D), _f32(dt_bias)
    batch, L, nheads, P = x.shape
    G, N = B.shape[2], B.shape[3]
    if dt.shape != (batch, L, nheads) or (z is not None and z.shape != x.shape):
        raise ValueError("dt must be (batch, L, nheads) and z like x")
    if B.shape != (batch, L, G, N) or C.shape != B.shape or A.shape != (nheads,):
        raise ValueError("B, C must be (batch, L, ngroups, dstate) and A (nheads,)")
    if pairs is None:
        n_pairs, pairs_arr = batch * nheads, None
    else:
        pairs_arr = np.ascontiguousarray(pairs, dtype=np.int64)
        n_pairs = pairs_arr.size
    h0_arr = None if h0 is None else np.ascontiguousarray(h0, dtype=np.float64).reshape(n_pairs, P, N)
    y = np.empty((n_pairs, L, P))
    h = np.empty((n_pairs, P, N))
    lib = _lib_override or _load()
    rc = lib.ssd_oracle_scan(batch, L, nheads, P, G, N, dtc, _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C),
                             _ptr(D), _ptr(z), _ptr(dt_bias), int(bool(dt_softplus)), _ptr(pairs_arr), n_pairs,
                             _ptr(h0_arr), _ptr(y), _ptr(h), int(threads))
    if rc != 0:
        raise ValueError("oracle rejected its arguments")
    if pairs is None:
        return (y.reshape(batch, nheads, L, P).transpose(0, 2, 1, 3).copy(),
                h.reshape(batch, nheads, P, N))
    return y, h


class Variant:
    """The oracle's entry points bound to another build of the oracle source.

    Used only by the tests that plant a mistake in a copy of the oracle source
    and check that the pins catch it.
    """

    def __init__(self, so_path: str):
        self._lib = _bind(so_path)

    def scan(self, **kw):
        return scan(_lib_override=self._lib, **kw)

    def state_update(self, **kw):
        return state_update(_lib_override=self._lib, **kw)

    def conv_scan(self, **kw):
        return conv_scan(_lib_override=self._lib, **kw)

    def conv_state_update(self, **kw):
        return conv_state_update(_lib_override=self._lib, **kw)

    def trap_scan(self, **kw):
        return trap_scan(_lib_override=self._lib, **kw)

    def scan_d(self, **kw):
        return scan_d(_lib_override=self._lib, **kw)

    def scan_bwd(self, **kw):
        return scan_bwd(_lib_override=self._lib, **kw)

    def ssd_rec(self, **kw):
        return ssd_rec(_lib_override=self._lib, **kw)

    def ssd_scan(self, **kw):
        return ssd_scan(_lib_override=self._lib, **kw)


def compile_source(src_paths, so_path: str) -> str:
    """Compile oracle source files (same flags as :func:`build`) into one library."""
    if isinstance(src_paths, str):
        src_paths = [src_paths]
    subprocess.check_call(["gcc", "-O2", "-fno-fast-math", "-fopenmp", "-fPIC", "-shared",
                           "-std=c11", *src_paths, "-o", so_path, "-lm"])
    return so_path


SOURCES = tuple(_SRCS)
