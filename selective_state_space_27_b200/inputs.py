"""Seeded synthetic inputs for the selective scan (S6) and its decode step.

This module is shared by the CUDA path's tests and benchmark and by the CPU
oracle's tests. It draws random numbers and rounds them to the storage dtype;
it performs none of the S6 arithmetic (no softplus, no exponentials of the
recurrence, no readout), so the two implementations it feeds stay independent.

The distributions follow the workload recipe of the S6 layer described in
"Notas sobre Mamba" (section "O mecanismo de seleção (S6)"): a diagonal
transition A = -exp(A_log) with the S4D-real initialisation A_log[d,n] =
log(n+1), so A[d,n] = -(n+1) exactly; a raw step Δ_raw ~ N(0, 0.5²) plus a
per-channel bias Δ_bias = log(expm1(dt)) with dt log-uniform in [1e-3, 1e-1]
(the inverse softplus of dt, so that softplus(Δ_bias) = dt); u, B, C, z ~
N(0, 1); D ~ U[0.5, 1.5].

bf16 tensors are drawn in fp32 and rounded to nearest-even; they are held on
the host as ``numpy.uint16`` bit patterns.
"""
from __future__ import annotations

import concurrent.futures as _cf
import dataclasses
import os

import numpy as np
from numpy.random import SeedSequence, default_rng

__all__ = [
    "ScanWorkload",
    "DecodeWorkload",
    "SCAN_WORKLOADS",
    "DECODE_WORKLOADS",
    "make_scan_inputs",
    "make_decode_state",
    "make_decode_step",
    "bf16_bits_from_f32",
    "f32_from_bf16_bits",
    "SsdWorkload",
    "SSD_WORKLOADS",
    "make_ssd_inputs",
    "make_ssd_state",
    "make_delta_regime",
    "DELTA_REGIMES",
]

BASE_SEED = 20261202

# One draw stream per tensor, so that the value of a tensor does not depend on
# which other tensors were drawn.
_STREAM = {"u": 1, "delta": 2, "B": 3, "C": 4, "z": 5, "D": 6, "dt": 7, "h0": 8, "conv_w": 9, "conv_b": 10,
           "conv_state": 11, "lambda_raw": 12, "ssd_x": 13, "ssd_dt": 14, "ssd_B": 15, "ssd_C": 16, "ssd_z": 17,
           "ssd_head": 18, "ssd_h0": 19, "regime": 20, "regime_pick": 21}
_CHUNK = 1 << 22


@dataclasses.dataclass(frozen=True)
class ScanWorkload:
    name: str
    batch: int
    dim: int          # d_inner
    dstate: int       # N
    seqlen: int       # L
    dtype: str        # "f32" or "bf16": dtype of u, delta, B, C, z and y
    has_z: bool
    seed: int

    @property
    def elements(self) -> int:
        """Scan elements (b, d, t, n) processed by one pass."""
        return self.batch * self.dim * self.seqlen * self.dstate


@dataclasses.dataclass(frozen=True)
class DecodeWorkload:
    name: str
    batch: int
    dim: int
    dstate: int
    steps: int
    dtype: str
    has_z: bool
    seed: int


SCAN_WORKLOADS = {
    "s6_tiny_f32": ScanWorkload("s6_tiny_f32", 1, 16, 4, 64, "f32", False, BASE_SEED + 0),
    "mamba130m_layer": ScanWorkload("mamba130m_layer", 8, 1536, 16, 2048, "bf16", True, BASE_SEED + 1),
    "mamba1p4b_layer": ScanWorkload("mamba1p4b_layer", 4, 4096, 16, 8192, "bf16", True, BASE_SEED + 2),
    "long_context_131k": ScanWorkload("long_context_131k", 1, 5120, 16, 131072, "bf16", True, BASE_SEED + 3),
}

DECODE_WORKLOADS = {
    "decode_b256_d5120": DecodeWorkload("decode_b256_d5120", 256, 5120, 16, 1000, "bf16", True, BASE_SEED + 4),
}


@dataclasses.dataclass(frozen=True)
class SsdWorkload:
    """A Mamba-2 SSD layer: x (batch, L, nheads, headdim), B and C (batch, L,
    ngroups, dstate)."""
    name: str
    batch: int
    seqlen: int
    nheads: int
    ngroups: int
    headdim: int
    dstate: int
    has_z: bool
    seed: int

    @property
    def elements(self) -> int:
        """State elements (b, t, h, p, n) updated by one pass."""
        return self.batch * self.seqlen * self.nheads * self.headdim * self.dstate


# The Mamba-2 layer of "Mamba-2 e State Space Duality (SSD)", section
# "Implementando Mamba-2 em pipelines de inferência": batch 4, 8192 tokens,
# d_model 2048 with expand 2 (d_inner 4096 = 64 heads of headdim 64), d_state
# 128, bf16; one group of B and C. The small case has a ragged last block.
SSD_WORKLOADS = {
    "ssd_small": SsdWorkload("ssd_small", 2, 300, 4, 1, 64, 128, True, BASE_SEED + 10),
    "mamba2_layer_d2048": SsdWorkload("mamba2_layer_d2048", 4, 8192, 64, 1, 64, 128, True, BASE_SEED + 11),
}


def _threads() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:  # pragma: no cover
        return max(1, os.cpu_count() or 1)


def _fill(out: np.ndarray, seed: int, stream: int, draw) -> None:
    """Fill ``out`` (flat, float32) chunk by chunk from independent child streams.

    Chunk ``c`` of a tensor always comes from ``SeedSequence(seed,
    spawn_key=(stream, c))``, so the result does not depend on the number of
    threads used.
    """
    flat = out.reshape(-1)
    n = flat.size
    nchunks = (n + _CHUNK - 1) // _CHUNK

    def one(c: int) -> None:
        g = default_rng(SeedSequence(seed, spawn_key=(stream, c)))
        sl = flat[c * _CHUNK:min(n, (c + 1) * _CHUNK)]
        draw(g, sl)

    if nchunks <= 1:
        for c in range(nchunks):
            one(c)
        return
    with _cf.ThreadPoolExecutor(min(_threads(), nchunks)) as ex:
        list(ex.map(one, range(nchunks)))


def _normal(shape, seed, stream, scale=1.0) -> np.ndarray:
    out = np.empty(shape, np.float32)

    def draw(g, sl):
        g.standard_normal(out=sl, dtype=np.float32)
        if scale != 1.0:
            sl *= np.float32(scale)

    _fill(out, seed, stream, draw)
    return out


def bf16_bits_from_f32(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (nearest, ties to even); return the bits."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, np.uint16)
    src = x.reshape(-1).view(np.uint32)
    dst = out.reshape(-1)
    n = src.size
    nchunks = max(1, (n + _CHUNK - 1) // _CHUNK)

    def one(c):
        s = src[c * _CHUNK:min(n, (c + 1) * _CHUNK)]
        lsb = (s >> np.uint32(16)) & np.uint32(1)
        r = (s + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
        dst[c * _CHUNK:min(n, (c + 1) * _CHUNK)] = r.astype(np.uint16)

    if nchunks == 1:
        one(0)
    else:
        with _cf.ThreadPoolExecutor(min(_threads(), nchunks)) as ex:
            list(ex.map(one, range(nchunks)))
    return out


def f32_from_bf16_bits(bits: np.ndarray) -> np.ndarray:
    """Widen bfloat16 bit patterns to float32 (exact)."""
    return (np.asarray(bits, np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _store(x32: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "f32":
        return x32
    if dtype == "bf16":
        return bf16_bits_from_f32(x32)
    raise ValueError(f"unknown dtype {dtype!r}")


def _channel_params(dim: int, dstate: int, seed: int):
    """A (dim, dstate), D (dim,), delta_bias (dim,), all float32."""
    # S4D-real initialisation A_log[d,n] = log(n+1): A = -exp(A_log) = -(n+1),
    # written out directly because it is an integer and exact in float32.
    n = np.arange(dstate, dtype=np.float64)
    A = np.broadcast_to(-(n + 1.0), (dim, dstate)).astype(np.float32).copy()
    gD = default_rng(SeedSequence(seed, spawn_key=(_STREAM["D"],)))
    D = gD.uniform(0.5, 1.5, size=dim).astype(np.float32)
    gdt = default_rng(SeedSequence(seed, spawn_key=(_STREAM["dt"],)))
    dt = np.exp(gdt.uniform(np.log(1e-3), np.log(1e-1), size=dim))
    delta_bias = np.log(np.expm1(dt)).astype(np.float32)
    return A, D, delta_bias


def make_scan_inputs(w: ScanWorkload, *, batch: int | None = None, dim: int | None = None,
                     dstate: int | None = None, seqlen: int | None = None,
                     dtype: str | None = None, has_z: bool | None = None,
                     seed: int | None = None) -> dict:
    """Draw one scan workload on the host.

    Keyword overrides give shapes of the same recipe (used for edge-case
    tests). Returns a dict with numpy arrays: ``u, delta, z`` (batch, dim, L),
    ``B, C`` (batch, dstate, L) in the storage dtype (float32, or uint16 bf16
    bits), and float32 ``A`` (dim, dstate), ``D`` (dim,), ``delta_bias``
    (dim,), plus the shape fields.
    """
    bt = w.batch if batch is None else batch
    dm = w.dim if dim is None else dim
    ns = w.dstate if dstate is None else dstate
    L = w.seqlen if seqlen is None else seqlen
    dt_ = w.dtype if dtype is None else dtype
    hz = w.has_z if has_z is None else has_z
    sd = w.seed if seed is None else seed

    A, D, delta_bias = _channel_params(dm, ns, sd)
    out = {
        "batch": bt, "dim": dm, "dstate": ns, "seqlen": L, "dtype": dt_,
        "u": _store(_normal((bt, dm, L), sd, _STREAM["u"]), dt_),
        "delta": _store(_normal((bt, dm, L), sd, _STREAM["delta"], 0.5), dt_),
        "B": _store(_normal((bt, ns, L), sd, _STREAM["B"]), dt_),
        "C": _store(_normal((bt, ns, L), sd, _STREAM["C"]), dt_),
        "z": _store(_normal((bt, dm, L), sd, _STREAM["z"]), dt_) if hz else None,
        "A": A, "D": D, "delta_bias": delta_bias,
    }
    return out


def make_decode_state(w: DecodeWorkload, *, batch=None, dim=None, dstate=None, seed=None) -> dict:
    """Initial fp32 state h0 ~ N(0,1) (batch, dim, dstate) and the per-channel parameters."""
    bt = w.batch if batch is None else batch
    dm = w.dim if dim is None else dim
    ns = w.dstate if dstate is None else dstate
    sd = w.seed if seed is None else seed
    A, D, delta_bias = _channel_params(dm, ns, sd)
    return {"batch": bt, "dim": dm, "dstate": ns, "dtype": w.dtype,
            "h0": _normal((bt, dm, ns), sd, _STREAM["h0"]), "A": A, "D": D,
            "delta_bias": delta_bias}


def make_decode_step(w: DecodeWorkload, step: int, *, batch=None, dim=None, dstate=None,
                     seed=None, dtype=None, has_z=None) -> dict:
    """Token inputs of decode step ``step``: x, delta, z (batch, dim); B, C (batch, dstate)."""
    bt = w.batch if batch is None else batch
    dm = w.dim if dim is None else dim
    ns = w.dstate if dstate is None else dstate
    sd = (w.seed if seed is None else seed) + 1 + step
    dt_ = w.dtype if dtype is None else dtype
    hz = w.has_z if has_z is None else has_z
    return {
        "x": _store(_normal((bt, dm), sd, _STREAM["u"]), dt_),
        "delta": _store(_normal((bt, dm), sd, _STREAM["delta"], 0.5), dt_),
        "B": _store(_normal((bt, ns), sd, _STREAM["B"]), dt_),
        "C": _store(_normal((bt, ns), sd, _STREAM["C"]), dt_),
        "z": _store(_normal((bt, dm), sd, _STREAM["z"]), dt_) if hz else None,
    }


def make_conv_params(dim: int, width: int = 4, seed: int = BASE_SEED) -> dict:
    """Depthwise convolution taps (dim, width) and bias (dim,), float32, drawn
    U(-1/sqrt(width), 1/sqrt(width)) like a default-initialised depthwise
    Conv1d (fan-in = width)."""
    bound = 1.0 / np.sqrt(width)
    gw = default_rng(SeedSequence(seed, spawn_key=(_STREAM["conv_w"],)))
    gb = default_rng(SeedSequence(seed, spawn_key=(_STREAM["conv_b"],)))
    return {"conv_w": gw.uniform(-bound, bound, size=(dim, width)).astype(np.float32),
            "conv_b": gb.uniform(-bound, bound, size=dim).astype(np.float32)}


def make_conv_state(batch: int, dim: int, width: int, dtype: str, seed: int = BASE_SEED) -> np.ndarray:
    """A convolution state (batch, dim, width) of N(0,1) inputs in the storage
    dtype (float32, or bf16 bits)."""
    return _store(_normal((batch, dim, width), seed, _STREAM["conv_state"]), dtype)


def make_lambda_raw(batch: int, dim: int, seqlen: int, dtype: str, seed: int = BASE_SEED) -> np.ndarray:
    """Pre-activation of the trapezoidal rule's per-token gate, N(0, 1) in the
    storage dtype (float32, or bf16 bits), shape (batch, dim, seqlen)."""
    return _store(_normal((batch, dim, seqlen), seed, _STREAM["lambda_raw"]), dtype)


def make_ssd_inputs(w: SsdWorkload, *, batch=None, seqlen=None, nheads=None, ngroups=None, has_z=None,
                    seed=None) -> dict:
    """Draw one Mamba-2 SSD workload on the host (bf16 bits for x, dt, B, C, z).

    Recipe (Mamba-2 initialisation): per head A = -U[1, 16] (A_log = log of a
    uniform draw in [1, 16]), D ~ U[0.5, 1.5], dt_bias = log(expm1(dt)) with dt
    log-uniform in [1e-3, 1e-1]; per token dt_raw ~ N(0, 0.5^2); x, B, C, z ~
    N(0, 1). Returns x, z (batch, L, nheads, headdim), dt (batch, L, nheads),
    B, C (batch, L, ngroups, dstate) as uint16 bf16 bits, and float32 A, D,
    dt_bias (nheads,), plus the shape fields.
    """
    bt = w.batch if batch is None else batch
    L = w.seqlen if seqlen is None else seqlen
    H = w.nheads if nheads is None else nheads
    G = w.ngroups if ngroups is None else ngroups
    hz = w.has_z if has_z is None else has_z
    sd = w.seed if seed is None else seed
    gh = default_rng(SeedSequence(sd, spawn_key=(_STREAM["ssd_head"],)))
    A = (-gh.uniform(1.0, 16.0, size=H)).astype(np.float32)
    D = gh.uniform(0.5, 1.5, size=H).astype(np.float32)
    dt0 = np.exp(gh.uniform(np.log(1e-3), np.log(1e-1), size=H))
    dt_bias = np.log(np.expm1(dt0)).astype(np.float32)
    P, N = w.headdim, w.dstate
    return {
        "batch": bt, "seqlen": L, "nheads": H, "ngroups": G, "headdim": P, "dstate": N,
        "x": bf16_bits_from_f32(_normal((bt, L, H, P), sd, _STREAM["ssd_x"])),
        "dt": bf16_bits_from_f32(_normal((bt, L, H), sd, _STREAM["ssd_dt"], 0.5)),
        "B": bf16_bits_from_f32(_normal((bt, L, G, N), sd, _STREAM["ssd_B"])),
        "C": bf16_bits_from_f32(_normal((bt, L, G, N), sd, _STREAM["ssd_C"])),
        "z": bf16_bits_from_f32(_normal((bt, L, H, P), sd, _STREAM["ssd_z"])) if hz else None,
        "A": A, "D": D, "dt_bias": dt_bias,
    }


def make_ssd_state(batch: int, nheads: int, headdim: int = 64, dstate: int = 128, seed: int = BASE_SEED) -> np.ndarray:
    """An initial SSD state (batch, nheads, headdim, dstate) float32 ~ N(0, 1)."""
    return _normal((batch, nheads, headdim, dstate), seed, _STREAM["ssd_h0"])


# Step values outside the layer recipe, for the method's degenerate regimes
# ("Notas sobre Mamba", section "O mecanismo de seleção (S6)": a large step
# resets the state to the current input, a step near zero keeps the state and
# ignores the input):
#   "large"  U[10, 50]    -- exp(delta A) underflows for every state
#   "edge"   U[15, 40]    -- a softplus argument on both sides of 20
#   "zero"   exactly 0    -- Abar = 1 and Bbar = 0
#   "mixed"  per element 0 (30%), |N(0, 0.5^2)| / 8 (50%) or U[10, 50] (20%):
#            resets and holds inside one sequence
DELTA_REGIMES = ("large", "edge", "zero", "mixed")


def make_delta_regime(shape, regime: str, dtype: str, seed: int = BASE_SEED) -> np.ndarray:
    """Raw step values of one of ``DELTA_REGIMES`` in the storage dtype
    (float32, or bf16 bits), shape ``shape``."""
    if regime not in DELTA_REGIMES:
        raise ValueError(f"unknown regime {regime!r}")
    out = np.zeros(shape, np.float32)
    if regime in ("large", "edge"):
        lo, hi = (10.0, 50.0) if regime == "large" else (15.0, 40.0)

        def draw(g, sl):
            sl[:] = g.uniform(lo, hi, size=sl.size).astype(np.float32)

        _fill(out, seed, _STREAM["regime"], draw)
    elif regime == "mixed":
        small = np.abs(_normal(shape, seed, _STREAM["regime"], 0.5)) / np.float32(8.0)
        big = np.empty(shape, np.float32)
        _fill(big, seed, _STREAM["regime"] + 100, lambda g, sl: sl.__setitem__(
            slice(None), g.uniform(10.0, 50.0, size=sl.size).astype(np.float32)))
        pick = np.empty(shape, np.float32)
        _fill(pick, seed, _STREAM["regime_pick"], lambda g, sl: sl.__setitem__(
            slice(None), g.random(size=sl.size, dtype=np.float32)))
        out = np.where(pick < 0.3, np.float32(0.0), np.where(pick < 0.8, small, big)).astype(np.float32)
    return _store(out, dtype)
