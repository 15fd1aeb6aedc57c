"""Helpers for the GPU parity tests: move seeded host inputs to the device, run
the CUDA path through the C ABI, and compare with the fp64 oracle."""
from __future__ import annotations

import numpy as np

import oracle

TOL = {"f32": 1e-4, "bf16": 5e-3}


def to_device(a, dtype):
    """numpy float32 or uint16 (bf16 bits) -> torch CUDA tensor of the storage dtype."""
    import torch
    if a is None:
        return None
    if dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(a)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def to_host64(t):
    import torch
    return t.detach().to(torch.float64).cpu().numpy()


def rel_err(got, ref) -> float:
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    scale = np.abs(ref).max()
    if scale == 0:
        return float(np.abs(got).max())
    return float(np.abs(got - ref).max() / scale)


def device_inputs(inp, *, use_z=True, use_D=True, use_bias=True):
    dt = inp["dtype"]
    return dict(
        u=to_device(inp["u"], dt), delta=to_device(inp["delta"], dt),
        B=to_device(inp["B"], dt), C=to_device(inp["C"], dt),
        z=to_device(inp["z"], dt) if (use_z and inp["z"] is not None) else None,
        A=to_device(inp["A"], "f32"),
        D=to_device(inp["D"], "f32") if use_D else None,
        delta_bias=to_device(inp["delta_bias"], "f32") if use_bias else None,
    )


def oracle_scan(inp, *, rows=None, use_z=True, use_D=True, use_bias=True, softplus=True, h0=None,
                threads=0):
    return oracle.scan(u=inp["u"], delta=inp["delta"], A=inp["A"], B=inp["B"], C=inp["C"],
                       D=inp["D"] if use_D else None,
                       z=inp["z"] if use_z else None,
                       delta_bias=inp["delta_bias"] if use_bias else None,
                       delta_softplus=softplus, dtype=inp["dtype"], rows=rows, h0=h0,
                       threads=threads)


def sample_rows(batch, dim, count, seed=0):
    """A fixed seeded set of rows b*dim+d, always including the first and last."""
    g = np.random.default_rng(seed)
    n = batch * dim
    if n <= count:
        return np.arange(n, dtype=np.int64)
    rows = set(g.choice(n, size=count - 2, replace=False).tolist())
    rows.update([0, n - 1])
    return np.array(sorted(rows), dtype=np.int64)
