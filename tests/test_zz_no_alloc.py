"""mamba_scan_fwd_noalloc: the scan entry point for callers that cannot allocate.

Some callers of this library cannot hand it a workspace: a plugin inside a
host application that owns all device memory and passes in only its tensors,
or a path where cudaMalloc is off limits because it can stall the device.
mamba_scan_fwd_noalloc keeps the multi-block carry workspace in a fixed
device array inside the library instead. These tests call it through the C ABI
and check that it gives the same y and final state as mamba_scan_fwd (with a
caller-allocated workspace), within the parity tolerance of the other tests,
on two calls in a row with different inputs -- the second call must not be
disturbed by what the first left in the shared array -- and that a call too
large for the array is refused without launching anything.

This file is named to be collected last, so that a run stopping at the first
failure has already run every other test; it also passes on its own.
"""
import ctypes

import numpy as np
import pytest

from selective_state_space_27_b200.inputs import SCAN_WORKLOADS, make_scan_inputs
from tests.gpu_util import TOL, device_inputs, rel_err, to_host64

pytestmark = pytest.mark.gpu

LAYER = SCAN_WORKLOADS["mamba130m_layer"]
MS_ERR_WORKSPACE = 6
SCRATCH_BYTES = 8 << 20


def _entry():
    import selective_state_space_27_b200 as ms
    lib = ms.load_library()
    fn = lib.mamba_scan_fwd_noalloc
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.POINTER(ms.ScanArgs), ctypes.c_void_p]
    return ms, lib, fn


def _call_noalloc(dev, dtype_t, force_segments):
    import torch
    ms, lib, fn = _entry()
    batch, dim, L = dev["u"].shape
    y = torch.full_like(dev["u"], float("nan"))
    hT = torch.full((batch, dim, dev["B"].shape[1]), float("nan"), device="cuda")
    args = ms.build_scan_args(dev["u"], dev["delta"], dev["A"], dev["B"], dev["C"], y, D=dev["D"],
                              z=dev["z"], delta_bias=dev["delta_bias"], final_state=hT,
                              force_segments=force_segments)
    rc = fn(ctypes.byref(args), torch.cuda.current_stream().cuda_stream)
    assert rc == 0, lib.mamba_last_error().decode()
    torch.cuda.synchronize()
    return to_host64(y), to_host64(hT)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("force_segments", [0, 3, 16])
def test_noalloc_matches_workspace_entry_point(dtype, force_segments):
    import torch
    ms, _, _ = _entry()
    for call, seed in enumerate((1001, 1002)):   # two calls in a row, different inputs
        inp = make_scan_inputs(LAYER, batch=2, dim=40, seqlen=4096 + 13, dtype=dtype, seed=seed)
        dev = device_inputs(inp)
        y_ref, h_ref = ms.scan_fwd(**dev, force_segments=force_segments)
        torch.cuda.synchronize()
        y, h = _call_noalloc(dev, dtype, force_segments)
        assert np.isfinite(y).all() and np.isfinite(h).all(), f"call {call}: output not written"
        assert rel_err(y, to_host64(y_ref)) <= TOL[dtype], f"call {call}: y differs"
        assert rel_err(h, to_host64(h_ref)) <= TOL[dtype], f"call {call}: final state differs"


def test_noalloc_refuses_more_than_the_built_in_array():
    import torch
    ms, lib, fn = _entry()
    batch, dim, N, L, segs = 2, 4096, 16, 64 * 64, 64
    assert batch * dim * segs * 2 * N * 4 > SCRATCH_BYTES
    u = torch.zeros((batch, dim, L), dtype=torch.bfloat16, device="cuda")
    Bm = torch.zeros((batch, N, L), dtype=torch.bfloat16, device="cuda")
    A = -torch.ones((dim, N), device="cuda")
    y = torch.full_like(u, 7.0)
    args = ms.build_scan_args(u, u, A, Bm, Bm, y, force_segments=segs)
    rc = fn(ctypes.byref(args), torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert rc == MS_ERR_WORKSPACE
    assert "scratch" in lib.mamba_last_error().decode()
    assert float(y.float().min()) == 7.0 and float(y.float().max()) == 7.0   # nothing launched
