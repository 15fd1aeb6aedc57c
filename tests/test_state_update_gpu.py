"""GPU parity of the single-token state update (decode) against the fp64 oracle."""
import numpy as np
import pytest

import oracle
from selective_state_space_27_b200.inputs import (DECODE_WORKLOADS, SCAN_WORKLOADS, make_decode_state,
                                                  make_decode_step, make_scan_inputs)
from tests.gpu_util import TOL, device_inputs, rel_err, sample_rows, to_device, to_host64
from tests.oracle_pins import read_selection_step

pytestmark = pytest.mark.gpu

DEC = DECODE_WORKLOADS["decode_b256_d5120"]


def _ms():
    import selective_state_space_27_b200 as ms
    return ms


def _step_on_gpu(state_t, st, dtype, prm, use_z=True):
    return _ms().state_update(state_t, to_device(st["x"], dtype), to_device(st["delta"], dtype),
                              prm["A"], to_device(st["B"], dtype), to_device(st["C"], dtype),
                              D=prm["D"], z=to_device(st["z"], dtype) if use_z else None,
                              delta_bias=prm["delta_bias"])


def test_selection_step_worked_example():
    """The page's single step ("Notas sobre Mamba", "O mecanismo de seleção (S6)"):
    h = 1, x = 1, A = -1, B = 1 gives h = 5.0067 for delta = 5 and 1.0000 for
    delta = 0.01 (4 decimals), on the float32 GPU path."""
    import torch
    ms = _ms()
    N = 4
    for delta, abar, bbar, h_new in read_selection_step():
        for Bval, expect in ((0.0, abar), (1.0, h_new)):
            state = torch.ones((1, 1, N), device="cuda")
            f = lambda v, shape: torch.full(shape, v, device="cuda", dtype=torch.float32)
            ms.state_update(state, f(1.0, (1, 1)), f(delta, (1, 1)), f(-1.0, (1, N)),
                            f(Bval, (1, N)), f(1.0, (1, N)), delta_softplus=False)
            torch.cuda.synchronize()
            got = np.round(state.cpu().numpy().astype(np.float64).reshape(-1), 4)
            assert np.all(np.abs(got - expect) < 1e-9), (delta, Bval, got, expect)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("N", [1, 3, 4, 16])
@pytest.mark.parametrize("use_z", [True, False])
def test_single_step(dtype, N, use_z):
    import torch
    d = make_decode_state(DEC, batch=5, dim=77, dstate=N, seed=31 + N)
    st = make_decode_step(DEC, 0, batch=5, dim=77, dstate=N, dtype=dtype, seed=31 + N)
    prm = {k: to_device(d[k], "f32") for k in ("A", "D", "delta_bias")}
    state_t = torch.from_numpy(d["h0"]).cuda()
    y = _step_on_gpu(state_t, st, dtype, prm, use_z)
    torch.cuda.synchronize()
    ref_state = d["h0"].astype(np.float64)
    yr = oracle.state_update(state=ref_state, x=st["x"], delta=st["delta"], A=d["A"], B=st["B"],
                             C=st["C"], D=d["D"], z=st["z"] if use_z else None,
                             delta_bias=d["delta_bias"], dtype=dtype)
    assert rel_err(to_host64(y), yr) <= TOL[dtype]
    assert rel_err(to_host64(state_t), ref_state) <= TOL[dtype]


def test_strided_state():
    """State rows with padding between them (batch and row strides != dense)."""
    import torch
    N = 16
    d = make_decode_state(DEC, batch=3, dim=40, dstate=N, seed=41)
    st = make_decode_step(DEC, 0, batch=3, dim=40, dstate=N, seed=41)
    prm = {k: to_device(d[k], "f32") for k in ("A", "D", "delta_bias")}
    big = torch.zeros((3, 41, 20), device="cuda")
    big[:, :40, :16] = torch.from_numpy(d["h0"]).cuda()
    state_t = big[:, :40, :16]
    y = _step_on_gpu(state_t, st, "bf16", prm)
    torch.cuda.synchronize()
    ref_state = d["h0"].astype(np.float64)
    yr = oracle.state_update(state=ref_state, x=st["x"], delta=st["delta"], A=d["A"], B=st["B"],
                             C=st["C"], D=d["D"], z=st["z"], delta_bias=d["delta_bias"], dtype="bf16")
    assert rel_err(to_host64(y), yr) <= TOL["bf16"]
    assert rel_err(to_host64(state_t), ref_state) <= TOL["bf16"]
    assert float(big[:, 40:, :].abs().max()) == 0.0 and float(big[:, :, 16:].abs().max()) == 0.0


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_decode_steps_reproduce_scan(dtype):
    """L single-token updates from h = 0 give the scan's y and final state."""
    import torch
    ms = _ms()
    w = SCAN_WORKLOADS["mamba130m_layer"]
    inp = make_scan_inputs(w, batch=2, dim=48, seqlen=200, dtype=dtype, seed=51)
    dev = device_inputs(inp)
    y_scan, h_scan = ms.scan_fwd(**dev)
    state = torch.zeros((2, 48, 16), device="cuda")
    ys = []
    for t in range(200):
        ys.append(ms.state_update(state, dev["u"][:, :, t].contiguous(), dev["delta"][:, :, t].contiguous(),
                                  dev["A"], dev["B"][:, :, t].contiguous(), dev["C"][:, :, t].contiguous(),
                                  D=dev["D"], z=dev["z"][:, :, t].contiguous(),
                                  delta_bias=dev["delta_bias"]))
    torch.cuda.synchronize()
    y_dec = torch.stack(ys, dim=-1)
    assert rel_err(to_host64(y_dec), to_host64(y_scan)) <= TOL[dtype]
    assert rel_err(to_host64(state), to_host64(h_scan)) <= TOL[dtype]


@pytest.mark.slow
def test_decode_workload_1000_steps_sampled_rows():
    """(256, 5120, 16) fp32 state, 1000 seeded bf16 tokens; y of every step and
    the final state checked on a seeded sample of rows."""
    import torch
    ms = _ms()
    w = DEC
    d = make_decode_state(w)
    rows = sample_rows(w.batch, w.dim, 256, seed=7)
    prm = {k: to_device(d[k], "f32") for k in ("A", "D", "delta_bias")}
    state_t = torch.from_numpy(d["h0"]).cuda()
    ref_state = d["h0"].reshape(-1, w.dstate)[rows].astype(np.float64).copy()
    worst = 0.0
    for s in range(w.steps):
        st = make_decode_step(w, s)
        y = ms.state_update(state_t, to_device(st["x"], "bf16"), to_device(st["delta"], "bf16"),
                            prm["A"], to_device(st["B"], "bf16"), to_device(st["C"], "bf16"),
                            D=prm["D"], z=to_device(st["z"], "bf16"), delta_bias=prm["delta_bias"])
        yr = oracle.state_update(state=ref_state, x=st["x"], delta=st["delta"], A=d["A"], B=st["B"],
                                 C=st["C"], D=d["D"], z=st["z"], delta_bias=d["delta_bias"],
                                 dtype="bf16", rows=rows)
        yg = to_host64(y).reshape(-1)[rows]
        worst = max(worst, rel_err(yg, yr))
    torch.cuda.synchronize()
    assert worst <= TOL["bf16"], worst
    hs = to_host64(state_t).reshape(-1, w.dstate)[rows]
    assert rel_err(hs, ref_state) <= TOL["bf16"]
