"""GPU parity of the exponential-trapezoidal selective scan (Mamba-3) against
the fp64 oracle. Bar as for the scan: 1e-4 (float32 inputs), 5e-3 (bfloat16
inputs) on y and on the final state."""
import numpy as np
import pytest

import oracle
from selective_state_space_27_b200.inputs import SCAN_WORKLOADS, make_lambda_raw, make_scan_inputs
from tests.gpu_util import TOL, device_inputs, oracle_scan, rel_err, to_device, to_host64

pytestmark = pytest.mark.gpu

LAYER = SCAN_WORKLOADS["mamba130m_layer"]


def _ms():
    import selective_state_space_27_b200 as ms
    return ms


def _trap_configs():
    # the fused variants are compiled for the 2-I/O-warp kernels (6 warps) with 2 or 4 lanes per row
    return [(c, lanes, warps) for c, lanes, _, warps, kind in _ms().scan_configs()
            if kind == 1 and lanes in (2, 4) and warps == 6]


def _oracle(inp, lam, *, h0=None, rows=None):
    return oracle.trap_scan(u=inp["u"], delta=inp["delta"], lambda_raw=lam, A=inp["A"], B=inp["B"], C=inp["C"],
                            D=inp["D"], z=inp["z"], delta_bias=inp["delta_bias"], dtype=inp["dtype"], h0=h0,
                            rows=rows)


def _run(dev, lam_t, *, plan=None, h0=None):
    import torch
    y, hT = _ms().trap_scan_fwd(dev["u"], dev["delta"], lam_t, dev["A"], dev["B"], dev["C"], D=dev["D"], z=dev["z"],
                                delta_bias=dev["delta_bias"], initial_state=h0, plan=plan)
    torch.cuda.synchronize()
    return to_host64(y), to_host64(hT)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("batch,dim,N,L,offset", [
    (1, 3, 16, 1, 0), (2, 37, 16, 33, 0), (2, 130, 16, 1000, 0), (3, 20, 5, 97, 0), (1, 64, 16, 64, 0),
    (2, 70, 16, 255, 1), (1, 9, 8, 31, 3),
])
def test_trap_scan_matches_oracle(dtype, batch, dim, N, L, offset):
    """Every configuration that runs the rule, and the automatic plan, on ragged
    rows and lengths, with an initial state, and (offset > 0) rows that are not
    16-byte aligned."""
    import torch
    ms = _ms()
    inp = make_scan_inputs(LAYER, batch=batch, dim=dim, dstate=N, seqlen=L + offset, dtype=dtype,
                           seed=3100 + dim + L)
    lam = make_lambda_raw(batch, dim, L + offset, dtype, seed=3200 + L)
    dev = device_inputs(inp)
    lam_t = to_device(lam, dtype)
    if offset:
        for k in ("u", "delta", "z", "B", "C"):
            dev[k] = dev[k][..., offset:]
            inp[k] = np.ascontiguousarray(inp[k][..., offset:])
        lam_t = lam_t[..., offset:]
        lam = np.ascontiguousarray(lam[..., offset:])
        inp["seqlen"] = L
    h0 = np.random.default_rng(dim).normal(size=(batch, dim, N)).astype(np.float32)
    yr, hr = _oracle(inp, lam, h0=h0.reshape(-1, N))
    plans = [None] + [ms.ScanPlan(config=c, warps_per_cta=w, segments=1) for c, _, w in _trap_configs()]
    for plan in plans:
        y, hT = _run(dev, lam_t, plan=plan, h0=torch.from_numpy(h0).cuda())
        tag = "auto" if plan is None else f"config {plan.config}"
        assert rel_err(y, yr) <= TOL[dtype], tag
        assert rel_err(hT, hr) <= TOL[dtype], tag


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("batch,dim,N,L", [(2, 100, 16, 300), (3, 40, 5, 257)])
def test_trap_scan_persistent_schedule(dtype, batch, dim, N, L):
    """The rule under the persistent schedule: every configuration that runs it
    at CTA counts from 1 to one per unit, including counts that cut units
    between CTAs (the CTA that takes a row over starts from the handed-over
    state and reads B at the step before its first one), on ragged lengths and
    a state size below 16."""
    import torch
    ms = _ms()
    inp = make_scan_inputs(LAYER, batch=batch, dim=dim, dstate=N, seqlen=L, dtype=dtype, seed=3500 + L)
    lam = make_lambda_raw(batch, dim, L, dtype, seed=3600 + L)
    dev = device_inputs(inp)
    lam_t = to_device(lam, dtype)
    h0 = np.random.default_rng(3700 + L).normal(size=(batch, dim, N)).astype(np.float32)
    h0_t = torch.from_numpy(h0).cuda()
    yr, hr = _oracle(inp, lam, h0=h0.reshape(-1, N))
    for c, lanes, w in _trap_configs():
        rows = 128 // lanes
        units = batch * ((dim + rows - 1) // rows)
        for ctas in sorted({1, 2, 3, max(1, units // 2), max(1, units - 1), units}):
            plan = ms.ScanPlan(config=c, warps_per_cta=w, segments=1, ctas=ctas)
            y, hT = _run(dev, lam_t, plan=plan, h0=h0_t)
            tag = f"config {c}, {ctas} CTAs of {units} units"
            assert rel_err(y, yr) <= TOL[dtype], tag
            assert rel_err(hT, hr) <= TOL[dtype], tag


def test_trap_with_lambda_one_is_the_euler_scan():
    """lambda = sigmoid(20) = 1 in float32: the rule reduces to exponential-Euler,
    so the result matches the plain scan's oracle."""
    inp = make_scan_inputs(LAYER, batch=2, dim=48, seqlen=300, dtype="f32", seed=3300)
    dev = device_inputs(inp)
    lam_t = to_device(np.full(inp["u"].shape, 20.0, np.float32), "f32")
    y, hT = _run(dev, lam_t)
    yr, hr = oracle_scan(inp)
    assert rel_err(y, yr) <= TOL["f32"] and rel_err(hT, hr) <= TOL["f32"]


def test_trap_scan_mamba130m_layer_full():
    """The Mamba-130M-shaped layer (bf16, gate) with lambda_raw ~ N(0, 1), every row."""
    inp = make_scan_inputs(LAYER)
    lam = make_lambda_raw(inp["batch"], inp["dim"], inp["seqlen"], "bf16")
    y, hT = _run(device_inputs(inp), to_device(lam, "bf16"))
    yr, hr = _oracle(inp, lam)
    assert rel_err(y, yr) <= TOL["bf16"] and rel_err(hT, hr) <= TOL["bf16"]


def test_trap_scan_rejects_unusable_plans():
    ms = _ms()
    inp = make_scan_inputs(LAYER, batch=1, dim=16, seqlen=64, seed=3400)
    dev = device_inputs(inp)
    lam_t = to_device(make_lambda_raw(1, 16, 64, "bf16"), "bf16")
    for cfg, lanes, _, warps, kind in ms.scan_configs():
        if kind == 1 and lanes in (2, 4):
            continue
        with pytest.raises(ms.MambaScanError) as ei:
            ms.trap_scan_fwd(dev["u"], dev["delta"], lam_t, dev["A"], dev["B"], dev["C"],
                             plan=ms.ScanPlan(config=cfg, warps_per_cta=warps, segments=1))
        assert ei.value.status == 2
