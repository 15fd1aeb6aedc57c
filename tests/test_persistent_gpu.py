"""GPU parity of the sequential scan kernels under the persistent schedule.

With ``ms_scan_plan.ctas > 0`` the chunks of all units (batch entry x block of
rows) are cut into equal ranges, one per CTA, and a unit whose chunks fall in
two ranges is continued by a second CTA from the state the first one hands
over. The recurrence is the same ("Notas sobre Mamba", section "A varredura
paralela ciente do hardware": the state stays on chip within a CTA; between
CTAs it passes once through memory), so the results must match the oracle at
the usual bar for every split: one CTA doing everything, ranges that end in
the middle of units, and one range per unit. The workspace's status word must
read 0 afterwards (no carry wait gave up).
"""
import numpy as np
import pytest

from selective_state_space_27_b200.inputs import SCAN_WORKLOADS, make_scan_inputs
from tests.gpu_util import TOL, device_inputs, oracle_scan, rel_err, to_host64

pytestmark = pytest.mark.gpu

LAYER = SCAN_WORKLOADS["mamba130m_layer"]


def _ms():
    import selective_state_space_27_b200 as ms
    return ms


def _sequential():
    return [(cfg, lanes, warps) for cfg, lanes, _, warps, kind in _ms().scan_configs() if kind == 1]


def _run(dev, plan, h0=None):
    import torch
    ms = _ms()
    args = ms.build_scan_args(dev["u"], dev["delta"], dev["A"], dev["B"], dev["C"], torch.empty_like(dev["u"]))
    ws = torch.empty(max(ms.plan_workspace_size(args, plan), 256), dtype=torch.uint8, device="cuda")
    y, hT = ms.scan_fwd(**dev, plan=plan, workspace=ws, initial_state=h0)
    assert ms.scan_status(ws) == 0, "a carry wait gave up"
    return to_host64(y), to_host64(hT)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("N,L", [(16, 1000 + 7), (5, 333)])
def test_every_split(dtype, N, L):
    """Every sequential configuration, CTA counts from 1 to one per unit."""
    import torch
    ms = _ms()
    batch, dim = 3, 70
    inp = make_scan_inputs(LAYER, batch=batch, dim=dim, dstate=N, seqlen=L, dtype=dtype, seed=8000 + N)
    dev = device_inputs(inp)
    h0 = np.random.default_rng(8001).normal(size=(batch, dim, N)).astype(np.float32)
    yr, hr = oracle_scan(inp, h0=h0.reshape(-1, N))
    for cfg, lanes, warps in _sequential():
        rows = 128 // lanes
        units = batch * ((dim + rows - 1) // rows)
        for ctas in sorted({1, 2, 3, units // 2 or 1, units}):
            if ctas > units:
                continue
            plan = ms.ScanPlan(config=cfg, warps_per_cta=warps, segments=1, ctas=ctas)
            y, hT = _run(dev, plan, h0=torch.from_numpy(h0).cuda())
            tag = f"config {cfg} (lanes {lanes}), {ctas} of {units} units"
            assert rel_err(y, yr) <= TOL[dtype], tag
            assert rel_err(hT, hr) <= TOL[dtype], tag


def test_long_rows_split_many_times():
    """Few rows, long sequences: ranges cut units at many chunk boundaries."""
    ms = _ms()
    inp = make_scan_inputs(LAYER, batch=1, dim=100, seqlen=20000 + 3, seed=8100)
    dev = device_inputs(inp)
    yr, hr = oracle_scan(inp)
    cfg = [c for c, lanes, _ in _sequential() if lanes == 4][0]
    for ctas in (2, 3, 4):   # 4 units of 32 rows
        y, hT = _run(dev, ms.ScanPlan(config=cfg, warps_per_cta=6, segments=1, ctas=ctas))
        assert rel_err(y, yr) <= TOL["bf16"], ctas
        assert rel_err(hT, hr) <= TOL["bf16"], ctas


def test_refused_plans():
    """More CTAs than units, or CTAs on an entry point that takes no workspace,
    are refused before any launch."""
    import ctypes

    import torch
    ms = _ms()
    inp = make_scan_inputs(LAYER, batch=1, dim=64, seqlen=100, seed=8200)
    dev = device_inputs(inp)
    cfg = [c for c, lanes, _ in _sequential() if lanes == 4][0]
    with pytest.raises(ms.MambaScanError) as ei:
        ms.scan_fwd(**dev, plan=ms.ScanPlan(config=cfg, warps_per_cta=6, segments=1, ctas=3))   # 2 units
    assert ei.value.status == 2
    lam = torch.zeros_like(dev["u"])
    with pytest.raises(ms.MambaScanError) as ei:
        ms.trap_scan_fwd(dev["u"], dev["delta"], lam, dev["A"], dev["B"], dev["C"],
                         plan=ms.ScanPlan(config=cfg, warps_per_cta=6, segments=1, ctas=3))
    assert ei.value.status == 2
    lib = ms.load_library()
    args = ms.build_scan_args(dev["u"], dev["delta"], dev["A"], dev["B"], dev["C"], torch.empty_like(dev["u"]))
    plan = ms.ScanPlan(config=cfg, warps_per_cta=6, segments=1, ctas=1)
    assert lib.mamba_trap_scan_fwd(ctypes.byref(args), lam.data_ptr(), lam.stride(0), lam.stride(1),
                                   ctypes.byref(plan), None) == 2
    torch.cuda.synchronize()


def test_automatic_plan_long_context_shape():
    """The automatic plan for the long-context layer's shape (1 x 5120 rows)
    uses the persistent schedule; checked on a shorter sequence in full."""
    import torch
    ms = _ms()
    inp = make_scan_inputs(SCAN_WORKLOADS["long_context_131k"], seqlen=2048 + 5, seed=8300)
    dev = device_inputs(inp)
    args = ms.build_scan_args(dev["u"], dev["delta"], dev["A"], dev["B"], dev["C"], torch.empty_like(dev["u"]))
    plan = ms.scan_plan(args)
    assert plan.ctas > 0, "expected the persistent schedule"
    y, hT = ms.scan_fwd(**dev)
    yr, hr = oracle_scan(inp)
    assert rel_err(to_host64(y), yr) <= TOL["bf16"]
    assert rel_err(to_host64(hT), hr) <= TOL["bf16"]
