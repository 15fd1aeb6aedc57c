"""GPU parity in the step size's degenerate regimes, for every scan kernel
configuration, the decode step and the Mamba-2 SSD forward.

"Notas sobre Mamba", section "O mecanismo de seleção (S6)", reads the step
delta as a gate: a large step resets the state to the current input (Abar =
exp(delta A) -> 0), a step near zero keeps the state and ignores the input
(Abar -> 1, Bbar -> 0). The layer recipe keeps delta between about 1e-3 and
0.5, so these cases come from their own generators (``make_delta_regime``):
steps of 10 to 50 (exp(delta A) far below the float32 range for A = -(n+1)),
softplus arguments on both sides of its identity threshold 20, steps that are
exactly zero, and sequences that mix the three. The bar is the same as for the
layer workloads: max|err| / max|ref| <= 1e-4 (float32) and 5e-3 (bf16) on y
and on the final state, against the fp64 oracle on the same inputs.
"""
import numpy as np
import pytest

import oracle
from selective_state_space_27_b200.inputs import (DECODE_WORKLOADS, SCAN_WORKLOADS, SSD_WORKLOADS,
                                                  make_decode_state, make_decode_step, make_delta_regime,
                                                  make_scan_inputs, make_ssd_inputs, make_ssd_state)
from tests.gpu_util import TOL, device_inputs, oracle_scan, rel_err, to_device, to_host64

pytestmark = pytest.mark.gpu

LAYER = SCAN_WORKLOADS["mamba130m_layer"]
DEC = DECODE_WORKLOADS["decode_b256_d5120"]
SSD = SSD_WORKLOADS["ssd_small"]

# (regime of the raw step, softplus on, bias): "edge" runs through the softplus
# with no bias (argument = raw step in [15, 40]); "edge_bias" puts the large
# value in the per-channel bias instead, under a recipe-sized raw step.
CASES = [("large", False, False), ("edge", True, False), ("edge_bias", True, True), ("zero", False, False),
         ("mixed", False, False)]


def _ms():
    import selective_state_space_27_b200 as ms
    return ms


def _scan_case(regime, dtype, *, batch=2, dim=70, N=16, L=296, seed=0, steep_A=False):
    inp = make_scan_inputs(LAYER, batch=batch, dim=dim, dstate=N, seqlen=L, dtype=dtype, seed=seed)
    if regime == "edge_bias":
        inp["delta_bias"] = make_delta_regime((dim,), "edge", "f32", seed + 1)
    else:
        inp["delta"] = make_delta_regime((batch, dim, L), regime, dtype, seed + 1)
    if steep_A:
        # A = -exp(U[3, 6]) per (d, n): -20 ... -400, so delta A << -100 already for steps near 1
        g = np.random.default_rng(seed + 2)
        inp["A"] = (-np.exp(g.uniform(3.0, 6.0, size=(dim, N)))).astype(np.float32)
    h0 = np.random.default_rng(seed + 3).normal(size=(batch, dim, N)).astype(np.float32)
    return inp, h0


def _plans():
    """(plan, tag) for every configuration: sequential kernels at their fixed
    CTA; chunked kernels at 2 warps with 3 segments (the multi-block carry)."""
    ms = _ms()
    out = []
    for cfg, lanes, states, max_warps, kind in ms.scan_configs():
        if kind == 1:
            out.append((ms.ScanPlan(config=cfg, warps_per_cta=max_warps, segments=1), f"sequential cfg {cfg}"))
        else:
            out.append((ms.ScanPlan(config=cfg, warps_per_cta=2, segments=3), f"chunked cfg {cfg}, 3 segments"))
    return out


def _check_scan(inp, h0, softplus, use_bias, plan=None, tag=""):
    import torch
    ms = _ms()
    dtype = inp["dtype"]
    dev = device_inputs(inp, use_bias=use_bias)
    y, hT = ms.scan_fwd(**dev, delta_softplus=softplus, initial_state=torch.from_numpy(h0).cuda(), plan=plan)
    torch.cuda.synchronize()
    y, hT = to_host64(y), to_host64(hT)
    yr, hr = oracle_scan(inp, use_bias=use_bias, softplus=softplus, h0=h0.reshape(-1, inp["dstate"]))
    assert np.isfinite(y).all() and np.isfinite(hT).all(), tag
    ey, eh = rel_err(y, yr), rel_err(hT, hr.reshape(hT.shape))
    assert ey <= TOL[dtype], f"{tag}: y error {ey:.3e}"
    assert eh <= TOL[dtype], f"{tag}: final state error {eh:.3e}"
    return hT


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("regime,softplus,use_bias", CASES)
def test_scan_every_configuration(dtype, regime, softplus, use_bias):
    """Each compiled scan configuration (and the automatic plan) on one regime."""
    inp, h0 = _scan_case(regime, dtype, seed=7000 + 10 * CASES.index((regime, softplus, use_bias)))
    for plan, tag in [(None, "automatic plan")] + _plans():
        hT = _check_scan(inp, h0, softplus, use_bias, plan=plan, tag=f"{regime}/{dtype}: {tag}")
        if regime == "zero":
            # Abar = 1 and Bbar u = 0 at every step: the state comes out unchanged
            assert np.array_equal(hT, h0.astype(np.float64)), f"{tag}: state changed under delta = 0"


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("regime", ["large", "mixed"])
def test_scan_steep_decay(dtype, regime):
    """delta A far below -100 (A down to -400) with the recipe's state size
    and a ragged state size, automatic and segmented plans."""
    for N, seed in ((16, 7100), (5, 7110)):
        inp, h0 = _scan_case(regime, dtype, N=N, seed=seed + (regime == "mixed"), steep_A=True)
        _check_scan(inp, h0, False, False, tag=f"steep {regime}/{dtype}/N={N}")
        ms = _ms()
        _check_scan(inp, h0, False, False, plan=ms.ScanPlan(config=0, warps_per_cta=2, segments=4),
                    tag=f"steep {regime}/{dtype}/N={N}, chunked cfg 0, 4 segments")


def test_scan_long_mixed_sequence_segments():
    """A 20k-step sequence of mixed resets and holds, cut into 8 segments by the
    multi-block carry (decay products that underflow inside a segment)."""
    inp, h0 = _scan_case("mixed", "bf16", batch=1, dim=24, L=20000 + 3, seed=7200)
    _check_scan(inp, h0, False, False, tag="mixed, automatic")
    inp["delta"] = make_delta_regime((1, 24, 20003), "mixed", "bf16", 7201)
    import selective_state_space_27_b200 as ms
    import torch
    dev = device_inputs(inp, use_bias=False)
    y, hT = ms.scan_fwd(**dev, delta_softplus=False, initial_state=torch.from_numpy(h0).cuda(), force_segments=8)
    torch.cuda.synchronize()
    yr, hr = oracle_scan(inp, use_bias=False, softplus=False, h0=h0.reshape(-1, 16))
    assert rel_err(to_host64(y), yr) <= TOL["bf16"]
    assert rel_err(to_host64(hT), hr.reshape(hT.shape)) <= TOL["bf16"]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("regime,softplus,use_bias", CASES)
def test_decode_steps(dtype, regime, softplus, use_bias):
    """Five decode steps in a row from a random state, each step's y and the
    state after every step against the oracle's decode step."""
    import torch
    ms = _ms()
    batch, dim, N = 3, 77, 16
    seed = 7300 + 10 * CASES.index((regime, softplus, use_bias))
    d = make_decode_state(DEC, batch=batch, dim=dim, dstate=N, seed=seed)
    bias = make_delta_regime((dim,), "edge", "f32", seed + 1) if regime == "edge_bias" else d["delta_bias"]
    prm = {"A": to_device(d["A"], "f32"), "D": to_device(d["D"], "f32"), "delta_bias": to_device(bias, "f32")}
    state_t = torch.from_numpy(d["h0"]).cuda()
    ref = d["h0"].astype(np.float64)
    for s in range(5):
        st = make_decode_step(DEC, s, batch=batch, dim=dim, dstate=N, dtype=dtype, seed=seed)
        if regime != "edge_bias":
            st["delta"] = make_delta_regime((batch, dim), regime, dtype, seed + 2 + s)
        before = state_t.clone()
        y = ms.state_update(state_t, to_device(st["x"], dtype), to_device(st["delta"], dtype), prm["A"],
                            to_device(st["B"], dtype), to_device(st["C"], dtype), D=prm["D"],
                            z=to_device(st["z"], dtype), delta_bias=prm["delta_bias"] if use_bias else None,
                            delta_softplus=softplus)
        torch.cuda.synchronize()
        yr = oracle.state_update(state=ref, x=st["x"], delta=st["delta"], A=d["A"], B=st["B"], C=st["C"],
                                 D=d["D"], z=st["z"], delta_bias=bias if use_bias else None,
                                 delta_softplus=softplus, dtype=dtype)
        tag = f"{regime}/{dtype} step {s}"
        assert rel_err(to_host64(y), yr) <= TOL[dtype], tag
        assert rel_err(to_host64(state_t), ref) <= TOL[dtype], tag
        if regime == "zero":
            assert torch.equal(state_t, before), f"{tag}: state changed under delta = 0"


@pytest.mark.parametrize("regime,softplus", [("large", True), ("mixed", False), ("zero", False)])
def test_ssd_large_decay(regime, softplus):
    """Mamba-2 SSD with |delta A| up to several hundred inside a 128-token block
    (A per head down to -16), across block boundaries, from a random state."""
    ms = _ms()
    batch, L, H = 2, 300, 4
    seed = 7400 + ("large", "mixed", "zero").index(regime)
    inp = make_ssd_inputs(SSD, batch=batch, seqlen=L, nheads=H, seed=seed)
    inp["dt"] = make_delta_regime((batch, L, H), regime, "bf16", seed + 1)
    h0 = make_ssd_state(batch, H, seed=seed + 2)
    dev = {k: to_device(inp[k], "bf16") for k in ("x", "dt", "B", "C", "z")}
    dev |= {k: to_device(inp[k], "f32") for k in ("A", "D")}
    y, hT = ms.ssd_fwd(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"], D=dev["D"], z=dev["z"], dt_bias=None,
                       dt_softplus=softplus, initial_state=to_device(h0, "f32"))
    y, hT = to_host64(y), to_host64(hT)
    yr, hr = oracle.ssd_scan(x=inp["x"], dt=inp["dt"], A=inp["A"], B=inp["B"], C=inp["C"], D=inp["D"], z=inp["z"],
                             dt_bias=None, dt_softplus=softplus, dtype="bf16", h0=h0.reshape(batch * H, 64, 128))
    assert np.isfinite(y).all() and np.isfinite(hT).all()
    assert rel_err(y, yr) <= TOL["bf16"], regime
    assert rel_err(hT, hr.reshape(hT.shape)) <= TOL["bf16"], regime
