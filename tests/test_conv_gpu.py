"""GPU parity of the convolution prologue (causal depthwise conv + SiLU fused
in front of the scan, and its decode step) against the fp64 oracle.

Bar as for the scan: max|y - y_ref| / max|y_ref| <= 1e-4 (float32 inputs) or
5e-3 (bfloat16 inputs), and the same on the final state; the convolution state
after a decode step must equal the oracle's exactly (it holds input values).
"""
import numpy as np
import pytest

import oracle
from selective_state_space_27_b200.inputs import (SCAN_WORKLOADS, f32_from_bf16_bits, make_conv_params,
                                                  make_conv_state, make_scan_inputs)
from tests.gpu_util import TOL, device_inputs, rel_err, to_device, to_host64

pytestmark = pytest.mark.gpu

LAYER = SCAN_WORKLOADS["mamba130m_layer"]


def _ms():
    import selective_state_space_27_b200 as ms
    return ms


def _conv_configs():
    # the fused variants are compiled for the 2-I/O-warp kernels (6 warps) with 2 or 4 lanes per row
    return [(c, lanes, warps) for c, lanes, _, warps, kind in _ms().scan_configs()
            if kind == 1 and lanes in (2, 4) and warps == 6]


def _oracle(inp, conv, *, silu=True, rows=None, h0=None):
    return oracle.conv_scan(x=inp["u"], conv_w=conv["conv_w"], conv_b=conv["conv_b"], conv_silu=silu,
                            delta=inp["delta"], A=inp["A"], B=inp["B"], C=inp["C"], D=inp["D"], z=inp["z"],
                            delta_bias=inp["delta_bias"], dtype=inp["dtype"], rows=rows, h0=h0)


def _run(dev, conv_t, *, silu=True, plan=None, h0=None):
    import torch
    ms = _ms()
    y, hT = ms.conv_scan_fwd(dev["u"], conv_t["conv_w"], dev["delta"], dev["A"], dev["B"], dev["C"], D=dev["D"],
                             z=dev["z"], delta_bias=dev["delta_bias"], conv_bias=conv_t["conv_b"],
                             conv_silu=silu, initial_state=h0, plan=plan)
    torch.cuda.synchronize()
    return to_host64(y), to_host64(hT)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("batch,dim,N,L,width,silu,offset", [
    (1, 3, 16, 1, 4, True, 0), (2, 37, 16, 33, 4, True, 0), (2, 130, 16, 1000, 4, True, 0),
    (3, 20, 5, 97, 3, False, 0), (1, 64, 16, 64, 1, True, 0), (2, 70, 16, 255, 2, True, 1),
    (1, 9, 8, 31, 4, False, 3),
])
def test_conv_scan_matches_oracle(dtype, batch, dim, N, L, width, silu, offset):
    """Every configuration that fuses the prologue, and the automatic plan, on
    ragged rows and lengths, widths 1-4, with and without the SiLU, an initial
    state, and (offset > 0) rows that are not 16-byte aligned."""
    import torch
    ms = _ms()
    inp = make_scan_inputs(LAYER, batch=batch, dim=dim, dstate=N, seqlen=L + offset, dtype=dtype,
                           seed=2100 + dim + L + width)
    dev = device_inputs(inp)
    if offset:
        for k in ("u", "delta", "z", "B", "C"):
            dev[k] = dev[k][..., offset:]
            inp[k] = np.ascontiguousarray(inp[k][..., offset:])
        inp["seqlen"] = L
    conv = make_conv_params(dim, width, seed=2200 + width)
    conv_t = {k: to_device(v, "f32") for k, v in conv.items()}
    h0 = np.random.default_rng(dim).normal(size=(batch, dim, N)).astype(np.float32)
    h0_t = torch.from_numpy(h0).cuda()
    yr, hr = _oracle(inp, conv, silu=silu, h0=h0.reshape(-1, N))
    plans = [None] + [ms.ScanPlan(config=c, warps_per_cta=w, segments=1) for c, _, w in _conv_configs()]
    for plan in plans:
        y, hT = _run(dev, conv_t, silu=silu, plan=plan, h0=h0_t)
        tag = "auto" if plan is None else f"config {plan.config}"
        assert rel_err(y, yr) <= TOL[dtype], tag
        assert rel_err(hT, hr) <= TOL[dtype], tag


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_conv_scan_persistent_schedule(dtype):
    """The prologue under the persistent schedule: every configuration that
    fuses it at CTA counts from 1 to one per unit, including counts that cut
    units between CTAs (the convolution's look-back then starts a piece in the
    middle of a row)."""
    import torch
    ms = _ms()
    batch, dim, N, L = 2, 100, 16, 300
    inp = make_scan_inputs(LAYER, batch=batch, dim=dim, dstate=N, seqlen=L, dtype=dtype, seed=2950)
    dev = device_inputs(inp)
    conv = make_conv_params(dim, 4, seed=2951)
    conv_t = {k: to_device(v, "f32") for k, v in conv.items()}
    h0 = np.random.default_rng(2952).normal(size=(batch, dim, N)).astype(np.float32)
    h0_t = torch.from_numpy(h0).cuda()
    yr, hr = _oracle(inp, conv, h0=h0.reshape(-1, N))
    for c, lanes, w in _conv_configs():
        rows = 128 // lanes
        units = batch * ((dim + rows - 1) // rows)
        for ctas in sorted({1, 2, 3, max(1, units // 2), max(1, units - 1), units}):
            plan = ms.ScanPlan(config=c, warps_per_cta=w, segments=1, ctas=ctas)
            y, hT = _run(dev, conv_t, plan=plan, h0=h0_t)
            tag = f"config {c}, {ctas} CTAs of {units} units"
            assert rel_err(y, yr) <= TOL[dtype], tag
            assert rel_err(hT, hr) <= TOL[dtype], tag


def test_conv_scan_persistent_on_side_stream():
    """The persistent schedule on a stream other than the current one, with
    the hand-over workspace allocated by the binding: work queued meanwhile on
    the current stream must not receive the workspace's memory while the scan
    still uses it."""
    import torch
    ms = _ms()
    batch, dim, N, L = 2, 100, 16, 3000
    inp = make_scan_inputs(LAYER, batch=batch, dim=dim, dstate=N, seqlen=L, seed=2960)
    dev = device_inputs(inp)
    conv = make_conv_params(dim, 4, seed=2961)
    conv_t = {k: to_device(v, "f32") for k, v in conv.items()}
    c, lanes, w = _conv_configs()[0]
    units = batch * ((dim + 128 // lanes - 1) // (128 // lanes))
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    y, hT = ms.conv_scan_fwd(dev["u"], conv_t["conv_w"], dev["delta"], dev["A"], dev["B"], dev["C"], D=dev["D"],
                             z=dev["z"], delta_bias=dev["delta_bias"], conv_bias=conv_t["conv_b"], stream=side,
                             plan=ms.ScanPlan(config=c, warps_per_cta=w, segments=1, ctas=max(1, units - 1)))
    junk = [torch.full((1 << 16,), 7, dtype=torch.uint8, device="cuda") for _ in range(64)]
    del junk
    side.synchronize()
    torch.cuda.synchronize()
    yr, hr = _oracle(inp, conv)
    assert rel_err(to_host64(y), yr) <= TOL["bf16"]
    assert rel_err(to_host64(hT), hr) <= TOL["bf16"]


def test_conv_scan_mamba130m_layer_full():
    """The Mamba-130M-shaped layer (bf16, gate) with a width-4 prologue, every row."""
    inp = make_scan_inputs(LAYER)
    conv = make_conv_params(inp["dim"], 4)
    dev = device_inputs(inp)
    y, hT = _run(dev, {k: to_device(v, "f32") for k, v in conv.items()})
    yr, hr = _oracle(inp, conv)
    assert rel_err(y, yr) <= TOL["bf16"] and rel_err(hT, hr) <= TOL["bf16"]


def test_conv_scan_rejects_unfusable_plans():
    """Chunked configurations and 8/16 lanes per row cannot fuse the prologue;
    width 5 and forced segments are refused before any launch."""
    import torch
    ms = _ms()
    inp = make_scan_inputs(LAYER, batch=1, dim=16, seqlen=64, seed=2300)
    dev = device_inputs(inp)
    conv_t = {k: to_device(v, "f32") for k, v in make_conv_params(16, 4).items()}
    for cfg, lanes, _, warps, kind in ms.scan_configs():
        if kind == 1 and lanes in (2, 4):
            continue
        with pytest.raises(ms.MambaScanError) as ei:
            ms.conv_scan_fwd(dev["u"], conv_t["conv_w"], dev["delta"], dev["A"], dev["B"], dev["C"],
                             plan=ms.ScanPlan(config=cfg, warps_per_cta=warps, segments=1))
        assert ei.value.status == 2
    wide = torch.zeros((16, 5), dtype=torch.float32, device="cuda")
    with pytest.raises(ms.MambaScanError) as ei:
        ms.conv_scan_fwd(dev["u"], wide, dev["delta"], dev["A"], dev["B"], dev["C"])
    assert ei.value.status == 2


def _decode_oracle_steps(inp_steps, conv, state0, cstate0, dtype):
    state = state0.astype(np.float64).copy()
    cstate = cstate0.copy()
    ys = []
    for st in inp_steps:
        ys.append(oracle.conv_state_update(state=state, conv_state=cstate, x=st["x"], conv_w=conv["conv_w"],
                                           conv_b=conv["conv_b"], delta=st["delta"], A=st["A"], B=st["B"],
                                           C=st["C"], D=st["D"], z=st["z"], delta_bias=st["delta_bias"],
                                           dtype=dtype))
    return np.stack(ys), state, cstate


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("width", [1, 3, 4])
def test_conv_state_update_matches_oracle(dtype, width):
    """20 decode steps with the convolution prologue from a random state and
    convolution state: y every step, the final state, and the convolution
    state (exactly: it holds input values)."""
    import torch
    ms = _ms()
    batch, dim, N, steps = 3, 70, 16, 20
    g = np.random.default_rng(2400 + width)
    scan = make_scan_inputs(LAYER, batch=batch, dim=dim, dstate=N, seqlen=steps, dtype=dtype, seed=2500 + width)
    conv = make_conv_params(dim, width, seed=2600 + width)
    cstate0 = make_conv_state(batch, dim, width, dtype, seed=2700 + width)
    state0 = g.normal(size=(batch, dim, N)).astype(np.float32)
    steps_np = [dict(x=np.ascontiguousarray(scan["u"][:, :, t]), delta=np.ascontiguousarray(scan["delta"][:, :, t]),
                     B=np.ascontiguousarray(scan["B"][:, :, t]), C=np.ascontiguousarray(scan["C"][:, :, t]),
                     z=np.ascontiguousarray(scan["z"][:, :, t]), A=scan["A"], D=scan["D"],
                     delta_bias=scan["delta_bias"]) for t in range(steps)]
    cs_ref = cstate0.astype(np.float64) if dtype == "f32" else f32_from_bf16_bits(cstate0).astype(np.float64)
    yr, hr, csr = _decode_oracle_steps(steps_np, conv, state0, cs_ref, dtype)
    state = torch.from_numpy(state0.copy()).cuda()
    cstate = to_device(cstate0, dtype)
    conv_t = {k: to_device(v, "f32") for k, v in conv.items()}
    ys = []
    for st in steps_np:
        d = {k: to_device(v, dtype if k in ("x", "delta", "B", "C", "z") else "f32") for k, v in st.items()}
        ys.append(to_host64(ms.conv_state_update(state, cstate, d["x"], conv_t["conv_w"], d["delta"], d["A"],
                                                 d["B"], d["C"], D=d["D"], z=d["z"], delta_bias=d["delta_bias"],
                                                 conv_bias=conv_t["conv_b"])))
    torch.cuda.synchronize()
    assert rel_err(np.stack(ys), yr) <= TOL[dtype]
    assert rel_err(to_host64(state), hr) <= TOL[dtype]
    assert np.array_equal(to_host64(cstate), csr)


def test_decode_continues_the_fused_scan():
    """A fused scan over the first L - 5 steps (final state kept) followed by 5
    decode steps whose convolution state holds the last inputs of the prefix
    reproduces the fused scan over all L steps."""
    import torch
    ms = _ms()
    batch, dim, N, L, width, P = 2, 64, 16, 64, 4, 59
    inp = make_scan_inputs(LAYER, batch=batch, dim=dim, dstate=N, seqlen=L, dtype="f32", seed=2800)
    conv = make_conv_params(dim, width, seed=2801)
    conv_t = {k: to_device(v, "f32") for k, v in conv.items()}
    yr, hr = _oracle(inp, conv)
    pre = {k: (np.ascontiguousarray(v[..., :P]) if k in ("u", "delta", "z", "B", "C") else v) for k, v in inp.items()}
    dev = device_inputs(pre)
    y_pre, h = _run(dev, conv_t)
    state = torch.from_numpy(h.astype(np.float32)).cuda()
    cstate = torch.from_numpy(np.ascontiguousarray(inp["u"][:, :, P - width:P])).cuda()
    ys = [y_pre]
    for t in range(P, L):
        d = {k: to_device(np.ascontiguousarray(inp[k][:, :, t]), "f32") for k in ("u", "delta", "z", "B", "C")}
        y = ms.conv_state_update(state, cstate, d["u"], conv_t["conv_w"], d["delta"], to_device(inp["A"], "f32"),
                                 d["B"], d["C"], D=to_device(inp["D"], "f32"), z=d["z"],
                                 delta_bias=to_device(inp["delta_bias"], "f32"), conv_bias=conv_t["conv_b"])
        ys.append(to_host64(y)[:, :, None])
    torch.cuda.synchronize()
    assert rel_err(np.concatenate(ys, axis=2), yr) <= TOL["f32"]
    assert rel_err(to_host64(state), hr) <= TOL["f32"]
