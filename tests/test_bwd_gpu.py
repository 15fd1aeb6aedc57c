"""GPU parity of the scan backward (gradients for sum(y dy) + sum(h_T dh_T))
against the fp64 oracle, whose gradients are pinned to finite differences.

Bar: max|g - g_ref| / max|g_ref| per gradient tensor <= 2e-4 with float32
inputs; with bfloat16 inputs <= 5e-3 for du, ddelta, dz (stored in bf16) and
<= 1e-3 for the float32 reductions (dA, dB, dC, dD, ddelta_bias, dh0), whose
summation order differs (atomics)."""
import numpy as np
import pytest

import oracle
from selective_state_space_27_b200.inputs import SCAN_WORKLOADS, bf16_bits_from_f32, make_scan_inputs
from tests.gpu_util import device_inputs, rel_err, to_device, to_host64

pytestmark = pytest.mark.gpu

LAYER = SCAN_WORKLOADS["mamba130m_layer"]
ROUNDED = ("du", "ddelta", "dz")


def _tol(dtype, name):
    if dtype == "f32":
        return 2e-4
    return 5e-3 if name in ROUNDED else 1e-3


def _check(inp, *, seed, use_h0=True, use_dhT=True, softplus=True, checkpointed=False):
    import torch
    import selective_state_space_27_b200 as ms
    dt = inp["dtype"]
    g = np.random.default_rng(seed)
    batch, dim, L, N = inp["batch"], inp["dim"], inp["seqlen"], inp["dstate"]
    dy = g.normal(size=(batch, dim, L)).astype(np.float32)
    dy_store = dy if dt == "f32" else bf16_bits_from_f32(dy)
    h0 = g.normal(size=(batch, dim, N)).astype(np.float32) if use_h0 else None
    dhT = g.normal(size=(batch, dim, N)).astype(np.float32) if use_dhT else None
    dev = device_inputs(inp)
    h0_dev = None if h0 is None else torch.from_numpy(h0).cuda()
    ckpt = None
    if checkpointed:
        # the forward keeps the states of every 8th step; its y and final state match the plain forward's
        # (bit for bit when the automatic plan is the same sequential kernel; a shape the planner gives
        # to a chunked kernel differs by rounding only)
        ckpt = torch.full((ms.checkpoint_numel(dev["u"], dev["B"]),), float("nan"), device="cuda")
        y_ck, hT_ck = ms.scan_fwd(dev["u"], dev["delta"], dev["A"], dev["B"], dev["C"], D=dev["D"], z=dev["z"],
                                  delta_bias=dev["delta_bias"], delta_softplus=softplus, initial_state=h0_dev,
                                  checkpoints=ckpt)
        y_pl, hT_pl = ms.scan_fwd(dev["u"], dev["delta"], dev["A"], dev["B"], dev["C"], D=dev["D"], z=dev["z"],
                                  delta_bias=dev["delta_bias"], delta_softplus=softplus, initial_state=h0_dev)
        torch.cuda.synchronize()
        fwd_tol = 1e-4 if dt == "f32" else 5e-3
        assert rel_err(to_host64(y_ck), to_host64(y_pl)) <= fwd_tol
        assert rel_err(to_host64(hT_ck), to_host64(hT_pl)) <= fwd_tol
    out = ms.scan_bwd(dev["u"], dev["delta"], dev["A"], dev["B"], dev["C"], to_device(dy_store, dt), D=dev["D"],
                      z=dev["z"], delta_bias=dev["delta_bias"], delta_softplus=softplus, initial_state=h0_dev,
                      dfinal_state=None if dhT is None else torch.from_numpy(dhT).cuda(), checkpoints=ckpt)
    torch.cuda.synchronize()
    ref = oracle.scan_bwd(u=inp["u"], delta=inp["delta"], A=inp["A"], B=inp["B"], C=inp["C"], dy=dy_store,
                          D=inp["D"], z=inp["z"], delta_bias=inp["delta_bias"], delta_softplus=softplus, h0=h0,
                          dhT=dhT)
    names = {"du": "du", "ddelta": "ddelta", "dz": "dz", "dA": "dA", "dB": "dB", "dC": "dC", "dD": "dD",
             "ddelta_bias": "ddelta_bias", "dinitial_state": "dh0"}
    absent = {"dz": inp["z"] is None, "dD": inp["D"] is None, "ddelta_bias": inp["delta_bias"] is None}
    for k, rk in names.items():
        if absent.get(k, False):       # no input, no gradient
            assert out[k] is None
            continue
        got = to_host64(out[k])
        assert np.isfinite(got).all(), k
        err = rel_err(got, ref[rk])
        assert err <= _tol(dt, k), f"{k}: {err:.2e}"


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("batch,dim,N,L", [(1, 3, 16, 1), (2, 37, 16, 33), (2, 20, 5, 100), (1, 16, 16, 256),
                                           (3, 50, 8, 17)])
def test_scan_bwd_matches_oracle(dtype, batch, dim, N, L):
    """Ragged rows (dim not a multiple of the CTA's 16 rows), ragged lengths
    (partial last chunk), dstate < 16, with z, D, delta_bias, h0 and dh_T."""
    inp = make_scan_inputs(LAYER, batch=batch, dim=dim, dstate=N, seqlen=L, dtype=dtype, seed=4100 + dim + L)
    _check(inp, seed=4200 + L)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("batch,dim,N,L", [(1, 3, 16, 1), (2, 37, 16, 33), (2, 20, 5, 100), (1, 16, 16, 256),
                                           (2, 40, 16, 1030)])
def test_scan_bwd_checkpointed_matches_oracle(dtype, batch, dim, N, L):
    """The training pair: the forward keeps the 8-step checkpoints (its y and
    final state unchanged), the backward recomputes from them. Ragged rows and
    lengths (partial last 8- and 16-step chunks), dstate < 16."""
    inp = make_scan_inputs(LAYER, batch=batch, dim=dim, dstate=N, seqlen=L, dtype=dtype, seed=4150 + dim + L)
    _check(inp, seed=4250 + L, checkpointed=True)


def test_scan_checkpoint_errors():
    """A short checkpoint buffer is refused by both calls; a forced segmented
    (chunked) plan cannot write checkpoints."""
    import torch
    import selective_state_space_27_b200 as ms
    inp = make_scan_inputs(LAYER, batch=1, dim=8, seqlen=64, dtype="f32", seed=4400)
    dev = device_inputs(inp)
    short = torch.zeros(ms.checkpoint_numel(dev["u"], dev["B"]) - 1, device="cuda")
    with pytest.raises(ms.MambaScanError, match="MS_ERR_WORKSPACE"):
        ms.scan_fwd(dev["u"], dev["delta"], dev["A"], dev["B"], dev["C"], D=dev["D"], z=dev["z"],
                    delta_bias=dev["delta_bias"], checkpoints=short)
    dy = torch.zeros_like(dev["u"])
    with pytest.raises(ms.MambaScanError, match="MS_ERR_WORKSPACE"):
        ms.scan_bwd(dev["u"], dev["delta"], dev["A"], dev["B"], dev["C"], dy, D=dev["D"], z=dev["z"],
                    delta_bias=dev["delta_bias"], checkpoints=short)
    full = torch.zeros(ms.checkpoint_numel(dev["u"], dev["B"]), device="cuda")
    with pytest.raises(ms.MambaScanError, match="MS_ERR_UNSUPPORTED"):
        ms.scan_fwd(dev["u"], dev["delta"], dev["A"], dev["B"], dev["C"], D=dev["D"], z=dev["z"],
                    delta_bias=dev["delta_bias"], force_segments=2, checkpoints=full)


@pytest.mark.parametrize("softplus", [True, False])
def test_scan_bwd_without_optional_terms(softplus):
    """No z, D, bias, h0 or dh_T (and raw delta with softplus off)."""
    inp = make_scan_inputs(LAYER, batch=2, dim=24, seqlen=70, dtype="f32", seed=4300)
    inp["z"], inp["D"], inp["delta_bias"] = None, None, None
    if not softplus:
        inp["delta"] = np.abs(inp["delta"]) * 0.1
    _check(inp, seed=4301, use_h0=False, use_dhT=False, softplus=softplus)


@pytest.mark.slow
@pytest.mark.parametrize("checkpointed", [False, True])
def test_scan_bwd_mamba130m_layer_full(checkpointed):
    """The Mamba-130M-shaped layer (bf16, gate), every row and gradient; with
    checkpoints from the forward, whose persistent schedule here cuts units
    between CTAs (the carry hand-over and the checkpoint stores meet)."""
    _check(make_scan_inputs(LAYER), seed=4400, checkpointed=checkpointed)
