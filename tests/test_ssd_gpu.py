"""GPU parity of the Mamba-2 chunked SSD forward (tcgen05 tensor cores)
against the fp64 oracle's recurrent form.

Bar: max|y - y_ref| / max|y_ref| <= 5e-3 (bf16 inputs, fp32 accumulation, the
block operands M' and the passed state rounded to bf16 for the tensor
cores), and the same on the final state. The kernel works in blocks of 128
tokens, so the lengths below cover one token, a single partial block, exact
blocks, a ragged last block and many blocks.
"""
import numpy as np
import pytest

import oracle
from selective_state_space_27_b200.inputs import SSD_WORKLOADS, make_ssd_inputs, make_ssd_state
from tests.gpu_util import TOL, rel_err, to_device, to_host64

pytestmark = pytest.mark.gpu

SMALL = SSD_WORKLOADS["ssd_small"]
LAYER = SSD_WORKLOADS["mamba2_layer_d2048"]


def _ms():
    import selective_state_space_27_b200 as ms
    return ms


def _dev(inp):
    return {k: to_device(inp[k], "bf16") for k in ("x", "dt", "B", "C", "z")} | \
        {k: to_device(inp[k], "f32") for k in ("A", "D", "dt_bias")}


def _oracle(inp, *, use_z=True, use_D=True, use_bias=True, softplus=True, pairs=None, h0=None):
    return oracle.ssd_scan(x=inp["x"], dt=inp["dt"], A=inp["A"], B=inp["B"], C=inp["C"],
                           D=inp["D"] if use_D else None, z=inp["z"] if use_z else None,
                           dt_bias=inp["dt_bias"] if use_bias else None, dt_softplus=softplus, dtype="bf16",
                           pairs=pairs, h0=h0)


def _run(dev, *, use_z=True, use_D=True, use_bias=True, softplus=True, h0=None):
    ms = _ms()
    y, hT = ms.ssd_fwd(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"], D=dev["D"] if use_D else None,
                       z=dev["z"] if use_z else None, dt_bias=dev["dt_bias"] if use_bias else None,
                       dt_softplus=softplus, initial_state=h0)
    return to_host64(y), to_host64(hT)


@pytest.mark.parametrize("batch,L,nheads,ngroups", [
    (1, 1, 1, 1), (1, 77, 2, 1), (2, 128, 2, 2), (1, 129, 3, 1), (2, 300, 4, 1), (1, 1000, 4, 2),
])
def test_ssd_matches_oracle(batch, L, nheads, ngroups):
    """Lengths from one token to many blocks (ragged and exact), one or two
    groups of B and C, gate, skip and biased softplus step."""
    inp = make_ssd_inputs(SMALL, batch=batch, seqlen=L, nheads=nheads, ngroups=ngroups, seed=3000 + L + nheads)
    y, hT = _run(_dev(inp))
    yr, hr = _oracle(inp)
    assert rel_err(y, yr) <= TOL["bf16"]
    assert rel_err(hT, hr) <= TOL["bf16"]


@pytest.mark.parametrize("use_z,use_D,use_bias,softplus", [
    (False, False, False, False), (False, True, True, True), (True, False, True, True), (True, True, False, True),
])
def test_ssd_optional_terms(use_z, use_D, use_bias, softplus):
    """Each optional term off in turn (no gate, no skip, no bias, raw step),
    from a nonzero initial state."""
    inp = make_ssd_inputs(SMALL, batch=2, seqlen=260, nheads=2, seed=3100)
    if not softplus:
        # a raw step must stay positive for a decaying state: use |dt_raw| / 8
        from selective_state_space_27_b200.inputs import bf16_bits_from_f32, f32_from_bf16_bits
        inp["dt"] = bf16_bits_from_f32(np.abs(f32_from_bf16_bits(inp["dt"])) / 8.0)
    h0 = make_ssd_state(2, 2, seed=3101)
    kw = dict(use_z=use_z, use_D=use_D, use_bias=use_bias, softplus=softplus)
    y, hT = _run(_dev(inp), h0=to_device(h0, "f32"), **kw)
    yr, hr = _oracle(inp, h0=h0.reshape(4, 64, 128), **kw)
    assert rel_err(y, yr) <= TOL["bf16"]
    assert rel_err(hT, hr.reshape(hT.shape)) <= TOL["bf16"]


def test_ssd_strided_views():
    """x, z and y as head slices of wider token rows, and B, C as slices of a
    shared (B | C) buffer, the way a fused input projection lays them out."""
    import torch
    ms = _ms()
    inp = make_ssd_inputs(SMALL, batch=2, seqlen=200, nheads=2, seed=3200)
    dev = _dev(inp)
    bc = torch.cat([dev["B"], dev["C"]], dim=3)             # (batch, L, 1, 256)
    B = bc[..., :128]
    C = bc[..., 128:]
    wide = torch.zeros((2, 200, 3, 64), dtype=torch.bfloat16, device="cuda")
    wide[:, :, 1:] = dev["x"]
    x = wide[:, :, 1:]
    yw = torch.zeros((2, 200, 5, 64), dtype=torch.bfloat16, device="cuda")
    y_out = yw[:, :, 2:4]
    y, hT = ms.ssd_fwd(x, dev["dt"], dev["A"], B.reshape(2, 200, 1, 128), C.reshape(2, 200, 1, 128),
                       D=dev["D"], z=dev["z"], dt_bias=dev["dt_bias"], out=y_out)
    torch.cuda.synchronize()
    yr, hr = _oracle(inp)
    assert rel_err(to_host64(y_out), yr) <= TOL["bf16"]
    assert rel_err(to_host64(hT), hr) <= TOL["bf16"]
    assert float(yw[:, :, :2].abs().max()) == 0.0 and float(yw[:, :, 4:].abs().max()) == 0.0


def test_ssd_continues_from_final_state():
    """Two calls, the second from the first's final state, equal one call
    over the whole sequence (state passing between blocks)."""
    inp = make_ssd_inputs(SMALL, batch=1, seqlen=400, nheads=2, seed=3300)
    dev = _dev(inp)
    ms = _ms()
    y, hT = ms.ssd_fwd(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"], D=dev["D"], z=dev["z"],
                       dt_bias=dev["dt_bias"])
    cut = 173
    part = {k: (v[:, :cut].contiguous() if k in ("x", "dt", "B", "C", "z") else v) for k, v in dev.items()}
    rest = {k: (v[:, cut:].contiguous() if k in ("x", "dt", "B", "C", "z") else v) for k, v in dev.items()}
    y1, h1 = ms.ssd_fwd(part["x"], part["dt"], part["A"], part["B"], part["C"], D=part["D"], z=part["z"],
                        dt_bias=part["dt_bias"])
    y2, h2 = ms.ssd_fwd(rest["x"], rest["dt"], rest["A"], rest["B"], rest["C"], D=rest["D"], z=rest["z"],
                        dt_bias=rest["dt_bias"], initial_state=h1)
    yr, hr = _oracle(inp)
    import torch
    assert rel_err(to_host64(torch.cat([y1, y2], dim=1)), yr) <= TOL["bf16"]
    assert rel_err(to_host64(h2), hr) <= TOL["bf16"]
    assert rel_err(to_host64(y), yr) <= TOL["bf16"]


def test_ssd_mamba2_layer_sampled_heads():
    """The Mamba-2 layer of batch 4 x 8192 tokens x 64 heads (d_inner 4096,
    d_state 128), in the launch configuration the benchmark times; the oracle
    checks a seeded sample of (batch, head) pairs in full (every token, every
    channel) and the final state of each."""
    inp = make_ssd_inputs(LAYER)
    y, hT = _run(_dev(inp))
    g = np.random.default_rng(7)
    n = LAYER.batch * LAYER.nheads
    pairs = sorted(set(g.choice(n, size=6, replace=False).tolist()) | {0, n - 1})
    yr, hr = _oracle(inp, pairs=pairs)
    for k, pr in enumerate(pairs):
        b, h = divmod(pr, LAYER.nheads)
        assert rel_err(y[b, :, h, :], yr[k]) <= TOL["bf16"], pr
        assert rel_err(hT[b, h], hr[k]) <= TOL["bf16"], pr
    assert np.isfinite(y).all() and np.isfinite(hT).all()


def test_ssd_rejects_unsupported_arguments():
    """float32 inputs, token strides that are not multiples of 8 elements and
    nheads not a multiple of ngroups are refused before any launch."""
    import torch
    ms = _ms()
    inp = make_ssd_inputs(SMALL, batch=1, seqlen=64, nheads=2, seed=3400)
    dev = _dev(inp)
    with pytest.raises(ms.MambaScanError) as ei:
        ms.ssd_fwd(dev["x"].float(), dev["dt"].float(), dev["A"], dev["B"].float(), dev["C"].float(),
                   out=torch.empty((1, 64, 2, 64), device="cuda"))
    assert ei.value.status == 2
    wide = torch.zeros((1, 64, 130), dtype=torch.bfloat16, device="cuda")   # token stride 130
    x_odd = wide[:, :, :128].unflatten(2, (2, 64))                         # strides (8320, 130, 64, 1)
    with pytest.raises(ms.MambaScanError) as ei:
        ms.ssd_fwd(x_odd, dev["dt"], dev["A"], dev["B"], dev["C"])
    assert ei.value.status == 3
    with pytest.raises(ms.MambaScanError) as ei:
        ms.ssd_fwd(dev["x"], dev["dt"], dev["A"], torch.cat([dev["B"]] * 4, dim=2)[:, :, :3].contiguous(),
                   torch.cat([dev["C"]] * 4, dim=2)[:, :, :3].contiguous())
    assert ei.value.status == 1


def test_ssd_one_group_per_head():
    """ngroups = nheads: every head reads its own B and C."""
    inp = make_ssd_inputs(SMALL, batch=2, seqlen=333, nheads=4, ngroups=4, seed=3500)
    y, hT = _run(_dev(inp))
    yr, hr = _oracle(inp)
    assert rel_err(y, yr) <= TOL["bf16"]
    assert rel_err(hT, hr) <= TOL["bf16"]


def test_ssd_mamba2_layer_from_initial_state():
    """The full Mamba-2 layer continued from a seeded nonzero state; sampled
    (batch, head) pairs against the oracle started from the same state."""
    import torch
    inp = make_ssd_inputs(LAYER, seed=LAYER.seed + 7)
    h0 = make_ssd_state(LAYER.batch, LAYER.nheads, seed=3600)
    y, hT = _run(_dev(inp), h0=torch.from_numpy(h0).cuda())
    pairs = [3, 77, 200, LAYER.batch * LAYER.nheads - 1]
    yr, hr = _oracle(inp, pairs=pairs, h0=h0.reshape(-1, 64, 128)[pairs])
    for k, pr in enumerate(pairs):
        b, h = divmod(pr, LAYER.nheads)
        assert rel_err(y[b, :, h, :], yr[k]) <= TOL["bf16"], pr
        assert rel_err(hT[b, h], hr[k]) <= TOL["bf16"], pr


def test_ssd_batch_slices():
    """x, dt, B, C, z and y as every other batch entry of larger tensors
    (batch strides twice the dense ones)."""
    import torch
    ms = _ms()
    inp = make_ssd_inputs(SMALL, batch=2, seqlen=150, nheads=2, seed=3700)
    dev = _dev(inp)
    big = {}
    for k in ("x", "dt", "B", "C", "z"):
        t = dev[k]
        b2 = torch.zeros((4,) + tuple(t.shape[1:]), dtype=t.dtype, device="cuda")
        b2[0::2] = t
        big[k] = b2[0::2]
    ybig = torch.zeros((4,) + tuple(dev["x"].shape[1:]), dtype=torch.bfloat16, device="cuda")
    y_out = ybig[0::2]
    _, hT = ms.ssd_fwd(big["x"], big["dt"], dev["A"], big["B"], big["C"], D=dev["D"], z=big["z"],
                       dt_bias=dev["dt_bias"], out=y_out)
    yr, hr = _oracle(inp)
    assert rel_err(to_host64(y_out), yr) <= TOL["bf16"]
    assert rel_err(to_host64(hT), hr) <= TOL["bf16"]
    assert float(ybig[1::2].abs().max()) == 0.0


@pytest.mark.parametrize("block", [1, 3])
def test_ssd_timeout_path(block):
    """The kernel's bounded pipeline waits: with block `block - 1`'s loads
    withheld (the fault-injection hook of ms_ssd_args) and a 2 ms wait limit,
    the wait for those loads runs out, the status word reads MS_ERR_TIMEOUT,
    the CTA drains the loads and products it did issue and exits, and the
    context stays usable: a normal call straight after it matches the oracle."""
    import torch
    ms = _ms()
    inp = make_ssd_inputs(SMALL, batch=2, seqlen=700, nheads=2, seed=3300 + block)
    dev = _dev(inp)
    ws = torch.zeros(ms.SSD_WORKSPACE_BYTES, dtype=torch.uint8, device="cuda")
    ms.ssd_fwd(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"], D=dev["D"], z=dev["z"], dt_bias=dev["dt_bias"],
               workspace=ws, check=False, wait_limit_us=2000, withhold_block=block)
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32)[0].item()) == 5   # MS_ERR_TIMEOUT
    with pytest.raises(ms.MambaScanError) as ei:
        ms.ssd_check(ws)
    assert ei.value.status == 5
    y, hT = ms.ssd_fwd(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"], D=dev["D"], z=dev["z"],
                       dt_bias=dev["dt_bias"], workspace=ws)
    yr, hr = _oracle(inp)
    assert rel_err(to_host64(y), yr) <= TOL["bf16"]
    assert rel_err(to_host64(hT), hr) <= TOL["bf16"]


def _ssd_ws_bytes(dev):
    import ctypes
    ms = _ms()
    args = ms.build_ssd_args(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"], dev["x"])
    n = ctypes.c_size_t(0)
    assert ms.load_library().mamba_ssd_workspace_size(ctypes.byref(args), ctypes.byref(n)) == 0
    return n.value


@pytest.mark.parametrize("batch,L,nheads,ngroups", [(2, 1000, 80, 2), (1, 1300, 150, 1)])
def test_ssd_persistent_schedule(batch, L, nheads, ngroups):
    """More (batch, head) pairs than SMs, leaving the last wave partly empty:
    the call takes the persistent schedule (a larger workspace), which cuts
    the chunks of all pairs evenly over the SMs and hands a pair's state from
    one CTA to the next. Every pair against the oracle, from an initial state."""
    import torch
    inp = make_ssd_inputs(SMALL, batch=batch, seqlen=L, nheads=nheads, ngroups=ngroups, seed=3800 + nheads)
    dev = _dev(inp)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    if batch * nheads <= sms or (batch * nheads) % sms == 0:
        pytest.skip("the shape fills whole waves of this device")
    assert _ssd_ws_bytes(dev) > _ms().SSD_WORKSPACE_BYTES
    h0 = make_ssd_state(batch, nheads, seed=3801)
    y, hT = _run(dev, h0=torch.from_numpy(h0).cuda())
    yr, hr = _oracle(inp, h0=h0.reshape(-1, 64, 128))
    assert rel_err(y, yr) <= TOL["bf16"]
    assert rel_err(hT, hr.reshape(hT.shape)) <= TOL["bf16"]
    # the same call with the smallest workspace runs one CTA per pair: same result
    ws = torch.zeros(_ms().SSD_WORKSPACE_BYTES, dtype=torch.uint8, device="cuda")
    y2, hT2 = _ms().ssd_fwd(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"], D=dev["D"], z=dev["z"],
                            dt_bias=dev["dt_bias"], initial_state=torch.from_numpy(h0).cuda(), workspace=ws)
    assert rel_err(to_host64(y2), yr) <= TOL["bf16"]
    assert rel_err(to_host64(hT2), hr.reshape(hT.shape)) <= TOL["bf16"]


def test_ssd_persistent_on_side_stream():
    """The persistent schedule on a stream other than the current one, with
    its hand-over workspace allocated by the binding, while the current stream
    churns the allocator."""
    import torch
    ms = _ms()
    inp = make_ssd_inputs(SMALL, batch=2, seqlen=700, nheads=80, seed=3950)
    dev = _dev(inp)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    if 160 <= sms or 160 % sms == 0:
        pytest.skip("the shape fills whole waves of this device")
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    y, hT = ms.ssd_fwd(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"], D=dev["D"], z=dev["z"],
                       dt_bias=dev["dt_bias"], stream=side, check=False)
    junk = [torch.full((1 << 16,), 7, dtype=torch.uint8, device="cuda") for _ in range(64)]
    del junk
    side.synchronize()
    torch.cuda.synchronize()
    yr, hr = _oracle(inp)
    assert rel_err(to_host64(y), yr) <= TOL["bf16"]
    assert rel_err(to_host64(hT), hr) <= TOL["bf16"]


def test_ssd_persistent_timeout_path():
    """The persistent schedule's bounded waits: with block 2's loads withheld
    and a 2 ms limit, every CTA gives up, still raises its hand-over flag (so
    no CTA waits on it for longer than the limit), drains and exits; the status
    word reads MS_ERR_TIMEOUT and a normal call straight after matches the
    oracle."""
    import torch
    ms = _ms()
    inp = make_ssd_inputs(SMALL, batch=2, seqlen=600, nheads=80, seed=3900)
    dev = _dev(inp)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    if 160 <= sms or 160 % sms == 0:
        pytest.skip("the shape fills whole waves of this device")
    nbytes = _ssd_ws_bytes(dev)
    assert nbytes > ms.SSD_WORKSPACE_BYTES
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    ms.ssd_fwd(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"], D=dev["D"], z=dev["z"], dt_bias=dev["dt_bias"],
               workspace=ws, check=False, wait_limit_us=2000, withhold_block=3)
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32)[0].item()) == 5   # MS_ERR_TIMEOUT
    y, hT = ms.ssd_fwd(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"], D=dev["D"], z=dev["z"],
                       dt_bias=dev["dt_bias"], workspace=ws)
    yr, hr = _oracle(inp)
    assert rel_err(to_host64(y), yr) <= TOL["bf16"]
    assert rel_err(to_host64(hT), hr) <= TOL["bf16"]


def test_ssd_withheld_block_past_the_end_is_harmless():
    """A withheld block index beyond the sequence changes nothing."""
    inp = make_ssd_inputs(SMALL, batch=1, seqlen=200, nheads=2, seed=3400)
    dev = _dev(inp)
    ms = _ms()
    y, hT = ms.ssd_fwd(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"], D=dev["D"], z=dev["z"],
                       dt_bias=dev["dt_bias"], withhold_block=50, wait_limit_us=100000)
    yr, hr = _oracle(inp)
    assert rel_err(to_host64(y), yr) <= TOL["bf16"]
    assert rel_err(to_host64(hT), hr) <= TOL["bf16"]
