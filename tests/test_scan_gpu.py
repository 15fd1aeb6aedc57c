"""GPU parity of the selective scan (C ABI via the binding) against the fp64 oracle.

Bar: max|y - y_ref| / max|y_ref| <= 1e-4 for float32 inputs and <= 5e-3 for
bfloat16 inputs (float32 arithmetic, bf16 output rounding), and the same bound
on the final state.
"""
import numpy as np
import pytest

from selective_state_space_27_b200.inputs import SCAN_WORKLOADS, make_scan_inputs
from tests.gpu_util import TOL, device_inputs, oracle_scan, rel_err, sample_rows, to_device, to_host64

pytestmark = pytest.mark.gpu

TINY = SCAN_WORKLOADS["s6_tiny_f32"]
LAYER = SCAN_WORKLOADS["mamba130m_layer"]


def _ms():
    import selective_state_space_27_b200 as ms
    return ms


def run_scan(inp, *, use_z=True, use_D=True, use_bias=True, softplus=True, force_segments=0,
             h0=None):
    import torch
    dev = device_inputs(inp, use_z=use_z, use_D=use_D, use_bias=use_bias)
    h0_t = None if h0 is None else torch.from_numpy(np.ascontiguousarray(h0, np.float32)).cuda()
    y, hT = _ms().scan_fwd(**dev, delta_softplus=softplus, force_segments=force_segments,
                           initial_state=h0_t)
    torch.cuda.synchronize()
    return to_host64(y), to_host64(hT)


def check(inp, *, rows=None, use_z=True, use_D=True, use_bias=True, softplus=True,
          force_segments=0, h0=None):
    y, hT = run_scan(inp, use_z=use_z, use_D=use_D, use_bias=use_bias, softplus=softplus,
                     force_segments=force_segments, h0=h0)
    h0_rows = None
    if h0 is not None:
        h0_rows = h0.reshape(-1, inp["dstate"]) if rows is None else h0.reshape(-1, inp["dstate"])[rows]
    yr, hr = oracle_scan(inp, rows=rows, use_z=use_z, use_D=use_D, use_bias=use_bias,
                         softplus=softplus, h0=h0_rows)
    L, N = inp["seqlen"], inp["dstate"]
    if rows is not None:
        y = y.reshape(-1, L)[rows]
        hT = hT.reshape(-1, N)[rows]
    tol = TOL[inp["dtype"]]
    ey, eh = rel_err(y, yr), rel_err(hT, hr)
    assert np.isfinite(y).all() and np.isfinite(hT).all()
    assert ey <= tol, f"y error {ey:.3e} > {tol}"
    assert eh <= tol, f"final state error {eh:.3e} > {tol}"
    return ey, eh


def test_tiny_f32_workload():
    inp = make_scan_inputs(TINY)
    check(inp)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("L", [1, 7, 16, 63, 64, 65, 127, 129, 1000, 2047, 2049])
def test_ragged_lengths(dtype, L):
    inp = make_scan_inputs(LAYER, batch=2, dim=37, dstate=16, seqlen=L, dtype=dtype, has_z=True,
                           seed=100 + L)
    check(inp)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("N", [1, 2, 3, 4, 8, 15, 16])
def test_state_sizes(dtype, N):
    inp = make_scan_inputs(LAYER, batch=3, dim=70, dstate=N, seqlen=300, dtype=dtype, seed=200 + N)
    check(inp)


@pytest.mark.parametrize("use_z,use_D,use_bias,softplus", [
    (False, True, True, True), (True, False, True, True), (True, True, False, True),
    (True, True, False, False), (False, False, False, False),
])
def test_optional_terms(use_z, use_D, use_bias, softplus):
    inp = make_scan_inputs(LAYER, batch=2, dim=64, seqlen=333, seed=300)
    if not softplus:
        # keep delta positive and small without softplus: use |raw| / 8 drawn from the same recipe
        from selective_state_space_27_b200.inputs import bf16_bits_from_f32, f32_from_bf16_bits
        inp["delta"] = bf16_bits_from_f32(np.abs(f32_from_bf16_bits(inp["delta"])) / 8)
    check(inp, use_z=use_z, use_D=use_D, use_bias=use_bias, softplus=softplus)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("segments", [2, 3, 7, 64])
def test_forced_segments(dtype, segments):
    inp = make_scan_inputs(LAYER, batch=2, dim=40, seqlen=4096 + 13, dtype=dtype, seed=400 + segments)
    check(inp, force_segments=segments)


def test_automatic_segments_few_rows_long_sequence():
    inp = make_scan_inputs(LAYER, batch=1, dim=16, seqlen=65536 + 5, seed=500)
    check(inp)


@pytest.mark.parametrize("segments", [0, 5])
def test_initial_state(segments):
    inp = make_scan_inputs(LAYER, batch=2, dim=33, seqlen=1500, seed=600)
    g = np.random.default_rng(601)
    h0 = g.normal(size=(2, 33, 16)).astype(np.float32)
    check(inp, h0=h0, force_segments=segments)


def _strided(a, dtype, pad):
    """Embed a (B, X, L) array in a wider buffer: batch stride grows by `pad` rows of L."""
    import torch
    t = to_device(a, dtype)
    Bn, X, L = t.shape
    big = torch.zeros((Bn, X + pad, L + 8), dtype=t.dtype, device=t.device)
    big[:, :X, :L] = t
    return big[:, :X, :L]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_strided_views(dtype):
    """Non-contiguous batch and row strides (aligned, so the vector path runs)."""
    import torch
    ms = _ms()
    inp = make_scan_inputs(LAYER, batch=3, dim=50, seqlen=640, dtype=dtype, seed=700)
    dev = device_inputs(inp)
    dev.update({k: _strided(inp[k], dtype, 3) for k in ("u", "delta", "z", "B", "C")})
    y_full = torch.zeros((3, 53, 648), dtype=dev["u"].dtype, device="cuda")
    y = y_full[:, :50, :640]
    _, hT = ms.scan_fwd(**dev, out=y)
    torch.cuda.synchronize()
    yr, hr = oracle_scan(inp)
    assert rel_err(to_host64(y), yr) <= TOL[dtype]
    assert rel_err(to_host64(hT), hr) <= TOL[dtype]
    # the padding of the output buffer is untouched
    assert float(y_full[:, 50:, :].abs().max()) == 0.0 and float(y_full[:, :, 640:].abs().max()) == 0.0


def test_misaligned_rows_use_scalar_path():
    """Row strides that break 16-byte alignment (odd L, contiguous) still match."""
    inp = make_scan_inputs(LAYER, batch=2, dim=9, seqlen=1023, seed=800)
    check(inp)


def test_deterministic():
    inp = make_scan_inputs(LAYER, batch=2, dim=64, seqlen=1024, seed=900)
    y1, h1 = run_scan(inp)
    y2, h2 = run_scan(inp)
    assert np.array_equal(y1, y2) and np.array_equal(h1, h2)


def test_mamba130m_layer_full():
    """The 130M-shaped layer workload (8, 1536, 16, 2048), every row."""
    inp = make_scan_inputs(LAYER)
    check(inp)


@pytest.mark.slow
def test_mamba1p4b_layer_sampled_rows():
    w = SCAN_WORKLOADS["mamba1p4b_layer"]
    inp = make_scan_inputs(w)
    check(inp, rows=sample_rows(w.batch, w.dim, 96, seed=1))


@pytest.mark.slow
def test_long_context_sampled_rows():
    w = SCAN_WORKLOADS["long_context_131k"]
    inp = make_scan_inputs(w)
    check(inp, rows=sample_rows(w.batch, w.dim, 24, seed=2))


@pytest.mark.slow
def test_long_context_forced_segments_sampled_rows():
    w = SCAN_WORKLOADS["long_context_131k"]
    inp = make_scan_inputs(w)
    check(inp, rows=sample_rows(w.batch, w.dim, 12, seed=3), force_segments=8)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_every_kernel_configuration(dtype):
    """Each compiled configuration, forced through mamba_scan_fwd_with_plan:
    chunked kernels at their smallest and largest CTA, with and without
    segments; sequential kernels at their fixed CTA (other shapes refused)."""
    import torch
    ms = _ms()
    # rows 16-byte aligned (every configuration can run) and a ragged last chunk
    inp = make_scan_inputs(LAYER, batch=2, dim=88, seqlen=1000, dtype=dtype, seed=1100)
    dev = device_inputs(inp)
    yr, hr = oracle_scan(inp)
    for cfg, lanes, states, max_warps, kind in ms.scan_configs():
        if kind == 1:
            for warps, segments in ((2, 1), (max_warps, 2)):
                with pytest.raises(ms.MambaScanError) as ei:
                    ms.scan_fwd(**dev, plan=ms.ScanPlan(config=cfg, warps_per_cta=warps, segments=segments))
                assert ei.value.status == 2
            shapes = [(max_warps, 1)]
        else:
            # the largest CTA whose shared memory fits (float32 tiles are twice as large)
            largest = None
            for warps in range(max_warps, 1, -1):
                try:
                    ms.scan_fwd(**dev, plan=ms.ScanPlan(config=cfg, warps_per_cta=warps, segments=1))
                    largest = warps
                    break
                except ms.MambaScanError as e:
                    assert e.status == 2
            assert largest is not None, f"config {cfg} runs at no CTA size"
            shapes = [(w, s) for w in sorted({2, largest}) for s in (1, 3)]
        for warps, segments in shapes:
            plan = ms.ScanPlan(config=cfg, warps_per_cta=warps, segments=segments)
            y, hT = ms.scan_fwd(**dev, plan=plan)
            torch.cuda.synchronize()
            tag = f"config {cfg} (kind {kind}, lanes {lanes}, states {states}), {warps} warps, {segments} segments"
            assert rel_err(to_host64(y), yr) <= TOL[dtype], tag
            assert rel_err(to_host64(hT), hr) <= TOL[dtype], tag


def _sequential_configs():
    return [(cfg, lanes, warps) for cfg, lanes, _, warps, kind in _ms().scan_configs() if kind == 1]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("batch,dim,N,L,offset", [
    (1, 3, 16, 1, 0), (2, 37, 16, 33, 0), (2, 130, 16, 1000, 0), (3, 20, 5, 97, 0),
    (1, 64, 1, 64, 0), (2, 70, 16, 255, 1), (1, 9, 8, 31, 3),
])
def test_sequential_kernels(dtype, batch, dim, N, L, offset):
    """Every sequential configuration on ragged rows, lengths and state sizes,
    with an initial state, and (offset > 0) rows that are not 16-byte aligned
    (the scalar load path), against the oracle."""
    import torch
    ms = _ms()
    inp = make_scan_inputs(LAYER, batch=batch, dim=dim, dstate=N, seqlen=L + offset, dtype=dtype,
                           seed=1500 + dim + L + N)
    dev = device_inputs(inp)
    if offset:   # drop the first `offset` steps of every row: views with misaligned row starts
        for k in ("u", "delta", "z", "B", "C"):
            dev[k] = dev[k][..., offset:]
        for k in ("u", "delta", "z", "B", "C"):
            inp[k] = np.ascontiguousarray(inp[k][..., offset:])
        inp["seqlen"] = L
    h0 = np.random.default_rng(dim).normal(size=(batch, dim, N)).astype(np.float32)
    yr, hr = oracle_scan(inp, h0=h0.reshape(-1, N))
    for cfg, lanes, warps in _sequential_configs():
        plan = ms.ScanPlan(config=cfg, warps_per_cta=warps, segments=1)
        y, hT = ms.scan_fwd(**dev, plan=plan, initial_state=torch.from_numpy(h0).cuda())
        torch.cuda.synchronize()
        tag = f"config {cfg} (lanes per row {lanes})"
        assert rel_err(to_host64(y), yr) <= TOL[dtype], tag
        assert rel_err(to_host64(hT), hr) <= TOL[dtype], tag


def test_plan_validation():
    """Unusable plans are refused before any launch."""
    import torch
    ms = _ms()
    inp = make_scan_inputs(LAYER, batch=1, dim=8, dstate=4, seqlen=128, seed=1200)
    dev = device_inputs(inp)
    configs = ms.scan_configs()
    pipelined = [c for c, _, states, _, kind in configs if states == 0 and kind == 0]
    for plan in [ms.ScanPlan(config=len(configs), warps_per_cta=4, segments=1),
                 ms.ScanPlan(config=0, warps_per_cta=1, segments=1),
                 ms.ScanPlan(config=0, warps_per_cta=4, segments=0),
                 ms.ScanPlan(config=pipelined[0], warps_per_cta=4, segments=1)]:   # needs dstate 16
        with pytest.raises(ms.MambaScanError) as ei:
            ms.scan_fwd(**dev, plan=plan)
        assert ei.value.status == 2
    torch.cuda.synchronize()
    # the automatic plan is one of the compiled configurations
    y = torch.empty_like(dev["u"])
    args = ms.build_scan_args(dev["u"], dev["delta"], dev["A"], dev["B"], dev["C"], y)
    plan = ms.scan_plan(args)
    assert 0 <= plan.config < len(configs) and plan.segments >= 1 and plan.warps_per_cta >= 2


def test_side_stream_with_segments():
    """A launch on a stream other than the current one, with the multi-block
    carry workspace allocated by the binding: work queued meanwhile on the
    current stream must not receive the workspace's memory while the scan
    still uses it."""
    import torch
    ms = _ms()
    inp = make_scan_inputs(LAYER, batch=2, dim=48, seqlen=6000 + 7, seed=1300)
    dev = device_inputs(inp)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    y, hT = ms.scan_fwd(**dev, force_segments=6, stream=side)
    # churn the allocator on the current stream while the side stream runs
    junk = [torch.full((1 << 16,), 7, dtype=torch.uint8, device="cuda") for _ in range(64)]
    del junk
    side.synchronize()
    torch.cuda.synchronize()
    yr, hr = oracle_scan(inp)
    assert rel_err(to_host64(y), yr) <= TOL["bf16"]
    assert rel_err(to_host64(hT), hr) <= TOL["bf16"]
