"""Pins of the fp64 oracle to facts other than itself.

Each ``pin_*`` function takes an oracle object (the ``oracle`` module, or an
``oracle.Variant`` built from a copy of its source with a planted mistake) and
raises ``AssertionError`` when the oracle disagrees with the fact it checks:
values printed by the pages for a worked example, closed forms, brute force on
tiny inputs, special cases that reduce to a library routine, and invariants.
None of them re-types the oracle's loop: each computes the expected value by a
different route (a convolution, a cumulative sum, an explicit matrix, a masked
matrix product, a single-step formula).
"""
from __future__ import annotations

import os

import numpy as np
from scipy.special import expit

HERE = os.path.dirname(os.path.abspath(__file__))
GOLDEN = os.path.join(HERE, "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


def _rel(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    scale = max(np.abs(b).max(), 1e-300)
    return float(np.abs(a - b).max() / scale)


def read_selection_step():
    rows = []
    with open(os.path.join(GOLDEN, "selection_step.txt")) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append([float(v) for v in line.split()])
    return rows


def pin_selection_step(orc):
    """The worked single step ("Notas sobre Mamba", "O mecanismo de seleção (S6)").

    h = 1, x = 1, A = -1, B = 1, softplus off, no bias: with B = 0 the new
    state is Abar itself; with B = 1 it is Abar + delta. Both must round to the
    page's printed 4-decimal values, for four identical state channels.
    """
    N = 4
    for delta, abar_p, bbar_p, h_p in read_selection_step():
        for Bval, expect in ((0.0, abar_p), (1.0, h_p)):
            state = np.ones((1, 1, N), np.float64)
            orc.state_update(state=state, x=_f32([[1.0]]), delta=_f32([[delta]]),
                             A=_f32(-np.ones((1, N))), B=_f32(np.full((1, N), Bval)),
                             C=_f32(np.ones((1, N))), delta_softplus=False)
            got = np.round(state.reshape(-1), 4)
            assert np.all(np.abs(got - expect) < 1e-9), (delta, Bval, state.reshape(-1), expect)
        # Bbar = delta * B with B = 1 is printed too: the state gained exactly delta.
        s0 = np.ones((1, 1, N))
        s1 = np.ones((1, 1, N))
        kw = dict(x=_f32([[1.0]]), delta=_f32([[delta]]), A=_f32(-np.ones((1, N))),
                  C=_f32(np.ones((1, N))), delta_softplus=False)
        orc.state_update(state=s0, B=_f32(np.zeros((1, N))), **kw)
        orc.state_update(state=s1, B=_f32(np.ones((1, N))), **kw)
        assert abs(round(float((s1 - s0).max()), 4) - bbar_p) < 1e-12


def pin_lti_convolution(orc, L=96, N=8, seed=11):
    """Constant delta, B and C make the system time invariant ("Notas sobre
    Mamba", "Preliminares"): y = K * x + D x with K_k = sum_n C_n Abar_n^k
    delta B_n and Abar = exp(delta A) -- first-order Bbar = delta B. Computed by
    np.convolve; agreement to 1e-12 relative.
    """
    g = _rng(seed)
    dim = 3
    A = -np.exp(g.normal(size=(dim, N))).astype(np.float32)
    Bv = g.normal(size=N).astype(np.float32)
    Cv = g.normal(size=N).astype(np.float32)
    D = g.uniform(0.5, 1.5, size=dim).astype(np.float32)
    x = g.normal(size=(1, dim, L)).astype(np.float32)
    delta = 0.0625
    Bt = np.repeat(Bv[None, :, None], L, axis=2)
    Ct = np.repeat(Cv[None, :, None], L, axis=2)
    y, h = orc.scan(u=x, delta=_f32(np.full((1, dim, L), delta)), A=A, B=_f32(Bt), C=_f32(Ct),
                    D=D, delta_softplus=False)
    k = np.arange(L)
    for d in range(dim):
        abar = np.exp(delta * A[d].astype(np.float64))
        K = ((Cv.astype(np.float64) * delta * Bv.astype(np.float64))[None, :]
             * np.power(abar[None, :], k[:, None])).sum(axis=1)
        ref = np.convolve(x[0, d].astype(np.float64), K)[:L] + float(D[d]) * x[0, d].astype(np.float64)
        assert _rel(y[0, d], ref) < 1e-12, (d, _rel(y[0, d], ref))
        # final state: sum_k abar^k delta B x_{L-1-k}
        href = (np.power(abar[None, :], k[::-1, None]) * (delta * Bv.astype(np.float64))[None, :]
                * x[0, d].astype(np.float64)[:, None]).sum(axis=0)
        assert _rel(h[0, d], href) < 1e-12


def pin_zero_delta(orc, L=40, N=5, seed=12):
    """delta = 0 keeps the state and ignores the token ("Notas sobre Mamba",
    "O mecanismo de seleção (S6)"): Abar = 1, Bbar = 0, so h stays 0 and
    y = D x silu(z), exactly.
    """
    g = _rng(seed)
    batch, dim = 2, 3
    x = g.normal(size=(batch, dim, L)).astype(np.float32)
    z = g.normal(size=(batch, dim, L)).astype(np.float32)
    D = g.uniform(0.5, 1.5, size=dim).astype(np.float32)
    A = -np.exp(g.normal(size=(dim, N))).astype(np.float32)
    B = g.normal(size=(batch, N, L)).astype(np.float32)
    C = g.normal(size=(batch, N, L)).astype(np.float32)
    y, h = orc.scan(u=x, delta=_f32(np.zeros((batch, dim, L))), A=A, B=B, C=C, D=D, z=z,
                    delta_softplus=False)
    assert np.all(h == 0.0)
    ref = D[None, :, None].astype(np.float64) * x * (z * expit(z.astype(np.float64)))
    assert _rel(y, ref) < 1e-15


def pin_linearity(orc, L=50, N=6, seed=13):
    """For fixed delta, B, C, z the map x -> (y, h_final) is linear ("Notas sobre
    Mamba", the recurrence of "O mecanismo de seleção (S6)"). Inputs are
    multiples of 1/8 so that 3 x1 - 2 x2 is exact in float32.
    """
    g = _rng(seed)
    batch, dim = 2, 4
    x1 = (g.integers(-16, 17, size=(batch, dim, L)) / 8.0).astype(np.float32)
    x2 = (g.integers(-16, 17, size=(batch, dim, L)) / 8.0).astype(np.float32)
    x3 = _f32(3.0 * x1 - 2.0 * x2)
    kw = dict(delta=_f32(g.normal(scale=0.5, size=(batch, dim, L))),
              A=_f32(-np.exp(g.normal(size=(dim, N)))),
              B=_f32(g.normal(size=(batch, N, L))), C=_f32(g.normal(size=(batch, N, L))),
              D=_f32(g.uniform(0.5, 1.5, size=dim)), z=_f32(g.normal(size=(batch, dim, L))),
              delta_bias=_f32(g.normal(size=dim) - 2.0), delta_softplus=True)
    y1, h1 = orc.scan(u=x1, **kw)
    y2, h2 = orc.scan(u=x2, **kw)
    y3, h3 = orc.scan(u=x3, **kw)
    assert _rel(y3, 3 * y1 - 2 * y2) < 1e-12
    assert _rel(h3, 3 * h1 - 2 * h2) < 1e-12
    # and not trivially linear: the map is not the zero map
    assert np.abs(y1).max() > 1e-3


def pin_scalar_state_closed_form(orc, L=60, seed=14):
    """N = 1: h_t = sum_{i<=t} exp(a (S_t - S_i)) delta_i B_i x_i with S the
    cumulative sum of delta -- the log-space cumulative product the pages use
    to build the decay mask ("Notas sobre Mamba", "A forma dual: atenção
    mascarada"). y_t = C_t h_t + D x_t.
    """
    g = _rng(seed)
    a = -0.75
    x = g.normal(size=(1, 1, L)).astype(np.float32)
    dl = g.uniform(0.01, 0.4, size=(1, 1, L)).astype(np.float32)
    B = g.normal(size=(1, 1, L)).astype(np.float32)
    C = g.normal(size=(1, 1, L)).astype(np.float32)
    D = np.array([0.9], np.float32)
    y, h = orc.scan(u=x, delta=dl, A=_f32([[a]]), B=B, C=C, D=D, delta_softplus=False)
    d64 = dl[0, 0].astype(np.float64)
    S = np.cumsum(d64)
    w = d64 * B[0, 0].astype(np.float64) * x[0, 0].astype(np.float64)
    href = np.array([np.sum(np.exp(a * (S[t] - S[:t + 1])) * w[:t + 1]) for t in range(L)])
    yref = C[0, 0].astype(np.float64) * href + float(D[0]) * x[0, 0].astype(np.float64)
    assert _rel(y[0, 0], yref) < 1e-12
    assert abs(h[0, 0, 0] - href[-1]) <= 1e-12 * max(1.0, abs(href[-1]))


def pin_unrolled_products(orc, seed=15):
    """Brute force on tiny inputs: y = M x + D x with the lower-triangular
    M_ji = sum_n C_j[n] (prod_{k=i+1..j} Abar_k[n]) Bbar_i[n] ("Notas sobre
    Mamba", "SSMs como matrizes semisseparáveis"), for every L <= 16 and
    random N <= 4, several batches and channels, softplus and bias on, gate on.
    """
    g = _rng(seed)
    for L in range(1, 17):
        N = int(g.integers(1, 5))
        batch, dim = 2, 3
        x = g.normal(size=(batch, dim, L)).astype(np.float32)
        raw = g.normal(scale=0.5, size=(batch, dim, L)).astype(np.float32)
        bias = (g.normal(size=dim) - 1.5).astype(np.float32)
        A = (-np.exp(g.normal(size=(dim, N)))).astype(np.float32)
        B = g.normal(size=(batch, N, L)).astype(np.float32)
        C = g.normal(size=(batch, N, L)).astype(np.float32)
        D = g.uniform(0.5, 1.5, size=dim).astype(np.float32)
        z = g.normal(size=(batch, dim, L)).astype(np.float32)
        y, h = orc.scan(u=x, delta=raw, A=A, B=B, C=C, D=D, z=z, delta_bias=bias,
                        delta_softplus=True)
        for b in range(batch):
            for d in range(dim):
                dl = np.logaddexp(0.0, raw[b, d].astype(np.float64) + float(bias[d]))
                abar = np.exp(dl[:, None] * A[d].astype(np.float64)[None, :])      # (L, N)
                bbar = dl[:, None] * B[b].T.astype(np.float64)                        # (L, N)
                M = np.zeros((L, L))
                for j in range(L):
                    for i in range(j + 1):
                        prod = np.prod(abar[i + 1:j + 1], axis=0) if j > i else np.ones(N)
                        M[j, i] = np.sum(C[b, :, j].astype(np.float64) * prod * bbar[i])
                xx = x[b, d].astype(np.float64)
                yref = (M @ xx + float(D[d]) * xx) * (z[b, d] * expit(z[b, d].astype(np.float64)))
                assert _rel(y[b, d], yref) < 1e-12, (L, N, b, d)
                hT = np.zeros(N)
                for i in range(L):
                    hT += np.prod(abar[i + 1:], axis=0) * bbar[i] * xx[i]
                assert _rel(h[b, d], hT) < 1e-12


def pin_scalar_transition_masked_form(orc, L=32, N=16, seed=16):
    """If A[d,n] = a for all n, Abar_t = a_t I and the scan equals the masked
    form y = (Lmask o (C B^T)) (delta x) + D x with Lmask_ji = prod_{k=i+1..j}
    a_k ("Notas sobre Mamba", "A forma dual: atenção mascarada"). Computed
    with matrix products.
    """
    g = _rng(seed)
    a = -0.375
    x = g.normal(size=(1, 1, L)).astype(np.float32)
    dl = g.uniform(0.05, 0.5, size=(1, 1, L)).astype(np.float32)
    B = g.normal(size=(1, N, L)).astype(np.float32)
    C = g.normal(size=(1, N, L)).astype(np.float32)
    D = np.array([1.25], np.float32)
    y, _ = orc.scan(u=x, delta=dl, A=_f32(np.full((1, N), a)), B=B, C=C, D=D,
                    delta_softplus=False)
    d64 = dl[0, 0].astype(np.float64)
    S = np.cumsum(a * d64)
    mask = np.tril(np.exp(S[:, None] - S[None, :]))
    Cm = C[0].T.astype(np.float64)
    Bm = B[0].T.astype(np.float64)
    xx = x[0, 0].astype(np.float64)
    yref = (mask * (Cm @ Bm.T)) @ (d64 * xx) + 1.25 * xx
    assert _rel(y[0, 0], yref) < 1e-12


def pin_segmentation(orc, L=77, m=30, N=4, seed=17):
    """Associativity of the recurrence ("Notas sobre Mamba", "A varredura
    paralela ciente do hardware"): the scan over [0, L) equals the scan over
    [0, m) continued from its final state over [m, L).
    """
    g = _rng(seed)
    batch, dim = 2, 3
    t = dict(u=g.normal(size=(batch, dim, L)), delta=g.normal(scale=0.5, size=(batch, dim, L)),
             z=g.normal(size=(batch, dim, L)), B=g.normal(size=(batch, N, L)),
             C=g.normal(size=(batch, N, L)))
    t = {k: _f32(v) for k, v in t.items()}
    p = dict(A=_f32(-np.exp(g.normal(size=(dim, N)))), D=_f32(g.uniform(0.5, 1.5, size=dim)),
             delta_bias=_f32(g.normal(size=dim) - 2.0), delta_softplus=True)
    y, h = orc.scan(**t, **p)
    y1, h1 = orc.scan(**{k: _f32(v[..., :m]) for k, v in t.items()}, **p)
    y2, h2 = orc.scan(**{k: _f32(v[..., m:]) for k, v in t.items()}, **p,
                      h0=h1.reshape(batch * dim, N))
    assert _rel(np.concatenate([y1, y2], axis=-1), y) < 1e-13
    assert _rel(h2, h) < 1e-13


def pin_decode_equals_scan(orc, L=25, N=16, seed=18):
    """L single-token steps from h = 0 reproduce the scan's y and final state
    (recurrent mode for generation, "Notas sobre Mamba", "Preliminares"; the
    step of "Mamba-2 e State Space Duality (SSD)").
    """
    g = _rng(seed)
    batch, dim = 3, 2
    t = dict(u=g.normal(size=(batch, dim, L)), delta=g.normal(scale=0.5, size=(batch, dim, L)),
             z=g.normal(size=(batch, dim, L)), B=g.normal(size=(batch, N, L)),
             C=g.normal(size=(batch, N, L)))
    t = {k: _f32(v) for k, v in t.items()}
    p = dict(A=_f32(-np.exp(g.normal(size=(dim, N)))), D=_f32(g.uniform(0.5, 1.5, size=dim)),
             delta_bias=_f32(g.normal(size=dim) - 2.0), delta_softplus=True)
    y, h = orc.scan(**t, **p)
    state = np.zeros((batch, dim, N))
    for s in range(L):
        ys = orc.state_update(state=state, x=_f32(t["u"][..., s]), delta=_f32(t["delta"][..., s]),
                              z=_f32(t["z"][..., s]), B=_f32(t["B"][..., s]),
                              C=_f32(t["C"][..., s]), **p)
        assert _rel(ys, y[..., s]) < 1e-14
    assert _rel(state, h) < 1e-14


def pin_large_delta_resets(orc, L=20, N=4, seed=19):
    """A large step forgets the past and absorbs the token ("Notas sobre
    Mamba", "O mecanismo de seleção (S6)"): with delta = 50, Abar underflows to
    below 1e-21 and h_t = delta B_t x_t, y_t = C_t . h_t + D x_t.
    """
    g = _rng(seed)
    x = g.normal(size=(1, 2, L)).astype(np.float32)
    B = g.normal(size=(1, N, L)).astype(np.float32)
    C = g.normal(size=(1, N, L)).astype(np.float32)
    A = _f32(-np.arange(1, N + 1)[None, :].repeat(2, 0))
    D = _f32([0.5, 1.5])
    y, h = orc.scan(u=x, delta=_f32(np.full((1, 2, L), 50.0)), A=A, B=B, C=C, D=D,
                    delta_softplus=False)
    for d in range(2):
        hb = 50.0 * B[0].astype(np.float64) * x[0, d].astype(np.float64)[None, :]
        yref = (C[0].astype(np.float64) * hb).sum(axis=0) + float(D[d]) * x[0, d].astype(np.float64)
        assert _rel(y[0, d], yref) < 1e-12
        assert _rel(h[0, d], hb[:, -1]) < 1e-12


def pin_softplus_of_biased_step(orc, seed=20):
    """delta = softplus(raw + bias) ("Notas sobre Mamba", "O mecanismo de
    seleção (S6)"): one step from h = 0 with B = x = 1 leaves h = delta, which
    must equal log(1 + exp(raw + bias)) from numpy's logaddexp; the bias is
    added before the softplus, so (raw, bias) and (raw + bias, 0) agree.
    """
    g = _rng(seed)
    raw = np.array([-9.0, -4.25, -1.0, 0.0, 0.75, 3.5, 12.0, 19.5, 25.0], np.float32)
    bias = np.float32(-0.5)
    for r in raw:
        hs = []
        for rr, bb in ((r, bias), (np.float32(r + bias), np.float32(0.0))):
            st = np.zeros((1, 1, 1))
            orc.state_update(state=st, x=_f32([[1.0]]), delta=_f32([[rr]]), A=_f32([[-1.0]]),
                             B=_f32([[1.0]]), C=_f32([[1.0]]), delta_bias=_f32([bb]),
                             delta_softplus=True)
            hs.append(float(st[0, 0, 0]))
        v = float(np.float32(r + bias))
        ref = float(np.logaddexp(0.0, v))
        assert abs(hs[1] - ref) <= 1e-12 * ref, (r, hs[1], ref)
        assert abs(hs[0] - hs[1]) <= 1e-12 * ref
    del g


def pin_gate(orc, L=33, N=3, seed=21):
    """The output is multiplied by SiLU(z) = z * sigmoid(z) ("Notas sobre Mamba",
    "O bloco Mamba"): y(z) = y(no z) * z * expit(z).
    """
    g = _rng(seed)
    t = dict(u=g.normal(size=(1, 2, L)), delta=g.normal(scale=0.5, size=(1, 2, L)),
             B=g.normal(size=(1, N, L)), C=g.normal(size=(1, N, L)))
    t = {k: _f32(v) for k, v in t.items()}
    p = dict(A=_f32(-np.exp(g.normal(size=(2, N)))), D=_f32([0.7, 1.1]),
             delta_bias=_f32([-2.0, -3.0]))
    z = g.normal(size=(1, 2, L)).astype(np.float32)
    y0, h0 = orc.scan(**t, **p)
    y1, h1 = orc.scan(**t, **p, z=z)
    assert _rel(y1, y0 * z * expit(z.astype(np.float64))) < 1e-14
    assert np.array_equal(h0, h1)


def pin_bf16_decoding(orc, seed=22):
    """bfloat16 inputs are read as the float32 value with the same top 16 bits:
    the bf16 scan equals the f32 scan of the widened values, and a few bit
    patterns have known values (0x3F80 = 1, 0xC040 = -3, 0x3E80 = 0.25).
    """
    g = _rng(seed)
    L, N = 9, 2
    known = np.array([0x3F80, 0xC040, 0x3E80], np.uint16)
    vals = np.array([1.0, -3.0, 0.25])
    st = np.zeros((1, 3, 1))
    orc.state_update(state=st, x=known.reshape(1, 3), delta=np.full((1, 3), 0x3F80, np.uint16),
                     A=_f32(-np.ones((3, 1))), B=np.full((1, 1), 0x3F80, np.uint16),
                     C=np.full((1, 1), 0x3F80, np.uint16), delta_softplus=False, dtype="bf16")
    assert np.allclose(st.reshape(-1), vals, rtol=0, atol=1e-15)

    def bits(a):
        return (np.asarray(a, np.float32).view(np.uint32) >> 16).astype(np.uint16)

    def widen(b):
        return (b.astype(np.uint32) << 16).view(np.float32)

    t = dict(u=g.normal(size=(1, 2, L)), delta=g.normal(scale=0.5, size=(1, 2, L)),
             B=g.normal(size=(1, N, L)), C=g.normal(size=(1, N, L)), z=g.normal(size=(1, 2, L)))
    tb = {k: bits(v) for k, v in t.items()}
    tf = {k: widen(v) for k, v in tb.items()}
    p = dict(A=_f32(-np.exp(g.normal(size=(2, N)))), D=_f32([0.7, 1.1]),
             delta_bias=_f32([-2.0, -3.0]))
    yb, hb = orc.scan(**tb, **p, dtype="bf16")
    yf, hf = orc.scan(**tf, **p, dtype="f32")
    assert np.array_equal(yb, yf) and np.array_equal(hb, hf)


# ---- convolution prologue ("Notas sobre Mamba", "O bloco Mamba": short
# depthwise convolution + SiLU before the SSM; width d_conv = 4 in "Mamba-2 e
# State Space Duality (SSD)"). Reading: causal, zero input before t = 0,
# w[d, K-1] weighs the current input.

def _conv_case(g, batch=2, dim=3, L=37, N=4, width=4):
    return dict(x=_f32(g.normal(size=(batch, dim, L))), conv_w=_f32(g.normal(size=(dim, width))),
                conv_b=_f32(g.normal(size=dim)), delta=_f32(g.normal(scale=0.5, size=(batch, dim, L))),
                A=_f32(-np.exp(g.normal(size=(dim, N)))), B=_f32(g.normal(size=(batch, N, L))),
                C=_f32(g.normal(size=(batch, N, L))), D=_f32(g.uniform(0.5, 1.5, size=dim)),
                delta_bias=_f32(g.normal(size=dim) - 2.0))


def pin_conv_matches_numpy_convolve(orc, seed=30):
    """The convolution output against numpy's full convolution truncated to
    the first L outputs (the causal form), for every width 1..4, with and
    without the SiLU (scipy's expit)."""
    g = _rng(seed)
    for width in (1, 2, 3, 4):
        case = _conv_case(g, width=width)
        for act in (False, True):
            _, _, u = orc.conv_scan(**case, conv_silu=act, return_u=True)
            x, w, b = case["x"].astype(np.float64), case["conv_w"].astype(np.float64), case["conv_b"]
            batch, dim, L = x.shape
            want = np.empty_like(x)
            for bi in range(batch):
                for d in range(dim):
                    pre = np.convolve(x[bi, d], w[d][::-1])[:L] + float(b[d])
                    want[bi, d] = pre * expit(pre) if act else pre
            assert _rel(u, want) <= 1e-12, (width, act)


def pin_conv_impulse_response(orc, seed=31):
    """A unit impulse at t0 returns the filter taps from t0 on, newest tap
    first, and nothing before t0 (causality)."""
    g = _rng(seed)
    case = _conv_case(g, batch=1, dim=2, L=16, width=4)
    case["x"] = np.zeros_like(case["x"])
    case["x"][0, 1, 5] = 1.0
    case["conv_b"] = np.zeros_like(case["conv_b"])
    _, _, u = orc.conv_scan(**case, conv_silu=False, return_u=True)
    w = case["conv_w"][1].astype(np.float64)
    want = np.zeros(16)
    want[5:9] = w[::-1]
    assert np.array_equal(u[0, 1], want)
    assert np.array_equal(u[0, 0], np.zeros(16))


def pin_conv_identity_filter_is_plain_scan(orc, seed=32):
    """Taps (0, ..., 0, 1), no bias, no SiLU: u = x, so the result is the plain
    scan of x, bit for bit."""
    g = _rng(seed)
    case = _conv_case(g, width=4)
    case["conv_w"] = _f32(np.tile([0.0, 0.0, 0.0, 1.0], (3, 1)))
    case["conv_b"] = None
    y, h = orc.conv_scan(**case, conv_silu=False)
    x = case.pop("x")
    for k in ("conv_w", "conv_b"):
        case.pop(k)
    y2, h2 = orc.scan(u=x, **case)
    assert np.array_equal(y, y2) and np.array_equal(h, h2)


def pin_conv_output_feeds_scan(orc, seed=33):
    """The scan of the fused path equals the plain scan of numpy's
    convolution + SiLU (rounded to float32, hence the tolerance)."""
    g = _rng(seed)
    case = _conv_case(g, width=3)
    y, h = orc.conv_scan(**case)
    x, w, b = case["x"].astype(np.float64), case["conv_w"].astype(np.float64), case["conv_b"]
    batch, dim, L = x.shape
    u = np.empty_like(x)
    for bi in range(batch):
        for d in range(dim):
            pre = np.convolve(x[bi, d], w[d][::-1])[:L] + float(b[d])
            u[bi, d] = pre * expit(pre)
    rest = {k: v for k, v in case.items() if k not in ("x", "conv_w", "conv_b")}
    y2, h2 = orc.scan(u=_f32(u), **rest)
    assert _rel(y, y2) <= 1e-5 and _rel(h, h2) <= 1e-5


def pin_conv_decode_equals_scan(orc, seed=34):
    """L decode steps with the convolution state reproduce the fused scan's
    outputs and final state, and leave the last `width` inputs in the
    convolution state, oldest first."""
    g = _rng(seed)
    case = _conv_case(g, batch=2, dim=3, L=19, N=5, width=4)
    y, h = orc.conv_scan(**case)
    batch, dim, L = case["x"].shape
    N = case["B"].shape[1]
    state = np.zeros((batch, dim, N))
    cstate = np.zeros((batch, dim, 4))
    ys = np.empty((batch, dim, L))
    for t in range(L):
        ys[:, :, t] = orc.conv_state_update(
            state=state, conv_state=cstate, x=_f32(case["x"][:, :, t]), conv_w=case["conv_w"],
            conv_b=case["conv_b"], delta=_f32(case["delta"][:, :, t]), A=case["A"],
            B=_f32(case["B"][:, :, t]), C=_f32(case["C"][:, :, t]), D=case["D"],
            delta_bias=case["delta_bias"])
    assert _rel(ys, y) <= 1e-12 and _rel(state, h) <= 1e-12
    assert np.array_equal(cstate, case["x"][:, :, L - 4:].astype(np.float64))


# ---- exponential-trapezoidal recurrence ("Notas sobre Mamba", section
# "Recorrência trapezoidal": h_t = alpha_t h_{t-1} + beta_t B_{t-1} x_{t-1}
# + gamma_t B_t x_t, lambda_t = sigmoid(.), B_{-1} x_{-1} = 0).

def _trap_case(g, batch=2, dim=3, L=29, N=5):
    return dict(u=_f32(g.normal(size=(batch, dim, L))), delta=_f32(g.normal(scale=0.5, size=(batch, dim, L))),
                lambda_raw=_f32(g.normal(size=(batch, dim, L))), A=_f32(-np.exp(g.normal(size=(dim, N)))),
                B=_f32(g.normal(size=(batch, N, L))), C=_f32(g.normal(size=(batch, N, L))),
                D=_f32(g.uniform(0.5, 1.5, size=dim)), z=_f32(g.normal(size=(batch, dim, L))),
                delta_bias=_f32(g.normal(size=dim) - 2.0))


def _read_trapezoid_check():
    rows = []
    with open(os.path.join(GOLDEN, "trapezoid_check.txt")) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                lam, val = line.split()
                rows.append((float(lam), float(val)))
    return rows


def _page_trajectories(orc, lam):
    """The section's experiment through the oracle: one channel, N = 6 states,
    the state trajectory read out one state at a time (C_t = e_n, no skip, no
    gate). Returns (trapezoidal, exponential-Euler) trajectories (L, N)."""
    g = np.random.default_rng(2)
    L, N = 24, 6
    A = -np.exp(g.normal(size=N))
    B = g.normal(size=(L, N))
    x = g.normal(size=L)
    delta = np.exp(g.normal(size=L) * 0.3)
    lam_raw = np.full(L, 40.0 if lam == 1.0 else 0.0)    # sigmoid(40) = 1 and sigmoid(0) = 1/2 in fp64
    common = dict(u=_f32(x.reshape(1, 1, L)), delta=_f32(delta.reshape(1, 1, L)), A=_f32(A.reshape(1, N)),
                  B=_f32(B.T.reshape(1, N, L)), delta_softplus=False)
    trap = np.empty((L, N))
    euler = np.empty((L, N))
    for n in range(N):
        C = np.zeros((1, N, L), np.float32)
        C[0, n, :] = 1.0
        trap[:, n] = orc.trap_scan(lambda_raw=_f32(lam_raw.reshape(1, 1, L)), C=C, **common)[0][0, 0]
        euler[:, n] = orc.scan(C=C, **common)[0][0, 0]
    return trap, euler


def pin_trap_page_check(orc):
    """The section's printed check: lambda = 1 reproduces exponential-Euler (to
    rounding), lambda = 1/2 differs by 1.50 (the printed value, 2 decimals)."""
    for lam, printed in _read_trapezoid_check():
        trap, euler = _page_trajectories(orc, lam)
        diff = float(np.abs(trap - euler).max())
        if lam == 1.0:
            assert diff <= 1e-13, diff
        else:
            assert f"{diff:.2e}" == f"{printed:.2e}", (diff, printed)


def pin_trap_unrolled_sum(orc, seed=40):
    """Brute force: h_t = sum_{s<=t} (prod_{k=s+1..t} alpha_k) (gamma_s B_s x_s
    + beta_s B_{s-1} x_{s-1}), built from cumulative products, then y = C h +
    D x times silu(z)."""
    g = _rng(seed)
    case = _trap_case(g, batch=1, dim=2, L=14, N=3)
    y, h = orc.trap_scan(**case)
    x = case["u"][0].astype(np.float64)
    dr = case["delta"][0].astype(np.float64) + case["delta_bias"][:, None]
    dt = np.logaddexp(0.0, dr)
    lam = expit(case["lambda_raw"][0].astype(np.float64))
    Bm = case["B"][0].astype(np.float64)          # (N, L)
    Cm = case["C"][0].astype(np.float64)
    L = x.shape[1]
    for d in range(2):
        ys = np.zeros(L)
        for n in range(3):
            alpha = np.exp(dt[d] * float(case["A"][d, n]))
            beta = (1.0 - lam[d]) * dt[d] * alpha
            gamma = lam[d] * dt[d]
            v = Bm[n] * x[d]
            src = gamma * v + beta * np.concatenate([[0.0], v[:-1]])
            ht = np.array([sum(np.prod(alpha[s + 1:t + 1]) * src[s] for s in range(t + 1)) for t in range(L)])
            ys += Cm[n] * ht
            assert abs(ht[-1] - h[0, d, n]) <= 1e-12 * max(1.0, abs(ht[-1]))
        zz = case["z"][0, d].astype(np.float64)
        ys = (ys + float(case["D"][d]) * x[d]) * zz * expit(zz)
        assert _rel(y[0, d], ys) <= 1e-12


def pin_trap_linearity(orc, seed=41):
    """Linear in x for fixed delta, lambda, B, C (no gate)."""
    g = _rng(seed)
    case = _trap_case(g)
    case["z"] = None
    x1, x2 = case.pop("u"), _f32(g.normal(size=case["delta"].shape))
    a, b = 0.75, -1.25
    y1, h1 = orc.trap_scan(u=x1, **case)
    y2, h2 = orc.trap_scan(u=x2, **case)
    y3, h3 = orc.trap_scan(u=_f32(a * x1.astype(np.float64) + b * x2.astype(np.float64)), **case)
    assert _rel(y3, a * y1 + b * y2) <= 1e-6 and _rel(h3, a * h1 + b * h2) <= 1e-6


# ---- backward pass (gradients of the scan, the training half the pages
# recompute instead of storing: "A varredura paralela ciente do hardware") ----

def _bwd_case(g, batch=2, dim=2, N=3, L=9, softplus=True):
    """Without the softplus the step is used as given, so it is drawn positive
    (a step of the discretised system; negative steps make the state grow and
    the finite differences lose digits)."""
    delta = g.normal(scale=0.5, size=(batch, dim, L))
    bias = g.normal(size=dim) - 1.0
    if not softplus:
        delta, bias = np.abs(delta), g.uniform(0.05, 0.2, size=dim)
    return dict(u=g.normal(size=(batch, dim, L)), delta=delta,
                A=-np.exp(g.normal(size=(dim, N))), B=g.normal(size=(batch, N, L)), C=g.normal(size=(batch, N, L)),
                D=g.uniform(0.5, 1.5, size=dim), z=g.normal(size=(batch, dim, L)),
                delta_bias=bias, h0=g.normal(size=(batch, dim, N)), delta_softplus=softplus)


def pin_double_forward_matches_scan(orc, seed=50):
    """The all-double forward (the backward's reference) computes the same
    values as the float32 scan on float32 inputs."""
    g = _rng(seed)
    case = _bwd_case(g)
    f32 = {k: (_f32(v) if isinstance(v, np.ndarray) else v) for k, v in case.items()}
    y1, h1 = orc.scan_d(**{k: (v.astype(np.float64) if isinstance(v, np.ndarray) else v) for k, v in f32.items()})
    h0 = f32.pop("h0")
    y2, h2 = orc.scan(**f32, h0=h0.reshape(-1, h0.shape[-1]))
    assert _rel(y1, y2) <= 1e-14 and _rel(h1, h2) <= 1e-14


def pin_backward_finite_differences(orc, seed=51, eps=1e-6):
    """Every gradient of sum(y dy) + sum(hT dhT) against central finite
    differences of the all-double forward, input by input, with and without
    the softplus."""
    for softplus in (True, False):
        g = _rng(seed + softplus)
        case = _bwd_case(g, softplus=softplus)
        dy = g.normal(size=case["u"].shape)
        dhT = g.normal(size=case["h0"].shape)
        grads = orc.scan_bwd(**case, dy=dy, dhT=dhT)

        def loss(c):
            y, h = orc.scan_d(**c)
            return float((y * dy).sum() + (h * dhT).sum())

        for name, gname in (("u", "du"), ("delta", "ddelta"), ("z", "dz"), ("A", "dA"), ("B", "dB"), ("C", "dC"),
                            ("D", "dD"), ("delta_bias", "ddelta_bias"), ("h0", "dh0")):
            base = case[name]
            fd = np.empty_like(base)
            for idx in np.ndindex(base.shape):
                plus = dict(case); minus = dict(case)
                bp = base.copy(); bm = base.copy()
                bp[idx] += eps; bm[idx] -= eps
                plus[name] = bp; minus[name] = bm
                fd[idx] = (loss(plus) - loss(minus)) / (2 * eps)
            assert _rel(grads[gname], fd) <= 1e-6, (softplus, name, _rel(grads[gname], fd))


def pin_backward_linear_in_output_gradients(orc, seed=52):
    """The gradients are linear in (dy, dhT)."""
    g = _rng(seed)
    case = _bwd_case(g)
    dy1, dy2 = g.normal(size=case["u"].shape), g.normal(size=case["u"].shape)
    dh1, dh2 = g.normal(size=case["h0"].shape), g.normal(size=case["h0"].shape)
    g1 = orc.scan_bwd(**case, dy=dy1, dhT=dh1)
    g2 = orc.scan_bwd(**case, dy=dy2, dhT=dh2)
    g3 = orc.scan_bwd(**case, dy=2.0 * dy1 - 3.0 * dy2, dhT=2.0 * dh1 - 3.0 * dh2)
    for k in g1:
        assert _rel(g3[k], 2.0 * g1[k] - 3.0 * g2[k]) <= 1e-12, k


def _read_ssd_dual_check():
    with open(os.path.join(GOLDEN, "ssd_dual_check.txt")) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                L, N, P, lo, hi, seed, printed = line.split()
                return int(L), int(N), int(P), float(lo), float(hi), int(seed), float(printed)
    raise AssertionError("ssd_dual_check.txt holds no case")


def pin_ssd_page_check(orc):
    """The page's printed duality check ("Notas sobre Mamba", "A forma dual:
    atenção mascarada"): on its own seeded inputs, the recurrent form equals
    Y = (Lmask o C B^T) X, Lmask_ji = prod_{k=i+1..j} a_k, to the rounding of
    fp64 (the page prints a largest difference of 9.44e-15). The mask here is
    built from explicit products, not from the page's cumulative log-sum.
    """
    L, N, P, lo, hi, seed, printed = _read_ssd_dual_check()
    g = _rng(seed)
    a = g.uniform(lo, hi, size=L)
    B = g.normal(size=(L, N))
    C = g.normal(size=(L, N))
    X = g.normal(size=(L, P))
    Y, _ = orc.ssd_rec(a=a, B=B, C=C, X=X)
    mask = np.zeros((L, L))
    for j in range(L):
        for i in range(j + 1):
            mask[j, i] = np.prod(a[i + 1:j + 1])
    Yq = (mask * (C @ B.T)) @ X
    diff = float(np.abs(Y - Yq).max())
    assert diff <= 100.0 * printed, diff


def _ssd_case(g, batch=2, L=23, nheads=4, ngroups=2, P=3, N=5, dtype="f32"):
    t = dict(x=g.normal(size=(batch, L, nheads, P)), dt=g.normal(scale=0.5, size=(batch, L, nheads)),
             B=g.normal(size=(batch, L, ngroups, N)), C=g.normal(size=(batch, L, ngroups, N)),
             z=g.normal(size=(batch, L, nheads, P)))
    t = {k: _f32(v) for k, v in t.items()}
    p = dict(A=_f32(-g.uniform(1.0, 16.0, size=nheads)), D=_f32(g.uniform(0.5, 1.5, size=nheads)),
             dt_bias=_f32(np.log(np.expm1(np.exp(g.uniform(np.log(1e-3), np.log(1e-1), size=nheads))))),
             dt_softplus=True)
    return t, p


def pin_ssd_equals_selective_scan(orc, seed=60):
    """A scalar transition per head is the selective scan with A[d, n] equal
    to the head's A for every n ("Notas sobre Mamba", "A forma dual: atenção
    mascarada"): each channel p of head h is an S6 row whose step, bias and
    skip are the head's and whose B and C are the head's group's. Checked
    against the (separately pinned) selective-scan oracle, including an
    initial state and the final state."""
    g = _rng(seed)
    batch, L, H, G, P, N = 2, 23, 4, 2, 3, 5
    t, p = _ssd_case(g, batch, L, H, G, P, N)
    h0 = g.normal(size=(batch * H, P, N))
    y, hT = orc.ssd_scan(**t, **p, h0=h0)
    for b in range(batch):
        for h in range(H):
            grp = h // (H // G)
            u = _f32(t["x"][b, :, h, :].T[None])
            z = _f32(t["z"][b, :, h, :].T[None])
            dl = _f32(np.broadcast_to(t["dt"][b, :, h], (1, P, L)))
            Bs = _f32(t["B"][b, :, grp, :].T[None])
            Cs = _f32(t["C"][b, :, grp, :].T[None])
            ys, hs = orc.scan(u=u, delta=dl, A=_f32(np.full((P, N), p["A"][h])), B=Bs, C=Cs,
                              D=_f32(np.full(P, p["D"][h])), z=z, delta_bias=_f32(np.full(P, p["dt_bias"][h])),
                              delta_softplus=True, h0=h0[b * H + h])
            assert _rel(y[b, :, h, :], ys[0].T) < 1e-12
            assert _rel(hT[b, h], hs[0]) < 1e-12


def pin_ssd_layer_quadratic(orc, seed=61):
    """The whole layer (softplus step with bias, skip, gate, two groups) in
    its dual form: per head, y = (Lmask o C_g B_g^T)(delta x) + D x, gated by
    z sigmoid(z), with Lmask_ji = exp(S_j - S_i), S = cumsum(delta A) ("Notas
    sobre Mamba", "A forma dual: atenção mascarada"; "Mamba-2 e State Space
    Duality (SSD)", "A teoria do State Space Duality (SSD) no Mamba-2").
    softplus and the sigmoid come from numpy and scipy."""
    g = _rng(seed)
    batch, L, H, G, P, N = 2, 31, 4, 2, 3, 6
    t, p = _ssd_case(g, batch, L, H, G, P, N)
    y, _ = orc.ssd_scan(**t, **p)
    for b in range(batch):
        for h in range(H):
            grp = h // (H // G)
            dl = np.logaddexp(0.0, t["dt"][b, :, h].astype(np.float64) + float(p["dt_bias"][h]))
            S = np.cumsum(dl * float(p["A"][h]))
            mask = np.tril(np.exp(S[:, None] - S[None, :]))
            Bm = t["B"][b, :, grp, :].astype(np.float64)
            Cm = t["C"][b, :, grp, :].astype(np.float64)
            X = t["x"][b, :, h, :].astype(np.float64)
            zz = t["z"][b, :, h, :].astype(np.float64)
            yref = ((mask * (Cm @ Bm.T)) @ (dl[:, None] * X) + float(p["D"][h]) * X) * zz * expit(zz)
            assert _rel(y[b, :, h, :], yref) < 1e-12


def pin_ssd_segmentation_and_pairs(orc, seed=62, m=11):
    """The layer over [0, L) equals the layer over [0, m) continued from its
    final state over [m, L) (state passing between blocks, "Notas sobre
    Mamba", "O algoritmo SSD"); a listed subset of (batch, head) pairs gives
    the same rows as the full run."""
    g = _rng(seed)
    batch, L, H, G, P, N = 2, 29, 4, 1, 4, 3
    t, p = _ssd_case(g, batch, L, H, G, P, N)
    y, hT = orc.ssd_scan(**t, **p)
    y1, h1 = orc.ssd_scan(**{k: _f32(v[:, :m]) for k, v in t.items()}, **p)
    y2, h2 = orc.ssd_scan(**{k: _f32(v[:, m:]) for k, v in t.items()}, **p, h0=h1.reshape(batch * H, P, N))
    assert _rel(np.concatenate([y1, y2], axis=1), y) < 1e-13
    assert _rel(h2, hT) < 1e-13
    ys, hs = orc.ssd_scan(**t, **p, pairs=[5, 0])
    assert np.array_equal(ys[0], y[1, :, 1, :]) and np.array_equal(ys[1], y[0, :, 0, :])
    assert np.array_equal(hs[0], hT[1, 1]) and np.array_equal(hs[1], hT[0, 0])


def pin_ssd_zero_step_keeps_state(orc, seed=63):
    """delta = 0 (no bias, no softplus): a_t = 1 and the input term vanishes,
    so the state stays at h0 and y_t = h0 C_t + D x_t ("Notas sobre Mamba",
    "O mecanismo de seleção (S6)": a small step keeps the state and ignores
    the token)."""
    g = _rng(seed)
    batch, L, H, G, P, N = 1, 9, 2, 1, 3, 4
    t, p = _ssd_case(g, batch, L, H, G, P, N)
    t["dt"] = _f32(np.zeros_like(t["dt"]))
    t.pop("z")
    h0 = g.normal(size=(batch * H, P, N))
    y, hT = orc.ssd_scan(**t, A=p["A"], D=p["D"], dt_softplus=False, h0=h0)
    for h in range(H):
        C = t["C"][0, :, 0, :].astype(np.float64)
        yref = C @ h0[h].T + float(p["D"][h]) * t["x"][0, :, h, :].astype(np.float64)
        assert _rel(y[0, :, h, :], yref) < 1e-14
        assert np.array_equal(hT[0, h], h0[h])


def pin_ssd_bf16_decoding(orc, seed=64):
    """bf16 inputs are read as their exact float32 values: the layer on bf16
    bit patterns equals the layer on the same values widened to float32."""
    g = _rng(seed)
    t, p = _ssd_case(g, 1, 13, 2, 1, 4, 3)
    bits = {k: (np.ascontiguousarray(v).view(np.uint32) >> np.uint32(16)).astype(np.uint16) for k, v in t.items()}
    wide = {k: (b.astype(np.uint32) << np.uint32(16)).view(np.float32) for k, b in bits.items()}
    y16, h16 = orc.ssd_scan(**bits, **p, dtype="bf16")
    y32, h32 = orc.ssd_scan(**wide, **p, dtype="f32")
    assert np.array_equal(y16, y32) and np.array_equal(h16, h32)
    assert _rel(y16, orc.ssd_scan(**t, **p, dtype="f32")[0]) > 1e-6


ALL_PINS = [
    pin_selection_step,
    pin_lti_convolution,
    pin_zero_delta,
    pin_linearity,
    pin_scalar_state_closed_form,
    pin_unrolled_products,
    pin_scalar_transition_masked_form,
    pin_segmentation,
    pin_decode_equals_scan,
    pin_large_delta_resets,
    pin_softplus_of_biased_step,
    pin_gate,
    pin_bf16_decoding,
    pin_conv_matches_numpy_convolve,
    pin_conv_impulse_response,
    pin_conv_identity_filter_is_plain_scan,
    pin_conv_output_feeds_scan,
    pin_conv_decode_equals_scan,
    pin_trap_page_check,
    pin_trap_unrolled_sum,
    pin_trap_linearity,
    pin_double_forward_matches_scan,
    pin_backward_finite_differences,
    pin_backward_linear_in_output_gradients,
    pin_ssd_page_check,
    pin_ssd_equals_selective_scan,
    pin_ssd_layer_quadratic,
    pin_ssd_segmentation_and_pairs,
    pin_ssd_zero_step_keeps_state,
    pin_ssd_bf16_decoding,
]
