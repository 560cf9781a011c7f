"""Pins for the fp64 oracle: each check ties the oracle to something other than
itself -- a brute-force direct sum, a closed form, a library routine, or an
invariant of the method -- so that a dropped term, a wrong sign or index, or a
transposed operand in ``oracle.c`` fails at least one test.  CPU only.
"""
import math

import numpy as np
import pytest
from scipy.special import expit

import oracle
from state_space_model_causal_b200 import inputs as gen


def _silu_ref(v):
    # logistic from scipy, not the oracle's 1/(1+exp(-v))
    return v * expit(v)


def _softplus_ref(v):
    return np.logaddexp(0.0, v)


def _conv_ref(x_row, w, bias, hist):
    """Causal cross-correlation through numpy.convolve: w[W-1] multiplies the
    current token, history (last W raw values, oldest first) pads the left."""
    W = len(w)
    if len(x_row) == 0:
        return np.zeros(0)
    padded = np.concatenate([hist[1:] if W > 1 else hist[:0], x_row])
    return np.convolve(padded, w[::-1], mode="valid") + bias


def _brute_force_scan(x, dt, A, Bm, Cm, Dv, z, dt_bias, softplus, cw, cb, cs, h0):
    """Direct, recurrence-free evaluation of the scan on tiny inputs:

    h_t[n] = exp(A_n * sum_{r<=t} delta_r) h0[n]
             + sum_{s<=t} exp(A_n * sum_{s<r<=t} delta_r) delta_s B_s[n] u_s
    y_t    = (sum_n C_t[n] h_t[n] + D u_t) * silu(z_t)
    """
    Bt, Dd, L = x.shape
    N = A.shape[1]
    G = Bm.shape[1]
    out = np.zeros((Bt, Dd, L))
    hT = np.zeros((Bt, Dd, N))
    for b in range(Bt):
        for d in range(Dd):
            g = d // (Dd // G)
            if cw is not None:
                W = cw.shape[1]
                hist = cs[b, d] if cs is not None else np.zeros(W)
                u = _silu_ref(_conv_ref(x[b, d], cw[d], cb[d] if cb is not None else 0.0, hist))
            else:
                u = x[b, d].copy()
            v = dt[b, d] + (dt_bias[d] if dt_bias is not None else 0.0)
            delta = _softplus_ref(v) if softplus else v
            for t in range(L):
                y = 0.0
                for n in range(N):
                    h = math.exp(A[d, n] * delta[: t + 1].sum()) * (h0[b, d, n] if h0 is not None else 0.0)
                    for s in range(t + 1):
                        h += math.exp(A[d, n] * delta[s + 1: t + 1].sum()) * delta[s] * Bm[b, g, n, s] * u[s]
                    y += Cm[b, g, n, t] * h
                    if t == L - 1:
                        hT[b, d, n] = h
                y += (Dv[d] if Dv is not None else 0.0) * u[t]
                if z is not None:
                    y *= _silu_ref(z[b, d, t])
                out[b, d, t] = y
    return out, hT


def _rand(shape, seed, name, scale=1.0):
    return gen.normal(shape, "pins", seed, name) * scale


@pytest.mark.parametrize("seed,Bt,Dd,L,N,G,W", [
    (0, 1, 1, 1, 1, 1, 0),
    (1, 1, 2, 5, 3, 1, 0),
    (2, 2, 3, 8, 4, 1, 4),
    (3, 1, 3, 7, 2, 3, 3),
    (4, 2, 2, 3, 4, 2, 4),   # L < W
    (5, 1, 2, 6, 3, 1, 1),   # W = 1
    (6, 1, 4, 5, 2, 2, 4),   # two channels per group
])
def test_scan_matches_brute_force(seed, Bt, Dd, L, N, G, W):
    x = _rand((Bt, Dd, L), seed, "x")
    dt = gen.uniform((Bt, Dd, L), -2.0, 1.0, "pins", seed, "dt")
    A = -np.abs(_rand((Dd, N), seed, "A")) - 0.1
    Bm = _rand((Bt, G, N, L), seed, "B")
    Cm = _rand((Bt, G, N, L), seed, "C")
    Dv = _rand((Dd,), seed, "D")
    z = _rand((Bt, Dd, L), seed, "z")
    db = _rand((Dd,), seed, "db", 0.5)
    h0 = _rand((Bt, Dd, N), seed, "h0")
    cw = _rand((Dd, W), seed, "cw", 0.5) if W else None
    cb = _rand((Dd,), seed, "cb") if W else None
    cs = _rand((Bt, Dd, W), seed, "cs") if W else None
    for softplus in (True, False):
        out, hf, _ = oracle.scan(x, dt, A, Bm, Cm, D=Dv, z=z, dt_bias=db, dt_softplus=softplus,
                                 conv_weight=cw, conv_bias=cb, conv_state=cs, h0=h0)
        ref, hT = _brute_force_scan(x, dt, A, Bm, Cm, Dv, z, db, softplus, cw, cb, cs, h0)
        np.testing.assert_allclose(out, ref, rtol=1e-11, atol=1e-12)
        np.testing.assert_allclose(hf, hT, rtol=1e-11, atol=1e-12)


def test_scan_optional_inputs_absent_match_brute_force():
    Bt, Dd, L, N = 1, 2, 6, 3
    x = _rand((Bt, Dd, L), 9, "x")
    dt = gen.uniform((Bt, Dd, L), -3.0, 0.0, "pins", 9, "dt")
    A = -np.abs(_rand((Dd, N), 9, "A"))
    Bm = _rand((Bt, 1, N, L), 9, "B")
    Cm = _rand((Bt, 1, N, L), 9, "C")
    out, hf, _ = oracle.scan(x, dt, A, Bm, Cm)
    ref, hT = _brute_force_scan(x, dt, A, Bm, Cm, None, None, None, True, None, None, None, None)
    np.testing.assert_allclose(out, ref, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(hf, hT, rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("A_val", [-0.7, -3.0, -0.01])
def test_scan_closed_form_constant_inputs(A_val):
    """Constant delta, A, B, C, x and h0 = 0: a = exp(delta A),
    h_t = delta B x (1 - a^(t+1)) / (1 - a), y_t = C h_t + D x."""
    L, N = 50, 2
    delta, Bv, Cv, xv, Dval = 0.3, 1.7, -0.4, 0.9, 0.25
    x = np.full((1, 1, L), xv)
    dt = np.full((1, 1, L), delta)
    A = np.full((1, N), A_val)
    Bm = np.full((1, 1, N, L), Bv)
    Cm = np.full((1, 1, N, L), Cv)
    out, hf, _ = oracle.scan(x, dt, A, Bm, Cm, D=np.array([Dval]), dt_softplus=False)
    a = math.exp(delta * A_val)
    t = np.arange(L)
    h = delta * Bv * xv * (1 - a ** (t + 1)) / (1 - a)
    np.testing.assert_allclose(out[0, 0], N * Cv * h + Dval * xv, rtol=1e-12)
    np.testing.assert_allclose(hf[0, 0], np.full(N, h[-1]), rtol=1e-12)


def test_scan_A_zero_is_prefix_sum():
    L, N = 40, 3
    x = _rand((1, 1, L), 11, "x")
    dt = np.abs(_rand((1, 1, L), 11, "dt"))
    Bm = _rand((1, 1, N, L), 11, "B")
    Cm = _rand((1, 1, N, L), 11, "C")
    out, _, _ = oracle.scan(x, dt, np.zeros((1, N)), Bm, Cm, dt_softplus=False)
    h = np.cumsum(dt[0, 0] * Bm[0, 0] * x[0, 0], axis=1)  # (N, L)
    np.testing.assert_allclose(out[0, 0], (Cm[0, 0] * h).sum(0), rtol=1e-11, atol=1e-12)


def test_scan_very_negative_A_has_no_memory():
    L, N = 20, 2
    x = _rand((1, 1, L), 12, "x")
    dt = np.full((1, 1, L), 1.0)
    Bm = _rand((1, 1, N, L), 12, "B")
    Cm = _rand((1, 1, N, L), 12, "C")
    out, _, _ = oracle.scan(x, dt, np.full((1, N), -1e4), Bm, Cm, dt_softplus=False)
    ref = (Cm[0, 0] * Bm[0, 0] * x[0, 0]).sum(0)
    np.testing.assert_allclose(out[0, 0], ref, rtol=1e-12)


def test_scan_B_zero_gives_skip_times_gate():
    s = gen.scan_inputs(2, 16, 3, 4, W=4, io="f32", seed=3, tag="pins")
    Bz = np.zeros_like(s.B)
    out, hf, _ = oracle.scan(s.x, s.dt, s.A, Bz, s.C, D=s.D, z=s.z, dt_bias=s.dt_bias,
                             conv_weight=s.conv_weight, conv_bias=s.conv_bias)
    u = np.stack([[_silu_ref(_conv_ref(s.x[b, d], s.conv_weight[d], 0.0, np.zeros(4)))
                   for d in range(3)] for b in range(2)])
    np.testing.assert_allclose(out, s.D[None, :, None] * u * _silu_ref(s.z), rtol=1e-12, atol=1e-14)
    assert np.all(hf == 0.0)


def test_scan_linear_in_x_without_conv():
    s = gen.scan_inputs(1, 24, 3, 4, io="f32", seed=4, tag="pins")
    x2 = _rand(s.x.shape, 4, "x2")
    alpha, beta = 0.6, -1.3
    kw = dict(D=s.D, z=s.z, dt_bias=s.dt_bias)
    y1, _, _ = oracle.scan(s.x, s.dt, s.A, s.B, s.C, **kw)
    y2, _, _ = oracle.scan(x2, s.dt, s.A, s.B, s.C, **kw)
    y12, _, _ = oracle.scan(alpha * s.x + beta * x2, s.dt, s.A, s.B, s.C, **kw)
    np.testing.assert_allclose(y12, alpha * y1 + beta * y2, rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("split", [1, 2, 3, 17, 39])
def test_scan_chunked_equals_sequential(split):
    s = gen.scan_inputs(2, 40, 3, 4, W=4, io="f32", seed=5, tag="pins", conv_state=True, h0=True)
    kw = dict(D=s.D, dt_bias=s.dt_bias, conv_weight=s.conv_weight, conv_bias=s.conv_bias)
    full, hf, csf = oracle.scan(s.x, s.dt, s.A, s.B, s.C, z=s.z, conv_state=s.conv_state,
                                h0=s.h0, **kw)
    a, h1, cs1 = oracle.scan(s.x[..., :split], s.dt[..., :split], s.A, s.B[..., :split],
                             s.C[..., :split], z=s.z[..., :split], conv_state=s.conv_state,
                             h0=s.h0, **kw)
    b, h2, cs2 = oracle.scan(s.x[..., split:], s.dt[..., split:], s.A, s.B[..., split:],
                             s.C[..., split:], z=s.z[..., split:], conv_state=cs1, h0=h1, **kw)
    np.testing.assert_allclose(np.concatenate([a, b], -1), full, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(h2, hf, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(cs2, csf, rtol=0, atol=0)


def _decode_steps_via_ssu(s, h, cs, t0, t1):
    """Run tokens t0..t1-1 through the single-token oracle (Mamba-1 layout
    mapped onto (B, H=1, P=D, N))."""
    Bt, Dd, _ = s.x.shape
    N = s.A.shape[1]
    outs = []
    st = h.reshape(Bt, 1, Dd, N)
    for t in range(t0, t1):
        o, st, cs = oracle.ssu(st, s.x[:, None, :, t], s.dt[:, None, :, t], s.A[None], s.B[..., t],
                               s.C[..., t], D=s.D[None], z=s.z[:, None, :, t],
                               dt_bias=s.dt_bias[None], conv_weight=s.conv_weight,
                               conv_bias=s.conv_bias, conv_state=cs)
        outs.append(o[:, 0])
    return np.stack(outs, -1), st.reshape(Bt, Dd, N), cs


@pytest.mark.parametrize("k", [1, 3, 6])
def test_prefill_then_decode_equals_full_prefill(k):
    L = 12
    s = gen.scan_inputs(2, L, 3, 4, W=4, io="f32", seed=6, tag="pins", conv_state=True, h0=True)
    kw = dict(D=s.D, dt_bias=s.dt_bias, conv_weight=s.conv_weight, conv_bias=s.conv_bias)
    full, hf, csf = oracle.scan(s.x, s.dt, s.A, s.B, s.C, z=s.z, conv_state=s.conv_state,
                                h0=s.h0, **kw)
    _, hp, csp = oracle.scan(s.x[..., :L - k], s.dt[..., :L - k], s.A, s.B[..., :L - k],
                             s.C[..., :L - k], z=s.z[..., :L - k], conv_state=s.conv_state,
                             h0=s.h0, **kw)
    dec, hd, csd = _decode_steps_via_ssu(s, hp, csp, L - k, L)
    np.testing.assert_allclose(dec, full[..., L - k:], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(hd, hf, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(csd.reshape(csf.shape), csf, rtol=0, atol=0)


def test_single_token_prefill_equals_one_update_without_conv():
    s = gen.scan_inputs(2, 1, 4, 5, io="f32", seed=7, tag="pins", h0=True)
    out, hf, _ = oracle.scan(s.x, s.dt, s.A, s.B, s.C, D=s.D, z=s.z, dt_bias=s.dt_bias, h0=s.h0)
    o, st, _ = oracle.ssu(s.h0[:, None], s.x[:, None, :, 0], s.dt[:, None, :, 0], s.A[None],
                          s.B[..., 0], s.C[..., 0], D=s.D[None], z=s.z[:, None, :, 0],
                          dt_bias=s.dt_bias[None])
    np.testing.assert_allclose(o[:, 0], out[..., 0], rtol=1e-13)
    np.testing.assert_allclose(st[:, 0], hf, rtol=1e-13)


@pytest.mark.parametrize("G", [1, 2, 4])
def test_mamba2_notation_matches_general_form(G):
    Bt, H, P, N = 3, 4, 5, 6
    s = gen.ssu_mamba2_inputs(Bt, H, P, N, G=G, io="f32", state="f32", seed=8, tag="pins",
                              with_z=True)
    o2, st2 = oracle.ssu_mamba2(s.state, s.x, s.dt, s.A, s.B, s.C, D=s.D, z=s.z,
                                dt_bias=s.dt_bias)
    og, stg, _ = oracle.ssu(s.state, s.x, s.dt[:, :, None], s.A[:, None, None], s.B, s.C,
                            D=s.D[:, None], z=s.z, dt_bias=s.dt_bias[:, None])
    np.testing.assert_allclose(o2, og, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(st2, stg, rtol=1e-13, atol=1e-14)


def test_mamba2_groups_map_consecutive_heads():
    """G groups: heads [g*H/G, (g+1)*H/G) read group g.  Equal to G separate
    calls with one group each on those head ranges."""
    Bt, H, P, N, G = 2, 6, 3, 4, 3
    s = gen.ssu_mamba2_inputs(Bt, H, P, N, G=G, io="f32", state="f32", seed=9, tag="pins",
                              with_z=True)
    o, st = oracle.ssu_mamba2(s.state, s.x, s.dt, s.A, s.B, s.C, D=s.D, z=s.z, dt_bias=s.dt_bias)
    hpg = H // G
    for g in range(G):
        hs = slice(g * hpg, (g + 1) * hpg)
        og, stg = oracle.ssu_mamba2(s.state[:, hs], s.x[:, hs], s.dt[:, hs], s.A[hs],
                                    s.B[:, g:g + 1], s.C[:, g:g + 1], D=s.D[hs], z=s.z[:, hs],
                                    dt_bias=s.dt_bias[hs])
        np.testing.assert_allclose(o[:, hs], og, rtol=1e-14)
        np.testing.assert_allclose(st[:, hs], stg, rtol=1e-14)


def _m2_prefill_inputs(seed, Bt, H, P, N, G, L):
    x = _rand((Bt, H, P, L), seed, "m2x")
    dt = gen.uniform((Bt, H, L), -3.0, 0.5, "pins", seed, "m2dt")
    A = -gen.uniform((H,), 0.2, 3.0, "pins", seed, "m2A")
    Bm = _rand((Bt, G, N, L), seed, "m2B")
    Cm = _rand((Bt, G, N, L), seed, "m2C")
    Dv = _rand((H,), seed, "m2D")
    z = _rand((Bt, H, P, L), seed, "m2z")
    db = _rand((H,), seed, "m2db", 0.5)
    h0 = _rand((Bt, H, P, N), seed, "m2h0")
    return x, dt, A, Bm, Cm, Dv, z, db, h0


@pytest.mark.parametrize("G", [1, 2])
def test_mamba2_prefill_matches_mamba1_scan_with_heads_expanded(G):
    """The Mamba-2-layout prefill equals the (separately pinned) Mamba-1 scan
    with one channel per (head, headdim) row: A, dt, dt_bias and D repeated
    over the head's rows and over n, no conv."""
    Bt, H, P, N, L = 2, 4, 3, 5, 9
    x, dt, A, Bm, Cm, Dv, z, db, h0 = _m2_prefill_inputs(11, Bt, H, P, N, G, L)
    out, hf = oracle.scan_mamba2(x, dt, A, Bm, Cm, D=Dv, z=z, dt_bias=db, h0=h0)
    D1 = H * P
    out1, hf1, _ = oracle.scan(x.reshape(Bt, D1, L), np.repeat(dt, P, axis=1),
                               np.repeat(A, P)[:, None] * np.ones((1, N)), Bm, Cm,
                               D=np.repeat(Dv, P), z=z.reshape(Bt, D1, L),
                               dt_bias=np.repeat(db, P), h0=h0.reshape(Bt, D1, N))
    np.testing.assert_allclose(out, out1.reshape(Bt, H, P, L), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(hf, hf1.reshape(Bt, H, P, N), rtol=1e-12, atol=1e-13)


def test_mamba2_prefill_equals_repeated_decode():
    """L prefill steps equal L single-token updates of the (separately pinned)
    Mamba-2 decode oracle, state carried from one to the next."""
    Bt, H, P, N, G, L = 2, 6, 3, 4, 3, 7
    x, dt, A, Bm, Cm, Dv, z, db, h0 = _m2_prefill_inputs(12, Bt, H, P, N, G, L)
    out, hf = oracle.scan_mamba2(x, dt, A, Bm, Cm, D=Dv, z=z, dt_bias=db, h0=h0)
    st = h0
    for t in range(L):
        o, st = oracle.ssu_mamba2(st, x[..., t], dt[..., t], A, Bm[..., t], Cm[..., t], D=Dv,
                                  z=z[..., t], dt_bias=db)
        np.testing.assert_allclose(out[..., t], o, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(hf, st, rtol=1e-13, atol=1e-14)


def test_mamba2_prefill_two_steps_by_hand():
    """One head, headdim 2, d_state 1, two steps, written out."""
    import math
    x = np.array([[[[0.5, -1.0], [2.0, 0.25]]]])      # (1, 1, 2, 2)
    dt = np.array([[[0.3, -0.2]]])
    A, Dv, db = np.array([-1.5]), np.array([0.7]), np.array([0.1])
    Bm = np.array([[[[1.2, -0.4]]]])                  # (1, 1, 1, 2)
    Cm = np.array([[[[0.9, 2.0]]]])
    out, hf = oracle.scan_mamba2(x, dt, A, Bm, Cm, D=Dv, dt_bias=db)
    sp = lambda v: math.log1p(math.exp(v))  # noqa: E731
    for p in range(2):
        h = 0.0
        for t in range(2):
            d = sp(dt[0, 0, t] + db[0])
            h = math.exp(d * A[0]) * h + d * Bm[0, 0, 0, t] * x[0, 0, p, t]
            assert out[0, 0, p, t] == pytest.approx(Cm[0, 0, 0, t] * h + Dv[0] * x[0, 0, p, t],
                                                    rel=1e-14, abs=1e-15)
        assert hf[0, 0, p, 0] == pytest.approx(h, rel=1e-14)


def test_ssu_single_step_matches_scan_brute_force_with_groups():
    """One decode step with state, conv and groups equals the brute-force scan
    of a single token whose conv history is the incoming conv state."""
    Bt, Dd, N, W, G = 2, 4, 3, 4, 2
    s = gen.scan_inputs(Bt, 1, Dd, N, G=G, W=W, io="f32", seed=10, tag="pins", conv_state=True,
                        h0=True)
    ref, hT = _brute_force_scan(s.x, s.dt, s.A, s.B, s.C, s.D, s.z, s.dt_bias, True,
                                s.conv_weight, s.conv_bias, s.conv_state, s.h0)
    # Mamba-1 channels as heads with headdim 1, so the group maps per channel.
    o, st, cs = oracle.ssu(s.h0[:, :, None, :], s.x[:, :, None, 0], s.dt[:, :, None, 0],
                           s.A[:, None, :], s.B[..., 0], s.C[..., 0], D=s.D[:, None],
                           z=s.z[:, :, None, 0], dt_bias=s.dt_bias[:, None],
                           conv_weight=s.conv_weight, conv_bias=s.conv_bias,
                           conv_state=s.conv_state)
    np.testing.assert_allclose(o[:, :, 0], ref[..., 0], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(st[:, :, 0], hT, rtol=1e-12, atol=1e-13)
    expect_cs = np.concatenate([s.conv_state[..., 1:], s.x[..., :1]], -1)
    np.testing.assert_array_equal(cs.reshape(Bt, Dd, W), expect_cs)


@pytest.mark.parametrize("W", [1, 2, 3, 4, 6])
def test_conv_impulse_response(W):
    L = 10
    w = _rand((1, W), 13, "w")
    x = np.zeros((1, 1, L))
    x[0, 0, 0] = 1.0
    out, _ = oracle.conv1d(x, w, bias=np.array([0.5]))
    expect = np.full(L, 0.5)
    for t in range(min(W, L)):
        expect[t] += w[0, W - 1 - t]
    np.testing.assert_allclose(out[0, 0], expect, rtol=0, atol=1e-15)


def test_conv_width_one_is_scaling():
    x = _rand((2, 3, 9), 14, "x")
    w = _rand((3, 1), 14, "w")
    b = _rand((3,), 14, "b")
    out, cs = oracle.conv1d(x, w, bias=b)
    np.testing.assert_allclose(out, w[None, :, :1] * x + b[None, :, None], rtol=1e-15)
    np.testing.assert_array_equal(cs[..., 0], x[..., -1])


@pytest.mark.parametrize("L", [0, 1, 2, 3, 4, 7])
def test_conv_matches_numpy_convolve_and_state(L):
    Bt, Dd, W = 2, 3, 4
    x = _rand((Bt, Dd, L), 15, "x")
    w = _rand((Dd, W), 15, "w")
    b = _rand((Dd,), 15, "b")
    cs = _rand((Bt, Dd, W), 15, "cs")
    for silu in (False, True):
        out, cso = oracle.conv1d(x, w, bias=b, conv_state=cs, silu=silu)
        for bb in range(Bt):
            for d in range(Dd):
                ref = _conv_ref(x[bb, d], w[d], b[d], cs[bb, d])
                if silu:
                    ref = _silu_ref(ref)
                np.testing.assert_allclose(out[bb, d], ref, rtol=1e-13, atol=1e-14)
                np.testing.assert_array_equal(cso[bb, d], np.concatenate([cs[bb, d], x[bb, d]])[-W:])


def test_activation_special_values():
    assert oracle.softplus(0.0) == pytest.approx(math.log(2.0), rel=1e-15)
    assert oracle.softplus(800.0) == pytest.approx(800.0, rel=1e-15)
    assert oracle.softplus(-800.0) == 0.0
    assert oracle.silu(0.0) == 0.0
    for v in (-3.0, -0.5, 0.25, 2.0, 30.0):
        # silu(v) - silu(-v) = v and softplus(v) - softplus(-v) = v
        assert oracle.silu(v) - oracle.silu(-v) == pytest.approx(v, rel=1e-14)
        assert oracle.softplus(v) - oracle.softplus(-v) == pytest.approx(v, rel=1e-14)


# ------------------------------------------------------- cache-dtype rounding --
def test_round_cache_matches_library_conversions():
    """The oracle's rounding of a state to its cache dtype equals numpy's
    float64 -> float16 conversion, torch's float32 -> bfloat16 conversion (on
    values exact in float32, so that no double rounding is involved) and the
    float64 -> float32 cast, including subnormals, ties and overflow."""
    import torch
    r = np.random.default_rng(0)
    v = r.standard_normal(20000) * 10.0 ** r.integers(-9, 6, 20000)
    edge = np.array([0.0, -0.0, 65504.0, 65519.99, 65520.0, -65520.0, 2.0 ** -24, 2.0 ** -25,
                     3 * 2.0 ** -26, 1 + 2.0 ** -11, 1 + 3 * 2.0 ** -11, 1e300])
    v = np.concatenate([v, edge])
    with np.errstate(over="ignore"):
        np.testing.assert_array_equal(oracle.round_cache(v, "f16"), v.astype(np.float16).astype(np.float64))
        np.testing.assert_array_equal(oracle.round_cache(v, "f32"), v.astype(np.float32).astype(np.float64))
    f = (r.standard_normal(20000) * 10.0 ** r.integers(-40, 38, 20000)).astype(np.float32)
    f = np.concatenate([f[np.isfinite(f)], np.float32([1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, 2.0 ** -130])])
    f = f.astype(np.float64)
    np.testing.assert_array_equal(oracle.round_cache(f, "bf16"),
                                  torch.from_numpy(f).float().bfloat16().double().numpy())
    np.testing.assert_array_equal(oracle.round_cache(v, None), v)


def test_round_cache_ties_go_to_even():
    """Hand values at exact ties: 1 + 2^-11 lies halfway between the fp16
    neighbours 1 and 1 + 2^-10 and goes to 1 (even last bit); 1 + 3 * 2^-11
    goes up to 1 + 2^-9; the same for bf16 one exponent step of 2^-8."""
    got = oracle.round_cache([1 + 2.0 ** -11, 1 + 3 * 2.0 ** -11, -(1 + 2.0 ** -11)], "f16")
    assert list(got) == [1.0, 1 + 2.0 ** -9, -1.0]
    got = oracle.round_cache([1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, 2 + 2.0 ** -7], "bf16")
    assert list(got) == [1.0, 1 + 2.0 ** -6, 2.0]


def test_ssu_cache_dtype_rounds_the_state_after_the_readout():
    """With cache_dtype the step's output is that of the unrounded update and
    the returned state is the unrounded state rounded to the cache dtype."""
    s = gen.ssu_mamba2_inputs(2, 4, 8, 16, io="f32", state="f32", seed=31, tag="round")
    o, st = oracle.ssu_mamba2(s.state, s.x, s.dt, s.A, s.B, s.C, D=s.D, dt_bias=s.dt_bias)
    for dt_ in ("f16", "bf16"):
        o2, st2 = oracle.ssu_mamba2(s.state, s.x, s.dt, s.A, s.B, s.C, D=s.D, dt_bias=s.dt_bias,
                                    cache_dtype=dt_)
        np.testing.assert_array_equal(o2, o)
        np.testing.assert_array_equal(st2, oracle.round_cache(st, dt_))
        assert not np.array_equal(st2, st)


# ----------------------------------------------------------- sequence pieces --
@pytest.mark.parametrize("softplus", [True, False])
def test_delta_sum_is_the_decay_exponent_of_the_scan(softplus):
    """With B = 0 the scan only decays its initial state, h_L = exp(A * S) h0
    with S the sum of the steps' delta: oracle.delta_sum must give that S (the
    scan is pinned to a recurrence-free brute force above)."""
    s = gen.scan_inputs(2, 9, 3, 2, io="f32", seed=11, tag="dsum", h0=True)
    dt = s.dt if softplus else np.abs(s.dt) * 0.05  # delta must stay positive without the softplus
    A = np.array([[-0.5, -1.0], [-0.25, -2.0], [-1.5, -0.75]])
    h0 = np.ones((2, 3, 2))
    _, hL, _ = oracle.scan(s.x, dt, A, np.zeros_like(s.B), s.C, D=s.D, z=s.z, dt_bias=s.dt_bias,
                           dt_softplus=softplus, h0=h0)
    S = oracle.delta_sum(dt, s.dt_bias, dt_softplus=softplus)
    np.testing.assert_allclose(hL, np.exp(A[None] * S[:, :, None]), rtol=1e-12, atol=0)
    assert oracle.delta_sum(dt[..., :0], s.dt_bias).tolist() == [[0.0] * 3] * 2


@pytest.mark.parametrize("cuts", [(5,), (3, 8), (1, 6, 11)])
def test_carry_fold_composes_sequence_pieces(cuts):
    """A prefill cut into consecutive pieces: each piece scanned from a zero
    state (conv history: the raw inputs just before it) ends in h_end(j).
    Folding h_in(j+1) = carry_fold(h_in(j), A, delta_sum(piece j), h_end(j))
    from h_in(0) = h0 must give the state the whole scan reaches at every cut,
    and each piece re-scanned from h_in(j) the whole scan's outputs."""
    L = 14
    s = gen.scan_inputs(2, L, 3, 4, W=4, io="f32", seed=12, tag="fold", conv_state=True, h0=True)
    kw = dict(D=s.D, dt_bias=s.dt_bias, conv_weight=s.conv_weight, conv_bias=s.conv_bias)
    piece = lambda a, t0, t1: a[..., t0:t1]  # noqa: E731
    full, hf, _ = oracle.scan(s.x, s.dt, s.A, s.B, s.C, z=s.z, conv_state=s.conv_state, h0=s.h0, **kw)
    bounds = (0,) + tuple(cuts) + (L,)
    h_in = s.h0
    cs = s.conv_state
    for j in range(len(bounds) - 1):
        t0, t1 = bounds[j], bounds[j + 1]
        args = [piece(a, t0, t1) for a in (s.x, s.dt)] + [s.A] + [piece(a, t0, t1) for a in (s.B, s.C)]
        out_j, _, cs_next = oracle.scan(*args, z=piece(s.z, t0, t1), conv_state=cs, h0=h_in, **kw)
        np.testing.assert_allclose(out_j, full[..., t0:t1], rtol=1e-11, atol=1e-12)
        _, h_end, _ = oracle.scan(*args, z=piece(s.z, t0, t1), conv_state=cs, h0=None, **kw)
        h_in = oracle.carry_fold(h_in, s.A, oracle.delta_sum(piece(s.dt, t0, t1), s.dt_bias), h_end)
        _, h_cut, _ = oracle.scan(*[piece(a, 0, t1) for a in (s.x, s.dt)], s.A,
                                  *[piece(a, 0, t1) for a in (s.B, s.C)], z=piece(s.z, 0, t1),
                                  conv_state=s.conv_state, h0=s.h0, **kw)
        np.testing.assert_allclose(h_in, h_cut, rtol=1e-11, atol=1e-12)
        cs = cs_next
    np.testing.assert_allclose(h_in, hf, rtol=1e-11, atol=1e-12)


def test_carry_fold_special_cases():
    """A = 0: no decay, the states add; S = 0: the same; a decay far below
    the smallest double: the earlier state is forgotten."""
    rng = np.random.default_rng(13)
    st, he = rng.standard_normal((2, 3, 4)), rng.standard_normal((2, 3, 4))
    A = -rng.uniform(0.5, 2.0, (3, 4))
    np.testing.assert_array_equal(oracle.carry_fold(st, np.zeros((3, 4)), np.ones((2, 3)), he), st + he)
    np.testing.assert_array_equal(oracle.carry_fold(st, A, np.zeros((2, 3)), he), st + he)
    np.testing.assert_array_equal(oracle.carry_fold(st, A, np.full((2, 3), 1e6), he), he)


# ---- double-gated short causal conv ("LFM2.5-1.2B-Thinking性能优化CUDA核心编程技巧"
# section 2.1 names the block; the reading out = Cg * conv(Bg * x) is the oracle's)

@pytest.mark.parametrize("L,W", [(0, 3), (1, 3), (2, 1), (3, 4), (5, 3), (9, 2), (11, 4)])
def test_gated_conv_matches_numpy_convolve_and_state(L, W):
    """The conv of the gated input through numpy.convolve, times the output
    gate; the outgoing state is the last W gated inputs."""
    Bt, Dd = 2, 3
    x, bg, cg = (_rand((Bt, Dd, L), 40, n) for n in ("x", "bg", "cg"))
    w = _rand((Dd, W), 40, "w")
    b = _rand((Dd,), 40, "b")
    cs = _rand((Bt, Dd, W), 40, "cs")
    out, cso = oracle.gated_conv1d(x, bg, cg, w, bias=b, conv_state=cs)
    for bb in range(Bt):
        for d in range(Dd):
            v = bg[bb, d] * x[bb, d]
            np.testing.assert_allclose(out[bb, d], cg[bb, d] * _conv_ref(v, w[d], b[d], cs[bb, d]),
                                       rtol=1e-13, atol=1e-14)
            np.testing.assert_array_equal(cso[bb, d], np.concatenate([cs[bb, d], v])[-W:])


def test_gated_conv_unit_gates_is_the_plain_conv():
    x = _rand((2, 4, 13), 41, "x")
    w, b = _rand((4, 3), 41, "w"), _rand((4,), 41, "b")
    cs = _rand((2, 4, 3), 41, "cs")
    one = np.ones_like(x)
    out, cso = oracle.gated_conv1d(x, one, one, w, bias=b, conv_state=cs)
    ref, csr = oracle.conv1d(x, w, bias=b, conv_state=cs, silu=False)
    np.testing.assert_array_equal(out, ref)
    np.testing.assert_array_equal(cso, csr)


@pytest.mark.parametrize("W", [1, 3, 4])
def test_gated_conv_impulse_response(W):
    """x = impulse at t0: out[t0 + j] = Cg[t0 + j] * (bias + w[W-1-j] * Bg[t0])."""
    L, t0 = 12, 3
    x = np.zeros((1, 1, L))
    x[0, 0, t0] = 1.0
    bg, cg = _rand((1, 1, L), 42, "bg"), _rand((1, 1, L), 42, "cg")
    w = _rand((1, W), 42, "w")
    out, _ = oracle.gated_conv1d(x, bg, cg, w, bias=np.array([0.25]))
    c = np.full(L, 0.25)
    for j in range(W):
        c[t0 + j] += w[0, W - 1 - j] * bg[0, 0, t0]
    np.testing.assert_allclose(out[0, 0], cg[0, 0] * c, rtol=1e-15, atol=1e-16)


def test_gated_conv_gates_act_before_and_after():
    """Changing the input gate at step t moves outputs t .. t+W-1; changing the
    output gate at step t moves output t alone; a zero input gate leaves
    Cg * bias."""
    L, W, t = 10, 4, 4
    x, bg, cg = (_rand((1, 2, L), 43, n) for n in ("x", "bg", "cg"))
    w, b = _rand((2, W), 43, "w"), _rand((2,), 43, "b")
    out, _ = oracle.gated_conv1d(x, bg, cg, w, bias=b)
    bg2 = bg.copy()
    bg2[..., t] += 1.0
    moved = np.abs(oracle.gated_conv1d(x, bg2, cg, w, bias=b)[0] - out) > 0
    assert moved[..., t:t + W].all() and not moved[..., :t].any() and not moved[..., t + W:].any()
    cg2 = cg.copy()
    cg2[..., t] += 1.0
    moved = np.abs(oracle.gated_conv1d(x, bg, cg2, w, bias=b)[0] - out) > 0
    assert moved[..., t].all() and moved.sum() == 2
    out0, cs0 = oracle.gated_conv1d(x, np.zeros_like(bg), cg, w, bias=b)
    np.testing.assert_array_equal(out0, cg * b[None, :, None])
    np.testing.assert_array_equal(cs0, np.zeros((1, 2, W)))


@pytest.mark.parametrize("k", [0, 1, 3, 7, 12])
def test_gated_conv_split_and_token_steps_equal_one_call(k):
    """The sequence cut at k with the state carried, and token-by-token
    decoding, equal one call over the whole sequence."""
    L, W = 12, 3
    x, bg, cg = (_rand((2, 3, L), 44, n) for n in ("x", "bg", "cg"))
    w, b = _rand((3, W), 44, "w"), _rand((3,), 44, "b")
    cs = _rand((2, 3, W), 44, "cs")
    full, csf = oracle.gated_conv1d(x, bg, cg, w, bias=b, conv_state=cs)
    o1, cs1 = oracle.gated_conv1d(x[..., :k], bg[..., :k], cg[..., :k], w, bias=b, conv_state=cs)
    o2, cs2 = oracle.gated_conv1d(x[..., k:], bg[..., k:], cg[..., k:], w, bias=b, conv_state=cs1)
    np.testing.assert_allclose(np.concatenate([o1, o2], -1), full, rtol=1e-14, atol=1e-15)
    np.testing.assert_array_equal(cs2, csf)
    st, steps = cs, []
    for t in range(L):
        o, st = oracle.gated_conv1d(x[..., t:t + 1], bg[..., t:t + 1], cg[..., t:t + 1], w, bias=b, conv_state=st)
        steps.append(o)
    np.testing.assert_allclose(np.concatenate(steps, -1), full, rtol=1e-14, atol=1e-15)
    np.testing.assert_array_equal(st, csf)
