"""Randomised invariants of the fp64 oracle (CPU, hypothesis).

The fixed-shape pins in test_oracle_pins.py tie the oracle to brute-force
sums, closed forms and invariants.  These tests draw shapes, split points
and seeds at random to show the same invariants hold away from the pinned
shapes:
  * a prefill split anywhere, state and conv state carried across, equals
    the whole prefill (Mamba-1 and Mamba-2 layouts);
  * without the conv and with h0 = 0, the output is linear in x (z fixed);
  * a prefill of the first tokens followed by single-token updates equals
    the whole prefill (Mamba-1 layout with the fused conv);
  * the Mamba-2-layout prefill equals the Mamba-1 scan with its per-head
    values repeated over the head's rows;
  * both prefills are causal: inputs at later steps leave earlier outputs
    bit-identical;
  * Mamba-1 channels are independent: one channel's inputs, parameters and
    states reach no other channel's outputs or states;
  * a prefill cut into pieces scanned from zero states is recovered exactly
    by composing the pieces' carries and adding the decayed incoming state's
    readout (the context-parallel decomposition), in both layouts;
  * the double-gated short conv: a split anywhere equals one call, the
    output is linear in x for fixed gates, and it is causal with a window of
    W steps for the input gate.
"""
import numpy as np
from hypothesis import given, settings
from hypothesis import strategies as st

import oracle
from state_space_model_causal_b200 import inputs as gen

SETTINGS = dict(max_examples=25, deadline=None)


@settings(**SETTINGS)
@given(Bt=st.integers(1, 2), D=st.integers(1, 6), L=st.integers(2, 24), N=st.integers(1, 6),
       W=st.sampled_from([0, 1, 3, 4]), frac=st.floats(0.05, 0.95), seed=st.integers(0, 10**6))
def test_mamba1_prefill_split_anywhere(Bt, D, L, N, W, frac, seed):
    split = max(1, min(L - 1, int(L * frac)))
    s = gen.scan_inputs(Bt, L, D, N, W=W, io="f32", seed=seed, tag="prop", conv_state=W > 0, h0=True)
    kw = dict(D=s.D, dt_bias=s.dt_bias, conv_weight=s.conv_weight, conv_bias=s.conv_bias)
    full, hf, csf = oracle.scan(s.x, s.dt, s.A, s.B, s.C, z=s.z, conv_state=s.conv_state, h0=s.h0, **kw)
    cut = lambda a, sl: a[..., sl]  # noqa: E731
    a, h1, cs1 = oracle.scan(cut(s.x, slice(0, split)), cut(s.dt, slice(0, split)), s.A,
                             cut(s.B, slice(0, split)), cut(s.C, slice(0, split)),
                             z=cut(s.z, slice(0, split)), conv_state=s.conv_state, h0=s.h0, **kw)
    b, h2, cs2 = oracle.scan(cut(s.x, slice(split, L)), cut(s.dt, slice(split, L)), s.A,
                             cut(s.B, slice(split, L)), cut(s.C, slice(split, L)),
                             z=cut(s.z, slice(split, L)), conv_state=cs1, h0=h1, **kw)
    np.testing.assert_allclose(np.concatenate([a, b], -1), full, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(h2, hf, rtol=1e-11, atol=1e-12)
    if W > 0:
        np.testing.assert_array_equal(cs2, csf)


@settings(**SETTINGS)
@given(Bt=st.integers(1, 2), H=st.integers(1, 4), P=st.integers(1, 5), N=st.integers(1, 8),
       L=st.integers(2, 20), G=st.sampled_from([1, 2]), frac=st.floats(0.05, 0.95),
       seed=st.integers(0, 10**6))
def test_mamba2_prefill_split_anywhere(Bt, H, P, N, L, G, frac, seed):
    H = H * G  # heads divisible by groups
    split = max(1, min(L - 1, int(L * frac)))
    s = gen.scan_m2_inputs(Bt, H, P, N, L, G=G, io="f32", seed=seed, tag="prop", h0=True)
    full, hf = oracle.scan_mamba2(s.x, s.dt, s.A, s.B, s.C, D=s.D, z=s.z, dt_bias=s.dt_bias, h0=s.h0)
    sl1, sl2 = slice(0, split), slice(split, L)
    a, h1 = oracle.scan_mamba2(s.x[..., sl1], s.dt[..., sl1], s.A, s.B[..., sl1], s.C[..., sl1], D=s.D,
                               z=s.z[..., sl1], dt_bias=s.dt_bias, h0=s.h0)
    b, h2 = oracle.scan_mamba2(s.x[..., sl2], s.dt[..., sl2], s.A, s.B[..., sl2], s.C[..., sl2], D=s.D,
                               z=s.z[..., sl2], dt_bias=s.dt_bias, h0=h1)
    np.testing.assert_allclose(np.concatenate([a, b], -1), full, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(h2, hf, rtol=1e-11, atol=1e-12)


@settings(**SETTINGS)
@given(D=st.integers(1, 5), L=st.integers(1, 16), N=st.integers(1, 5), alpha=st.floats(-3, 3),
       seed=st.integers(0, 10**6))
def test_mamba1_output_linear_in_x_without_conv(D, L, N, alpha, seed):
    s = gen.scan_inputs(1, L, D, N, W=0, io="f32", seed=seed, tag="prop_lin")
    x2 = gen.normal(s.x.shape, "prop_lin", seed, "x2")
    kw = dict(D=s.D, z=s.z, dt_bias=s.dt_bias)
    y1, _, _ = oracle.scan(s.x, s.dt, s.A, s.B, s.C, **kw)
    y2, _, _ = oracle.scan(x2, s.dt, s.A, s.B, s.C, **kw)
    y12, _, _ = oracle.scan(s.x + alpha * x2, s.dt, s.A, s.B, s.C, **kw)
    np.testing.assert_allclose(y12, y1 + alpha * y2, rtol=1e-10, atol=1e-11)


@settings(**SETTINGS)
@given(Bt=st.integers(1, 2), D=st.integers(1, 4), N=st.integers(1, 4), L=st.integers(2, 10),
       k=st.integers(1, 4), seed=st.integers(0, 10**6))
def test_mamba1_prefill_then_single_token_updates(Bt, D, N, L, k, seed):
    k = min(k, L - 1)
    s = gen.scan_inputs(Bt, L, D, N, W=4, io="f32", seed=seed, tag="prop_pd", conv_state=True, h0=True)
    kw = dict(D=s.D, dt_bias=s.dt_bias, conv_weight=s.conv_weight, conv_bias=s.conv_bias)
    full, hf, csf = oracle.scan(s.x, s.dt, s.A, s.B, s.C, z=s.z, conv_state=s.conv_state, h0=s.h0, **kw)
    head = slice(0, L - k)
    _, h, cs = oracle.scan(s.x[..., head], s.dt[..., head], s.A, s.B[..., head], s.C[..., head],
                           z=s.z[..., head], conv_state=s.conv_state, h0=s.h0, **kw)
    st_ = h.reshape(Bt, 1, D, N)
    for t in range(L - k, L):
        o, st_, cs = oracle.ssu(st_, s.x[:, None, :, t], s.dt[:, None, :, t], s.A[None], s.B[..., t],
                                s.C[..., t], D=s.D[None], z=s.z[:, None, :, t], dt_bias=s.dt_bias[None],
                                conv_weight=s.conv_weight, conv_bias=s.conv_bias, conv_state=cs)
        np.testing.assert_allclose(o[:, 0], full[..., t], rtol=1e-11, atol=1e-12)
        cs = cs.reshape(Bt, D, -1)
    np.testing.assert_allclose(st_.reshape(Bt, D, N), hf, rtol=1e-11, atol=1e-12)


@settings(**SETTINGS)
@given(Bt=st.integers(1, 2), H=st.integers(1, 3), P=st.integers(1, 4), N=st.integers(1, 6),
       L=st.integers(1, 12), seed=st.integers(0, 10**6))
def test_mamba2_prefill_equals_mamba1_scan_with_heads_repeated(Bt, H, P, N, L, seed):
    s = gen.scan_m2_inputs(Bt, H, P, N, L, io="f32", seed=seed, tag="prop_x", h0=True)
    y2, h2 = oracle.scan_mamba2(s.x, s.dt, s.A, s.B, s.C, D=s.D, z=s.z, dt_bias=s.dt_bias, h0=s.h0)
    D1 = H * P
    y1, h1, _ = oracle.scan(s.x.reshape(Bt, D1, L), np.repeat(s.dt, P, axis=1),
                            np.repeat(s.A, P)[:, None] * np.ones((1, N)), s.B, s.C, D=np.repeat(s.D, P),
                            z=s.z.reshape(Bt, D1, L), dt_bias=np.repeat(s.dt_bias, P),
                            h0=s.h0.reshape(Bt, D1, N))
    np.testing.assert_allclose(y2, y1.reshape(Bt, H, P, L), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(h2, h1.reshape(Bt, H, P, N), rtol=1e-12, atol=1e-13)


@settings(**SETTINGS)
@given(Bt=st.integers(1, 2), D=st.integers(1, 4), L=st.integers(2, 16), N=st.integers(1, 4),
       W=st.sampled_from([0, 2, 4]), frac=st.floats(0.05, 0.95), seed=st.integers(0, 10**6))
def test_mamba1_prefill_is_causal(Bt, D, L, N, W, frac, seed):
    """Changing every input at steps >= t' leaves all outputs before t'
    bit-identical (the conv looks back only, the scan runs forward)."""
    cut = max(1, min(L - 1, int(L * frac)))
    s = gen.scan_inputs(Bt, L, D, N, W=W, io="f32", seed=seed, tag="prop_c", conv_state=W > 0, h0=True)
    kw = dict(D=s.D, dt_bias=s.dt_bias, conv_weight=s.conv_weight, conv_bias=s.conv_bias,
              conv_state=s.conv_state, h0=s.h0)
    y, _, _ = oracle.scan(s.x, s.dt, s.A, s.B, s.C, z=s.z, **kw)
    late = lambda a, name: np.concatenate(  # noqa: E731
        [a[..., :cut], gen.normal(a[..., cut:].shape, "prop_c2", seed, name)], -1)
    y2, _, _ = oracle.scan(late(s.x, "x"), late(s.dt, "dt"), s.A, late(s.B, "B"), late(s.C, "C"),
                           z=late(s.z, "z"), **kw)
    np.testing.assert_array_equal(y2[..., :cut], y[..., :cut])
    assert not np.array_equal(y2[..., cut:], y[..., cut:])


@settings(**SETTINGS)
@given(Bt=st.integers(1, 2), H=st.integers(1, 3), P=st.integers(1, 4), N=st.integers(1, 6),
       L=st.integers(2, 12), frac=st.floats(0.05, 0.95), seed=st.integers(0, 10**6))
def test_mamba2_prefill_is_causal(Bt, H, P, N, L, frac, seed):
    cut = max(1, min(L - 1, int(L * frac)))
    s = gen.scan_m2_inputs(Bt, H, P, N, L, io="f32", seed=seed, tag="prop_c", h0=True)
    y, _ = oracle.scan_mamba2(s.x, s.dt, s.A, s.B, s.C, D=s.D, z=s.z, dt_bias=s.dt_bias, h0=s.h0)
    late = lambda a, name: np.concatenate(  # noqa: E731
        [a[..., :cut], gen.normal(a[..., cut:].shape, "prop_c2", seed, name)], -1)
    y2, _ = oracle.scan_mamba2(late(s.x, "x"), late(s.dt, "dt"), s.A, late(s.B, "B"), late(s.C, "C"),
                               D=s.D, z=late(s.z, "z"), dt_bias=s.dt_bias, h0=s.h0)
    np.testing.assert_array_equal(y2[..., :cut], y[..., :cut])
    assert not np.array_equal(y2[..., cut:], y[..., cut:])


@settings(**SETTINGS)
@given(Bt=st.integers(1, 2), D=st.integers(2, 5), L=st.integers(1, 12), N=st.integers(1, 4),
       W=st.sampled_from([0, 4]), pick=st.integers(0, 10**6), seed=st.integers(0, 10**6))
def test_mamba1_channels_are_independent(Bt, D, L, N, W, pick, seed):
    """Channel d's x, dt, z, A row, D, dt_bias, conv weights and states affect
    channel d's outputs and states only (B and C are shared)."""
    d = pick % D
    s = gen.scan_inputs(Bt, L, D, N, W=W, io="f32", seed=seed, tag="prop_i", conv_state=W > 0, h0=True)

    def run(t):
        return oracle.scan(t.x, t.dt, t.A, t.B, t.C, z=t.z, D=t.D, dt_bias=t.dt_bias,
                           conv_weight=t.conv_weight, conv_bias=t.conv_bias, conv_state=t.conv_state, h0=t.h0)

    y, hf, csf = run(s)
    o = gen.scan_inputs(Bt, L, D, N, W=W, io="f32", seed=seed + 1, tag="prop_i", conv_state=W > 0, h0=True)
    for name, axis in (("x", 1), ("dt", 1), ("z", 1), ("A", 0), ("D", 0), ("dt_bias", 0), ("h0", 1),
                       ("conv_weight", 0), ("conv_bias", 0), ("conv_state", 1)):
        a, b = getattr(s, name), getattr(o, name)
        if a is None:
            continue
        a = a.copy()
        idx = [slice(None)] * a.ndim
        idx[axis] = d
        a[tuple(idx)] = b[tuple(idx)]
        setattr(s, name, a)
    y2, hf2, csf2 = run(s)
    keep = [k for k in range(D) if k != d]
    np.testing.assert_array_equal(y2[:, keep], y[:, keep])
    np.testing.assert_array_equal(hf2[:, keep], hf[:, keep])
    if W > 0:
        np.testing.assert_array_equal(csf2[:, keep], csf[:, keep])


@settings(**SETTINGS)
@given(Bt=st.integers(1, 2), H=st.integers(1, 3), P=st.integers(1, 3), N=st.integers(1, 5),
       L=st.integers(4, 16), R=st.integers(2, 4), seed=st.integers(0, 10**6))
def test_mamba2_prefill_context_parallel_decomposition(Bt, H, P, N, L, R, seed):
    """A sequence cut into R pieces, each scanned from a zero state, is put
    back together by composing the pieces' carries h -> Lambda*h + h_r (Lambda
    the head's decay over the piece) and adding, at each step t of a piece,
    silu(z_t) * C_t . (lambda_t * h_in), lambda_t the decay since the piece began."""
    s = gen.scan_m2_inputs(Bt, H, P, N, L, io="f32", seed=seed, tag="prop_cp", h0=True)
    full, hfull = oracle.scan_mamba2(s.x, s.dt, s.A, s.B, s.C, D=s.D, z=s.z, dt_bias=s.dt_bias, h0=s.h0)
    delta = np.vectorize(oracle.softplus)(s.dt + s.dt_bias[None, :, None])  # (B, H, L)
    cuts = np.linspace(0, L, R + 1).astype(int)
    h_in = s.h0.copy()  # (B, H, P, N): the true state entering the current piece
    for r in range(R):
        sl = slice(cuts[r], cuts[r + 1])
        y0, h_r = oracle.scan_mamba2(s.x[..., sl], s.dt[..., sl], s.A, s.B[..., sl], s.C[..., sl], D=s.D,
                                     z=s.z[..., sl], dt_bias=s.dt_bias, h0=None)
        lam = np.exp(np.cumsum(delta[..., sl], -1) * s.A[None, :, None])  # (B, H, Lr)
        carry = np.einsum("bnt,bhpn->bhpt", s.C[:, 0, :, sl], h_in) * lam[:, :, None, :]  # one group
        silu_z = s.z[..., sl] / (1.0 + np.exp(-s.z[..., sl]))
        np.testing.assert_allclose(y0 + silu_z * carry, full[..., sl], rtol=1e-9, atol=1e-11)
        h_in = lam[..., -1][:, :, None, None] * h_in + h_r
    np.testing.assert_allclose(h_in, hfull, rtol=1e-9, atol=1e-11)


@settings(**SETTINGS)
@given(Bt=st.integers(1, 2), D=st.integers(1, 4), N=st.integers(1, 5), L=st.integers(4, 16),
       R=st.integers(2, 4), W=st.sampled_from([0, 4]), seed=st.integers(0, 10**6))
def test_mamba1_prefill_context_parallel_decomposition(Bt, D, N, L, R, W, seed):
    """The same decomposition in the Mamba-1 layout: the decay is per (d, n)
    element, and a piece's conv history is the W raw inputs before it."""
    s = gen.scan_inputs(Bt, L, D, N, W=W, io="f32", seed=seed, tag="prop_cp1", conv_state=W > 0, h0=True)
    kw = dict(D=s.D, dt_bias=s.dt_bias, conv_weight=s.conv_weight, conv_bias=s.conv_bias)
    full, hfull, _ = oracle.scan(s.x, s.dt, s.A, s.B, s.C, z=s.z, conv_state=s.conv_state, h0=s.h0, **kw)
    delta = np.vectorize(oracle.softplus)(s.dt + s.dt_bias[None, :, None])  # (B, D, L)
    raw = np.concatenate([s.conv_state, s.x], -1) if W else None  # W history entries, then x
    cuts = np.linspace(0, L, R + 1).astype(int)
    h_in = s.h0.copy()  # (B, D, N)
    for r in range(R):
        sl = slice(cuts[r], cuts[r + 1])
        cs = raw[..., cuts[r]:cuts[r] + W].copy() if W else None
        y0, h_r, _ = oracle.scan(s.x[..., sl], s.dt[..., sl], s.A, s.B[..., sl], s.C[..., sl], z=s.z[..., sl],
                                 conv_state=cs, h0=None, **kw)
        lam = np.exp(np.cumsum(delta[..., sl], -1)[:, :, None, :] * s.A[None, :, :, None])  # (B, D, N, Lr)
        carry = np.einsum("bnt,bdnt,bdn->bdt", s.C[:, 0, :, sl], lam, h_in)  # one group
        silu_z = s.z[..., sl] / (1.0 + np.exp(-s.z[..., sl]))
        np.testing.assert_allclose(y0 + silu_z * carry, full[..., sl], rtol=1e-9, atol=1e-11)
        h_in = lam[..., -1] * h_in + h_r
    np.testing.assert_allclose(h_in, hfull, rtol=1e-9, atol=1e-11)


# ---- double-gated short causal conv (reading: out = Cg * conv(Bg * x))
@settings(**SETTINGS)
@given(Bt=st.integers(1, 2), D=st.integers(1, 5), L=st.integers(2, 24), W=st.integers(1, 8),
       frac=st.floats(0.05, 0.95), seed=st.integers(0, 10**6))
def test_gated_conv_split_anywhere(Bt, D, L, W, frac, seed):
    """A sequence cut anywhere, the conv state carried across, equals one call."""
    split = max(1, min(L - 1, int(L * frac)))
    s = gen.gated_conv_inputs(Bt, L, D, W, io="f32", seed=seed, tag="prop_gc", conv_state=True)
    full, csf = oracle.gated_conv1d(s.x, s.bg, s.cg, s.weight, bias=s.bias, conv_state=s.conv_state)
    a, b = slice(0, split), slice(split, L)
    o1, cs1 = oracle.gated_conv1d(s.x[..., a], s.bg[..., a], s.cg[..., a], s.weight, bias=s.bias,
                                  conv_state=s.conv_state)
    o2, cs2 = oracle.gated_conv1d(s.x[..., b], s.bg[..., b], s.cg[..., b], s.weight, bias=s.bias, conv_state=cs1)
    np.testing.assert_allclose(np.concatenate([o1, o2], -1), full, rtol=1e-13, atol=1e-14)
    np.testing.assert_array_equal(cs2, csf)


@settings(**SETTINGS)
@given(D=st.integers(1, 5), L=st.integers(1, 16), W=st.integers(1, 6), alpha=st.floats(-3, 3),
       seed=st.integers(0, 10**6))
def test_gated_conv_linear_in_x_with_the_gates_fixed(D, L, W, alpha, seed):
    """Without bias and state, x -> out is linear for fixed gates."""
    s = gen.gated_conv_inputs(1, L, D, W, io="f32", seed=seed, tag="prop_gc_lin", bias=False)
    x2 = gen.normal(s.x.shape, seed, "prop_gc_lin", "x2")
    f = lambda x: oracle.gated_conv1d(x, s.bg, s.cg, s.weight)[0]  # noqa: E731
    np.testing.assert_allclose(f(s.x + alpha * x2), f(s.x) + alpha * f(x2), rtol=1e-11, atol=1e-12)


@settings(**SETTINGS)
@given(Bt=st.integers(1, 2), D=st.integers(1, 4), L=st.integers(2, 16), W=st.integers(1, 8),
       frac=st.floats(0.05, 0.95), seed=st.integers(0, 10**6))
def test_gated_conv_is_causal_with_a_window_of_W(Bt, D, L, W, frac, seed):
    """Changing x, Bg and Cg from step t on leaves outputs before t
    bit-identical; changing only the input gate at step t moves outputs t ..
    t+W-1 at most."""
    t = max(1, min(L - 1, int(L * frac)))
    s = gen.gated_conv_inputs(Bt, L, D, W, io="f32", seed=seed, tag="prop_gc_causal", conv_state=True)
    base, _ = oracle.gated_conv1d(s.x, s.bg, s.cg, s.weight, bias=s.bias, conv_state=s.conv_state)
    x2, bg2, cg2 = s.x.copy(), s.bg.copy(), s.cg.copy()
    x2[..., t:] += 1.0
    bg2[..., t:] -= 0.5
    cg2[..., t:] *= 2.0
    moved, _ = oracle.gated_conv1d(x2, bg2, cg2, s.weight, bias=s.bias, conv_state=s.conv_state)
    np.testing.assert_array_equal(moved[..., :t], base[..., :t])
    bg3 = s.bg.copy()
    bg3[..., t] += 1.0
    only, _ = oracle.gated_conv1d(s.x, bg3, s.cg, s.weight, bias=s.bias, conv_state=s.conv_state)
    np.testing.assert_array_equal(only[..., :t], base[..., :t])
    np.testing.assert_array_equal(only[..., t + W:], base[..., t + W:])
