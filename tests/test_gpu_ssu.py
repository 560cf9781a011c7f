"""GPU parity of the single-token state update (ssm_selective_state_update)
against the fp64 oracle, both layouts, through the C ABI."""
import numpy as np
import pytest

import oracle
from state_space_model_causal_b200 import inputs as gen
from tests.parity import TOL, N, T, assert_close

pytestmark = pytest.mark.gpu


def _ssu(**kw):
    from state_space_model_causal_b200 import ssm_selective_state_update
    return ssm_selective_state_update(**kw)


# ------------------------------------------------------------------ Mamba-1 --
def _m1_gpu(s, conv_state_dtype=None):
    cs_dt = conv_state_dtype or s.conv_state_dtype
    st = T(s.state, s.state_dtype)
    cs = T(s.conv_state, cs_dt)
    out = _ssu(state=st, x=T(s.x, s.io), dt=T(s.dt, s.io), A=T(s.A, "f32"), B=T(s.B, s.io),
               C=T(s.C, s.io), D=T(s.D, "f32"), z=T(s.z, s.io), dt_bias=T(s.dt_bias, "f32"),
               conv_weight=T(s.conv_weight, "f32"), conv_bias=T(s.conv_bias, "f32"), conv_state=cs)
    return out, st, cs


def _m1_oracle(s):
    Bt, D, N_ = s.state.shape
    o, st, cs = oracle.ssu(s.state[:, :, None, :], s.x[:, :, None], s.dt[:, :, None], s.A[:, None, :],
                           s.B, s.C, D=s.D[:, None], z=None if s.z is None else s.z[:, :, None],
                           dt_bias=s.dt_bias[:, None], conv_weight=s.conv_weight,
                           conv_bias=s.conv_bias, conv_state=s.conv_state)
    return o[:, :, 0], st[:, :, 0], None if cs is None else cs.reshape(Bt, D, -1)


def test_decode_2p8b_full_layer():
    """Mamba-1 2.8B-shaped decode step: B=245, D=5120, N=16, W=4, fp32 state
    and conv state, fp16 x/dt/z/B/C; every row compared."""
    import torch
    s = gen.decode_2p8b(slab=0)
    out, st, cs = _m1_gpu(s)
    torch.cuda.synchronize()
    o, sref, csref = _m1_oracle(s)
    assert_close(N(out), o, TOL["f16"], "out")
    assert_close(N(st), sref, TOL["f16"], "state")
    np.testing.assert_array_equal(N(cs), csref)


@pytest.mark.parametrize("state_dt,io", [("f32", "f32"), ("f16", "f16"), ("bf16", "bf16"),
                                         ("f32", "bf16")])
@pytest.mark.parametrize("N_", [16, 8, 32, 5])
def test_mamba1_dtypes_and_dstate(state_dt, io, N_):
    s = gen.ssu_mamba1_inputs(7, 96, N_, W=4, io=io, state=state_dt, seed=1, tag=f"m1{N_}")
    out, st, cs = _m1_gpu(s)
    o, sref, csref = _m1_oracle(s)
    tol = TOL[io] if state_dt == "f32" else TOL["f16"]
    assert_close(N(out), o, tol, "out")
    assert_close(N(st), sref, tol, "state")
    np.testing.assert_array_equal(N(cs), csref)


def test_mamba1_multi_step_decode():
    """Three consecutive decode steps on the same caches."""
    import torch
    s = gen.ssu_mamba1_inputs(9, 64, 16, W=4, io="f32", state="f32", seed=2, tag="steps")
    st = T(s.state, "f32")
    cs = T(s.conv_state, "f32")
    sref, csref = s.state, s.conv_state
    for k in range(3):
        x = gen.round_to(gen.normal((9, 64), "steps", k, "x"), "f32")
        out = _ssu(state=st, x=T(x, "f32"), dt=T(s.dt, "f32"), A=T(s.A, "f32"), B=T(s.B, "f32"),
                   C=T(s.C, "f32"), D=T(s.D, "f32"), z=T(s.z, "f32"), dt_bias=T(s.dt_bias, "f32"),
                   conv_weight=T(s.conv_weight, "f32"), conv_bias=T(s.conv_bias, "f32"),
                   conv_state=cs)
        torch.cuda.synchronize()
        s2 = gen.SsuInputs(sref, x, s.dt, s.A, s.B, s.C, s.D, s.z, s.dt_bias, s.conv_weight,
                           s.conv_bias, csref)
        o, sref, csref = _m1_oracle(s2)
        assert_close(N(out), o, 1e-5, f"out step {k}")
    assert_close(N(st), sref, 1e-5, "state")
    np.testing.assert_array_equal(N(cs), csref)


def test_mamba1_without_conv_and_fp16_conv_state():
    s = gen.ssu_mamba1_inputs(5, 32, 16, W=0, io="f16", state="f32", seed=3, tag="noconv")
    st = T(s.state, "f32")
    out = _ssu(state=st, x=T(s.x, "f16"), dt=T(s.dt, "f16"), A=T(s.A, "f32"), B=T(s.B, "f16"),
               C=T(s.C, "f16"), D=T(s.D, "f32"), z=T(s.z, "f16"), dt_bias=T(s.dt_bias, "f32"))
    o, sref, _ = _m1_oracle(s)
    assert_close(N(out), o, TOL["f16"], "out")
    assert_close(N(st), sref, TOL["f16"], "state")
    s = gen.ssu_mamba1_inputs(5, 32, 16, W=4, io="f16", state="f32", conv_state_dtype="f16",
                              seed=4, tag="cs16")
    out, st, cs = _m1_gpu(s)
    o, sref, csref = _m1_oracle(s)
    assert_close(N(out), o, TOL["f16"], "out")
    np.testing.assert_array_equal(N(cs), csref)


# ------------------------------------------------------------------ Mamba-2 --
def _m2_gpu(s, **extra):
    st = T(s.state, s.state_dtype)
    out = _ssu(state=st, x=T(s.x, s.io), dt=T(s.dt, s.io), A=T(s.A, "f32"), B=T(s.B, s.io),
               C=T(s.C, s.io), D=T(s.D, "f32"), z=T(s.z, s.io), dt_bias=T(s.dt_bias, "f32"), **extra)
    return out, st


def _m2_oracle(s):
    if s.dt.ndim == 2:
        return oracle.ssu_mamba2(s.state, s.x, s.dt, s.A, s.B, s.C, D=s.D, z=s.z, dt_bias=s.dt_bias)
    o, st, _ = oracle.ssu(s.state, s.x, s.dt, s.A[:, None, None], s.B, s.C, D=s.D[:, None], z=s.z,
                          dt_bias=s.dt_bias[:, None])
    return o, st


@pytest.mark.parametrize("cache", ["f16", "f32"])
@pytest.mark.parametrize("R", [8, 80, 1024, 8192])
def test_mamba2_64x128_effective_batch(cache, R):
    """H=80, P=64, N=128, G=1, fp16 inputs, fp16/fp32 cache."""
    import torch
    s = gen.mamba2_64x128(R, cache=cache)
    out, st = _m2_gpu(s)
    torch.cuda.synchronize()
    o, sref = _m2_oracle(s)
    assert_close(N(out), o, TOL["f16"], "out")
    assert_close(N(st), sref, TOL["f16"], "state")


def test_mamba2_launch_sizes_in_any_order():
    """The library opts each kernel into its shared memory once and remembers
    it; launches of one kernel with stages of different sizes, largest first,
    then smaller, then between, then the largest again, must all run and
    match the oracle (a remembered size must never meet a lower limit)."""
    import torch
    for R in (1024, 8, 80, 1024, 16):
        s = gen.mamba2_64x128(R, cache="f16")
        out, st = _m2_gpu(s)
        torch.cuda.synchronize()
        o, sref = _m2_oracle(s)
        assert_close(N(out), o, TOL["f16"], f"out R={R}")
        assert_close(N(st), sref, TOL["f16"], f"state R={R}")


@pytest.mark.parametrize("cache", ["bf16", "f32"])
@pytest.mark.parametrize("R", [8, 32, 512, 2048])
def test_mamba2_128x256_effective_batch(cache, R):
    """H=32, P=128, N=256, G=1, bf16 inputs, bf16/fp32 cache."""
    import torch
    s = gen.mamba2_128x256(R, cache=cache)
    out, st = _m2_gpu(s)
    torch.cuda.synchronize()
    o, sref = _m2_oracle(s)
    assert_close(N(out), o, TOL["bf16"], "out")
    assert_close(N(st), sref, TOL["bf16"], "state")


def _full_size_sampled(H, P, N_, R, cache, io, samples=24):
    """Largest effective batch, inputs drawn on the device; sampled (b, h)
    rows are copied out before the in-place update and checked one by one."""
    import torch
    Bt, Hr = gen.effective_batch_shape(R, H)
    tag = ("full", H, P, N_, R, cache)
    st = gen.device_normal((Bt, Hr, P, N_), cache, *tag, "state")
    x = gen.device_normal((Bt, Hr, P), io, *tag, "x")
    dt = gen.device_uniform((Bt, Hr), -4.0, -1.0, io, *tag, "dt")
    Bm = gen.device_normal((Bt, 1, N_), io, *tag, "B")
    Cm = gen.device_normal((Bt, 1, N_), io, *tag, "C")
    A = T(gen.round_to(-gen.uniform((Hr,), 1.0, 16.0, *tag, "A"), "f32"), "f32")
    db = T(gen.round_to(gen.dt_bias_draw((Hr,), *tag, "db"), "f32"), "f32")
    Dv = torch.ones(Hr, device="cuda")
    rng = np.random.default_rng(7)
    picks = [(int(b), int(h)) for b, h in zip(rng.integers(0, Bt, samples), rng.integers(0, Hr, samples))]
    picks += [(0, 0), (Bt - 1, Hr - 1)]
    before = {bh: N(st[bh[0], bh[1]]) for bh in picks}
    out = _ssu(state=st, x=x, dt=dt, A=A, B=Bm, C=Cm, D=Dv, dt_bias=db)
    torch.cuda.synchronize()
    An, dbn = N(A), N(db)
    for (b, h), s0 in before.items():
        o, sref = oracle.ssu_mamba2(s0[None, None], N(x[b, h])[None, None], N(dt[b, h]).reshape(1, 1),
                                    An[h:h + 1], N(Bm[b])[None], N(Cm[b])[None], D=np.ones(1),
                                    dt_bias=dbn[h:h + 1])
        assert_close(N(out[b, h]), o[0, 0], TOL[io], f"out[{b},{h}]")
        assert_close(N(st[b, h]), sref[0, 0], TOL[io], f"state[{b},{h}]")
    del st
    torch.cuda.empty_cache()


@pytest.mark.parametrize("cache", ["f16", "f32"])
def test_mamba2_64x128_largest_effective_batch_sampled(cache):
    _full_size_sampled(80, 64, 128, 131072, cache, "f16")


@pytest.mark.parametrize("cache", ["bf16", "f32"])
def test_mamba2_128x256_largest_effective_batch_sampled(cache):
    _full_size_sampled(32, 128, 256, 65536, cache, "bf16")


@pytest.mark.parametrize("G", [2, 4])
def test_mamba2_groups(G):
    s = gen.ssu_mamba2_inputs(3, 8, 16, 64, G=G, io="f16", state="f32", seed=5, tag=f"g{G}",
                              with_z=True)
    out, st = _m2_gpu(s)
    o, sref = _m2_oracle(s)
    assert_close(N(out), o, TOL["f16"], "out")
    assert_close(N(st), sref, TOL["f16"], "state")


def test_mamba2_dt_per_row_and_full_A_and_no_D():
    import torch
    s = gen.ssu_mamba2_inputs(3, 4, 16, 32, io="f32", state="f32", seed=6, tag="perrow",
                              dt_per_head=False, with_z=True, with_D=False)
    Afull = np.ascontiguousarray(np.broadcast_to(s.A[:, None, None], (4, 16, 32)) *
                                 (1.0 + 0.01 * np.arange(32)))
    st = T(s.state, "f32")
    out = _ssu(state=st, x=T(s.x, "f32"), dt=T(s.dt, "f32"), A=T(Afull, "f32"), B=T(s.B, "f32"),
               C=T(s.C, "f32"), z=T(s.z, "f32"), dt_bias=T(s.dt_bias, "f32"))
    torch.cuda.synchronize()
    o, sref, _ = oracle.ssu(s.state, s.x, s.dt, Afull, s.B, s.C, z=s.z, dt_bias=s.dt_bias[:, None])
    assert_close(N(out), o, 1e-5, "out")
    assert_close(N(st), sref, 1e-5, "state")


def test_mamba2_slot_indices_with_padding_rows():
    """Continuous batching: 5 requests over a pool of 9 cache slots, one
    padding row (-1) that must leave everything untouched."""
    import torch
    pool = gen.ssu_mamba2_inputs(9, 6, 8, 64, io="f16", state="f16", seed=7, tag="pool")
    s = gen.ssu_mamba2_inputs(5, 6, 8, 64, io="f16", state="f16", seed=8, tag="req", with_z=True)
    idx = np.array([4, 0, -1, 7, 2], dtype=np.int32)
    st = T(pool.state, "f16")
    out0 = torch.full((5, 6, 8), 7.0, dtype=torch.float16, device="cuda")
    _ssu(state=st, x=T(s.x, "f16"), dt=T(s.dt, "f16"), A=T(s.A, "f32"), B=T(s.B, "f16"),
         C=T(s.C, "f16"), D=T(s.D, "f32"), z=T(s.z, "f16"), dt_bias=T(s.dt_bias, "f32"),
         state_batch_indices=torch.from_numpy(idx).cuda(), out=out0)
    torch.cuda.synchronize()
    got_state, got_out = N(st), N(out0)
    expect_state = pool.state.copy()
    for b, slot in enumerate(idx):
        if slot < 0:
            assert np.all(got_out[b] == 7.0)
            continue
        o, sref = oracle.ssu_mamba2(pool.state[slot:slot + 1], s.x[b:b + 1], s.dt[b:b + 1], s.A,
                                    s.B[b:b + 1], s.C[b:b + 1], D=s.D, z=s.z[b:b + 1],
                                    dt_bias=s.dt_bias)
        expect_state[slot] = sref[0]
        assert_close(got_out[b], o[0], TOL["f16"], f"out[{b}]")
    untouched = [k for k in range(9) if k not in idx]
    np.testing.assert_array_equal(got_state[untouched], pool.state[untouched])
    assert_close(got_state, expect_state, TOL["f16"], "pool")


def test_mamba2_strided_state_view_and_generic_layouts():
    """State as a view into a larger pool (non-contiguous batch dim), and a
    layout whose dstate is not contiguous (generic kernel)."""
    import torch
    s = gen.ssu_mamba2_inputs(4, 6, 8, 64, io="f16", state="f32", seed=9, tag="view", with_z=True)
    big = torch.zeros(4, 10, 8, 64, device="cuda")
    big[:, 2:8] = T(s.state, "f32")
    view = big[:, 2:8]
    out, _ = _m2_gpu(s)  # reference run of the same problem on a dense copy
    out2 = _ssu(state=view, x=T(s.x, "f16"), dt=T(s.dt, "f16"), A=T(s.A, "f32"), B=T(s.B, "f16"),
                C=T(s.C, "f16"), D=T(s.D, "f32"), z=T(s.z, "f16"), dt_bias=T(s.dt_bias, "f32"))
    torch.cuda.synchronize()
    o, sref = _m2_oracle(s)
    assert_close(N(out2), o, TOL["f16"], "out (view)")
    assert_close(N(view), sref, TOL["f16"], "state (view)")
    assert torch.count_nonzero(big[:, :2]) == 0 and torch.count_nonzero(big[:, 8:]) == 0
    # dstate-major storage: element (b,h,p,n) at n*B*H*P + ...
    tr = T(np.ascontiguousarray(np.moveaxis(s.state, -1, 0)), "f32")
    stg = tr.permute(1, 2, 3, 0)
    out3 = _ssu(state=stg, x=T(s.x, "f16"), dt=T(s.dt, "f16"), A=T(s.A, "f32"), B=T(s.B, "f16"),
                C=T(s.C, "f16"), D=T(s.D, "f32"), z=T(s.z, "f16"), dt_bias=T(s.dt_bias, "f32"))
    torch.cuda.synchronize()
    assert_close(N(out3), o, TOL["f16"], "out (generic)")
    assert_close(N(stg), sref, TOL["f16"], "state (generic)")


def test_empty_batch_is_a_no_op():
    import torch
    st = torch.zeros(0, 4, 8, 16, device="cuda")
    x = torch.zeros(0, 4, 8, device="cuda")
    out = _ssu(state=st, x=x, dt=torch.zeros(0, 4, device="cuda"), A=torch.ones(4, device="cuda"),
               B=torch.zeros(0, 1, 16, device="cuda"), C=torch.zeros(0, 1, 16, device="cuda"))
    torch.cuda.synchronize()
    assert out.shape == (0, 4, 8)


def test_mamba2_dt_per_row_with_scalar_A():
    """dt given per (head, headdim) row with one A per head: the bulk-copy
    kernel's per-row discretisation branch."""
    import torch
    s = gen.ssu_mamba2_inputs(5, 6, 32, 128, io="f16", state="f16", seed=11, tag="dtrow",
                              dt_per_head=False, with_z=True)
    out, st = _m2_gpu(s)
    torch.cuda.synchronize()
    o, sref = _m2_oracle(s)
    assert_close(N(out), o, TOL["f16"], "out")
    assert_close(N(st), sref, TOL["f16"], "state")


def test_bulk_copy_kernels_leave_the_device_error_word_clear():
    import torch
    from state_space_model_causal_b200 import LaunchInfo, ssm_device_error
    s = gen.mamba2_64x128(4096, cache="f16")
    info = LaunchInfo()
    st = T(s.state, "f16")
    from state_space_model_causal_b200 import ssm_selective_state_update
    ssm_selective_state_update(st, T(s.x, "f16"), T(s.dt, "f16"), T(s.A, "f32"), T(s.B, "f16"),
                               T(s.C, "f16"), D=T(s.D, "f32"), dt_bias=T(s.dt_bias, "f32"), info=info)
    assert info.as_dict()["kernel"] == "ssu_tma"
    assert ssm_device_error() == 0
    torch.cuda.synchronize()


def test_mamba1_slot_indices_with_padding_rows():
    """Mamba-1 decode over a pool of 6 cache slots (state and conv state) for 4
    requests, one of them a padding row; the bulk-copy kernel must leave the
    padding row's output and every unused slot untouched."""
    import torch
    pool = gen.ssu_mamba1_inputs(6, 64, 16, W=4, io="f16", state="f32", seed=12, tag="pool1")
    s = gen.ssu_mamba1_inputs(4, 64, 16, W=4, io="f16", state="f32", seed=13, tag="req1")
    idx = np.array([5, -1, 0, 3], dtype=np.int32)
    st = T(pool.state, "f32")
    cs = T(pool.conv_state, "f32")
    out = torch.full((4, 64), 3.0, dtype=torch.float16, device="cuda")
    from state_space_model_causal_b200 import LaunchInfo
    info = LaunchInfo()
    _ssu(state=st, x=T(s.x, "f16"), dt=T(s.dt, "f16"), A=T(s.A, "f32"), B=T(s.B, "f16"),
         C=T(s.C, "f16"), D=T(s.D, "f32"), z=T(s.z, "f16"), dt_bias=T(s.dt_bias, "f32"),
         conv_weight=T(s.conv_weight, "f32"), conv_bias=T(s.conv_bias, "f32"), conv_state=cs,
         state_batch_indices=torch.from_numpy(idx).cuda(), out=out, info=info)
    torch.cuda.synchronize()
    assert info.as_dict()["kernel"] == "ssu_row_tma"
    got_st, got_cs, got_out = N(st), N(cs), N(out)
    for b, slot in enumerate(idx):
        if slot < 0:
            assert np.all(got_out[b] == 3.0)
            continue
        one = gen.SsuInputs(pool.state[slot:slot + 1], s.x[b:b + 1], s.dt[b:b + 1], s.A,
                            s.B[b:b + 1], s.C[b:b + 1], s.D, s.z[b:b + 1], s.dt_bias,
                            s.conv_weight, s.conv_bias, pool.conv_state[slot:slot + 1])
        o, sref, csref = _m1_oracle(one)
        assert_close(got_out[b], o[0], TOL["f16"], f"out[{b}]")
        assert_close(got_st[slot], sref[0], TOL["f16"], f"state[{slot}]")
        np.testing.assert_array_equal(got_cs[slot], csref[0])
    for slot in (1, 2, 4):
        np.testing.assert_array_equal(got_st[slot], pool.state[slot])
        np.testing.assert_array_equal(got_cs[slot], pool.conv_state[slot])


# ------------------------------------------------- several steps, 16-bit caches --
@pytest.mark.parametrize("cache,io,P,N_", [("f16", "f16", 64, 128), ("bf16", "bf16", 128, 256)])
def test_mamba2_multi_step_decode_16bit_cache(cache, io, P, N_):
    """Eight consecutive decode steps on one fp16 / bf16 cache.  The GPU stores
    the state rounded to the cache dtype after every step; the oracle rounds
    its fp64 state the same way (cache_dtype), so outputs and the cache stay
    comparable step after step."""
    import torch
    s = gen.ssu_mamba2_inputs(4, 8, P, N_, io=io, state=cache, seed=41, tag=f"steps{cache}", with_z=True)
    st = T(s.state, cache)
    sref = s.state
    for k in range(8):
        tg = ("steps16", cache, k)
        x = gen.round_to(gen.normal((4, 8, P), *tg, "x"), io)
        dt = gen.round_to(gen.uniform((4, 8), -4.0, -1.0, *tg, "dt"), io)
        Bm = gen.round_to(gen.normal((4, 1, N_), *tg, "B"), io)
        Cm = gen.round_to(gen.normal((4, 1, N_), *tg, "C"), io)
        z = gen.round_to(gen.normal((4, 8, P), *tg, "z"), io)
        out = _ssu(state=st, x=T(x, io), dt=T(dt, io), A=T(s.A, "f32"), B=T(Bm, io), C=T(Cm, io),
                   D=T(s.D, "f32"), z=T(z, io), dt_bias=T(s.dt_bias, "f32"))
        torch.cuda.synchronize()
        o, sref = oracle.ssu_mamba2(sref, x, dt, s.A, Bm, Cm, D=s.D, z=z, dt_bias=s.dt_bias,
                                    cache_dtype=cache)
        assert_close(N(out), o, TOL[io], f"out step {k}")
        assert_close(N(st), sref, TOL[io], f"cache after step {k}", ulps=k + 1)


@pytest.mark.parametrize("cache", ["f16", "bf16"])
def test_mamba1_multi_step_decode_16bit_cache(cache):
    """Six consecutive Mamba-1 decode steps (fused conv roll) on a 16-bit ssm
    cache, compared step by step with the oracle rounding its state the same way."""
    import torch
    io = cache
    s = gen.ssu_mamba1_inputs(9, 64, 16, W=4, io=io, state=cache, seed=42, tag=f"m1steps{cache}")
    st = T(s.state, cache)
    cs = T(s.conv_state, "f32")
    sref, csref = s.state, s.conv_state
    for k in range(6):
        tg = ("m1steps16", cache, k)
        x = gen.round_to(gen.normal((9, 64), *tg, "x"), io)
        dt = gen.round_to(gen.uniform((9, 64), -4.0, -1.0, *tg, "dt"), io)
        out = _ssu(state=st, x=T(x, io), dt=T(dt, io), A=T(s.A, "f32"), B=T(s.B, io), C=T(s.C, io),
                   D=T(s.D, "f32"), z=T(s.z, io), dt_bias=T(s.dt_bias, "f32"),
                   conv_weight=T(s.conv_weight, "f32"), conv_bias=T(s.conv_bias, "f32"), conv_state=cs)
        torch.cuda.synchronize()
        o, st_ref, cs_ref = oracle.ssu(sref[:, :, None, :], x[:, :, None], dt[:, :, None], s.A[:, None, :],
                                       s.B, s.C, D=s.D[:, None], z=s.z[:, :, None],
                                       dt_bias=s.dt_bias[:, None], conv_weight=s.conv_weight,
                                       conv_bias=s.conv_bias, conv_state=csref, cache_dtype=cache)
        sref, csref = st_ref[:, :, 0], cs_ref.reshape(9, 64, -1)
        assert_close(N(out), o[:, :, 0], TOL[io], f"out step {k}")
        assert_close(N(st), sref, TOL[io], f"cache after step {k}", ulps=k + 1)
    np.testing.assert_array_equal(N(cs), csref)
