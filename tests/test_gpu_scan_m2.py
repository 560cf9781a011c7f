"""GPU parity of the Mamba-2-layout prefill (ssm_selective_scan_fwd with a
rank-4 x) against the fp64 oracle, on the same seeded inputs, through the C
ABI.  The fast kernel reads the time-major memory of the Mamba-2 model: x
stored as (B, L, H, P) and passed as its (B, H, P, L) view."""
import numpy as np
import pytest

import oracle
from state_space_model_causal_b200 import inputs as gen
from tests.parity import TOL, N, T, assert_close

pytestmark = pytest.mark.gpu


def _time_major(a, dtype, perm):
    """Store a (logical layout) array in memory order `perm` and return the
    logical view of that storage."""
    import torch
    store = T(np.ascontiguousarray(np.transpose(a, perm)), dtype)
    inv = np.argsort(perm)
    return store.permute(*[int(i) for i in inv])


def run_m2_gpu(s, *, layout="time_major", with_state=True, softplus=True, info=None):
    import torch
    from state_space_model_causal_b200 import ssm_selective_scan_fwd
    io = s.io
    Bt, H, P, L = s.x.shape
    N_ = s.B.shape[2]
    if layout == "time_major":
        x = _time_major(s.x, io, (0, 3, 1, 2))
        z = _time_major(s.z, io, (0, 3, 1, 2)) if s.z is not None else None
        dt = _time_major(s.dt, io, (0, 2, 1))
        Bm = _time_major(s.B, io, (0, 3, 1, 2))
        Cm = _time_major(s.C, io, (0, 3, 1, 2))
        out = _time_major(np.zeros(s.x.shape), io, (0, 3, 1, 2))
    else:
        x, dt, Bm, Cm = T(s.x, io), T(s.dt, io), T(s.B, io), T(s.C, io)
        z = T(s.z, io) if s.z is not None else None
        out = torch.empty_like(x)
    h = None
    if with_state:
        h = T(s.h0 if s.h0 is not None else np.zeros((Bt, H, P, N_)), "f32")
    ssm_selective_scan_fwd(x, dt, T(s.A, "f32"), Bm, Cm, D=T(s.D, "f32"), z=z,
                           dt_bias=T(s.dt_bias, "f32"), dt_softplus=softplus, ssm_state=h, out=out,
                           info=info)
    torch.cuda.synchronize()
    return N(out), N(h)


def run_m2_oracle(s, softplus=True):
    return oracle.scan_mamba2(s.x, s.dt, s.A, s.B, s.C, D=s.D, z=s.z, dt_bias=s.dt_bias,
                              dt_softplus=softplus, h0=s.h0)


def _check(s, *, layout="time_major", kernel=None, tol=None, with_state=True, softplus=True):
    from state_space_model_causal_b200 import LaunchInfo
    info = LaunchInfo()
    out, h = run_m2_gpu(s, layout=layout, with_state=with_state, softplus=softplus, info=info)
    if kernel:
        assert info.as_dict()["kernel"] == kernel
    ref, href = run_m2_oracle(s, softplus=softplus)
    tol = tol or (1e-5 if s.io == "f32" else TOL[s.io])
    assert_close(out, ref, tol, "out")
    if with_state:
        assert_close(h, href, tol, "ssm_state")


def test_m2_prefill_fp32_ragged_chunk_groups():
    """fp32, N=64, P=8 (one partial row block), L=40 (ragged last chunk), two
    groups, incoming state."""
    s = gen.scan_m2_inputs(2, 4, 8, 64, 40, G=2, io="f32", seed=1, tag="m2a", h0=True)
    _check(s, kernel="scan_m2")


@pytest.mark.parametrize("io", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("N_,P", [(64, 64), (128, 64), (128, 24), (256, 64), (256, 40)])
def test_m2_prefill_fast_kernel_variants(io, N_, P):
    s = gen.scan_m2_inputs(2, 3, P, N_, 37, io=io, seed=2, tag=f"m2v{N_}{P}{io}", h0=True)
    _check(s, kernel="scan_m2")


@pytest.mark.parametrize("N_,P,layout", [(16, 8, "time_major"), (48, 8, "time_major"),
                                          (128, 6, "time_major"), (128, 8, "time_last"),
                                          (300 // 2, 5, "time_last")])
def test_m2_prefill_generic_kernel(N_, P, layout):
    s = gen.scan_m2_inputs(2, 2, P, N_, 21, io="f32", seed=3, tag=f"m2g{N_}{P}", h0=True)
    _check(s, layout=layout, kernel="scan_m2_generic")


def test_m2_prefill_optional_inputs_absent_and_no_softplus():
    s = gen.scan_m2_inputs(2, 4, 16, 128, 33, io="f32", seed=4, tag="m2o", with_z=False,
                           with_D=False, with_dt_bias=False)
    _check(s, kernel="scan_m2", with_state=False)
    s = gen.scan_m2_inputs(2, 4, 16, 128, 33, io="f32", seed=5, tag="m2sp", with_dt_bias=False)
    s.dt = np.abs(s.dt) * 0.01  # delta = dt must stay positive without the softplus
    _check(s, kernel="scan_m2", softplus=False)


@pytest.mark.parametrize("L", [1, 15, 16, 17])
def test_m2_prefill_short_sequences(L):
    s = gen.scan_m2_inputs(1, 2, 8, 128, L, io="f32", seed=6, tag=f"m2L{L}", h0=True)
    _check(s, kernel="scan_m2")


def test_m2_prefill_empty_sequence_leaves_state_unchanged():
    import torch
    from state_space_model_causal_b200 import ssm_selective_scan_fwd
    h0 = gen.round_to(np.random.default_rng(0).standard_normal((1, 2, 8, 64)), "f32")
    h = T(h0, "f32")
    x = torch.zeros(1, 2, 8, 0, device="cuda")
    bc = torch.zeros(1, 1, 64, 0, device="cuda")
    ssm_selective_scan_fwd(x, torch.zeros(1, 2, 0, device="cuda"), T(np.full(2, -1.0), "f32"), bc,
                           bc.clone(), ssm_state=h)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(N(h), h0)


def test_m2_prefill_then_decode_matches_oracle():
    """Long sequence (several chunks) then two Mamba-2 decode steps on the GPU
    state: the decoded outputs equal the oracle's prefill over all steps."""
    import torch
    from state_space_model_causal_b200 import ssm_selective_state_update
    Bt, H, P, N_, L, k = 2, 4, 16, 128, 70, 2
    s = gen.scan_m2_inputs(Bt, H, P, N_, L, io="f32", seed=7, tag="m2pd", h0=True)
    head = gen.ScanM2Inputs(s.x[..., :L - k], s.dt[..., :L - k], s.A, s.B[..., :L - k],
                            s.C[..., :L - k], s.D, s.z[..., :L - k], s.dt_bias, s.h0, "f32")
    _, h = run_m2_gpu(head)
    st = T(h, "f32")
    outs = []
    for t in range(L - k, L):
        o = ssm_selective_state_update(st, T(s.x[..., t], "f32"), T(s.dt[..., t], "f32"), T(s.A, "f32"),
                                       T(s.B[..., t], "f32"), T(s.C[..., t], "f32"), D=T(s.D, "f32"),
                                       z=T(s.z[..., t], "f32"), dt_bias=T(s.dt_bias, "f32"))
        outs.append(N(o))
    torch.cuda.synchronize()
    ref, href = run_m2_oracle(s)
    assert_close(np.stack(outs, -1), ref[..., L - k:], 1e-5, "decoded outputs")
    assert_close(N(st), href, 1e-5, "final state")


def test_m2_prefill_full_size_sampled_heads():
    """Mamba-2 2.7B-shaped prefill (B=8, L=2048, H=80, P=64, N=128, fp16), the
    shape the benchmark times, inputs drawn on the device; 6 sampled (b, h)
    heads are checked against the oracle."""
    import torch
    from state_space_model_causal_b200 import LaunchInfo, ssm_selective_scan_fwd
    Bt, L, H, P, N_ = 8, 2048, 80, 64, 128
    tag = ("test", "m2_full")
    xs = gen.device_normal((Bt, L, H, P), "f16", *tag, "x")
    zs = gen.device_normal((Bt, L, H, P), "f16", *tag, "z")
    dts = gen.device_uniform((Bt, L, H), -4.0, -1.0, "f16", *tag, "dt")
    Bs = gen.device_normal((Bt, L, 1, N_), "f16", *tag, "B")
    Cs = gen.device_normal((Bt, L, 1, N_), "f16", *tag, "C")
    A = -torch.from_numpy(gen.uniform((H,), 1.0, 16.0, *tag, "A").astype(np.float32)).cuda()
    db = torch.from_numpy(gen.dt_bias_draw((H,), *tag, "db").astype(np.float32)).cuda()
    Dv = torch.ones(H, device="cuda")
    h = gen.device_normal((Bt, H, P, N_), "f32", *tag, "h0")
    h0 = h.clone()
    outs = torch.empty_like(xs)
    view = lambda t: t.permute(0, 2, 3, 1)  # noqa: E731  (B, L, H, P) -> (B, H, P, L)
    info = LaunchInfo()
    ssm_selective_scan_fwd(view(xs), dts.permute(0, 2, 1), A, view(Bs), view(Cs), D=Dv, z=view(zs),
                           dt_bias=db, ssm_state=h, out=view(outs), info=info)
    torch.cuda.synchronize()
    assert info.as_dict()["kernel"] == "scan_m2"
    rng = np.random.default_rng(7)
    picks = [(int(b), int(hh)) for b, hh in zip(rng.integers(0, Bt, 4), rng.integers(0, H, 4))]
    picks += [(0, 0), (Bt - 1, H - 1)]
    An, dbn = N(A), N(db)
    for b, hh in picks:
        sub = gen.ScanM2Inputs(N(view(xs)[b:b + 1, hh:hh + 1]), N(dts.permute(0, 2, 1)[b:b + 1, hh:hh + 1]),
                               An[hh:hh + 1], N(view(Bs)[b:b + 1]), N(view(Cs)[b:b + 1]), np.ones(1),
                               N(view(zs)[b:b + 1, hh:hh + 1]), dbn[hh:hh + 1], N(h0[b:b + 1, hh:hh + 1]),
                               "f16")
        ref, href = run_m2_oracle(sub)
        assert_close(N(view(outs)[b:b + 1, hh:hh + 1]), ref, TOL["f16"], f"out[{b},{hh}]")
        assert_close(N(h[b:b + 1, hh:hh + 1]), href, TOL["f16"], f"state[{b},{hh}]")
    del xs, zs, outs
    torch.cuda.empty_cache()


# ------------------------------------------- balanced slices with hand-overs --
def _m2_slots(N_):
    import torch
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    return sms * 3  # resident CTAs of the fast kernel (3 per SM)


@pytest.mark.parametrize("io,N_,P,L", [("f16", 128, 64, 200), ("bf16", 256, 128, 72), ("f32", 64, 64, 56)])
def test_m2_prefill_balanced_slices_match_oracle_and_whole_units(io, N_, P, L):
    """More (batch, head, row block) units than resident CTAs: CTAs take equal
    slices of the (unit, 16-step chunk) list and hand 32 KB state tiles over
    through the workspace.  Results match the oracle and equal the run
    without a workspace (one whole unit per CTA) bit for bit."""
    from state_space_model_causal_b200 import ssm_selective_scan_workspace_size
    rpc = 512 // (N_ // 16)
    blocks = -(-P // rpc)
    H = 8
    Bt = -(-(_m2_slots(N_) + 31) // (H * blocks))
    s = gen.scan_m2_inputs(Bt, H, P, N_, L, io=io, seed=5, tag=f"m2bal{io}{N_}", h0=True,
                           with_z=True)
    x = _time_major(s.x, io, (0, 3, 1, 2))
    assert ssm_selective_scan_workspace_size(
        x, _time_major(s.dt, io, (0, 2, 1)), T(s.A, "f32"), _time_major(s.B, io, (0, 3, 1, 2)),
        _time_major(s.C, io, (0, 3, 1, 2))) > 0, "problem too small to split"
    _check(s, kernel="scan_m2")
    # the same call without a workspace runs whole units: identical results
    import torch
    from state_space_model_causal_b200 import ssm_selective_scan_fwd

    def run(workspace):
        out = _time_major(np.zeros(s.x.shape), io, (0, 3, 1, 2))
        h = T(s.h0, "f32")
        ssm_selective_scan_fwd(x, _time_major(s.dt, io, (0, 2, 1)), T(s.A, "f32"),
                               _time_major(s.B, io, (0, 3, 1, 2)), _time_major(s.C, io, (0, 3, 1, 2)),
                               D=T(s.D, "f32"), z=_time_major(s.z, io, (0, 3, 1, 2)),
                               dt_bias=T(s.dt_bias, "f32"), ssm_state=h, out=out, workspace=workspace)
        torch.cuda.synchronize()
        return N(out), N(h)

    a, b = run("auto"), run(None)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])


@pytest.mark.parametrize("io", ["f32", "f16"])
def test_m2_prefill_rescaled_and_direct_chunks(io):
    """The kernel runs a 16-step chunk in the rescaled form (state divided by
    the running decay product) while every partial decay product of the chunk
    stays within 2^+-64, else in the direct form.  dt is raised on alternate 24-step spans,
    so that chunks are mild, strong or mixed: with dt_bias = 0 a strong step
    has delta = softplus(0.5) = 0.97, a decay of 2^-22.5 per step at A = -16
    (direct form) and 2^-1.4 at A = -1 (rescaled form even when strong).
    Both forms must match the oracle, state included."""
    s = gen.scan_m2_inputs(2, 3, 64, 128, 100, io=io, seed=9, tag=f"m2rs{io}", h0=True)
    s.A = np.array([-16.0, -4.0, -1.0])
    s.dt_bias = np.zeros(3)
    strong = (np.arange(100) // 24) % 2 == 1
    dt = np.array(s.dt, dtype=np.float64)
    dt[:, :, strong] = 0.5
    s.dt = gen.round_to(dt, io)
    _check(s, kernel="scan_m2")


def test_m2_prefill_rescaled_form_long_mild_decay():
    """Weak decay over a long sequence (delta * A ~ -0.02 per step): every
    chunk runs in the rescaled form and the state builds up over hundreds of
    steps; fp32 I/O at the fp32 bound."""
    s = gen.scan_m2_inputs(1, 2, 64, 64, 640, io="f32", seed=10, tag="m2mild", h0=True)
    s.A = np.array([-1.0, -2.0])
    s.dt = gen.round_to(np.full(s.dt.shape, -3.9), "f32")
    s.dt_bias = np.array([-0.05, -0.05])
    _check(s, kernel="scan_m2")
