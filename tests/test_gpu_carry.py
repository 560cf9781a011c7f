"""GPU parity of the sequence-piece calls (ssm_scan_delta_sum,
ssm_scan_carry_fold) against the fp64 oracle, and of a prefill cut into
pieces and joined by them -- on one GPU, piece after piece, and through the
context-parallel driver with ranks emulated by host threads -- against the
oracle's whole-sequence prefill."""
import threading

import numpy as np
import pytest

import oracle
from state_space_model_causal_b200 import inputs as gen
from tests.parity import TOL, N, T, assert_close

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("io,softplus,bias", [("f32", True, True), ("f16", True, True),
                                              ("bf16", True, False), ("f32", False, True)])
@pytest.mark.parametrize("L", [0, 1, 37, 512])
def test_delta_sum_matches_oracle(io, softplus, bias, L):
    from state_space_model_causal_b200 import ssm_scan_delta_sum
    s = gen.scan_inputs(3, max(L, 1), 40, 4, io=io, seed=20 + L, tag="dsum")
    dt = s.dt[..., :L] if softplus else gen.round_to(np.abs(s.dt[..., :L]) * 0.05, io)
    db = s.dt_bias if bias else None
    got = ssm_scan_delta_sum(T(dt, io), T(db, "f32") if bias else None, dt_softplus=softplus)
    ref = oracle.delta_sum(dt, db, dt_softplus=softplus)
    if L == 0:
        assert np.array_equal(N(got), np.zeros((3, 40)))
    else:
        assert_close(N(got), ref, 1e-5, "delta sum")


def test_delta_sum_strided_view():
    """dt as a strided view (every other time step of a wider buffer)."""
    import torch
    from state_space_model_causal_b200 import ssm_scan_delta_sum
    s = gen.scan_inputs(2, 64, 16, 4, io="f32", seed=27, tag="dsumv")
    wide = T(s.dt, "f32")
    view = wide[..., ::2]
    got = ssm_scan_delta_sum(view, T(s.dt_bias, "f32"))
    torch.cuda.synchronize()
    assert_close(N(got), oracle.delta_sum(s.dt[..., ::2], s.dt_bias), 1e-5, "delta sum (view)")


@pytest.mark.parametrize("S_scale", [0.0, 0.05, 3.0])
def test_carry_fold_matches_oracle(S_scale):
    import torch
    from state_space_model_causal_b200 import ssm_scan_carry_fold
    rng = np.random.default_rng(30)
    st = gen.round_to(rng.standard_normal((3, 40, 16)), "f32")
    he = gen.round_to(rng.standard_normal((3, 40, 16)), "f32")
    A = gen.round_to(-rng.uniform(1.0, 16.0, (40, 16)), "f32")
    S = gen.round_to(rng.uniform(0.0, 1.0, (3, 40)) * S_scale, "f32")
    g = T(st, "f32")
    ssm_scan_carry_fold(g, T(A, "f32"), T(S, "f32"), T(he, "f32"))
    torch.cuda.synchronize()
    assert_close(N(g), oracle.carry_fold(st, A, S, he), 1e-5, "carry fold")


def _pieces(total, cuts):
    b = (0,) + tuple(cuts) + (total,)
    return [(b[i], b[i + 1]) for i in range(len(b) - 1)]


@pytest.mark.parametrize("io,cuts", [("f16", (96,)), ("f16", (40, 104, 200)), ("f32", (64, 128))])
def test_prefill_in_pieces_joined_on_one_gpu(io, cuts):
    """Pieces scanned from zero states with their records, the states entering
    them composed by carry folds, each piece re-scanned from its state: the
    outputs and final caches of the whole prefill."""
    import torch
    from state_space_model_causal_b200 import (ssm_scan_carry_fold, ssm_scan_delta_sum,
                                               ssm_selective_scan_fwd)
    L = 256
    s = gen.scan_inputs(2, L, 64, 16, W=4, io=io, seed=31, tag="pieces", conv_state=True, h0=True)
    ref, href, csref = oracle.scan(s.x, s.dt, s.A, s.B, s.C, D=s.D, z=s.z, dt_bias=s.dt_bias,
                                   conv_weight=s.conv_weight, conv_bias=s.conv_bias,
                                   conv_state=s.conv_state, h0=s.h0)
    kw = dict(D=T(s.D, "f32"), dt_bias=T(s.dt_bias, "f32"), conv_weight=T(s.conv_weight, "f32"),
              conv_bias=T(s.conv_bias, "f32"))
    A = T(s.A, "f32")
    h_in = T(s.h0, "f32")
    cs = T(s.conv_state, "f32")
    outs = []
    for t0, t1 in _pieces(L, cuts):
        sl = lambda a: T(np.ascontiguousarray(a[..., t0:t1]), io)  # noqa: E731
        x, dt, z, Bm, Cm = sl(s.x), sl(s.dt), sl(s.z), sl(s.B), sl(s.C)
        h_end = torch.zeros_like(h_in)
        cs_zero_start = cs.clone()
        ssm_selective_scan_fwd(x, dt, A, Bm, Cm, z=z, conv_state=cs_zero_start, ssm_state=h_end, **kw)
        S = ssm_scan_delta_sum(dt, kw["dt_bias"])
        h = h_in.clone()
        out = ssm_selective_scan_fwd(x, dt, A, Bm, Cm, z=z, conv_state=cs, ssm_state=h, **kw)
        outs.append(N(out))
        ssm_scan_carry_fold(h_in, A, S, h_end)  # the state entering the next piece
        torch.cuda.synchronize()
        assert_close(N(h_in), N(h), 2 * TOL[io], "composed vs scanned state")
    tol = 2 * TOL[io]
    assert_close(np.concatenate(outs, -1), ref, tol, "out")
    assert_close(N(h_in), href, tol, "final ssm state")
    np.testing.assert_array_equal(N(cs), gen.round_to(csref, "f32"))


class _ThreadComm:
    """The collective of ranks emulated by host threads of one process: the
    ranks' kernels share one stream and never wait on one another; only the
    host threads meet at the barrier."""

    def __init__(self, rank, world, shared):
        self.rank, self.world_size, self.sh = rank, world, shared

    def all_gather(self, t):
        self.sh["slots"][self.rank] = t.clone()
        self.sh["barrier"].wait()
        got = [v.clone() for v in self.sh["slots"]]
        self.sh["barrier"].wait()
        return got


@pytest.mark.parametrize("io,lengths", [("f16", (128, 128)), ("f16", (96, 40, 64, 56)), ("f32", (64, 72, 120))])
def test_context_parallel_driver_with_emulated_ranks(io, lengths):
    """The driver of state_space_model_causal_b200.context_parallel, one host
    thread per rank on one GPU: every rank's outputs are the whole prefill's
    over its piece, and the last rank ends with the final caches."""
    import torch
    from state_space_model_causal_b200.context_parallel import prefill_context_parallel
    L = sum(lengths)
    s = gen.scan_inputs(2, L, 48, 16, W=4, io=io, seed=32, tag="cpdrv", conv_state=True, h0=True)
    ref, href, csref = oracle.scan(s.x, s.dt, s.A, s.B, s.C, D=s.D, z=s.z, dt_bias=s.dt_bias,
                                   conv_weight=s.conv_weight, conv_bias=s.conv_bias,
                                   conv_state=s.conv_state, h0=s.h0)
    R = len(lengths)
    bounds = np.cumsum((0,) + tuple(lengths))
    shared = {"slots": [None] * R, "barrier": threading.Barrier(R, timeout=120)}
    results, errors = [None] * R, []
    dev = torch.device("cuda", 0)

    def rank_main(r):
        try:
            torch.cuda.set_device(dev)
            t0, t1 = int(bounds[r]), int(bounds[r + 1])
            sl = lambda a: T(np.ascontiguousarray(a[..., t0:t1]), io)  # noqa: E731
            h = T(s.h0, "f32") if r == 0 else torch.zeros(2, 48, 16, device=dev)
            cs = T(s.conv_state, "f32") if r == 0 else torch.zeros(2, 48, 4, device=dev)
            out = prefill_context_parallel(
                sl(s.x), sl(s.dt), T(s.A, "f32"), sl(s.B), sl(s.C), D=T(s.D, "f32"), z=sl(s.z),
                dt_bias=T(s.dt_bias, "f32"), conv_weight=T(s.conv_weight, "f32"),
                conv_bias=T(s.conv_bias, "f32"), conv_state=cs, ssm_state=h,
                comm=_ThreadComm(r, R, shared))
            torch.cuda.synchronize()
            results[r] = (N(out), N(h), N(cs))
        except Exception as e:  # reported below; the barrier is broken for the others
            errors.append(repr(e))
            shared["barrier"].abort()

    threads = [threading.Thread(target=rank_main, args=(r,)) for r in range(R)]
    for th in threads:
        th.start()
    for th in threads:
        th.join(timeout=300)
    assert not errors, errors
    tol = 2 * TOL[io]
    assert_close(np.concatenate([res[0] for res in results], -1), ref, tol, "out")
    assert_close(results[-1][1], href, tol, "final ssm state")
    np.testing.assert_array_equal(results[-1][2], gen.round_to(csref, "f32"))


def test_carry_fold_mamba2_layout_matches_oracle():
    """Rank-4 state, A and the sums per head: the oracle's fold with A and S
    repeated over the head's rows."""
    import torch
    from state_space_model_causal_b200 import ssm_scan_carry_fold
    rng = np.random.default_rng(33)
    st = gen.round_to(rng.standard_normal((2, 3, 8, 32)), "f32")
    he = gen.round_to(rng.standard_normal((2, 3, 8, 32)), "f32")
    A = gen.round_to(-rng.uniform(1.0, 16.0, 3), "f32")
    S = gen.round_to(rng.uniform(0.0, 0.3, (2, 3)), "f32")
    g = T(st, "f32")
    ssm_scan_carry_fold(g, T(A, "f32"), T(S, "f32"), T(he, "f32"))
    torch.cuda.synchronize()
    rows = lambda a: a.reshape(2, 24, 32)  # noqa: E731
    ref = oracle.carry_fold(rows(st), np.repeat(A, 8)[:, None].repeat(32, 1), np.repeat(S, 8, axis=1), rows(he))
    assert_close(N(g).reshape(2, 24, 32), ref, 1e-5, "carry fold (Mamba-2 layout)")


def _time_major(a, dtype, perm):
    import torch  # noqa: F401
    store = T(np.ascontiguousarray(np.transpose(a, perm)), dtype)
    return store.permute(*[int(i) for i in np.argsort(perm)])


@pytest.mark.parametrize("io,lengths", [("f16", (64, 48)), ("f32", (32, 40, 56))])
def test_context_parallel_driver_mamba2_layout_with_emulated_ranks(io, lengths):
    """The driver on Mamba-2-layout pieces (time-major rows, as the model
    stores them), one host thread per rank on one GPU, against the oracle's
    whole-sequence Mamba-2-layout prefill."""
    import torch
    from state_space_model_causal_b200.context_parallel import prefill_context_parallel
    L = sum(lengths)
    s = gen.scan_m2_inputs(2, 3, 64, 128, L, io=io, seed=34, tag="cpm2", h0=True)
    ref, href = oracle.scan_mamba2(s.x, s.dt, s.A, s.B, s.C, D=s.D, z=s.z, dt_bias=s.dt_bias, h0=s.h0)
    R = len(lengths)
    bounds = np.cumsum((0,) + tuple(lengths))
    shared = {"slots": [None] * R, "barrier": threading.Barrier(R, timeout=120)}
    results, errors = [None] * R, []
    dev = torch.device("cuda", 0)

    def rank_main(r):
        try:
            torch.cuda.set_device(dev)
            t0, t1 = int(bounds[r]), int(bounds[r + 1])
            sl = lambda a: np.ascontiguousarray(a[..., t0:t1])  # noqa: E731
            x = _time_major(sl(s.x), io, (0, 3, 1, 2))
            z = _time_major(sl(s.z), io, (0, 3, 1, 2))
            dt = _time_major(sl(s.dt), io, (0, 2, 1))
            Bm = _time_major(sl(s.B), io, (0, 3, 1, 2))
            Cm = _time_major(sl(s.C), io, (0, 3, 1, 2))
            out = _time_major(np.zeros(x.shape), io, (0, 3, 1, 2))
            h = T(s.h0, "f32") if r == 0 else torch.zeros(2, 3, 64, 128, device=dev)
            prefill_context_parallel(x, dt, T(s.A, "f32"), Bm, Cm, D=T(s.D, "f32"), z=z,
                                     dt_bias=T(s.dt_bias, "f32"), ssm_state=h, out=out,
                                     comm=_ThreadComm(r, R, shared))
            torch.cuda.synchronize()
            results[r] = (N(out), N(h))
        except Exception as e:
            errors.append(repr(e))
            shared["barrier"].abort()

    threads = [threading.Thread(target=rank_main, args=(r,)) for r in range(R)]
    for th in threads:
        th.start()
    for th in threads:
        th.join(timeout=300)
    assert not errors, errors
    tol = 2 * (1e-5 if io == "f32" else TOL[io])
    assert_close(np.concatenate([res[0] for res in results], -1), ref, tol, "out")
    assert_close(results[-1][1], href, tol, "final ssm state")
