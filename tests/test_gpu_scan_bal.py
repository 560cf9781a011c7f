"""GPU parity of the load-balanced prefill (SSM_KERNEL_SCAN_BAL) against the
fp64 oracle, through the C ABI, on problems with more (batch entry,
16-channel) units than the GPU runs warps at once, so that warps hand running
states over to one another through the workspace.  The hand-over passes the
exact fp32 state, so the split run must also equal the run without a
workspace (whole units per warp) bit for bit."""
import ctypes

import numpy as np
import pytest

from state_space_model_causal_b200 import inputs as gen
from tests.parity import TOL, N, T, assert_close, run_scan_oracle

pytestmark = pytest.mark.gpu


def _slots():
    """Warps the balanced prefill keeps resident: SMs x 2 CTAs x 4 warps."""
    import torch
    return torch.cuda.get_device_properties(0).multi_processor_count * 2 * 4


def _inputs(io, L, extra_units=37, Bt=3, W=4, seed=0, **kw):
    """A problem with `extra_units` more units than resident warps."""
    units = _slots() + extra_units
    D = 16 * -(-units // Bt)
    return gen.scan_inputs(Bt, L, D, 16, W=W, io=io, seed=seed, tag=f"bal{io}{L}{W}",
                           conv_state=W > 0, h0=True, **kw)


def _run(s, workspace="auto", info=None):
    import torch
    from state_space_model_causal_b200 import ssm_selective_scan_fwd
    io = s.io
    Bt, D, L = s.x.shape
    W = 0 if s.conv_weight is None else s.conv_weight.shape[1]
    h = T(s.h0, "f32")
    cs = T(s.conv_state if s.conv_state is not None else np.zeros((Bt, D, max(W, 1))), "f32") if W else None
    out = ssm_selective_scan_fwd(T(s.x, io), T(s.dt, io), T(s.A, "f32"), T(s.B, io), T(s.C, io),
                                 D=T(s.D, "f32"), z=T(s.z, io), dt_bias=T(s.dt_bias, "f32"),
                                 conv_weight=T(s.conv_weight, "f32"), conv_bias=T(s.conv_bias, "f32"),
                                 conv_state=cs, ssm_state=h, workspace=workspace, info=info)
    torch.cuda.synchronize()
    return N(out), N(h), N(cs)


def _check_against_oracle(s, got):
    out, h, cs = got
    ref, href, csref = run_scan_oracle(s)
    assert_close(out, ref, TOL[s.io], "out")
    assert_close(h, href, TOL[s.io], "ssm_state")
    if csref is not None:
        np.testing.assert_array_equal(cs, csref)


@pytest.mark.parametrize("io,L", [("f16", 72), ("bf16", 104), ("f32", 40), ("f16", 8)])
def test_balanced_split_matches_oracle_and_whole_units(io, L):
    """Slices of ~3 chunks (L=72: chunks of 32, 32 and a ragged 8) start and
    end inside units; outputs, final ssm and conv states match the oracle, and
    equal the no-workspace run bit for bit."""
    from state_space_model_causal_b200 import LaunchInfo, ssm_selective_scan_workspace_size
    s = _inputs(io, L)
    info = LaunchInfo()
    split = _run(s, info=info)
    assert info.as_dict()["kernel"] == "scan_bal"
    Bt, D, _ = s.x.shape
    assert ssm_selective_scan_workspace_size(T(s.x, io), T(s.dt, io), T(s.A, "f32"), T(s.B, io),
                                             T(s.C, io)) > 0, "problem too small to split"
    _check_against_oracle(s, split)
    whole = _run(s, workspace=None)
    for a, b, name in zip(split, whole, ("out", "ssm_state", "conv_state")):
        np.testing.assert_array_equal(a, b, err_msg=name)


def test_balanced_split_without_conv_gate_or_state():
    s = _inputs("f16", 64, W=0, seed=1, with_z=False)
    _check_against_oracle(s, _run(s))


def test_balanced_split_groups():
    """Two groups of B/C rows: every 16-channel unit stays inside one group."""
    units = _slots() + 53
    D = 32 * -(-units // 4)  # Bt=2 below, D % 32 == 0 so each group holds whole units
    s = gen.scan_inputs(2, 48, D, 16, G=2, W=4, io="f16", seed=2, tag="balg", conv_state=True, h0=True)
    _check_against_oracle(s, _run(s))


def test_workspace_is_reused_across_calls_and_shapes():
    """The workspace's generation counter lets one buffer serve call after
    call (hand-over flags of earlier calls never match); different shapes
    through the same buffer stay correct."""
    import torch
    from state_space_model_causal_b200 import ssm_selective_scan_workspace_size
    s1 = _inputs("f16", 72, seed=3)
    s2 = _inputs("f16", 40, extra_units=400, Bt=2, seed=4)
    need = max(ssm_selective_scan_workspace_size(T(s.x, "f16"), T(s.dt, "f16"), T(s.A, "f32"),
                                                 T(s.B, "f16"), T(s.C, "f16")) for s in (s1, s2))
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    first = _run(s1, workspace=ws)
    for s in (s1, s2, s1, s2):
        got = _run(s, workspace=ws)
        _check_against_oracle(s, got)
    for a, b in zip(first, _run(s1, workspace=ws)):
        np.testing.assert_array_equal(a, b)


def test_workspace_errors():
    """Too small or misaligned workspace: SSM_ERR_WORKSPACE; a workspace that
    overlaps an operand: SSM_ERR_ALIAS.  Nothing is launched."""
    import torch
    from state_space_model_causal_b200 import SsmError, ssm_selective_scan_fwd, ssm_selective_scan_workspace_size
    s = _inputs("f16", 40, seed=5)
    x, dt, A, B, C = T(s.x, "f16"), T(s.dt, "f16"), T(s.A, "f32"), T(s.B, "f16"), T(s.C, "f16")
    need = ssm_selective_scan_workspace_size(x, dt, A, B, C)
    assert need > 0
    small = torch.zeros(need - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(SsmError) as e:
        ssm_selective_scan_fwd(x, dt, A, B, C, workspace=small)
    assert e.value.name == "SSM_ERR_WORKSPACE"
    big = torch.zeros(need + 512, dtype=torch.uint8, device="cuda")
    with pytest.raises(SsmError) as e:
        ssm_selective_scan_fwd(x, dt, A, B, C, workspace=big[16:])
    assert e.value.name == "SSM_ERR_WORKSPACE"
    out = torch.empty_like(x)
    with pytest.raises(SsmError) as e:
        ssm_selective_scan_fwd(x, dt, A, B, C, out=out,
                               workspace=out.view(torch.uint8).reshape(-1)[:need])
    assert e.value.name == "SSM_ERR_ALIAS"


def test_no_device_error_after_split_runs():
    from state_space_model_causal_b200 import ssm_device_error
    s = _inputs("f16", 72, seed=6)
    _run(s)
    assert ssm_device_error() == 0


def test_balanced_softplus_slow_path_and_large_steps():
    """dt + dt_bias spanning (-8, 30): e^v crosses 1/16 (the warp-uniform
    log1pf path) and passes 20 (delta = v), mixed within one warp's lanes."""
    s = _inputs("f32", 40, seed=7, W=4)
    r = np.random.default_rng(7)
    s.dt = gen.round_to(r.uniform(-8.0, 30.0, s.dt.shape) - s.dt_bias[None, :, None], "f32")
    # large steps drive exp(delta * A) to zero: the state forgets, outputs stay finite
    _check_against_oracle(s, _run(s))


def test_balanced_without_softplus():
    """dt_softplus = 0: delta = dt + dt_bias as given (kept positive)."""
    import torch
    from state_space_model_causal_b200 import ssm_selective_scan_fwd
    s = _inputs("f16", 48, seed=8, W=4)
    s.dt = gen.round_to(np.abs(s.dt) * 0.01, "f16")
    s.dt_bias = np.zeros_like(s.dt_bias)
    io = "f16"
    h = T(s.h0, "f32")
    cs = T(s.conv_state, "f32")
    out = ssm_selective_scan_fwd(T(s.x, io), T(s.dt, io), T(s.A, "f32"), T(s.B, io), T(s.C, io),
                                 D=T(s.D, "f32"), z=T(s.z, io), dt_bias=T(s.dt_bias, "f32"),
                                 dt_softplus=False, conv_weight=T(s.conv_weight, "f32"),
                                 conv_bias=T(s.conv_bias, "f32"), conv_state=cs, ssm_state=h)
    torch.cuda.synchronize()
    ref, href, csref = run_scan_oracle(s, softplus=False)
    assert_close(N(out), ref, TOL[io], "out")
    assert_close(N(h), href, TOL[io], "ssm_state")
    np.testing.assert_array_equal(N(cs), csref)


# ----------------------------------------------------- context-parallel prefill --
@pytest.mark.parametrize("io,Bt,D,L,W", [("f16", 1, 256, 512, 4), ("f32", 2, 96, 416, 4),
                                         ("bf16", 1, 64, 200, 0)])
def test_context_parallel_pieces_match_oracle(io, Bt, D, L, W):
    """Few (batch, 16-channel) units: the sequence is cut into pieces scanned in
    two passes (zero-state pieces with end-state records, then re-scans from
    the composed states); outputs, final ssm and conv states match the oracle
    and the plain sequential run (no workspace)."""
    s = gen.scan_inputs(Bt, L, D, 16, W=W, io=io, seed=20, tag=f"cp{io}{L}", conv_state=W > 0, h0=True)
    got = _run(s)
    _check_against_oracle(s, got)
    # both runs are within tol of the oracle, so within 2 tol of each other
    plain = _run(s, workspace=None)
    for a, b, name in zip(got, plain, ("out", "ssm_state", "conv_state")):
        if name == "conv_state":
            np.testing.assert_array_equal(a, b)
        else:
            assert_close(a, b, 2 * TOL[io], f"{name} vs sequential")


def test_context_parallel_full_length_b1_with_hand_overs():
    """The 2.8B-shaped layer at batch 1 (320 units): 5 pieces, 1280
    piece-units per pass, so the passes also hand states between warps."""
    s = gen.scan_inputs(1, 2048, 5120, 16, W=4, io="f16", seed=3, tag="cp_b1", conv_state=True, h0=True)
    _check_against_oracle(s, _run(s))
