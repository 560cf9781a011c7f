"""The allocation-free prefill entry point, ssm_selective_scan_fwd_noalloc.

Some callers cannot allocate device memory (a plugin or custom-operator
interface that receives its tensors but no allocator, or a serving loop that
must not allocate once running), so they cannot hand the fast prefill the
workspace it uses to pass running states between warps.  This entry point
takes that scratch from a fixed device array inside the library instead.

The test calls it through the C ABI on a problem large enough to need the
scratch (more 16-channel units than resident warps), twice in a row on
different inputs, and compares each call's outputs and final states with
those of ssm_selective_scan_fwd given its own workspace.  The second call
checks that what the first call left in the shared array does not leak into
the next one.  This file is collected last so that a run which stops at the
first failure has already run every other test."""
import numpy as np
import pytest

from state_space_model_causal_b200 import inputs as gen
from tests.parity import TOL, N, T, assert_close

pytestmark = pytest.mark.gpu


def _problem(seed):
    import torch
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    units = sms * 2 * 4 + 29  # more units than the prefill's resident warps
    Bt = 3
    D = 16 * -(-units // Bt)
    return gen.scan_inputs(Bt, 72, D, 16, W=4, io="f16", seed=seed, tag=f"noalloc{seed}",
                           conv_state=True, h0=True)


def _call(fn, s):
    """Run one entry point on fresh copies of the inputs and caches."""
    import torch
    io = s.io
    x = T(s.x, io)
    h = T(s.h0, "f32")
    cs = T(s.conv_state, "f32")
    out = torch.empty_like(x)
    fn(x, T(s.dt, io), T(s.A, "f32"), T(s.B, io), T(s.C, io), D=T(s.D, "f32"), z=T(s.z, io),
       dt_bias=T(s.dt_bias, "f32"), conv_weight=T(s.conv_weight, "f32"),
       conv_bias=T(s.conv_bias, "f32"), conv_state=cs, ssm_state=h, out=out)
    torch.cuda.synchronize()
    return N(out), N(h), N(cs)


def test_noalloc_prefill_matches_the_workspace_entry_point_twice_in_a_row():
    from state_space_model_causal_b200 import (ssm_device_error, ssm_selective_scan_fwd,
                                               ssm_selective_scan_fwd_noalloc,
                                               ssm_selective_scan_workspace_size)
    for seed in (11, 12):
        s = _problem(seed)
        # the problem does need the hand-over scratch
        assert ssm_selective_scan_workspace_size(T(s.x, s.io), T(s.dt, s.io), T(s.A, "f32"),
                                                 T(s.B, s.io), T(s.C, s.io)) > 0
        got = _call(ssm_selective_scan_fwd_noalloc, s)
        ref = _call(ssm_selective_scan_fwd, s)
        for g, r, what in zip(got, ref, ("out", "ssm_state", "conv_state")):
            assert np.isfinite(g).all(), what
            assert_close(g, r, TOL[s.io], f"{what} (call with seed {seed})")
        assert ssm_device_error() == 0


def test_noalloc_prefill_refuses_a_caller_workspace():
    """The scratch is the library's own: a call that also passes a workspace
    is refused with SSM_ERR_WORKSPACE before anything runs."""
    import ctypes

    import torch
    from state_space_model_causal_b200 import binding
    s = _problem(13)
    tensors = [T(s.x, s.io), T(s.dt, s.io), T(s.A, "f32"), T(s.B, s.io), T(s.C, s.io)]
    out = torch.empty_like(tensors[0])
    ws = torch.zeros(1 << 20, dtype=torch.uint8, device="cuda")
    a = binding.ScanArgs()
    a.struct_size = ctypes.sizeof(binding.ScanArgs)
    a.x, a.dt, a.A, a.B, a.C = map(binding.describe, tensors)
    a.out = binding.describe(out)
    a.dt_softplus = 1
    a.workspace, a.workspace_bytes = ws.data_ptr(), ws.numel()
    st = binding.library().ssm_selective_scan_fwd_noalloc(ctypes.byref(a),
                                                          torch.cuda.current_stream().cuda_stream)
    assert binding.STATUS[st] == "SSM_ERR_WORKSPACE"
