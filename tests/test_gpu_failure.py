"""Failure detection on the GPU without a GPU fault.

The bulk-copy state-update kernels give up a wait on a shared-memory stage
after a cycle budget, record it in the library's device error record and
exit; the host reads it with ssm_device_error() / ssm_device_error_info().
These tests make one wait run out on purpose, through the failure-test build
of the library (libssm_causal_testhooks.so, the only build that reads the
switches): SSM_TEST_DROP_ITEM names a work item whose copies are never
started (a flag that nothing sets) and SSM_TEST_WAIT_CYCLES shortens the
budget to about 10 ms.  The call must return without a CUDA error, the record
must name the kernel and the dropped item as the first unfinished one, read
once and then clear, and the context must stay usable: the next call,
without the switches, matches the oracle.  The product library, given the
same switches, ignores them."""
import os

import numpy as np
import pytest

from state_space_model_causal_b200 import inputs as gen
from tests.parity import TOL, N, assert_close
from tests.test_gpu_ssu import _m1_gpu, _m1_oracle, _m2_gpu, _m2_oracle

pytestmark = pytest.mark.gpu


class _env:
    def __init__(self, **kv):
        self.kv, self.old = kv, {}

    def __enter__(self):
        for k, v in self.kv.items():
            self.old[k] = os.environ.get(k)
            os.environ[k] = v

    def __exit__(self, *exc):
        for k, v in self.old.items():
            if v is None:
                os.environ.pop(k, None)
            else:
                os.environ[k] = v


def _expect_timeout_then_clean(run_dropped, run_clean, check, kernel):
    import torch
    from state_space_model_causal_b200 import LaunchInfo, binding, ssm_device_error, ssm_device_error_info
    info = LaunchInfo()
    with binding.using_library(binding.TESTHOOKS_LIB_PATH):
        assert ssm_device_error() == 0
        with _env(SSM_TEST_DROP_ITEM="5", SSM_TEST_WAIT_CYCLES="20000000"):
            run_dropped(info)
            torch.cuda.synchronize()  # no CUDA error: the kernel returned
        rep = ssm_device_error_info()
        assert rep == {"code": 1, "kernel": kernel, "first_item": 5}, rep
        assert ssm_device_error() == 0  # read and cleared
        check(run_clean())
        assert ssm_device_error() == 0
    return info


def test_mamba1_bulk_copy_wait_runs_out_and_is_reported():
    s = gen.ssu_mamba1_inputs(16, 512, 16, W=4, io="f16", state="f32", seed=21, tag="fail1")

    def check(res):
        out, st, cs = res
        o, sref, csref = _m1_oracle(s)
        assert_close(N(out), o, TOL["f16"], "out")
        assert_close(N(st), sref, TOL["f16"], "state")
        np.testing.assert_array_equal(N(cs), csref)

    info = _expect_timeout_then_clean(lambda info: _m1_gpu(s), lambda: _m1_gpu(s), check, "ssu_row_tma")
    assert info is not None


def test_mamba2_bulk_copy_wait_runs_out_and_is_reported():
    s = gen.ssu_mamba2_inputs(16, 8, 64, 128, io="f16", state="f16", seed=22, tag="fail2")

    def check(res):
        out, st = res
        o, sref = _m2_oracle(s)
        assert_close(N(out), o, TOL["f16"], "out")
        assert_close(N(st), sref, TOL["f16"], "state")

    _expect_timeout_then_clean(lambda info: _m2_gpu(s), lambda: _m2_gpu(s), check, "ssu_tma")


def test_product_library_ignores_the_failure_test_switches():
    """The shipped library never reads SSM_TEST_*: with the switches set the
    update completes, matches the oracle and leaves the record clear."""
    import torch
    from state_space_model_causal_b200 import ssm_device_error
    s = gen.ssu_mamba2_inputs(16, 8, 64, 128, io="f16", state="f16", seed=23, tag="fail3")
    with _env(SSM_TEST_DROP_ITEM="5", SSM_TEST_WAIT_CYCLES="20000000"):
        out, st = _m2_gpu(s)
        torch.cuda.synchronize()
    assert ssm_device_error() == 0
    o, sref = _m2_oracle(s)
    assert_close(N(out), o, TOL["f16"], "out")
    assert_close(N(st), sref, TOL["f16"], "state")


def test_the_kernels_under_test_are_the_bulk_copy_ones():
    """The two cases above go through the kernels with bounded waits."""
    from state_space_model_causal_b200 import LaunchInfo, ssm_selective_state_update
    from tests.parity import T
    s1 = gen.ssu_mamba1_inputs(16, 512, 16, W=4, io="f16", state="f32", seed=21, tag="fail1")
    info = LaunchInfo()
    ssm_selective_state_update(T(s1.state, "f32"), T(s1.x, "f16"), T(s1.dt, "f16"), T(s1.A, "f32"),
                               T(s1.B, "f16"), T(s1.C, "f16"), D=T(s1.D, "f32"), z=T(s1.z, "f16"),
                               dt_bias=T(s1.dt_bias, "f32"), conv_weight=T(s1.conv_weight, "f32"),
                               conv_bias=T(s1.conv_bias, "f32"), conv_state=T(s1.conv_state, "f32"),
                               info=info)
    assert info.as_dict()["kernel"] == "ssu_row_tma" and info.work_items > 5
    s2 = gen.ssu_mamba2_inputs(16, 8, 64, 128, io="f16", state="f16", seed=22, tag="fail2")
    info = LaunchInfo()
    ssm_selective_state_update(T(s2.state, "f16"), T(s2.x, "f16"), T(s2.dt, "f16"), T(s2.A, "f32"),
                               T(s2.B, "f16"), T(s2.C, "f16"), D=T(s2.D, "f32"), dt_bias=T(s2.dt_bias, "f32"),
                               info=info)
    assert info.as_dict()["kernel"] == "ssu_tma" and info.work_items > 5


def test_prefill_hand_over_wait_runs_out_and_is_reported():
    """The balanced prefill: worker w never publishes the state it hands to
    worker w + 1 (SSM_TEST_DROP_WORKER, test build only).  w + 1 gives up its
    bounded wait, scans its piece of that unit from a zero state, and the
    record names the prefill kernel and that unit; every other unit's outputs
    are complete, and the next call without the switch matches the oracle.
    The product library ignores the switch."""
    import torch
    from state_space_model_causal_b200 import (LaunchInfo, binding, ssm_device_error, ssm_device_error_info,
                                               ssm_selective_scan_fwd)
    from tests.parity import T, run_scan_oracle
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    Bt, L = 3, 72
    units_wanted = sms * 2 * 4 + 29  # more 16-channel units than resident warps: slices hand over
    D = 16 * -(-units_wanted // Bt)
    s = gen.scan_inputs(Bt, L, D, 16, W=4, io="f16", seed=50, tag="dropworker", conv_state=True, h0=True)
    ref, href, _ = run_scan_oracle(s)

    def call():
        info = LaunchInfo()
        out = ssm_selective_scan_fwd(T(s.x, "f16"), T(s.dt, "f16"), T(s.A, "f32"), T(s.B, "f16"),
                                     T(s.C, "f16"), D=T(s.D, "f32"), z=T(s.z, "f16"),
                                     dt_bias=T(s.dt_bias, "f32"), conv_weight=T(s.conv_weight, "f32"),
                                     conv_bias=T(s.conv_bias, "f32"), conv_state=T(s.conv_state, "f32"),
                                     ssm_state=T(s.h0, "f32"), info=info)
        torch.cuda.synchronize()
        return N(out), info

    out, info = call()  # product library: plan of the split
    assert binding.KERNELS[info.kernel] == "scan_bal"
    workers, units, nck = info.grid * 4, info.work_items, -(-L // 32)
    total = units * nck
    # a worker whose slice ends inside a unit: it hands that unit's state over
    w = next(v for v in range(workers - 1) if ((v + 1) * total // workers) % nck != 0)
    lost = ((w + 1) * total // workers) // nck  # the unit its successor continues
    with binding.using_library(binding.TESTHOOKS_LIB_PATH):
        assert ssm_device_error() == 0
        with _env(SSM_TEST_DROP_WORKER=str(w), SSM_TEST_WAIT_CYCLES="20000000"):
            out_d, _ = call()
        rep = ssm_device_error_info()
        assert rep == {"code": 1, "kernel": "scan_bal", "first_item": lost}, rep
        assert ssm_device_error() == 0  # read and cleared
        # every other unit (batch entry b, channels 16c .. 16c+15) is complete
        nblk = D // 16
        keep = np.ones((Bt, D), dtype=bool)
        keep[lost // nblk, 16 * (lost % nblk):16 * (lost % nblk + 1)] = False
        assert_close(out_d[keep], ref[keep], TOL["f16"], "outputs of the other units")
        out_c, _ = call()  # the switch gone: complete again
        assert_close(out_c, ref, TOL["f16"], "out after the failure")
        assert ssm_device_error() == 0
    with _env(SSM_TEST_DROP_WORKER=str(w), SSM_TEST_WAIT_CYCLES="20000000"):
        out_p, _ = call()  # product library: the switch has no effect
    assert_close(out_p, ref, TOL["f16"], "out (product library)")
    assert ssm_device_error() == 0
