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
