"""GPU parity of the whole-unit prefill kernel (scan_vec_kernel), which the
planner selects only under the tuning switch SSM_SCAN_KERNEL=vec.  The library
reads its switches once per process, so each case runs in a child process
with the switch set; the child checks the chosen kernel and the results
against the fp64 oracle and reports through its exit status."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import sys
import numpy as np
import torch
from state_space_model_causal_b200 import inputs as gen, LaunchInfo, ssm_selective_scan_fwd
from state_space_model_causal_b200.binding import KERNELS
from tests.parity import TOL, T, N, assert_close, run_scan_oracle

io, Bt, L, D, W, sw = sys.argv[1], int(sys.argv[2]), int(sys.argv[3]), int(sys.argv[4]), int(sys.argv[5]), sys.argv[6]
s = gen.scan_inputs(Bt, L, D, 16, W=W, io=io, seed=3, tag="scan_vec_child", conv_state=W > 0, h0=True)
info = LaunchInfo()
cs = T(s.conv_state, "f32") if W else None
h = T(s.h0, "f32")
out = ssm_selective_scan_fwd(T(s.x, io), T(s.dt, io), T(s.A, "f32"), T(s.B, io), T(s.C, io),
                             D=T(s.D, "f32"), z=T(s.z, io), dt_bias=T(s.dt_bias, "f32"),
                             conv_weight=T(s.conv_weight, "f32") if W else None,
                             conv_bias=T(s.conv_bias, "f32") if W else None,
                             conv_state=cs, ssm_state=h, info=info)
torch.cuda.synchronize()
assert KERNELS[info.kernel] == "scan_vec", KERNELS[info.kernel]
ref, href, csref = run_scan_oracle(s)
assert_close(N(out), ref, TOL[io], "out")
assert_close(N(h), href, TOL[io], "ssm_state")
if W:
    np.testing.assert_array_equal(N(cs), gen.round_to(csref, "f32"))
print("ok", KERNELS[info.kernel])
"""


@pytest.mark.parametrize("io,Bt,L,D,W,sw", [("f16", 2, 96, 48, 4, "0"), ("bf16", 1, 40, 32, 4, "2"),
                                             ("f32", 2, 64, 32, 0, "0"), ("f16", 1, 72, 64, 4, "3")])
def test_whole_unit_prefill_kernel_matches_oracle(io, Bt, L, D, W, sw):
    env = dict(os.environ, SSM_SCAN_KERNEL="vec", SSM_SCAN_SW_PAIRS=sw)
    r = subprocess.run([sys.executable, "-c", CHILD, io, str(Bt), str(L), str(D), str(W), sw],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "ok scan_vec" in r.stdout
