"""The context-parallel driver's host logic on CPU: two and three gloo ranks
under torch.distributed.run, each holding one piece of the sequences.  The
library calls are replaced by the fp64 oracle (this test's own stand-in; the
product path calls the CUDA library), so what is checked is the driver's data
flow -- the halo and record all-gathers, which rank folds which records, the
caches each rank ends with -- against the oracle's whole-sequence prefill."""
import os
import re
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


WORKER = r"""
import sys
sys.path.insert(0, sys.argv[1])
import datetime
import numpy as np
import torch
import torch.distributed as dist
import oracle
from state_space_model_causal_b200 import inputs as gen
from state_space_model_causal_b200.context_parallel import TorchCollective, prefill_context_parallel

class OracleOps:
    # the three library calls, evaluated by the oracle on CPU tensors
    def scan(self, x, dt, A, B, C, D=None, z=None, dt_bias=None, dt_softplus=True, conv_weight=None,
             conv_bias=None, conv_state=None, ssm_state=None, out=None):
        n = lambda t: None if t is None else t.double().numpy()
        if x.dim() == 4:  # Mamba-2 layout
            o, h = oracle.scan_mamba2(n(x), n(dt), n(A), n(B), n(C), D=n(D), z=n(z), dt_bias=n(dt_bias),
                                      dt_softplus=dt_softplus, h0=n(ssm_state))
            out.copy_(torch.from_numpy(o))
            ssm_state.copy_(torch.from_numpy(h))
            return out
        o, h, cs = oracle.scan(n(x), n(dt), n(A), n(B), n(C), D=n(D), z=n(z), dt_bias=n(dt_bias),
                               dt_softplus=dt_softplus, conv_weight=n(conv_weight),
                               conv_bias=n(conv_bias), conv_state=n(conv_state), h0=n(ssm_state))
        out.copy_(torch.from_numpy(o))
        ssm_state.copy_(torch.from_numpy(h))
        if conv_state is not None:
            conv_state.copy_(torch.from_numpy(cs))
        return out
    def delta_sum(self, dt, dt_bias, dt_softplus):
        n = lambda t: None if t is None else t.double().numpy()
        return torch.from_numpy(oracle.delta_sum(n(dt), n(dt_bias), dt_softplus)).float()
    def carry_fold(self, state, A, S, h_end):
        st, a, sm, he = (t.double().numpy() for t in (state, A, S, h_end))
        if st.ndim == 4:  # Mamba-2 layout: heads' rows as channels, A and S repeated over them
            Bt, H, P, Nn = st.shape
            st, he = st.reshape(Bt, H * P, Nn), he.reshape(Bt, H * P, Nn)
            a, sm = np.repeat(a, P)[:, None].repeat(Nn, 1), np.repeat(sm, P, axis=1)
        state.copy_(torch.from_numpy(oracle.carry_fold(st, a, sm, he)).reshape(state.shape))
        return state

dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
comm = TorchCollective()
r, R = comm.rank, comm.world_size
lengths = [int(v) for v in sys.argv[2].split(",")]
assert len(lengths) == R
L = sum(lengths)
f = lambda a: torch.from_numpy(np.ascontiguousarray(a)).double()
if sys.argv[3] == "mamba2":
    s = gen.scan_m2_inputs(2, 3, 4, 5, L, io="f32", seed=41, tag="cphost2", h0=True)
    ref, href = oracle.scan_mamba2(s.x, s.dt, s.A, s.B, s.C, D=s.D, z=s.z, dt_bias=s.dt_bias, h0=s.h0)
    b = np.cumsum([0] + lengths)
    t0, t1 = int(b[r]), int(b[r + 1])
    sl = lambda a: f(a[..., t0:t1])
    h = f(s.h0) if r == 0 else torch.zeros(2, 3, 4, 5, dtype=torch.float64)
    out = prefill_context_parallel(sl(s.x), sl(s.dt), f(s.A), sl(s.B), sl(s.C), D=f(s.D), z=sl(s.z),
                                   dt_bias=f(s.dt_bias), ssm_state=h, comm=comm, ops=OracleOps())
    np.testing.assert_allclose(out.numpy(), ref[..., t0:t1], rtol=2e-6, atol=2e-6)
    if r == R - 1:
        np.testing.assert_allclose(h.numpy(), href, rtol=2e-6, atol=2e-6)
    dist.barrier()
    dist.destroy_process_group()
    print(f"ok rank {r}", flush=True)
    sys.exit(0)
s = gen.scan_inputs(2, L, 6, 4, W=4, io="f32", seed=40, tag="cphost", conv_state=True, h0=True)
ref, href, csref = oracle.scan(s.x, s.dt, s.A, s.B, s.C, D=s.D, z=s.z, dt_bias=s.dt_bias,
                               conv_weight=s.conv_weight, conv_bias=s.conv_bias,
                               conv_state=s.conv_state, h0=s.h0)
b = np.cumsum([0] + lengths)
t0, t1 = int(b[r]), int(b[r + 1])
sl = lambda a: f(a[..., t0:t1])
h = f(s.h0) if r == 0 else torch.zeros(2, 6, 4, dtype=torch.float64)
cs = f(s.conv_state) if r == 0 else torch.zeros(2, 6, 4, dtype=torch.float64)
out = prefill_context_parallel(sl(s.x), sl(s.dt), f(s.A), sl(s.B), sl(s.C), D=f(s.D), z=sl(s.z),
                               dt_bias=f(s.dt_bias), conv_weight=f(s.conv_weight),
                               conv_bias=f(s.conv_bias), conv_state=cs, ssm_state=h,
                               comm=comm, ops=OracleOps())
np.testing.assert_allclose(out.numpy(), ref[..., t0:t1], rtol=2e-6, atol=2e-6)
if r == R - 1:
    np.testing.assert_allclose(h.numpy(), href, rtol=2e-6, atol=2e-6)
    np.testing.assert_allclose(cs.numpy(), csref, rtol=0, atol=0)
dist.barrier()
dist.destroy_process_group()
print(f"ok rank {r}", flush=True)
"""


@pytest.mark.parametrize("lengths,layout", [("9,14", "mamba1"), ("5,11,7", "mamba1"), ("6,13,9", "mamba2")])
def test_context_parallel_driver_on_gloo_ranks(lengths, layout, tmp_path):
    worker = tmp_path / "worker.py"
    worker.write_text(WORKER)
    R = len(lengths.split(","))
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={R}",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), str(worker), ROOT, lengths, layout]
    res = subprocess.run(cmd, capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert res.returncode == 0, (res.stdout + res.stderr)[-4000:]
    # the ranks' lines may interleave: count the reports, not the lines
    assert sorted(re.findall(r"ok rank (\d+)", res.stdout)) == [str(r) for r in range(R)]
