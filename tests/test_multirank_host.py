"""Host logic of the multi-GPU run (replicas only) on CPU: two gloo ranks.

The per-rank step times are combined as the maximum over ranks, the
whole-job value counts every rank's units, only rank 0 prints, and the
reference arm runs on rank 0 alone.  No GPU and no NCCL are involved."""
import json
import os
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
import json, os, sys
sys.path.insert(0, sys.argv[1])
import datetime
import torch.distributed as dist
import bench
dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
rank, world = dist.get_rank(), dist.get_world_size()
ms = [2.0, 3.5][rank]                      # rank 1 is the slow one
step = bench.max_over_ranks(ms, dist, "cpu")
value = bench.job_throughput(world, 1e9, step)
dist.barrier()
dist.destroy_process_group()
if rank == 0:
    print(json.dumps({"ms": step, "value": value, "world": world}), flush=True)
"""


def test_two_gloo_ranks_take_the_slowest_step_and_count_all_units(tmp_path):
    worker = tmp_path / "worker.py"
    worker.write_text(WORKER)
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), str(worker), ROOT]
    res = subprocess.run(cmd, capture_output=True, text=True, timeout=240, cwd=ROOT)
    assert res.returncode == 0, res.stderr[-3000:]
    lines = [ln for ln in res.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, res.stdout  # rank 0 only
    d = json.loads(lines[0])
    assert d["world"] == 2 and d["ms"] == pytest.approx(3.5)
    # 2 ranks x 1e9 units in 3.5 ms
    assert d["value"] == pytest.approx(2 * 1e9 / 3.5e-3 / 1e9)


def test_single_process_needs_no_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(1.25, None, "cpu") == 1.25
    assert bench.job_throughput(1, 2e9, 4.0) == pytest.approx(500.0)


def test_reference_arm_runs_on_rank_zero_only():
    """Under torchrun the reference arm's non-zero ranks exit 0 and print nothing."""
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    res = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--gpus", "2", "--steps", "1",
                          "--warmup", "3"], capture_output=True, text=True, timeout=120, cwd=ROOT, env=env)
    assert res.returncode == 0, res.stderr[-2000:]
    assert res.stdout.strip() == ""


@pytest.mark.parametrize("kind,entry,rows", [
    ("m1_decode", {"bytes_per_call": 206208320}, 1),
    ("m2_decode", {"bytes_per_call": 4331209248, "batch": 1639, "heads": 80, "P": 64, "N": 128}, 1),
    ("m2_prefill", {}, 1),
    ("gated_conv", {"roofline": {"algorithmic_bytes_per_launch": 134414336}}, 1),
    ("conv1d", {"roofline": {"algorithmic_bytes_per_launch": 168448000}}, 8),
])
def test_oracle_beside_each_sub_line_runs_on_the_host(kind, entry, rows):
    """The oracle timings attached to the bench's sub-lines run on the host
    (no GPU) and report a positive rate in the line's unit."""
    sys.path.insert(0, ROOT)
    import bench
    r = bench.oracle_beside(entry, kind, rows=rows)
    assert r["value"] > 0 and r["kind"] == "oracle" and r["cores"] == 1
    assert r["unit"] == ("Gelem/s" if kind == "m2_prefill" else "GB/s")
