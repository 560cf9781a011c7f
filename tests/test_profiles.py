"""The committed ncu summaries and the bench's use of them (CPU only).

Each summary under profiles/ that records DRAM traffic must be internally
consistent (bytes per launch = reads + writes, the stated ratio to the
algorithmic bytes), and the bench must report a summary's traffic only while
the kernel sources still hash to the value recorded in it."""
import glob
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _fields(path):
    rec = {}
    for line in open(path):
        if ":" in line and not line.startswith("#"):
            k, v = line.split(":", 1)
            rec[k.strip()] = v.strip()
    return rec


SUMMARIES = sorted(p for p in glob.glob(os.path.join(ROOT, "profiles", "*.txt"))
                   if "dram_bytes_per_launch" in _fields(p))


def test_there_are_traffic_summaries_for_every_bench_kernel():
    names = {os.path.basename(p) for p in SUMMARIES}
    for need in ("scan_bal_prefill_2p8b.txt", "scan_m2_prefill_2p7b.txt", "ssu_row_tma_decode_2p8b.txt",
                 "ssu_head_tma_mamba2_64x128_f16_R131072.txt", "ssu_head_tma_mamba2_64x128_f32_R131072.txt",
                 "ssu_head_tma_mamba2_128x256_bf16_R65536.txt", "ssu_head_tma_mamba2_128x256_f32_R65536.txt",
                 "gated_conv_lfm.txt", "conv1d_2p8b.txt"):
        assert need in names


@pytest.mark.parametrize("path", SUMMARIES, ids=os.path.basename)
def test_summary_is_consistent(path):
    rec = _fields(path)
    for key in ("kernel", "source_sha256_16", "source_files", "algorithmic_bytes_per_launch",
                "dram_bytes_read_MB", "dram_bytes_write_MB", "dram_bytes_per_launch", "traffic_over_algorithmic"):
        assert key in rec, key
    total = float(rec["dram_bytes_per_launch"])
    rw = (float(rec["dram_bytes_read_MB"]) + float(rec["dram_bytes_write_MB"])) * 1e6
    assert total == pytest.approx(rw, abs=1.0e4)  # the MB figures carry two decimals each
    ratio = total / float(rec["algorithmic_bytes_per_launch"])
    assert ratio == pytest.approx(float(rec["traffic_over_algorithmic"]), abs=1e-3)
    for f in rec["source_files"].split(","):
        assert os.path.isfile(os.path.join(ROOT, f.strip())), f


def test_bench_reports_traffic_only_for_the_profiled_source(tmp_path, monkeypatch):
    csrc = tmp_path / "state_space_model_causal_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "k.cu").write_text("__global__ void k() {}\n")
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    digest = bench.src_hash("k.cu")
    (tmp_path / "profiles" / "k.txt").write_text(
        f"# summary\nsource_sha256_16: {digest}\ndram_bytes_per_launch: 12345\n")
    assert bench.profiled_traffic("k.txt", ["k.cu"]) == 12345.0
    (csrc / "k.cu").write_text("__global__ void k() { }\n")  # the kernel changed since the capture
    assert bench.profiled_traffic("k.txt", ["k.cu"]) is None
    assert bench.profiled_traffic("missing.txt", ["k.cu"]) is None
