"""Benchmark of the Mamba hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]
                    [--sweep] [--no-decode]

Headline (one JSON line on rank 0): the fused prefill -- causal conv1d (W=4)
+ SiLU + selective scan + D skip + SiLU(z) gate -- of a Mamba-2.8B-shaped
layer, batch 4, L=2048, d_inner=5120, d_state=16, fp16 I/O, fp32 parameters
and state; value = scan elements B*L*D*N per second (Gelem/s).  One step is
one call of ssm_selective_scan_fwd on inputs already resident in HBM; L2 is
flushed before every step and only the kernel is inside each step's event
pair.  The same line carries the decode updates (ssm_selective_state_update)
measured in the same run: HBM GB/s and fraction of the measured copy peak for
the Mamba-1 2.8B-shaped decode step (64 layer slabs) and the Mamba-2 layouts at
their largest effective batch, and the double-gated short conv of an
LFM2-style conv block (HBM GB/s).

Multi-GPU: the work does not need an exchange between GPUs (every (b, d)
recurrence is independent), so N ranks run independent replicas (weak
scaling, no data-path collective); value = all ranks' elements / the slowest
rank's time.  --impl reference times the fp64 CPU oracle on a bounded sample of
the same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

METRIC = "scan Gelem/s (B·L·D·N) prefill; SSU decode HBM GB/s vs B200 peak, per batch"
WORKLOAD = "mamba1-2.8b-prefill: conv1d(W=4)+SiLU+selective-scan+gate, B=4 L=2048 D=5120 N=16, fp16 I/O"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_HBM_GBS = 6650.0
SFU_EX2_PER_CLK_PER_SM = 16  # nominal SFU ex2 throughput per SM per clock
# SFU operations per (b, t, d, n) element of the fused prefill: the decay
# exp(delta*A), plus per (b, t, d) the exponentials of the conv SiLU, the
# softplus and the gate (their reciprocals run on the FMA pipe), over N = 16
PREFILL_SFU_PER_ELEM = 1.0 + 3.0 / 16
NUM_SMS = 148
SM_MAX_MHZ = 1965.0


# --------------------------------------------------------------- helpers --
def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p.get("sm_max_mhz", SM_MAX_MHZ)), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, SM_MAX_MHZ, "fallback"


def probe_rates():
    """Every `name: value` line of profiles/sfu_pipe_rates.txt (the figures
    `python bench.py --peaks` printed on this machine's B200s)."""
    rec = {}
    try:
        for line in open(os.path.join(ROOT, "profiles", "sfu_pipe_rates.txt")):
            if ":" in line and not line.startswith("#"):
                k, v = line.split(":", 1)
                try:
                    rec[k.strip()] = float(v)
                except ValueError:
                    pass
    except OSError:
        pass
    return rec


def sfu_rate():
    """ex2 operations per clock per SM: the rate `python bench.py --peaks`
    measured on this machine's B200s (recorded in profiles/sfu_pipe_rates.txt),
    else the nominal 16."""
    try:
        for line in open(os.path.join(ROOT, "profiles", "sfu_pipe_rates.txt")):
            if line.startswith("ex2_per_clk_per_sm:"):
                return float(line.split(":", 1)[1]), "measured (bench.py --peaks)"
    except OSError:
        pass
    return float(SFU_EX2_PER_CLK_PER_SM), "nominal"


# Microbenchmark of the SFU: 16 independent chains per thread, inputs changed
# by an FMA every iteration, 8 warps per SM sub-partition.
PEAKS_SRC = r"""
#include <cstdio>
#include <cuda_runtime.h>
__device__ __forceinline__ float ex2(float x) { float y; asm volatile("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x)); return y; }
__device__ __forceinline__ float rcp(float x) { float y; asm volatile("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x)); return y; }
template <int OP> __global__ void k(float* out, int iters) {
  float x[16], acc[16];
  for (int j = 0; j < 16; ++j) { x[j] = -0.01f * (threadIdx.x + j); acc[j] = 0.f; }
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int j = 0; j < 16; ++j) { x[j] = fmaf(x[j], 0.9999f, -1e-4f); acc[j] += OP == 0 ? ex2(x[j]) : rcp(x[j] - 3.0f); }
  }
  float s = 0; for (int j = 0; j < 16; ++j) s += acc[j];
  if (s == 1234.5f) out[0] = s;
}
// STREAM-style copy: four 16-byte loads in flight per thread, then the stores
__global__ void copy16(const float4* __restrict__ a, float4* __restrict__ b, size_t n) {
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += 4 * stride) {
    float4 v[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) if (i + k * stride < n) v[k] = a[i + k * stride];
#pragma unroll
    for (int k = 0; k < 4; ++k) if (i + k * stride < n) b[i + k * stride] = v[k];
  }
}
int main() {
  float* d; if (cudaMalloc(&d, 4) != cudaSuccess) return 1;
  int sms, clk; cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, 0); cudaDeviceGetAttribute(&clk, cudaDevAttrClockRate, 0);
  cudaEvent_t a, b; cudaEventCreate(&a); cudaEventCreate(&b);
  for (int op = 0; op < 2; ++op) {
    const int iters = 4096, blocks = sms * 8;
    auto L = [&] { if (op == 0) k<0><<<blocks, 128>>>(d, iters); else k<1><<<blocks, 128>>>(d, iters); };
    L(); cudaDeviceSynchronize(); cudaEventRecord(a); L(); cudaEventRecord(b); cudaEventSynchronize(b);
    float ms; cudaEventElapsedTime(&ms, a, b);
    printf("%s_per_clk_per_sm: %.3f\n", op == 0 ? "ex2" : "rcp", (double)blocks * 128 * 16 * iters / (ms * 1e-3) / sms / (clk * 1e3));
  }
  {
    const size_t bytes = (size_t)2 << 30;  // 2 GiB each way, far beyond L2
    float4 *x, *y;
    if (cudaMalloc(&x, bytes) != cudaSuccess || cudaMalloc(&y, bytes) != cudaSuccess) return 1;
    cudaMemset(x, 0, bytes);
    const size_t n = bytes / 16;
    float best = 1e30f;
    for (int rep = 0; rep < 12; ++rep) {  // kernel copies, then the runtime's device-to-device copy
      cudaEventRecord(a);
      if (rep < 6) copy16<<<sms * 4, 512>>>(x, y, n);
      else cudaMemcpyAsync(y, x, bytes, cudaMemcpyDeviceToDevice, 0);
      cudaEventRecord(b);
      cudaEventSynchronize(b);
      float ms; cudaEventElapsedTime(&ms, a, b);
      if (rep != 0 && rep != 6 && ms < best) best = ms;  // the first of each kind warms up
    }
    printf("hbm_copy_gbs: %.1f\n", 2.0 * bytes / (best * 1e-3) / 1e9);
    cudaFree(x); cudaFree(y);
  }
  return cudaGetLastError() == cudaSuccess ? 0 : 1;
}
"""


def run_peaks():
    """Compile and run the SFU microbenchmark; print its rates at the max SM clock."""
    import tempfile
    with tempfile.TemporaryDirectory() as tmp:
        src = os.path.join(tmp, "sfu.cu")
        exe = os.path.join(tmp, "sfu")
        with open(src, "w") as f:
            f.write(PEAKS_SRC)
        subprocess.check_call(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-o", exe, src])
        out = subprocess.run([exe], capture_output=True, text=True, check=True).stdout
    print(out, end="", flush=True)
    return 0


def src_hash(*names):
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "state_space_model_causal_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(summary_name, source_files):
    """DRAM bytes per launch recorded in a committed ncu summary, if that
    summary was taken on the current kernel source (else None)."""
    path = os.path.join(ROOT, "profiles", summary_name)
    try:
        rec = {}
        for line in open(path):
            if ":" in line and not line.startswith("#"):
                k, v = line.split(":", 1)
                rec[k.strip()] = v.strip()
        if rec.get("source_sha256_16") != src_hash(*source_files):
            return None
        return float(rec["dram_bytes_per_launch"])
    except Exception:
        return None


class ClockSampler:
    """Samples this GPU's SM clock and clock-event reasons through NVML every
    few milliseconds while the timed region runs (read-only queries)."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"))

    def __init__(self, uuid, period_s=0.005):
        self.uuid = uuid
        self.period = period_s
        self.samples = []
        self.max_mhz = None
        self._stop = None
        self._thread = None
        self.error = None

    def __enter__(self):
        import threading
        try:
            import pynvml
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByUUID(self.uuid)
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
            masks = [(n, getattr(pynvml, attr)) for n, attr in self.REASONS]
        except Exception as e:  # no NVML: record why, keep running
            self.error = f"nvml unavailable: {e}"
            return self
        self._stop = threading.Event()

        def run():
            while not self._stop.is_set():
                try:
                    mhz = float(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM))
                    r = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                    self.samples.append((mhz, [n for n, m in masks if r & m]))
                except Exception as e:
                    self.error = str(e)
                    return
                self._stop.wait(self.period)

        self._thread = threading.Thread(target=run, daemon=True)
        self._thread.start()
        return self

    def __exit__(self, *exc):
        if self._thread is not None:
            self._stop.set()
            self._thread.join(timeout=2)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0,
                    "note": self.error or "no samples"}
        reasons = sorted({r for _, rs in self.samples for r in rs})
        return {"sm_mhz": statistics.median(m for m, _ in self.samples),
                "sm_max_mhz": self.max_mhz, "reasons": reasons, "samples": len(self.samples),
                "source": "NVML, 5 ms period, during the timed steps"}


def device_uuid(dev):
    import torch
    try:
        u = str(torch.cuda.get_device_properties(dev).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        return None


# --------------------------------------------------------------- prefill --
class Prefill:
    """Device-resident inputs and the call of the 2.8B-shaped prefill."""

    def __init__(self, dev, seed=0, Bt=4):
        import torch
        from state_space_model_causal_b200 import inputs as gen
        self.gen = gen
        s = gen.prefill_2p8b(seed=seed, Bt=Bt)
        self.s = s
        self.Bt, self.D, self.L = s.x.shape
        self.N = s.A.shape[1]
        self.W = s.conv_weight.shape[1]
        t = lambda a, dt: gen.to_torch(np.ascontiguousarray(a), dt, dev)  # noqa: E731
        self.x, self.dt, self.z = t(s.x, "f16"), t(s.dt, "f16"), t(s.z, "f16")
        self.B, self.C = t(s.B, "f16"), t(s.C, "f16")
        self.A, self.Dv = t(s.A, "f32"), t(s.D, "f32")
        self.db, self.cw, self.cb = t(s.dt_bias, "f32"), t(s.conv_weight, "f32"), t(s.conv_bias, "f32")
        self.h = torch.zeros(self.Bt, self.D, self.N, device=dev)
        self.cs = torch.zeros(self.Bt, self.D, self.W, device=dev)
        self.out = torch.empty_like(self.x)
        self.elems = self.Bt * self.L * self.D * self.N

    def algorithmic_bytes(self):
        BLD = self.Bt * self.L * self.D
        io = 4 * BLD * 2                                  # x, dt, z in + out, fp16
        bc = 2 * self.Bt * self.N * self.L * 2            # B, C
        params = self.D * self.N * 4 + self.D * 4 * 3 + self.D * self.W * 4
        states = self.Bt * self.D * (self.N + self.W) * 4  # final ssm/conv state written
        return io + bc + params + states

    def run(self, stream=None):
        from state_space_model_causal_b200 import ssm_selective_scan_fwd
        ssm_selective_scan_fwd(self.x, self.dt, self.A, self.B, self.C, D=self.Dv, z=self.z,
                               dt_bias=self.db, conv_weight=self.cw, conv_bias=self.cb,
                               conv_state=self.cs, ssm_state=self.h, out=self.out, stream=stream)


class PrefillM2:
    """Mamba-2-layout prefill, Mamba-2 2.7B-shaped layer (d_inner 5120 = 80 heads x
    headdim 64, dstate 128, one group), B=8, L=2048, fp16 I/O, fp32 state.  Inputs
    are drawn on the device and stored time-major as the model holds them (x as
    (B, L, H, P)), passed as their (B, H, P, L) views."""

    def __init__(self, dev, Bt=8, L=2048, H=80, P=64, N=128):
        import torch
        from state_space_model_causal_b200 import inputs as gen
        tag = ("bench", "prefill_m2")
        self.Bt, self.L, self.H, self.P, self.N = Bt, L, H, P, N
        view = lambda t: t.permute(0, 2, 3, 1)  # noqa: E731
        self.x = view(gen.device_normal((Bt, L, H, P), "f16", *tag, "x", device=dev))
        self.z = view(gen.device_normal((Bt, L, H, P), "f16", *tag, "z", device=dev))
        self.dt = gen.device_uniform((Bt, L, H), -4.0, -1.0, "f16", *tag, "dt", device=dev).permute(0, 2, 1)
        self.B = view(gen.device_normal((Bt, L, 1, N), "f16", *tag, "B", device=dev))
        self.C = view(gen.device_normal((Bt, L, 1, N), "f16", *tag, "C", device=dev))
        self.A = -torch.from_numpy(gen.uniform((H,), 1.0, 16.0, *tag, "A").astype(np.float32)).to(dev)
        self.db = torch.from_numpy(gen.dt_bias_draw((H,), *tag, "db").astype(np.float32)).to(dev)
        self.Dv = torch.ones(H, device=dev)
        self.h = gen.device_normal((Bt, H, P, N), "f32", *tag, "h0", device=dev)
        self.out = view(torch.empty(Bt, L, H, P, dtype=torch.float16, device=dev))
        self.elems = Bt * L * H * P * N

    def algorithmic_bytes(self):
        io = 3 * self.Bt * self.L * self.H * self.P * 2 + self.Bt * self.L * self.H * 2  # x, z, out; dt
        bc = 2 * self.Bt * self.L * self.N * 2
        state = 2 * self.Bt * self.H * self.P * self.N * 4  # read and written
        return io + bc + state + 3 * self.H * 4

    def run(self):
        from state_space_model_causal_b200 import ssm_selective_scan_fwd
        ssm_selective_scan_fwd(self.x, self.dt, self.A, self.B, self.C, D=self.Dv, z=self.z,
                               dt_bias=self.db, ssm_state=self.h, out=self.out)


def prefill_mamba2(dev, hbm_peak, sm_max, steps=20, warmup=3):
    """Mamba-2-layout prefill: CUDA events per step, L2 flushed before each."""
    import torch
    pm = PrefillM2(dev)
    flush = L2Flush(dev)
    ms = time_prefill(pm, steps, warmup, dev, flush)
    mean = statistics.mean(ms)
    gel = pm.elems / (mean * 1e-3) / 1e9
    # FP32 pipe: 128 lanes per SM.  Per state element and step the recurrence
    # needs at least two FP32 operations (the state update and the readout,
    # as the kernel's rescaled form does them); written directly it needs
    # three (delta*x*B, the decay FMA, the readout FMA).  The peak is the
    # two-operation floor; the three-operation figure is reported beside it.
    fp32_peak = NUM_SMS * 128 * sm_max * 1e6 / 2 / 1e9  # Gelem/s
    fp32_peak_direct = fp32_peak * 2 / 3
    alg = pm.algorithmic_bytes()
    gbs = alg / (mean * 1e-3) / 1e9
    traffic = profiled_traffic("scan_m2_prefill_2p7b.txt", ["scan_m2.cu", "common.cuh"])
    del pm
    torch.cuda.empty_cache()
    return {"workload": "mamba2-2.7b-prefill: B=8 L=2048 H=80 P=64 N=128 G=1, fp16 I/O, fp32 state, "
                        "time-major rows",
            "us_per_call": round(mean * 1e3, 2), "Gelem_s": round(gel, 1),
            "roofline": {"bound": "alu", "achieved": round(gel, 1), "peak": round(fp32_peak, 1),
                         "unit": "Gelem/s", "frac": round(gel / fp32_peak, 4), "traffic": traffic,
                         "peak_kind": "FP32 pipe 128 lanes/SM x 148 SMs x max SM clock / 2 ops per element",
                         "frac_of_direct_form_bound": round(gel / fp32_peak_direct, 4),
                         "hbm_achieved_gbs": round(gbs, 1), "hbm_peak_gbs": hbm_peak,
                         "hbm_frac": round(gbs / hbm_peak, 4), "algorithmic_bytes_per_launch": alg},
            "l2": "flushed before every step (256 MiB write, then a 256 MiB read of another buffer, so no dirty line is left to write back)", "gpu_launches": steps}


def prefill_single_sequence(dev, sfu_peak, hbm_peak, steps=20, warmup=3):
    """The 2.8B-shaped prefill at batch 1 (320 units of 16 channels, fewer
    than the 1184 worker warps): the context-parallel mode, two launches per
    call (pieces from zero states with carry records, then the re-scan from
    the composed states).  CUDA events per call, L2 flushed before each."""
    import torch
    from state_space_model_causal_b200 import LaunchInfo, ssm_selective_scan_fwd
    pf = Prefill(dev, Bt=1)
    # the plan: work_items = base units x (pieces - 1) per pass; pieces of
    # ceil(chunks / pieces) 32-step chunks; pass 1 runs pieces 0 .. S-2 and
    # pass 2 pieces 1 .. S-1, so per base unit (S-2) * piece + all chunks run
    info = LaunchInfo()
    ssm_selective_scan_fwd(pf.x, pf.dt, pf.A, pf.B, pf.C, D=pf.Dv, z=pf.z, dt_bias=pf.db,
                           conv_weight=pf.cw, conv_bias=pf.cb, conv_state=pf.cs, ssm_state=pf.h,
                           out=pf.out, info=info)
    nck = -(-pf.L // 32)
    base_units = pf.Bt * pf.D // 16
    pieces = info.work_items // base_units + 1
    piece = -(-nck // pieces)
    work_factor = ((pieces - 2) * piece + nck) / nck
    flush = L2Flush(dev)
    ms = time_prefill(pf, steps, warmup, dev, flush)
    mean = statistics.mean(ms)
    gel = pf.elems / (mean * 1e-3) / 1e9
    alg = pf.algorithmic_bytes()
    del pf
    torch.cuda.empty_cache()
    return {"workload": "mamba1-2.8b-prefill, one sequence: B=1 L=2048 D=5120 N=16 W=4, fp16 I/O "
                        "(context-parallel pieces, two launches per call)",
            "us_per_call": round(mean * 1e3, 2), "Gelem_s": round(gel, 1),
            "roofline": {"bound": "alu", "achieved": round(gel, 1), "peak": round(sfu_peak, 1),
                         "unit": "Gelem/s", "frac": round(gel / sfu_peak, 4), "traffic": None,
                         "peak_kind": "SFU ex2 rate x 148 SMs x max SM clock (one exp per element)",
                         "pieces": pieces, "executed_work_factor": round(work_factor, 4),
                         "frac_of_executed_work": round(gel * work_factor / sfu_peak, 4),
                         "hbm_achieved_gbs": round(alg / (mean * 1e-3) / 1e9, 1), "hbm_peak_gbs": hbm_peak},
            "l2": "flushed before every step (256 MiB write, then a 256 MiB read of another buffer, so no dirty line is left to write back)", "gpu_launches": 2 * steps}


class GatedConv:
    """The double-gated short conv of an LFM2-style conv block, B=4, L=2048,
    D=2048, W=3, fp16: x and both gates are the three D-wide slices of one
    token-major (B, L, 3D) projection output (drawn on the device), the output
    is token-major (B, L, D), the conv state fp32."""

    def __init__(self, dev, Bt=4, L=2048, D=2048, W=3):
        import torch
        from state_space_model_causal_b200 import inputs as gen
        tag = ("bench", "gated_conv")
        self.Bt, self.L, self.D, self.W = Bt, L, D, W
        self.proj = gen.device_normal((Bt, L, 3 * D), "f16", *tag, "proj", device=dev)
        self.bg, self.cg, self.x = (self.proj[:, :, i * D:(i + 1) * D].transpose(1, 2) for i in range(3))
        self.w = gen.device_normal((D, W), "f32", *tag, "w", std=0.2, device=dev)
        self.b = gen.device_normal((D,), "f32", *tag, "b", std=0.1, device=dev)
        self.cs = torch.zeros(Bt, D, W, device=dev)
        self.out = torch.empty(Bt, L, D, dtype=torch.float16, device=dev).transpose(1, 2)
        self.elems = Bt * L * D

    def algorithmic_bytes(self):
        io = 4 * self.Bt * self.L * self.D * 2            # x, b_gate, c_gate in, out
        params = self.D * (self.W + 1) * 4
        state = self.Bt * self.D * (2 * self.W - 1) * 4   # W-1 entries read, W written
        return io + params + state

    def run(self):
        from state_space_model_causal_b200 import ssm_gated_conv1d_fwd
        ssm_gated_conv1d_fwd(self.x, self.bg, self.cg, self.w, bias=self.b, conv_state=self.cs, out=self.out)


def gated_conv_lfm(dev, hbm_peak, steps=20, warmup=3):
    """The double-gated conv: CUDA events per call, L2 flushed before each."""
    import torch
    gc = GatedConv(dev)
    flush = L2Flush(dev)
    ms = time_prefill(gc, steps, warmup, dev, flush)
    mean = statistics.mean(ms)
    alg = gc.algorithmic_bytes()
    gbs = alg / (mean * 1e-3) / 1e9
    traffic = profiled_traffic("gated_conv_lfm.txt", ["gconv.cu", "common.cuh"])
    entry = {"workload": "double-gated short conv (LFM2-style conv block): B=4 L=2048 D=2048 W=3, fp16 "
                         "x/gates (slices of one token-major projection), token-major out, fp32 state",
             "us_per_call": round(mean * 1e3, 2), "Gelem_s": round(gc.elems / (mean * 1e-3) / 1e9, 1),
             "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm_peak, "unit": "GB/s",
                          "frac": round(gbs / hbm_peak, 4), "traffic": traffic,
                          "algorithmic_bytes_per_launch": alg},
             "l2": "flushed before every step (256 MiB write, then a 256 MiB read of another buffer, so no dirty line is left to write back)", "gpu_launches": steps}
    del gc
    torch.cuda.empty_cache()
    return entry


class Conv1d:
    """The standalone causal conv1d of one Mamba-1 2.8B layer: x (B=4,
    D=5120, L=2048) fp16 time-contiguous, W=4, bias, SiLU, an fp32 conv state
    read and written."""

    def __init__(self, dev, Bt=4, D=5120, L=2048, W=4):
        import torch
        from state_space_model_causal_b200 import inputs as gen
        tag = ("bench", "conv1d")
        self.Bt, self.D, self.L, self.W = Bt, D, L, W
        self.x = gen.device_normal((Bt, D, L), "f16", *tag, "x", device=dev)
        self.w = gen.device_normal((D, W), "f32", *tag, "w", std=0.2, device=dev)
        self.b = gen.device_normal((D,), "f32", *tag, "b", std=0.1, device=dev)
        self.cs = gen.device_normal((Bt, D, W), "f32", *tag, "cs", device=dev)
        self.out = torch.empty_like(self.x)
        self.elems = Bt * D * L

    def algorithmic_bytes(self):
        io = 2 * self.Bt * self.D * self.L * 2            # x in, out
        params = self.D * (self.W + 1) * 4
        state = self.Bt * self.D * (2 * self.W - 1) * 4   # W-1 entries read, W written
        return io + params + state

    def run(self):
        from state_space_model_causal_b200 import ssm_causal_conv1d_fwd
        ssm_causal_conv1d_fwd(self.x, self.w, bias=self.b, conv_state=self.cs, silu=True, out=self.out)


def conv1d_2p8b(dev, hbm_peak, steps=20, warmup=3):
    """The standalone conv1d: CUDA events per call, L2 flushed before each."""
    import torch
    cv = Conv1d(dev)
    flush = L2Flush(dev)
    ms = time_prefill(cv, steps, warmup, dev, flush)
    mean = statistics.mean(ms)
    alg = cv.algorithmic_bytes()
    gbs = alg / (mean * 1e-3) / 1e9
    traffic = profiled_traffic("conv1d_2p8b.txt", ["conv1d.cu", "common.cuh"])
    entry = {"workload": "mamba1-2.8b conv1d: B=4 D=5120 L=2048 W=4, fp16 time-contiguous x/out, bias, "
                         "SiLU, fp32 conv state",
             "us_per_call": round(mean * 1e3, 2), "Gelem_s": round(cv.elems / (mean * 1e-3) / 1e9, 1),
             "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm_peak, "unit": "GB/s",
                          "frac": round(gbs / hbm_peak, 4), "traffic": traffic,
                          "algorithmic_bytes_per_launch": alg},
             "l2": "flushed before every step (256 MiB write, then a 256 MiB read of another buffer, so no dirty line is left to write back)", "gpu_launches": steps}
    del cv
    torch.cuda.empty_cache()
    return entry


LEAD_CYCLES = 200_000  # ~0.1 ms of device time queued ahead of each timed call


class L2Flush:
    """Empties L2 between timed steps: writes a buffer twice the L2 size,
    then reads another one as large.  The read evicts the dirty lines of the
    write (and of the previous step's outputs) before the timed call starts,
    so the call neither finds its inputs in L2 nor pays for write-backs that
    are not its own."""

    def __init__(self, dev):
        import torch
        self.w = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
        self.r = torch.zeros(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
        self.out = torch.empty((), dtype=torch.float32, device=dev)

    def __call__(self):
        import torch
        self.w.zero_()
        torch.sum(self.r, 0, out=self.out)


def time_prefill(pf, steps, warmup, dev, flush):
    """Per-step CUDA events around the kernel only, L2 flushed before each
    step.  A short device-side sleep follows the flush, so that the host has
    already queued the call (whose Python marshalling takes tens of
    microseconds) when the start event fires: the pair then brackets device
    work only, which matters for kernels of a few tens of microseconds."""
    import torch
    stream = torch.cuda.current_stream(dev)
    for _ in range(warmup):
        flush()
        pf.run()
    torch.cuda.synchronize(dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    for a, b in ev:
        flush()
        torch.cuda._sleep(LEAD_CYCLES)
        a.record(stream)
        pf.run()
        b.record(stream)
    torch.cuda.synchronize(dev)
    return [a.elapsed_time(b) for a, b in ev]


def time_prefill_e2e(pf, steps, warmup, dev):
    """Same metric end to end: pinned host inputs -> device, the C-ABI call,
    result back to pinned host memory, all inside each step's event pair."""
    import torch
    host = {k: getattr(pf, k).cpu().pin_memory() for k in ("x", "dt", "z", "B", "C")}
    back = {k: torch.empty_like(getattr(pf, k), device="cpu").pin_memory()
            for k in ("out", "h", "cs")}
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = sum(v.numel() * v.element_size() for v in back.values())
    stream = torch.cuda.current_stream(dev)

    def step():
        for k, v in host.items():
            getattr(pf, k).copy_(v, non_blocking=True)
        pf.h.zero_()
        pf.cs.zero_()
        pf.run()
        for k, v in back.items():
            v.copy_(getattr(pf, k), non_blocking=True)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize(dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    for a, b in ev:
        a.record(stream)
        step()
        b.record(stream)
    torch.cuda.synchronize(dev)
    ms = [a.elapsed_time(b) for a, b in ev]
    return ms, h2d, d2h


def time_prefill_e2e_pipelined(pf, steps, warmup, dev):
    """The end-to-end metric with the steps pipelined the way a stream of
    prefills runs: two sets of device buffers; step i's inputs go up on a
    copy stream while step i-1 computes on a second stream and step i-2's
    results come down on a third (the two copy directions use separate copy
    engines).  Every step still copies all its inputs from pinned host memory
    and reads its results back.  Returns (ms per step, H2D bytes, D2H bytes)
    from events around the whole run: the first upload to the last download."""
    import torch
    from state_space_model_causal_b200 import ssm_selective_scan_fwd
    names_in, names_out = ("x", "dt", "z", "B", "C"), ("out", "h", "cs")
    host = {k: getattr(pf, k).cpu().pin_memory() for k in names_in}
    back = [{k: torch.empty_like(getattr(pf, k), device="cpu").pin_memory() for k in names_out}
            for _ in range(2)]
    sets = [{k: getattr(pf, k) for k in names_in + names_out}]
    sets.append({k: torch.empty_like(v) for k, v in sets[0].items()})
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = sum(v.numel() * v.element_size() for v in back[0].values())
    up, comp, down = (torch.cuda.Stream(dev) for _ in range(3))
    done_comp = [torch.cuda.Event() for _ in range(2)]   # set j's inputs consumed
    done_down = [torch.cuda.Event() for _ in range(2)]   # set j's results read back
    ready = [torch.cuda.Event() for _ in range(2)]       # set j's inputs uploaded
    for j in range(2):  # nothing pending yet
        done_comp[j].record(comp)
        done_down[j].record(down)

    def step(i):
        j = i % 2
        S, hb = sets[j], back[j]
        with torch.cuda.stream(up):
            up.wait_event(done_comp[j])
            for k in names_in:
                S[k].copy_(host[k], non_blocking=True)
            ready[j].record(up)
        with torch.cuda.stream(comp):
            comp.wait_event(ready[j])
            comp.wait_event(done_down[j])
            S["h"].zero_()
            S["cs"].zero_()
            ssm_selective_scan_fwd(S["x"], S["dt"], pf.A, S["B"], S["C"], D=pf.Dv, z=S["z"],
                                   dt_bias=pf.db, conv_weight=pf.cw, conv_bias=pf.cb,
                                   conv_state=S["cs"], ssm_state=S["h"], out=S["out"], stream=comp)
            done_comp[j].record(comp)
        with torch.cuda.stream(down):
            down.wait_event(done_comp[j])
            for k in names_out:
                hb[k].copy_(S[k], non_blocking=True)
            done_down[j].record(down)

    for i in range(warmup):
        step(i)
    torch.cuda.synchronize(dev)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(up)
    for i in range(steps):
        step(i)
    b.record(down)
    torch.cuda.synchronize(dev)
    return a.elapsed_time(b) / steps, h2d, d2h


# ---------------------------------------------------------------- decode --
def graph_time(calls, replays, dev, warm_eager=3):
    """Per-call microseconds: `calls` (a list of closures) captured in one
    CUDA graph, 5 warm replays, `replays` timed replays (events per replay)."""
    import torch
    for _ in range(warm_eager):
        for c in calls:
            c()
    torch.cuda.synchronize(dev)
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream(dev)
    s.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            for c in calls:
                c()
    torch.cuda.current_stream(dev).wait_stream(s)
    for _ in range(5):
        g.replay()
    torch.cuda.synchronize(dev)
    lat = []
    for _ in range(replays):
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        g.replay()
        b.record()
        b.synchronize()
        lat.append(a.elapsed_time(b))
    del g
    per_call = [1000.0 * l / len(calls) for l in lat]
    return statistics.mean(per_call), statistics.median(per_call)


def decode_mamba1_2p8b(dev, hbm_peak, slabs=64, replays=20):
    """Mamba-1 2.8B-shaped decode: B=245, D=5120, N=16, W=4; fp32 ssm and conv
    state ~ N(0,1), fp16 x/dt/z/B/C; one independent slab per layer, each call
    of the graph on the next slab (13.2 GB per replay, far above L2)."""
    import torch
    from state_space_model_causal_b200 import inputs as gen, ssm_selective_state_update
    Bt, D, N, W = 245, 5120, 16, 4
    tag = ("bench", "decode_2p8b")
    calls, bufs = [], []
    for k in range(slabs):
        st = gen.device_normal((Bt, D, N), "f32", *tag, k, "state", device=dev)
        cs = gen.device_normal((Bt, D, W), "f32", *tag, k, "cs", device=dev)
        x = gen.device_normal((Bt, D), "f16", *tag, k, "x", device=dev)
        dt = gen.device_uniform((Bt, D), -4.0, -1.0, "f16", *tag, k, "dt", device=dev)
        z = gen.device_normal((Bt, D), "f16", *tag, k, "z", device=dev)
        Bm = gen.device_normal((Bt, 1, N), "f16", *tag, k, "B", device=dev)
        Cm = gen.device_normal((Bt, 1, N), "f16", *tag, k, "C", device=dev)
        A = -torch.arange(1, N + 1, device=dev, dtype=torch.float32).repeat(D, 1)
        Dv = torch.ones(D, device=dev)
        db = torch.from_numpy(gen.dt_bias_draw((D,), *tag, k, "db").astype(np.float32)).to(dev)
        cw = gen.device_normal((D, W), "f32", *tag, k, "cw", std=0.2, device=dev)
        cb = torch.zeros(D, device=dev)
        out = torch.empty_like(x)
        b = (st, x, dt, A, Bm, Cm, Dv, z, db, cw, cb, cs, out)
        bufs.append(b)
        calls.append(lambda b=b: ssm_selective_state_update(
            b[0], b[1], b[2], b[3], b[4], b[5], D=b[6], z=b[7], dt_bias=b[8], conv_weight=b[9],
            conv_bias=b[10], conv_state=b[11], out=b[12]))
    us, med = graph_time(calls, replays, dev)
    BD = Bt * D
    nbytes = (BD * N * 4 * 2 + BD * ((W - 1) + W) * 4 + BD * 2 * 3 + BD * 2
              + Bt * N * 2 * 2 + D * N * 4 + D * 4 * 3 + D * W * 4)
    gbs = nbytes / (us * 1e-6) / 1e9
    del bufs, calls
    torch.cuda.empty_cache()
    traffic = profiled_traffic("ssu_row_tma_decode_2p8b.txt", ["ssu.cu", "common.cuh", "tma.cuh"])
    return {"workload": "mamba1-2.8b-decode: B=245 D=5120 N=16 W=4, fp32 ssm/conv state, fp16 io, 64 slabs",
            "us_per_call": round(us, 3), "us_median": round(med, 3), "bytes_per_call": nbytes,
            "GBps": round(gbs, 1), "frac_of_hbm_peak": round(gbs / hbm_peak, 4),
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm_peak, "unit": "GB/s",
                         "frac": round(gbs / hbm_peak, 4), "traffic": traffic},
            "l2": "each call on a different 100 MB slab", "gpu_launches_per_replay": slabs}


def decode_mamba2(dev, hbm_peak, H, P, N, R, cache, io, method="cold", replays=10, calls_per_graph=5):
    """Mamba-2 SSU at effective batch R, timed one of two ways:

    * "cold": the calls of the graph rotate over ceil(2 * L2 / slab) state
      slabs (at least `calls_per_graph` calls, one per slab when there are
      more slabs), so no call finds its state in L2;
    * "pages": the timing method of the vLLM SSU benchmark -- 20 eager warm-up
      calls, a graph of 10 calls on the same buffers, 5 warm replays, 100
      timed replays; at small R the state stays in L2.
    """
    import torch
    from state_space_model_causal_b200 import inputs as gen, ssm_selective_state_update
    Bt, Hr = gen.effective_batch_shape(R, H)
    es = 4 if cache == "f32" else 2
    state_bytes = Bt * Hr * P * N * es
    if method == "pages":
        nslab, ncalls, warm_eager, replays = 1, 10, 20, 100
    else:
        nslab = max(1, math.ceil(2 * L2_BYTES / state_bytes))
        ncalls, warm_eager = max(calls_per_graph, nslab), 3
    tag = ("bench", "mamba2", H, P, N, R, cache)
    A = -torch.from_numpy(gen.uniform((Hr,), 1.0, 16.0, *tag, "A").astype(np.float32)).to(dev)
    db = torch.from_numpy(gen.dt_bias_draw((Hr,), *tag, "db").astype(np.float32)).to(dev)
    Dv = torch.ones(Hr, device=dev)
    calls, bufs = [], []
    for k in range(nslab):
        st = gen.device_normal((Bt, Hr, P, N), cache, *tag, k, "state", device=dev)
        x = gen.device_normal((Bt, Hr, P), io, *tag, k, "x", device=dev)
        dt = gen.device_uniform((Bt, Hr), -4.0, -1.0, io, *tag, k, "dt", device=dev)
        Bm = gen.device_normal((Bt, 1, N), io, *tag, k, "B", device=dev)
        Cm = gen.device_normal((Bt, 1, N), io, *tag, k, "C", device=dev)
        out = torch.empty_like(x)
        b = (st, x, dt, Bm, Cm, out)
        bufs.append(b)
    for i in range(ncalls):
        b = bufs[i % nslab]
        calls.append(lambda b=b: ssm_selective_state_update(
            b[0], b[1], b[2], A, b[3], b[4], D=Dv, dt_bias=db, out=b[5]))
    us, med = graph_time(calls, replays, dev, warm_eager=warm_eager)
    rows = Bt * Hr * P
    nbytes = rows * N * es * 2 + rows * 2 * 2 + Bt * Hr * 2 + Bt * N * 2 * 2 + Hr * 4 * 3
    gbs = nbytes / (us * 1e-6) / 1e9
    del bufs, calls
    torch.cuda.empty_cache()
    traffic = profiled_traffic(f"ssu_head_tma_mamba2_{P}x{N}_{cache}_R{R}.txt",
                               ["ssu.cu", "common.cuh", "tma.cuh"])
    l2 = (f"{nslab} state slabs rotated ({nslab * state_bytes / 2**20:.0f} MiB, >= 2 x L2 or one slab larger)"
          if method == "cold" else f"same buffers, {state_bytes / 2**20:.1f} MiB of state")
    return {"workload": f"mamba2-ssu: H={H} P={P} N={N} G=1, {io} io, {cache} cache",
            "method": method,
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm_peak, "unit": "GB/s",
                         "frac": round(gbs / hbm_peak, 4), "traffic": traffic},
            "requested_R": R, "effective_batch": Bt * Hr, "batch": Bt, "heads": Hr, "P": P, "N": N,
            "us_per_call": round(us, 3), "us_median": round(med, 3), "bytes_per_call": nbytes,
            "GBps": round(gbs, 1), "frac_of_hbm_peak": round(gbs / hbm_peak, 4), "l2": l2,
            "calls_per_graph": ncalls}


def eager_latency(dev, R, calls=300):
    """Host cost of one eager ssm_selective_state_update call (Mamba-2 layout,
    H=80 P=64 N=128, fp16): the wall time per call of `calls` back-to-back
    calls of the C entry point with its argument struct built once (library
    checks, planning and launch), and through the Python binding (argument
    marshalling included).  The GPU work of these sizes is shorter than the
    host path, so the host path is what is timed."""
    import ctypes

    import torch
    from state_space_model_causal_b200 import binding, inputs as gen, ssm_selective_state_update
    H, P, N = 80, 64, 128
    Bt, Hr = gen.effective_batch_shape(R, H)
    tag = ("bench", "eager", R)
    st = gen.device_normal((Bt, Hr, P, N), "f16", *tag, "state", device=dev)
    x = gen.device_normal((Bt, Hr, P), "f16", *tag, "x", device=dev)
    dt = gen.device_uniform((Bt, Hr), -4.0, -1.0, "f16", *tag, "dt", device=dev)
    Bm = gen.device_normal((Bt, 1, N), "f16", *tag, "B", device=dev)
    Cm = gen.device_normal((Bt, 1, N), "f16", *tag, "C", device=dev)
    A = -torch.linspace(1.0, 16.0, Hr, device=dev)
    Dv, db = torch.ones(Hr, device=dev), torch.full((Hr,), -3.0, device=dev)
    out = torch.empty_like(x)
    a = binding.SsuArgs()
    a.struct_size = ctypes.sizeof(binding.SsuArgs)
    a.state, a.x, a.dt, a.A, a.B, a.C, a.D, a.dt_bias, a.out = map(binding.describe, (st, x, dt, A, Bm, Cm, Dv, db, out))
    a.dt_softplus = 1
    lib = binding.library()
    stream = torch.cuda.current_stream(dev).cuda_stream
    for _ in range(20):
        if lib.ssm_selective_state_update(ctypes.byref(a), stream) != 0:
            raise RuntimeError("ssm_selective_state_update refused the eager-latency case")
    torch.cuda.synchronize(dev)
    t0 = time.perf_counter()
    for _ in range(calls):
        lib.ssm_selective_state_update(ctypes.byref(a), stream)
    t_c = (time.perf_counter() - t0) / calls
    torch.cuda.synchronize(dev)
    t0 = time.perf_counter()
    for _ in range(calls):
        ssm_selective_state_update(st, x, dt, A, Bm, Cm, D=Dv, dt_bias=db, out=out)
    t_py = (time.perf_counter() - t0) / calls
    torch.cuda.synchronize(dev)
    return {"requested_R": R, "effective_batch": Bt * Hr, "c_call_us": round(t_c * 1e6, 2),
            "python_call_us": round(t_py * 1e6, 2)}


# ------------------------------------------------------------- reference --
def oracle_prefill_sample(channels, seed=0):
    """Time the fp64 oracle on `channels` full-length (b, d) channels of the
    2.8B-shaped prefill recipe (at most the workload's 4 x 5120); returns
    (seconds, elements)."""
    import oracle
    from state_space_model_causal_b200 import inputs as gen
    channels = max(1, min(4 * 5120, channels))
    Bt = -(-channels // 5120)
    s = gen.prefill_2p8b(seed=seed, Bt=Bt, D=-(-channels // Bt))
    t0 = time.perf_counter()
    oracle.scan(s.x, s.dt, s.A, s.B, s.C, D=s.D, z=s.z, dt_bias=s.dt_bias,
                conv_weight=s.conv_weight, conv_bias=s.conv_bias)
    dt = time.perf_counter() - t0
    return dt, s.x.shape[0] * s.x.shape[1] * s.x.shape[2] * s.A.shape[1]


def oracle_beside(entry, kind, rows=None):
    """Time the fp64 oracle (one host thread) on a bounded sample of a sub-line's
    workload and express it in that line's unit, so that every measured kernel
    has the oracle timed beside it.  kind: "m1_decode", "m2_decode",
    "m2_prefill", "gated_conv" or "conv1d"; rows overrides the sample size
    (tests)."""
    import oracle
    from state_space_model_causal_b200 import inputs as gen
    if kind == "m1_decode":
        Bt = rows or 245
        s = gen.ssu_mamba1_inputs(Bt, 5120, 16, W=4, io="f16", state="f32", seed=0, tag="oracle_beside")
        t0 = time.perf_counter()
        oracle.ssu(s.state[:, :, None, :], s.x[:, :, None], s.dt[:, :, None], s.A[:, None, :], s.B, s.C,
                   D=s.D[:, None], z=s.z[:, :, None], dt_bias=s.dt_bias[:, None],
                   conv_weight=s.conv_weight, conv_bias=s.conv_bias, conv_state=s.conv_state)
        dt = time.perf_counter() - t0
        per_row = entry["bytes_per_call"] / (245 * 5120)
        value, unit = Bt * 5120 * per_row / dt / 1e9, "GB/s"
        sample = f"{Bt} of the 245 batch rows (all 5120 channels), one decode step"
    elif kind == "m2_decode":
        H, P, N = entry["heads"], entry["P"], entry["N"]
        Bt = rows or 16
        s = gen.ssu_mamba2_inputs(Bt, H, P, N, io="f32", state="f32", seed=0, tag="oracle_beside")
        t0 = time.perf_counter()
        oracle.ssu_mamba2(s.state, s.x, s.dt, s.A, s.B, s.C, D=s.D, dt_bias=s.dt_bias)
        dt = time.perf_counter() - t0
        per_b = entry["bytes_per_call"] / entry["batch"]
        value, unit = Bt * per_b / dt / 1e9, "GB/s"
        sample = f"{Bt} batch rows x {H} heads, one decode step"
    elif kind == "gated_conv":
        Bt = rows or 1
        s = gen.gated_conv_inputs(Bt, 2048, 2048, 3, io="f16", seed=0, tag="oracle_beside")
        t0 = time.perf_counter()
        oracle.gated_conv1d(s.x, s.bg, s.cg, s.weight, bias=s.bias)
        dt = time.perf_counter() - t0
        per_elem = entry["roofline"]["algorithmic_bytes_per_launch"] / (4 * 2048 * 2048)
        value, unit = Bt * 2048 * 2048 * per_elem / dt / 1e9, "GB/s"
        sample = f"{Bt} of the 4 batch entries, all 2048 channels, full L=2048"
    elif kind == "conv1d":
        chans = rows or 5120
        s = gen.normal((1, chans, 2048), "oracle_beside", "conv1d", "x")
        w = gen.normal((chans, 4), "oracle_beside", "conv1d", "w", std=0.2)
        b = gen.normal((chans,), "oracle_beside", "conv1d", "b", std=0.1)
        cs = gen.normal((1, chans, 4), "oracle_beside", "conv1d", "cs")
        t0 = time.perf_counter()
        oracle.conv1d(s, w, bias=b, conv_state=cs, silu=True)
        dt = time.perf_counter() - t0
        per_elem = entry["roofline"]["algorithmic_bytes_per_launch"] / (4 * 5120 * 2048)
        value, unit = chans * 2048 * per_elem / dt / 1e9, "GB/s"
        sample = f"{chans} of the 20480 (b, d) rows, full L=2048"
    elif kind == "m2_prefill":
        heads = rows or 8
        s = gen.scan_m2_inputs(1, heads, 64, 128, 2048, io="f16", seed=0, tag="oracle_beside")
        t0 = time.perf_counter()
        oracle.scan_mamba2(s.x, s.dt, s.A, s.B, s.C, D=s.D, z=s.z, dt_bias=s.dt_bias)
        dt = time.perf_counter() - t0
        value, unit = heads * 64 * 128 * 2048 / dt / 1e9, "Gelem/s"
        sample = f"{heads} of the 640 (b, h) heads, full L=2048"
    else:
        raise ValueError(kind)
    return {"value": round(value, 6), "unit": unit, "cores": 1, "kind": "oracle",
            "sample": f"{sample}; fp64 sequential C on one host thread, {dt:.2f} s"}


def oracle_prefill_threads(channels, threads, seed=0):
    """The oracle on `channels` channels of the prefill recipe split into
    `threads` contiguous channel ranges, one host thread each (the C oracle
    runs with the GIL released, and channels are independent); returns
    (wall seconds, elements)."""
    from concurrent.futures import ThreadPoolExecutor

    import oracle
    from state_space_model_causal_b200 import inputs as gen
    channels = max(threads, min(4 * 5120, channels))
    Bt = -(-channels // 5120)
    s = gen.prefill_2p8b(seed=seed, Bt=Bt, D=-(-channels // Bt))
    Dd = s.x.shape[1]
    cuts = [Dd * i // threads for i in range(threads + 1)]
    parts = [slice(cuts[i], cuts[i + 1]) for i in range(threads) if cuts[i + 1] > cuts[i]]

    def one(sl):
        oracle.scan(s.x[:, sl], s.dt[:, sl], s.A[sl], s.B, s.C, D=s.D[sl], z=s.z[:, sl],
                    dt_bias=s.dt_bias[sl], conv_weight=s.conv_weight[sl], conv_bias=s.conv_bias[sl])

    with ThreadPoolExecutor(len(parts)) as pool:
        t0 = time.perf_counter()
        list(pool.map(one, parts))
        dt = time.perf_counter() - t0
    return dt, s.x.shape[0] * Dd * s.x.shape[2] * s.A.shape[1]


def cpu_baseline(target_s=10.0):
    """The fp64 oracle timed on the host: on every core the process may use
    (one channel range per thread), plus the one-thread figure beside it."""
    import oracle
    oracle.build()
    t1, e1 = oracle_prefill_sample(64)
    one_thread = e1 / t1 / 1e9
    cores = max(1, min(64, len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity")
                       else (os.cpu_count() or 1)))
    ch = max(cores, min(4 * 5120, int(64 * cores * target_s / max(t1, 1e-3))))
    t, e = oracle_prefill_threads(ch, cores)
    ch = e // (2048 * 16)
    return {"value": round(e / t / 1e9, 6), "unit": "Gelem/s", "cores": cores, "kind": "oracle",
            "single_thread_value": round(one_thread, 6),
            "sample": f"{ch} of the 20480 (b,d) channels of the 2.8B-shaped prefill, full "
                      f"L=2048, fp64 C over {cores} host threads (one channel range each), "
                      f"{t:.1f} s; one thread: 64 channels in {t1:.3f} s"}


# ------------------------------------------------------- multi-rank host --
def max_over_ranks(ms_step, pg, device):
    """The step time of the job: the slowest rank's (every rank calls this
    once, in the same order).  pg is torch.distributed or None."""
    if pg is None:
        return float(ms_step)
    import torch
    t = torch.tensor([float(ms_step)], dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world, units_per_rank, ms_step):
    """Whole-job units per second (Gunits/s): every rank processes the same
    fixed work (weak scaling), the job is as slow as its slowest rank."""
    return world * units_per_rank / (ms_step * 1e-3) / 1e9


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    oracle.build()
    cores = max(1, min(64, len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity")
                       else (os.cpu_count() or 1)))
    t, _ = oracle_prefill_sample(64)
    # up to 5 s of CPU work per step over every host core, less when there
    # are many steps, so that the whole run stays near two and a half minutes
    per_step_s = max(0.5, min(5.0, 150.0 / max(1, args.steps + args.warmup)))
    ch = max(64, min(4 * 5120, int(64 * cores * per_step_s / max(t, 1e-3))))
    for _ in range(args.warmup):
        oracle_prefill_threads(ch, cores)
    times, elems = [], 0
    for _ in range(args.steps):
        t, e = oracle_prefill_threads(ch, cores)
        times.append(t)
        elems = e
    ch = elems // (2048 * 16)
    ms = 1000.0 * statistics.mean(times)
    value = elems / (ms / 1000.0) / 1e9
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "Gelem/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms, 3), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD, "sample": f"{ch} channels x L=2048 per step",
                       "l2": "n/a (host)"},
            "cpu_baseline": {"value": round(value, 6), "unit": "Gelem/s", "cores": cores,
                             "kind": "oracle",
                             "sample": f"{ch} (b,d) channels x L=2048 per step over {cores} threads"},
            "e2e": {"value": round(value, 6), "unit": "Gelem/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- sweep --
def run_sweep(dev, hbm_peak):
    """Mamba-2 SSU per effective batch, both timing methods, both cache dtypes
    of both configs; then the eager host latency per call."""
    out = []
    grids = ((80, 64, 128, ("f16", "f32"), "f16",
              (8, 16, 32, 64, 128, 256, 512, 1024, 2048, 4096, 8192, 16384, 32768, 65536, 131072)),
             (32, 128, 256, ("bf16", "f32"), "bf16",
              (8, 16, 32, 64, 128, 256, 512, 1024, 2048, 4096, 8192, 16384, 32768, 65536)))
    for H, P, N, caches, io, Rs in grids:
        for cache in caches:
            for R in Rs:
                for method in (("pages", "cold") if R <= 2048 else ("cold",)):
                    r = decode_mamba2(dev, hbm_peak, H, P, N, R, cache, io, method=method, replays=20)
                    print(json.dumps(r), flush=True)
                    out.append(r)
    for R in (8, 64, 256, 1024):
        r = eager_latency(dev, R)
        print(json.dumps({"eager_host_latency": r}), flush=True)
        out.append(r)
    return out


# ------------------------------------------------------ single cases --
def run_only(args, dev):
    """Warm-up then timed launches of one case, nothing else (profiling)."""
    import torch
    from state_space_model_causal_b200 import inputs as gen, ssm_selective_state_update
    if args.only == "prefill":
        pf = Prefill(dev)
        fn = pf.run
    elif args.only == "prefill_m2":
        pm = PrefillM2(dev)
        fn = pm.run
    elif args.only == "gated_conv":
        gc = GatedConv(dev)
        fn = gc.run
    elif args.only == "conv1d":
        cv = Conv1d(dev)
        fn = cv.run
    elif args.only == "decode_m1":
        Bt, D, N, W = args.B, 5120, 16, 4  # default: two layers' worth of rows, 200 MB of state
        tag = ("only", "decode_m1")
        st = gen.device_normal((Bt, D, N), "f32", *tag, "state", device=dev)
        cs = gen.device_normal((Bt, D, W), "f32", *tag, "cs", device=dev)
        x = gen.device_normal((Bt, D), "f16", *tag, "x", device=dev)
        dt = gen.device_uniform((Bt, D), -4.0, -1.0, "f16", *tag, "dt", device=dev)
        z = gen.device_normal((Bt, D), "f16", *tag, "z", device=dev)
        Bm = gen.device_normal((Bt, 1, N), "f16", *tag, "B", device=dev)
        Cm = gen.device_normal((Bt, 1, N), "f16", *tag, "C", device=dev)
        A = -torch.arange(1, N + 1, device=dev, dtype=torch.float32).repeat(D, 1)
        Dv, db = torch.ones(D, device=dev), torch.full((D,), -3.0, device=dev)
        cw = gen.device_normal((D, W), "f32", *tag, "cw", std=0.2, device=dev)
        out = torch.empty_like(x)
        fn = lambda: ssm_selective_state_update(st, x, dt, A, Bm, Cm, D=Dv, z=z, dt_bias=db,  # noqa
                                                conv_weight=cw, conv_state=cs, out=out)
    else:
        H, P, N, cache, io = {"m2_f16": (80, 64, 128, "f16", "f16"),
                              "m2_f32": (80, 64, 128, "f32", "f16"),
                              "m2_bf16": (32, 128, 256, "bf16", "bf16"),
                              "m2_f32_256": (32, 128, 256, "f32", "bf16")}[args.only]
        Bt, Hr = gen.effective_batch_shape(args.R, H)
        tag = ("only", args.only, args.R)
        st = gen.device_normal((Bt, Hr, P, N), cache, *tag, "state", device=dev)
        x = gen.device_normal((Bt, Hr, P), io, *tag, "x", device=dev)
        dt = gen.device_uniform((Bt, Hr), -4.0, -1.0, io, *tag, "dt", device=dev)
        Bm = gen.device_normal((Bt, 1, N), io, *tag, "B", device=dev)
        Cm = gen.device_normal((Bt, 1, N), io, *tag, "C", device=dev)
        A = -torch.linspace(1.0, 16.0, Hr, device=dev)
        Dv, db = torch.ones(Hr, device=dev), torch.full((Hr,), -3.0, device=dev)
        out = torch.empty_like(x)
        fn = lambda: ssm_selective_state_update(st, x, dt, A, Bm, Cm, D=Dv, dt_bias=db, out=out)  # noqa
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize(dev)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(args.steps):
        fn()
    b.record()
    torch.cuda.synchronize(dev)
    print(f"{args.only}: {a.elapsed_time(b) * 1000 / args.steps:.1f} us per launch", flush=True)
    return 0


# ----------------------------------------------------------------- main --
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--sweep", action="store_true", help="per-effective-batch decode sweep lines")
    ap.add_argument("--peaks", action="store_true", help="measure the SFU ex2 / rcp rates and exit")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--only", choices=["prefill", "prefill_m2", "decode_m1", "m2_f16", "m2_f32",
                                       "m2_bf16", "m2_f32_256", "gated_conv", "conv1d"],
                    help="run --warmup then --steps launches of one case and exit "
                         "(for profiler captures; prints no JSON line)")
    ap.add_argument("--R", type=int, default=16384, help="effective batch for --only m2_*")
    ap.add_argument("--B", type=int, default=490, help="batch for --only decode_m1")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    if args.impl == "reference":
        return run_reference(args)
    if args.peaks:
        return run_peaks()

    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
        pg = dist

    import state_space_model_causal_b200 as pkg
    pkg.library()  # fails loudly when the extension is missing
    hbm_peak, sm_max, peak_src = peaks()
    if args.sweep:
        if rank == 0:
            run_sweep(dev, hbm_peak)
        return 0

    if args.only:
        return run_only(args, dev)

    pf = Prefill(dev)
    flush = L2Flush(dev)

    if pg:
        pg.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(device_uuid(dev)) as clk:
        ms = time_prefill(pf, args.steps, args.warmup, dev, flush)
    torch.cuda.synchronize(dev)
    if pg:
        pg.barrier()
    ms_step = max_over_ranks(statistics.mean(ms), pg, dev)
    value = job_throughput(world, pf.elems, ms_step)

    # roofline of the prefill kernel: one exp(delta*A) per element on the SFU
    ex2_rate, ex2_kind = sfu_rate()
    sfu_peak = NUM_SMS * ex2_rate * sm_max * 1e6 / 1e9  # Gelem/s
    alg_bytes = pf.algorithmic_bytes()
    hbm_gbs = alg_bytes / (ms_step * 1e-3) / 1e9
    traffic = profiled_traffic("scan_bal_prefill_2p8b.txt", ["scan_bal.cu", "common.cuh"])
    achieved = pf.elems / (ms_step * 1e-3) / 1e9
    roofline = {"bound": "alu", "achieved": round(achieved, 2),
                "peak": round(sfu_peak, 1), "unit": "Gelem/s",
                "frac": round(achieved / sfu_peak, 4),
                "traffic": traffic,
                "peak_kind": f"SFU ex2 {ex2_rate:g}/clk/SM ({ex2_kind}) x {NUM_SMS} SMs x max SM clock",
                "sfu_ops_per_elem": PREFILL_SFU_PER_ELEM,
                "frac_all_sfu_ops": round(achieved * PREFILL_SFU_PER_ELEM / sfu_peak, 4),
                "hbm_achieved_gbs": round(hbm_gbs, 1), "hbm_peak_gbs": hbm_peak,
                "hbm_frac": round(hbm_gbs / hbm_peak, 4), "hbm_peak_kind": peak_src,
                "algorithmic_bytes_per_launch": alg_bytes}

    e2e_ms, h2d, d2h = time_prefill_e2e(pf, max(3, args.steps // 4), 3, dev)
    e2e_serial = world * pf.elems / (statistics.mean(e2e_ms) * 1e-3) / 1e9
    e2e_pipe_ms, _, _ = time_prefill_e2e_pipelined(pf, max(6, args.steps // 4), 3, dev)
    e2e_val = world * pf.elems / (e2e_pipe_ms * 1e-3) / 1e9

    prefill_m2 = prefill_mamba2(dev, hbm_peak, sm_max) if not args.no_decode else None
    prefill_b1 = prefill_single_sequence(dev, sfu_peak, hbm_peak) if not args.no_decode else None
    gated_conv = gated_conv_lfm(dev, hbm_peak) if not args.no_decode else None
    conv1d = conv1d_2p8b(dev, hbm_peak) if not args.no_decode else None

    decode = []
    if not args.no_decode:
        decode.append(decode_mamba1_2p8b(dev, hbm_peak))
        decode.append(decode_mamba2(dev, hbm_peak, 80, 64, 128, 131072, "f16", "f16"))
        decode.append(decode_mamba2(dev, hbm_peak, 80, 64, 128, 131072, "f32", "f16"))
        decode.append(decode_mamba2(dev, hbm_peak, 32, 128, 256, 65536, "bf16", "bf16"))
        decode.append(decode_mamba2(dev, hbm_peak, 32, 128, 256, 65536, "f32", "bf16"))

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        cpu = cpu_baseline()
        # the oracle timed beside every other measured kernel, in its line's unit
        if prefill_m2:
            prefill_m2["oracle"] = oracle_beside(prefill_m2, "m2_prefill")
        if prefill_b1:  # the same per-channel work as the headline's sample
            prefill_b1["oracle"] = dict(cpu, sample="the headline's cpu_baseline (same recipe, per channel): "
                                                    + cpu["sample"])
        for i, entry in enumerate(decode):
            entry["oracle"] = oracle_beside(entry, "m1_decode" if i == 0 else "m2_decode")
        if gated_conv:
            gated_conv["oracle"] = oracle_beside(gated_conv, "gated_conv")
        if conv1d:
            conv1d["oracle"] = oracle_beside(conv1d, "conv1d")

    if pg:
        pg.barrier()
        pg.destroy_process_group()
    if rank != 0:
        return 0
    line = {"metric": METRIC, "value": round(value, 2), "unit": "Gelem/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic",
            "config": {"workload": WORKLOAD, "global_batch": 4 * world, "seq_len": 2048,
                       "d_inner": 5120, "d_state": 16, "conv_width": 4, "io_dtype": "f16",
                       "parallelism": f"replicas x{world}",
                       "l2": "flushed before every step (256 MiB write, then a 256 MiB read of another "
                             "buffer, so no dirty line is left to write back); inputs 338 MB > 126 MB L2"},
            "roofline": roofline, "cpu_baseline": cpu,
            "e2e": {"value": round(e2e_val, 3), "unit": "Gelem/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_pipe_ms, 3),
                    "method": "pipelined: step i's inputs upload while step i-1 computes and step i-2's "
                              "results download (two device buffer sets, three streams), events from "
                              "the first upload to the last download",
                    "serial_value": round(e2e_serial, 3),
                    "serial_method": "one step at a time: upload, call, download inside each step's events"},
            "gpu_launches": args.steps, "clocks": clk.summary(),
            "peaks": {"hbm_gbs": hbm_peak, "hbm_kind": peak_src,
                      "hbm_copy_probe_gbs": probe_rates().get("hbm_copy_gbs"),
                      "ex2_per_clk_per_sm": ex2_rate, "ex2_kind": ex2_kind,
                      "note": "roofline fractions use hbm_gbs (MEASURED_PEAKS.json, else the fallback "
                              "figure); the copy probe of bench.py --peaks is context"},
            "prefill_mamba2": prefill_m2,
            "prefill_one_sequence": prefill_b1,
            "gated_conv": gated_conv,
            "conv1d": conv1d,
            "decode": decode}
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
