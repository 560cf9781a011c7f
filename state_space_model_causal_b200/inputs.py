"""Seeded synthetic inputs for the Mamba hot path.

This module is the ONLY code shared by the CUDA path's tests/benchmark and the
fp64 oracle.  It draws random numbers and rounds them to the storage dtype; it
holds none of the method's arithmetic (no conv, softplus, SiLU, exponential or
scan).  Every tensor comes from its own counter-based stream (numpy's Philox,
keyed by a hash of ``(seed, workload, tensor name, slab)``), is drawn in fp64
and rounded to its I/O dtype with round-to-nearest-even; the rounded values,
widened back to float64, are what both sides consume.

Workload recipes (the pages run real Mamba-2.8B / Mamba2 / Falcon-H1 layers;
these seeded tensors stand in for them -- no dataset items, no weights):

* ``scan_small``   B=1, L=128, D=64, N=16, fp32 I/O, no conv, h0 = 0.
* ``prefill_2p8b`` B=4, L=2048, D=5120, N=16, W=4, fp16 I/O, fp32 params/state.
* ``decode_2p8b``  B=245, D=5120, N=16, W=4, fp32 ssm/conv state ~ N(0,1),
  fp16 x/dt/z/B/C, one independent slab per layer.
* ``mamba2_64x128`` H=80, P=64, N=128, G=1, fp16 inputs, fp16/fp32 state.
* ``mamba2_128x256`` H=32, P=128, N=256, G=1, bf16 inputs, bf16/fp32 state.
* ``gated_conv_lfm``  double-gated short conv: B=4, L=2048, D=2048, W=3, fp16
  x and gates, fp32 weights and state (the LFM2.5 page gives only the model's
  size; the width and the conv width are choices, stated as such).

Distributions: x, z, B, C ~ N(0, 1); dt ~ U(-4, -1); dt_bias = the inverse of
softplus applied to U(1e-3, 0.1), i.e. log(expm1(u)); Mamba-1 A[d, n] = -(n+1);
Mamba-2 A[h] = -U(1, 16); D = 1; conv weight ~ N(0, sigma=0.2), conv bias 0;
states ~ N(0, 1) where a state is given.  Gated conv: x and both gates ~ N(0, 1),
weight ~ N(0, sigma=0.2), bias ~ N(0, sigma=0.1).
"""
from __future__ import annotations

import dataclasses
import hashlib
from typing import Optional

import numpy as np

IO_DTYPES = ("f32", "f16", "bf16")


# --------------------------------------------------------------------------
# streams and rounding
# --------------------------------------------------------------------------
def stream_key(*tags) -> int:
    """64-bit Philox key for a tuple of tags (seed, workload, name, slab...)."""
    h = hashlib.sha256("/".join(str(t) for t in tags).encode()).digest()
    return int.from_bytes(h[:8], "little")


def rng(*tags) -> np.random.Generator:
    return np.random.Generator(np.random.Philox(key=stream_key(*tags)))


def _bf16_bits(a32: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 bit patterns, round to nearest even (finite inputs)."""
    u = np.ascontiguousarray(a32, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def round_to(a, dtype: str) -> np.ndarray:
    """Round float64 values to ``dtype`` (RNE); return them as float64."""
    a = np.asarray(a, dtype=np.float64)
    if dtype == "f64":
        return a.copy()
    if dtype == "f32":
        return a.astype(np.float32).astype(np.float64)
    if dtype == "f16":
        return a.astype(np.float16).astype(np.float64)
    if dtype == "bf16":
        bits = _bf16_bits(a.astype(np.float32)).astype(np.uint32) << 16
        return bits.view(np.float32).astype(np.float64)
    raise ValueError(f"unknown dtype {dtype}")


def to_storage(a, dtype: str) -> np.ndarray:
    """float64 values (already representable) -> numpy array in storage form.
    bf16 is returned as its uint16 bit patterns."""
    a = np.asarray(a, dtype=np.float64)
    if dtype == "f32":
        return a.astype(np.float32)
    if dtype == "f16":
        return a.astype(np.float16)
    if dtype == "bf16":
        return _bf16_bits(a.astype(np.float32))
    raise ValueError(f"unknown dtype {dtype}")


def torch_dtype(dtype: str):
    import torch
    return {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}[dtype]


def to_torch(a, dtype: str, device="cpu", pin: bool = False):
    """float64 values -> torch tensor of ``dtype`` on ``device`` (bit-exact)."""
    import torch
    s = to_storage(a, dtype)
    if dtype == "bf16":
        t = torch.from_numpy(s.view(np.int16).copy()).view(torch.bfloat16)
    else:
        t = torch.from_numpy(np.ascontiguousarray(s).copy())
    if pin:
        t = t.pin_memory()
    return t.to(device) if str(device) != "cpu" else t


def from_torch(t) -> np.ndarray:
    """torch tensor (any of the three dtypes, any device) -> float64 numpy."""
    import torch
    return t.detach().to("cpu", torch.float64).numpy()


def normal(shape, *tags, std=1.0):
    return rng(*tags).standard_normal(size=shape) * std


def uniform(shape, lo, hi, *tags):
    return rng(*tags).uniform(lo, hi, size=shape)


def dt_bias_draw(shape, *tags):
    """dt_bias so that softplus(dt_bias) ~ U(1e-3, 0.1): log(expm1(u))."""
    u = uniform(shape, 1e-3, 0.1, *tags)
    return np.log(np.expm1(u))


# --------------------------------------------------------------------------
# prefill (Mamba-1 layout)
# --------------------------------------------------------------------------
@dataclasses.dataclass
class ScanInputs:
    x: np.ndarray            # (B, D, L)
    dt: np.ndarray           # (B, D, L)
    A: np.ndarray            # (D, N) fp32 values
    B: np.ndarray            # (B, G, N, L)
    C: np.ndarray            # (B, G, N, L)
    D: Optional[np.ndarray]  # (D,)
    z: Optional[np.ndarray]  # (B, D, L)
    dt_bias: Optional[np.ndarray]  # (D,)
    conv_weight: Optional[np.ndarray]  # (D, W)
    conv_bias: Optional[np.ndarray]    # (D,)
    conv_state: Optional[np.ndarray]   # (B, D, W)
    h0: Optional[np.ndarray]           # (B, D, N) fp32 values
    io: str = "f32"


def scan_inputs(Bt, L, D, N, *, G=1, W=0, io="f32", seed=0, tag="scan", with_z=True,
                with_D=True, with_dt_bias=True, conv_state=False, h0=False) -> ScanInputs:
    """Seeded prefill inputs; ``W=0`` means no fused conv."""
    t = (seed, tag)
    x = round_to(normal((Bt, D, L), *t, "x"), io)
    dt = round_to(uniform((Bt, D, L), -4.0, -1.0, *t, "dt"), io)
    A = round_to(-np.broadcast_to(np.arange(1, N + 1, dtype=np.float64), (D, N)), "f32")
    Bm = round_to(normal((Bt, G, N, L), *t, "B"), io)
    Cm = round_to(normal((Bt, G, N, L), *t, "C"), io)
    Dv = np.ones(D) if with_D else None
    z = round_to(normal((Bt, D, L), *t, "z"), io) if with_z else None
    db = round_to(dt_bias_draw((D,), *t, "dt_bias"), "f32") if with_dt_bias else None
    cw = cb = cs = None
    if W:
        cw = round_to(normal((D, W), *t, "conv_w", std=0.2), "f32")
        cb = np.zeros(D)
        if conv_state:
            cs = round_to(normal((Bt, D, W), *t, "conv_state"), io)
    hh = round_to(normal((Bt, D, N), *t, "h0"), "f32") if h0 else None
    return ScanInputs(x, dt, np.ascontiguousarray(A), Bm, Cm, Dv, z, db, cw, cb, cs, hh, io)


def scan_small(seed=0) -> ScanInputs:
    """B=1, L=128, D=64, N=16, fp32, no conv, h0 = 0."""
    return scan_inputs(1, 128, 64, 16, io="f32", seed=seed, tag="scan_small")


def prefill_2p8b(seed=0, Bt=4, L=2048, D=5120, N=16, W=4) -> ScanInputs:
    """Mamba-1 2.8B-shaped prefill: conv width 4 + SiLU + scan, fp16 I/O."""
    return scan_inputs(Bt, L, D, N, W=W, io="f16", seed=seed, tag="prefill_2p8b")


# --------------------------------------------------------------------------
# decode (single-token state update)
# --------------------------------------------------------------------------
# prefill (Mamba-2 layout)
# --------------------------------------------------------------------------
@dataclasses.dataclass
class ScanM2Inputs:
    x: np.ndarray            # (B, H, P, L)
    dt: np.ndarray           # (B, H, L)
    A: np.ndarray            # (H,) fp32 values
    B: np.ndarray            # (B, G, N, L)
    C: np.ndarray            # (B, G, N, L)
    D: Optional[np.ndarray]  # (H,)
    z: Optional[np.ndarray]  # (B, H, P, L)
    dt_bias: Optional[np.ndarray]  # (H,)
    h0: Optional[np.ndarray]       # (B, H, P, N) fp32 values
    io: str = "f32"


def scan_m2_inputs(Bt, H, P, N, L, *, G=1, io="f32", seed=0, tag="scan_m2", with_z=True,
                   with_D=True, with_dt_bias=True, h0=False) -> ScanM2Inputs:
    """Seeded Mamba-2-layout prefill inputs, distributions of the Mamba-2 SSU
    configs: x, z, B, C ~ N(0,1); dt ~ U(-4,-1); A = -U(1,16) per head; D = 1."""
    t = (seed, tag)
    x = round_to(normal((Bt, H, P, L), *t, "x"), io)
    dt = round_to(uniform((Bt, H, L), -4.0, -1.0, *t, "dt"), io)
    A = round_to(-uniform((H,), 1.0, 16.0, *t, "A"), "f32")
    Bm = round_to(normal((Bt, G, N, L), *t, "B"), io)
    Cm = round_to(normal((Bt, G, N, L), *t, "C"), io)
    Dv = np.ones(H) if with_D else None
    z = round_to(normal((Bt, H, P, L), *t, "z"), io) if with_z else None
    db = round_to(dt_bias_draw((H,), *t, "dt_bias"), "f32") if with_dt_bias else None
    hh = round_to(normal((Bt, H, P, N), *t, "h0"), "f32") if h0 else None
    return ScanM2Inputs(x, dt, A, Bm, Cm, Dv, z, db, hh, io)


# --------------------------------------------------------------------------
@dataclasses.dataclass
class SsuInputs:
    state: np.ndarray        # Mamba-1: (B, D, N); Mamba-2: (B, H, P, N)
    x: np.ndarray            # (B, D) or (B, H, P)
    dt: np.ndarray           # (B, D) or (B, H)
    A: np.ndarray            # (D, N) or (H,)
    B: np.ndarray            # (B, G, N)
    C: np.ndarray            # (B, G, N)
    D: Optional[np.ndarray]  # (D,) or (H,)
    z: Optional[np.ndarray]
    dt_bias: Optional[np.ndarray]
    conv_weight: Optional[np.ndarray] = None  # (D, W)
    conv_bias: Optional[np.ndarray] = None    # (D,)
    conv_state: Optional[np.ndarray] = None   # (B, D, W)
    io: str = "f16"
    state_dtype: str = "f32"
    conv_state_dtype: str = "f32"


def ssu_mamba1_inputs(Bt, D, N, *, W=4, G=1, io="f16", state="f32", conv_state_dtype="f32",
                      seed=0, tag="decode_2p8b", slab=0, with_z=True) -> SsuInputs:
    t = (seed, tag, slab)
    st = round_to(normal((Bt, D, N), *t, "state"), state)
    x = round_to(normal((Bt, D), *t, "x"), io)
    dt = round_to(uniform((Bt, D), -4.0, -1.0, *t, "dt"), io)
    A = round_to(-np.broadcast_to(np.arange(1, N + 1, dtype=np.float64), (D, N)), "f32")
    Bm = round_to(normal((Bt, G, N), *t, "B"), io)
    Cm = round_to(normal((Bt, G, N), *t, "C"), io)
    z = round_to(normal((Bt, D), *t, "z"), io) if with_z else None
    db = round_to(dt_bias_draw((D,), *t, "dt_bias"), "f32")
    cw = cb = cs = None
    if W:
        cw = round_to(normal((D, W), *t, "conv_w", std=0.2), "f32")
        cb = np.zeros(D)
        cs = round_to(normal((Bt, D, W), *t, "conv_state"), conv_state_dtype)
    return SsuInputs(st, x, dt, np.ascontiguousarray(A), Bm, Cm, np.ones(D), z, db, cw, cb, cs,
                     io, state, conv_state_dtype)


def decode_2p8b(slab=0, seed=0, Bt=245, D=5120, N=16, W=4) -> SsuInputs:
    """Mamba-1 2.8B-shaped decode step for one layer slab."""
    return ssu_mamba1_inputs(Bt, D, N, W=W, io="f16", state="f32", seed=seed, slab=slab)


def effective_batch_shape(R: int, H: int):
    """Effective batch R = batch * nheads.  R >= H: batch = ceil(R / H) with
    all H heads; R < H: batch 1 running the first R heads.  Returns
    (batch, heads_run)."""
    if R >= H:
        return -(-R // H), H
    return 1, R


def ssu_mamba2_inputs(Bt, H, P, N, *, G=1, io="f16", state="f16", seed=0, tag="mamba2",
                      with_z=False, with_D=True, dt_per_head=True) -> SsuInputs:
    t = (seed, tag)
    st = round_to(normal((Bt, H, P, N), *t, "state"), state)
    x = round_to(normal((Bt, H, P), *t, "x"), io)
    dshape = (Bt, H) if dt_per_head else (Bt, H, P)
    dt = round_to(uniform(dshape, -4.0, -1.0, *t, "dt"), io)
    A = round_to(-uniform((H,), 1.0, 16.0, *t, "A"), "f32")
    Bm = round_to(normal((Bt, G, N), *t, "B"), io)
    Cm = round_to(normal((Bt, G, N), *t, "C"), io)
    z = round_to(normal((Bt, H, P), *t, "z"), io) if with_z else None
    db = round_to(dt_bias_draw((H,), *t, "dt_bias"), "f32")
    Dv = np.ones(H) if with_D else None
    return SsuInputs(st, x, dt, A, Bm, Cm, Dv, z, db, io=io, state_dtype=state)


def mamba2_64x128(R, cache="f16", seed=0) -> SsuInputs:
    Bt, Hr = effective_batch_shape(R, 80)
    return ssu_mamba2_inputs(Bt, Hr, 64, 128, io="f16", state=cache, seed=seed,
                             tag=f"mamba2_64x128/R{R}")


def mamba2_128x256(R, cache="bf16", seed=0) -> SsuInputs:
    Bt, Hr = effective_batch_shape(R, 32)
    return ssu_mamba2_inputs(Bt, Hr, 128, 256, io="bf16", state=cache, seed=seed,
                             tag=f"mamba2_128x256/R{R}")


# --------------------------------------------------------------------------
# double-gated short causal conv
# --------------------------------------------------------------------------
@dataclasses.dataclass
class GatedConvInputs:
    x: np.ndarray                     # (B, D, L)
    bg: np.ndarray                    # (B, D, L) input gate
    cg: np.ndarray                    # (B, D, L) output gate
    weight: np.ndarray                # (D, W) fp32 values
    bias: Optional[np.ndarray]        # (D,)
    conv_state: Optional[np.ndarray]  # (B, D, W)
    io: str


def gated_conv_inputs(Bt, L, D, W, *, io="f16", seed=0, tag="gated_conv", bias=True,
                      conv_state=False, state_dtype="f32") -> GatedConvInputs:
    t = (seed, tag)
    x = round_to(normal((Bt, D, L), *t, "x"), io)
    bg = round_to(normal((Bt, D, L), *t, "bg"), io)
    cg = round_to(normal((Bt, D, L), *t, "cg"), io)
    w = round_to(normal((D, W), *t, "w", std=0.2), "f32")
    b = round_to(normal((D,), *t, "b", std=0.1), "f32") if bias else None
    cs = round_to(normal((Bt, D, W), *t, "conv_state"), state_dtype) if conv_state else None
    return GatedConvInputs(x, bg, cg, w, b, cs, io)


def gated_conv_lfm(seed=0, Bt=4, L=2048, D=2048, W=3) -> GatedConvInputs:
    """The double-gated conv workload: fp16 x and gates, a 3-wide conv."""
    return gated_conv_inputs(Bt, L, D, W, io="f16", seed=seed, tag="gated_conv_lfm")


# --------------------------------------------------------------------------
# device-side draws for sizes too large to draw on the host quickly
# --------------------------------------------------------------------------
def device_normal(shape, dtype: str, *tags, std=1.0, device="cuda"):
    """N(0, std) drawn by torch's Philox generator on ``device`` in fp32 and
    rounded to ``dtype``; the same tags give the same values."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(stream_key(*tags) & 0x7FFFFFFFFFFFFFFF)
    t = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(torch_dtype(dtype))


def device_uniform(shape, lo, hi, dtype: str, *tags, device="cuda"):
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(stream_key(*tags) & 0x7FFFFFFFFFFFFFFF)
    t = torch.rand(shape, generator=g, device=device, dtype=torch.float32)
    t.mul_(hi - lo).add_(lo)
    return t.to(torch_dtype(dtype))
