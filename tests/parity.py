"""Shared helpers for the GPU parity tests: tolerance, rel-L2, and runners that
feed the same rounded inputs to the CUDA path (through the C ABI binding) and
to the fp64 oracle."""
from __future__ import annotations

import numpy as np

import oracle
from state_space_model_causal_b200 import inputs as gen

# rel-L2 bounds: 1e-5 for fp32 I/O, 3e-3 for fp16/bf16 I/O (state in any dtype)
TOL = {"f32": 1e-5, "f16": 3e-3, "bf16": 3e-3}


def rel_l2(got, ref) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    den = np.linalg.norm(ref.ravel())
    num = np.linalg.norm((got - ref).ravel())
    return float(num / den) if den > 0 else float(num)


def assert_close(got, ref, tol, what=""):
    err = rel_l2(got, ref)
    if not err <= tol:
        diff = np.abs(np.asarray(got, np.float64) - np.asarray(ref, np.float64))
        i = np.unravel_index(np.argmax(diff), diff.shape)
        raise AssertionError(f"{what}: rel-L2 {err:.3e} > {tol:.1e}; max |diff| {diff[i]:.3e} at {i}")
    return err


def T(a, dtype, device="cuda"):
    """float64 numpy -> torch tensor of dtype on device (None passes through)."""
    if a is None:
        return None
    return gen.to_torch(np.ascontiguousarray(a), dtype, device)


def N(t):
    return None if t is None else gen.from_torch(t)


# --------------------------------------------------------------- prefill --
def run_scan_gpu(s: gen.ScanInputs, *, with_state=True, conv_state_dtype="f32", softplus=True):
    import torch
    from state_space_model_causal_b200 import ssm_selective_scan_fwd
    io = s.io
    Bt, D, L = s.x.shape
    N_ = s.A.shape[1]
    x, dt, z = T(s.x, io), T(s.dt, io), T(s.z, io)
    Bm, Cm = T(s.B, io), T(s.C, io)
    A = T(s.A, "f32")
    Dv = T(s.D, "f32")
    db = T(s.dt_bias, "f32")
    cw = T(s.conv_weight, "f32")
    cb = T(s.conv_bias, "f32")
    cs = None
    if s.conv_weight is not None and with_state:
        W = s.conv_weight.shape[1]
        cs0 = s.conv_state if s.conv_state is not None else np.zeros((Bt, D, W))
        cs = T(cs0, conv_state_dtype)
    h = None
    if with_state:
        h = T(s.h0 if s.h0 is not None else np.zeros((Bt, D, N_)), "f32")
    out = ssm_selective_scan_fwd(x, dt, A, Bm, Cm, D=Dv, z=z, dt_bias=db, dt_softplus=softplus,
                                 conv_weight=cw, conv_bias=cb, conv_state=cs, ssm_state=h)
    torch.cuda.synchronize()
    return N(out), N(h), N(cs)


def run_scan_oracle(s: gen.ScanInputs, softplus=True):
    return oracle.scan(s.x, s.dt, s.A, s.B, s.C, D=s.D, z=s.z, dt_bias=s.dt_bias,
                       dt_softplus=softplus, conv_weight=s.conv_weight, conv_bias=s.conv_bias,
                       conv_state=s.conv_state, h0=s.h0)
