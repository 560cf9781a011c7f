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


# significand bits (with the implicit one) and smallest normal exponent of
# the storage dtypes an output can come back in
_FORMATS = (("bf16", 8, -126), ("f16", 11, -14), ("f32", 24, -126))


def storage_ulp(got, ref):
    """A unit in the last place, at |ref|, of the coarsest storage dtype in
    which every value of `got` is exactly representable (bf16, fp16 or fp32;
    0 for anything finer)."""
    g = np.asarray(got, np.float64)
    for name, bits, emin in _FORMATS:
        if np.array_equal(gen.round_to(g, name), g, equal_nan=True):
            e = np.floor(np.log2(np.maximum(np.abs(np.asarray(ref, np.float64)), 2.0 ** emin)))
            return 2.0 ** (e - (bits - 1))
    return 0.0


def assert_close(got, ref, tol, what="", ulps=0.5):
    """rel-L2 over the whole tensor <= tol (the acceptance bound), and every
    element within tol * (|ref| + rms(ref)) plus `ulps` units in the last place
    of the dtype the output is stored in, so that a wrong tile or tail cannot
    hide in the norm of a large tensor.  One stored rounding is half an ulp;
    a cache that both sides round to its dtype after each of k steps can
    drift apart by up to one ulp per step (each step adds one rounding on
    either side to the decayed earlier difference), so such comparisons pass
    ulps=k."""
    err = rel_l2(got, ref)
    g = np.asarray(got, np.float64)
    r = np.asarray(ref, np.float64)
    diff = np.abs(g - r)
    if not err <= tol:
        i = np.unravel_index(np.argmax(diff), diff.shape)
        raise AssertionError(f"{what}: rel-L2 {err:.3e} > {tol:.1e}; max |diff| {diff[i]:.3e} at {i}")
    if r.size:
        rms = float(np.sqrt(np.mean(r * r)))
        bound = tol * (np.abs(r) + rms) + ulps * storage_ulp(g, r)
        bad = ~(diff <= bound)
        if bad.any():
            ratio = np.where(bad, diff / np.maximum(bound, 1e-300), 0.0)
            i = np.unravel_index(np.argmax(ratio), ratio.shape)
            raise AssertionError(f"{what}: element {i} off by {diff[i]:.3e} > {bound[i]:.3e} "
                                 f"(= tol * (|ref| + rms) + {ulps} ulp), got {g[i]!r} want {r[i]!r}; "
                                 f"{int(bad.sum())} such elements; rel-L2 {err:.3e}")
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
