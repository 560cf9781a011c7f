"""fp64 CPU oracle for the Mamba hot path -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline /
reference legs may import this package.  The product (the CUDA library and its
binding in ``state_space_model_causal_b200``) never imports, links or calls it,
and this package never imports the product.  The arithmetic lives in
``oracle.c`` (plain C, double precision, sequential loops); this module only
compiles it with gcc, marshals numpy arrays to contiguous float64 and returns
the results.

Functions (see the header comment of ``oracle.c`` for the definitions):

* :func:`conv1d` -- causal depthwise conv1d, optional SiLU, conv-state out
  (operator "causal-conv1d", "feat(llama.cu): 适配 mamba 模型" section 2.1).
* :func:`scan` -- fused prefill: conv -> SiLU -> softplus(dt + dt_bias) ->
  selective scan -> D skip -> SiLU(z) gate, per channel sequentially over t
  (operators "causal-conv1d, selective-scan, silu, element-mul", same section).
* :func:`ssu` -- single-token selective_state_update in the general
  (B, H, P, N) form, with optional fused conv-state roll (Mamba-1 decode);
  argument list of the selective_state_update call in "[XPU] Add tuned Mamba
  SSU configs for Intel Arc Pro B70", section 关键源码片段.
* :func:`ssu_mamba2` -- the same update in the Mamba-2 notation (scalar A,
  dt, D and dt_bias per head, ngroups), written separately in C.
* :func:`delta_sum` and :func:`carry_fold` -- a prefill cut into sequence
  pieces: the sum of a piece's steps delta, and the state entering the next
  piece, exp(A * sum delta) * h_in + h_end (the pieces of a context-parallel
  prefill; the long-context claim of "feat(llama.cu): 适配 mamba 模型" section
  6.1).
* :func:`gated_conv1d` -- the double-gated short causal conv of the
  "double-gated LIV convolution blocks" named in "LFM2.5-1.2B-Thinking性能优化
  CUDA核心编程技巧" section 2.1, on the reading out = Cg * conv(Bg * x) (the
  page prints no equation; see ``oracle.c``).
* :func:`round_cache` -- a state rounded to its cache dtype (fp32, fp16, bf16;
  nearest, ties to even); :func:`ssu` and :func:`ssu_mamba2` apply it to the
  updated state when given ``cache_dtype``, after the step's readout has used
  the unrounded state, so that several consecutive decode steps can be
  compared with a GPU cache kept in that dtype.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

_dp = ctypes.POINTER(ctypes.c_double)
_i64 = ctypes.c_int64


def build(force: bool = False) -> str:
    """Compile ``oracle.c`` into ``liboracle.so`` next to it (gcc, -O2, no fast-math)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c99", "-fno-fast-math", "-ffp-contract=off", "-shared", "-fPIC",
             _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def configure(lib):
    """Declare the C signatures on a loaded oracle library and return it."""
    lib.oracle_round_cache.restype = ctypes.c_int
    lib.oracle_round_cache.argtypes = [_dp, _i64, ctypes.c_int]
    lib.oracle_silu.restype = ctypes.c_double
    lib.oracle_silu.argtypes = [ctypes.c_double]
    lib.oracle_softplus.restype = ctypes.c_double
    lib.oracle_softplus.argtypes = [ctypes.c_double]
    lib.oracle_conv1d.restype = ctypes.c_int
    lib.oracle_conv1d.argtypes = [_i64] * 4 + [_dp] * 4 + [ctypes.c_int] + [_dp] * 2
    lib.oracle_scan.restype = ctypes.c_int
    lib.oracle_scan.argtypes = [_i64] * 6 + [_dp] * 8 + [ctypes.c_int] + [_dp] * 4 + [_dp] * 3
    lib.oracle_ssu.restype = ctypes.c_int
    lib.oracle_ssu.argtypes = [_i64] * 6 + [_dp] * 9 + [ctypes.c_int] + [_dp] * 3 + [_dp]
    lib.oracle_ssu_mamba2.restype = ctypes.c_int
    lib.oracle_ssu_mamba2.argtypes = [_i64] * 5 + [_dp] * 8 + [_dp] + [ctypes.c_int] + [_dp]
    lib.oracle_scan_mamba2.restype = ctypes.c_int
    lib.oracle_scan_mamba2.argtypes = [_i64] * 6 + [_dp] * 8 + [ctypes.c_int] + [_dp] * 3
    lib.oracle_delta_sum.restype = ctypes.c_int
    lib.oracle_delta_sum.argtypes = [_i64] * 3 + [_dp] * 2 + [ctypes.c_int] + [_dp]
    lib.oracle_carry_fold.restype = ctypes.c_int
    lib.oracle_carry_fold.argtypes = [_i64] * 3 + [_dp] * 4
    lib.oracle_gated_conv1d.restype = ctypes.c_int
    lib.oracle_gated_conv1d.argtypes = [_i64] * 4 + [_dp] * 8
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            _lib = configure(ctypes.CDLL(build()))
    return _lib


def _in(a, shape=None):
    """Optional input -> (contiguous float64 array or None, pointer or NULL)."""
    if a is None:
        return None, None
    arr = np.ascontiguousarray(np.asarray(a, dtype=np.float64))
    if shape is not None:
        arr = np.ascontiguousarray(np.broadcast_to(arr, shape))
    return arr, arr.ctypes.data_as(_dp)


def _out(shape):
    arr = np.zeros(shape, dtype=np.float64)
    return arr, arr.ctypes.data_as(_dp)


def silu(v: float) -> float:
    return _load().oracle_silu(float(v))


def softplus(v: float) -> float:
    return _load().oracle_softplus(float(v))


def conv1d(x, weight, bias=None, conv_state=None, silu=False):
    """x (B, D, L), weight (D, W) -> (out (B, D, L), conv_state_out (B, D, W))."""
    lib = _load()
    x_, px = _in(x)
    B, D, L = x_.shape
    w_, pw = _in(weight)
    W = w_.shape[1]
    _, pb = _in(bias, (D,)) if bias is not None else (None, None)
    _, pcs = _in(conv_state, (B, D, W)) if conv_state is not None else (None, None)
    out, po = _out((B, D, L))
    cso, pcso = _out((B, D, W))
    rc = lib.oracle_conv1d(B, D, L, W, px, pw, pb, pcs, int(bool(silu)), po, pcso)
    if rc != 0:
        raise ValueError("oracle_conv1d rejected its arguments")
    return out, cso


def scan(x, dt, A, B, C, D=None, z=None, dt_bias=None, dt_softplus=True,
         conv_weight=None, conv_bias=None, conv_state=None, h0=None):
    """Fused prefill.  x, dt, z (Bt, Dd, L); A (Dd, N); B, C (Bt, G, N, L) or
    (Bt, N, L); D, dt_bias, conv_bias (Dd); conv_weight (Dd, W);
    conv_state (Bt, Dd, W); h0 (Bt, Dd, N).

    Returns (out, h_final, conv_state_out); conv_state_out is None without conv.
    """
    lib = _load()
    x_, px = _in(x)
    Bt, Dd, L = x_.shape
    A_, pA = _in(A)
    N = A_.shape[1]
    Bm = np.asarray(B, dtype=np.float64)
    Cm = np.asarray(C, dtype=np.float64)
    if Bm.ndim == 3:
        Bm = Bm[:, None]
    if Cm.ndim == 3:
        Cm = Cm[:, None]
    G = Bm.shape[1]
    _, pB = _in(Bm)
    _, pC = _in(Cm)
    _, pdt = _in(dt, (Bt, Dd, L))
    _, pD = _in(D, (Dd,)) if D is not None else (None, None)
    _, pz = _in(z, (Bt, Dd, L)) if z is not None else (None, None)
    _, pdb = _in(dt_bias, (Dd,)) if dt_bias is not None else (None, None)
    W = 0
    pcw = pcb = pcs = None
    if conv_weight is not None:
        cw_, pcw = _in(conv_weight)
        W = cw_.shape[1]
        _, pcb = _in(conv_bias, (Dd,)) if conv_bias is not None else (None, None)
        _, pcs = _in(conv_state, (Bt, Dd, W)) if conv_state is not None else (None, None)
    _, ph0 = _in(h0, (Bt, Dd, N)) if h0 is not None else (None, None)
    out, po = _out((Bt, Dd, L))
    hf, phf = _out((Bt, Dd, N))
    cso, pcso = (_out((Bt, Dd, W)) if conv_weight is not None else (None, None))
    rc = lib.oracle_scan(Bt, Dd, L, N, G, W, px, pdt, pA, pB, pC, pD, pz, pdb,
                         int(bool(dt_softplus)), pcw, pcb, pcs, ph0, po, phf, pcso)
    if rc != 0:
        raise ValueError("oracle_scan rejected its arguments")
    return out, hf, cso


_CACHE_CODES = {None: 0, "f64": 0, "f32": 1, "f16": 2, "bf16": 3}


def round_cache(a, dtype):
    """Values of ``a`` rounded to ``dtype`` ("f32", "f16", "bf16"; None or
    "f64" keeps them), nearest with ties to even, returned as float64."""
    out = np.array(a, dtype=np.float64, copy=True, order="C")
    rc = _load().oracle_round_cache(out.ctypes.data_as(_dp), out.size, _CACHE_CODES[dtype])
    if rc != 0:
        raise ValueError("oracle_round_cache rejected its arguments")
    return out


def ssu(state, x, dt, A, B, C, D=None, z=None, dt_bias=None, dt_softplus=True,
        conv_weight=None, conv_bias=None, conv_state=None, cache_dtype=None):
    """General single-token update.  state (Bt, H, P, N); x, z (Bt, H, P);
    dt broadcastable to (Bt, H, P); A broadcastable to (H, P, N);
    B, C (Bt, G, N); D, dt_bias broadcastable to (H, P); conv_weight (H*P, W);
    conv_bias (H*P); conv_state (Bt, H*P, W).

    Returns (out, new_state, new_conv_state or None); inputs are not modified.
    cache_dtype rounds the returned state to that dtype (see round_cache).
    """
    lib = _load()
    st = np.array(state, dtype=np.float64, copy=True, order="C")
    Bt, H, P, N = st.shape
    pst = st.ctypes.data_as(_dp)
    _, px = _in(x, (Bt, H, P))
    _, pdt = _in(dt, (Bt, H, P))
    _, pA = _in(A, (H, P, N))
    Bm = np.asarray(B, dtype=np.float64)
    Cm = np.asarray(C, dtype=np.float64)
    if Bm.ndim == 2:
        Bm = Bm[:, None]
    if Cm.ndim == 2:
        Cm = Cm[:, None]
    G = Bm.shape[1]
    _, pB = _in(Bm)
    _, pC = _in(Cm)
    _, pD = _in(D, (H, P)) if D is not None else (None, None)
    _, pz = _in(z, (Bt, H, P)) if z is not None else (None, None)
    _, pdb = _in(dt_bias, (H, P)) if dt_bias is not None else (None, None)
    W = 0
    pcw = pcb = pcs = None
    cs = None
    if conv_weight is not None:
        cw_, pcw = _in(np.asarray(conv_weight).reshape(H * P, -1))
        W = cw_.shape[1]
        _, pcb = _in(np.asarray(conv_bias).reshape(-1), (H * P,)) if conv_bias is not None else (None, None)
        cs = np.array(conv_state, dtype=np.float64, copy=True, order="C").reshape(Bt, H * P, W)
        pcs = cs.ctypes.data_as(_dp)
    out, po = _out((Bt, H, P))
    rc = lib.oracle_ssu(Bt, H, P, N, G, W, pst, px, pdt, pA, pB, pC, pD, pz, pdb,
                        int(bool(dt_softplus)), pcw, pcb, pcs, po)
    if rc != 0:
        raise ValueError("oracle_ssu rejected its arguments")
    if _CACHE_CODES[cache_dtype]:
        st = round_cache(st, cache_dtype)
    return out, st, cs


def ssu_mamba2(state, x, dt, A, B, C, D=None, z=None, dt_bias=None, dt_softplus=True,
               cache_dtype=None):
    """Mamba-2 notation.  state (Bt, H, P, N); x, z (Bt, H, P); dt (Bt, H);
    A, D, dt_bias (H); B, C (Bt, G, N).  Returns (out, new_state); cache_dtype
    rounds the returned state to that dtype (see round_cache)."""
    lib = _load()
    st = np.array(state, dtype=np.float64, copy=True, order="C")
    Bt, H, P, N = st.shape
    pst = st.ctypes.data_as(_dp)
    _, px = _in(x, (Bt, H, P))
    _, pdt = _in(dt, (Bt, H))
    _, pA = _in(A, (H,))
    Bm = np.asarray(B, dtype=np.float64)
    Cm = np.asarray(C, dtype=np.float64)
    if Bm.ndim == 2:
        Bm = Bm[:, None]
    if Cm.ndim == 2:
        Cm = Cm[:, None]
    G = Bm.shape[1]
    _, pB = _in(Bm)
    _, pC = _in(Cm)
    _, pD = _in(D, (H,)) if D is not None else (None, None)
    _, pz = _in(z, (Bt, H, P)) if z is not None else (None, None)
    _, pdb = _in(dt_bias, (H,)) if dt_bias is not None else (None, None)
    out, po = _out((Bt, H, P))
    rc = lib.oracle_ssu_mamba2(Bt, H, P, N, G, pst, px, pdt, pA, pB, pC, pD, pz, pdb,
                               int(bool(dt_softplus)), po)
    if rc != 0:
        raise ValueError("oracle_ssu_mamba2 rejected its arguments")
    if _CACHE_CODES[cache_dtype]:
        st = round_cache(st, cache_dtype)
    return out, st


def scan_mamba2(x, dt, A, B, C, D=None, z=None, dt_bias=None, dt_softplus=True, h0=None):
    """Prefill, Mamba-2 layout.  x, z (Bt, H, P, L); dt (Bt, H, L); A, D, dt_bias (H);
    B, C (Bt, G, N, L) or (Bt, N, L); h0 (Bt, H, P, N).  Returns (out, h_final)."""
    lib = _load()
    xa, px = _in(x)
    Bt, H, P, L = xa.shape
    _, pdt = _in(dt, (Bt, H, L))
    _, pA = _in(A, (H,))
    Bm = np.asarray(B, dtype=np.float64)
    Cm = np.asarray(C, dtype=np.float64)
    if Bm.ndim == 3:
        Bm = Bm[:, None]
    if Cm.ndim == 3:
        Cm = Cm[:, None]
    G, N = Bm.shape[1], Bm.shape[2]
    _, pB = _in(Bm, (Bt, G, N, L))
    _, pC = _in(Cm, (Bt, G, N, L))
    _, pD = _in(D, (H,)) if D is not None else (None, None)
    _, pz = _in(z, (Bt, H, P, L)) if z is not None else (None, None)
    _, pdb = _in(dt_bias, (H,)) if dt_bias is not None else (None, None)
    _, ph0 = _in(h0, (Bt, H, P, N)) if h0 is not None else (None, None)
    out, po = _out((Bt, H, P, L))
    hf, phf = _out((Bt, H, P, N))
    rc = lib.oracle_scan_mamba2(Bt, H, P, N, G, L, px, pdt, pA, pB, pC, pD, pz, pdb,
                                int(bool(dt_softplus)), ph0, po, phf)
    if rc != 0:
        raise ValueError("oracle_scan_mamba2 rejected its arguments")
    return out, hf


def delta_sum(dt, dt_bias=None, dt_softplus=True):
    """S (Bt, Dd): the sum over t of delta = softplus(dt + dt_bias) (dt + dt_bias
    without the softplus); dt (Bt, Dd, L), dt_bias (Dd)."""
    lib = _load()
    dt_, pdt = _in(dt)
    Bt, Dd, L = dt_.shape
    _, pdb = _in(dt_bias, (Dd,)) if dt_bias is not None else (None, None)
    out, po = _out((Bt, Dd))
    if lib.oracle_delta_sum(Bt, Dd, L, pdt, pdb, int(bool(dt_softplus)), po) != 0:
        raise ValueError("oracle_delta_sum rejected its arguments")
    return out


def carry_fold(state, A, S, h_end):
    """exp(A * S) * state + h_end: the state entering the next sequence piece,
    from the state entering this one (state), the piece's sum of delta (S) and
    its end state from a zero start (h_end).  state, h_end (Bt, Dd, N); A (Dd, N);
    S (Bt, Dd).  Returns a new array."""
    lib = _load()
    st = np.array(state, dtype=np.float64, copy=True, order="C")
    Bt, Dd, N = st.shape
    _, pA = _in(A, (Dd, N))
    _, pS = _in(S, (Bt, Dd))
    _, ph = _in(h_end, (Bt, Dd, N))
    if lib.oracle_carry_fold(Bt, Dd, N, pA, pS, ph, st.ctypes.data_as(_dp)) != 0:
        raise ValueError("oracle_carry_fold rejected its arguments")
    return st


def gated_conv1d(x, Bg, Cg, weight, bias=None, conv_state=None):
    """out = Cg * (bias + causal conv of Bg * x).  x, Bg, Cg (B, D, L); weight
    (D, W); bias (D); conv_state (B, D, W), the last W gated inputs before x.
    Returns (out (B, D, L), conv_state_out (B, D, W))."""
    lib = _load()
    x_, px = _in(x)
    B, D, L = x_.shape
    _, pB = _in(Bg, (B, D, L))
    _, pC = _in(Cg, (B, D, L))
    w_, pw = _in(weight)
    W = w_.shape[1]
    _, pb = _in(bias, (D,)) if bias is not None else (None, None)
    _, pcs = _in(conv_state, (B, D, W)) if conv_state is not None else (None, None)
    out, po = _out((B, D, L))
    cso, pcso = _out((B, D, W))
    if lib.oracle_gated_conv1d(B, D, L, W, px, pB, pC, pw, pb, pcs, po, pcso) != 0:
        raise ValueError("oracle_gated_conv1d rejected its arguments")
    return out, cso
