"""Thin ctypes binding of libssm_causal.so (declared in include/ssm_causal.h).

Argument marshalling only: torch tensors are described by (device pointer,
dtype, shape, strides) and handed to the C entry points together with the
current CUDA stream of their device.  All tensors of one call must live on
one CUDA device; the call runs with that device current.  Every step of the computation runs in the library's
CUDA kernels; there is no CPU or PyTorch fallback.  If the shared library is
missing, importing the functions raises instead of degrading silently.

The entry points keep the C names:

* :func:`ssm_causal_conv1d_fwd`
* :func:`ssm_selective_scan_fwd`
* :func:`ssm_selective_state_update`
* :func:`ssm_scan_delta_sum`, :func:`ssm_scan_carry_fold` (sequence pieces)
* :func:`ssm_gated_conv1d_fwd` (double-gated short causal conv)
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional, Sequence

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libssm_causal.so")
# the same library built with the failure-test switches (tests only)
TESTHOOKS_LIB_PATH = os.path.join(_HERE, "libssm_causal_testhooks.so")
MAX_DIMS = 5

SSM_F32, SSM_F16, SSM_BF16, SSM_I32 = 0, 1, 2, 3
SSM_FLAG_DRY_RUN = 0x1

STATUS = {
    0: "SSM_OK", 1: "SSM_ERR_NULL", 2: "SSM_ERR_SHAPE", 3: "SSM_ERR_DTYPE", 4: "SSM_ERR_STRIDE",
    5: "SSM_ERR_UNSUPPORTED", 6: "SSM_ERR_CUDA", 7: "SSM_ERR_INTERNAL", 8: "SSM_ERR_VERSION",
    9: "SSM_ERR_ALIAS", 10: "SSM_ERR_WORKSPACE",
}
KERNELS = {
    0: "none", 1: "conv1d", 2: "conv1d_generic", 3: "scan_chunked", 4: "scan_generic",
    5: "ssu_vec", 6: "ssu_generic", 7: "scan_vec", 8: "ssu_row", 9: "ssu_tma", 10: "ssu_row_tma",
    11: "scan_m2", 12: "scan_m2_generic", 13: "scan_bal", 14: "delta_sum", 15: "carry_fold",
    16: "gated_conv", 17: "gated_conv_generic", 18: "gated_conv_rows",
}


class SsmError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(msg)
        self.status = status
        self.name = STATUS.get(status, str(status))


class Tensor(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("dtype", ctypes.c_int32), ("ndim", ctypes.c_int32),
                ("shape", ctypes.c_int64 * MAX_DIMS), ("stride", ctypes.c_int64 * MAX_DIMS)]


class LaunchInfo(ctypes.Structure):
    _fields_ = [("struct_size", ctypes.c_uint32), ("kernel", ctypes.c_int32),
                ("grid", ctypes.c_int32), ("block", ctypes.c_int32),
                ("smem_bytes", ctypes.c_int32), ("rows_per_item", ctypes.c_int32),
                ("work_items", ctypes.c_int64)]

    def as_dict(self):
        return {"kernel": KERNELS.get(self.kernel, self.kernel), "grid": self.grid,
                "block": self.block, "smem_bytes": self.smem_bytes,
                "rows_per_item": self.rows_per_item, "work_items": self.work_items}


class ErrorReport(ctypes.Structure):
    _fields_ = [("struct_size", ctypes.c_uint32), ("code", ctypes.c_int32),
                ("kernel", ctypes.c_int32), ("reserved", ctypes.c_int32),
                ("first_item", ctypes.c_int64)]

    def as_dict(self):
        return {"code": self.code, "kernel": KERNELS.get(self.kernel, self.kernel) if self.code else None,
                "first_item": self.first_item}


class Conv1dArgs(ctypes.Structure):
    _fields_ = [("struct_size", ctypes.c_uint32), ("flags", ctypes.c_uint32),
                ("x", Tensor), ("weight", Tensor), ("bias", Tensor), ("conv_state", Tensor),
                ("silu", ctypes.c_int32), ("out", Tensor),
                ("info", ctypes.POINTER(LaunchInfo))]


class ScanArgs(ctypes.Structure):
    _fields_ = [("struct_size", ctypes.c_uint32), ("flags", ctypes.c_uint32),
                ("x", Tensor), ("dt", Tensor), ("A", Tensor), ("B", Tensor), ("C", Tensor),
                ("D", Tensor), ("z", Tensor), ("dt_bias", Tensor), ("dt_softplus", ctypes.c_int32),
                ("conv_weight", Tensor), ("conv_bias", Tensor), ("conv_state", Tensor),
                ("ssm_state", Tensor), ("out", Tensor), ("info", ctypes.POINTER(LaunchInfo)),
                ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_uint64)]


class SsuArgs(ctypes.Structure):
    _fields_ = [("struct_size", ctypes.c_uint32), ("flags", ctypes.c_uint32),
                ("state", Tensor), ("x", Tensor), ("dt", Tensor), ("A", Tensor), ("B", Tensor),
                ("C", Tensor), ("D", Tensor), ("z", Tensor), ("dt_bias", Tensor),
                ("dt_softplus", ctypes.c_int32), ("conv_weight", Tensor), ("conv_bias", Tensor),
                ("conv_state", Tensor), ("state_batch_indices", Tensor), ("out", Tensor),
                ("info", ctypes.POINTER(LaunchInfo))]


class DeltaSumArgs(ctypes.Structure):
    _fields_ = [("struct_size", ctypes.c_uint32), ("flags", ctypes.c_uint32),
                ("dt", Tensor), ("dt_bias", Tensor), ("dt_softplus", ctypes.c_int32), ("out", Tensor),
                ("info", ctypes.POINTER(LaunchInfo))]


class CarryFoldArgs(ctypes.Structure):
    _fields_ = [("struct_size", ctypes.c_uint32), ("flags", ctypes.c_uint32),
                ("state", Tensor), ("A", Tensor), ("delta_sum", Tensor), ("h_end", Tensor),
                ("info", ctypes.POINTER(LaunchInfo))]


class GatedConvArgs(ctypes.Structure):
    _fields_ = [("struct_size", ctypes.c_uint32), ("flags", ctypes.c_uint32),
                ("x", Tensor), ("b_gate", Tensor), ("c_gate", Tensor), ("weight", Tensor),
                ("bias", Tensor), ("conv_state", Tensor), ("out", Tensor),
                ("info", ctypes.POINTER(LaunchInfo))]


_lock = threading.Lock()
_lib = None
_override = None  # a library swapped in by using_library() (failure tests)


def library():
    """Load libssm_causal.so (raises if it has not been built)."""
    global _lib
    if _override is not None:
        return _override
    with _lock:
        if _lib is None:
            _lib = _open(LIB_PATH)
    return _lib


class using_library:
    """Route every call of this binding to another build of the library (the
    failure-test build at TESTHOOKS_LIB_PATH) for the duration of the block."""

    def __init__(self, path):
        self.path = path
        self.saved = None

    def __enter__(self):
        global _override
        self.saved = _override
        _override = _open(self.path)
        return _override

    def __exit__(self, *exc):
        global _override
        _override = self.saved


def _open(path):
    """Load one build of the library and declare its entry points."""
    if not os.path.exists(path):
        raise ImportError(
            f"{path} is missing: build it with "
            "`python -m state_space_model_causal_b200.build` (there is no fallback)")
    lib = ctypes.CDLL(path)
    for name, argt in (("ssm_causal_conv1d_fwd", Conv1dArgs),
                       ("ssm_selective_scan_fwd", ScanArgs),
                       ("ssm_selective_state_update", SsuArgs),
                       ("ssm_scan_delta_sum", DeltaSumArgs),
                       ("ssm_scan_carry_fold", CarryFoldArgs),
                       ("ssm_gated_conv1d_fwd", GatedConvArgs)):
        fn = getattr(lib, name)
        fn.restype = ctypes.c_int
        fn.argtypes = [ctypes.POINTER(argt), ctypes.c_void_p]
    lib.ssm_selective_scan_fwd_noalloc.restype = ctypes.c_int
    lib.ssm_selective_scan_fwd_noalloc.argtypes = [ctypes.POINTER(ScanArgs), ctypes.c_void_p]
    lib.ssm_selective_scan_workspace_size.restype = ctypes.c_int
    lib.ssm_selective_scan_workspace_size.argtypes = [ctypes.POINTER(ScanArgs),
                                                      ctypes.POINTER(ctypes.c_uint64)]
    lib.ssm_status_string.restype = ctypes.c_char_p
    lib.ssm_status_string.argtypes = [ctypes.c_int]
    lib.ssm_abi_version.restype = ctypes.c_int
    lib.ssm_device_error.restype = ctypes.c_int
    lib.ssm_device_error.argtypes = [ctypes.POINTER(ctypes.c_int), ctypes.c_void_p]
    lib.ssm_device_error_info.restype = ctypes.c_int
    lib.ssm_device_error_info.argtypes = [ctypes.POINTER(ErrorReport), ctypes.c_void_p]
    lib.ssm_test_clamp_wait_budget.restype = ctypes.c_longlong
    lib.ssm_test_clamp_wait_budget.argtypes = [ctypes.c_longlong]
    lib.ssm_struct_size.restype = ctypes.c_size_t
    lib.ssm_struct_size.argtypes = [ctypes.c_int]
    for which, st in enumerate((Tensor, Conv1dArgs, ScanArgs, SsuArgs, LaunchInfo, ErrorReport,
                                DeltaSumArgs, CarryFoldArgs, GatedConvArgs)):
        if lib.ssm_struct_size(which) != ctypes.sizeof(st):
            raise ImportError(f"struct layout mismatch for {st.__name__}")
    return lib


# ------------------------------------------------------------ descriptors --
def raw_tensor(ptr: int, dtype: int, shape: Sequence[int], stride: Optional[Sequence[int]] = None):
    """Descriptor from a raw pointer (used for host-side argument checks)."""
    t = Tensor()
    t.data = ptr
    t.dtype = dtype
    t.ndim = len(shape)
    if stride is None:
        stride, acc = [], 1
        for s in reversed(shape):
            stride.insert(0, acc)
            acc *= max(int(s), 1)
    for i, (s, st) in enumerate(zip(shape, stride)):
        t.shape[i] = int(s)
        t.stride[i] = int(st)
    return t


def _dtype_code(t) -> int:
    import torch
    codes = {torch.float32: SSM_F32, torch.float16: SSM_F16, torch.bfloat16: SSM_BF16,
             torch.int32: SSM_I32}
    if t.dtype not in codes:
        raise TypeError(f"unsupported dtype {t.dtype}")
    return codes[t.dtype]


def describe(t) -> Tensor:
    """torch.Tensor (CUDA) or None -> ssm_tensor."""
    if t is None:
        return Tensor()
    if not t.is_cuda:
        raise ValueError("libssm_causal takes CUDA tensors only (no CPU fallback)")
    if t.dim() == 0 or t.dim() > MAX_DIMS:
        raise ValueError(f"rank {t.dim()} is outside 1..{MAX_DIMS}")
    return raw_tensor(t.data_ptr() if t.numel() > 0 else max(t.data_ptr(), 16), _dtype_code(t),
                      tuple(t.shape), tuple(t.stride()))


def device_of(tensors):
    """The one CUDA device that every given tensor (None = absent) lives on;
    a call whose tensors span devices is refused before anything launches."""
    devs = {(t.device.type, t.device.index) for t in tensors if t is not None}
    if len(devs) != 1:
        raise ValueError(f"all tensors of a call must be on one CUDA device, got {sorted(devs)}")
    return next(t.device for t in tensors if t is not None)


def _run(fn, args, tensors, stream):
    """Call a C entry point on the device of its tensors (switching the
    current device only when it differs) and on `stream`, else on that
    device's current stream."""
    import torch
    dev = device_of(tensors)

    def go():
        if stream is not None:
            handle = stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
        else:
            handle = torch.cuda.current_stream(dev).cuda_stream
        return fn(ctypes.byref(args), handle)

    if dev.index is not None and dev.index != torch.cuda.current_device():
        with torch.cuda.device(dev):
            return go()
    return go()


def _check(status: int, what: str):
    if status != 0:
        msg = library().ssm_status_string(status).decode()
        raise SsmError(status, f"{what}: {msg}")


def _info_ptr(info: Optional[LaunchInfo]):
    if info is None:
        return None
    info.struct_size = ctypes.sizeof(LaunchInfo)
    return ctypes.pointer(info)


# ------------------------------------------------------------ entry points --
def ssm_selective_scan_fwd_noalloc(x, dt, A, B, C, D=None, z=None, dt_bias=None, dt_softplus=True,
                                   conv_weight=None, conv_bias=None, conv_state=None, ssm_state=None,
                                   out=None, stream=None, info: Optional[LaunchInfo] = None):
    """The prefill of ssm_selective_scan_fwd for callers that cannot allocate
    device memory: the scratch comes from the library's fixed device array
    (see include/ssm_causal.h).  `out` must be given: this call allocates
    nothing, not even its output."""
    if out is None:
        raise ValueError("ssm_selective_scan_fwd_noalloc allocates nothing: pass `out`")
    a = ScanArgs()
    a.struct_size = ctypes.sizeof(ScanArgs)
    (a.x, a.dt, a.A, a.B, a.C, a.D, a.z, a.dt_bias, a.conv_weight, a.conv_bias, a.conv_state,
     a.ssm_state, a.out) = map(describe, (x, dt, A, B, C, D, z, dt_bias, conv_weight, conv_bias,
                                          conv_state, ssm_state, out))
    a.dt_softplus = int(bool(dt_softplus))
    a.info = _info_ptr(info)
    _check(_run(library().ssm_selective_scan_fwd_noalloc, a,
                (x, dt, A, B, C, D, z, dt_bias, conv_weight, conv_bias, conv_state, ssm_state, out), stream),
           "ssm_selective_scan_fwd_noalloc")
    return out


def ssm_selective_scan_workspace_size(x, dt, A, B, C, D=None, z=None, dt_bias=None,
                                      dt_softplus=True, conv_weight=None, conv_bias=None,
                                      conv_state=None, ssm_state=None, out=None) -> int:
    """Bytes of workspace ssm_selective_scan_fwd can use for these arguments on
    their device (0: none)."""
    import torch
    if out is None:
        out = torch.empty_like(x)
    a = ScanArgs()
    a.struct_size = ctypes.sizeof(ScanArgs)
    (a.x, a.dt, a.A, a.B, a.C, a.D, a.z, a.dt_bias, a.conv_weight, a.conv_bias, a.conv_state,
     a.ssm_state, a.out) = map(describe, (x, dt, A, B, C, D, z, dt_bias, conv_weight, conv_bias,
                                          conv_state, ssm_state, out))
    a.dt_softplus = int(bool(dt_softplus))
    tensors = (x, dt, A, B, C, D, z, dt_bias, conv_weight, conv_bias, conv_state, ssm_state, out)
    need = ctypes.c_uint64(0)
    with _on_device(device_of(tensors)):
        _check(library().ssm_selective_scan_workspace_size(ctypes.byref(a), ctypes.byref(need)),
               "ssm_selective_scan_workspace_size")
    return need.value


def ssm_causal_conv1d_fwd(x, weight, bias=None, conv_state=None, silu=False, out=None,
                          stream=None, info: Optional[LaunchInfo] = None):
    """Causal depthwise conv1d.  x (B, D, L); weight (D, W) f32; bias (D);
    conv_state (B, D, W) in/out.  Returns out (B, D, L)."""
    import torch
    if out is None:
        out = torch.empty_like(x)
    a = Conv1dArgs()
    a.struct_size = ctypes.sizeof(Conv1dArgs)
    a.x, a.weight, a.bias, a.conv_state, a.out = map(describe, (x, weight, bias, conv_state, out))
    a.silu = int(bool(silu))
    a.info = _info_ptr(info)
    _check(_run(library().ssm_causal_conv1d_fwd, a, (x, weight, bias, conv_state, out), stream),
           "ssm_causal_conv1d_fwd")
    return out


def ssm_selective_scan_fwd(x, dt, A, B, C, D=None, z=None, dt_bias=None, dt_softplus=True,
                           conv_weight=None, conv_bias=None, conv_state=None, ssm_state=None,
                           out=None, stream=None, info: Optional[LaunchInfo] = None,
                           workspace="auto"):
    """Fused prefill (see include/ssm_causal.h).  Returns out (B, D, L).

    workspace: "auto" (default) passes a cached zero-initialised workspace of
    the size the library asks for (one per device and stream); None passes no
    workspace (the prefill then runs without hand-overs); a uint8 CUDA tensor
    is passed as given."""
    import torch
    if out is None:
        out = torch.empty_like(x)
    a = ScanArgs()
    a.struct_size = ctypes.sizeof(ScanArgs)
    (a.x, a.dt, a.A, a.B, a.C, a.D, a.z, a.dt_bias, a.conv_weight, a.conv_bias, a.conv_state,
     a.ssm_state, a.out) = map(describe, (x, dt, A, B, C, D, z, dt_bias, conv_weight, conv_bias,
                                          conv_state, ssm_state, out))
    a.dt_softplus = int(bool(dt_softplus))
    a.info = _info_ptr(info)
    tensors = (x, dt, A, B, C, D, z, dt_bias, conv_weight, conv_bias, conv_state, ssm_state, out)
    dev = device_of(tensors)
    with _on_device(dev):
        if isinstance(workspace, str):
            if workspace != "auto":
                raise ValueError(f"workspace must be 'auto', None or a tensor, not {workspace!r}")
            need = ctypes.c_uint64(0)
            _check(library().ssm_selective_scan_workspace_size(ctypes.byref(a), ctypes.byref(need)),
                   "ssm_selective_scan_workspace_size")
            if need.value:
                ws = _workspace(dev, stream, need.value)
                a.workspace, a.workspace_bytes = ws.data_ptr(), ws.numel() * ws.element_size()
        elif workspace is not None:
            a.workspace, a.workspace_bytes = workspace.data_ptr(), workspace.numel() * workspace.element_size()
        _check(_run(library().ssm_selective_scan_fwd, a, tensors, stream), "ssm_selective_scan_fwd")
    return out


# Prefill workspaces: one per (device, stream), zero-filled when allocated and
# grown by reallocation; the library keeps it consistent from call to call.
_ws_lock = threading.Lock()
_workspaces = {}


def _stream_handle(dev, stream):
    import torch
    if stream is not None:
        return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
    return torch.cuda.current_stream(dev).cuda_stream


def _workspace(dev, stream, nbytes):
    """The zero-initialised workspace of (dev, stream), at least nbytes long
    (256-byte aligned: torch's allocator aligns blocks to 512 bytes)."""
    import torch
    handle = _stream_handle(dev, stream)
    key = (dev.index, handle)
    with _ws_lock:
        ws = _workspaces.get(key)
        if ws is None or ws.numel() < nbytes:
            # allocated and zero-filled on the stream the prefill runs on, so
            # the fill is ordered before the kernel; a replaced buffer is
            # recycled by the caching allocator only after that stream's
            # queued work
            ext = torch.cuda.ExternalStream(handle, device=dev)
            with torch.cuda.stream(ext):
                ws = torch.zeros(nbytes, dtype=torch.uint8, device=dev)
            _workspaces[key] = ws
        return ws


class _on_device:
    """Make `dev` current for the block (no-op when it already is)."""

    def __init__(self, dev):
        self.dev = dev
        self.ctx = None

    def __enter__(self):
        import torch
        if self.dev.index is not None and self.dev.index != torch.cuda.current_device():
            self.ctx = torch.cuda.device(self.dev)
            self.ctx.__enter__()
        return self

    def __exit__(self, *exc):
        if self.ctx is not None:
            self.ctx.__exit__(*exc)


def ssm_selective_state_update(state, x, dt, A, B, C, D=None, z=None, dt_bias=None,
                               dt_softplus=True, conv_weight=None, conv_bias=None,
                               conv_state=None, state_batch_indices=None, out=None, stream=None,
                               info: Optional[LaunchInfo] = None):
    """One decode step; state (and conv_state) updated in place.  Returns out."""
    import torch
    if out is None:
        out = torch.empty_like(x)
    a = SsuArgs()
    a.struct_size = ctypes.sizeof(SsuArgs)
    (a.state, a.x, a.dt, a.A, a.B, a.C, a.D, a.z, a.dt_bias, a.conv_weight, a.conv_bias,
     a.conv_state, a.state_batch_indices, a.out) = map(
        describe, (state, x, dt, A, B, C, D, z, dt_bias, conv_weight, conv_bias, conv_state,
                   state_batch_indices, out))
    a.dt_softplus = int(bool(dt_softplus))
    a.info = _info_ptr(info)
    _check(_run(library().ssm_selective_state_update, a,
                (state, x, dt, A, B, C, D, z, dt_bias, conv_weight, conv_bias, conv_state,
                 state_batch_indices, out), stream),
           "ssm_selective_state_update")
    return out


def ssm_scan_delta_sum(dt, dt_bias=None, dt_softplus=True, out=None, stream=None,
                       info: Optional[LaunchInfo] = None):
    """Sum over t of a sequence piece's delta (see include/ssm_causal.h):
    dt (B, D, L) -> (B, D) float32."""
    import torch
    if out is None:
        out = torch.empty(dt.shape[0], dt.shape[1], dtype=torch.float32, device=dt.device)
    a = DeltaSumArgs()
    a.struct_size = ctypes.sizeof(DeltaSumArgs)
    a.dt, a.dt_bias, a.out = map(describe, (dt, dt_bias, out))
    a.dt_softplus = int(bool(dt_softplus))
    a.info = _info_ptr(info)
    _check(_run(library().ssm_scan_delta_sum, a, (dt, dt_bias, out), stream), "ssm_scan_delta_sum")
    return out


def ssm_scan_carry_fold(state, A, delta_sum, h_end, stream=None, info: Optional[LaunchInfo] = None):
    """state <- exp(A * delta_sum) * state + h_end in place: the state entering
    the next sequence piece (see include/ssm_causal.h).  Returns state."""
    a = CarryFoldArgs()
    a.struct_size = ctypes.sizeof(CarryFoldArgs)
    a.state, a.A, a.delta_sum, a.h_end = map(describe, (state, A, delta_sum, h_end))
    a.info = _info_ptr(info)
    _check(_run(library().ssm_scan_carry_fold, a, (state, A, delta_sum, h_end), stream),
           "ssm_scan_carry_fold")
    return state


def ssm_gated_conv1d_fwd(x, b_gate, c_gate, weight, bias=None, conv_state=None, out=None,
                         stream=None, info: Optional[LaunchInfo] = None):
    """Double-gated short causal conv: out = c_gate * (bias + causal conv of
    b_gate * x) (see include/ssm_causal.h).  x, b_gate, c_gate (B, D, L);
    weight (D, W) f32; bias (D); conv_state (B, D, W) in/out, the last W gated
    inputs.  Without ``out``, the output takes x's layout: channels contiguous
    (B, L, D storage) when x has unit channel stride, else (B, D, L).  Returns out."""
    import torch
    if out is None:
        if x.dim() == 3 and x.stride(1) == 1 and x.shape[1] > 1:
            out = torch.empty((x.shape[0], x.shape[2], x.shape[1]), dtype=x.dtype,
                              device=x.device).transpose(1, 2)
        else:
            out = torch.empty(x.shape, dtype=x.dtype, device=x.device)
    a = GatedConvArgs()
    a.struct_size = ctypes.sizeof(GatedConvArgs)
    a.x, a.b_gate, a.c_gate, a.weight, a.bias, a.conv_state, a.out = map(
        describe, (x, b_gate, c_gate, weight, bias, conv_state, out))
    a.info = _info_ptr(info)
    _check(_run(library().ssm_gated_conv1d_fwd, a, (x, b_gate, c_gate, weight, bias, conv_state, out), stream),
           "ssm_gated_conv1d_fwd")
    return out


def ssm_device_error(stream=None) -> int:
    """Wait for the current stream and return (and clear) the library's device
    error word: 0 = none, 1 = a kernel gave up a bounded wait and exited early."""
    import torch
    code = ctypes.c_int(0)
    st = stream.cuda_stream if stream is not None else torch.cuda.current_stream().cuda_stream
    _check(library().ssm_device_error(ctypes.byref(code), st), "ssm_device_error")
    return code.value


def ssm_device_error_info(stream=None) -> dict:
    """Wait for the stream, then read and clear the library's device error
    record: {"code": 0 | 1, "kernel": name of the reporting kernel or None,
    "first_item": lowest unfinished work item or -1} (see
    include/ssm_causal.h, ssm_device_error_info)."""
    import torch
    rep = ErrorReport()
    rep.struct_size = ctypes.sizeof(ErrorReport)
    st = stream.cuda_stream if stream is not None else torch.cuda.current_stream().cuda_stream
    _check(library().ssm_device_error_info(ctypes.byref(rep), st), "ssm_device_error_info")
    return rep.as_dict()
