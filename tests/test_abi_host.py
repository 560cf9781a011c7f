"""Host-side checks of the C ABI (no GPU needed, nothing is launched).

The library must load, export every function that include/ssm_causal.h
declares, agree with the binding on struct layouts, and reject every invalid
argument with its documented status before any CUDA call.  Valid calls are
made in dry-run mode (SSM_FLAG_DRY_RUN), which checks and plans but launches
nothing, so the chosen kernel and launch shape can be inspected on the CPU.
"""
import ctypes
import os
import re

import pytest

from state_space_model_causal_b200 import binding as bd

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ssm_causal.h")

F32, F16, BF16, I32 = bd.SSM_F32, bd.SSM_F16, bd.SSM_BF16, bd.SSM_I32
OK, ENULL, ESHAPE, EDTYPE, ESTRIDE, EUNSUP, ECUDA, EINT, EVER, EALIAS, EWORKSPACE = range(11)


@pytest.fixture(scope="module")
def lib():
    return bd.library()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*[A-Za-z_][\w\s\*]*?\b(ssm_\w+)\s*\(", src, flags=re.M)))


def test_header_declares_the_three_entry_points():
    fns = declared_functions()
    for name in ("ssm_causal_conv1d_fwd", "ssm_selective_scan_fwd", "ssm_selective_state_update",
                 "ssm_scan_delta_sum", "ssm_scan_carry_fold", "ssm_gated_conv1d_fwd",
                 "ssm_status_string", "ssm_abi_version", "ssm_struct_size"):
        assert name in fns


def test_library_exports_every_declared_symbol(lib):
    missing = [f for f in declared_functions() if not hasattr(lib, f)]
    assert not missing, f"declared but not exported: {missing}"


def test_abi_version_and_struct_layouts(lib):
    assert lib.ssm_abi_version() == 4
    for which, st in enumerate((bd.Tensor, bd.Conv1dArgs, bd.ScanArgs, bd.SsuArgs, bd.LaunchInfo,
                                bd.ErrorReport, bd.DeltaSumArgs, bd.CarryFoldArgs, bd.GatedConvArgs)):
        assert lib.ssm_struct_size(which) == ctypes.sizeof(st)
    assert lib.ssm_struct_size(99) == 0


def test_failure_test_wait_budget_has_a_floor(lib):
    """A failure test may shorten the bounded waits, never below 10^7 cycles
    (~5 ms), so a wait for copies still in flight cannot be cut short; the
    clean-up wait after a give-up always uses the full budget."""
    assert lib.ssm_test_clamp_wait_budget(1) == 10_000_000
    assert lib.ssm_test_clamp_wait_budget(0) == 10_000_000
    assert lib.ssm_test_clamp_wait_budget(20_000_000) == 20_000_000
    test_lib = bd._open(bd.TESTHOOKS_LIB_PATH)
    assert test_lib.ssm_test_clamp_wait_budget(5) == 10_000_000


def test_error_report_checks_its_arguments(lib):
    assert lib.ssm_device_error_info(None, None) == ENULL
    rep = bd.ErrorReport()
    rep.struct_size = 3
    assert lib.ssm_device_error_info(ctypes.byref(rep), None) == EVER


def test_status_strings(lib):
    for code, name in bd.STATUS.items():
        assert lib.ssm_status_string(code).decode().startswith(name)
    assert lib.ssm_status_string(1234).decode() == "unknown ssm_status"


# ---------------------------------------------------------------- helpers --
class FakeMem:
    """Hands out distinct, 256-byte-aligned fake device addresses far apart."""

    def __init__(self):
        self.next = 1 << 40

    def __call__(self, dtype, shape, stride=None):
        ptr = self.next
        self.next += 1 << 36
        return bd.raw_tensor(ptr, dtype, shape, stride)


def scan_args(mem, Bn=4, D=5120, L=2048, N=16, G=None, W=4, io=F16, **over):
    a = bd.ScanArgs()
    a.struct_size = ctypes.sizeof(bd.ScanArgs)
    a.flags = bd.SSM_FLAG_DRY_RUN
    a.x = mem(io, (Bn, D, L))
    a.dt = mem(io, (Bn, D, L))
    a.A = mem(F32, (D, N))
    bshape = (Bn, N, L) if G is None else (Bn, G, N, L)
    a.B = mem(io, bshape)
    a.C = mem(io, bshape)
    a.D = mem(F32, (D,))
    a.z = mem(io, (Bn, D, L))
    a.dt_bias = mem(F32, (D,))
    a.dt_softplus = 1
    if W:
        a.conv_weight = mem(F32, (D, W))
        a.conv_bias = mem(F32, (D,))
        a.conv_state = mem(F32, (Bn, D, W))
    a.ssm_state = mem(F32, (Bn, D, N))
    a.out = mem(io, (Bn, D, L))
    for k, v in over.items():
        setattr(a, k, v)
    return a


def ssu_m1_args(mem, Bn=245, D=5120, N=16, W=4, io=F16, st=F32, **over):
    a = bd.SsuArgs()
    a.struct_size = ctypes.sizeof(bd.SsuArgs)
    a.flags = bd.SSM_FLAG_DRY_RUN
    a.state = mem(st, (Bn, D, N))
    a.x = mem(io, (Bn, D))
    a.dt = mem(io, (Bn, D))
    a.A = mem(F32, (D, N))
    a.B = mem(io, (Bn, 1, N))
    a.C = mem(io, (Bn, 1, N))
    a.D = mem(F32, (D,))
    a.z = mem(io, (Bn, D))
    a.dt_bias = mem(F32, (D,))
    a.dt_softplus = 1
    if W:
        a.conv_weight = mem(F32, (D, W))
        a.conv_bias = mem(F32, (D,))
        a.conv_state = mem(F32, (Bn, D, W))
    a.out = mem(io, (Bn, D))
    for k, v in over.items():
        setattr(a, k, v)
    return a


def ssu_m2_args(mem, Bn=8, H=80, P=64, N=128, G=1, io=F16, st=F16, **over):
    a = bd.SsuArgs()
    a.struct_size = ctypes.sizeof(bd.SsuArgs)
    a.flags = bd.SSM_FLAG_DRY_RUN
    a.state = mem(st, (Bn, H, P, N))
    a.x = mem(io, (Bn, H, P))
    a.dt = mem(io, (Bn, H))
    a.A = mem(F32, (H,))
    a.B = mem(io, (Bn, G, N))
    a.C = mem(io, (Bn, G, N))
    a.D = mem(F32, (H,))
    a.dt_bias = mem(F32, (H,))
    a.dt_softplus = 1
    a.out = mem(io, (Bn, H, P))
    for k, v in over.items():
        setattr(a, k, v)
    return a


def conv_args(mem, Bn=2, D=64, L=100, W=4, io=F16, **over):
    a = bd.Conv1dArgs()
    a.struct_size = ctypes.sizeof(bd.Conv1dArgs)
    a.flags = bd.SSM_FLAG_DRY_RUN
    a.x = mem(io, (Bn, D, L))
    a.weight = mem(F32, (D, W))
    a.bias = mem(F32, (D,))
    a.conv_state = mem(F32, (Bn, D, W))
    a.silu = 1
    a.out = mem(io, (Bn, D, L))
    for k, v in over.items():
        setattr(a, k, v)
    return a


def call(lib, fn, args):
    info = bd.LaunchInfo()
    info.struct_size = ctypes.sizeof(bd.LaunchInfo)
    args.info = ctypes.pointer(info)
    st = getattr(lib, fn)(ctypes.byref(args), None)
    return st, info


# ------------------------------------------------------------- valid plans --
def test_prefill_2p8b_plan(lib):
    """Without a workspace every warp takes whole (batch, 16-channel) units:
    1280 units, 4 warps per CTA."""
    st, info = call(lib, "ssm_selective_scan_fwd", scan_args(FakeMem()))
    assert st == OK
    assert bd.KERNELS[info.kernel] == "scan_bal"
    assert info.block == 128 and info.rows_per_item == 16
    assert info.work_items == 4 * 5120 // 16
    assert info.grid == 4 * 5120 // 16 // 4


def ws_bytes(workers):
    """256-byte header, one 32-bit flag per worker rounded up to 256 bytes,
    one 1088-byte hand-over slot (16 x 16 state, 16 sums of delta) per worker."""
    return 256 + (workers * 4 + 255) // 256 * 256 + workers * 1088


def test_prefill_workspace_size_and_balanced_plan(lib):
    """1280 units > 148 SMs x 2 CTAs x 4 warps = 1184 resident warps: the
    dry-run plan asks for the hand-over workspace and, given one, runs
    exactly one persistent wave of 296 CTAs."""
    mem = FakeMem()
    a = scan_args(mem)
    need = ctypes.c_uint64(0)
    assert lib.ssm_selective_scan_workspace_size(ctypes.byref(a), ctypes.byref(need)) == OK
    assert need.value == ws_bytes(1184)
    a.workspace, a.workspace_bytes = mem.next, need.value
    mem.next += 1 << 36
    st, info = call(lib, "ssm_selective_scan_fwd", a)
    assert st == OK and bd.KERNELS[info.kernel] == "scan_bal"
    assert info.grid == 148 * 2 and info.work_items == 1280
    assert lib.ssm_selective_scan_workspace_size(ctypes.byref(a), None) == ENULL


def test_prefill_context_parallel_plan(lib):
    """B=1: 320 units fill under 60% of the 1184 resident warps, so the
    sequence is cut into 5 pieces of 13 chunks (the last one 12): each of the
    two passes runs 4 pieces per unit, 1280 piece-units (more than the
    warps, so the passes hand over too).  The workspace adds one record
    (16 x 16 state + 16 sums of delta) per unit and piece 0..3."""
    mem = FakeMem()
    a = scan_args(mem, Bn=1, D=5120)
    need = ctypes.c_uint64(123)
    assert lib.ssm_selective_scan_workspace_size(ctypes.byref(a), ctypes.byref(need)) == OK
    assert need.value == ws_bytes(1184) + 320 * 4 * 1088
    a.workspace, a.workspace_bytes = mem.next, need.value
    mem.next += 1 << 36
    st, info = call(lib, "ssm_selective_scan_fwd", a)
    assert st == OK and bd.KERNELS[info.kernel] == "scan_bal"
    assert info.work_items == 1280 and info.grid == 296


def test_prefill_context_parallel_plan_short_batch(lib):
    """B=1, D=64, L=512 (4 units of 16 channels, 16 chunks): as many pieces as
    leave at least two chunks each with the last piece shorter -- 8 pieces of
    2 chunks, 7 per pass -- so 28 piece-units per pass, no hand-overs between
    warps (28 < 1184), and one record per unit and piece 0..6."""
    mem = FakeMem()
    a = scan_args(mem, Bn=1, D=64, L=512)
    need = ctypes.c_uint64(123)
    assert lib.ssm_selective_scan_workspace_size(ctypes.byref(a), ctypes.byref(need)) == OK
    assert need.value == ws_bytes(1184) + 4 * 7 * 1088
    a.workspace, a.workspace_bytes = mem.next, need.value
    mem.next += 1 << 36
    st, info = call(lib, "ssm_selective_scan_fwd", a)
    assert st == OK and bd.KERNELS[info.kernel] == "scan_bal"
    assert info.work_items == 28


def test_prefill_small_problem_needs_no_workspace(lib):
    mem = FakeMem()
    need = ctypes.c_uint64(123)
    a = scan_args(mem, Bn=2, D=64, L=100)  # chunked kernel
    assert lib.ssm_selective_scan_workspace_size(ctypes.byref(a), ctypes.byref(need)) == OK
    assert need.value == 0


def test_prefill_workspace_errors(lib):
    mem = FakeMem()
    need = ws_bytes(1184)
    a = scan_args(mem)
    a.workspace, a.workspace_bytes = mem.next, need - 1
    mem.next += 1 << 36
    assert call(lib, "ssm_selective_scan_fwd", a)[0] == EWORKSPACE   # too small
    a.workspace, a.workspace_bytes = mem.next + 16, need
    assert call(lib, "ssm_selective_scan_fwd", a)[0] == EWORKSPACE   # not 256-byte aligned
    a.workspace, a.workspace_bytes = a.out.data, need
    assert call(lib, "ssm_selective_scan_fwd", a)[0] == EALIAS       # overlaps the output
    a.workspace, a.workspace_bytes = a.A.data - 256, need
    assert call(lib, "ssm_selective_scan_fwd", a)[0] == EALIAS       # overlaps A


def test_unaligned_or_odd_prefill_layouts_use_the_chunked_kernel(lib):
    mem = FakeMem()
    st, info = call(lib, "ssm_selective_scan_fwd", scan_args(mem, Bn=2, D=64, L=100))
    assert st == OK and bd.KERNELS[info.kernel] == "scan_chunked"  # L % 8 != 0
    st, info = call(lib, "ssm_selective_scan_fwd", scan_args(mem, Bn=2, D=64, L=64, N=32))
    assert st == OK and bd.KERNELS[info.kernel] == "scan_chunked"  # d_state > 16
    st, info = call(lib, "ssm_selective_scan_fwd", scan_args(mem, Bn=2, D=64, L=64, W=3))
    assert st == OK and bd.KERNELS[info.kernel] == "scan_chunked"  # conv width 3
    a = scan_args(mem, Bn=2, D=64, L=64)
    a.x.data += 2                                                  # 2-byte aligned rows
    st, info = call(lib, "ssm_selective_scan_fwd", a)
    assert st == OK and bd.KERNELS[info.kernel] == "scan_chunked"


def test_small_scan_plan_and_generic_for_large_state(lib):
    mem = FakeMem()
    st, info = call(lib, "ssm_selective_scan_fwd", scan_args(mem, Bn=1, D=64, L=128, W=0, io=F32))
    assert st == OK and bd.KERNELS[info.kernel] == "scan_bal"
    st, info = call(lib, "ssm_selective_scan_fwd", scan_args(mem, Bn=1, D=8, L=16, N=128, W=0))
    assert st == OK and bd.KERNELS[info.kernel] == "scan_generic"


def test_scan_groups_choose_generic_when_tile_straddles_groups(lib):
    mem = FakeMem()
    st, info = call(lib, "ssm_selective_scan_fwd", scan_args(mem, Bn=1, D=64, L=8, G=4))
    assert st == OK and bd.KERNELS[info.kernel] == "scan_bal"  # 16 channels per group
    st, info = call(lib, "ssm_selective_scan_fwd", scan_args(mem, Bn=1, D=24, L=8, G=3))
    assert st == OK and bd.KERNELS[info.kernel] == "scan_generic"  # 8 channels per group


def test_decode_2p8b_plan(lib):
    st, info = call(lib, "ssm_selective_state_update", ssu_m1_args(FakeMem()))
    assert st == OK and bd.KERNELS[info.kernel] == "ssu_row_tma"
    # one bulk-copy pipeline per warp, 32 channels (one per lane) per work item
    assert info.block == 128 and info.rows_per_item == 32
    assert 0 < info.grid <= 148 * 5 and info.work_items == 245 * (5120 // 32)
    assert 0 < info.smem_bytes <= 48 * 1024 and info.smem_bytes % 128 == 0
    # a channel count that is not a multiple of 8 takes the register-streaming row kernel
    st, info = call(lib, "ssm_selective_state_update", ssu_m1_args(FakeMem(), D=100))
    assert st == OK and bd.KERNELS[info.kernel] == "ssu_row"


@pytest.mark.parametrize("P,N,st_dt,io", [(64, 128, F16, F16), (64, 128, F32, F16),
                                          (128, 256, BF16, BF16), (128, 256, F32, BF16)])
@pytest.mark.parametrize("R", [8, 128, 4096, 131072])
def test_mamba2_plans_use_bulk_copy_kernel(lib, P, N, st_dt, io, R):
    H = 80 if N == 128 else 32
    Bn, Hr = (-(-R // H), H) if R >= H else (1, R)
    st, info = call(lib, "ssm_selective_state_update",
                    ssu_m2_args(FakeMem(), Bn=Bn, H=Hr, P=P, N=N, io=io, st=st_dt))
    assert st == OK and bd.KERNELS[info.kernel] == "ssu_tma"
    assert 0 < info.grid <= 148 * 3
    assert 0 < info.smem_bytes <= 76 * 1024 and info.smem_bytes % 128 == 0
    assert info.work_items * info.rows_per_item >= Bn * Hr * P


def test_mamba2_groups_items_do_not_straddle_groups(lib):
    st, info = call(lib, "ssm_selective_state_update", ssu_m2_args(FakeMem(), Bn=3, H=12, P=8, N=128, G=4))
    assert st == OK and bd.KERNELS[info.kernel] == "ssu_tma"
    # headdim 6: an item's fp16 x values cannot start 16-byte aligned -> streaming kernel
    st, info = call(lib, "ssm_selective_state_update", ssu_m2_args(FakeMem(), Bn=3, H=12, P=6, N=128, G=4))
    assert st == OK and bd.KERNELS[info.kernel] == "ssu_vec"
    # rows that are not dense (row stride > row size) take the register-streaming kernel
    m = FakeMem()
    a = ssu_m2_args(m, Bn=3, H=12, P=6, N=128, G=4)
    a.state = m(F16, (3, 12, 6, 128), (12 * 6 * 256, 6 * 256, 256, 1))
    st, info = call(lib, "ssm_selective_state_update", a)
    assert st == OK and bd.KERNELS[info.kernel] == "ssu_vec"
    # full A per element takes the per-row kernel; its items must not straddle a group
    m = FakeMem()
    a = ssu_m2_args(m, Bn=3, H=12, P=6, N=16, G=4, st=F32)
    a.A = m(F32, (12, 6, 16))
    st, info = call(lib, "ssm_selective_state_update", a)
    assert st == OK and bd.KERNELS[info.kernel] == "ssu_row"
    assert (12 // 4 * 6) % info.rows_per_item == 0


def test_ssu_generic_for_unaligned_rows(lib):
    mem = FakeMem()
    st, info = call(lib, "ssm_selective_state_update", ssu_m2_args(mem, N=3, st=F32))
    assert st == OK and bd.KERNELS[info.kernel] == "ssu_generic"
    # dstate not contiguous
    a = ssu_m2_args(mem, Bn=2, H=4, P=8, N=16, st=F32)
    a.state = mem(F32, (2, 4, 8, 16), (4 * 8 * 16 * 2, 8 * 16 * 2, 16 * 2, 2))
    st, info = call(lib, "ssm_selective_state_update", a)
    assert st == OK and bd.KERNELS[info.kernel] == "ssu_generic"


def test_empty_problems_launch_nothing(lib):
    mem = FakeMem()
    st, info = call(lib, "ssm_selective_scan_fwd", scan_args(mem, Bn=2, D=16, L=0))
    assert st == OK and info.kernel == 0 and info.grid == 0
    st, info = call(lib, "ssm_selective_state_update", ssu_m2_args(mem, Bn=0))
    assert st == OK and info.kernel == 0
    st, info = call(lib, "ssm_causal_conv1d_fwd", conv_args(mem, L=0))
    assert st == OK and info.kernel == 0


def test_conv_plan(lib):
    """L a multiple of the vector width: the 16-byte vector kernel, units of
    U 256-step blocks (fp16) of a row -- U = 8 for fp16 and fp32 up to W = 4,
    else 4 -- on persistent CTAs of 8 warps (at most 3 per SM of the dry-run
    B200); otherwise (or W - 1 above the vector width, or unit time stride
    missing) the warp-per-row kernel."""
    st, info = call(lib, "ssm_causal_conv1d_fwd", conv_args(FakeMem()))
    assert st == OK and bd.KERNELS[info.kernel] == "conv1d_generic" and info.grid == 2 * 64 // 4
    # 128 rows of 8 blocks, fp16, W = 4: one unit of 8 blocks per row
    st, info = call(lib, "ssm_causal_conv1d_fwd", conv_args(FakeMem(), L=2048))
    assert st == OK and bd.KERNELS[info.kernel] == "conv1d" and info.block == 256
    assert info.grid == 2 * 64 // 8 and info.work_items == 2 * 64
    # bf16: units of 4 blocks, two per row
    st, info = call(lib, "ssm_causal_conv1d_fwd", conv_args(FakeMem(), L=2048, io=BF16))
    assert st == OK and bd.KERNELS[info.kernel] == "conv1d" and info.work_items == 2 * 64 * 2
    # fp16, W = 5: units of 4 blocks
    st, info = call(lib, "ssm_causal_conv1d_fwd", conv_args(FakeMem(), L=2048, W=5))
    assert st == OK and bd.KERNELS[info.kernel] == "conv1d" and info.work_items == 2 * 64 * 2
    # many units: the grid stops at 148 SMs x 3 CTAs
    st, info = call(lib, "ssm_causal_conv1d_fwd", conv_args(FakeMem(), Bn=4, D=5120, L=2048))
    assert st == OK and bd.KERNELS[info.kernel] == "conv1d" and info.grid == 148 * 3
    assert info.work_items == 4 * 5120
    # a ragged last block: ceil(264 / 256) = 2 blocks, one unit per row
    st, info = call(lib, "ssm_causal_conv1d_fwd", conv_args(FakeMem(), Bn=1, D=3, L=264))
    assert st == OK and bd.KERNELS[info.kernel] == "conv1d" and info.work_items == 3 and info.grid == 1
    # fp32: 4 steps per vector, so W = 6 needs the generic kernel; W = 5 does not
    st, info = call(lib, "ssm_causal_conv1d_fwd", conv_args(FakeMem(), L=64, W=6, io=F32))
    assert st == OK and bd.KERNELS[info.kernel] == "conv1d_generic"
    st, info = call(lib, "ssm_causal_conv1d_fwd", conv_args(FakeMem(), L=64, W=5, io=F32))
    assert st == OK and bd.KERNELS[info.kernel] == "conv1d"


def test_conv_plan_matches_its_rules_on_random_shapes(lib):
    """The planner's choice, unroll, unit count and grid for 300 random
    contiguous shapes, against the rules stated plainly: the vector kernel
    when L is a multiple of V and W - 1 <= V; U = 8 for fp16 and fp32 up to
    W = 4, else 4; units = rows x ceil(ceil(L / 32V) / U); grid =
    min(ceil(units / 8), 148 x 3)."""
    import numpy as np
    rng = np.random.default_rng(11)
    for _ in range(300):
        io = [F32, F16, BF16][rng.integers(3)]
        Bn, D = int(rng.integers(1, 5)), int(rng.integers(1, 300))
        L, W = int(rng.integers(1, 5000)), int(rng.integers(1, 9))
        st, info = call(lib, "ssm_causal_conv1d_fwd", conv_args(FakeMem(), Bn=Bn, D=D, L=L, W=W, io=io))
        assert st == OK
        V = 4 if io == F32 else 8
        rows = Bn * D
        if L % V or W - 1 > V:
            assert bd.KERNELS[info.kernel] == "conv1d_generic", (io, Bn, D, L, W)
            continue
        U = 8 if io in (F32, F16) and W <= 4 else 4
        units = rows * (-(-(-(-L // (32 * V))) // U))
        assert bd.KERNELS[info.kernel] == "conv1d", (io, Bn, D, L, W)
        assert info.work_items == units and info.grid == min(-(-units // 8), 148 * 3), (io, Bn, D, L, W)


# ------------------------------------------------------------ error paths --
def test_null_args_and_version(lib):
    for fn in ("ssm_causal_conv1d_fwd", "ssm_selective_scan_fwd", "ssm_selective_state_update"):
        assert getattr(lib, fn)(None, None) == ENULL
    a = scan_args(FakeMem())
    a.struct_size -= 8
    assert lib.ssm_selective_scan_fwd(ctypes.byref(a), None) == EVER
    a = scan_args(FakeMem())
    info = bd.LaunchInfo()
    info.struct_size = 3
    a.info = ctypes.pointer(info)
    assert lib.ssm_selective_scan_fwd(ctypes.byref(a), None) == EVER


def _expect(lib, fn, args, status):
    st, _ = call(lib, fn, args)
    assert st == status, f"{fn}: expected {bd.STATUS[status]}, got {bd.STATUS.get(st, st)}"


def test_scan_error_paths(lib):
    fn = "ssm_selective_scan_fwd"
    m = FakeMem()
    _expect(lib, fn, scan_args(m, x=bd.Tensor()), ENULL)                       # missing x
    _expect(lib, fn, scan_args(m, dt=m(F16, (4, 5120, 2047))), ESHAPE)         # dt length
    _expect(lib, fn, scan_args(m, A=m(F16, (5120, 16))), EDTYPE)               # A not f32
    _expect(lib, fn, scan_args(m, dt=m(F32, (4, 5120, 2048))), EDTYPE)         # mixed io
    _expect(lib, fn, scan_args(m, x=m(F16, (4, 5120, 2048), (5120 * 2048, 2048, -1))), ESTRIDE)
    _expect(lib, fn, scan_args(m, out=m(F16, (4, 5120, 2048), (5120 * 2048, 2048, 0))), ESTRIDE)
    _expect(lib, fn, scan_args(m, Bn=1, D=10, L=4, G=3), ESHAPE)               # G does not divide D
    _expect(lib, fn, scan_args(m, Bn=1, D=8, L=4, N=300), EUNSUP)              # N > 256
    _expect(lib, fn, scan_args(m, Bn=1, D=8, L=4, W=9), EUNSUP)                # W > 8
    a = scan_args(m, Bn=1, D=8, L=4, W=0)
    a.conv_state = m(F32, (1, 8, 4))
    _expect(lib, fn, a, ENULL)                                                 # state without weight
    a = scan_args(m, Bn=1, D=8, L=4)
    a.out = a.x                                                                # in-place out
    _expect(lib, fn, a, EALIAS)
    a = scan_args(m, Bn=1, D=8, L=4)
    a.ssm_state = a.conv_state
    _expect(lib, fn, a, ESHAPE)
    a = scan_args(m, Bn=1, D=8, L=4)
    a.x.data += 1                                                              # misaligned element
    _expect(lib, fn, a, ESTRIDE)
    a = scan_args(m, Bn=1, D=8, L=4)
    a.x.dtype = 7
    _expect(lib, fn, a, EDTYPE)
    a = scan_args(m, Bn=1, D=8, L=4)
    a.x.ndim = 0
    _expect(lib, fn, a, ESHAPE)


def test_ssu_error_paths(lib):
    fn = "ssm_selective_state_update"
    m = FakeMem()
    _expect(lib, fn, ssu_m2_args(m, state=bd.Tensor()), ENULL)
    _expect(lib, fn, ssu_m2_args(m, x=m(F16, (8, 80, 63))), ESHAPE)
    _expect(lib, fn, ssu_m2_args(m, A=m(F16, (80,))), EDTYPE)
    _expect(lib, fn, ssu_m2_args(m, H=80, G=3), ESHAPE)                        # G does not divide H
    _expect(lib, fn, ssu_m2_args(m, N=512, st=F32), EUNSUP)
    _expect(lib, fn, ssu_m2_args(m, state=m(F16, (8, 80, 64, 128), (0, 8192, 128, 1))), ESTRIDE)
    _expect(lib, fn, ssu_m1_args(m, W=9), EUNSUP)
    a = ssu_m1_args(m)
    a.conv_state = bd.Tensor()
    _expect(lib, fn, a, ENULL)                                                 # conv weight without state
    a = ssu_m1_args(m)
    a.out = a.x
    _expect(lib, fn, a, EALIAS)
    a = ssu_m1_args(m, Bn=4, D=8)
    a.state = m(F32, (6, 8, 16))                                               # slots != batch
    a.conv_state = m(F32, (6, 8, 4))
    _expect(lib, fn, a, ESHAPE)
    a.state_batch_indices = m(I32, (4,))
    _expect(lib, fn, a, OK)                                                    # ... unless indexed
    a.state_batch_indices = m(F32, (4,))
    _expect(lib, fn, a, EDTYPE)
    a = ssu_m1_args(m, Bn=4, D=8)
    a.dt = m(F16, (4, 8, 1))                                                   # rank-3 dt is Mamba-2 only
    _expect(lib, fn, a, ESHAPE)


def test_conv_error_paths(lib):
    fn = "ssm_causal_conv1d_fwd"
    m = FakeMem()
    _expect(lib, fn, conv_args(m, weight=bd.Tensor()), ENULL)
    _expect(lib, fn, conv_args(m, out=m(F32, (2, 64, 100))), EDTYPE)
    _expect(lib, fn, conv_args(m, weight=m(F32, (64, 9))), EUNSUP)
    _expect(lib, fn, conv_args(m, weight=m(F32, (64, 0))), ESHAPE)
    _expect(lib, fn, conv_args(m, conv_state=m(F32, (2, 64, 3))), ESHAPE)
    a = conv_args(m)
    a.out = a.x
    _expect(lib, fn, a, EALIAS)
    a = conv_args(m)                      # the state inside x
    a.conv_state = bd.raw_tensor(a.x.data, F32, (2, 64, 4), None)
    _expect(lib, fn, a, EALIAS)
    a = conv_args(m)                      # the state inside out
    a.conv_state = bd.raw_tensor(a.out.data + 256, F32, (2, 64, 4), None)
    _expect(lib, fn, a, EALIAS)
    # broadcast (self-overlapping) out or state: refused, not raced
    _expect(lib, fn, conv_args(m, out=m(F16, (2, 64, 100), (0, 100, 1))), ESTRIDE)
    _expect(lib, fn, conv_args(m, conv_state=m(F32, (2, 64, 4), (4 * 64, 0, 1))), ESTRIDE)


def test_oversized_tensors_are_rejected_before_any_arithmetic(lib):
    """Element counts, offsets and byte spans past 2^56 would overflow the
    int64 extent and alias arithmetic: such tensors are refused up front."""
    m = FakeMem()
    big = 1 << 30
    _expect(lib, "ssm_selective_scan_fwd", scan_args(m, x=m(F16, (big, big, 1 << 10))), EUNSUP)  # count
    _expect(lib, "ssm_selective_scan_fwd",
            scan_args(m, out=m(F16, (4, 5120, 2048), (1 << 62, 2048, 1))), EUNSUP)          # offset
    _expect(lib, "ssm_causal_conv1d_fwd", conv_args(m, x=m(F32, (1, 1, 1 << 55))), EUNSUP)  # bytes
    _expect(lib, "ssm_selective_state_update",
            ssu_m2_args(m, state=m(F16, (8, 80, 64, 128), (1 << 60, 8192, 128, 1))), EUNSUP)
    # an empty tensor touches no memory, whatever its other sizes and strides
    a = conv_args(m, Bn=0, x=m(F16, (0, 64, 100), (1 << 62, 100, 1)))
    a.out = m(F16, (0, 64, 100))
    a.conv_state = m(F32, (0, 64, 4))
    st, info = call(lib, "ssm_causal_conv1d_fwd", a)
    assert st == OK and info.kernel == 0


def test_binding_rejects_cpu_tensors():
    torch = pytest.importorskip("torch")
    x = torch.zeros(1, 2, 3)
    with pytest.raises(ValueError, match="CUDA tensors only"):
        bd.describe(x)


def test_binding_refuses_a_call_whose_tensors_span_devices():
    torch = pytest.importorskip("torch")

    class Stub:  # stands for a CUDA tensor: only its device is read
        def __init__(self, index):
            self.device = torch.device("cuda", index)

    a, b, c = Stub(0), Stub(0), Stub(1)
    assert bd.device_of((a, None, b)) == torch.device("cuda", 0)
    assert bd.device_of((None, c)) == torch.device("cuda", 1)
    with pytest.raises(ValueError, match="one CUDA device"):
        bd.device_of((a, c))
    with pytest.raises(ValueError, match="one CUDA device"):
        bd.device_of((None, None))


def test_binding_runs_on_the_tensors_device_and_stream(monkeypatch):
    """The entry point gets the tensors' device's current stream (or the
    stream given), and the current device is switched only when the tensors
    live on another one.  torch.cuda is stubbed: nothing touches a GPU."""
    torch = pytest.importorskip("torch")
    state = {"current": 0, "switched_to": []}

    class FakeStream:
        def __init__(self, handle):
            self.cuda_stream = handle

    class FakeDeviceCtx:
        def __init__(self, dev):
            self.dev = dev

        def __enter__(self):
            state["switched_to"].append(self.dev.index)
            self.prev, state["current"] = state["current"], self.dev.index

        def __exit__(self, *exc):
            state["current"] = self.prev

    monkeypatch.setattr(torch.cuda, "current_device", lambda: state["current"])
    monkeypatch.setattr(torch.cuda, "current_stream", lambda dev: FakeStream(1000 + dev.index))
    monkeypatch.setattr(torch.cuda, "device", FakeDeviceCtx)

    class Stub:
        def __init__(self, index):
            self.device = torch.device("cuda", index)

    seen = []

    def fake_entry(args_ref, handle):
        seen.append((handle, state["current"]))
        return 0

    args = bd.ScanArgs()
    assert bd._run(fake_entry, args, (Stub(0), None, Stub(0)), None) == 0
    assert seen[-1] == (1000, 0) and state["switched_to"] == []          # same device: no switch
    assert bd._run(fake_entry, args, (Stub(1), Stub(1)), None) == 0
    assert seen[-1] == (1001, 1) and state["switched_to"] == [1]          # ran on device 1
    assert state["current"] == 0                                          # and switched back
    assert bd._run(fake_entry, args, (Stub(0),), FakeStream(77)) == 0
    assert seen[-1] == (77, 0)                                            # the given stream
    assert bd._run(fake_entry, args, (Stub(0),), 88) == 0
    assert seen[-1] == (88, 0)                                            # a raw handle


# ------------------------------------------------- Mamba-2-layout prefill --
def scan_m2_args(mem, Bn=8, H=80, P=64, N=128, L=2048, G=1, io=F16, time_major=True, **over):
    """x (B, H, P, L) as the view of (B, L, H, P) storage when time_major."""
    a = bd.ScanArgs()
    a.struct_size = ctypes.sizeof(bd.ScanArgs)
    a.flags = bd.SSM_FLAG_DRY_RUN
    if time_major:
        a.x = mem(io, (Bn, H, P, L), (L * H * P, P, 1, H * P))
        a.z = mem(io, (Bn, H, P, L), (L * H * P, P, 1, H * P))
        a.out = mem(io, (Bn, H, P, L), (L * H * P, P, 1, H * P))
        a.dt = mem(io, (Bn, H, L), (L * H, 1, H))
        a.B = mem(io, (Bn, G, N, L), (L * G * N, N, 1, G * N))
        a.C = mem(io, (Bn, G, N, L), (L * G * N, N, 1, G * N))
    else:
        a.x = mem(io, (Bn, H, P, L))
        a.z = mem(io, (Bn, H, P, L))
        a.out = mem(io, (Bn, H, P, L))
        a.dt = mem(io, (Bn, H, L))
        a.B = mem(io, (Bn, G, N, L))
        a.C = mem(io, (Bn, G, N, L))
    a.A = mem(F32, (H,))
    a.D = mem(F32, (H,))
    a.dt_bias = mem(F32, (H,))
    a.dt_softplus = 1
    a.ssm_state = mem(F32, (Bn, H, P, N))
    for k, v in over.items():
        setattr(a, k, v)
    return a


def test_m2_prefill_plan_fast_kernel(lib):
    st, info = call(lib, "ssm_selective_scan_fwd", scan_m2_args(FakeMem()))
    assert st == OK and bd.KERNELS[info.kernel] == "scan_m2"
    # one CTA of 128 threads per (batch, head): 64 headdim rows x 128 state entries
    assert info.block == 128 and info.rows_per_item == 64 and info.grid == 8 * 80
    assert 0 < info.smem_bytes <= 227 * 1024
    st, info = call(lib, "ssm_selective_scan_fwd", scan_m2_args(FakeMem(), H=32, P=128, N=256, io=BF16))
    assert st == OK and bd.KERNELS[info.kernel] == "scan_m2"
    assert info.rows_per_item == 32 and info.grid == 8 * 32 * 4 and info.smem_bytes <= 227 * 1024


@pytest.mark.parametrize("over,why", [
    (dict(time_major=False), "time-last rows"),
    (dict(N=96), "dstate not 64/128/256"),
    (dict(P=12), "headdim not a multiple of 8"),
])
def test_m2_prefill_plan_generic_kernel(lib, over, why):
    st, info = call(lib, "ssm_selective_scan_fwd", scan_m2_args(FakeMem(), **over))
    assert st == OK and bd.KERNELS[info.kernel] == "scan_m2_generic", why


def test_m2_prefill_errors(lib):
    mem = FakeMem()
    a = scan_m2_args(mem)
    a.conv_weight = mem(F32, (80 * 64, 4))
    assert call(lib, "ssm_selective_scan_fwd", a)[0] == EUNSUP  # conv is its own call
    assert call(lib, "ssm_selective_scan_fwd", scan_m2_args(mem, A=mem(F32, (80, 128))))[0] == ESHAPE
    assert call(lib, "ssm_selective_scan_fwd", scan_m2_args(mem, G=3))[0] == ESHAPE  # H % G
    assert call(lib, "ssm_selective_scan_fwd", scan_m2_args(mem, N=300))[0] == EUNSUP
    assert call(lib, "ssm_selective_scan_fwd", scan_m2_args(mem, D=mem(F32, (64,))))[0] == ESHAPE
    assert call(lib, "ssm_selective_scan_fwd", scan_m2_args(mem, z=mem(F32, (8, 80, 64, 2048))))[0] == EDTYPE
    assert call(lib, "ssm_selective_scan_fwd",
                scan_m2_args(mem, ssm_state=mem(F16, (8, 80, 64, 128))))[0] == EDTYPE
    a = scan_m2_args(mem)
    a.out = a.x
    assert call(lib, "ssm_selective_scan_fwd", a)[0] == EALIAS
    a = scan_m2_args(mem, L=0)
    st, info = call(lib, "ssm_selective_scan_fwd", a)
    assert st == OK and bd.KERNELS[info.kernel] == "none"


def test_plain_c_client_links_and_runs(tmp_path, lib):
    """A C program built against include/ssm_causal.h and linked to the .so
    (no Python, no torch types) plans a prefill and a decode and gets every
    documented error status."""
    import subprocess
    src = os.path.join(ROOT, "tests", "c_abi_client.c")
    exe = tmp_path / "c_abi_client"
    libdir = os.path.dirname(bd.LIB_PATH)
    subprocess.check_call(["gcc", "-std=c99", "-O1", "-I", os.path.join(ROOT, "include"), src, "-o", str(exe),
                           "-L", libdir, "-lssm_causal", f"-Wl,-rpath,{libdir}"])
    res = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert res.returncode == 0, res.stdout + res.stderr
    assert "fails 0" in res.stdout


# ----------------------------------------------------------- sequence pieces --
def delta_sum_args(mem, Bn=2, D=64, L=300, io=F16, **over):
    a = bd.DeltaSumArgs()
    a.struct_size = ctypes.sizeof(bd.DeltaSumArgs)
    a.flags = bd.SSM_FLAG_DRY_RUN
    a.dt = mem(io, (Bn, D, L))
    a.dt_bias = mem(F32, (D,))
    a.dt_softplus = 1
    a.out = mem(F32, (Bn, D))
    for k, v in over.items():
        setattr(a, k, v)
    return a


def carry_fold_args(mem, Bn=2, D=64, N=16, **over):
    a = bd.CarryFoldArgs()
    a.struct_size = ctypes.sizeof(bd.CarryFoldArgs)
    a.flags = bd.SSM_FLAG_DRY_RUN
    a.state = mem(F32, (Bn, D, N))
    a.A = mem(F32, (D, N))
    a.delta_sum = mem(F32, (Bn, D))
    a.h_end = mem(F32, (Bn, D, N))
    for k, v in over.items():
        setattr(a, k, v)
    return a


def test_delta_sum_plan_and_checks(lib):
    """One warp per (b, d) row, 8 rows per 256-thread CTA; fp32 output of
    shape (B, D); dt of any float dtype; bias optional; empty rows launch
    nothing; an output over dt is refused."""
    mem = FakeMem()
    st, info = call(lib, "ssm_scan_delta_sum", delta_sum_args(mem))
    assert st == OK and bd.KERNELS[info.kernel] == "delta_sum"
    assert info.grid == 2 * 64 // 8 and info.block == 256 and info.work_items == 128
    st, _ = call(lib, "ssm_scan_delta_sum", delta_sum_args(mem, io=F32, dt_bias=bd.Tensor()))
    assert st == OK
    st, _ = call(lib, "ssm_scan_delta_sum", delta_sum_args(mem, L=0))  # writes zeros
    assert st == OK
    st, info = call(lib, "ssm_scan_delta_sum", delta_sum_args(mem, Bn=0, out=mem(F32, (0, 64))))
    assert st == OK and bd.KERNELS[info.kernel] == "none"
    assert call(lib, "ssm_scan_delta_sum", delta_sum_args(mem, out=mem(F16, (2, 64))))[0] == EDTYPE
    assert call(lib, "ssm_scan_delta_sum", delta_sum_args(mem, out=mem(F32, (2, 63))))[0] == ESHAPE
    assert call(lib, "ssm_scan_delta_sum", delta_sum_args(mem, dt_bias=mem(F32, (65,))))[0] == ESHAPE
    a = delta_sum_args(mem)
    a.out = bd.raw_tensor(a.dt.data, F32, (2, 64))
    assert call(lib, "ssm_scan_delta_sum", a)[0] == EALIAS
    a = delta_sum_args(mem)
    a.struct_size -= 8
    assert call(lib, "ssm_scan_delta_sum", a)[0] == EVER


def test_carry_fold_plan_and_checks(lib):
    """Elementwise over B*D*N with a grid-stride loop of at most 16 CTAs per
    SM; every tensor fp32 with matching shapes; the state may not overlap an
    input."""
    mem = FakeMem()
    st, info = call(lib, "ssm_scan_carry_fold", carry_fold_args(mem))
    assert st == OK and bd.KERNELS[info.kernel] == "carry_fold"
    assert info.grid == 2 * 64 * 16 // 256 and info.rows_per_item == 16 and info.work_items == 128
    st, info = call(lib, "ssm_scan_carry_fold", carry_fold_args(mem, Bn=64, D=5120, N=16))
    assert st == OK and info.grid == 148 * 16
    assert call(lib, "ssm_scan_carry_fold", carry_fold_args(mem, A=mem(F32, (64, 15))))[0] == ESHAPE
    assert call(lib, "ssm_scan_carry_fold", carry_fold_args(mem, delta_sum=mem(F16, (2, 64))))[0] == EDTYPE
    a = carry_fold_args(mem)
    a.h_end = bd.raw_tensor(a.state.data, F32, (2, 64, 16))
    assert call(lib, "ssm_scan_carry_fold", a)[0] == EALIAS
    st, info = call(lib, "ssm_scan_carry_fold", carry_fold_args(mem, Bn=0, state=mem(F32, (0, 64, 16)),
                                                                  delta_sum=mem(F32, (0, 64)),
                                                                  h_end=mem(F32, (0, 64, 16))))
    assert st == OK and bd.KERNELS[info.kernel] == "none"


def test_carry_fold_mamba2_layout_plan(lib):
    """Rank-4 state (B, H, P, N) with A and the sums per head."""
    mem = FakeMem()
    a = carry_fold_args(mem, state=mem(F32, (2, 8, 64, 128)), A=mem(F32, (8,)), delta_sum=mem(F32, (2, 8)),
                        h_end=mem(F32, (2, 8, 64, 128)))
    st, info = call(lib, "ssm_scan_carry_fold", a)
    assert st == OK and bd.KERNELS[info.kernel] == "carry_fold"
    assert info.rows_per_item == 64 * 128 and info.work_items == 16
    a = carry_fold_args(mem, state=mem(F32, (2, 8, 64, 128)), A=mem(F32, (8, 64)), delta_sum=mem(F32, (2, 8)),
                        h_end=mem(F32, (2, 8, 64, 128)))
    assert call(lib, "ssm_scan_carry_fold", a)[0] == ESHAPE
    a = carry_fold_args(mem, state=mem(F32, (2, 8, 64)), A=mem(F32, (8,)), delta_sum=mem(F32, (2, 8)),
                        h_end=mem(F32, (2, 8, 64)))
    assert call(lib, "ssm_scan_carry_fold", a)[0] == ESHAPE  # rank 3 needs A (D, N)


# ------------------------------------------------------------- gated conv --
def gconv_args(mem, Bn=4, D=2048, L=2048, W=3, io=F16, layout="tokens", **over):
    """layout "tokens": x, b_gate, c_gate are the three D-wide slices of one
    (B, L, 3D) projection output and out is (B, L, D) storage, all viewed as
    (B, D, L); "rows": every tensor (B, D, L) contiguous."""
    a = bd.GatedConvArgs()
    a.struct_size = ctypes.sizeof(bd.GatedConvArgs)
    a.flags = bd.SSM_FLAG_DRY_RUN
    es = 4 if io == F32 else 2
    if layout == "tokens":
        proj = mem(io, (Bn, L, 3 * D))
        st = (L * 3 * D, 1, 3 * D)
        a.b_gate, a.c_gate, a.x = (bd.raw_tensor(proj.data + i * D * es, io, (Bn, D, L), st) for i in range(3))
        a.out = mem(io, (Bn, D, L), (L * D, 1, D))
    else:
        a.x, a.b_gate, a.c_gate, a.out = (mem(io, (Bn, D, L)) for _ in range(4))
    a.weight = mem(F32, (D, W))
    a.bias = mem(F32, (D,))
    a.conv_state = mem(F32, (Bn, D, W))
    for k, v in over.items():
        setattr(a, k, v)
    return a


def test_gated_conv_plan_token_major_layout(lib):
    """The three slices of a (B, L, 3D) projection: 16-byte vectors of 8
    channels; segments sized to one wave of 2 CTAs of 256 threads per SM
    (4 x 256 vectors x 74 segments of 28 steps = 296 CTAs), a 96 KB ring of
    8 steps x 3 vectors per thread."""
    st, info = call(lib, "ssm_gated_conv1d_fwd", gconv_args(FakeMem()))
    assert st == OK and bd.KERNELS[info.kernel] == "gated_conv"
    assert info.block == 256 and info.rows_per_item == 8 and info.smem_bytes == 8 * 3 * 256 * 16
    assert info.work_items == 4 * 256 * 74 and info.grid == 2 * 148
    st, info = call(lib, "ssm_gated_conv1d_fwd", gconv_args(FakeMem(), io=F32))
    assert st == OK and bd.KERNELS[info.kernel] == "gated_conv" and info.rows_per_item == 4
    # one decode step: one segment of one step per vector
    st, info = call(lib, "ssm_gated_conv1d_fwd", gconv_args(FakeMem(), Bn=245, L=1))
    assert st == OK and bd.KERNELS[info.kernel] == "gated_conv" and info.work_items == 245 * 256
    # a long, narrow problem keeps segments of at least 8 steps (>= W - 1, so
    # only a row's first segment reads the state it later overwrites)
    for L, segs in ((20, 2), (17, 2), (15, 1), (8, 1), (64, 8), (65, 8)):
        st, info = call(lib, "ssm_gated_conv1d_fwd", gconv_args(FakeMem(), Bn=1, D=8, L=L, W=8))
        assert st == OK and info.work_items == segs, (L, info.work_items)


def test_gated_conv_time_contiguous_rows_plan(lib):
    """(B, D, L) rows with unit step stride: one warp per (row, segment of
    whole 256-step blocks), about 32 warps per SM (8192 rows: one segment)."""
    m = FakeMem()
    st, info = call(lib, "ssm_gated_conv1d_fwd", gconv_args(m, layout="rows"))
    assert st == OK and bd.KERNELS[info.kernel] == "gated_conv_rows" and info.smem_bytes == 0
    assert info.work_items == 4 * 2048 and info.grid == 4 * 2048 // 8 and info.block == 256
    # few rows: segments of whole blocks (one row of 2048 steps -> 8 segments of 256)
    st, info = call(lib, "ssm_gated_conv1d_fwd", gconv_args(m, layout="rows", Bn=1, D=1))
    assert st == OK and bd.KERNELS[info.kernel] == "gated_conv_rows" and info.work_items == 8
    # fp32: vectors of 4 steps, so W - 1 <= 4
    st, info = call(lib, "ssm_gated_conv1d_fwd", gconv_args(m, layout="rows", io=F32, W=5))
    assert st == OK and bd.KERNELS[info.kernel] == "gated_conv_rows"
    st, info = call(lib, "ssm_gated_conv1d_fwd", gconv_args(m, layout="rows", io=F32, W=6))
    assert st == OK and bd.KERNELS[info.kernel] == "gated_conv_generic"


def test_gated_conv_other_layouts_use_the_generic_kernel(lib):
    m = FakeMem()
    st, info = call(lib, "ssm_gated_conv1d_fwd", gconv_args(m, layout="rows", L=2044))  # L not a multiple of 8
    assert st == OK and bd.KERNELS[info.kernel] == "gated_conv_generic" and info.rows_per_item == 1
    assert info.smem_bytes == 0
    st, info = call(lib, "ssm_gated_conv1d_fwd", gconv_args(m, D=2044))  # D not a multiple of 8
    assert st == OK and bd.KERNELS[info.kernel] == "gated_conv_generic"
    a = gconv_args(m)
    a.x = bd.raw_tensor(a.x.data + 2, F16, (4, 2048, 2048), (2048 * 3 * 2048, 1, 3 * 2048))  # 2-byte offset
    st, info = call(lib, "ssm_gated_conv1d_fwd", a)
    assert st == OK and bd.KERNELS[info.kernel] == "gated_conv_generic"


def test_gated_conv_error_paths(lib):
    fn = "ssm_gated_conv1d_fwd"
    m = FakeMem()
    assert lib.ssm_gated_conv1d_fwd(None, None) == ENULL
    _expect(lib, fn, gconv_args(m, weight=bd.Tensor()), ENULL)
    _expect(lib, fn, gconv_args(m, c_gate=bd.Tensor()), ENULL)
    _expect(lib, fn, gconv_args(m, weight=m(F32, (2048, 9))), EUNSUP)
    _expect(lib, fn, gconv_args(m, weight=m(F32, (2048, 0))), ESHAPE)
    _expect(lib, fn, gconv_args(m, b_gate=m(F16, (4, 2048, 2047))), ESHAPE)
    _expect(lib, fn, gconv_args(m, b_gate=m(BF16, (4, 2048, 2048))), EDTYPE)
    _expect(lib, fn, gconv_args(m, out=m(F32, (4, 2048, 2048))), EDTYPE)
    _expect(lib, fn, gconv_args(m, bias=m(F16, (2048,))), EDTYPE)
    _expect(lib, fn, gconv_args(m, conv_state=m(F32, (4, 2048, 4))), ESHAPE)
    _expect(lib, fn, gconv_args(m, conv_state=m(BF16, (4, 2048, 3))), EDTYPE)
    a = gconv_args(m)
    a.out = a.c_gate
    _expect(lib, fn, a, EALIAS)
    a = gconv_args(m)
    a.conv_state = bd.raw_tensor(a.out.data, F32, (4, 2048, 3))
    _expect(lib, fn, a, EALIAS)
    a = gconv_args(m)
    a.struct_size -= 8
    _expect(lib, fn, a, EVER)
    # outputs and the in/out state may not broadcast (stride 0)
    _expect(lib, fn, gconv_args(m, out=m(F16, (4, 2048, 2048), (2048 * 2048, 0, 2048))), ESTRIDE)
    _expect(lib, fn, gconv_args(m, conv_state=m(F32, (4, 2048, 3), (3 * 2048, 3, 0))), ESTRIDE)
    # inputs may: one gate shared by every batch entry
    st, info = call(lib, fn, gconv_args(m, layout="rows", b_gate=m(F16, (4, 2048, 2048), (0, 2048, 1))))
    assert st == OK and bd.KERNELS[info.kernel] == "gated_conv_rows"
    st, info = call(lib, fn, gconv_args(m, L=0))  # the state is left as it is
    assert st == OK and bd.KERNELS[info.kernel] == "none"
    st, info = call(lib, fn, gconv_args(m, Bn=0, conv_state=m(F32, (0, 2048, 3))))
    assert st == OK and bd.KERNELS[info.kernel] == "none"
