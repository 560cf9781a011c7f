"""GPU parity of the standalone causal conv1d, and out-of-bounds guards: every
output and cache is placed inside a larger buffer whose surrounding bands
hold a fixed bit pattern, which must survive every kernel unchanged."""
import numpy as np
import pytest

import oracle
from state_space_model_causal_b200 import inputs as gen
from tests.parity import TOL, N, T, assert_close

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("io", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("L,W", [(1, 4), (3, 4), (4, 4), (255, 4), (256, 4), (257, 4), (700, 4),
                                 (50, 1), (50, 2), (50, 8)])
@pytest.mark.parametrize("silu", [False, True])
def test_conv1d_matches_oracle(io, L, W, silu):
    import torch
    from state_space_model_causal_b200 import ssm_causal_conv1d_fwd
    Bt, D = 2, 6
    x = gen.round_to(gen.normal((Bt, D, L), "conv", L, W, "x"), io)
    w = gen.round_to(gen.normal((D, W), "conv", L, W, "w", std=0.2), "f32")
    b = gen.round_to(gen.normal((D,), "conv", L, W, "b"), "f32")
    cs = gen.round_to(gen.normal((Bt, D, W), "conv", L, W, "cs"), "f32")
    csg = T(cs, "f32")
    out = ssm_causal_conv1d_fwd(T(x, io), T(w, "f32"), bias=T(b, "f32"), conv_state=csg, silu=silu)
    torch.cuda.synchronize()
    ref, csref = oracle.conv1d(x, w, bias=b, conv_state=cs, silu=silu)
    assert_close(N(out), ref, TOL[io], "out")
    np.testing.assert_array_equal(N(csg), csref)


def _conv_kernel(io, L, W):
    """The kernel the planner picks for contiguous (B, D, L) tensors."""
    V = 4 if io == "f32" else 8
    return "conv1d" if L % V == 0 and W - 1 <= V else "conv1d_generic"


@pytest.mark.parametrize("io", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("Bt,D,L,W", [(2, 3, 8, 4), (1, 2, 256, 4), (1, 2, 264, 4), (1, 1, 4096, 4),
                                      (3, 5, 776, 1), (2, 3, 520, 5), (1, 4, 1032, 8), (2, 2, 2048, 7)])
@pytest.mark.parametrize("silu", [False, True])
def test_conv1d_vector_rows_match_oracle(io, Bt, D, L, W, silu):
    """The 16-byte vector kernel: L = 8 (less than one block), one block of
    256 steps exactly, a ragged last block, long rows cut into many segments
    (few rows), widths 1..8 (fp32 takes the warp-per-row kernel above W = 5),
    with an incoming state."""
    import torch
    from state_space_model_causal_b200 import LaunchInfo, binding, ssm_causal_conv1d_fwd
    tag = ("convv", Bt, D, L, W)
    x = gen.round_to(gen.normal((Bt, D, L), *tag, "x"), io)
    w = gen.round_to(gen.normal((D, W), *tag, "w", std=0.2), "f32")
    b = gen.round_to(gen.normal((D,), *tag, "b"), "f32")
    cs = gen.round_to(gen.normal((Bt, D, W), *tag, "cs"), "f32")
    csg = T(cs, "f32")
    info = LaunchInfo()
    out = ssm_causal_conv1d_fwd(T(x, io), T(w, "f32"), bias=T(b, "f32"), conv_state=csg, silu=silu, info=info)
    torch.cuda.synchronize()
    assert binding.KERNELS[info.kernel] == _conv_kernel(io, L, W)
    ref, csref = oracle.conv1d(x, w, bias=b, conv_state=cs, silu=silu)
    assert_close(N(out), ref, TOL[io], "out")
    np.testing.assert_array_equal(N(csg), csref)


@pytest.mark.parametrize("io", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("Bt,D,L,W", [(1, 3600, 8, 4), (2, 1800, 1032, 4), (1, 4000, 264, 1), (1, 3560, 520, 5),
                                      (1, 3600, 16, 8), (1, 3600, 4, 5), (3, 1500, 2048, 3), (2, 1800, 4096, 4)])
def test_conv1d_vector_many_rows_match_oracle(io, Bt, D, L, W):
    """More units than the persistent grid's warps (148 SMs x 4 CTAs x 8),
    so each warp takes several units across row ends: rows of one short
    block, rows of several blocks with a ragged last one, L below the width
    (fp32, L = 4, W = 5), widths 1..8, SiLU, bias and an incoming state."""
    import torch
    from state_space_model_causal_b200 import LaunchInfo, binding, ssm_causal_conv1d_fwd
    tag = ("convm", Bt, D, L, W)
    x = gen.round_to(gen.normal((Bt, D, L), *tag, "x"), io)
    w = gen.round_to(gen.normal((D, W), *tag, "w", std=0.2), "f32")
    b = gen.round_to(gen.normal((D,), *tag, "b"), "f32")
    cs = gen.round_to(gen.normal((Bt, D, W), *tag, "cs"), "f32")
    csg = T(cs, "f32")
    info = LaunchInfo()
    out = ssm_causal_conv1d_fwd(T(x, io), T(w, "f32"), bias=T(b, "f32"), conv_state=csg, silu=True, info=info)
    torch.cuda.synchronize()
    assert binding.KERNELS[info.kernel] == _conv_kernel(io, L, W)
    ref, csref = oracle.conv1d(x, w, bias=b, conv_state=cs, silu=True)
    assert_close(N(out), ref, TOL[io], "out")
    np.testing.assert_array_equal(N(csg), csref)


@pytest.mark.parametrize("io", ["f16", "bf16"])
@pytest.mark.parametrize("D", [7, 3600])
def test_conv1d_vector_state_in_io_dtype_and_padded_rows(io, D):
    """A conv state in the io dtype, no bias, and x / out rows that sit in a
    wider (B, D, L + 16) buffer (aligned, not contiguous)."""
    import torch
    from state_space_model_causal_b200 import LaunchInfo, binding, ssm_causal_conv1d_fwd
    Bt, L, W = 2, 512, 4
    x = gen.round_to(gen.normal((Bt, D, L), "convp", "x"), io)
    w = gen.round_to(gen.normal((D, W), "convp", "w", std=0.2), "f32")
    cs = gen.round_to(gen.normal((Bt, D, W), "convp", "cs"), io)
    xb = torch.zeros((Bt, D, L + 16), dtype=T(x, io).dtype, device="cuda")
    xb[:, :, :L] = T(x, io)
    ob = torch.full_like(xb, 7.0)
    csg = T(cs, io)
    info = LaunchInfo()
    ssm_causal_conv1d_fwd(xb[:, :, :L], T(w, "f32"), conv_state=csg, silu=True, out=ob[:, :, :L], info=info)
    torch.cuda.synchronize()
    assert binding.KERNELS[info.kernel] == _conv_kernel(io, L, W)
    ref, csref = oracle.conv1d(x, w, conv_state=cs, silu=True)
    assert_close(N(ob[:, :, :L]), ref, TOL[io], "out")
    assert bool(torch.all(ob[:, :, L:] == 7.0))
    np.testing.assert_array_equal(N(csg), gen.round_to(csref, io))


@pytest.mark.parametrize("D", [5, 1800])
def test_conv1d_vector_decode_after_prefill(D):
    """A vector-kernel prefill's outgoing state (few rows, or more rows than
    the grid has warps) feeds token-by-token calls (the warp-per-row kernel
    at L = 1); together they equal one oracle call."""
    import torch
    from state_space_model_causal_b200 import ssm_causal_conv1d_fwd
    Bt, L, W, extra = 2, 256, 4, 6
    x = gen.round_to(gen.normal((Bt, D, L + extra), "convd", "x"), "f16")
    w = gen.round_to(gen.normal((D, W), "convd", "w", std=0.2), "f32")
    cs = gen.round_to(gen.normal((Bt, D, W), "convd", "cs"), "f32")
    csg = T(cs, "f32")
    xt = T(x, "f16")
    outs = [N(ssm_causal_conv1d_fwd(xt[:, :, :L].contiguous(), T(w, "f32"), conv_state=csg, silu=True))]
    for t in range(L, L + extra):
        outs.append(N(ssm_causal_conv1d_fwd(xt[:, :, t:t + 1].contiguous(), T(w, "f32"), conv_state=csg,
                                            silu=True)))
    torch.cuda.synchronize()
    ref, csref = oracle.conv1d(x, w, conv_state=cs, silu=True)
    assert_close(np.concatenate(outs, -1), ref, TOL["f16"], "out")
    np.testing.assert_array_equal(N(csg), csref)


def test_conv1d_without_state_at_the_prefill_shape():
    """No conv state: zeros before t = 0 and nothing written; 16 sampled rows
    of the 2.8B prefill's x against the oracle."""
    import torch
    from state_space_model_causal_b200 import LaunchInfo, binding, ssm_causal_conv1d_fwd
    s = gen.prefill_2p8b(seed=0)
    info = LaunchInfo()
    out = ssm_causal_conv1d_fwd(T(s.x, "f16"), T(s.conv_weight, "f32"),
                                bias=T(s.conv_bias, "f32"), silu=True, info=info)
    torch.cuda.synchronize()
    assert binding.KERNELS[info.kernel] == "conv1d"
    got = N(out)
    rng = np.random.default_rng(3)
    for b, d in zip(rng.integers(0, 4, 16), rng.integers(0, 5120, 16)):
        ref, _ = oracle.conv1d(s.x[b:b + 1, d:d + 1], s.conv_weight[d:d + 1],
                               bias=s.conv_bias[d:d + 1], silu=True)
        assert_close(got[b:b + 1, d:d + 1], ref, TOL["f16"], f"row ({b},{d})")


def test_conv1d_full_size_every_element():
    """The benchmark's launch (B=4, D=5120, L=2048, W=4, fp16, bias, SiLU, an
    fp32 conv state read and written) against the oracle on every output
    element and every state entry."""
    import torch
    from state_space_model_causal_b200 import LaunchInfo, binding, ssm_causal_conv1d_fwd
    tag = ("convfull",)
    x = gen.round_to(gen.normal((4, 5120, 2048), *tag, "x"), "f16")
    w = gen.round_to(gen.normal((5120, 4), *tag, "w", std=0.2), "f32")
    b = gen.round_to(gen.normal((5120,), *tag, "b", std=0.1), "f32")
    cs = gen.round_to(gen.normal((4, 5120, 4), *tag, "cs"), "f32")
    csg = T(cs, "f32")
    info = LaunchInfo()
    out = ssm_causal_conv1d_fwd(T(x, "f16"), T(w, "f32"), bias=T(b, "f32"), conv_state=csg, silu=True, info=info)
    torch.cuda.synchronize()
    assert binding.KERNELS[info.kernel] == "conv1d"
    ref, csref = oracle.conv1d(x, w, bias=b, conv_state=cs, silu=True)
    assert_close(N(out), ref, TOL["f16"], "out")
    np.testing.assert_array_equal(N(csg), csref)


# ------------------------------------------------------------ canary bands --
CANARY_WORDS = 4096  # 16 KiB of pattern on each side


def _banded(shape, dtype):
    """Tensor of `shape`/`dtype` carved out of a uint8 buffer with canary
    bands of 0xA5 bytes before and after it."""
    import torch
    es = {torch.float32: 4, torch.float16: 2, torch.bfloat16: 2}[dtype]
    n = int(np.prod(shape)) * es
    pad = CANARY_WORDS * 4
    buf = torch.full((pad + n + pad,), 0xA5, dtype=torch.uint8, device="cuda")
    t = buf[pad:pad + n].view(dtype).view(*shape)
    return buf, t, pad, n


def _bands_intact(buf, pad, n):
    import torch
    return bool(torch.all(buf[:pad] == 0xA5)) and bool(torch.all(buf[pad + n:] == 0xA5))


def test_prefill_writes_stay_inside_outputs():
    import torch
    from state_space_model_causal_b200 import ssm_selective_scan_fwd
    s = gen.scan_inputs(3, 77, 40, 16, W=4, io="f16", seed=20, tag="canary", conv_state=True,
                        h0=True)
    bo, out, po, no = _banded((3, 40, 77), torch.float16)
    bh, h, ph, nh = _banded((3, 40, 16), torch.float32)
    bc, cs, pc, nc = _banded((3, 40, 4), torch.float32)
    h.copy_(T(s.h0, "f32"))
    cs.copy_(T(s.conv_state, "f32"))
    ssm_selective_scan_fwd(T(s.x, "f16"), T(s.dt, "f16"), T(s.A, "f32"), T(s.B, "f16"),
                           T(s.C, "f16"), D=T(s.D, "f32"), z=T(s.z, "f16"),
                           dt_bias=T(s.dt_bias, "f32"), conv_weight=T(s.conv_weight, "f32"),
                           conv_bias=T(s.conv_bias, "f32"), conv_state=cs, ssm_state=h, out=out)
    torch.cuda.synchronize()
    for buf, pad, n in ((bo, po, no), (bh, ph, nh), (bc, pc, nc)):
        assert _bands_intact(buf, pad, n)


@pytest.mark.parametrize("layout", ["mamba1", "mamba2"])
def test_ssu_writes_stay_inside_caches(layout):
    import torch
    from state_space_model_causal_b200 import ssm_selective_state_update
    if layout == "mamba1":
        s = gen.ssu_mamba1_inputs(5, 72, 16, W=4, io="f16", state="f32", seed=21, tag="canary1")
        bst, st, pst, nst = _banded(s.state.shape, torch.float32)
        bcs, cs, pcs, ncs = _banded(s.conv_state.shape, torch.float32)
        st.copy_(T(s.state, "f32"))
        cs.copy_(T(s.conv_state, "f32"))
        bo, out, po, no = _banded(s.x.shape, torch.float16)
        ssm_selective_state_update(st, T(s.x, "f16"), T(s.dt, "f16"), T(s.A, "f32"), T(s.B, "f16"),
                                   T(s.C, "f16"), D=T(s.D, "f32"), z=T(s.z, "f16"),
                                   dt_bias=T(s.dt_bias, "f32"), conv_weight=T(s.conv_weight, "f32"),
                                   conv_bias=T(s.conv_bias, "f32"), conv_state=cs, out=out)
        bands = [(bst, pst, nst), (bcs, pcs, ncs), (bo, po, no)]
    else:
        s = gen.ssu_mamba2_inputs(3, 5, 24, 128, io="bf16", state="bf16", seed=22, tag="canary2")
        bst, st, pst, nst = _banded(s.state.shape, torch.bfloat16)
        st.copy_(T(s.state, "bf16"))
        bo, out, po, no = _banded(s.x.shape, torch.bfloat16)
        ssm_selective_state_update(st, T(s.x, "bf16"), T(s.dt, "bf16"), T(s.A, "f32"),
                                   T(s.B, "bf16"), T(s.C, "bf16"), D=T(s.D, "f32"),
                                   dt_bias=T(s.dt_bias, "f32"), out=out)
        bands = [(bst, pst, nst), (bo, po, no)]
    torch.cuda.synchronize()
    for buf, pad, n in bands:
        assert _bands_intact(buf, pad, n)


def test_conv1d_writes_stay_inside_outputs():
    import torch
    from state_space_model_causal_b200 import ssm_causal_conv1d_fwd
    x = gen.round_to(gen.normal((2, 9, 301), "cc", "x"), "f16")
    w = gen.round_to(gen.normal((9, 4), "cc", "w"), "f32")
    bo, out, po, no = _banded((2, 9, 301), torch.float16)
    bc, cs, pc, nc = _banded((2, 9, 4), torch.float32)
    cs.zero_()
    ssm_causal_conv1d_fwd(T(x, "f16"), T(w, "f32"), conv_state=cs, silu=True, out=out)
    torch.cuda.synchronize()
    assert _bands_intact(bo, po, no) and _bands_intact(bc, pc, nc)
