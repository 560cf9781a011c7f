"""GPU parity of the double-gated short causal conv (ssm_gated_conv1d_fwd)
against the fp64 oracle: out = Cg * (bias + causal conv of Bg * x), the
reading of the "double-gated LIV convolution blocks" of
"LFM2.5-1.2B-Thinking性能优化CUDA核心编程技巧" (section 2.1).

Both layouts: "tokens" (x, Bg, Cg the three D-wide slices of one (B, L, 3D)
projection output, out (B, L, D) storage: the 16-byte vector kernel) and
"rows" (every tensor (B, D, L): the time-contiguous kernel when L is a
multiple of the vector width, else the generic one).  The outgoing conv state
holds gated inputs, which are exact in fp32 for 16-bit inputs and correctly
rounded for fp32 inputs, so it is compared bit for bit."""
import numpy as np
import pytest

import oracle
from state_space_model_causal_b200 import inputs as gen
from tests.parity import TOL, N, T, assert_close

pytestmark = pytest.mark.gpu


def _device(s, layout, state_dtype="f32"):
    """Device tensors of a GatedConvInputs in the given layout."""
    import torch
    Bt, D, L = s.x.shape
    if layout == "tokens":
        proj = np.concatenate([s.bg, s.cg, s.x], axis=1).transpose(0, 2, 1)  # (B, L, 3D)
        pt = T(proj, s.io)
        bg, cg, x = (pt[:, :, i * D:(i + 1) * D].transpose(1, 2) for i in range(3))
        out = torch.empty((Bt, L, D), dtype=x.dtype, device=x.device).transpose(1, 2)
    else:
        x, bg, cg = T(s.x, s.io), T(s.bg, s.io), T(s.cg, s.io)
        out = torch.empty_like(x)
    cs = T(s.conv_state, state_dtype) if s.conv_state is not None else None
    return x, bg, cg, out, cs


def _run(s, layout, state_dtype="f32"):
    import torch
    from state_space_model_causal_b200 import LaunchInfo, binding, ssm_gated_conv1d_fwd
    x, bg, cg, out, cs = _device(s, layout, state_dtype)
    info = LaunchInfo()
    ssm_gated_conv1d_fwd(x, bg, cg, T(s.weight, "f32"), bias=T(s.bias, "f32"), conv_state=cs, out=out,
                         info=info)
    torch.cuda.synchronize()
    return N(out), N(cs), binding.KERNELS[info.kernel]


def expected_kernel(layout, io, L, W):
    """The kernel the planner picks for contiguous test tensors."""
    V = 4 if io == "f32" else 8
    if layout == "tokens" or L == 1:
        return "gated_conv"
    return "gated_conv_rows" if L % V == 0 and W - 1 <= V else "gated_conv_generic"


@pytest.mark.parametrize("layout", ["tokens", "rows"])
@pytest.mark.parametrize("io", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("Bt,L,D,W", [(2, 1, 16, 3), (2, 5, 16, 4), (1, 37, 24, 3), (3, 300, 32, 4),
                                      (2, 129, 8, 1), (1, 64, 16, 8), (2, 7, 16, 8), (1, 17, 8, 8),
                                      (1, 23, 8, 8), (2, 65, 8, 7)])
def test_gated_conv_matches_oracle(layout, io, Bt, L, D, W):
    """Ragged lengths, lengths below the conv width, widths 1..8, many
    segments per row (few channel vectors), with bias and an incoming state."""
    s = gen.gated_conv_inputs(Bt, L, D, W, io=io, seed=1, tag=f"gc/{L}/{D}/{W}", conv_state=True)
    got, cs, kern = _run(s, layout)
    assert kern == expected_kernel(layout, io, L, W)
    ref, csref = oracle.gated_conv1d(s.x, s.bg, s.cg, s.weight, bias=s.bias, conv_state=s.conv_state)
    assert_close(got, ref, TOL[io], "out")
    np.testing.assert_array_equal(cs, gen.round_to(csref, "f32"))


@pytest.mark.parametrize("io", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("Bt,L,W", [(2, 1, 3), (3, 5, 4), (1, 37, 3), (2, 300, 4), (2, 129, 1), (1, 64, 8),
                                    (2, 2100, 3)])
def test_gated_conv_whole_warp_rows_match_oracle(io, Bt, L, W):
    """Rows of exactly 32 channel vectors (D = 256 at 16-bit, 128 at fp32),
    so that every warp's threads share one (batch, segment) row; ragged
    segment lengths, widths 1..8, an incoming state."""
    D = 128 if io == "f32" else 256
    s = gen.gated_conv_inputs(Bt, L, D, W, io=io, seed=7, tag=f"gcw/{L}/{W}", conv_state=True)
    got, cs, kern = _run(s, "tokens")
    assert kern == "gated_conv"
    ref, csref = oracle.gated_conv1d(s.x, s.bg, s.cg, s.weight, bias=s.bias, conv_state=s.conv_state)
    assert_close(got, ref, TOL[io], "out")
    np.testing.assert_array_equal(cs, gen.round_to(csref, "f32"))


@pytest.mark.parametrize("io", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("Bt,L,D,W", [(2, 256, 4, 3), (1, 264, 3, 4), (1, 2048, 2, 4), (3, 520, 5, 1),
                                      (1, 8, 2, 5), (2, 776, 3, 8)])
def test_gated_conv_time_contiguous_rows_match_oracle(io, Bt, L, D, W):
    """(B, D, L) rows: one block of 256 steps exactly, a ragged last block,
    rows cut into segments (few rows), L = 8, widths 1..8 (fp32 takes the
    strided kernel above W = 5), with an incoming state."""
    s = gen.gated_conv_inputs(Bt, L, D, W, io=io, seed=9, tag=f"gcr/{L}/{D}/{W}", conv_state=True)
    got, cs, kern = _run(s, "rows")
    assert kern == expected_kernel("rows", io, L, W)
    ref, csref = oracle.gated_conv1d(s.x, s.bg, s.cg, s.weight, bias=s.bias, conv_state=s.conv_state)
    assert_close(got, ref, TOL[io], "out")
    np.testing.assert_array_equal(cs, gen.round_to(csref, "f32"))


@pytest.mark.parametrize("io", ["f16", "bf16"])
def test_gated_conv_state_in_the_io_dtype_and_no_bias(io):
    s = gen.gated_conv_inputs(2, 50, 32, 3, io=io, seed=2, tag="gc/io_state", bias=False, conv_state=True,
                              state_dtype=io)
    got, cs, kern = _run(s, "tokens", state_dtype=io)
    assert kern == "gated_conv"
    ref, csref = oracle.gated_conv1d(s.x, s.bg, s.cg, s.weight, conv_state=s.conv_state)
    assert_close(got, ref, TOL[io], "out")
    np.testing.assert_array_equal(cs, gen.round_to(csref, io))


@pytest.mark.parametrize("layout,L", [("tokens", 40), ("rows", 40), ("rows", 300)])
def test_gated_conv_without_state_starts_from_zeros(layout, L):
    s = gen.gated_conv_inputs(2, L, 16, 4, io="f16", seed=3, tag="gc/nostate")
    got, cs, _ = _run(s, layout)
    assert cs is None
    ref, _ = oracle.gated_conv1d(s.x, s.bg, s.cg, s.weight, bias=s.bias)
    assert_close(got, ref, TOL["f16"], "out")


@pytest.mark.parametrize("D", [64, 256])
def test_gated_conv_decode_steps_equal_one_prefill(D):
    """Token-by-token calls (L = 1) through the conv state give the prefill's
    outputs and final state; each step also matches the oracle's step."""
    import torch
    from state_space_model_causal_b200 import ssm_gated_conv1d_fwd
    Bt, L, W = 3, 12, 3
    s = gen.gated_conv_inputs(Bt, L, D, W, io="f16", seed=4, tag="gc/decode", conv_state=True)
    x, bg, cg, _, cs = _device(s, "tokens")
    w, b = T(s.weight, "f32"), T(s.bias, "f32")
    steps = []
    for t in range(L):
        o = ssm_gated_conv1d_fwd(x[:, :, t:t + 1], bg[:, :, t:t + 1], cg[:, :, t:t + 1], w, bias=b, conv_state=cs)
        steps.append(N(o))
    torch.cuda.synchronize()
    ref, csref = oracle.gated_conv1d(s.x, s.bg, s.cg, s.weight, bias=s.bias, conv_state=s.conv_state)
    assert_close(np.concatenate(steps, -1), ref, TOL["f16"], "decoded out")
    np.testing.assert_array_equal(N(cs), gen.round_to(csref, "f32"))
    full, csf, _ = _run(s, "tokens")
    np.testing.assert_array_equal(np.concatenate(steps, -1), full)
    np.testing.assert_array_equal(N(cs), csf)


def test_gated_conv_full_size_every_element():
    """The benchmark's workload (B=4, L=2048, D=2048, W=3, fp16, token-major
    slices of one projection output), in the launch the benchmark times,
    against the oracle on every element."""
    s = gen.gated_conv_lfm(seed=0)
    got, _, kern = _run(s, "tokens")
    assert kern == "gated_conv"
    ref, _ = oracle.gated_conv1d(s.x, s.bg, s.cg, s.weight, bias=s.bias)
    assert_close(got, ref, TOL["f16"], "out")


def test_gated_conv_empty_and_zero_length():
    import torch
    from state_space_model_causal_b200 import LaunchInfo, binding, ssm_gated_conv1d_fwd
    s = gen.gated_conv_inputs(2, 0, 16, 3, io="f16", seed=5, tag="gc/empty", conv_state=True)
    x, bg, cg, out, cs = _device(s, "rows")
    before = N(cs)
    info = LaunchInfo()
    ssm_gated_conv1d_fwd(x, bg, cg, T(s.weight, "f32"), bias=T(s.bias, "f32"), conv_state=cs, out=out, info=info)
    torch.cuda.synchronize()
    assert binding.KERNELS[info.kernel] == "none"
    np.testing.assert_array_equal(N(cs), before)


def test_gated_conv_input_gate_broadcast_over_the_batch():
    """One input gate for every batch entry (batch stride 0), rows layout."""
    import torch
    from state_space_model_causal_b200 import ssm_gated_conv1d_fwd
    s = gen.gated_conv_inputs(3, 40, 16, 4, io="f16", seed=8, tag="gc/bcast", conv_state=True)
    bg1 = s.bg[:1]
    bgt = T(bg1, "f16").expand(3, -1, -1)
    cs = T(s.conv_state, "f32")
    out = ssm_gated_conv1d_fwd(T(s.x, "f16"), bgt, T(s.cg, "f16"), T(s.weight, "f32"), bias=T(s.bias, "f32"),
                               conv_state=cs)
    torch.cuda.synchronize()
    bg_full = np.broadcast_to(bg1, s.bg.shape)
    ref, csref = oracle.gated_conv1d(s.x, bg_full, s.cg, s.weight, bias=s.bias, conv_state=s.conv_state)
    assert_close(N(out), ref, TOL["f16"], "out")
    np.testing.assert_array_equal(N(cs), gen.round_to(csref, "f32"))
