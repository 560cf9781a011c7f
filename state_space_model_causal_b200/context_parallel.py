"""Context-parallel prefill: one sequence piece per rank of a process group,
in the Mamba-1 layout (with the fused conv) or the Mamba-2 layout.

The selective scan is a first-order linear recurrence in h, so a sequence cut
into consecutive pieces composes (the long-context point of "feat(llama.cu):
适配 mamba 模型", section 6.1: the scan is linear in the sequence length).
Rank r holds steps [t_r, t_{r+1}) of every sequence of the batch and runs:

1. *halo*: an all-gather of every rank's last W raw inputs, so that rank r's
   conv history is the previous rank's tail (rank 0 keeps the sequence's
   incoming conv state);
2. *pass 1*: ``ssm_selective_scan_fwd`` over its piece -- rank 0 from the
   sequence's initial state (its outputs and end state are final), every
   other rank from a zero state, giving its end state h_end(r) -- and
   ``ssm_scan_delta_sum`` for the piece's sum of delta S(r);
3. *exchange*: an all-gather of the records (h_end, S) over the ranks,
   B*D*(N+1) floats per rank (B*H*(P*N+1) in the Mamba-2 layout);
4. *pass 2* (ranks r > 0): h_in(r) composed from the records by r - 1
   ``ssm_scan_carry_fold`` calls, h_in(j+1) = exp(A * S(j)) * h_in(j) +
   h_end(j) from h_in(1) = h_end(0), then ``ssm_selective_scan_fwd`` over the
   piece from h_in(r) for the outputs and the caches.

Every step of the method runs in the library's kernels; this module only
moves the halo and the records through the collective (NCCL over NVLink on
GPUs, or any backend that implements ``all_gather``).  The last rank ends
with the sequence's final caches.  Ranks r > 0 scan their piece twice (the
fix-up of the Mamba-1 layout needs one exponential per element, as much as
the scan itself; the Mamba-2 layout runs the same two passes), so the speedup
over one GPU is about R / 2 for R ranks.
"""
from __future__ import annotations

from typing import List


class TorchCollective:
    """The collective of a ``torch.distributed`` process group (default group
    when ``group`` is None)."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.rank = dist.get_rank(group)
        self.world_size = dist.get_world_size(group)

    def all_gather(self, t) -> List:
        out = [t.new_empty(t.shape) for _ in range(self.world_size)]
        self.dist.all_gather(out, t.contiguous(), group=self.group)
        return out


class LibraryOps:
    """The library calls the driver is built from (the C-ABI binding)."""

    def __init__(self):
        from . import binding
        self.b = binding

    def scan(self, x, dt, A, B, C, **kw):
        return self.b.ssm_selective_scan_fwd(x, dt, A, B, C, **kw)

    def delta_sum(self, dt, dt_bias, dt_softplus):
        return self.b.ssm_scan_delta_sum(dt, dt_bias=dt_bias, dt_softplus=dt_softplus)

    def carry_fold(self, state, A, S, h_end):
        return self.b.ssm_scan_carry_fold(state, A, S, h_end)


def prefill_context_parallel(x, dt, A, B, C, *, D=None, z=None, dt_bias=None, dt_softplus=True,
                             conv_weight=None, conv_bias=None, conv_state=None, ssm_state=None,
                             out=None, comm=None, ops=None):
    """Prefill of this rank's piece of the sequences (see
    ``ssm_selective_scan_fwd``).  Mamba-1 layout: x, dt, z (B, D, L_r); A (D, N);
    B, C (B, N, L_r) or (B, G, N, L_r); ssm_state (B, D, N).  Mamba-2 layout:
    x, z (B, H, P, L_r); dt (B, H, L_r); A (H); B, C (B, G, N, L_r);
    ssm_state (B, H, P, N); no fused conv.  conv_state (B, D, W) and ssm_state
    are the sequences' incoming caches on rank 0 (ignored elsewhere); each
    rank's are updated in place with the caches at the end of its piece, so
    the last rank's are the sequences' final ones.  A conv width W needs
    pieces of at least W steps.  comm: an object with ``rank``, ``world_size``
    and ``all_gather(tensor) -> list`` (default: the torch.distributed group).
    Returns out, shaped like x."""
    import torch
    comm = comm if comm is not None else TorchCollective()
    ops = ops if ops is not None else LibraryOps()
    r, R = comm.rank, comm.world_size
    L = x.shape[-1]
    if x.dim() == 4:  # Mamba-2 layout: the state is (B, H, P, N)
        if conv_weight is not None:
            raise ValueError("the Mamba-2-layout prefill takes no fused conv")
        state_shape = (x.shape[0], x.shape[1], x.shape[2], B.shape[-2])
    else:
        state_shape = (x.shape[0], x.shape[1], A.shape[1])
    Bt, Dd = x.shape[0], x.shape[1]
    W = conv_weight.shape[1] if conv_weight is not None else 0
    if W and L < W:
        raise ValueError(f"every piece needs at least the conv width ({W}) of steps, got {L}")
    if out is None:
        out = torch.empty_like(x)
    kw = dict(D=D, z=z, dt_bias=dt_bias, dt_softplus=dt_softplus, conv_weight=conv_weight,
              conv_bias=conv_bias)

    # 1. halo: the last W raw inputs of every piece (copies, no arithmetic)
    history = None
    if W:
        tails = comm.all_gather(x[..., L - W:].to(torch.float32).contiguous())
        if r == 0:
            history = (conv_state.to(torch.float32).clone() if conv_state is not None
                       else torch.zeros(Bt, Dd, W, dtype=torch.float32, device=x.device))
        else:
            history = tails[r - 1].clone()

    # 2. pass 1: rank 0 from the initial state (final results), the others from zero
    h = torch.zeros(state_shape, dtype=torch.float32, device=x.device)
    if r == 0 and ssm_state is not None:
        h.copy_(ssm_state)
    cs = history.clone() if W else None
    first_out = out if r == 0 else torch.empty_like(x)
    ops.scan(x, dt, A, B, C, conv_state=cs, ssm_state=h, out=first_out, **kw)
    S = ops.delta_sum(dt, dt_bias, dt_softplus)

    # 3. exchange the records
    h_ends = comm.all_gather(h)
    sums = comm.all_gather(S)

    # 4. pass 2: compose the state entering this piece, scan it again
    if r > 0:
        h = h_ends[0].clone()
        for j in range(1, r):
            ops.carry_fold(h, A, sums[j], h_ends[j])
        cs = history.clone() if W else None
        ops.scan(x, dt, A, B, C, conv_state=cs, ssm_state=h, out=out, **kw)
    if ssm_state is not None:
        ssm_state.copy_(h)
    if conv_state is not None and W:
        conv_state.copy_(cs)
    return out
