"""Context-parallel relay of the carried state between GPUs.

For sequences longer than one GPU should hold, every rank of a process group
takes one time segment of every (batch, head) sequence: rank r holds tokens
[r*T_r, (r+1)*T_r).  The recurrence couples the segments only through the
state at a segment boundary (per head a dv x dk fp32 matrix, 64 KB at
d = 128), and the state-to-state map of a segment is a full linear operator on
the state, so the segments cannot be summarised and combined in a scan: the
state has to be handed on.

Forward, on every rank:
  1. the state-independent chunk work (kron_delta_fwd_phase, LOCAL), at once
     on all ranks;
  2. rank r > 0 receives S0 from rank r-1, straight into its own memory (a
     point-to-point NCCL transfer over NVLink; rank 0 uses the given S0);
  3. the chunk chain and the outputs (CARRY); the final state goes to rank
     r+1 while this rank's output kernel runs.
Backward, mirrored: the dST-independent per-chunk work first, then rank r <
P-1 receives dST from rank r+1, runs the reverse chain and the rest, and
sends its dS0 to rank r-1.

The chains run one rank after the other; the chunk-local work (more than
half of a step) is split P ways and overlaps the upstream chains.  No
collective and no multicast: one send and one receive per rank and
direction, each of B*H*dv*dk*4 bytes.

The operations a rank runs on its segment come from an ops object with the
methods of ``CudaSegmentOps``, the default, which runs the library's kernels
through the C ABI (there is no other implementation in the package).
"""
from __future__ import annotations

from dataclasses import dataclass, field

__all__ = ["CudaSegmentOps", "RelayContext", "relay_fwd", "relay_bwd"]


@dataclass
class RelayContext:
    """What the forward of one segment keeps for its backward."""
    inputs: tuple
    S_in: object            # the state received at the segment start (None = zero on rank 0)
    save: dict = field(default_factory=dict)


class CudaSegmentOps:
    """Segment operations on the current CUDA device through the C ABI."""

    def __init__(self, stream=None):
        self.stream = stream

    def new_state(self, like, B, H, dv, dk):
        import torch
        return torch.empty((B, H, dv, dk), dtype=torch.float32, device=like.device)

    def fwd_local(self, inputs, save):
        import delta_rule_linear_kron_b200 as kd
        q, k, v, beta, c, logf = inputs
        out, ST, ws = kd.fwd(q, k, v, beta, c, logf, None, save=save, phase=kd.KD_PHASE_LOCAL,
                             stream=self.stream)
        return dict(out=out, ST=ST, ws=ws, save=save)

    def fwd_carry(self, inputs, S_in, st):
        import delta_rule_linear_kron_b200 as kd
        q, k, v, beta, c, logf = inputs
        out, ST, _ = kd.fwd(q, k, v, beta, c, logf, S_in, out=st["out"], state_out=st["ST"], save=st["save"],
                            workspace=st["ws"], phase=kd.KD_PHASE_CARRY, stream=self.stream)
        return out, ST

    def bwd_local(self, inputs, S_in, st, dO):
        import delta_rule_linear_kron_b200 as kd
        q, k, v, beta, c, logf = inputs
        B, T, H, dk = q.shape
        dv = v.shape[-1]
        ws = kd._alloc_ws(kd.workspace_size(kd.KD_WS_BWD, B, H, T, dk, dv, kd._dtype_code(q)), q.device)
        g = kd.bwd(q, k, v, beta, c, logf, S_in, dO, None, fwd_workspace=st["ws"], workspace=ws,
                   phase=kd.KD_PHASE_LOCAL, stream=self.stream)
        return dict(g=g, ws=ws)

    def bwd_carry(self, inputs, S_in, st, dO, dST, bst):
        import delta_rule_linear_kron_b200 as kd
        q, k, v, beta, c, logf = inputs
        return kd.bwd(q, k, v, beta, c, logf, S_in, dO, dST, fwd_workspace=st["ws"], workspace=bst["ws"],
                      phase=kd.KD_PHASE_CARRY, grads=bst["g"], stream=self.stream)


def _ranks(group):
    import torch.distributed as dist
    rank = dist.get_rank(group)
    world = dist.get_world_size(group)

    def glob(r):
        return r if group is None else dist.get_global_rank(group, r)
    return rank, world, glob


def relay_fwd(q, k, v, beta, c, logf, S0=None, *, group=None, ops=None, save=True):
    """Forward of this rank's time segment (inputs [B, T_r, H, d]).  S0 is used
    on rank 0 only.  Returns (out, ST, ctx): ST is the state after the whole
    sequence on the last rank and None elsewhere; ctx feeds relay_bwd."""
    import torch.distributed as dist
    ops = CudaSegmentOps() if ops is None else ops
    rank, world, glob = _ranks(group)
    inputs = (q, k, v, beta, c, logf)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    st = ops.fwd_local(inputs, save)
    if rank == 0:
        S_in = S0
    else:
        S_in = ops.new_state(q, B, H, dv, dk)
        dist.recv(S_in, src=glob(rank - 1), group=group)
    out, ST = ops.fwd_carry(inputs, S_in, st)
    if rank < world - 1:
        dist.send(ST, dst=glob(rank + 1), group=group)
        ST = None
    return out, ST, RelayContext(inputs=inputs, S_in=S_in, save=st)


def relay_bwd(ctx, dO, dST=None, *, group=None, ops=None):
    """Backward of this rank's segment for the loss <dO, out> (all ranks) +
    <dST, ST> (dST used on the last rank only).  Returns the gradient dict
    (dq, dk, dv, dbeta, dc, dlogf, dS0); dS0 is the gradient of the initial
    state on rank 0 and the gradient of the received state elsewhere."""
    import torch.distributed as dist
    ops = CudaSegmentOps() if ops is None else ops
    rank, world, glob = _ranks(group)
    q, k, v = ctx.inputs[:3]
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    bst = ops.bwd_local(ctx.inputs, ctx.S_in, ctx.save, dO)
    if rank == world - 1:
        dS_in = dST
    else:
        dS_in = ops.new_state(q, B, H, dv, dk)
        dist.recv(dS_in, src=glob(rank + 1), group=group)
    g = ops.bwd_carry(ctx.inputs, ctx.S_in, ctx.save, dO, dS_in, bst)
    if rank > 0:
        dist.send(g["dS0"], dst=glob(rank - 1), group=group)
    return g
