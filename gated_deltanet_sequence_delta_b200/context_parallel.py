"""Context-parallel prefill: the sequences of one call cut into consecutive segments, one
per rank of a torch.distributed process group (rank r holds tokens r T_seg .. (r+1) T_seg - 1
of every sequence), so that a long prefill is spread over several GPUs.

Over a segment the gated delta rule is affine in the state it starts from (the product form
of the update in the "Gated DeltaNet" research log, with H = S^T):
    H_end = A H_start + B,     o_t = o0_t + H_start^T c_t.
Each rank runs its segment twice through ``gdn_chunk_prefill``: from a zero state (giving
o0 and B) and with v = 0 from H_start = I (giving c and A).  The only exchange is an
all-gather of every segment's (A, B), 2 x 64 KB per (sequence, value head); then
``gdn_cp_combine`` scans them to this rank's H_start and the final state, and corrects o.
The state never waits on another rank's kernels: the collective sits between launches.
"""
from __future__ import annotations

import torch

from . import binding as B


def segment_transitions(q, k, v, g, beta, BT: int = 64, scale: float = 1.0, qk_l2norm: bool = True):
    """This rank's segment, dense [N, T_seg, ...] tensors on the GPU.  Returns (o0, Bs, c, As):
    o0 [N, T_seg, HV, Dv] and Bs [N, HV, Dk, Dv] from a zero start, c and As from the run
    with v = 0 starting at the identity (Dk = Dv).  The tensor-core shapes take one call that
    shares the chunk-local stage between the two runs; the others take two prefills."""
    N, _, _, Dk = q.shape
    HV, Dv = v.shape[-2:]
    if Dk != Dv:
        raise ValueError("context-parallel prefill needs Dk == Dv")
    try:
        return B.gdn_cp_segment(q, k, v, g, beta, BT=BT, scale=scale, qk_l2norm=qk_l2norm)
    except B.GDNError as err:
        if err.status != 4:   # anything but UNSUPPORTED is a real failure
            raise
    o0, Bs = B.gdn_chunk_prefill(q, k, v, g, beta, BT=BT, scale=scale, qk_l2norm=qk_l2norm)
    eye = torch.eye(Dk, dtype=torch.float32, device=q.device).expand(N, HV, Dk, Dk).contiguous()
    c, As = B.gdn_chunk_prefill(q, k, torch.zeros_like(v), g, beta, initial_state=eye, BT=BT, scale=scale,
                                qk_l2norm=qk_l2norm)
    return o0, Bs, c, As


def gather_transitions(As, Bs, group=None):
    """All-gather every rank's (A, B) in rank order: returns A_all, B_all [R, N, HV, Dk, Dv]."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    A_all = torch.empty((world,) + tuple(As.shape), dtype=As.dtype, device=As.device)
    B_all = torch.empty((world,) + tuple(Bs.shape), dtype=Bs.dtype, device=Bs.device)
    dist.all_gather(list(A_all.unbind(0)), As.contiguous(), group=group)
    dist.all_gather(list(B_all.unbind(0)), Bs.contiguous(), group=group)
    return A_all, B_all


def cp_chunk_prefill(q, k, v, g, beta, initial_state=None, group=None, BT: int = 64, scale: float = 1.0,
                     qk_l2norm: bool = True):
    """Context-parallel prefill of this rank's segment.  q, k [N, T_seg, HK, Dk], v [N, T_seg,
    HV, Dv], g, beta [N, T_seg, HV] on the rank's GPU; initial_state [N, HV, Dk, Dv] (the
    state before segment 0, read on every rank) or None.  Returns (o of this segment, the
    sequences' final states, this segment's start states); the final states are the same on
    every rank."""
    import torch.distributed as dist
    rank = dist.get_rank(group)
    o, Bs, c, As = segment_transitions(q, k, v, g, beta, BT=BT, scale=scale, qk_l2norm=qk_l2norm)
    A_all, B_all = gather_transitions(As, Bs, group)
    start, final = B.gdn_cp_combine(A_all, B_all, o, c, rank, initial_state=initial_state)
    return o, final, start
