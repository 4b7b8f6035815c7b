"""Context-parallel prefill on one GPU with the ranks emulated one after another (no rank
waits on another: the all-gather is a host-side stack): every segment through
context_parallel.segment_transitions (two gdn_chunk_prefill runs), then gdn_cp_combine
per segment; the outputs and final states against the oracle over the whole sequences."""
import numpy as np
import pytest

from gated_deltanet_sequence_delta_b200 import inputs as I
from harness import TOL, assert_close, gpu_gates, oracle_gates, to_dev, to_np

pytestmark = pytest.mark.gpu


def _run(io, R, T_seg, N, HK, HV, seed):
    import torch
    import oracle
    import gated_deltanet_sequence_delta_b200 as G
    from gated_deltanet_sequence_delta_b200 import context_parallel as CP
    T = R * T_seg
    inp = I.make_prefill(N, T, HK, HV, 128, 128, io_dtype=io, seed=seed, h0_std=0.02)
    q, k, v = to_dev(inp.q).view(N, T, HK, 128), to_dev(inp.k).view(N, T, HK, 128), to_dev(inp.v).view(N, T, HV, 128)
    g, beta = gpu_gates(inp)
    g, beta = g.view(N, T, HV), beta.view(N, T, HV)
    h0 = to_dev(inp.h0)
    parts = []
    for r in range(R):
        sl = slice(r * T_seg, (r + 1) * T_seg)
        seg = [t[:, sl].contiguous() for t in (q, k, v, g, beta)]
        parts.append(CP.segment_transitions(*seg, BT=inp.BT))
    A_all = torch.stack([p[3] for p in parts])
    B_all = torch.stack([p[1] for p in parts])
    outs, finals, starts = [], [], []
    for r in range(R):
        o, _, c, _ = parts[r]
        start, final = G.gdn_cp_combine(A_all, B_all, o, c, r, initial_state=h0)
        outs.append(o)
        finals.append(final)
        starts.append(start)
    o_cp = torch.cat(outs, dim=1)
    # oracle over the whole sequences, on the same rounded inputs, with its own gates
    g_ref, b_ref = oracle_gates(inp)
    o_ref, h_ref = oracle.recurrence(inp.q.f64().reshape(N, T, HK, 128), inp.k.f64().reshape(N, T, HK, 128),
                                     inp.v.f64().reshape(N, T, HV, 128), g_ref, b_ref,
                                     h0=inp.h0.astype(np.float64))
    tol = TOL[io]
    assert_close(to_np(o_cp), o_ref, tol, f"context-parallel o ({io})", out_bf16=io == I.BF16)
    for r in range(R):
        assert_close(to_np(finals[r]), h_ref, tol, f"final state seen by rank {r}")
    # every rank's start state is the state at its segment's first token
    _, h_mid = oracle.recurrence(inp.q.f64().reshape(N, T, HK, 128)[:, :T_seg * 2],
                                 inp.k.f64().reshape(N, T, HK, 128)[:, :T_seg * 2],
                                 inp.v.f64().reshape(N, T, HV, 128)[:, :T_seg * 2], g_ref[:, :T_seg * 2],
                                 b_ref[:, :T_seg * 2], h0=inp.h0.astype(np.float64))
    assert_close(to_np(starts[2]), h_mid, tol, "start state of segment 2")
    assert G.gdn_cp_status() == 0


@pytest.mark.parametrize("io", [I.BF16, I.F32])
def test_cp_four_segments_gqa(io):
    """Four ragged segments of 200 tokens (not whole chunks), one sequence, HK=2, HV=4."""
    _run(io, 4, 200, 1, 2, 4, 91)


def test_cp_two_sequences():
    """Two dense sequences, four segments of 256 tokens each, HK=HV=4, bf16."""
    _run(I.BF16, 4, 256, 2, 4, 4, 92)


def test_cp_segment_matches_two_prefills():
    """gdn_cp_segment (one chunk-local stage, two carries) against gdn_chunk_prefill from
    zero (o, final state: bit for bit) and gdn_chunk_prefill with v = 0 from the identity
    (c, A: to the usual tolerance; the fp16 data scale of the two carries may differ)."""
    import torch
    import gated_deltanet_sequence_delta_b200 as G
    inp = I.make_prefill(2, 300, 2, 4, 128, 128, io_dtype=I.BF16, seed=93)
    q, k, v = to_dev(inp.q).view(2, 300, 2, 128), to_dev(inp.k).view(2, 300, 2, 128), to_dev(inp.v).view(2, 300, 4, 128)
    g, beta = gpu_gates(inp)
    g, beta = g.view(2, 300, 4), beta.view(2, 300, 4)
    o, hT, c, A = G.gdn_cp_segment(q, k, v, g, beta)
    o2, hT2 = G.gdn_chunk_prefill(q, k, v, g, beta)
    eye = torch.eye(128, dtype=torch.float32, device="cuda").expand(2, 4, 128, 128).contiguous()
    c2, A2 = G.gdn_chunk_prefill(q, k, torch.zeros_like(v), g, beta, initial_state=eye)
    assert torch.equal(o, o2) and torch.equal(hT, hT2)
    assert_close(to_np(c), to_np(c2), TOL[I.BF16], "c", out_bf16=True)
    assert_close(to_np(A), to_np(A2), TOL[I.BF16], "A")


def test_cp_product_function_through_a_process_group():
    """context_parallel.cp_chunk_prefill as a user calls it: a real NCCL process group of
    one rank on this GPU, so that gather_transitions runs its all-gathers on CUDA tensors
    and gdn_cp_combine consumes what they return; against the oracle."""
    import datetime
    import oracle
    import torch
    import torch.distributed as dist
    from gated_deltanet_sequence_delta_b200 import context_parallel as CP
    N, T, HK, HV = 2, 300, 2, 4
    inp = I.make_prefill(N, T, HK, HV, 128, 128, io_dtype=I.BF16, seed=94, h0_std=0.02)
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", store=dist.HashStore(), rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60))
    try:
        g, beta = gpu_gates(inp)
        o, final, start = CP.cp_chunk_prefill(to_dev(inp.q), to_dev(inp.k), to_dev(inp.v), g.view(N, T, HV),
                                              beta.view(N, T, HV), initial_state=to_dev(inp.h0))
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    g_ref, b_ref = oracle_gates(inp)
    o_ref, h_ref = oracle.recurrence(inp.q.f64(), inp.k.f64(), inp.v.f64(), g_ref, b_ref,
                                     h0=inp.h0.astype(np.float64))
    tol = TOL[I.BF16]
    assert_close(to_np(o), o_ref, tol, "cp_chunk_prefill, one rank: o", out_bf16=True)
    assert_close(to_np(final), h_ref, tol, "cp_chunk_prefill, one rank: final state")
    # the only segment starts from the initial state
    assert_close(to_np(start), inp.h0.astype(np.float64), 1e-6, "cp_chunk_prefill, one rank: start state")
