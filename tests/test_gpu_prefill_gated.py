"""gdn_chunk_prefill_gated: the chunked prefill with the gate prologue (the gate code of the
Qwen3-next page, section 2.1) formed inside the chunk-local kernel.  It must be bit for bit
gdn_gates followed by gdn_chunk_prefill (same formula, same arithmetic), on dense and packed
layouts, bf16 and fp32 gate inputs and every grouped-head ratio the tensor-core path takes;
and it is checked against the oracle's gates and recurrence directly."""
import numpy as np
import pytest

from gated_deltanet_sequence_delta_b200 import inputs as I
from harness import TOL, assert_close, oracle_prefill, to_dev, to_np

pytestmark = pytest.mark.gpu


def _both(inp, ab_bf16):
    import torch
    import gated_deltanet_sequence_delta_b200 as G
    q, k, v = to_dev(inp.q), to_dev(inp.k), to_dev(inp.v)
    a, b = to_dev(inp.a), to_dev(inp.b)
    if ab_bf16:
        a, b = a.to(torch.bfloat16), b.to(torch.bfloat16)
    A_log, dt_bias = to_dev(inp.A_log), to_dev(inp.dt_bias)
    h0 = None if inp.h0 is None else to_dev(inp.h0)
    cu = None if inp.cu_seqlens is None else to_dev(inp.cu_seqlens)
    g, beta = G.gdn_gates(a, b, A_log, dt_bias)
    o1, h1 = G.gdn_chunk_prefill(q, k, v, g, beta, initial_state=h0, cu_seqlens=cu, scale=inp.scale,
                                 qk_l2norm=inp.l2norm)
    o2, h2 = G.gdn_chunk_prefill_gated(q, k, v, a, b, A_log, dt_bias, initial_state=h0, cu_seqlens=cu,
                                       scale=inp.scale, qk_l2norm=inp.l2norm)
    return (o1, h1), (o2, h2)


@pytest.mark.parametrize("ab_bf16", [False, True])
@pytest.mark.parametrize("groups", [(2, 2), (2, 4), (2, 8)])
def test_gated_equals_gates_then_prefill_dense(groups, ab_bf16):
    import torch
    HK, HV = groups
    inp = I.make_prefill(2, 333, HK, HV, 128, 128, io_dtype=I.BF16, seed=401, h0_std=0.05)
    (o1, h1), (o2, h2) = _both(inp, ab_bf16)
    assert torch.equal(o1, o2) and torch.equal(h1, h2)


def test_gated_equals_gates_then_prefill_packed():
    import torch
    lens = [1, 64, 0, 191, 70]
    inp = I.make_prefill(1, int(sum(lens)), 2, 4, 128, 128, io_dtype=I.BF16, seed=402, h0_std=0.05,
                         cu_seqlens=I.cu_from_lengths(lens), scale=0.5, qk_norm=(0.1, 10.0))
    (o1, h1), (o2, h2) = _both(inp, False)
    assert torch.equal(o1, o2) and torch.equal(h1, h2)


def test_gated_vs_oracle_long_workload_heads():
    """The long workload (T=32768, HK=16, HV=32) through the fused-gate entry point, against
    the oracle's own gates and recurrence on eight value heads."""
    inp = I.long_prefill()
    _, (o, hT) = _both(inp, False)
    heads = [0, 1, 7, 12, 19, 24, 30, 31]
    o_ref, h_ref = oracle_prefill(inp, heads)
    tol = TOL[I.BF16]
    assert_close(to_np(o[:, :, heads]), o_ref, tol, "gated prefill, long workload: o", out_bf16=True)
    assert_close(to_np(hT[:, heads]), h_ref, tol, "gated prefill, long workload: final state")


def test_gated_unsupported_shapes_rejected():
    import torch
    import gated_deltanet_sequence_delta_b200 as G
    inp = I.make_prefill(1, 100, 2, 4, 64, 64, io_dtype=I.BF16, seed=403)
    with pytest.raises(G.GDNError) as e:
        G.gdn_chunk_prefill_gated(to_dev(inp.q), to_dev(inp.k), to_dev(inp.v), to_dev(inp.a), to_dev(inp.b),
                                  to_dev(inp.A_log), to_dev(inp.dt_bias))
    assert e.value.status == 4
