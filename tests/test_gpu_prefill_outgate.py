"""gdn_chunk_prefill_outgate on the GPU: the chunked prefill with the output epilogue
(zero-centred RMSNorm over each head's Dv values times 1 + w, sigmoid gate of z) fused
into the output store, where a head's four column slices exchange their partial sums of
squares inside a thread-block cluster.  Checked against the oracle's recurrence followed
by its output epilogue, for dense, packed and full-size inputs."""
import numpy as np
import pytest

from gated_deltanet_sequence_delta_b200 import inputs as I
from harness import TOL, assert_close, gpu_gates, oracle_prefill, to_dev, to_np

pytestmark = pytest.mark.gpu
EPS = 1e-6


def _check(inp, seed):
    import oracle
    import gated_deltanet_sequence_delta_b200 as G
    n_tok = inp.B * inp.T
    z, w = I.outgate_inputs(n_tok, inp.HV, inp.Dv, inp.io_dtype, seed)
    g, beta = gpu_gates(inp)
    zd = to_dev(z).view(inp.B, inp.T, inp.HV, inp.Dv)
    o, hT = G.gdn_chunk_prefill_outgate(
        to_dev(inp.q), to_dev(inp.k), to_dev(inp.v), g, beta, zd, to_dev(w), EPS,
        initial_state=None if inp.h0 is None else to_dev(inp.h0),
        cu_seqlens=None if inp.cu_seqlens is None else to_dev(inp.cu_seqlens),
        BT=inp.BT, scale=inp.scale, qk_l2norm=inp.l2norm)
    o_core, h_ref = oracle_prefill(inp)
    o_ref = oracle.out_gate(o_core, z.f64().reshape(o_core.shape), w.astype(np.float64), eps=EPS)
    tol = TOL[inp.io_dtype]
    eo = assert_close(to_np(o), o_ref, tol, f"{inp.name}: gated output", out_bf16=True)
    eh = assert_close(to_np(hT), h_ref, tol, f"{inp.name}: final state")
    return eo, eh


def test_outgate_dense_ragged():
    _check(I.make_prefill(2, 333, 2, 4, 128, 128, io_dtype=I.BF16, seed=81, h0_std=0.05), 82)


def test_outgate_gqa_group4():
    _check(I.make_prefill(1, 200, 2, 8, 128, 128, io_dtype=I.BF16, seed=87, h0_std=0.05), 88)


def test_outgate_mha_single_chunk_and_tail():
    _check(I.make_prefill(1, 70, 4, 4, 128, 128, io_dtype=I.BF16, seed=83, h0_std=0.05), 84)


def test_outgate_packed_sequences():
    lens = [5, 130, 64, 250]
    cu = I.cu_from_lengths(lens)
    _check(I.make_prefill(1, int(cu[-1]), 2, 4, 128, 128, io_dtype=I.BF16, seed=85, h0_std=0.05,
                          cu_seqlens=cu), 86)


def test_outgate_long_workload_all_heads():
    """T=32768, HK=16, HV=32: the output epilogue on every head."""
    _check(I.long_prefill(), 87)
