"""A bounded wait that runs out, on the GPU, without any fault: the test hook
gdn_testing_stall makes one CTA of a kernel wait for copies that are never issued (a
flag that nothing sets).  The wait gives up at its limit, the kernel records
GDN_DEVERR_TIMEOUT, lets what it did issue land, frees its tensor memory and returns; the
status call reports the timeout, the context stays usable, and the next call on the same
process is correct against the oracle."""
import numpy as np
import pytest

from gated_deltanet_sequence_delta_b200 import inputs as I
from harness import check_prefill, gpu_gates, to_dev
from test_gpu_decode import _run_steps

pytestmark = pytest.mark.gpu

DEVERR_TIMEOUT = 2


def test_decode_wait_runs_out_then_recovers():
    import torch
    import gated_deltanet_sequence_delta_b200 as G
    setup = I.decode(B=4, H=8, D=128, io_dtype=I.BF16, seed=331)
    q, k, v, a, b = setup.step(0)
    state = to_dev(setup.state0.copy())
    g, beta = G.gdn_gates(to_dev(a), to_dev(b), to_dev(setup.A_log), to_dev(setup.dt_bias))
    assert G.gdn_decode_status() == 0
    G.testing_stall(G.STALL_DECODE)
    try:
        G.gdn_decode_step(to_dev(q), to_dev(k), to_dev(v), g, beta, state)
        torch.cuda.synchronize()   # the call returned and the launch finished
    finally:
        G.testing_stall(G.STALL_NONE)
    assert G.gdn_decode_status() == DEVERR_TIMEOUT
    assert G.gdn_decode_status() == 0   # the status call cleared the word
    _run_steps(setup, 4)                # the same process, a fresh state: correct again
    assert G.gdn_decode_status() == 0


def test_prefill_prep_wait_runs_out_then_recovers():
    import torch
    import gated_deltanet_sequence_delta_b200 as G
    inp = I.make_prefill(1, 300, 2, 4, 128, 128, io_dtype=I.BF16, seed=332, h0_std=0.05)
    g, beta = gpu_gates(inp)
    need = G.prefill_workspace_bytes(300, 1, 2, 4, 128, 128, 64, 1)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    G.testing_stall(G.STALL_PREFILL_PREP)
    try:
        G.gdn_chunk_prefill(to_dev(inp.q), to_dev(inp.k), to_dev(inp.v), g, beta, initial_state=to_dev(inp.h0),
                            workspace=ws)
        torch.cuda.synchronize()
    finally:
        G.testing_stall(G.STALL_NONE)
    assert G.gdn_chunk_prefill_status(ws) == DEVERR_TIMEOUT
    check_prefill(inp)                  # the same process: correct again


def test_stall_hook_rejects_unknown_site():
    import gated_deltanet_sequence_delta_b200 as G
    with pytest.raises(G.GDNError):
        G.testing_stall(7)
