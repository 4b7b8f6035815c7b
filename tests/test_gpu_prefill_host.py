"""gdn_chunk_prefill_host: gates + chunked prefill for host buffers, streamed through the
GPU in pieces.  Checked against the oracle (the same bound as every prefill), against the
device-buffer path (a single piece is bit-identical; several pieces differ only by the
per-piece scale of the fp16 intermediates), and for slot reuse across calls."""
import numpy as np
import pytest

from gated_deltanet_sequence_delta_b200 import inputs as I
from harness import TOL, assert_close, gpu_prefill, oracle_prefill, to_dev, to_np

pytestmark = pytest.mark.gpu


def _host(t):
    """Pinned CPU torch tensor of an inputs.Tensor or array."""
    return to_dev(t, device="cpu").contiguous().pin_memory()


def _run_host(inp, piece_tokens, with_h0=True):
    import gated_deltanet_sequence_delta_b200 as G
    import torch
    a, b = _host(inp.a.reshape(inp.B, inp.T, inp.HV)), _host(inp.b.reshape(inp.B, inp.T, inp.HV))
    h0 = _host(inp.h0) if (with_h0 and inp.h0 is not None) else None
    o, hT = G.gdn_chunk_prefill_host(_host(inp.q), _host(inp.k), _host(inp.v), a, b, _host(inp.A_log),
                                     _host(inp.dt_bias), initial_state=h0, BT=inp.BT, scale=inp.scale,
                                     qk_l2norm=inp.l2norm, piece_tokens=piece_tokens)
    torch.cuda.current_stream().synchronize()
    return o, hT


@pytest.mark.parametrize("io,T,piece", [(I.BF16, 1000, 256), (I.BF16, 700, 64), (I.F32, 333, 128)])
def test_host_pipeline_matches_oracle(io, T, piece):
    inp = I.make_prefill(2, T, 2, 4, 128, 128, io_dtype=io, seed=41, h0_std=0.05)
    o, hT = _run_host(inp, piece)
    o_ref, h_ref = oracle_prefill(inp)
    tol = TOL[io]
    assert_close(to_np(o), o_ref, tol, "host pipeline: o", out_bf16=io == I.BF16)
    assert_close(to_np(hT), h_ref, tol, "host pipeline: final state")


def test_host_pipeline_single_piece_is_the_device_path():
    import torch
    inp = I.make_prefill(1, 640, 2, 4, 128, 128, io_dtype=I.BF16, seed=43, h0_std=0.05)
    o_h, h_h = _run_host(inp, 4096)
    o_d, h_d, _, _ = gpu_prefill(inp)
    assert torch.equal(o_h, o_d.cpu()) and torch.equal(h_h, h_d.cpu())


def test_host_pipeline_pieces_close_to_device_path():
    inp = I.make_prefill(1, 2048, 2, 4, 128, 128, io_dtype=I.BF16, seed=44, h0_std=0.05)
    o_h, h_h = _run_host(inp, 512)
    o_d, h_d, _, _ = gpu_prefill(inp)
    # the two differ only by the fp16 rounding of intermediates under different scales
    assert_close(to_np(o_h), to_np(o_d), 5e-3, "pieces vs one call: o", out_bf16=True)
    assert_close(to_np(h_h), to_np(h_d), 5e-3, "pieces vs one call: state")


def test_host_pipeline_back_to_back_calls_and_empty_sequence():
    import gated_deltanet_sequence_delta_b200 as G
    import torch
    inp1 = I.make_prefill(1, 900, 2, 2, 128, 128, io_dtype=I.BF16, seed=45, h0_std=0.05)
    inp2 = I.make_prefill(1, 500, 2, 2, 128, 128, io_dtype=I.BF16, seed=46)
    # enqueue both before synchronising: the second call reuses the first call's slots
    a1, b1 = _host(inp1.a.reshape(1, 900, 2)), _host(inp1.b.reshape(1, 900, 2))
    a2, b2 = _host(inp2.a.reshape(1, 500, 2)), _host(inp2.b.reshape(1, 500, 2))
    r1 = G.gdn_chunk_prefill_host(_host(inp1.q), _host(inp1.k), _host(inp1.v), a1, b1, _host(inp1.A_log),
                                  _host(inp1.dt_bias), initial_state=_host(inp1.h0), piece_tokens=128)
    r2 = G.gdn_chunk_prefill_host(_host(inp2.q), _host(inp2.k), _host(inp2.v), a2, b2, _host(inp2.A_log),
                                  _host(inp2.dt_bias), piece_tokens=192)
    torch.cuda.current_stream().synchronize()
    for inp, (o, hT) in ((inp1, r1), (inp2, r2)):
        o_ref, h_ref = oracle_prefill(inp)
        assert_close(to_np(o), o_ref, TOL[I.BF16], f"{inp.seed}: o", out_bf16=True)
        assert_close(to_np(hT), h_ref, TOL[I.BF16], f"{inp.seed}: state")
    # T = 0: the final state is the initial state
    inp0 = I.make_prefill(1, 64, 2, 2, 128, 128, io_dtype=I.BF16, seed=47, h0_std=0.05)
    empty = lambda *s: torch.empty(s, dtype=torch.bfloat16).pin_memory()
    o0, h0 = G.gdn_chunk_prefill_host(empty(1, 0, 2, 128), empty(1, 0, 2, 128), empty(1, 0, 2, 128),
                                      torch.empty(1, 0, 2).pin_memory(), torch.empty(1, 0, 2).pin_memory(),
                                      _host(inp0.A_log), _host(inp0.dt_bias), initial_state=_host(inp0.h0))
    torch.cuda.current_stream().synchronize()
    assert torch.equal(h0, _host(inp0.h0))
