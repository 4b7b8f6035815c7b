"""gdn_chunk_prefill_static_ws: the prefill entry point for callers that may not
allocate device memory (its scratch is a fixed device array inside the library).
Its output must match gdn_chunk_prefill's on the same inputs, within the parity
tolerance the other GPU tests use, on consecutive calls that reuse the shared
scratch.  Called through the C ABI directly.  This file is collected last so a
failure here leaves every other test already run."""
import ctypes

import numpy as np
import pytest

from gated_deltanet_sequence_delta_b200 import inputs as I
from harness import TOL, assert_close, gpu_gates, to_dev, to_np

pytestmark = pytest.mark.gpu


def _static_fn():
    from gated_deltanet_sequence_delta_b200 import binding
    L = binding.lib()
    f = L.gdn_chunk_prefill_static_ws
    vp, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
    f.argtypes = [vp, vp, vp, ctypes.c_int, vp, vp, vp, vp, i32, i64, i32, i32, i32, i32, i32, i32,
                  ctypes.c_float, i32, vp, vp, vp]
    f.restype = ctypes.c_int
    return f


def _call_static(f, inp, g, beta):
    import torch
    q, k, v = to_dev(inp.q), to_dev(inp.k), to_dev(inp.v)
    h0 = None if inp.h0 is None else to_dev(inp.h0)
    cu = None if inp.cu_seqlens is None else to_dev(inp.cu_seqlens)
    N = inp.n_seqs
    o = torch.full((inp.B, inp.T, inp.HV, inp.Dv), float("nan"), dtype=q.dtype, device="cuda")
    hT = torch.full((N, inp.HV, inp.Dk, inp.Dv), float("nan"), device="cuda")
    dt = 1 if inp.io_dtype == I.BF16 else 0
    ptr = lambda t: None if t is None else t.data_ptr()
    st = f(ptr(q), ptr(k), ptr(v), dt, ptr(g), ptr(beta), ptr(h0), ptr(cu), inp.B, inp.T, N,
           inp.HK, inp.HV, inp.Dk, inp.Dv, inp.BT, inp.scale, int(inp.l2norm), ptr(o), ptr(hT),
           torch.cuda.current_stream().cuda_stream)
    assert st == 0, f"gdn_chunk_prefill_static_ws returned {st}"
    torch.cuda.synchronize()
    return o, hT


def test_static_scratch_matches_workspace_entry_point():
    import gated_deltanet_sequence_delta_b200 as G
    f = _static_fn()
    cases = [
        I.make_prefill(1, 700, 2, 4, 128, 128, io_dtype=I.BF16, seed=41, h0_std=0.05),
        I.make_prefill(1, 300, 2, 4, 128, 128, io_dtype=I.BF16, seed=42, h0_std=0.02,
                       cu_seqlens=I.cu_from_lengths([100, 1, 199])),
    ]
    for inp in cases:          # two calls in a row, different shapes, shared scratch
        g, beta = gpu_gates(inp)
        o_s, h_s = _call_static(f, inp, g, beta)
        o_w, h_w = G.gdn_chunk_prefill(
            to_dev(inp.q), to_dev(inp.k), to_dev(inp.v), g, beta,
            initial_state=None if inp.h0 is None else to_dev(inp.h0),
            cu_seqlens=None if inp.cu_seqlens is None else to_dev(inp.cu_seqlens), BT=inp.BT)
        tol = TOL[inp.io_dtype]
        assert_close(to_np(o_s), to_np(o_w), tol, "static scratch: o", out_bf16=True)
        assert_close(to_np(h_s), to_np(h_w), tol, "static scratch: final state")


def test_static_scratch_rejects_oversized_problem():
    from gated_deltanet_sequence_delta_b200 import binding
    f = _static_fn()
    A = 0x7f0000000000           # never dereferenced: the call must fail before any launch
    MB = 1 << 20
    T = 1 << 20                  # needs far more than the fixed scratch
    st = f(A, A + 512 * MB, A + 1024 * MB, 1, A + 2048 * MB, A + 2304 * MB, None, None, 1, T, 1,
           16, 32, 128, 128, 64, 1.0, 1, A + 4096 * MB, A + 8192 * MB, None)
    assert st == 6, binding.lib().gdn_status_string(st)
