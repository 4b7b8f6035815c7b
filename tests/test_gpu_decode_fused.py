"""gdn_decode_step_fused on the GPU: raw projections through the kernel-4 causal
convolution (identity or SiLU), the gates and the decode step in one kernel, against the
oracle's convolution, gates and one-token recurrence, with the convolution state and the
recurrent state carried over several steps."""
import numpy as np
import pytest

from gated_deltanet_sequence_delta_b200 import inputs as I
from harness import TOL, assert_close, to_dev, to_np

pytestmark = pytest.mark.gpu


def _run(setup, n_steps, act, eps=None):
    """eps given: the output epilogue too (gdn_decode_step_fused_outgate), against the oracle's
    out_gate on the oracle's core output."""
    import torch
    import oracle
    import gated_deltanet_sequence_delta_b200 as G
    bs = setup.base
    B, HK, HV, D = bs.B, bs.HK, bs.HV, bs.Dk
    state = to_dev(bs.state0.copy())
    # the library's convolution state is tap-major [B, 3, C]; the oracle's is [B, C, 3]
    cs = [to_dev(np.ascontiguousarray(setup.conv_state0.transpose(0, 2, 1))),
          torch.empty((B, 3, setup.C), dtype=torch.float32, device="cuda")]
    w = to_dev(setup.conv_w)
    A_log, dt_bias = to_dev(bs.A_log), to_dev(bs.dt_bias)
    ref_state = bs.state0.astype(np.float64)
    ref_cs = setup.conv_state0.astype(np.float64)
    tol = TOL[bs.io_dtype]
    nw = setup.out_w()
    for s in range(n_steps):
        x, a, b = setup.step(s)
        og = None
        if eps is not None:
            z = setup.out_z(s)
            og = (to_dev(z), to_dev(nw), eps)
        o, _ = G.gdn_decode_step_fused(to_dev(x), w, cs[s % 2], to_dev(a), to_dev(b), A_log, dt_bias, state,
                                       HK=HK, conv_act=act, scale=bs.scale, conv_state_out=cs[(s + 1) % 2],
                                       outgate=og)
        # oracle: convolution, gates, one-token recurrence
        y, ref_cs = oracle.conv(x.f64()[:, None, :], setup.conv_w, ref_cs, act)
        y = y[:, 0]
        q = y[:, :HK * D].reshape(B, HK, D)
        k = y[:, HK * D:2 * HK * D].reshape(B, HK, D)
        v = y[:, 2 * HK * D:].reshape(B, HV, D)
        g, beta = oracle.gates(a.astype(np.float64), b.astype(np.float64), bs.A_log.astype(np.float64),
                               bs.dt_bias.astype(np.float64))
        o_ref, ref_state = oracle.decode_step(q, k, v, g, beta, ref_state, scale=bs.scale, l2norm=bs.l2norm)
        if eps is not None:
            o_ref = oracle.out_gate(o_ref, z.f64(), nw.astype(np.float64), eps=eps)
        what = "fused step" if eps is None else f"fused step with output epilogue (eps {eps:g})"
        assert_close(to_np(o), o_ref, tol, f"{what} {s}: o", out_bf16=bs.io_dtype == I.BF16)
        assert_close(to_np(state), ref_state, tol, f"fused step {s}: state")
        # the convolution state holds exactly the three newest inputs
        np.testing.assert_array_equal(to_np(cs[(s + 1) % 2]).transpose(0, 2, 1), ref_cs,
                                      err_msg=f"step {s}: conv state")
    assert G.gdn_decode_status() == 0


@pytest.mark.parametrize("io,act", [(I.BF16, 1), (I.BF16, 0), (I.F32, 1)])
def test_fused_decode_small(io, act):
    _run(I.decode_fused(B=3, H=4, D=128, io_dtype=io, seed=71, HK=2), 6, act)


def test_fused_decode_workload_shape():
    """B=64, H=32, d=128, bf16, SiLU: four steps on every (sequence, head)."""
    _run(I.decode_fused(seed=72), 4, 1)


@pytest.mark.parametrize("io,eps", [(I.BF16, 1e-6), (I.BF16, 1e-3), (I.F32, 1e-6)])
def test_fused_decode_output_epilogue(io, eps):
    """The decode step from raw projections with the output epilogue (zero-centred RMSNorm
    times 1 + w, sigmoid gate of z) applied before the store, eps 1e-6 and the Qwen3-next
    page's 1e-3."""
    _run(I.decode_fused(B=3, H=4, D=128, io_dtype=io, seed=73, HK=2), 5, 1, eps=eps)


def test_fused_decode_output_epilogue_workload_shape():
    """B=64, H=32, d=128, bf16: four steps with the output epilogue on every (sequence, head)."""
    _run(I.decode_fused(seed=74), 4, 1, eps=1e-6)
