"""Parity where the data's dynamic range, not its shape, is the hard part.

* A sequence with a loud stretch followed by a quiet one: v times 10^3 over its first
  four chunks, then a forced reset (g = -20) on one token, then ordinary v.  The
  tensor-core path carries its fp16 intermediates with one power-of-two data scale per
  sequence, set by the loud stretch, so the quiet stretch's state and Delta sit 10^3
  below the scale's top.  Each stretch is checked against its own RMS, so that the loud
  stretch cannot hide an error in the quiet one.
* The output epilogue at eps = 1e-3, the RMSNorm epsilon the Qwen3-next page (section
  4.2) gives for bf16, on ordinary rows and on rows whose mean square is near eps (v
  scaled by 0.03), where eps is no longer negligible.
"""
import numpy as np
import pytest

from gated_deltanet_sequence_delta_b200 import inputs as I
from harness import TOL, assert_close, gpu_gates, gpu_prefill, oracle_prefill, to_dev, to_np

pytestmark = pytest.mark.gpu


def _loud_then_quiet(B, T, HK, HV, seed, loud_tokens, reset_token, gain, cu=None):
    inp = I.make_prefill(B, T, HK, HV, 128, 128, io_dtype=I.BF16, seed=seed, h0_std=0.02, cu_seqlens=cu)
    v = inp.v.f32().copy()
    v[:, :loud_tokens] *= gain
    inp.v = I.Tensor(I.f32_to_bf16_bits(v), I.BF16)
    mask = np.zeros(B * T, dtype=bool)
    mask.reshape(B, T)[:, reset_token] = True
    inp.g_reset = mask
    inp.name = f"loud x{gain:g} then quiet"
    return inp


@pytest.mark.parametrize("gain", [1e3, pytest.param(1e4, marks=pytest.mark.xfail(
    strict=True, reason="one fp16 data scale per sequence: a stretch 10^4 louder than the rest leaves "
                        "the quiet stretch's state and Delta too close to the fp16 subnormals"))])
@pytest.mark.parametrize("groups", [(2, 4), (4, 4)])
def test_loud_stretch_then_quiet_stretch(groups, gain):
    HK, HV = groups
    T, loud, reset = 768, 256, 300
    inp = _loud_then_quiet(2, T, HK, HV, 321, loud, reset, gain)
    o, hT, _, _ = gpu_prefill(inp)
    o_ref, h_ref = oracle_prefill(inp)
    og = to_np(o)
    tol = TOL[I.BF16]
    for name, sl in (("loud", slice(0, loud)), ("decaying", slice(loud, reset)), ("quiet", slice(reset, T))):
        assert_close(og[:, sl], o_ref[:, sl], tol, f"{inp.name}: o over the {name} stretch", out_bf16=True)
    assert_close(to_np(hT), h_ref, tol, f"{inp.name}: final state")


def test_loud_sequence_packed_before_quiet_one():
    """Packed: a loud sequence (v x 10^3) and then a quiet one; each sequence has its own
    data scale, so the quiet one must be as exact as on its own."""
    lens = [300, 257]
    cu = I.cu_from_lengths(lens)
    inp = I.make_prefill(1, int(cu[-1]), 2, 4, 128, 128, io_dtype=I.BF16, seed=322, h0_std=0.02, cu_seqlens=cu)
    v = inp.v.f32().copy()
    v[:, :300] *= 1e3
    inp.v = I.Tensor(I.f32_to_bf16_bits(v), I.BF16)
    o, hT, _, _ = gpu_prefill(inp)
    o_ref, h_ref = oracle_prefill(inp)
    og, hg = to_np(o), to_np(hT)
    tol = TOL[I.BF16]
    assert_close(og[:, :300], o_ref[:, :300], tol, "packed loud sequence: o", out_bf16=True)
    assert_close(og[:, 300:], o_ref[:, 300:], tol, "packed quiet sequence: o", out_bf16=True)
    assert_close(hg[0], h_ref[0], tol, "packed loud sequence: state")
    assert_close(hg[1], h_ref[1], tol, "packed quiet sequence: state")


@pytest.mark.parametrize("v_gain", [1.0, 0.03])
def test_outgate_eps_1e3(v_gain):
    import oracle
    import gated_deltanet_sequence_delta_b200 as G
    eps = 1e-3
    inp = I.make_prefill(2, 333, 2, 4, 128, 128, io_dtype=I.BF16, seed=323, h0_std=0.05 * v_gain)
    if v_gain != 1.0:
        inp.v = I.Tensor(I.f32_to_bf16_bits(inp.v.f32() * np.float32(v_gain)), I.BF16)
    n_tok = inp.B * inp.T
    z, w = I.outgate_inputs(n_tok, inp.HV, inp.Dv, inp.io_dtype, 324)
    g, beta = gpu_gates(inp)
    zd = to_dev(z).view(inp.B, inp.T, inp.HV, inp.Dv)
    o, hT = G.gdn_chunk_prefill_outgate(to_dev(inp.q), to_dev(inp.k), to_dev(inp.v), g, beta, zd, to_dev(w), eps,
                                        initial_state=to_dev(inp.h0), BT=inp.BT)
    o_core, h_ref = oracle_prefill(inp)
    ms = float(np.mean(o_core * o_core))
    o_ref = oracle.out_gate(o_core, z.f64().reshape(o_core.shape), w.astype(np.float64), eps=eps)
    tol = TOL[I.BF16]
    assert_close(to_np(o), o_ref, tol, f"gated output, eps 1e-3, mean(o^2) {ms:.2e}", out_bf16=True)
    assert_close(to_np(hT), h_ref, tol, "gated output, eps 1e-3: final state")
    if v_gain != 1.0:
        # the case is only meaningful if eps moves the result: the epilogue with eps = 1e-6
        # must differ from it by more than the tolerance
        o_small = oracle.out_gate(o_core, z.f64().reshape(o_core.shape), w.astype(np.float64), eps=1e-6)
        rms = float(np.sqrt(np.mean(o_ref * o_ref)))
        assert np.max(np.abs(o_small - o_ref)) > 10 * tol * rms
