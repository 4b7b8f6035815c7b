"""Shared test harness: run a seeded workload through the CUDA library (via the C
ABI binding) and through the CPU oracle, and compare them.

Tolerances (the bar every GPU parity test uses):
  * bf16 q/k/v with fp32 state: max |x_gpu - x_ref| <= 2e-2 * RMS(x_ref)
  * fp32 mode:                  max |x_gpu - x_ref| <= 1e-4 * RMS(x_ref)
applied to the outputs o and to the final states, separately.

bf16 outputs.  Rounding the exact result to bf16 (round to nearest) moves an
element x by up to 2^-8 |x|.  In these workloads max|o| is 8-10 times RMS(o), so
that rounding alone can exceed 2e-2 * RMS(o) even for a perfect kernel.  For a
bf16 output the bound is therefore applied to the arithmetic:
    |o_gpu - o_ref| <= tol * RMS(o_ref) + 2^-8 |o_ref|      (elementwise)
the second term being the representation bound of the output format.  fp32
outputs and the (always fp32) final states take the bound as stated.
"""
from __future__ import annotations

import numpy as np

from gated_deltanet_sequence_delta_b200 import inputs as I

TOL = {I.BF16: 2e-2, I.F32: 1e-4}


def rms_err(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    rms = float(np.sqrt(np.mean(ref * ref))) if ref.size else 0.0
    err = float(np.max(np.abs(got - ref))) if ref.size else 0.0
    assert np.all(np.isfinite(got)), "non-finite values in GPU result"
    return err, rms


BF16_REP = 2.0 ** -8   # relative representation bound of round-to-nearest bf16


# Every comparison made through assert_close, for the run's parity report (printed in the
# pytest terminal summary): (what, max|err| / RMS(ref), the part of it beyond the output's
# own bf16 rounding, RMS(err) / RMS(ref), tolerance).  RMS(err) shows a systematic bias that
# the per-element bound could hide.
PARITY_LOG: list = []


def assert_close(got, ref, tol, what="", out_bf16=False):
    """max|got - ref| <= tol * RMS(ref) (plus 2^-8 |ref| per element when ``got``
    was rounded to bf16).  Returns the arithmetic error relative to RMS(ref)."""
    err, rms = rms_err(got, ref)
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if ref.size == 0:
        return 0.0
    d = got - ref
    excess = np.abs(d) - (BF16_REP * np.abs(ref) if out_bf16 else 0.0)
    arith = float(max(np.max(excess), 0.0))
    den = max(rms, 1e-30)
    PARITY_LOG.append((what, err / den, arith / den, float(np.sqrt(np.mean(d * d))) / den, tol))
    assert arith <= tol * den, (
        f"{what}: max|err| {err:.3e} (beyond output rounding {arith:.3e}) > {tol:g} * RMS {rms:.3e}")
    return arith / den


# ---------------------------------------------------------------------------
# device side
# ---------------------------------------------------------------------------
def to_dev(t, device="cuda"):
    import torch
    if isinstance(t, I.Tensor):
        if t.dtype == I.BF16:
            return torch.from_numpy(np.ascontiguousarray(t.data).view(np.int16)).view(torch.bfloat16).to(device)
        return torch.from_numpy(np.ascontiguousarray(t.data)).to(device)
    return torch.from_numpy(np.ascontiguousarray(t)).to(device)


def to_np(x):
    import torch
    return x.detach().to(torch.float64).cpu().numpy()


def gpu_gates(inp):
    import gated_deltanet_sequence_delta_b200 as G
    a = to_dev(inp.a)
    b = to_dev(inp.b)
    g, beta = G.gdn_gates(a, b, to_dev(inp.A_log), to_dev(inp.dt_bias))
    if inp.g_reset is not None:
        import torch
        mask = to_dev(inp.g_reset).view(inp.B, inp.T)
        g[mask] = -20.0
    return g, beta


def gpu_prefill(inp, BT=None, with_state=True):
    """Gates then chunked prefill on the GPU; returns device tensors (o, hT, g, beta)."""
    import gated_deltanet_sequence_delta_b200 as G
    g, beta = gpu_gates(inp)
    o, hT = G.gdn_chunk_prefill(
        to_dev(inp.q), to_dev(inp.k), to_dev(inp.v), g, beta,
        initial_state=None if inp.h0 is None else to_dev(inp.h0),
        cu_seqlens=None if inp.cu_seqlens is None else to_dev(inp.cu_seqlens),
        BT=BT or inp.BT, scale=inp.scale, qk_l2norm=inp.l2norm, output_final_state=with_state)
    return o, hT, g, beta


# ---------------------------------------------------------------------------
# oracle side
# ---------------------------------------------------------------------------
def oracle_gates(inp):
    import oracle
    g, beta = oracle.gates(inp.a.astype(np.float64), inp.b.astype(np.float64),
                           inp.A_log.astype(np.float64), inp.dt_bias.astype(np.float64))
    if inp.g_reset is not None:
        g.reshape(-1, inp.HV)[inp.g_reset] = -20.0
    return g, beta


def oracle_prefill(inp, heads=None):
    """Oracle o [B, T, len(heads), Dv] and hT [N, len(heads), Dk, Dv] for the given
    value heads (all heads by default)."""
    import oracle
    g, beta = oracle_gates(inp)
    cu = None if inp.cu_seqlens is None else inp.cu_seqlens.astype(np.int64)
    if heads is None or list(heads) == list(range(inp.HV)):
        # every head in one call: the oracle spreads (sequence, head) pairs over the host cores
        q, k, v = inp.q.f64(), inp.k.f64(), inp.v.f64()
        h0 = None if inp.h0 is None else inp.h0.astype(np.float64)
        if cu is None:
            return oracle.recurrence(q, k, v, g, beta, h0=h0, scale=inp.scale, l2norm=inp.l2norm)
        o, hT = oracle.recurrence(q[0], k[0], v[0], g[0], beta[0], h0=h0, cu_seqlens=cu, scale=inp.scale,
                                  l2norm=inp.l2norm)
        return o[None], hT
    # selected heads: each value head with its own copy of its q/k head, all in one call
    heads = list(heads)
    G_ = inp.HV // inp.HK
    kh = [h // G_ for h in heads]
    q = inp.q.f64((slice(None), slice(None), kh))
    k = inp.k.f64((slice(None), slice(None), kh))
    v = inp.v.f64((slice(None), slice(None), heads))
    h0 = None if inp.h0 is None else inp.h0[:, heads].astype(np.float64)
    gs, bs = g[:, :, heads], beta[:, :, heads]
    if cu is None:
        return oracle.recurrence(q, k, v, gs, bs, h0=h0, scale=inp.scale, l2norm=inp.l2norm)
    o, hT = oracle.recurrence(q[0], k[0], v[0], gs[0], bs[0], h0=h0, cu_seqlens=cu, scale=inp.scale,
                              l2norm=inp.l2norm)
    return o[None], hT


def check_prefill(inp, heads=None, BT=None, tol=None):
    """Run both sides and assert parity on o and the final state; returns the
    relative errors (err / RMS) for o and state."""
    tol = TOL[inp.io_dtype] if tol is None else tol
    o, hT, _, _ = gpu_prefill(inp, BT=BT)
    heads_l = list(range(inp.HV)) if heads is None else list(heads)
    o_ref, h_ref = oracle_prefill(inp, heads_l)
    o_g = to_np(o[:, :, heads_l])
    h_g = to_np(hT[:, heads_l])
    eo = assert_close(o_g, o_ref, tol, f"{inp.name}: o", out_bf16=inp.io_dtype == I.BF16)
    eh = assert_close(h_g, h_ref, tol, f"{inp.name}: final state")
    return eo, eh
