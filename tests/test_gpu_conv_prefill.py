"""gdn_conv_prefill on the GPU: the kernel-4 causal convolution over whole sequences, from
raw q | k | v projections to the prefill's q, k, v, against the oracle's convolution
(dense and packed layouts with empty and short sequences, identity and SiLU, with and
without a carried state, bf16 and fp32, head dims 64 and 128); the carried convolution
state is compared bit for bit.  At the long workload's size, sampled windows.  End to end:
raw projections -> convolution -> chunked prefill -> two fused decode steps, against the
oracle run over the whole sequences."""
import numpy as np
import pytest

from gated_deltanet_sequence_delta_b200 import inputs as I
from harness import TOL, assert_close, to_dev, to_np

pytestmark = pytest.mark.gpu

# the convolution is four fp32 products and the activation: far inside this bound, relative
# to RMS(y); bf16 outputs add their own rounding (2^-8 |y|) on top
CONV_TOL = 1e-5


def _tap_major(state):   # oracle [N, C, 3] -> library [N, 3, C]
    return None if state is None else np.ascontiguousarray(state.transpose(0, 2, 1))


def _gpu_conv(x, w, state0, cu, B, T, HK, HV, D, act):
    import gated_deltanet_sequence_delta_b200 as G
    C = w.shape[0]
    xd = to_dev(x).view(B, T, C)
    cs = to_dev(_tap_major(state0)) if state0 is not None else None
    cud = to_dev(np.asarray(cu, dtype=np.int32)) if cu is not None else None
    return G.gdn_conv_prefill(xd, to_dev(w), HK, HV, D, D, conv_state_in=cs, cu_seqlens=cud, conv_act=act)


def _oracle_conv(x64, w, state0, bounds, act):
    """The oracle's convolution per sequence [bounds[n], bounds[n + 1])."""
    import oracle
    C = w.shape[0]
    N = len(bounds) - 1
    y = np.zeros_like(x64)
    st = np.zeros((N, C, 3))
    for n in range(N):
        s, e = int(bounds[n]), int(bounds[n + 1])
        s0 = state0[n:n + 1].astype(np.float64) if state0 is not None else None
        if e > s:
            yy, ss = oracle.conv(x64[None, s:e], w, s0, act)
            y[s:e] = yy[0]
            st[n] = ss[0]
        elif s0 is not None:
            st[n] = s0[0]
    return y, st


def _check(io, act, D, HK, HV, with_state, B=None, T=None, lens=None, seed=0):
    packed = lens is not None
    if packed:
        bounds = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
        B_, T_, N = 1, int(bounds[-1]), len(lens)
    else:
        bounds = np.arange(B + 1, dtype=np.int64) * T
        B_, T_, N = B, T, B
    x, w, st0 = I.conv_prefill_inputs(B_ * T_, N, HK, HV, D, io, seed, with_state)
    q, k, v, cs = _gpu_conv(x, w, st0, bounds if packed else None, B_, T_, HK, HV, D, act)
    n = B_ * T_
    y = np.concatenate([to_np(q).reshape(n, -1), to_np(k).reshape(n, -1), to_np(v).reshape(n, -1)], axis=1)
    y_ref, st_ref = _oracle_conv(x.f64(), w, st0, bounds, act)
    err = assert_close(y, y_ref, CONV_TOL, f"conv y ({io}, act {act})", out_bf16=io == I.BF16)
    np.testing.assert_array_equal(to_np(cs).transpose(0, 2, 1), st_ref, err_msg="conv state")
    import gated_deltanet_sequence_delta_b200 as G
    assert G.gdn_conv_status() == 0
    return err


@pytest.mark.parametrize("io,act,with_state", [(I.BF16, 1, True), (I.BF16, 0, False), (I.F32, 1, True),
                                               (I.F32, 0, False)])
def test_conv_dense(io, act, with_state):
    """Two dense sequences of 70 tokens (ragged against the kernel's 32-token runs)."""
    _check(io, act, 128, 2, 4, with_state, B=2, T=70, seed=81)


@pytest.mark.parametrize("io", [I.BF16, I.F32])
def test_conv_packed_short_and_empty(io):
    """Packed sequences of 0-100 tokens (empty ones first and in the middle; several
    sequence starts inside one 32-token run), head dim 64."""
    _check(io, 1, 64, 2, 4, True, lens=[0, 1, 2, 3, 5, 31, 32, 33, 64, 100, 0, 7], seed=82)


def test_conv_no_state_out():
    """conv_state_out may be omitted."""
    import gated_deltanet_sequence_delta_b200 as G
    x, w, _ = I.conv_prefill_inputs(40, 1, 2, 4, 128, I.BF16, 83, False)
    q, k, v, cs = G.gdn_conv_prefill(to_dev(x).view(1, 40, -1), to_dev(w), 2, 4, output_conv_state=False)
    assert cs is None
    y_ref, _ = _oracle_conv(x.f64(), w, None, [0, 40], 1)
    assert_close(to_np(q).reshape(40, -1), y_ref[:, :256], CONV_TOL, "q", out_bf16=True)


def test_conv_long_workload_sampled():
    """T=32768, HK=16, HV=32, d=128 (C = 8192), bf16, SiLU, with a carried state: windows
    at the sequence start, across run boundaries and at the end, on 96 channels spread
    over q, k and v; the carried state out is the last three inputs, bit for bit."""
    import oracle
    import torch
    T, HK, HV, D = 32768, 16, 32, 128
    x, w, st0 = I.conv_prefill_inputs(T, 1, HK, HV, D, I.BF16, 84, True)
    q, k, v, cs = _gpu_conv(x, w, st0, None, 1, T, HK, HV, D, 1)
    C = w.shape[0]
    rng = np.random.default_rng(5)
    ch = np.sort(np.concatenate([rng.choice(HK * D, 32, replace=False),
                                 HK * D + rng.choice(HK * D, 32, replace=False),
                                 2 * HK * D + rng.choice(HV * D, 32, replace=False)]))
    chd = torch.from_numpy(ch)

    def gpu_rows(t0, t1):
        parts = [q.view(T, -1), k.view(T, -1), v.view(T, -1)]
        full = torch.cat([p[t0:t1] for p in parts], dim=1)   # [t1 - t0, C] on the device
        return to_np(full[:, chd.to(full.device)])

    for t0 in (0, 1, 29, 32, 1000, 16381, T - 8):
        t1 = t0 + 8
        # the three inputs before t0: the carried state, then the sequence's own rows
        prev = np.concatenate([st0[0].T.astype(np.float64), x.f64(slice(0, t0))], axis=0)[-3:]
        state = prev[:, ch].T[None]                            # [1, channels, 3]
        y_ref, _ = oracle.conv(x.f64((slice(t0, t1), ch))[None], w[ch], state, 1)
        assert_close(gpu_rows(t0, t1), y_ref[0], CONV_TOL, f"conv window at {t0}", out_bf16=True)
    last = x.f64(slice(T - 3, T))                              # [3, C], oldest first
    np.testing.assert_array_equal(to_np(cs)[0], last, err_msg="conv state out")
    assert cs.shape == (1, 3, C)


def _end_to_end(outgate):
    """Three packed sequences (37, 130, 64 tokens) from raw projections: the convolution,
    the chunked prefill from a carried state, then two fused decode steps that take over
    both states; against the oracle's convolution, gates and recurrence over the whole
    sequences (prefill tokens followed by the two decoded tokens).  gdn_conv_prefill hands
    the prefill q, k, v in the io dtype, so the oracle rounds the prefill tokens'
    convolution output to bf16 at the same point; the fused decode step keeps its q, k, v
    in fp32, and so does the oracle for the decoded tokens.  outgate: the output epilogue on
    both calls (gdn_chunk_prefill_outgate, then the decode step's), against the oracle's
    epilogue over the whole sequences."""
    import oracle
    import torch
    import gated_deltanet_sequence_delta_b200 as G
    lens = [37, 130, 64]
    HK, HV, D, io, act = 2, 4, 128, I.BF16, 1
    N, n_pre = len(lens), sum(lens)
    bounds = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    x, w, st0 = I.conv_prefill_inputs(n_pre, N, HK, HV, D, io, 85, True)
    xdec, _, _ = I.conv_prefill_inputs(2 * N, N, HK, HV, D, io, 86, False)     # step s: rows s N .. s N + N - 1
    rng = np.random.default_rng(87)
    a = rng.standard_normal((n_pre + 2 * N, HV)).astype(np.float32)            # prefill rows, then decode rows
    b = rng.standard_normal((n_pre + 2 * N, HV)).astype(np.float32)
    A_log, dt_bias, _ = I.gate_params(87, HV)
    h0 = (0.02 * rng.standard_normal((N, HV, D, D))).astype(np.float32)
    eps = 1e-3                                                                  # the Qwen3-next page's value
    z, wn = I.outgate_inputs(n_pre + 2 * N, HV, D, io, 88)                     # prefill rows, then decode rows
    zd = to_dev(z).view(n_pre + 2 * N, HV, D)
    wnd = to_dev(wn)

    # ---- GPU: convolution, gates, prefill, then two decode steps from raw projections
    q, k, v, cs = _gpu_conv(x, w, st0, bounds, 1, n_pre, HK, HV, D, act)
    ad, bd = to_dev(a), to_dev(b)
    Ad, dd = to_dev(A_log), to_dev(dt_bias)
    g, beta = G.gdn_gates(ad[:n_pre].view(1, n_pre, HV), bd[:n_pre].view(1, n_pre, HV), Ad, dd)
    cud = to_dev(bounds.astype(np.int32))
    if outgate:
        o_pre, hT = G.gdn_chunk_prefill_outgate(q, k, v, g, beta, zd[:n_pre].view(1, n_pre, HV, D), wnd, eps,
                                                initial_state=to_dev(h0), cu_seqlens=cud)
    else:
        o_pre, hT = G.gdn_chunk_prefill(q, k, v, g, beta, initial_state=to_dev(h0), cu_seqlens=cud)
    wd = to_dev(w)
    cs_next = torch.empty_like(cs)
    o_dec = []
    for s in range(2):
        rows = slice(n_pre + s * N, n_pre + (s + 1) * N)
        og = (zd[rows].contiguous(), wnd, eps) if outgate else None
        o_s, _ = G.gdn_decode_step_fused(to_dev(xdec).view(2 * N, -1)[s * N:(s + 1) * N], wd, cs, ad[rows], bd[rows],
                                         Ad, dd, hT, HK=HK, conv_act=act, conv_state_out=cs_next, outgate=og)
        o_dec.append(to_np(o_s))
        cs, cs_next = cs_next, cs
    assert G.gdn_decode_status() == 0

    # ---- oracle over the whole sequences (each: its prefill tokens, then its two decoded tokens)
    order = []
    for n in range(N):
        order += list(range(int(bounds[n]), int(bounds[n + 1])))
        order += [n_pre + n, n_pre + N + n]
    order = np.asarray(order)
    x_all = np.concatenate([x.f64(), xdec.f64()], axis=0)[order]
    full_bounds = np.concatenate([[0], np.cumsum(np.asarray(lens) + 2)]).astype(np.int64)
    y, st_ref = _oracle_conv(x_all, w, st0, full_bounds, act)
    pre_rows = np.concatenate([np.arange(full_bounds[n], full_bounds[n] + lens[n]) for n in range(N)])
    y[pre_rows] = I.bf16_bits_to_f32(I.f32_to_bf16_bits(y[pre_rows].astype(np.float32)))
    qr = y[:, :HK * D].reshape(-1, HK, D)
    kr = y[:, HK * D:2 * HK * D].reshape(-1, HK, D)
    vr = y[:, 2 * HK * D:].reshape(-1, HV, D)
    g_ref, beta_ref = oracle.gates(a[order].astype(np.float64), b[order].astype(np.float64),
                                   A_log.astype(np.float64), dt_bias.astype(np.float64))
    o_ref, hT_ref = oracle.recurrence(qr, kr, vr, g_ref, beta_ref, h0=h0, cu_seqlens=full_bounds)
    if outgate:
        o_ref = oracle.out_gate(o_ref, z.f64().reshape(n_pre + 2 * N, HV, D)[order], wn.astype(np.float64), eps=eps)
    tol = TOL[io]
    assert_close(to_np(o_pre).reshape(n_pre, HV, D), o_ref[pre_rows], tol, "prefill o", out_bf16=True)
    for s in range(2):
        dec_rows = full_bounds[:-1] + np.asarray(lens) + s
        assert_close(o_dec[s], o_ref[dec_rows], tol, f"decode step {s} o", out_bf16=True)
    assert_close(to_np(hT), hT_ref, tol, "final state")
    np.testing.assert_array_equal(to_np(cs).transpose(0, 2, 1), st_ref, err_msg="conv state after decoding")


def test_conv_prefill_decode_end_to_end():
    _end_to_end(outgate=False)


def test_conv_prefill_decode_end_to_end_output_epilogue():
    """The same sequences with the output epilogue on the prefill and on both decode steps:
    the two calls apply one epilogue, so the decoded tokens continue the prefilled ones."""
    _end_to_end(outgate=True)
