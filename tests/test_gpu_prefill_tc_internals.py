"""White-box check of the tensor-core prefill's chunk-local stage: after a call,
the workspace holds, per (chunk, value head), fp16 W = T diag(b gamma) K_hat,
U = T diag(b) V (stored as fp16(U / 2^e) with 2^e alongside, e from max|v|),
P = scale * (exp(G_i - G_j) q_hat_i . k_hat_j)_{i>=j}, the per-row scalars, and per
(chunk, q/k head) the normalised fp16 K_hat and Q_hat tiles.  They are recomputed
here in numpy fp64 from the same inputs (the gates from the oracle) and compared at
fp16 accuracy.  This pins the first kernel separately from the serial state carry.
The workspace layout is the library's private business; this test mirrors it."""
import numpy as np
import pytest

from gated_deltanet_sequence_delta_b200 import inputs as I
from harness import oracle_gates, to_dev

pytestmark = pytest.mark.gpu


def _ru(x, a):
    return (x + a - 1) // a * a


def _layout(n_tokens, n_seqs, HK, HV):
    max_chunks = (n_tokens + 63) // 64 + n_seqs
    rows = max_chunks * HV * 64
    off_w = _ru(256 + (n_seqs + 1) * 4, 1024)
    off_u = _ru(off_w + rows * 128 * 2, 1024)
    off_p = _ru(off_u + rows * 128 * 2, 1024)
    off_qk = _ru(off_p + rows * 64 * 2, 1024)
    off_sc = _ru(off_qk + max_chunks * HK * 128 * 128 * 2, 1024)
    return max_chunks, off_w, off_u, off_p, off_qk, off_sc


def _f16_view(ws, off, n):
    import torch
    return ws[off:off + 2 * n].view(torch.float16).float().cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("HK,HV", [(2, 4), (2, 2)])
def test_chunk_local_stage(HK, HV):
    import torch
    import gated_deltanet_sequence_delta_b200 as G
    T = 150
    inp = I.make_prefill(1, T, HK, HV, 128, 128, io_dtype=I.BF16, seed=31, h0_std=0.05)
    g, beta = oracle_gates(inp)
    tg = torch.from_numpy(g.astype(np.float32)).cuda()
    tb = torch.from_numpy(beta.astype(np.float32)).cuda()
    need = G.prefill_workspace_bytes(T, 1, HK, HV, 128, 128, 64, 1)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    G.gdn_chunk_prefill(to_dev(inp.q), to_dev(inp.k), to_dev(inp.v), tg, tb,
                        initial_state=to_dev(inp.h0), workspace=ws, scale=0.5)
    torch.cuda.synchronize()
    assert G.gdn_chunk_prefill_status(ws) == 0
    max_chunks, off_w, off_u, off_p, off_qk, off_sc = _layout(T, 1, HK, HV)
    rows = max_chunks * HV * 64
    W = _f16_view(ws, off_w, rows * 128).reshape(max_chunks, HV, 64, 128)
    U = _f16_view(ws, off_u, rows * 128).reshape(max_chunks, HV, 64, 128)
    P = _f16_view(ws, off_p, rows * 64).reshape(max_chunks, HV, 64, 64)
    QK = _f16_view(ws, off_qk, max_chunks * HK * 128 * 128).reshape(max_chunks, HK, 128, 128)
    SC = ws[off_sc:off_sc + 4 * max_chunks * HV * 256].view(torch.float32).cpu().numpy()
    SC = SC.astype(np.float64).reshape(max_chunks, HV, 256)
    U = U * SC[:, :, 129][:, :, None, None]

    q, k, v = inp.q.f64()[0], inp.k.f64()[0], inp.v.f64()[0]
    rq = 1 / np.sqrt(np.sum(q * q, -1) + 1e-6)
    rk = 1 / np.sqrt(np.sum(k * k, -1) + 1e-6)
    Gq = HV // HK
    for c in range((T + 63) // 64):
        s, e = 64 * c, min(T, 64 * c + 64)
        cn = e - s
        for h in range(HV):
            hk = h // Gq
            Kh = k[s:e, hk] * rk[s:e, hk, None]
            Qh = q[s:e, hk] * rq[s:e, hk, None]
            V = v[s:e, h]
            bt = beta[0, s:e, h]
            Gc = np.cumsum(g[0, s:e, h])
            ii, jj = np.meshgrid(np.arange(cn), np.arange(cn), indexing="ij")
            Gam = np.exp(np.where(ii >= jj, Gc[:, None] - Gc[None, :], -np.inf))
            L = np.where(ii > jj, bt[:, None] * Gam * (Kh @ Kh.T), 0.0)
            Tm = np.linalg.inv(np.eye(cn) + L)
            W_ref = Tm @ ((bt * np.exp(Gc))[:, None] * Kh)
            U_ref = Tm @ (bt[:, None] * V)
            P_ref = 0.5 * Gam * (Qh @ Kh.T)
            a_ref = 0.5 * np.exp(Gc)
            d_ref = np.exp(Gc[-1] - Gc)
            tag = f"chunk {c} head {h}"
            for name, got, ref in (("W", W[c, h, :cn], W_ref), ("U", U[c, h, :cn], U_ref),
                                   ("P", P[c, h, :cn, :cn], P_ref)):
                scale_ = np.max(np.abs(ref)) + 1e-30
                err = np.max(np.abs(got - ref)) / scale_
                assert err < 4e-3, f"{tag} {name}: max err / max|ref| = {err:.3e}"
            np.testing.assert_allclose(SC[c, h, :cn], a_ref, rtol=1e-4, err_msg=tag + " a")
            np.testing.assert_allclose(SC[c, h, 64:64 + cn], d_ref, rtol=1e-4, err_msg=tag + " d")
            np.testing.assert_allclose(SC[c, h, 128], np.exp(Gc[-1]), rtol=1e-4, err_msg=tag + " gC")
            np.testing.assert_allclose(SC[c, h, 130], np.abs(V).max(), rtol=1e-6, err_msg=tag + " vmax")
            assert 0.5 <= np.abs(V).max() / SC[c, h, 129] < 1.0   # U is stored as fp16(U * 2^-e) with max|v| * 2^-e in [0.5, 1)
            assert np.all(W[c, h, cn:] == 0) and np.all(U[c, h, cn:] == 0)
            if h % Gq == 0:
                np.testing.assert_allclose(QK[c, hk, :cn], Kh, atol=2e-3 * np.abs(Kh).max(), err_msg=tag + " K_hat")
                np.testing.assert_allclose(QK[c, hk, 64:64 + cn], Qh, atol=2e-3 * np.abs(Qh).max(),
                                           err_msg=tag + " Q_hat")
