"""fp64 chunked form of the gated delta rule -- test infrastructure only.

This is NOT the oracle of record (that is the token-by-token recurrence in
``gdn_oracle.c``).  It writes out, in plain numpy fp64, the chunk-parallel
reformulation that the prefill kernels are built on, so that a test can show
the algebra itself equals the recurrence before any kernel is trusted with it.
It shares no code with the CUDA path.

The "QWEN3.5" Q&A page (question 1) describes the scheme: time is cut into
chunks of BT tokens, work inside a chunk is parallel, and the state is carried
serially from chunk to chunk.  The pages give no equations for it; the ones
below follow from the recurrence alone.  With H0 = S^T the state at the start
of a chunk (Dk x Dv), rows k_i, q_i, v_i of the chunk, and G_i the running sum
of the log-decays g inside the chunk (so gamma_i = exp(G_i)):

    delta_i = beta_i (v_i - alpha_i k_i H_{i-1})     H_i = alpha_i H_{i-1} + k_i^T delta_i
    (I + L) Delta = diag(beta) V - diag(beta gamma) K H0,
        L_ij = beta_i exp(G_i - G_j) k_i . k_j            (i > j, else 0)
    Delta = U - W H0,  with  T = (I + L)^{-1},
        W = T diag(beta gamma) K,   U = T diag(beta) V
    O = diag(gamma) Q H0 + P Delta,
        P_ij = exp(G_i - G_j) q_i . k_j                   (i >= j, else 0)
    H_C = gamma_C H0 + (diag(exp(G_C - G)) K)^T Delta

Every exponent that is evaluated is <= 0.
"""
from __future__ import annotations

import numpy as np
from scipy.linalg import solve_triangular


def _l2n(x: np.ndarray) -> np.ndarray:
    return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + 1e-6)


def chunked(q, k, v, g, beta, h0=None, cu_seqlens=None, BT: int = 64,
            scale: float = 1.0, l2norm: bool = True):
    """Same arguments and results as the oracle's ``recurrence`` (packed form
    when ``cu_seqlens`` is given, else dense [B, T, ...])."""
    q, k, v, g, beta = (np.asarray(x, dtype=np.float64) for x in (q, k, v, g, beta))
    out_shape = v.shape
    if cu_seqlens is None:
        B, T = q.shape[:2]
        cu = np.arange(B + 1, dtype=np.int64) * T
    else:
        cu = np.asarray(cu_seqlens, dtype=np.int64)
    HK, Dk = q.shape[-2:]
    HV, Dv = v.shape[-2:]
    q = q.reshape(-1, HK, Dk)
    k = k.reshape(-1, HK, Dk)
    v = v.reshape(-1, HV, Dv)
    g = g.reshape(-1, HV)
    beta = beta.reshape(-1, HV)
    if l2norm:
        q = _l2n(q)
        k = _l2n(k)
    n_seqs = cu.size - 1
    G_ = HV // HK
    o = np.zeros((q.shape[0], HV, Dv))
    hT = np.zeros((n_seqs, HV, Dk, Dv))
    for n in range(n_seqs):
        for h in range(HV):
            hk = h // G_
            H = (np.zeros((Dk, Dv)) if h0 is None
                 else np.array(np.asarray(h0, dtype=np.float64).reshape(n_seqs, HV, Dk, Dv)[n, h]))
            for s in range(cu[n], cu[n + 1], BT):
                e = min(s + BT, cu[n + 1])
                Q, K, V = q[s:e, hk], k[s:e, hk], v[s:e, h]
                bt = beta[s:e, h]
                G = np.cumsum(g[s:e, h])
                gam = np.exp(G)
                C = e - s
                ii, jj = np.meshgrid(np.arange(C), np.arange(C), indexing="ij")
                diff = np.where(ii >= jj, G[:, None] - G[None, :], -np.inf)
                Gam = np.exp(diff)                      # 0 above the diagonal
                L = np.where(ii > jj, bt[:, None] * Gam * (K @ K.T), 0.0)
                I = np.eye(C)
                W = solve_triangular(I + L, (bt * gam)[:, None] * K, lower=True,
                                     unit_diagonal=True)
                U = solve_triangular(I + L, bt[:, None] * V, lower=True,
                                     unit_diagonal=True)
                D = U - W @ H
                P = Gam * (Q @ K.T)
                o[s:e, h] = scale * (gam[:, None] * (Q @ H) + P @ D)
                H = gam[-1] * H + (np.exp(G[-1] - G)[:, None] * K).T @ D
            hT[n, h] = H
    return o.reshape(out_shape), hT
