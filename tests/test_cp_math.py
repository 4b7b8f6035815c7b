"""The decomposition behind the context-parallel prefill, on the oracle alone (CPU): for each
segment of a sequence, B and o0 are the run from a zero state, A and c the run with v = 0 from
the identity; the scan H_start(r + 1) = A_r H_start(r) + B_r and the correction
o_t = o0_t + H_start^T c_t must reproduce the run over the whole sequence.  Three segments of
unequal length, two sequences, grouped heads, a scale other than 1 (c carries it) and an
initial state."""
import numpy as np

import oracle


def test_three_segments_gqa_scale_and_start_state():
    rng = np.random.default_rng(21)
    N, HK, HV, D = 2, 1, 2, 8
    bounds = [0, 13, 30, 41]   # segment token ranges
    T = bounds[-1]
    q = rng.standard_normal((N, T, HK, D))
    k = rng.standard_normal((N, T, HK, D))
    v = rng.standard_normal((N, T, HV, D))
    g = -np.abs(rng.standard_normal((N, T, HV))) * 0.2
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((N, T, HV))))
    h0 = 0.1 * rng.standard_normal((N, HV, D, D))
    scale = 0.7
    o_ref, h_ref = oracle.recurrence(q, k, v, g, beta, h0=h0, scale=scale)
    eye = np.broadcast_to(np.eye(D), (N, HV, D, D)).copy()
    H = h0.copy()
    for r in range(len(bounds) - 1):
        sl = slice(bounds[r], bounds[r + 1])
        seg = [x[:, sl] for x in (q, k, v, g, beta)]
        o0, Bs = oracle.recurrence(*seg, scale=scale)
        c, As = oracle.recurrence(seg[0], seg[1], np.zeros_like(seg[2]), seg[3], seg[4], h0=eye, scale=scale)
        o = o0 + np.einsum("nthk,nhkj->nthj", c, H)
        np.testing.assert_allclose(o, o_ref[:, sl], rtol=0, atol=1e-10)
        H = np.einsum("nhij,nhjk->nhik", As, H) + Bs
    np.testing.assert_allclose(H, h_ref, rtol=0, atol=1e-10)


def test_transition_is_the_product_of_the_updates():
    """A of one segment equals the ordered product of the per-token maps
    alpha_t (I - beta_t k_t k_t^T) (k unit-normalised, as the oracle does), a brute-force
    check of the v = 0, identity-start run."""
    rng = np.random.default_rng(22)
    T, D = 6, 5
    q = rng.standard_normal((1, T, 1, D))
    k = rng.standard_normal((1, T, 1, D))
    g = -np.abs(rng.standard_normal((1, T, 1))) * 0.3
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((1, T, 1))))
    eye = np.eye(D)[None, None].copy()
    _, A = oracle.recurrence(q, k, np.zeros((1, T, 1, D)), g, beta, h0=eye)
    P = np.eye(D)
    for t in range(T):
        kt = k[0, t, 0] / np.sqrt(np.sum(k[0, t, 0] ** 2) + 1e-6)
        P = np.exp(g[0, t, 0]) * (np.eye(D) - beta[0, t, 0] * np.outer(kt, kt)) @ P
    np.testing.assert_allclose(A[0, 0], P, rtol=0, atol=1e-12)
