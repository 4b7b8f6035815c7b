"""Pins of the CPU oracle to facts fixed outside the oracle itself.

Every function takes an oracle handle (``oracle.OracleLib``) so the same checks
can be run against the real build and against builds with a planted mistake
(``test_oracle_mutants.py``).  Each pin states the passage or the mathematics it
rests on; none re-types the oracle's loop:

* gate values against library routines (scipy's expit, numpy's logaddexp) and
  against values worked by hand (``golden/gates_hand.json``);
* a two-token example worked by hand (``golden/hand_worked_2x2.json``);
* the special cases the pages name: no write keeps the state; a full write of a
  unit key retrieves exactly; a near-zero decay clears history;
* the online-learning view: each update is one gradient step on
  1/2 ||S k - v||^2 after weight decay, with the gradient taken numerically;
* a brute-force expanded product of the per-token transition matrices;
* structural facts: linearity in (v, S0), contraction bound, independence of
  packed sequences, grouped-head mapping, state carry, the chunked algebra;
* the output epilogue: a hand-worked example (``golden/out_gate_hand.json``), scale
  invariance, unit RMS of the plain norm, the gate against scipy, the place of eps;
* the convolution prologue: a hand-worked example (``golden/conv_hand.json``),
  the impulse response, the state as the three past inputs, state carry,
  linearity, and SiLU against scipy's logistic function.
"""
from __future__ import annotations

import json
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def _unit(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def _rand_problem(rng, B=1, T=12, HK=1, HV=1, Dk=6, Dv=6, unit_keys=True):
    q = rng.standard_normal((B, T, HK, Dk))
    k = rng.standard_normal((B, T, HK, Dk))
    if unit_keys:
        q, k = _unit(q), _unit(k)
    v = rng.standard_normal((B, T, HV, Dv))
    g = -rng.uniform(0.0, 1.5, (B, T, HV))
    beta = rng.uniform(0.0, 1.0, (B, T, HV))
    h0 = rng.standard_normal((B, HV, Dk, Dv))
    return q, k, v, g, beta, h0


# ---------------------------------------------------------------------------
# gates ("Gated DeltaNet ... Qwen3-next" page, section 2.1)
# ---------------------------------------------------------------------------
def pin_gates_library(orc):
    """g = -exp(A_log) softplus(a + dt_bias), beta = sigmoid(b) against scipy /
    numpy routines, over ordinary and extreme arguments."""
    from scipy.special import expit
    rng = _rng(11)
    HV = 5
    a = np.concatenate([rng.standard_normal((40, HV)) * 3,
                        np.linspace(-60, 60, 5 * HV).reshape(5, HV)])
    b = np.concatenate([rng.standard_normal((40, HV)) * 3,
                        np.linspace(-40, 40, 5 * HV).reshape(5, HV)])
    A_log = np.log(rng.uniform(1, 16, HV))
    dt_bias = rng.standard_normal(HV)
    g, beta = orc.gates(a, b, A_log, dt_bias)
    g_ref = -np.exp(A_log) * np.logaddexp(0.0, a + dt_bias)
    np.testing.assert_allclose(g, g_ref, rtol=1e-13, atol=1e-300)
    np.testing.assert_allclose(beta, expit(b), rtol=1e-13, atol=1e-300)
    assert np.all(g <= 0)


def pin_gates_hand(orc):
    rows = json.load(open(os.path.join(GOLDEN, "gates_hand.json")))["rows"]
    a = np.array([[r["a"]] for r in rows])
    b = np.array([[r["b"]] for r in rows])
    for i, r in enumerate(rows):
        g, beta = orc.gates(a[i:i + 1], b[i:i + 1], np.array([r["A_log"]]),
                            np.array([r["dt_bias"]]))
        np.testing.assert_allclose(g[0, 0], r["g"], rtol=1e-14)
        np.testing.assert_allclose(beta[0, 0], r["beta"], rtol=1e-14)


def pin_gates_dt_construction(orc):
    """With a = 0 and dt_bias = log(expm1(dt)), softplus(dt_bias) = dt, so
    g = -exp(A_log) * dt (the workloads' dt parametrisation)."""
    dt = np.exp(np.linspace(np.log(1e-3), np.log(1e-1), 7))
    A_log = np.log(np.linspace(1, 16, 7))
    g, _ = orc.gates(np.zeros((1, 7)), np.zeros((1, 7)), A_log, np.log(np.expm1(dt)))
    np.testing.assert_allclose(g[0], -np.exp(A_log) * dt, rtol=1e-12)


# ---------------------------------------------------------------------------
# recurrence (research-log page, third update rule; tutorial page section 6)
# ---------------------------------------------------------------------------
def pin_hand_worked(orc):
    d = json.load(open(os.path.join(GOLDEN, "hand_worked_2x2.json")))
    q = np.array(d["q"])[None, :, None, :]
    k = np.array(d["k"])[None, :, None, :]
    v = np.array(d["v"])[None, :, None, :]
    g = np.array(d["g"])[None, :, None]
    beta = np.array(d["beta"])[None, :, None]
    h0 = np.array(d["S0"]).T[None, None]
    o, hT = orc.recurrence(q, k, v, g, beta, h0=h0, l2norm=False)
    np.testing.assert_allclose(o[0, :, 0], np.array(d["o"]), atol=1e-14)
    np.testing.assert_allclose(hT[0, 0], np.array(d["S_final"]).T, atol=1e-14)


def pin_no_write_keeps_state(orc):
    """alpha = 1, beta = 0: S never changes and o_t = S_0 q_t (scale applied)."""
    rng = _rng(1)
    q, k, v, _, _, h0 = _rand_problem(rng, B=2, T=9, HK=2, HV=4, Dk=5, Dv=7)
    g = np.zeros(v.shape[:3])
    beta = np.zeros(v.shape[:3])
    o, hT = orc.recurrence(q, k, v, g, beta, h0=h0, scale=0.75, l2norm=False)
    np.testing.assert_array_equal(hT, h0)
    for h in range(4):
        expect = 0.75 * np.einsum("btc,cr->btr", q[:, :, h // 2], h0[0, h])
        np.testing.assert_allclose(o[0, :, h], expect[0], rtol=1e-13, atol=1e-13)
        expect1 = 0.75 * np.einsum("tc,cr->tr", q[1, :, h // 2], h0[1, h])
        np.testing.assert_allclose(o[1, :, h], expect1, rtol=1e-13, atol=1e-13)


def pin_orthonormal_retrieval(orc):
    """alpha = 1, beta = 1, orthonormal keys: the delta rule replaces the value
    stored under a key exactly, so S k_j returns the latest v written under k_j
    (research-log page: DeltaNet 'exactly replaces a key-value pair')."""
    rng = _rng(2)
    D = 8
    Qm, _ = np.linalg.qr(rng.standard_normal((D, D)))
    keys = Qm.T                              # rows are orthonormal
    order = [0, 1, 2, 0, 3, 1, 4, 0, 5]
    T = len(order)
    k = keys[order][None, :, None, :]
    v = rng.standard_normal((1, T, 1, D))
    q = k.copy()                             # read back the key just written
    g = np.zeros((1, T, 1))
    beta = np.ones((1, T, 1))
    o, hT = orc.recurrence(q, k, v, g, beta, h0=None, l2norm=False)
    np.testing.assert_allclose(o[0, :, 0], v[0, :, 0], atol=1e-12)
    latest = {}
    for t, j in enumerate(order):
        latest[j] = v[0, t, 0]
    S = hT[0, 0].T
    for j, vj in latest.items():
        np.testing.assert_allclose(S @ keys[j], vj, atol=1e-12)
    for j in set(range(D)) - set(order):      # never-written keys read zero
        np.testing.assert_allclose(S @ keys[j], 0.0, atol=1e-12)


def pin_full_write_any_decay(orc):
    """For any decay and any prior state, a beta = 1 write of a unit key gives
    S_t k_t = v_t, because the decayed read along k_t is cleared before the write
    (decay first, then the beta write: Q&A page, question 2a)."""
    rng = _rng(3)
    q, k, v, g, _, h0 = _rand_problem(rng, T=10, Dk=6, Dv=5)
    beta = np.ones(g.shape)
    o, _ = orc.recurrence(k, k, v, g, beta, h0=h0, l2norm=False)
    np.testing.assert_allclose(o[0, :, 0], v[0, :, 0], atol=1e-12)


def pin_sgd_step(orc):
    """Each update is S_t = X - beta grad L(X) with X = alpha S_{t-1} and
    L(X) = 1/2 ||X k - v||^2 (research-log page, online-learning view).
    The gradient is taken by central differences, exact for a quadratic up to
    rounding."""
    rng = _rng(4)
    Dk, Dv = 4, 3
    S = rng.standard_normal((Dv, Dk))
    for t in range(5):
        k = _unit(rng.standard_normal(Dk))
        v = rng.standard_normal(Dv)
        g = -rng.uniform(0, 2)
        b = rng.uniform(0, 1)
        X = np.exp(g) * S

        def L(M):
            r = M @ k - v
            return 0.5 * float(r @ r)

        grad = np.zeros_like(X)
        eps = 1e-3
        for i in range(Dv):
            for j in range(Dk):
                E = np.zeros_like(X)
                E[i, j] = eps
                grad[i, j] = (L(X + E) - L(X - E)) / (2 * eps)
        S_expect = X - b * grad
        _, hT = orc.recurrence(k[None, None, None], k[None, None, None],
                               v[None, None, None], np.array([[[g]]]), np.array([[[b]]]),
                               h0=S.T[None, None], l2norm=False)
        np.testing.assert_allclose(hT[0, 0].T, S_expect, rtol=1e-9, atol=1e-10)
        S = hT[0, 0].T


def pin_bruteforce_product(orc):
    """S_T = S_0 prod_t M_t + sum_t beta_t v_t k_t^T prod_{s>t} M_s with
    M_t = alpha_t (I - beta_t k_t k_t^T), as dense matrices, for T <= 16, d <= 8;
    every o_t = S_t q_t from the same expansion truncated at t."""
    rng = _rng(5)
    for (T, Dk, Dv) in [(16, 8, 8), (7, 3, 5), (11, 6, 2)]:
        q = rng.standard_normal((1, T, 1, Dk))
        k = rng.standard_normal((1, T, 1, Dk))     # not unit: the rule does not need it
        v = rng.standard_normal((1, T, 1, Dv))
        g = -rng.uniform(0, 1, (1, T, 1))
        beta = rng.uniform(0, 1, (1, T, 1))
        S0 = rng.standard_normal((Dv, Dk))
        M = [np.exp(g[0, t, 0]) * (np.eye(Dk) - beta[0, t, 0] * np.outer(k[0, t, 0], k[0, t, 0]))
             for t in range(T)]

        def S_at(tt):
            P = np.eye(Dk)
            for t in range(tt + 1):
                P = P @ M[t]
            S = S0 @ P
            for t in range(tt + 1):
                R = np.eye(Dk)
                for s in range(t + 1, tt + 1):
                    R = R @ M[s]
                S = S + beta[0, t, 0] * np.outer(v[0, t, 0], k[0, t, 0]) @ R
            return S

        o, hT = orc.recurrence(q, k, v, g, beta, h0=S0.T[None, None], l2norm=False, scale=1.3)
        for t in range(T):
            np.testing.assert_allclose(o[0, t, 0], 1.3 * S_at(t) @ q[0, t, 0], rtol=1e-10, atol=1e-10)
        np.testing.assert_allclose(hT[0, 0].T, S_at(T - 1), rtol=1e-10, atol=1e-10)


def pin_reset_clears_history(orc):
    """alpha -> 0 (g = -60) clears the state (tutorial page, section 6: alpha near 0
    wipes the previous state): right after the token the state is beta v k^T, and
    later outputs do not depend on what came before."""
    rng = _rng(6)
    q, k, v, g, beta, h0 = _rand_problem(rng, T=14, Dk=5, Dv=4)
    t0 = 6
    g[0, t0, 0] = -60.0
    o1, _ = orc.recurrence(q, k, v, g, beta, h0=h0, l2norm=False)
    q2, k2, v2 = q.copy(), k.copy(), v.copy()
    q2[0, :t0] = _unit(rng.standard_normal(q2[0, :t0].shape))
    k2[0, :t0] = _unit(rng.standard_normal(k2[0, :t0].shape))
    v2[0, :t0] = rng.standard_normal(v2[0, :t0].shape)
    o2, hT2 = orc.recurrence(q2, k2, v2, g, beta, h0=-3 * h0, l2norm=False)
    np.testing.assert_allclose(o1[0, t0:], o2[0, t0:], atol=1e-20)
    _, h_at = orc.recurrence(q[:, :t0 + 1], k[:, :t0 + 1], v[:, :t0 + 1], g[:, :t0 + 1],
                             beta[:, :t0 + 1], h0=h0, l2norm=False)
    expect = beta[0, t0, 0] * np.outer(k[0, t0, 0], v[0, t0, 0])   # H = S^T = beta k v^T
    np.testing.assert_allclose(h_at[0, 0], expect, atol=1e-20)


def pin_linearity(orc):
    """For fixed q, k, g, beta the map (v, S0) -> (o, S_T) is linear."""
    rng = _rng(7)
    q, k, v1, g, beta, h1 = _rand_problem(rng, B=2, T=10, HK=1, HV=2, Dk=5, Dv=6)
    v2 = rng.standard_normal(v1.shape)
    h2 = rng.standard_normal(h1.shape)
    oa, ha = orc.recurrence(q, k, v1, g, beta, h0=h1, l2norm=True)
    ob, hb = orc.recurrence(q, k, v2, g, beta, h0=h2, l2norm=True)
    oc, hc = orc.recurrence(q, k, 2 * v1 - 0.5 * v2, g, beta, h0=2 * h1 - 0.5 * h2, l2norm=True)
    np.testing.assert_allclose(oc, 2 * oa - 0.5 * ob, rtol=1e-11, atol=1e-11)
    np.testing.assert_allclose(hc, 2 * ha - 0.5 * hb, rtol=1e-11, atol=1e-11)


def pin_contraction_bound(orc):
    """With unit keys and beta in [0, 1], ||I - beta k k^T||_2 <= 1, hence
    ||S_t||_F <= alpha_t ||S_{t-1}||_F + beta_t ||v_t||."""
    rng = _rng(8)
    q, k, v, g, beta, h0 = _rand_problem(rng, T=30, Dk=6, Dv=6)
    H = h0
    for t in range(30):
        sl = slice(t, t + 1)
        _, Hn = orc.recurrence(q[:, sl], k[:, sl], v[:, sl], g[:, sl], beta[:, sl], h0=H,
                               l2norm=False)
        bound = np.exp(g[0, t, 0]) * np.linalg.norm(H) + beta[0, t, 0] * np.linalg.norm(v[0, t, 0])
        assert np.linalg.norm(Hn) <= bound * (1 + 1e-12)
        H = Hn


def pin_packed_sequences_independent(orc):
    """Packed sequences (cu_seqlens) are independent problems, each with its own
    initial state; a run over the pack equals one run per sequence."""
    rng = _rng(9)
    lens = [5, 1, 0, 9, 3]
    cu = np.concatenate([[0], np.cumsum(lens)])
    Ttot = int(cu[-1])
    q, k, v, g, beta, _ = _rand_problem(rng, B=1, T=Ttot, HK=2, HV=4, Dk=4, Dv=3)
    h0 = rng.standard_normal((len(lens), 4, 4, 3))
    o, hT = orc.recurrence(q[0], k[0], v[0], g[0], beta[0], h0=h0, cu_seqlens=cu)
    for n in range(len(lens)):
        s, e = cu[n], cu[n + 1]
        if e == s:
            np.testing.assert_array_equal(hT[n], h0[n])
            continue
        on, hn = orc.recurrence(q[:, s:e], k[:, s:e], v[:, s:e], g[:, s:e], beta[:, s:e],
                                h0=h0[n:n + 1])
        np.testing.assert_allclose(o[s:e], on[0], rtol=1e-13, atol=1e-14)
        np.testing.assert_allclose(hT[n], hn[0], rtol=1e-13, atol=1e-14)


def pin_grouped_heads(orc):
    """Value head h reads q/k head h // (HV / HK) (contiguous groups): a grouped
    run equals an ungrouped run with each q/k head repeated over its group."""
    rng = _rng(10)
    q, k, v, g, beta, h0 = _rand_problem(rng, B=1, T=8, HK=2, HV=6, Dk=4, Dv=4)
    o, hT = orc.recurrence(q, k, v, g, beta, h0=h0)
    qr = np.repeat(q, 3, axis=2)
    kr = np.repeat(k, 3, axis=2)
    o2, h2 = orc.recurrence(qr, kr, v, g, beta, h0=h0)
    np.testing.assert_allclose(o, o2, rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(hT, h2, rtol=1e-14, atol=1e-15)
    # and the grouping is contiguous, not round-robin: head 1 uses q/k head 0
    qs = q.copy()
    qs[:, :, 1] += 1.0
    o3, _ = orc.recurrence(qs, k, v, g, beta, h0=h0)
    np.testing.assert_array_equal(o3[:, :, :3], o[:, :, :3])


def pin_l2norm(orc):
    """q/k L2 normalisation x / sqrt(sum x^2 + 1e-6): a full write of a key of
    squared norm s into a zero state stores ||k_hat|| = sqrt(s / (s + 1e-6))
    times ||v||; the result is scale-invariant for ordinary norms; a zero key
    writes nothing."""
    rng = _rng(12)
    for s in [1e-8, 1e-6, 1e-3, 1.0, 1e4]:
        kk = _unit(rng.standard_normal(5)) * np.sqrt(s)
        vv = rng.standard_normal(3)
        _, hT = orc.recurrence(kk[None, None, None], kk[None, None, None], vv[None, None, None],
                               np.zeros((1, 1, 1)), np.ones((1, 1, 1)), l2norm=True)
        np.testing.assert_allclose(np.linalg.norm(hT), np.sqrt(s / (s + 1e-6)) * np.linalg.norm(vv),
                                   rtol=1e-12)
    q, k, v, g, beta, h0 = _rand_problem(rng, T=6, Dk=4, Dv=4)
    o1, h1 = orc.recurrence(1e3 * q, 1e3 * k, v, g, beta, h0=h0, l2norm=True)
    o2, h2 = orc.recurrence(1e4 * q, 7e3 * k, v, g, beta, h0=h0, l2norm=True)
    np.testing.assert_allclose(o1, o2, rtol=1e-9, atol=1e-9)
    np.testing.assert_allclose(h1, h2, rtol=1e-9, atol=1e-9)
    z = np.zeros_like(k)
    _, hz = orc.recurrence(q, z, v, g, beta, h0=h0, l2norm=True)
    assert np.all(np.isfinite(hz))


def pin_state_carry(orc):
    """Resuming from the final state of a prefix equals one run over the whole
    sequence (the initial_state / last_state carry of the prefill call)."""
    rng = _rng(13)
    q, k, v, g, beta, h0 = _rand_problem(rng, B=2, T=17, HK=1, HV=2, Dk=5, Dv=5)
    o, hT = orc.recurrence(q, k, v, g, beta, h0=h0)
    oa, ha = orc.recurrence(q[:, :7], k[:, :7], v[:, :7], g[:, :7], beta[:, :7], h0=h0)
    ob, hb = orc.recurrence(q[:, 7:], k[:, 7:], v[:, 7:], g[:, 7:], beta[:, 7:], h0=ha)
    np.testing.assert_allclose(np.concatenate([oa, ob], axis=1), o, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(hb, hT, rtol=1e-13, atol=1e-14)


def pin_chunked_algebra(orc):
    """The chunk-parallel reformulation (oracle/chunked.py, derived from the
    recurrence; the Q&A page, question 1, says chunking only reorganises the
    same computation) equals the token-by-token oracle for several chunk sizes,
    ragged tails and packed sequences."""
    from oracle.chunked import chunked
    rng = _rng(14)
    lens = [37, 64, 1, 100, 0, 65]
    cu = np.concatenate([[0], np.cumsum(lens)])
    Ttot = int(cu[-1])
    q, k, v, g, beta, _ = _rand_problem(rng, B=1, T=Ttot, HK=2, HV=4, Dk=8, Dv=6,
                                        unit_keys=False)
    g = -rng.uniform(0, 3, g.shape)          # strong decays: G reaches about -150
    h0 = rng.standard_normal((len(lens), 4, 8, 6))
    o, hT = orc.recurrence(q[0], k[0], v[0], g[0], beta[0], h0=h0, cu_seqlens=cu, scale=0.5)
    for BT in (16, 32, 64):
        oc, hc = chunked(q[0], k[0], v[0], g[0], beta[0], h0=h0, cu_seqlens=cu, BT=BT, scale=0.5)
        np.testing.assert_allclose(oc, o, rtol=1e-10, atol=1e-11)
        np.testing.assert_allclose(hc, hT, rtol=1e-10, atol=1e-11)


# ---------------------------------------------------------------------------
# the convolution prologue (Qwen3-next page, section 3.1; kernel size 4 from the
# tutorial page, section 6)
# ---------------------------------------------------------------------------
def pin_conv_hand(orc):
    """A two-channel, three-token example with a non-zero state, worked by hand."""
    d = json.load(open(os.path.join(GOLDEN, "conv_hand.json")))
    y, st = orc.conv(np.array(d["x"])[None], np.array(d["w"]), np.array(d["state"])[None])
    np.testing.assert_array_equal(y[0], np.array(d["y"]))
    np.testing.assert_array_equal(st[0], np.array(d["state_out"]))


def pin_conv_impulse_response(orc):
    """A unit impulse at t = 0 from a zero state returns the taps newest first:
    y_t = w[3 - t] for t < 4, then 0 (causality and tap order)."""
    rng = _rng(61)
    C = 3
    w = rng.standard_normal((C, 4))
    x = np.zeros((1, 7, C))
    x[0, 0, :] = 1.0
    y, st = orc.conv(x, w)
    for t in range(7):
        want = w[:, 3 - t] if t < 4 else np.zeros(C)
        np.testing.assert_array_equal(y[0, t], want)
    np.testing.assert_array_equal(st[0], np.zeros((C, 3)))


def pin_conv_state_is_past_input(orc):
    """The state stands for the three inputs before the first token: a call with
    state s equals a zero-state call on [s; x] without its first three outputs, and
    its returned state is the last three inputs."""
    rng = _rng(62)
    B, T, C = 2, 9, 4
    w = rng.standard_normal((C, 4))
    s = rng.standard_normal((B, C, 3))
    x = rng.standard_normal((B, T, C))
    y, st = orc.conv(x, w, s)
    xx = np.concatenate([np.transpose(s, (0, 2, 1)), x], axis=1)
    yy, _ = orc.conv(xx, w)
    np.testing.assert_allclose(y, yy[:, 3:], rtol=0, atol=1e-14)
    np.testing.assert_array_equal(st, np.transpose(x[:, -3:], (0, 2, 1)))


def pin_conv_state_carry(orc):
    """One call over T tokens equals two calls over the two halves with the state carried."""
    rng = _rng(63)
    B, T, C = 2, 11, 5
    w = rng.standard_normal((C, 4))
    x = rng.standard_normal((B, T, C))
    s0 = rng.standard_normal((B, C, 3))
    for act in (0, 1):
        y, st = orc.conv(x, w, s0, act)
        y1, s1 = orc.conv(x[:, :4], w, s0, act)
        y2, s2 = orc.conv(x[:, 4:], w, s1, act)
        np.testing.assert_array_equal(y, np.concatenate([y1, y2], axis=1))
        np.testing.assert_array_equal(st, s2)


def pin_conv_linear_and_silu(orc):
    """Without an activation the convolution is linear in (x, state); SiLU is the
    identity output times scipy's logistic sigmoid of it."""
    from scipy.special import expit
    rng = _rng(64)
    B, T, C = 1, 8, 3
    w = rng.standard_normal((C, 4))
    x1, x2 = rng.standard_normal((2, B, T, C))
    s1, s2 = rng.standard_normal((2, B, C, 3))
    y1, _ = orc.conv(x1, w, s1)
    y2, _ = orc.conv(x2, w, s2)
    y12, _ = orc.conv(2.0 * x1 - 3.0 * x2, w, 2.0 * s1 - 3.0 * s2)
    np.testing.assert_allclose(y12, 2.0 * y1 - 3.0 * y2, rtol=1e-13, atol=1e-13)
    ys, _ = orc.conv(x1, w, s1, act=1)
    np.testing.assert_allclose(ys, y1 * expit(y1), rtol=1e-14, atol=1e-15)


# ---------------------------------------------------------------------------
# the output epilogue (Qwen3-next page, section 3.2; GDN resource-allocation page)
# ---------------------------------------------------------------------------
def pin_out_gate_hand(orc):
    """A two-value row worked by hand."""
    d = json.load(open(os.path.join(GOLDEN, "out_gate_hand.json")))
    out = orc.out_gate(np.array([d["o"]]), np.array([d["z"]]), np.array(d["w"]), eps=d["eps"])
    np.testing.assert_allclose(out[0], np.array(d["out"]), rtol=1e-15)


def pin_out_gate_properties(orc):
    """With eps = 0: scaling o by c > 0 changes nothing; with w = 0 and an open gate the
    row has unit RMS (the plain RMSNorm); the gate multiplies by scipy's logistic
    sigmoid of z; the sign of each element is that of o."""
    from scipy.special import expit
    rng = _rng(65)
    rows, D = 5, 16
    o = rng.standard_normal((rows, D))
    z = rng.standard_normal((rows, D))
    w = 0.3 * rng.standard_normal(D)
    out = orc.out_gate(o, z, w, eps=0.0)
    np.testing.assert_allclose(orc.out_gate(7.5 * o, z, w, eps=0.0), out, rtol=1e-13)
    plain = orc.out_gate(o, np.full_like(z, 40.0), np.zeros(D), eps=0.0)
    np.testing.assert_allclose(np.sqrt(np.mean(plain ** 2, axis=-1)), np.ones(rows), rtol=1e-12)
    gated0 = orc.out_gate(o, np.full_like(z, 40.0), w, eps=0.0)
    np.testing.assert_allclose(out, gated0 * expit(z) / expit(40.0), rtol=1e-13)
    assert np.all(np.sign(out) == np.sign(o))


def pin_out_gate_eps(orc):
    """eps sits inside the square root with the mean: a zero row stays zero, and a row of
    RMS s gets the factor 1 / sqrt(s^2 + eps)."""
    D = 8
    o = np.full((1, D), 1e-3)
    out = orc.out_gate(o, np.full((1, D), 40.0), np.zeros(D), eps=1e-6)
    np.testing.assert_allclose(out, o / np.sqrt(1e-6 + 1e-6), rtol=1e-12)
    assert np.all(orc.out_gate(np.zeros((1, D)), np.zeros((1, D)), np.zeros(D)) == 0.0)


ALL_PINS = [
    pin_gates_library, pin_gates_hand, pin_gates_dt_construction, pin_hand_worked,
    pin_no_write_keeps_state, pin_orthonormal_retrieval, pin_full_write_any_decay,
    pin_sgd_step, pin_bruteforce_product, pin_reset_clears_history, pin_linearity,
    pin_contraction_bound, pin_packed_sequences_independent, pin_grouped_heads, pin_l2norm,
    pin_state_carry, pin_chunked_algebra,
    pin_conv_hand, pin_conv_impulse_response, pin_conv_state_is_past_input, pin_conv_state_carry,
    pin_conv_linear_and_silu, pin_out_gate_hand, pin_out_gate_properties, pin_out_gate_eps,
]
