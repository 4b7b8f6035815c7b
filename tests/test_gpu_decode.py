"""gdn_decode_step on the GPU against the oracle's one-token recurrence."""
import numpy as np
import pytest

from gated_deltanet_sequence_delta_b200 import inputs as I
from harness import TOL, assert_close, to_dev, to_np

pytestmark = pytest.mark.gpu


def _run_steps(setup, n_steps, sample=None, check_every=1, fused_gates=False):
    """Run n_steps decode steps on the GPU from setup.state0; the oracle follows the
    (b, h) pairs in ``sample`` (all pairs if None).  With ``fused_gates`` the GPU forms the
    gates inside the step (gdn_decode_step_gated).  Returns max relative errors."""
    import oracle
    import gated_deltanet_sequence_delta_b200 as G
    B, HK, HV = setup.B, setup.HK, setup.HV
    Gq = HV // HK
    state = to_dev(setup.state0.copy())
    A_log, dt_bias = to_dev(setup.A_log), to_dev(setup.dt_bias)
    pairs = [(b, h) for b in range(B) for h in range(HV)] if sample is None else sample
    ref_state = np.stack([setup.state0[b, h] for (b, h) in pairs]).astype(np.float64)[:, None]
    tol = TOL[setup.io_dtype]
    worst_o = worst_s = 0.0
    for s in range(n_steps):
        q, k, v, a, b = setup.step(s)
        if fused_gates:
            o = G.gdn_decode_step_gated(to_dev(q), to_dev(k), to_dev(v), to_dev(a), to_dev(b), A_log, dt_bias,
                                        state, scale=setup.scale, qk_l2norm=setup.l2norm)
        else:
            g, beta = G.gdn_gates(to_dev(a), to_dev(b), A_log, dt_bias)
            o = G.gdn_decode_step(to_dev(q), to_dev(k), to_dev(v), g, beta, state, scale=setup.scale,
                                  qk_l2norm=setup.l2norm)
        g_ref, beta_ref = oracle.gates(a.astype(np.float64), b.astype(np.float64),
                                       setup.A_log.astype(np.float64), setup.dt_bias.astype(np.float64))
        bi = np.array([p[0] for p in pairs])
        hi = np.array([p[1] for p in pairs])
        qf, kf, vf = q.f64(), k.f64(), v.f64()
        o_ref, ref_state_new = oracle.decode_step(
            qf[bi, hi // Gq][:, None], kf[bi, hi // Gq][:, None], vf[bi, hi][:, None],
            g_ref[bi, hi][:, None], beta_ref[bi, hi][:, None], ref_state,
            scale=setup.scale, l2norm=setup.l2norm)
        ref_state = ref_state_new
        if (s + 1) % check_every == 0 or s == n_steps - 1:
            o_g = to_np(o)[bi, hi]
            worst_o = max(worst_o, assert_close(o_g, o_ref[:, 0], tol, f"decode step {s}: o",
                                                out_bf16=setup.io_dtype == I.BF16))
            st_g = to_np(state[bi, hi])
            worst_s = max(worst_s, assert_close(st_g, ref_state[:, 0], tol, f"decode step {s}: state"))
    return worst_o, worst_s


@pytest.mark.parametrize("io", [I.F32, I.BF16])
@pytest.mark.parametrize("D", [(128, 128), (64, 64), (128, 64), (64, 128)])
def test_decode_small(io, D):
    Dk, Dv = D
    setup = I.decode(B=3, H=4, D=Dk, io_dtype=io, seed=5, HK=2)
    if Dv != Dk:
        import dataclasses
        rng = np.random.default_rng(9)
        setup = dataclasses.replace(setup, Dv=Dv,
                                    state0=(0.02 * rng.standard_normal((3, 4, Dk, Dv))).astype(np.float32))
    _run_steps(setup, 12)


def test_decode_workload_first_steps_all_heads():
    """B=64, H=32, d=128, bf16: the first 16 steps on every (sequence, head)."""
    import gated_deltanet_sequence_delta_b200 as G
    setup = I.decode()
    _run_steps(setup, 16)
    assert G.gdn_decode_status() == 0   # no bounded wait expired


def test_decode_workload_all_steps_all_heads():
    """All 1024 steps of the B=64, H=32, d=128 workload on every (sequence, head), checked
    every 64 steps and at the end."""
    import gated_deltanet_sequence_delta_b200 as G
    setup = I.decode()
    _run_steps(setup, I.DECODE_STEPS, check_every=64)
    assert G.gdn_decode_status() == 0


def test_decode_workload_all_steps_sampled():
    """All 1024 steps of the B=64, H=32, d=128 workload; the oracle follows 12
    sampled (sequence, head) pairs, checked every 64 steps and at the end."""
    setup = I.decode()
    rng = np.random.default_rng(123)
    pairs = sorted({(int(rng.integers(64)), int(rng.integers(32))) for _ in range(12)} | {(0, 0), (63, 31)})
    _run_steps(setup, I.DECODE_STEPS, sample=pairs, check_every=64)
    import gated_deltanet_sequence_delta_b200 as G
    assert G.gdn_decode_status() == 0


@pytest.mark.parametrize("io,ab", [(I.BF16, I.BF16), (I.BF16, I.F32), (I.F32, I.F32)])
@pytest.mark.parametrize("D", [128, 64])
def test_decode_gated_equals_gates_then_step(io, ab, D):
    """The fused-gate step is bit-identical to gdn_gates followed by gdn_decode_step."""
    import torch
    import gated_deltanet_sequence_delta_b200 as G
    setup = I.decode(B=5, H=8, D=D, io_dtype=io, seed=17, HK=4)
    A_log, dt_bias = to_dev(setup.A_log), to_dev(setup.dt_bias)
    st1 = to_dev(setup.state0.copy())
    st2 = st1.clone()
    for s in range(4):
        q, k, v, a, b = setup.step(s)
        da, db = to_dev(a), to_dev(b)
        if ab == I.BF16:
            da, db = da.to(torch.bfloat16), db.to(torch.bfloat16)
        g, beta = G.gdn_gates(da, db, A_log, dt_bias)
        o1 = G.gdn_decode_step(to_dev(q), to_dev(k), to_dev(v), g, beta, st1, scale=setup.scale)
        o2 = G.gdn_decode_step_gated(to_dev(q), to_dev(k), to_dev(v), da, db, A_log, dt_bias, st2,
                                     scale=setup.scale)
        assert torch.equal(o1, o2), f"step {s}: o differs"
        assert torch.equal(st1, st2), f"step {s}: state differs"


def test_decode_gated_workload_vs_oracle():
    """B=64, H=32, d=128, bf16, gates fused: 16 steps on every (sequence, head)."""
    import gated_deltanet_sequence_delta_b200 as G
    setup = I.decode()
    _run_steps(setup, 16, fused_gates=True)
    assert G.gdn_decode_status() == 0


def test_decode_no_write_no_decay_keeps_state():
    """beta = 0, alpha = 1: the state is bit-for-bit unchanged (fp32)."""
    import torch
    import gated_deltanet_sequence_delta_b200 as G
    rng = np.random.default_rng(1)
    B, H, D = 4, 8, 128
    st0 = torch.from_numpy(rng.standard_normal((B, H, D, D)).astype(np.float32)).cuda()
    st = st0.clone()
    q = torch.randn(B, H, D, device="cuda")
    k = torch.randn(B, H, D, device="cuda")
    v = torch.randn(B, H, D, device="cuda")
    zeros = torch.zeros(B, H, device="cuda")
    G.gdn_decode_step(q, k, v, zeros, zeros, st)
    assert torch.equal(st, st0)
