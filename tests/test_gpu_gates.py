"""gdn_gates on the GPU against the oracle's fp64 gates."""
import numpy as np
import pytest

from harness import to_dev, to_np

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("ab_dtype", ["f32", "bf16"])
def test_gates_match_oracle(ab_dtype):
    import torch
    import oracle
    import gated_deltanet_sequence_delta_b200 as G
    rng = np.random.default_rng(0)
    HV = 32
    a = np.concatenate([rng.standard_normal((1000, HV)) * 4,
                        np.linspace(-80, 80, 8 * HV).reshape(8, HV)]).astype(np.float32)
    b = np.concatenate([rng.standard_normal((1000, HV)) * 4,
                        np.linspace(-60, 60, 8 * HV).reshape(8, HV)]).astype(np.float32)
    A_log = np.log(rng.uniform(1, 16, HV)).astype(np.float32)
    dt = np.exp(rng.uniform(np.log(1e-3), np.log(1e-1), HV))
    dt_bias = np.log(np.expm1(dt)).astype(np.float32)
    ta, tb = to_dev(a), to_dev(b)
    if ab_dtype == "bf16":
        ta, tb = ta.to(torch.bfloat16), tb.to(torch.bfloat16)
        a = ta.float().cpu().numpy()
        b = tb.float().cpu().numpy()
    g, beta = G.gdn_gates(ta, tb, to_dev(A_log), to_dev(dt_bias))
    g_ref, beta_ref = oracle.gates(a, b, A_log, dt_bias)
    g_g, b_g = to_np(g), to_np(beta)
    # fp32 transcendental evaluation: a few ulp of relative error
    np.testing.assert_allclose(g_g, g_ref, rtol=2e-6, atol=1e-30)
    np.testing.assert_allclose(b_g, beta_ref, rtol=2e-6, atol=1e-30)


def test_gates_empty_and_shapes():
    import torch
    import gated_deltanet_sequence_delta_b200 as G
    z = torch.empty((0, 4), device="cuda")
    g, beta = G.gdn_gates(z, z.clone(), torch.zeros(4, device="cuda"), torch.zeros(4, device="cuda"))
    assert g.shape == (0, 4) and beta.shape == (0, 4)
