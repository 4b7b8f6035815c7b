"""gdn_chunk_prefill on the GPU against the oracle, plus self-consistency and edge
cases.  Small cases compare every element; the full-size workloads compare
sampled value heads over the whole sequence (the oracle computes those heads
one by one)."""
import numpy as np
import pytest

from gated_deltanet_sequence_delta_b200 import inputs as I
from harness import TOL, assert_close, check_prefill, gpu_prefill, oracle_prefill, to_dev, to_np

pytestmark = pytest.mark.gpu


def test_tiny_workload_fp32():
    """B=1, T=256, H=2, d=64, fp32, BT=64: every element at 1e-4 * RMS."""
    check_prefill(I.tiny())


@pytest.mark.parametrize("BT", [16, 32, 64])
@pytest.mark.parametrize("D", [64, 128])
def test_fp32_chunk_sizes_ragged(BT, D):
    inp = I.make_prefill(2, 203, 2, 4, D, D, io_dtype=I.F32, seed=7, BT=BT, h0_std=0.1)
    check_prefill(inp)


@pytest.mark.parametrize("D", [(128, 128), (64, 64), (64, 128), (128, 64)])
def test_bf16_dense_ragged(D):
    Dk, Dv = D
    inp = I.make_prefill(2, 333, 2, 4, Dk, Dv, io_dtype=I.BF16, seed=8, h0_std=0.05)
    check_prefill(inp)


@pytest.mark.parametrize("io", [I.F32, I.BF16])
def test_varlen_small(io):
    lens = [1, 63, 64, 65, 0, 200, 129, 7]
    inp = I.make_prefill(1, int(sum(lens)), 2, 4, 128, 128, io_dtype=io, seed=9, h0_std=0.05,
                         cu_seqlens=I.cu_from_lengths(lens))
    check_prefill(inp)


@pytest.mark.parametrize("packed", [False, True])
def test_bf16_gqa_group4(packed):
    """Four value heads per q/k head (HK=2, HV=8) on the tensor-core path: dense ragged or
    packed sequences, with initial states."""
    if packed:
        lens = [70, 1, 191, 0, 64]
        inp = I.make_prefill(1, int(sum(lens)), 2, 8, 128, 128, io_dtype=I.BF16, seed=12, h0_std=0.05,
                             cu_seqlens=I.cu_from_lengths(lens))
    else:
        inp = I.make_prefill(2, 333, 2, 8, 128, 128, io_dtype=I.BF16, seed=12, h0_std=0.05)
    check_prefill(inp)


def test_stress_gates_small():
    """Forced resets (g = -20) and full writes (b = +20) at 1% each, T=4096."""
    inp = I.make_prefill(1, 4096, 4, 4, 128, 128, io_dtype=I.BF16, seed=10, h0_std=0.02,
                         reset_frac=0.01, write_frac=0.01)
    check_prefill(inp)


def test_single_token_and_empty():
    for T in (1, 2):
        check_prefill(I.make_prefill(1, T, 1, 2, 128, 128, io_dtype=I.BF16, seed=11, h0_std=0.1))
    import gated_deltanet_sequence_delta_b200 as G
    import torch
    # all-empty packed batch: final states equal the initial ones
    h0 = torch.randn(3, 2, 128, 128, device="cuda")
    cu = torch.zeros(4, dtype=torch.int32, device="cuda")
    e = torch.empty((1, 0, 1, 128), dtype=torch.bfloat16, device="cuda")
    ev = torch.empty((1, 0, 2, 128), dtype=torch.bfloat16, device="cuda")
    eg = torch.empty((1, 0, 2), device="cuda")
    o, hT = G.gdn_chunk_prefill(e, e, ev, eg, eg, initial_state=h0, cu_seqlens=cu)
    assert o.shape == (1, 0, 2, 128)
    assert torch.equal(hT, h0)


def test_bt_independence_fp32():
    """BT changes rounding only: BT = 16, 32, 64 agree to fp32 accuracy."""
    inp = I.make_prefill(1, 500, 2, 2, 128, 128, io_dtype=I.F32, seed=12, h0_std=0.1)
    outs = [gpu_prefill(inp, BT=bt) for bt in (16, 32, 64)]
    for o, hT, _, _ in outs[1:]:
        assert_close(to_np(o), to_np(outs[0][0]), 1e-5, "o across BT")
        assert_close(to_np(hT), to_np(outs[0][1]), 1e-5, "state across BT")


def test_bt_independence_bf16():
    """bf16 with 128-dim heads: BT = 64 on the tensor cores (fp16 intermediates), BT = 32
    and 16 on CUDA cores (fp32 throughout).  Each agrees with the oracle within the bf16
    bound; the two CUDA-core chunk lengths give the same fp32 final state to fp32 accuracy
    (the chunk length changes only where sums are rounded).  Their bf16 outputs are not
    compared with each other: two roundings of nearly equal values may land one bf16 step
    apart, more than the half step the bound allows against the exact result."""
    inp = I.make_prefill(2, 333, 2, 4, 128, 128, io_dtype=I.BF16, seed=13, h0_std=0.05)
    o_ref, h_ref = oracle_prefill(inp)
    tol = TOL[I.BF16]
    outs = {}
    for bt in (64, 32, 16):
        o, hT, _, _ = gpu_prefill(inp, BT=bt)
        assert_close(to_np(o), o_ref, tol, f"bf16, BT {bt}: o", out_bf16=True)
        assert_close(to_np(hT), h_ref, tol, f"bf16, BT {bt}: final state")
        outs[bt] = (to_np(o), to_np(hT))
    assert_close(outs[16][1], outs[32][1], TOL[I.F32], "bf16 state, BT 16 against BT 32")


@pytest.mark.parametrize("io", [I.F32, I.BF16])
def test_varlen_equals_separate_calls(io):
    import gated_deltanet_sequence_delta_b200 as G
    lens = [70, 0, 129, 64, 5]
    inp = I.make_prefill(1, int(sum(lens)), 2, 4, 128, 128, io_dtype=io, seed=13, h0_std=0.05,
                         cu_seqlens=I.cu_from_lengths(lens))
    o, hT, g, beta = gpu_prefill(inp)
    q, k, v, h0 = to_dev(inp.q), to_dev(inp.k), to_dev(inp.v), to_dev(inp.h0)
    cu = inp.cu_seqlens
    for n in range(len(lens)):
        s, e = int(cu[n]), int(cu[n + 1])
        on, hn = G.gdn_chunk_prefill(q[:, s:e].contiguous(), k[:, s:e].contiguous(),
                                     v[:, s:e].contiguous(), g[:, s:e].contiguous(),
                                     beta[:, s:e].contiguous(), initial_state=h0[n:n + 1].contiguous())
        assert np.array_equal(to_np(on), to_np(o[:, s:e]))
        assert np.array_equal(to_np(hn[0]), to_np(hT[n]))


@pytest.mark.parametrize("io", [I.F32, I.BF16])
def test_state_carry_and_decode_continuation(io):
    """prefill(T) = prefill(first part) then prefill(rest) from its final state, and
    prefill(T) then one decode step = prefill(T + 1)."""
    import gated_deltanet_sequence_delta_b200 as G
    inp = I.make_prefill(1, 257, 2, 4, 128, 128, io_dtype=io, seed=14, h0_std=0.05)
    o, hT, g, beta = gpu_prefill(inp)
    q, k, v, h0 = to_dev(inp.q), to_dev(inp.k), to_dev(inp.v), to_dev(inp.h0)
    tol = TOL[io]
    for cut in (64, 100):
        oa, ha = G.gdn_chunk_prefill(q[:, :cut].contiguous(), k[:, :cut].contiguous(),
                                     v[:, :cut].contiguous(), g[:, :cut].contiguous(),
                                     beta[:, :cut].contiguous(), initial_state=h0)
        ob, hb = G.gdn_chunk_prefill(q[:, cut:].contiguous(), k[:, cut:].contiguous(),
                                     v[:, cut:].contiguous(), g[:, cut:].contiguous(),
                                     beta[:, cut:].contiguous(), initial_state=ha)
        assert_close(to_np(oa), to_np(o[:, :cut]), tol, "carry: first part", out_bf16=io == I.BF16)
        assert_close(to_np(ob), to_np(o[:, cut:]), tol, "carry: second part", out_bf16=io == I.BF16)
        assert_close(to_np(hb), to_np(hT), tol, "carry: state")
    T = 256
    op, hp = G.gdn_chunk_prefill(q[:, :T].contiguous(), k[:, :T].contiguous(), v[:, :T].contiguous(),
                                 g[:, :T].contiguous(), beta[:, :T].contiguous(), initial_state=h0)
    st = hp.clone()
    od = G.gdn_decode_step(q[:, T].contiguous(), k[:, T].contiguous(), v[:, T].contiguous(),
                           g[:, T].contiguous(), beta[:, T].contiguous(), st)
    assert_close(to_np(od), to_np(o[:, T]), tol, "decode continuation: o", out_bf16=io == I.BF16)
    assert_close(to_np(st), to_np(hT), tol, "decode continuation: state")


def test_in_place_state_and_canaries():
    """final_state may be the initial_state buffer; nothing past the outputs is written."""
    import torch
    import gated_deltanet_sequence_delta_b200 as G
    inp = I.make_prefill(1, 130, 2, 4, 128, 128, io_dtype=I.BF16, seed=15, h0_std=0.05)
    o_ref, h_ref, g, beta = gpu_prefill(inp)
    q, k, v = to_dev(inp.q), to_dev(inp.k), to_dev(inp.v)
    n_o = o_ref.numel()
    o_buf = torch.full((n_o + 4096,), 7.0, dtype=torch.bfloat16, device="cuda")
    st_buf = torch.full((h_ref.numel() + 4096,), -3.0, device="cuda")
    st_buf[:h_ref.numel()] = to_dev(inp.h0).flatten()
    o = o_buf[:n_o].view(o_ref.shape)
    st = st_buf[:h_ref.numel()].view(h_ref.shape)
    G.gdn_chunk_prefill(q, k, v, g, beta, initial_state=st, o=o, final_state=st)
    assert torch.equal(o, o_ref) and torch.equal(st, h_ref)
    assert torch.all(o_buf[n_o:] == 7.0) and torch.all(st_buf[h_ref.numel():] == -3.0)


def test_bad_cu_seqlens_reported_and_nothing_written():
    import torch
    import gated_deltanet_sequence_delta_b200 as G
    inp = I.make_prefill(1, 96, 1, 2, 128, 128, io_dtype=I.BF16, seed=16)
    q, k, v = to_dev(inp.q), to_dev(inp.k), to_dev(inp.v)
    g = torch.zeros(1, 96, 2, device="cuda")
    for bad in ([0, 50, 40, 96], [1, 50, 96], [0, 50, 95]):
        cu = torch.tensor(bad, dtype=torch.int32, device="cuda")
        n = len(bad) - 1
        ws = torch.empty(G.prefill_workspace_bytes(96, n, 1, 2, 128, 128, 64, 1), dtype=torch.uint8,
                         device="cuda")
        o = torch.full((1, 96, 2, 128), 5.0, dtype=torch.bfloat16, device="cuda")
        hT = torch.full((n, 2, 128, 128), 9.0, device="cuda")
        G.gdn_chunk_prefill(q, k, v, g, g, cu_seqlens=cu, o=o, final_state=hT, workspace=ws)
        assert G.gdn_chunk_prefill_status(ws) == 1
        assert torch.all(o == 5.0) and torch.all(hT == 9.0)
    cu = torch.tensor([0, 40, 96], dtype=torch.int32, device="cuda")
    ws = torch.empty(G.prefill_workspace_bytes(96, 2, 1, 2, 128, 128, 64, 1), dtype=torch.uint8,
                     device="cuda")
    G.gdn_chunk_prefill(q, k, v, g, g, cu_seqlens=cu, workspace=ws)
    assert G.gdn_chunk_prefill_status(ws) == 0


# ---------------------------------------------------------------------------
# full-size workloads: every value head (the 256K-token one in batches of eight heads,
# so that the oracle's fp64 copies stay within a few GB of host memory)
# ---------------------------------------------------------------------------
def test_long_workload_all_heads():
    """T=32768, HK=16, HV=32, d=128, bf16, BT=64: all 32 value heads."""
    inp = I.long_prefill()
    check_prefill(inp)


def test_varlen_workload_all_heads():
    """65536 packed tokens (lengths U[512, 8192]), per-sequence initial states, all heads."""
    inp = I.varlen()
    check_prefill(inp)


def test_stress_workload_all_heads():
    """T=262144, H=32, forced resets and full writes at 1% each: every value head, the
    oracle taking eight heads at a time."""
    inp = I.stress()
    o, hT, _, _ = gpu_prefill(inp)
    tol = TOL[inp.io_dtype]
    for h0 in range(0, inp.HV, 8):
        heads = list(range(h0, h0 + 8))
        o_ref, h_ref = oracle_prefill(inp, heads)
        assert_close(to_np(o[:, :, heads]), o_ref, tol, f"stress: o, heads {h0}-{h0 + 7}", out_bf16=True)
        assert_close(to_np(hT[:, heads]), h_ref, tol, f"stress: final state, heads {h0}-{h0 + 7}")
        del o_ref, h_ref
