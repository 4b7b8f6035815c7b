"""Context-parallel prefill on CPU with two gloo ranks (spawned processes): each rank takes
one segment of the same sequence, forms the segment's affine transition (A, B) and its
outputs o0 and c with the oracle (which stands in for the GPU kernels here), exchanges
(A, B) through context_parallel.gather_transitions, and checks the scan to its start
state, the final state and its corrected outputs against the oracle run over the whole
sequence.  This pins the decomposition H_end = A H_start + B, o_t = o0_t + H_start^T c_t
(exact in fp64) and the collective's plumbing; the combine kernel is checked on the GPU."""
import os
import socket
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _problem(T, HK, HV, D, seed):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((T, HK, D))
    k = rng.standard_normal((T, HK, D))
    v = rng.standard_normal((T, HV, D))
    g = -np.abs(rng.standard_normal((T, HV))) * 0.3
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((T, HV))))
    h0 = 0.1 * rng.standard_normal((1, HV, D, D))
    return q, k, v, g, beta, h0


def _rank_main(rank, world, port, out_dir, T_seg, HK, HV, D):
    import datetime
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import oracle
    from gated_deltanet_sequence_delta_b200 import context_parallel as CP
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        q, k, v, g, beta, h0 = _problem(world * T_seg, HK, HV, D, 11)
        seg = slice(rank * T_seg, (rank + 1) * T_seg)
        cu = np.array([0, T_seg])
        o0, Bs = oracle.recurrence(q[seg], k[seg], v[seg], g[seg], beta[seg], cu_seqlens=cu)
        eye = np.broadcast_to(np.eye(D), (1, HV, D, D)).copy()
        c, As = oracle.recurrence(q[seg], k[seg], np.zeros_like(v[seg]), g[seg], beta[seg], h0=eye, cu_seqlens=cu)
        A_all, B_all = CP.gather_transitions(torch.from_numpy(As), torch.from_numpy(Bs))
        A_all, B_all = A_all.numpy(), B_all.numpy()
        H = h0.copy()
        start = None
        for r in range(world):   # the scan the combine step performs
            if r == rank:
                start = H.copy()
            H = np.einsum("nhij,nhjk->nhik", A_all[r], H) + B_all[r]
        o = o0 + np.einsum("thk,hkj->thj", c, start[0])
        np.savez(os.path.join(out_dir, f"rank{rank}.npz"), o=o, start=start, final=H)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_context_parallel(tmp_path):
    import torch.multiprocessing as mp
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import oracle
    world, T_seg, HK, HV, D = 2, 37, 1, 2, 8
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path), T_seg, HK, HV, D), nprocs=world,
                       join=True, start_method="spawn")
    q, k, v, g, beta, h0 = _problem(world * T_seg, HK, HV, D, 11)
    o_ref, h_ref = oracle.recurrence(q, k, v, g, beta, h0=h0, cu_seqlens=np.array([0, world * T_seg]))
    _, h_mid = oracle.recurrence(q[:T_seg], k[:T_seg], v[:T_seg], g[:T_seg], beta[:T_seg], h0=h0,
                                 cu_seqlens=np.array([0, T_seg]))
    res = [np.load(tmp_path / f"rank{r}.npz") for r in range(world)]
    np.testing.assert_allclose(res[0]["start"], h0, rtol=0, atol=1e-12)
    np.testing.assert_allclose(res[1]["start"], h_mid, rtol=0, atol=1e-10)
    for r in range(world):
        np.testing.assert_allclose(res[r]["final"], h_ref, rtol=0, atol=1e-10)
        np.testing.assert_allclose(res[r]["o"], o_ref[r * T_seg:(r + 1) * T_seg], rtol=0, atol=1e-10)
