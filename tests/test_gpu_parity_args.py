"""Parity of the API's arguments that the workloads leave at their defaults: ``scale``
other than 1, ``qk_l2norm`` off, and q / k rows whose norms are far from 1, on every
prefill and decode kernel, each against the oracle element by element.

With the norm on, q and k rows get norms drawn from U(0.1, 10), so the kernels'
normalisation is far from the identity.  With it off, the norms are drawn from
U(0.1, 1): the rule is then stable only for beta |k|^2 <= 1 (the transition
I - beta k k^T has the eigenvalue 1 - beta |k|^2), so larger raw keys would make every
implementation diverge, the oracle included.  The paths:

* tensor-core prefill: bf16, Dk = Dv = 128, GQA groups 1, 2 and 4;
* CUDA-core prefill: fp32 (d = 128, BT 32 and 64) and bf16 with d = 64;
* staged decode (d = 128, bf16 and fp32) and per-thread decode (d = 64; 128 x 64);
* the decode step with the gates fused in, and the decode step from raw projections.
"""
import dataclasses

import numpy as np
import pytest

from gated_deltanet_sequence_delta_b200 import inputs as I
from harness import check_prefill
from test_gpu_decode import _run_steps

pytestmark = pytest.mark.gpu

# (qk_l2norm, q/k norm range, scale)
MODES = {
    "l2_norms_0.1-10_scale_0.5": (True, (0.1, 10.0), 0.5),
    "no_l2_norms_0.1-1_scale_0.125": (False, (0.1, 1.0), 0.125),
}


@pytest.mark.parametrize("mode", list(MODES))
@pytest.mark.parametrize("path", ["tc_bf16_g2", "tc_bf16_g1_packed", "tc_bf16_g4", "cudacore_f32_d128",
                                  "cudacore_f32_bt32", "cudacore_bf16_d64"])
def test_prefill_scale_norm_args(path, mode):
    l2, rng, scale = MODES[mode]
    kw = dict(scale=scale, l2norm=l2, qk_norm=rng, h0_std=0.05)
    if path == "tc_bf16_g2":
        inp = I.make_prefill(2, 333, 2, 4, 128, 128, io_dtype=I.BF16, seed=301, **kw)
    elif path == "tc_bf16_g1_packed":
        lens = [1, 64, 130, 0, 77]
        inp = I.make_prefill(1, int(sum(lens)), 3, 3, 128, 128, io_dtype=I.BF16, seed=302,
                             cu_seqlens=I.cu_from_lengths(lens), **kw)
    elif path == "tc_bf16_g4":
        inp = I.make_prefill(1, 260, 2, 8, 128, 128, io_dtype=I.BF16, seed=303, **kw)
    elif path == "cudacore_f32_d128":
        inp = I.make_prefill(2, 203, 2, 4, 128, 128, io_dtype=I.F32, seed=304, **kw)
    elif path == "cudacore_f32_bt32":
        inp = I.make_prefill(1, 150, 1, 2, 128, 128, io_dtype=I.F32, seed=305, BT=32, **kw)
    else:
        inp = I.make_prefill(2, 150, 2, 4, 64, 64, io_dtype=I.BF16, seed=306, **kw)
    inp.name = f"{path} {mode}"
    check_prefill(inp)


@pytest.mark.parametrize("mode", list(MODES))
@pytest.mark.parametrize("io", [I.BF16, I.F32])
@pytest.mark.parametrize("D", [(128, 128), (64, 64), (128, 64)])
def test_decode_scale_norm_args(D, io, mode):
    l2, rng, scale = MODES[mode]
    Dk, Dv = D
    setup = I.decode(B=3, H=4, D=Dk, io_dtype=io, seed=311, HK=2)
    if Dv != Dk:
        r = np.random.default_rng(312)
        setup = dataclasses.replace(setup, Dv=Dv, state0=(0.02 * r.standard_normal((3, 4, Dk, Dv))).astype(np.float32))
    setup = dataclasses.replace(setup, scale=scale, l2norm=l2, qk_norm=rng)
    _run_steps(setup, 8)


@pytest.mark.parametrize("mode", list(MODES))
@pytest.mark.parametrize("D", [128, 64])
def test_decode_gated_scale_norm_args(D, mode):
    l2, rng, scale = MODES[mode]
    setup = dataclasses.replace(I.decode(B=5, H=8, D=D, io_dtype=I.BF16, seed=313, HK=4), scale=scale, l2norm=l2,
                                qk_norm=rng)
    _run_steps(setup, 6, fused_gates=True)


@pytest.mark.parametrize("scale", [0.5, 2.0 ** -3.5])
def test_fused_decode_scale(scale):
    """The decode step from raw projections with scale != 1 (its q, k come out of the
    convolution with arbitrary norms, so the in-kernel normalisation is always exercised)."""
    from test_gpu_decode_fused import _run
    setup = I.decode_fused(B=3, H=4, D=128, io_dtype=I.BF16, seed=314, HK=2)
    setup = dataclasses.replace(setup, base=dataclasses.replace(setup.base, scale=scale))
    _run(setup, 4, 1)
