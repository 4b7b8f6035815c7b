"""Seeded synthetic inputs for the Gated DeltaNet core.

This module only draws random numbers and rounds them to the storage dtype; it
holds none of the method's arithmetic.  It is the one module that both the CUDA
path's tests/bench and the CPU oracle consume, so that the two sides always see
bit-identical inputs.

Workloads (shapes follow the pages' setting: head dim 128, hybrid-model head
counts, 32K-256K contexts):

* ``tiny``    B=1, T=256, HK=HV=2, D=64, fp32, BT=64, zero initial state, seed 0
* ``decode``  B=64, HK=HV=32, D=128, bf16 q/k/v, fp32 state ~ N(0, 0.02^2),
              1024 consecutive one-token steps, seed 1
* ``long``    B=1, T=32768, HK=16, HV=32, D=128, bf16, BT=64, zero state, seed 2
* ``varlen``  65536 packed tokens, lengths ~ U_int[512, 8192] (last truncated),
              HK=16, HV=32, D=128, bf16, initial states ~ N(0, 0.02^2), seed 3
* ``stress``  B=1, T=262144, HK=HV=32, D=128, bf16, initial state
              ~ N(0, 0.02^2); 1% of tokens forced to g = -20 after the gates,
              1% (drawn independently) forced to b = +20 before them; seed 4

Value recipe (every workload): q, k ~ N(0, 1) then scaled to unit L2 norm per
(token, head); v ~ N(0, 1); a, b ~ N(0, 1) per (token, value head);
A_log = log(U(1, 16)) per value head; dt log-uniform in [1e-3, 1e-1] per value
head and dt_bias = log(expm1(dt)).  bf16 tensors are rounded to nearest-even
here, before either side sees them.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

F32 = "f32"
BF16 = "bf16"


# ---------------------------------------------------------------------------
# bf16 storage helpers (bit manipulation only)
# ---------------------------------------------------------------------------
def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (nearest, ties to even); return uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = ((u >> 16) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + r) >> 16).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


@dataclass
class Tensor:
    """A host tensor stored in its io dtype: float32 array, or uint16 bf16 bits."""
    data: np.ndarray
    dtype: str  # F32 | BF16

    @property
    def shape(self):
        return self.data.shape

    def f32(self, index=...) -> np.ndarray:
        d = self.data[index]
        return bf16_bits_to_f32(d) if self.dtype == BF16 else np.asarray(d, dtype=np.float32)

    def f64(self, index=...) -> np.ndarray:
        return self.f32(index).astype(np.float64)


def _store(x32: np.ndarray, dtype: str) -> Tensor:
    if dtype == BF16:
        return Tensor(f32_to_bf16_bits(x32), BF16)
    return Tensor(np.ascontiguousarray(x32, dtype=np.float32), F32)


# ---------------------------------------------------------------------------
# Draws
# ---------------------------------------------------------------------------
def _rng(seed: int, *stream: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, *stream])))


_STREAM = {"q": 1, "k": 2, "v": 3, "a": 4, "b": 5, "A_log": 6, "dt": 7, "h0": 8,
           "lens": 9, "reset": 10, "write": 11, "qnorm": 12, "knorm": 13}

_BLOCK = 1 << 24  # elements per generation block, bounds temporary fp32 memory


def _normal_rows(rng, rows: int, inner: tuple, dtype: str, unit_norm: bool, norm_rng=None,
                 norm_range=None) -> Tensor:
    """rows x inner standard normals (optionally unit-L2 along the last axis),
    generated in row blocks and stored in ``dtype``.  With ``norm_range`` = (lo, hi)
    each unit row is then given an L2 norm drawn from U(lo, hi) by ``norm_rng``."""
    n_inner = int(np.prod(inner)) if inner else 1
    store_dtype = np.uint16 if dtype == BF16 else np.float32
    out = np.empty((rows,) + tuple(inner), dtype=store_dtype)
    block = max(1, _BLOCK // n_inner)
    for r0 in range(0, rows, block):
        r1 = min(rows, r0 + block)
        x = rng.standard_normal((r1 - r0,) + tuple(inner), dtype=np.float32)
        if unit_norm:
            x /= np.sqrt(np.sum(x * x, axis=-1, keepdims=True, dtype=np.float32))
            if norm_range is not None:
                lo, hi = norm_range
                x *= norm_rng.uniform(lo, hi, x.shape[:-1] + (1,)).astype(np.float32)
        out[r0:r1] = f32_to_bf16_bits(x) if dtype == BF16 else x
    return Tensor(out, dtype)


def gate_params(seed: int, HV: int):
    """A_log = log(U(1,16)); dt log-uniform [1e-3, 1e-1]; dt_bias = log(expm1(dt))."""
    A_log = np.log(_rng(seed, _STREAM["A_log"]).uniform(1.0, 16.0, HV)).astype(np.float32)
    u = _rng(seed, _STREAM["dt"]).uniform(np.log(1e-3), np.log(1e-1), HV)
    dt = np.exp(u)
    dt_bias = np.log(np.expm1(dt)).astype(np.float32)
    return A_log, dt_bias, dt.astype(np.float32)


@dataclass
class PrefillInputs:
    name: str
    B: int                 # batch rows of the dense layout (1 when packed)
    T: int                 # tokens per row (total tokens when packed)
    HK: int
    HV: int
    Dk: int
    Dv: int
    BT: int
    io_dtype: str
    seed: int
    q: Tensor              # [B, T, HK, Dk]
    k: Tensor              # [B, T, HK, Dk]
    v: Tensor              # [B, T, HV, Dv]
    a: np.ndarray          # [B, T, HV] float32
    b: np.ndarray          # [B, T, HV] float32
    A_log: np.ndarray      # [HV] float32
    dt_bias: np.ndarray    # [HV] float32
    h0: np.ndarray | None  # [N, HV, Dk, Dv] float32
    cu_seqlens: np.ndarray | None = None   # [N+1] int32 (packed form)
    g_reset: np.ndarray | None = None      # [B*T] bool: g forced to -20 after the gates
    scale: float = 1.0
    l2norm: bool = True
    extra: dict = field(default_factory=dict)

    @property
    def n_seqs(self) -> int:
        return self.B if self.cu_seqlens is None else int(self.cu_seqlens.size - 1)

    @property
    def n_tokens(self) -> int:
        return self.B * self.T

    def seq_bounds(self):
        if self.cu_seqlens is None:
            return [(i * self.T, (i + 1) * self.T) for i in range(self.B)]
        c = self.cu_seqlens
        return [(int(c[i]), int(c[i + 1])) for i in range(c.size - 1)]


def make_prefill(B: int, T: int, HK: int, HV: int, Dk: int, Dv: int, *, io_dtype: str,
                 seed: int, BT: int = 64, h0_std: float = 0.0, cu_seqlens=None,
                 reset_frac: float = 0.0, write_frac: float = 0.0, name: str = "custom",
                 scale: float = 1.0, l2norm: bool = True, qk_norm=None) -> PrefillInputs:
    """Draw one prefill problem with the value recipe in the module docstring.  With
    ``qk_norm`` = (lo, hi) the q and k rows get L2 norms drawn from U(lo, hi) instead of
    unit norm (``scale`` and ``l2norm`` are passed to both sides as they are)."""
    rows = B * T
    q = _normal_rows(_rng(seed, _STREAM["q"]), rows, (HK, Dk), io_dtype, True,
                     _rng(seed, _STREAM["qnorm"]), qk_norm)
    k = _normal_rows(_rng(seed, _STREAM["k"]), rows, (HK, Dk), io_dtype, True,
                     _rng(seed, _STREAM["knorm"]), qk_norm)
    v = _normal_rows(_rng(seed, _STREAM["v"]), rows, (HV, Dv), io_dtype, False)
    a = _rng(seed, _STREAM["a"]).standard_normal((rows, HV), dtype=np.float32)
    b = _rng(seed, _STREAM["b"]).standard_normal((rows, HV), dtype=np.float32)
    A_log, dt_bias, dt = gate_params(seed, HV)
    n_seqs = B if cu_seqlens is None else len(cu_seqlens) - 1
    h0 = None
    if h0_std > 0:
        h0 = (h0_std * _rng(seed, _STREAM["h0"]).standard_normal(
            (n_seqs, HV, Dk, Dv), dtype=np.float32)).astype(np.float32)
    g_reset = None
    if reset_frac > 0:
        n = max(1, int(round(reset_frac * rows)))
        g_reset = np.zeros(rows, dtype=bool)
        g_reset[_rng(seed, _STREAM["reset"]).choice(rows, n, replace=False)] = True
    if write_frac > 0:
        n = max(1, int(round(write_frac * rows)))
        idx = _rng(seed, _STREAM["write"]).choice(rows, n, replace=False)
        b[idx, :] = 20.0
    cu = None if cu_seqlens is None else np.asarray(cu_seqlens, dtype=np.int32)
    inp = PrefillInputs(
        name=name, B=B, T=T, HK=HK, HV=HV, Dk=Dk, Dv=Dv, BT=BT, io_dtype=io_dtype, seed=seed,
        q=Tensor(q.data.reshape(B, T, HK, Dk), io_dtype),
        k=Tensor(k.data.reshape(B, T, HK, Dk), io_dtype),
        v=Tensor(v.data.reshape(B, T, HV, Dv), io_dtype),
        a=a.reshape(B, T, HV), b=b.reshape(B, T, HV), A_log=A_log, dt_bias=dt_bias,
        h0=h0, cu_seqlens=cu, g_reset=g_reset, scale=scale, l2norm=l2norm)
    inp.extra["dt"] = dt
    return inp


def outgate_inputs(n_tokens: int, HV: int, Dv: int, io_dtype: str, seed: int):
    """Gate inputs z [n_tokens, HV, Dv] ~ N(0, 1) in the io dtype and norm weights
    w [Dv] ~ N(0, 0.3^2) fp32 for the output epilogue."""
    z = _store(_rng(seed, 300, 1).standard_normal((n_tokens, HV, Dv), dtype=np.float32), io_dtype)
    w = (0.3 * _rng(seed, 300, 2).standard_normal(Dv, dtype=np.float32)).astype(np.float32)
    return z, w


def conv_prefill_inputs(n_tokens: int, n_seqs: int, HK: int, HV: int, D: int, io_dtype: str, seed: int,
                        with_state: bool = True):
    """Raw q | k | v projection rows x [n_tokens, C] (C = 2 HK D + HV D) ~ N(0, 1) in the io
    dtype, convolution weights conv_w [C, 4] ~ N(0, 0.5^2) fp32 and initial convolution
    states [n_seqs, C, 3] ~ N(0, 1) fp32 (None without ``with_state``): the recipe of the
    decode step from raw projections, over whole sequences."""
    C = 2 * HK * D + HV * D
    x = _normal_rows(_rng(seed, 400, 1), n_tokens, (C,), io_dtype, False)
    conv_w = (0.5 * _rng(seed, 400, 2).standard_normal((C, 4), dtype=np.float32)).astype(np.float32)
    state = _rng(seed, 400, 3).standard_normal((n_seqs, C, 3), dtype=np.float32) if with_state else None
    return x, conv_w, state


def varlen_lengths(seed: int, total: int = 65536, lo: int = 512, hi: int = 8192) -> np.ndarray:
    """Sequence lengths ~ U_int[lo, hi] until they sum to ``total`` (last one truncated)."""
    rng = _rng(seed, _STREAM["lens"])
    lens = []
    acc = 0
    while acc < total:
        L = int(rng.integers(lo, hi + 1))
        L = min(L, total - acc)
        lens.append(L)
        acc += L
    return np.asarray(lens, dtype=np.int64)


def cu_from_lengths(lens) -> np.ndarray:
    return np.concatenate([[0], np.cumsum(np.asarray(lens, dtype=np.int64))]).astype(np.int32)


# ---------------------------------------------------------------------------
# Named workloads
# ---------------------------------------------------------------------------
def tiny() -> PrefillInputs:
    return make_prefill(1, 256, 2, 2, 64, 64, io_dtype=F32, seed=0, BT=64, name="tiny")


def long_prefill(T: int = 32768) -> PrefillInputs:
    return make_prefill(1, T, 16, 32, 128, 128, io_dtype=BF16, seed=2, BT=64, name="long")


def varlen(total: int = 65536) -> PrefillInputs:
    cu = cu_from_lengths(varlen_lengths(3, total))
    return make_prefill(1, total, 16, 32, 128, 128, io_dtype=BF16, seed=3, BT=64,
                        h0_std=0.02, cu_seqlens=cu, name="varlen")


def stress(T: int = 262144) -> PrefillInputs:
    return make_prefill(1, T, 32, 32, 128, 128, io_dtype=BF16, seed=4, BT=64, h0_std=0.02,
                        reset_frac=0.01, write_frac=0.01, name="stress")


WORKLOADS = {"tiny": tiny, "long": long_prefill, "varlen": varlen, "stress": stress}


# ---------------------------------------------------------------------------
# Decode workload
# ---------------------------------------------------------------------------
@dataclass
class DecodeSetup:
    B: int
    HK: int
    HV: int
    Dk: int
    Dv: int
    io_dtype: str
    seed: int
    state0: np.ndarray     # [B, HV, Dk, Dv] float32
    A_log: np.ndarray
    dt_bias: np.ndarray
    scale: float = 1.0
    l2norm: bool = True
    qk_norm: tuple | None = None   # (lo, hi): q, k row norms ~ U(lo, hi) instead of 1

    def step(self, s: int):
        """Inputs of step ``s``: q, k [B, HK, Dk], v [B, HV, Dv] (Tensor),
        a, b [B, HV] float32.  Each step has its own seeded stream."""
        seed = self.seed
        q = _normal_rows(_rng(seed, 100, s, 1), self.B, (self.HK, self.Dk), self.io_dtype, True,
                         _rng(seed, 100, s, 6), self.qk_norm)
        k = _normal_rows(_rng(seed, 100, s, 2), self.B, (self.HK, self.Dk), self.io_dtype, True,
                         _rng(seed, 100, s, 7), self.qk_norm)
        v = _normal_rows(_rng(seed, 100, s, 3), self.B, (self.HV, self.Dv), self.io_dtype, False)
        a = _rng(seed, 100, s, 4).standard_normal((self.B, self.HV), dtype=np.float32)
        b = _rng(seed, 100, s, 5).standard_normal((self.B, self.HV), dtype=np.float32)
        return q, k, v, a, b


def decode(B: int = 64, H: int = 32, D: int = 128, io_dtype: str = BF16, seed: int = 1,
           HK: int | None = None) -> DecodeSetup:
    HK = H if HK is None else HK
    A_log, dt_bias, _ = gate_params(seed, H)
    state0 = (0.02 * _rng(seed, _STREAM["h0"]).standard_normal((B, H, D, D), dtype=np.float32))
    return DecodeSetup(B=B, HK=HK, HV=H, Dk=D, Dv=D, io_dtype=io_dtype, seed=seed,
                       state0=state0.astype(np.float32), A_log=A_log, dt_bias=dt_bias)


DECODE_STEPS = 1024


@dataclass
class FusedDecodeSetup:
    """A decode workload fed by raw projections: per step x [B, C] with C = 2 HK Dk +
    HV Dv (q | k | v channels), a, b [B, HV]; a kernel-4 convolution with weights
    conv_w [C, 4] ~ N(0, 0.5^2) and an initial convolution state conv_state0 [B, C, 3]
    ~ N(0, 1).  x ~ N(0, 1) rounded to the io dtype."""
    base: DecodeSetup
    conv_w: np.ndarray
    conv_state0: np.ndarray

    @property
    def C(self) -> int:
        b = self.base
        return 2 * b.HK * b.Dk + b.HV * b.Dv

    def out_z(self, s: int) -> Tensor:
        """Output-gate input of step ``s``: z [B, HV, Dv] ~ N(0, 1) in the io dtype."""
        b = self.base
        return _store(_rng(b.seed, 200, s, 9).standard_normal((b.B, b.HV, b.Dv), dtype=np.float32), b.io_dtype)

    def out_w(self) -> np.ndarray:
        """Output-norm weight w [Dv] ~ N(0, 0.3^2) fp32 (the recipe of outgate_inputs)."""
        b = self.base
        return (0.3 * _rng(b.seed, 200, 0, 10).standard_normal(b.Dv, dtype=np.float32)).astype(np.float32)

    def step(self, s: int):
        b = self.base
        x = _store(_rng(b.seed, 200, s, 1).standard_normal((b.B, self.C), dtype=np.float32), b.io_dtype)
        a = _rng(b.seed, 200, s, 4).standard_normal((b.B, b.HV), dtype=np.float32)
        bb = _rng(b.seed, 200, s, 5).standard_normal((b.B, b.HV), dtype=np.float32)
        return x, a, bb


def decode_fused(B: int = 64, H: int = 32, D: int = 128, io_dtype: str = BF16, seed: int = 1,
                 HK: int | None = None) -> FusedDecodeSetup:
    base = decode(B=B, H=H, D=D, io_dtype=io_dtype, seed=seed, HK=HK)
    C = 2 * base.HK * D + H * D
    conv_w = (0.5 * _rng(seed, 200, 0, 7).standard_normal((C, 4), dtype=np.float32)).astype(np.float32)
    conv_state0 = _rng(seed, 200, 0, 8).standard_normal((B, C, 3), dtype=np.float32)
    return FusedDecodeSetup(base=base, conv_w=conv_w, conv_state0=conv_state0)
