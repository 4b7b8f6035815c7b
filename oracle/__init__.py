"""CPU fp64 oracle of the Gated DeltaNet core -- test infrastructure only.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  The CUDA
library never imports, links or calls it, and this package imports nothing of
the CUDA library: the two share no code.  Only the seeded input generator module
(which holds none of the method's arithmetic) feeds both.

The arithmetic lives in ``gdn_oracle.c`` (plain fp64, one token at a time; see
its header for the formulas and the pages they come from).  This module builds
that file with gcc (OpenMP, -O2, no BLAS) and marshals numpy arrays to it.

Public functions (all fp64 numpy in, fp64 numpy out):

* ``gates(a, b, A_log, dt_bias) -> (g, beta)`` -- the gate formula of the
  "Gated DeltaNet ... Qwen3-next" page, section 2.1.
* ``recurrence(q, k, v, g, beta, h0=None, cu_seqlens=None, scale=1.0,
  l2norm=True) -> (o, hT)`` -- the gated delta rule of the Gated DeltaNet
  research-log page (third update rule), token by token.
* ``decode_step(q, k, v, g, beta, state, ...) -> (o, new_state)`` -- the same
  recurrence for one token per sequence, the incremental update of the
  "QWEN3.5" Q&A page (question 2a).
* ``out_gate(o, z, w, eps=1e-6) -> out`` -- the output epilogue: zero-centred
  RMSNorm over the last axis (Qwen3-next page, section 3.2) times (1 + w), times a
  sigmoid gate of z (the GDN resource-allocation page).
* ``conv(x, w, state=None, act=0) -> (y, new_state)`` -- the causal depthwise
  convolution of kernel 4 that the Qwen3-next page (section 3.1) puts before the
  gated update, with its rolling state of the three previous inputs.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import sys

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
DEFAULT_LIB = os.path.join(_BUILD_DIR, "libgdn_oracle.so")

_dp = ctypes.POINTER(ctypes.c_double)
_ip = ctypes.POINTER(ctypes.c_int64)


def build(src: str = _SRC, out: str = DEFAULT_LIB, force: bool = False) -> str:
    """Compile ``src`` into the shared library ``out`` (gcc -O2 -fopenmp)."""
    if (not force and os.path.exists(out)
            and os.path.getmtime(out) >= os.path.getmtime(src)):
        return out
    os.makedirs(os.path.dirname(out), exist_ok=True)
    tmp = out + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
           src, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


def _ptr(a: np.ndarray | None, kind=_dp):
    if a is None:
        return ctypes.cast(None, kind)
    return a.ctypes.data_as(kind)


def _f64(x) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


class OracleLib:
    """ctypes handle on one build of the oracle library."""

    def __init__(self, path: str):
        self.path = path
        lib = ctypes.CDLL(path)
        lib.gdn_oracle_gates.argtypes = [_dp, _dp, _dp, _dp, ctypes.c_int64,
                                         ctypes.c_int64, _dp, _dp]
        lib.gdn_oracle_gates.restype = None
        lib.gdn_oracle_recurrence.argtypes = [
            _dp, _dp, _dp, _dp, _dp, _dp, _ip, ctypes.c_int64, ctypes.c_int64,
            ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_double,
            ctypes.c_int, _dp, _dp, ctypes.c_int]
        lib.gdn_oracle_recurrence.restype = ctypes.c_int
        lib.gdn_oracle_conv.argtypes = [_dp, _dp, _dp, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                         ctypes.c_int, _dp, _dp]
        lib.gdn_oracle_conv.restype = None
        lib.gdn_oracle_out_gate.argtypes = [_dp, _dp, _dp, ctypes.c_int64, ctypes.c_int64, ctypes.c_double, _dp]
        lib.gdn_oracle_out_gate.restype = None
        lib.gdn_oracle_max_threads.argtypes = []
        lib.gdn_oracle_max_threads.restype = ctypes.c_int
        self.lib = lib

    def max_threads(self) -> int:
        return int(self.lib.gdn_oracle_max_threads())

    # -- gates -----------------------------------------------------------
    def gates(self, a, b, A_log, dt_bias):
        a = _f64(a)
        b = _f64(b)
        A_log = _f64(A_log)
        dt_bias = _f64(dt_bias)
        HV = A_log.shape[-1]
        if a.shape != b.shape or a.shape[-1] != HV or dt_bias.shape != (HV,):
            raise ValueError("gates: a, b must be [..., HV]; A_log, dt_bias [HV]")
        n = a.size // HV
        g = np.empty_like(a)
        beta = np.empty_like(a)
        self.lib.gdn_oracle_gates(_ptr(a), _ptr(b), _ptr(A_log), _ptr(dt_bias),
                                  n, HV, _ptr(g), _ptr(beta))
        return g, beta

    # -- recurrence ------------------------------------------------------
    def recurrence(self, q, k, v, g, beta, h0=None, cu_seqlens=None,
                   scale: float = 1.0, l2norm: bool = True, threads: int = 0):
        """Run the gated delta rule.

        Dense form: q, k [B, T, HK, Dk]; v [B, T, HV, Dv]; g, beta [B, T, HV];
        h0 [B, HV, Dk, Dv] or None.  Returns o [B, T, HV, Dv] and
        hT [B, HV, Dk, Dv].

        Packed form (``cu_seqlens`` given): q, k [T_total, HK, Dk] (a leading
        batch axis of 1 is accepted); returns o [T_total, HV, Dv] (same leading
        axes as v) and hT [N, HV, Dk, Dv].
        """
        q, k, v, g, beta = map(_f64, (q, k, v, g, beta))
        out_shape = v.shape
        if cu_seqlens is None:
            if q.ndim != 4:
                raise ValueError("dense form wants q of shape [B, T, HK, Dk]")
            B, T = q.shape[:2]
            cu = np.arange(B + 1, dtype=np.int64) * T
        else:
            cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64))
        n_seqs = cu.size - 1
        HK, Dk = q.shape[-2:]
        HV, Dv = v.shape[-2:]
        q = q.reshape(-1, HK, Dk)
        k = k.reshape(-1, HK, Dk)
        v = v.reshape(-1, HV, Dv)
        g = g.reshape(-1, HV)
        beta = beta.reshape(-1, HV)
        T_total = q.shape[0]
        if (k.shape != q.shape or v.shape[0] != T_total or g.shape != (T_total, HV)
                or beta.shape != (T_total, HV) or cu[-1] != T_total):
            raise ValueError("recurrence: inconsistent shapes")
        if h0 is not None:
            h0 = _f64(h0).reshape(n_seqs, HV, Dk, Dv)
        o = np.empty((T_total, HV, Dv))
        hT = np.empty((n_seqs, HV, Dk, Dv))
        rc = self.lib.gdn_oracle_recurrence(
            _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(h0),
            _ptr(cu, _ip), n_seqs, HK, HV, Dk, Dv, float(scale), int(bool(l2norm)),
            _ptr(o), _ptr(hT), int(threads))
        if rc != 0:
            raise ValueError(f"gdn_oracle_recurrence failed with code {rc}")
        return o.reshape(out_shape), hT

    # -- output epilogue ---------------------------------------------------
    def out_gate(self, o, z, w, eps: float = 1e-6):
        """o, z [..., D]; w [D].  Returns o * rsqrt(mean(o^2) + eps) * (1 + w) * sigmoid(z)."""
        o = _f64(o)
        z = _f64(z)
        w = _f64(w)
        D = o.shape[-1]
        if z.shape != o.shape or w.shape != (D,):
            raise ValueError("out_gate: o, z must share a shape [..., D]; w must be [D]")
        out = np.empty_like(o)
        self.lib.gdn_oracle_out_gate(_ptr(o), _ptr(z), _ptr(w), o.size // D, D, float(eps), _ptr(out))
        return out

    # -- convolution prologue --------------------------------------------
    def conv(self, x, w, state=None, act: int = 0):
        """x [B, T, C]; w [C, 4] (taps oldest first); state [B, C, 3] or None.
        Returns (y [B, T, C], new state [B, C, 3])."""
        x = _f64(x)
        w = _f64(w)
        if x.ndim != 3 or w.shape != (x.shape[2], 4):
            raise ValueError("conv: x must be [B, T, C] and w [C, 4]")
        B, T, C = x.shape
        if state is not None:
            state = _f64(state)
            if state.shape != (B, C, 3):
                raise ValueError("conv: state must be [B, C, 3]")
        y = np.empty_like(x)
        new_state = np.empty((B, C, 3))
        self.lib.gdn_oracle_conv(_ptr(x), _ptr(w), _ptr(state), B, T, C, int(act), _ptr(y), _ptr(new_state))
        return y, new_state

    def decode_step(self, q, k, v, g, beta, state, scale: float = 1.0,
                    l2norm: bool = True, threads: int = 0):
        """One token per sequence: q, k [B, HK, Dk]; v [B, HV, Dv];
        g, beta [B, HV]; state [B, HV, Dk, Dv].  Returns (o [B, HV, Dv],
        new state [B, HV, Dk, Dv]); the input state is not modified."""
        q = _f64(q)
        B = q.shape[0]
        cu = np.arange(B + 1, dtype=np.int64)
        return self.recurrence(q, k, v, g, beta, h0=state, cu_seqlens=cu,
                               scale=scale, l2norm=l2norm, threads=threads)


_DEFAULT: OracleLib | None = None


def default() -> OracleLib:
    global _DEFAULT
    if _DEFAULT is None:
        _DEFAULT = OracleLib(build())
    return _DEFAULT


def gates(a, b, A_log, dt_bias):
    return default().gates(a, b, A_log, dt_bias)


def recurrence(q, k, v, g, beta, h0=None, cu_seqlens=None, scale=1.0,
               l2norm=True, threads=0):
    return default().recurrence(q, k, v, g, beta, h0=h0, cu_seqlens=cu_seqlens,
                                scale=scale, l2norm=l2norm, threads=threads)


def out_gate(o, z, w, eps=1e-6):
    return default().out_gate(o, z, w, eps=eps)


def conv(x, w, state=None, act=0):
    return default().conv(x, w, state=state, act=act)


def decode_step(q, k, v, g, beta, state, scale=1.0, l2norm=True, threads=0):
    return default().decode_step(q, k, v, g, beta, state, scale=scale,
                                 l2norm=l2norm, threads=threads)


def max_threads() -> int:
    return default().max_threads()


if __name__ == "__main__":  # pragma: no cover
    print(build(force="--force" in sys.argv))
