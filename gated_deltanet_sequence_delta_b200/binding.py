"""Thin Python binding over the C ABI of ``include/gdn.h`` (``libgdn.so``).

Argument marshalling only: every step of the computation runs in the library's
CUDA kernels.  PyTorch provides device memory and the current stream; outputs
that the caller does not pass are allocated here with ``torch.empty``.

The library is loaded on first use.  If ``libgdn.so`` is missing or cannot be
loaded, every call raises ``GDNLibraryError``: there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libgdn.so")
HEADER = os.path.join(os.path.dirname(_PKG), "include", "gdn.h")

GDN_F32, GDN_BF16 = 0, 1
STATUS_NAMES = {0: "GDN_OK", 1: "GDN_ERR_NULL", 2: "GDN_ERR_SHAPE", 3: "GDN_ERR_ALIGN",
                4: "GDN_ERR_UNSUPPORTED", 5: "GDN_ERR_ALIAS", 6: "GDN_ERR_WORKSPACE",
                7: "GDN_ERR_CUDA", 8: "GDN_ERR_DEVICE"}


class GDNLibraryError(RuntimeError):
    pass


class GDNError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(msg)
        self.status = status


_i32, _i64, _f32, _vp, _sz = ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_void_p, ctypes.c_size_t
_SIGS = {
    "gdn_status_string": ([ctypes.c_int], ctypes.c_char_p),
    "gdn_abi_version": ([], ctypes.c_int),
    "gdn_last_cuda_error": ([], ctypes.c_int),
    "gdn_kernel_launches": ([], ctypes.c_uint64),
    "gdn_gates": ([_vp, _vp, ctypes.c_int, _vp, _vp, _i64, _i32, _vp, _vp, _vp], ctypes.c_int),
    "gdn_chunk_prefill_workspace_bytes": ([_i64, _i32, _i32, _i32, _i32, _i32, _i32, ctypes.c_int], _sz),
    "gdn_chunk_prefill": ([_vp, _vp, _vp, ctypes.c_int, _vp, _vp, _vp, _vp, _i32, _i64, _i32, _i32,
                           _i32, _i32, _i32, _i32, _f32, _i32, _vp, _vp, _vp, _sz, _vp], ctypes.c_int),
    "gdn_chunk_prefill_status": ([_vp, _vp, ctypes.POINTER(_i32)], ctypes.c_int),
    "gdn_chunk_prefill_gated": ([_vp, _vp, _vp, ctypes.c_int, _vp, _vp, ctypes.c_int, _vp, _vp, _vp, _vp, _i32, _i64,
                                 _i32, _i32, _i32, _i32, _i32, _i32, _f32, _i32, _vp, _vp, _vp, _sz, _vp],
                                ctypes.c_int),
    "gdn_chunk_prefill_outgate": ([_vp, _vp, _vp, ctypes.c_int, _vp, _vp, _vp, _vp, _i32, _i64, _i32, _i32,
                                   _i32, _i32, _i32, _i32, _f32, _i32, _vp, _vp, _f32, _vp, _vp, _vp, _sz, _vp],
                                  ctypes.c_int),
    "gdn_decode_step": ([_vp, _vp, _vp, ctypes.c_int, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32,
                         _f32, _i32, _vp, _vp], ctypes.c_int),
    "gdn_decode_status": ([ctypes.POINTER(_i32)], ctypes.c_int),
    "gdn_testing_stall": ([_i32], ctypes.c_int),
    "gdn_conv_status": ([ctypes.POINTER(_i32)], ctypes.c_int),
    "gdn_cp_status": ([ctypes.POINTER(_i32)], ctypes.c_int),
    "gdn_cp_segment": ([_vp, _vp, _vp, ctypes.c_int, _vp, _vp, _vp, _vp, _i32, _i64, _i32, _i32, _i32, _i32, _i32,
                        _i32, _f32, _i32, _vp, _vp, _vp, _vp, _vp, _sz, _vp], ctypes.c_int),
    "gdn_cp_combine": ([_vp, _vp, _vp, _i32, _i32, _i32, _i64, _i32, _i32, _i32, ctypes.c_int, _vp, _vp, _vp, _vp,
                        _vp], ctypes.c_int),
    "gdn_decode_step_fused": ([_vp, ctypes.c_int, _vp, _vp, _vp, _i32, _vp, _vp, ctypes.c_int, _vp, _vp, _vp,
                               _i32, _i32, _i32, _i32, _i32, _f32, _i32, _vp, _vp], ctypes.c_int),
    "gdn_decode_step_fused_outgate": ([_vp, ctypes.c_int, _vp, _vp, _vp, _i32, _vp, _vp, ctypes.c_int, _vp, _vp,
                                       _vp, _i32, _i32, _i32, _i32, _i32, _f32, _i32, _vp, _vp, _f32, _vp, _vp],
                                      ctypes.c_int),
    "gdn_chunk_prefill_host_workspace_bytes": ([_i32, _i64, _i32, _i32, _i32, _i32, _i32, ctypes.c_int,
                                                ctypes.c_int, _i64], _sz),
    "gdn_chunk_prefill_host": ([_vp, _vp, _vp, ctypes.c_int, _vp, _vp, ctypes.c_int, _vp, _vp, _vp, _i32, _i64,
                                _i32, _i32, _i32, _i32, _i32, _f32, _i32, _i64, _vp, _vp, _vp, _sz, _vp],
                               ctypes.c_int),
    "gdn_conv_prefill": ([_vp, ctypes.c_int, _vp, _vp, _vp, _i32, _i64, _i32, _i32, _i32, _i32, _i32, _i32,
                          _vp, _vp, _vp, _vp, _vp], ctypes.c_int),
    "gdn_decode_step_gated": ([_vp, _vp, _vp, ctypes.c_int, _vp, _vp, ctypes.c_int, _vp, _vp, _vp, _i32, _i32,
                               _i32, _i32, _i32, _f32, _i32, _vp, _vp], ctypes.c_int),
}

_LIB = None


def header_functions(path: str = HEADER) -> list[str]:
    """Names of the functions ``include/gdn.h`` declares."""
    src = open(path).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*GDN_API\b[^(;]*?\b(gdn_\w+)\s*\(", src, re.M)))


def lib(path: str | None = None):
    """The loaded library (raises GDNLibraryError if it is not built)."""
    global _LIB
    if _LIB is not None and path is None:
        return _LIB
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise GDNLibraryError(
            f"{p} is not built; run `python -m gated_deltanet_sequence_delta_b200.build`")
    try:
        L = ctypes.CDLL(p)
    except OSError as e:  # pragma: no cover
        raise GDNLibraryError(f"cannot load {p}: {e}") from e
    for name, (argtypes, restype) in _SIGS.items():
        fn = getattr(L, name)
        fn.argtypes = argtypes
        fn.restype = restype
    if path is None:
        _LIB = L
    return L


def kernel_launches() -> int:
    """Kernels the library has launched in this process so far."""
    return int(lib().gdn_kernel_launches())


def _check(status: int, what: str):
    if status != 0:
        name = lib().gdn_status_string(status).decode()
        extra = ""
        if status == 7:
            extra = f" (cudaError {lib().gdn_last_cuda_error()})"
        raise GDNError(status, f"{what}: {name}{extra}")


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return GDN_BF16
    if t.dtype == torch.float32:
        return GDN_F32
    raise TypeError(f"unsupported dtype {t.dtype} (bf16 or fp32)")


def _ptr(t: torch.Tensor | None):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensors must be CUDA tensors")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return t.data_ptr()


def _hptr(t: torch.Tensor | None):
    """Address of a contiguous host (CPU) tensor, None for None."""
    if t is None:
        return None
    if t.is_cuda or not t.is_contiguous():
        raise ValueError("host tensors must be contiguous CPU tensors")
    return t.data_ptr()


def _stream():
    return torch.cuda.current_stream().cuda_stream


# ---------------------------------------------------------------------------
def gdn_gates(a: torch.Tensor, b: torch.Tensor, A_log: torch.Tensor, dt_bias: torch.Tensor,
              g: torch.Tensor | None = None, beta: torch.Tensor | None = None):
    """g = -exp(A_log) softplus(a + dt_bias), beta = sigmoid(b).
    a, b [..., HV] fp32/bf16; A_log, dt_bias [HV] fp32.  Returns fp32 (g, beta)."""
    HV = A_log.shape[-1]
    if a.shape != b.shape or a.shape[-1] != HV or a.dtype != b.dtype:
        raise ValueError("a, b must share shape [..., HV] and dtype")
    if A_log.dtype != torch.float32 or dt_bias.dtype != torch.float32:
        raise TypeError("A_log, dt_bias must be fp32")
    g = torch.empty(a.shape, dtype=torch.float32, device=a.device) if g is None else g
    beta = torch.empty(a.shape, dtype=torch.float32, device=a.device) if beta is None else beta
    n = a.numel() // HV
    st = lib().gdn_gates(_ptr(a), _ptr(b), _dtype_code(a), _ptr(A_log), _ptr(dt_bias), n, HV,
                         _ptr(g), _ptr(beta), _stream())
    _check(st, "gdn_gates")
    return g, beta


def prefill_workspace_bytes(n_tokens, n_seqs, HK, HV, Dk, Dv, BT, io_dtype) -> int:
    return int(lib().gdn_chunk_prefill_workspace_bytes(n_tokens, n_seqs, HK, HV, Dk, Dv, BT, io_dtype))


def gdn_chunk_prefill(q, k, v, g, beta, initial_state=None, cu_seqlens=None, BT: int = 64,
                      scale: float = 1.0, qk_l2norm: bool = True, output_final_state: bool = True,
                      o=None, final_state=None, workspace=None, outgate=None):
    """Chunked prefill.  Dense: q, k [B, T, HK, Dk], v [B, T, HV, Dv], g, beta [B, T, HV].
    Packed: B = 1 and cu_seqlens int32 [N + 1].  Returns (o, final_state or None)."""
    B, T, HK, Dk = q.shape
    HV, Dv = v.shape[-2:]
    if k.shape != q.shape or v.shape[:2] != (B, T) or g.shape != (B, T, HV) or beta.shape != g.shape:
        raise ValueError("inconsistent q/k/v/g/beta shapes")
    if k.dtype != q.dtype or v.dtype != q.dtype:
        raise TypeError("q, k, v must share one dtype")
    if g.dtype != torch.float32 or beta.dtype != torch.float32:
        raise TypeError("g, beta must be fp32")
    if cu_seqlens is not None:
        if cu_seqlens.dtype != torch.int32:
            raise TypeError("cu_seqlens must be int32")
        N = cu_seqlens.numel() - 1
    else:
        N = B
    dcode = _dtype_code(q)
    if o is None:
        o = torch.empty((B, T, HV, Dv), dtype=q.dtype, device=q.device)
    if final_state is None and output_final_state:
        final_state = torch.empty((N, HV, Dk, Dv), dtype=torch.float32, device=q.device)
    need = prefill_workspace_bytes(B * T, N, HK, HV, Dk, Dv, BT, dcode)
    if need == 0:
        _check(4, "gdn_chunk_prefill")
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    if outgate is None:
        st = lib().gdn_chunk_prefill(
            _ptr(q), _ptr(k), _ptr(v), dcode, _ptr(g), _ptr(beta), _ptr(initial_state),
            _ptr(cu_seqlens), B, T, N, HK, HV, Dk, Dv, BT, float(scale), int(bool(qk_l2norm)),
            _ptr(o), _ptr(final_state), _ptr(workspace), workspace.numel(), _stream())
        _check(st, "gdn_chunk_prefill")
    else:
        z, norm_w, eps = outgate
        if z.shape != o.shape or z.dtype != q.dtype or norm_w.shape != (Dv,) or norm_w.dtype != torch.float32:
            raise ValueError("z must be shaped and typed like o; norm_w fp32 [Dv]")
        st = lib().gdn_chunk_prefill_outgate(
            _ptr(q), _ptr(k), _ptr(v), dcode, _ptr(g), _ptr(beta), _ptr(initial_state),
            _ptr(cu_seqlens), B, T, N, HK, HV, Dk, Dv, BT, float(scale), int(bool(qk_l2norm)),
            _ptr(z), _ptr(norm_w), float(eps), _ptr(o), _ptr(final_state), _ptr(workspace), workspace.numel(),
            _stream())
        _check(st, "gdn_chunk_prefill_outgate")
    return o, final_state


def gdn_chunk_prefill_gated(q, k, v, a, b, A_log, dt_bias, initial_state=None, cu_seqlens=None, BT: int = 64,
                            scale: float = 1.0, qk_l2norm: bool = True, output_final_state: bool = True,
                            o=None, final_state=None, workspace=None):
    """Chunked prefill with the gate prologue fused in: a, b [B, T, HV] (fp32 or bf16) and
    A_log, dt_bias [HV] fp32 instead of g, beta (bit-identical to gdn_gates followed by
    gdn_chunk_prefill).  Tensor-core shapes only.  Returns (o, final_state or None)."""
    B, T, HK, Dk = q.shape
    HV, Dv = v.shape[-2:]
    if k.shape != q.shape or v.shape[:2] != (B, T) or a.shape != (B, T, HV) or b.shape != a.shape:
        raise ValueError("inconsistent q/k/v/a/b shapes")
    if k.dtype != q.dtype or v.dtype != q.dtype or b.dtype != a.dtype:
        raise TypeError("q, k, v must share one dtype, and a, b another")
    if A_log.dtype != torch.float32 or dt_bias.dtype != torch.float32:
        raise TypeError("A_log, dt_bias must be fp32")
    N = cu_seqlens.numel() - 1 if cu_seqlens is not None else B
    dcode = _dtype_code(q)
    if o is None:
        o = torch.empty((B, T, HV, Dv), dtype=q.dtype, device=q.device)
    if final_state is None and output_final_state:
        final_state = torch.empty((N, HV, Dk, Dv), dtype=torch.float32, device=q.device)
    need = prefill_workspace_bytes(B * T, N, HK, HV, Dk, Dv, BT, dcode)
    if need == 0:
        _check(4, "gdn_chunk_prefill_gated")
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    st = lib().gdn_chunk_prefill_gated(
        _ptr(q), _ptr(k), _ptr(v), dcode, _ptr(a), _ptr(b), _dtype_code(a), _ptr(A_log), _ptr(dt_bias),
        _ptr(initial_state), _ptr(cu_seqlens), B, T, N, HK, HV, Dk, Dv, BT, float(scale), int(bool(qk_l2norm)),
        _ptr(o), _ptr(final_state), _ptr(workspace), workspace.numel(), _stream())
    _check(st, "gdn_chunk_prefill_gated")
    return o, final_state


def gdn_chunk_prefill_outgate(q, k, v, g, beta, z, norm_w, eps: float = 1e-6, **kw):
    """gdn_chunk_prefill with the output epilogue: each output row of a value head becomes
    o * rsqrt(mean(o^2) + eps) * (1 + norm_w) * sigmoid(z); z like o, norm_w fp32 [Dv].
    Keyword arguments as gdn_chunk_prefill."""
    return gdn_chunk_prefill(q, k, v, g, beta, outgate=(z, norm_w, eps), **kw)


def gdn_chunk_prefill_status(workspace: torch.Tensor) -> int:
    """Synchronise the current stream and return the workspace's device error word."""
    word = _i32(0)
    st = lib().gdn_chunk_prefill_status(_ptr(workspace), _stream(), ctypes.byref(word))
    if st not in (0, 8):
        _check(st, "gdn_chunk_prefill_status")
    return int(word.value)


def gdn_decode_step(q, k, v, g, beta, state, scale: float = 1.0, qk_l2norm: bool = True, o=None):
    """One token per sequence: q, k [B, HK, Dk]; v [B, HV, Dv]; g, beta [B, HV] fp32;
    state [B, HV, Dk, Dv] fp32 updated in place.  Returns o [B, HV, Dv]."""
    B, HK, Dk = q.shape
    HV, Dv = v.shape[-2:]
    if k.shape != q.shape or v.shape[0] != B or g.shape != (B, HV) or beta.shape != (B, HV):
        raise ValueError("inconsistent decode shapes")
    if state.shape != (B, HV, Dk, Dv) or state.dtype != torch.float32:
        raise ValueError("state must be fp32 [B, HV, Dk, Dv]")
    if o is None:
        o = torch.empty((B, HV, Dv), dtype=q.dtype, device=q.device)
    st = lib().gdn_decode_step(_ptr(q), _ptr(k), _ptr(v), _dtype_code(q), _ptr(g), _ptr(beta),
                               _ptr(state), B, HK, HV, Dk, Dv, float(scale), int(bool(qk_l2norm)),
                               _ptr(o), _stream())
    _check(st, "gdn_decode_step")
    return o


def gdn_decode_step_gated(q, k, v, a, b, A_log, dt_bias, state, scale: float = 1.0, qk_l2norm: bool = True,
                          o=None):
    """gdn_decode_step with the gates formed in the kernel: a, b [B, HV] (fp32 or bf16),
    A_log, dt_bias [HV] fp32 instead of g, beta.  Returns o [B, HV, Dv]."""
    B, HK, Dk = q.shape
    HV, Dv = v.shape[-2:]
    if k.shape != q.shape or v.shape[0] != B or a.shape != (B, HV) or b.shape != (B, HV):
        raise ValueError("inconsistent decode shapes")
    if a.dtype != b.dtype or A_log.shape != (HV,) or dt_bias.shape != (HV,):
        raise ValueError("a, b must share a dtype; A_log, dt_bias must be [HV]")
    if A_log.dtype != torch.float32 or dt_bias.dtype != torch.float32:
        raise ValueError("A_log and dt_bias must be fp32")
    if state.shape != (B, HV, Dk, Dv) or state.dtype != torch.float32:
        raise ValueError("state must be fp32 [B, HV, Dk, Dv]")
    if o is None:
        o = torch.empty((B, HV, Dv), dtype=q.dtype, device=q.device)
    st = lib().gdn_decode_step_gated(_ptr(q), _ptr(k), _ptr(v), _dtype_code(q), _ptr(a), _ptr(b), _dtype_code(a),
                                     _ptr(A_log), _ptr(dt_bias), _ptr(state), B, HK, HV, Dk, Dv, float(scale),
                                     int(bool(qk_l2norm)), _ptr(o), _stream())
    _check(st, "gdn_decode_step_gated")
    return o


def prefill_host_workspace_bytes(B, T, HK, HV, Dk, Dv, BT, io_dtype, ab_dtype, piece_tokens) -> int:
    return int(lib().gdn_chunk_prefill_host_workspace_bytes(B, T, HK, HV, Dk, Dv, BT, io_dtype, ab_dtype,
                                                            piece_tokens))


def gdn_chunk_prefill_host(q, k, v, a, b, A_log, dt_bias, initial_state=None, BT: int = 64, scale: float = 1.0,
                           qk_l2norm: bool = True, piece_tokens: int = 4096, o=None, final_state=None,
                           workspace=None):
    """Gates + chunked prefill for host (CPU) tensors, pipelined through the GPU in pieces
    of ``piece_tokens`` tokens: q, k [B, T, HK, Dk]; v [B, T, HV, Dv]; a, b [B, T, HV];
    A_log, dt_bias [HV]; initial_state [B, HV, Dk, Dv] or None.  Returns host tensors
    (o, final_state).  Pinned host memory lets the copies overlap; the call synchronises
    nothing but the current stream waits for all of it."""
    B, T, HK, Dk = q.shape
    HV, Dv = v.shape[-2:]
    for t in (q, k, v, a, b, A_log, dt_bias):
        if t.is_cuda or not t.is_contiguous():
            raise ValueError("host inputs must be contiguous CPU tensors")
    if k.shape != q.shape or v.shape[:2] != (B, T) or a.shape != (B, T, HV) or b.shape != (B, T, HV):
        raise ValueError("inconsistent prefill shapes")
    if A_log.dtype != torch.float32 or dt_bias.dtype != torch.float32 or a.dtype != b.dtype:
        raise ValueError("A_log, dt_bias must be fp32; a, b must share a dtype")
    io, ab = _dtype_code(q), _dtype_code(a)
    if o is None:
        o = torch.empty((B, T, HV, Dv), dtype=q.dtype).pin_memory()
    if final_state is None:
        final_state = torch.empty((B, HV, Dk, Dv), dtype=torch.float32).pin_memory()
    need = prefill_host_workspace_bytes(B, T, HK, HV, Dk, Dv, BT, io, ab, piece_tokens)
    if need == 0:
        raise GDNError(4, "gdn_chunk_prefill_host: unsupported sizes")
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device="cuda")
    st = lib().gdn_chunk_prefill_host(_hptr(q), _hptr(k), _hptr(v), io, _hptr(a), _hptr(b), ab, _hptr(A_log),
                                      _hptr(dt_bias), _hptr(initial_state), B, T, HK, HV, Dk, Dv, BT, float(scale),
                                      int(bool(qk_l2norm)), int(piece_tokens), _hptr(o), _hptr(final_state),
                                      _ptr(workspace), workspace.numel(), _stream())
    _check(st, "gdn_chunk_prefill_host")
    return o, final_state


def gdn_decode_step_fused(x, conv_w, conv_state_in, a, b, A_log, dt_bias, state, HK: int, conv_act: int = 1,
                          scale: float = 1.0, qk_l2norm: bool = True, conv_state_out=None, o=None, outgate=None):
    """The decode step from raw projections: x [B, C] (C = 2 HK Dk + HV Dv, q | k | v),
    conv_w [C, 4], conv_state_in [B, 3, C] (tap-major, oldest first); a, b [B, HV];
    A_log, dt_bias [HV]; state [B, HV, Dk, Dv] updated in place.  With outgate = (z, norm_w,
    eps), z [B, HV, Dv] like o and norm_w [Dv] fp32, each output row becomes
    o * rsqrt(mean(o^2) + eps) * (1 + norm_w) * sigmoid(z) (gdn_decode_step_fused_outgate).
    Returns (o [B, HV, Dv], conv_state_out [B, 3, C])."""
    B, HV, Dk, Dv = state.shape
    C = 2 * HK * Dk + HV * Dv
    if x.shape != (B, C) or conv_w.shape != (C, 4) or conv_state_in.shape != (B, 3, C):
        raise ValueError("inconsistent fused decode shapes")
    if a.shape != (B, HV) or b.shape != (B, HV) or a.dtype != b.dtype:
        raise ValueError("a, b must be [B, HV] of one dtype")
    if conv_state_out is None:
        conv_state_out = torch.empty_like(conv_state_in)
    if o is None:
        o = torch.empty((B, HV, Dv), dtype=x.dtype, device=x.device)
    if outgate is None:
        st = lib().gdn_decode_step_fused(_ptr(x), _dtype_code(x), _ptr(conv_w), _ptr(conv_state_in),
                                         _ptr(conv_state_out), int(conv_act), _ptr(a), _ptr(b), _dtype_code(a),
                                         _ptr(A_log), _ptr(dt_bias), _ptr(state), B, HK, HV, Dk, Dv, float(scale),
                                         int(bool(qk_l2norm)), _ptr(o), _stream())
        _check(st, "gdn_decode_step_fused")
    else:
        z, norm_w, eps = outgate
        if z.shape != o.shape or z.dtype != x.dtype or norm_w.shape != (Dv,) or norm_w.dtype != torch.float32:
            raise ValueError("z must be shaped and typed like o; norm_w fp32 [Dv]")
        st = lib().gdn_decode_step_fused_outgate(_ptr(x), _dtype_code(x), _ptr(conv_w), _ptr(conv_state_in),
                                                 _ptr(conv_state_out), int(conv_act), _ptr(a), _ptr(b),
                                                 _dtype_code(a), _ptr(A_log), _ptr(dt_bias), _ptr(state), B, HK, HV,
                                                 Dk, Dv, float(scale), int(bool(qk_l2norm)), _ptr(z), _ptr(norm_w),
                                                 float(eps), _ptr(o), _stream())
        _check(st, "gdn_decode_step_fused_outgate")
    return o, conv_state_out


def gdn_conv_prefill(x, conv_w, HK: int, HV: int, Dk: int = 128, Dv: int = 128, conv_state_in=None,
                     cu_seqlens=None, conv_act: int = 1, output_conv_state: bool = True,
                     q=None, k=None, v=None, conv_state_out=None):
    """The prefill prologue: x [B, T, C] raw q | k | v projections (C = 2 HK Dk + HV Dv;
    packed: B = 1 with cu_seqlens int32 [N + 1]); conv_w [C, 4]; conv_state_in [N, 3, C]
    fp32 or None.  Returns (q [B, T, HK, Dk], k, v [B, T, HV, Dv], conv_state_out [N, 3, C]
    or None)."""
    B, T, C = x.shape
    if C != 2 * HK * Dk + HV * Dv or conv_w.shape != (C, 4) or conv_w.dtype != torch.float32:
        raise ValueError("x must be [B, T, 2 HK Dk + HV Dv] and conv_w fp32 [C, 4]")
    if cu_seqlens is not None:
        if cu_seqlens.dtype != torch.int32:
            raise TypeError("cu_seqlens must be int32")
        N = cu_seqlens.numel() - 1
    else:
        N = B
    if conv_state_in is not None and (conv_state_in.shape != (N, 3, C) or conv_state_in.dtype != torch.float32):
        raise ValueError("conv_state_in must be fp32 [N, 3, C]")
    if q is None:
        q = torch.empty((B, T, HK, Dk), dtype=x.dtype, device=x.device)
    if k is None:
        k = torch.empty((B, T, HK, Dk), dtype=x.dtype, device=x.device)
    if v is None:
        v = torch.empty((B, T, HV, Dv), dtype=x.dtype, device=x.device)
    if conv_state_out is None and output_conv_state:
        conv_state_out = torch.empty((N, 3, C), dtype=torch.float32, device=x.device)
    st = lib().gdn_conv_prefill(_ptr(x), _dtype_code(x), _ptr(conv_w), _ptr(conv_state_in), _ptr(cu_seqlens),
                                B, T, N, HK, HV, Dk, Dv, int(conv_act), _ptr(q), _ptr(k), _ptr(v),
                                _ptr(conv_state_out), _stream())
    _check(st, "gdn_conv_prefill")
    return q, k, v, conv_state_out


def gdn_cp_segment(q, k, v, g, beta, initial_state=None, cu_seqlens=None, BT: int = 64, scale: float = 1.0,
                   qk_l2norm: bool = True, workspace=None):
    """One rank's segment of a context-parallel prefill in one call (tensor-core shapes):
    returns (o, final_state) of the segment's prefill and (c, A) of its transition run
    (v = 0 from the identity), sharing one chunk-local stage."""
    B_, T, HK, Dk = q.shape
    HV, Dv = v.shape[-2:]
    N = cu_seqlens.numel() - 1 if cu_seqlens is not None else B_
    dcode = _dtype_code(q)
    o = torch.empty((B_, T, HV, Dv), dtype=q.dtype, device=q.device)
    c = torch.empty_like(o)
    final_state = torch.empty((N, HV, Dk, Dv), dtype=torch.float32, device=q.device)
    transition = torch.empty((N, HV, Dk, Dk), dtype=torch.float32, device=q.device)
    need = prefill_workspace_bytes(B_ * T, N, HK, HV, Dk, Dv, BT, dcode)
    if need == 0:
        _check(4, "gdn_cp_segment")
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    st = lib().gdn_cp_segment(_ptr(q), _ptr(k), _ptr(v), dcode, _ptr(g), _ptr(beta), _ptr(initial_state),
                              _ptr(cu_seqlens), B_, T, N, HK, HV, Dk, Dv, BT, float(scale), int(bool(qk_l2norm)),
                              _ptr(o), _ptr(final_state), _ptr(c), _ptr(transition), _ptr(workspace),
                              workspace.numel(), _stream())
    _check(st, "gdn_cp_segment")
    return o, final_state, c, transition


def gdn_cp_combine(A_all, B_all, o, c, rank: int, initial_state=None, start_state=None, final_state=None,
                   output_final_state: bool = True):
    """The exchange step of a context-parallel prefill: A_all, B_all [R, N, HV, 128, 128]
    fp32 (every segment's transition and zero-start final state), o [N, T_seg, HV, 128]
    (this segment's zero-start output, corrected in place) and c (its transition outputs).
    Returns (start_state, final_state or None)."""
    R, N, HV, Dk, Dv = A_all.shape
    if B_all.shape != A_all.shape or A_all.dtype != torch.float32 or B_all.dtype != torch.float32:
        raise ValueError("A_all, B_all must be fp32 [R, N, HV, Dk, Dv] of one shape")
    T_seg = o.shape[1]
    if o.shape != (N, T_seg, HV, Dv) or c.shape != o.shape or c.dtype != o.dtype:
        raise ValueError("o, c must be [N, T_seg, HV, Dv] of one dtype")
    if start_state is None:
        start_state = torch.empty((N, HV, Dk, Dv), dtype=torch.float32, device=o.device)
    if final_state is None and output_final_state:
        final_state = torch.empty((N, HV, Dk, Dv), dtype=torch.float32, device=o.device)
    st = lib().gdn_cp_combine(_ptr(A_all), _ptr(B_all), _ptr(initial_state), R, int(rank), N, T_seg, HV, Dk, Dv,
                              _dtype_code(o), _ptr(o), _ptr(c), _ptr(start_state), _ptr(final_state), _stream())
    _check(st, "gdn_cp_combine")
    return start_state, final_state


def gdn_cp_status() -> int:
    """Synchronise the device, return gdn_cp_combine's error word and clear it."""
    word = _i32(0)
    st = lib().gdn_cp_status(ctypes.byref(word))
    if st not in (0, 8):
        _check(st, "gdn_cp_status")
    return int(word.value)


def gdn_conv_status() -> int:
    """Synchronise the device, return the convolution kernel's error word and clear it."""
    word = _i32(0)
    st = lib().gdn_conv_status(ctypes.byref(word))
    if st not in (0, 8):
        _check(st, "gdn_conv_status")
    return int(word.value)


def gdn_decode_status() -> int:
    """Synchronise the device, return its decode error word and clear it."""
    word = _i32(0)
    st = lib().gdn_decode_status(ctypes.byref(word))
    if st not in (0, 8):
        _check(st, "gdn_decode_status")
    return int(word.value)


STALL_NONE, STALL_DECODE, STALL_PREFILL_PREP = 0, 1, 2


def testing_stall(site: int):
    """Test hook: make one CTA of the chosen kernel wait for copies that are never issued,
    so that its bounded wait runs out (STALL_NONE restores normal operation)."""
    _check(lib().gdn_testing_stall(int(site)), "gdn_testing_stall")
