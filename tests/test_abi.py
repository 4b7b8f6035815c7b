"""The C-ABI library loads, exports what include/gdn.h declares, and rejects bad
arguments on the host before launching anything (no GPU needed: every call here
fails validation, or has nothing to do, before any CUDA call)."""
import ctypes
import subprocess

import pytest

from gated_deltanet_sequence_delta_b200 import binding, build as gbuild


@pytest.fixture(scope="module")
def L():
    gbuild.build()
    return binding.lib()


def test_exports_every_declared_symbol(L):
    names = binding.header_functions()
    assert {"gdn_gates", "gdn_chunk_prefill", "gdn_decode_step"} <= set(names)
    nm = subprocess.run(["nm", "-D", "--defined-only", binding.LIB_PATH], capture_output=True,
                        text=True, check=True).stdout
    exported = {line.split()[-1] for line in nm.splitlines() if " T " in line}
    for n in names:
        assert n in exported, n
        assert getattr(L, n) is not None
    # nothing but the declared API is exported (hidden visibility elsewhere)
    assert {e for e in exported if e.startswith("gdn")} == set(names)


def test_version_and_strings(L):
    assert L.gdn_abi_version() == 1
    for s in range(9):
        assert L.gdn_status_string(s).decode().startswith("GDN_")
    assert b"unknown" in L.gdn_status_string(99)
    assert L.gdn_last_cuda_error() == 0


A = 0x7f0000000000          # fake, 16-byte aligned device addresses: never dereferenced
MB = 1 << 20


def _prefill(L, **kw):
    args = dict(q=A, k=A + 64 * MB, v=A + 128 * MB, io=1, g=A + 192 * MB, beta=A + 200 * MB,
                h0=None, cu=None, B=1, T=128, N=1, HK=2, HV=4, Dk=128, Dv=128, BT=64, scale=1.0,
                l2=1, o=A + 256 * MB, hT=A + 384 * MB, ws=A + 448 * MB, ws_bytes=1 << 20)
    args.update(kw)
    return L.gdn_chunk_prefill(args["q"], args["k"], args["v"], args["io"], args["g"], args["beta"],
                               args["h0"], args["cu"], args["B"], args["T"], args["N"], args["HK"],
                               args["HV"], args["Dk"], args["Dv"], args["BT"], args["scale"],
                               args["l2"], args["o"], args["hT"], args["ws"], args["ws_bytes"], None)


def test_prefill_validation(L):
    assert _prefill(L, q=None) == 1                       # NULL
    assert _prefill(L, HV=3) == 2                         # HV % HK
    assert _prefill(L, B=2, N=1) == 2                     # dense needs N == B
    assert _prefill(L, cu=A + 500 * MB, B=2, N=2) == 2    # packed needs B == 1
    assert _prefill(L, Dk=96) == 4                        # unsupported head dim
    assert _prefill(L, BT=48) == 4                        # chunk length not 16, 32 or 64
    assert _prefill(L, io=1, BT=128) == 4
    assert _prefill(L, ws=None) == 6
    assert _prefill(L, ws_bytes=16) == 6
    assert _prefill(L, q=A + 8) == 3                      # misaligned
    assert _prefill(L, o=A + 64) == 5                     # o overlaps q
    assert _prefill(L, hT=A + 256 * MB + 4096) == 5       # final state overlaps o
    assert _prefill(L, h0=A + 384 * MB + 64) == 5         # partial overlap of states
    assert _prefill(L, N=0, B=0) == 0                     # nothing to do: no launch


def _prefill_outgate(L, **kw):
    args = dict(q=A, k=A + 64 * MB, v=A + 128 * MB, io=1, g=A + 192 * MB, beta=A + 200 * MB,
                h0=None, cu=None, B=1, T=128, N=1, HK=2, HV=4, Dk=128, Dv=128, BT=64, scale=1.0,
                l2=1, z=A + 512 * MB, nw=A + 600 * MB, eps=1e-6, o=A + 256 * MB, hT=A + 384 * MB,
                ws=A + 448 * MB, ws_bytes=1 << 20)
    args.update(kw)
    return L.gdn_chunk_prefill_outgate(args["q"], args["k"], args["v"], args["io"], args["g"], args["beta"],
                                       args["h0"], args["cu"], args["B"], args["T"], args["N"], args["HK"],
                                       args["HV"], args["Dk"], args["Dv"], args["BT"], args["scale"],
                                       args["l2"], args["z"], args["nw"], args["eps"], args["o"], args["hT"],
                                       args["ws"], args["ws_bytes"], None)


def test_prefill_outgate_validation(L):
    assert _prefill_outgate(L, z=None) == 1
    assert _prefill_outgate(L, nw=None) == 1
    assert _prefill_outgate(L, eps=-1.0) == 2
    assert _prefill_outgate(L, eps=float("nan")) == 2
    assert _prefill_outgate(L, io=0, BT=64) == 4          # fp32: no tensor-core path, no epilogue
    assert _prefill_outgate(L, HV=6, HK=2) == 4            # GQA group 3
    assert _prefill_outgate(L, z=A + 512 * MB + 4) == 3    # misaligned
    assert _prefill_outgate(L, o=A + 512 * MB + 64) == 5   # o over z
    assert _prefill_outgate(L, N=0, B=0) == 0              # nothing to do


def _cp_segment(L, **kw):
    args = dict(q=A, k=A + 64 * MB, v=A + 128 * MB, io=1, g=A + 192 * MB, beta=A + 200 * MB,
                h0=None, cu=None, B=1, T=128, N=1, HK=2, HV=4, Dk=128, Dv=128, BT=64, scale=1.0,
                l2=1, o=A + 256 * MB, hT=A + 384 * MB, c=A + 512 * MB, tr=A + 600 * MB,
                ws=A + 448 * MB, ws_bytes=1 << 20)
    args.update(kw)
    return L.gdn_cp_segment(args["q"], args["k"], args["v"], args["io"], args["g"], args["beta"], args["h0"],
                            args["cu"], args["B"], args["T"], args["N"], args["HK"], args["HV"], args["Dk"],
                            args["Dv"], args["BT"], args["scale"], args["l2"], args["o"], args["hT"], args["c"],
                            args["tr"], args["ws"], args["ws_bytes"], None)


def test_cp_segment_validation(L):
    assert _cp_segment(L, c=None) == 1
    assert _cp_segment(L, tr=None) == 1                   # the transition output is required
    assert _cp_segment(L, Dv=64) == 4                     # Dk == Dv only
    assert _cp_segment(L, io=0, BT=64) == 4               # fp32: no tensor-core path
    assert _cp_segment(L, HV=6, HK=2) == 4                # GQA group 3
    assert _cp_segment(L, c=A + 256 * MB + 64) == 5       # c over o
    assert _cp_segment(L, tr=A + 384 * MB) == 5           # transition over the final state
    assert _cp_segment(L, N=0, B=0) == 0                  # nothing to do


def test_prefill_workspace_query(L):
    assert L.gdn_chunk_prefill_workspace_bytes(32768, 1, 16, 32, 128, 128, 64, 1) >= 256
    assert L.gdn_chunk_prefill_workspace_bytes(256, 1, 2, 2, 64, 64, 64, 0) >= 256
    assert L.gdn_chunk_prefill_workspace_bytes(256, 1, 2, 3, 64, 64, 64, 0) == 0
    assert L.gdn_chunk_prefill_workspace_bytes(256, 1, 2, 2, 80, 64, 64, 0) == 0
    # beyond the 32-bit coordinates of the tile copies
    assert L.gdn_chunk_prefill_workspace_bytes(2 ** 31, 1, 16, 32, 128, 128, 64, 1) == 0
    assert L.gdn_chunk_prefill_workspace_bytes(2 ** 26, 1, 32, 32, 128, 128, 64, 1) == 0
    assert L.gdn_chunk_prefill_workspace_bytes(2 ** 20, 1, 32, 32, 128, 128, 64, 1) > 0
    # chunk lengths: 16, 32 and 64 in both dtypes; bf16 at 16 or 32 takes the CUDA-core path,
    # whose workspace is the status word alone, far less than the tensor-core path's tiles
    tc = L.gdn_chunk_prefill_workspace_bytes(4096, 1, 2, 4, 128, 128, 64, 1)
    for bt in (16, 32):
        cc = L.gdn_chunk_prefill_workspace_bytes(4096, 1, 2, 4, 128, 128, bt, 1)
        assert 0 < cc < tc, (bt, cc, tc)
        assert L.gdn_chunk_prefill_workspace_bytes(4096, 1, 2, 4, 128, 128, bt, 0) > 0
    for bt in (8, 48, 128):
        assert L.gdn_chunk_prefill_workspace_bytes(4096, 1, 2, 4, 128, 128, bt, 1) == 0


def test_gates_validation(L):
    f = L.gdn_gates
    assert f(A, A + MB, 0, None, A + 3 * MB, 10, 4, A + 4 * MB, A + 5 * MB, None) == 1
    assert f(A, A + MB, 0, A + 2 * MB, A + 3 * MB, 10, 0, A + 4 * MB, A + 5 * MB, None) == 2
    assert f(A, A + MB, 0, A + 2 * MB, A + 3 * MB, -1, 4, A + 4 * MB, A + 5 * MB, None) == 2
    assert f(A, A + MB, 0, A + 2 * MB, A + 3 * MB, 10, 4, A + 16, A + 5 * MB, None) == 5
    assert f(A, A + MB, 0, A + 2 * MB, A + 3 * MB, 10, 4, A + 4 * MB, A + 4 * MB + 16, None) == 5
    assert f(A + 4, A + MB, 0, A + 2 * MB, A + 3 * MB, 10, 4, A + 4 * MB, A + 5 * MB, None) == 3
    assert f(None, None, 0, A + 2 * MB, A + 3 * MB, 0, 4, None, None, None) == 0   # empty: no launch


def test_decode_validation(L):
    f = L.gdn_decode_step
    base = [A, A + MB, A + 2 * MB, 1, A + 3 * MB, A + 4 * MB, A + 16 * MB, 4, 2, 4, 128, 128, 1.0, 1,
            A + 8 * MB, None]
    def call(**kw):
        a = list(base)
        for i, val in kw.items():
            a[int(i[1:])] = val
        return f(*a)
    assert call(a6=None) == 1
    assert call(a9=3) == 2
    assert call(a10=32) == 4
    assert call(a3=7) == 4
    assert call(a14=A + 16 * MB + 128) == 5     # o inside the state
    assert call(a6=A + 2 * MB) == 5             # state over v
    assert call(a0=A + 2) == 3
    assert call(a7=0) == 0                      # B = 0: nothing to do


def test_decode_gated_validation(L):
    f = L.gdn_decode_step_gated
    # q, k, v, io, a, b, ab, A_log, dt_bias, state, B, HK, HV, Dk, Dv, scale, l2, o, stream
    base = [A, A + MB, A + 2 * MB, 1, A + 3 * MB, A + 4 * MB, 0, A + 5 * MB, A + 6 * MB, A + 16 * MB,
            4, 2, 4, 128, 128, 1.0, 1, A + 8 * MB, None]
    def call(**kw):
        a = list(base)
        for i, val in kw.items():
            a[int(i[1:])] = val
        return f(*a)
    assert call(a4=None) == 1                   # a missing
    assert call(a8=None) == 1                   # dt_bias missing
    assert call(a12=3) == 2                     # HV % HK
    assert call(a6=7) == 4                      # bad ab dtype
    assert call(a13=32) == 4                    # head dim
    assert call(a5=A + 4 * MB + 4) == 3         # b misaligned
    assert call(a17=A + 3 * MB) == 5            # o over a
    assert call(a9=A + 5 * MB) == 5             # state over A_log
    assert call(a10=0) == 0                     # B = 0: nothing to do


def test_prefill_host_validation(L):
    f = L.gdn_chunk_prefill_host
    ws_need = L.gdn_chunk_prefill_host_workspace_bytes(1, 1000, 2, 4, 128, 128, 64, 1, 0, 256)
    assert ws_need > 0
    assert L.gdn_chunk_prefill_host_workspace_bytes(1, 1000, 2, 4, 128, 128, 64, 1, 0, 100) == 0   # piece % BT
    assert L.gdn_chunk_prefill_host_workspace_bytes(1, 1000, 2, 4, 32, 128, 64, 1, 0, 256) == 0    # head dim
    # q, k, v, io, a, b, ab, A_log, dt_bias, h0, B, T, HK, HV, Dk, Dv, BT, scale, l2, piece, o, hT, ws, bytes, stream
    base = [A, A + MB, A + 2 * MB, 1, A + 3 * MB, A + 4 * MB, 0, A + 5 * MB, A + 6 * MB, None,
            1, 1000, 2, 4, 128, 128, 64, 1.0, 1, 256, A + 8 * MB, A + 9 * MB, A + 16 * MB, ws_need, None]
    def call(**kw):
        a = list(base)
        for i, val in kw.items():
            a[int(i[1:])] = val
        return f(*a)
    assert call(a19=100) == 2                   # piece not a multiple of BT
    assert call(a19=0) == 2
    assert call(a13=3) == 2                     # HV % HK
    assert call(a14=32) == 4                    # head dim
    assert call(a6=9) == 4                      # ab dtype
    assert call(a0=None) == 1
    assert call(a8=None) == 1
    assert call(a22=None) == 6                  # no workspace
    assert call(a23=ws_need - 1) == 6           # workspace too small
    assert call(a22=A + 16 * MB + 16) == 3      # workspace not 256-byte aligned
    assert call(a10=0) == 0                     # B = 0: nothing to do


def test_decode_fused_validation(L):
    f = L.gdn_decode_step_fused
    # x, io, w, cs_in, cs_out, act, a, b, ab, A_log, dt_bias, state, B, HK, HV, Dk, Dv, scale, l2, o, stream
    base = [A, 1, A + MB, A + 2 * MB, A + 3 * MB, 1, A + 4 * MB, A + 5 * MB, 0, A + 6 * MB, A + 7 * MB,
            A + 16 * MB, 4, 2, 4, 128, 128, 1.0, 1, A + 9 * MB, None]
    def call(**kw):
        a = list(base)
        for i, val in kw.items():
            a[int(i[1:])] = val
        return f(*a)
    assert call(a0=None) == 1
    assert call(a2=None) == 1
    assert call(a5=2) == 4                      # activation code
    assert call(a15=64) == 4                    # d = 128 only
    assert call(a14=3) == 2                     # HV % HK
    assert call(a3=A + 2 * MB + 4) == 3         # conv_state_in misaligned
    assert call(a4=A + 2 * MB) == 5             # conv_state_out over conv_state_in
    assert call(a19=A + 16 * MB) == 5           # o over the state
    assert call(a12=0) == 0                     # B = 0: nothing to do


def test_conv_prefill_validation(L):
    f = L.gdn_conv_prefill
    # x, io, w, cs_in, cu, B, T, N, HK, HV, Dk, Dv, act, q, k, v, cs_out, stream
    base = [A, 1, A + MB, A + 2 * MB, None, 2, 100, 2, 2, 4, 128, 128, 1, A + 8 * MB, A + 9 * MB, A + 10 * MB,
            A + 11 * MB, None]
    def call(**kw):
        a = list(base)
        for i, val in kw.items():
            a[int(i[1:])] = val
        return f(*a)
    assert call(a0=None) == 1                   # x
    assert call(a2=None) == 1                   # weights
    assert call(a12=2) == 4                     # activation code
    assert call(a10=96) == 4                    # head dim
    assert call(a4=A + 12 * MB) == 2            # packed needs B = 1
    assert call(a7=3) == 2                      # dense: n_seqs = B
    assert call(a8=0) == 2                      # HK
    assert call(a13=A + 8 * MB + 4) == 3        # q misaligned
    assert call(a13=A) == 5                     # q over x
    assert call(a16=A + 2 * MB) == 5            # conv_state_out over conv_state_in
    assert call(a14=A + 8 * MB + 64) == 5       # k over q
    assert call(a5=0, a7=0) == 0                # no sequences: nothing to do


def test_cp_combine_validation(L):
    f = L.gdn_cp_combine
    # A_all, B_all, h0, R, rank, N, T_seg, HV, Dk, Dv, io, o, c, start, final, stream
    base = [A, A + 4 * MB, None, 2, 1, 1, 100, 2, 128, 128, 1, A + 8 * MB, A + 9 * MB, A + 10 * MB, A + 11 * MB,
            None]
    def call(**kw):
        a = list(base)
        for i, val in kw.items():
            a[int(i[1:])] = val
        return f(*a)
    assert call(a4=2) == 2                      # rank past R
    assert call(a3=0) == 2                      # R
    assert call(a8=64, a9=64) == 4              # d = 128 only
    assert call(a0=None) == 1
    assert call(a13=None) == 1                  # start state is required
    assert call(a11=A + 8 * MB + 4) == 3        # o misaligned
    assert call(a11=A + 9 * MB) == 5            # o over c
    assert call(a13=A + 4 * MB) == 5            # start state over B_all
    assert call(a14=A + 10 * MB) == 5           # final over start
    assert call(a10=0, a6=65535 * 128 + 1) == 4  # fp32: more token tiles than a grid row holds
    assert call(a5=2, a6=(1 << 30)) == 4         # bf16: past 32-bit tile coordinates
    assert call(a5=0) == 0                      # no sequences: nothing to do


def test_decode_status_null(L):
    assert L.gdn_decode_status(None) == 1
    assert L.gdn_conv_status(None) == 1
    assert L.gdn_cp_status(None) == 1


def test_missing_library_fails_loudly(tmp_path):
    with pytest.raises(binding.GDNLibraryError):
        binding.lib(str(tmp_path / "nope.so"))


def test_static_scratch_entry_point_reports_sizes_like_the_workspace_one(L):
    """gdn_chunk_prefill_static_ws rejects the sizes gdn_chunk_prefill rejects, with the same
    status, before it touches its scratch (so no GPU is needed here)."""
    f = L.gdn_chunk_prefill_static_ws
    vp, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
    f.argtypes = [vp, vp, vp, ctypes.c_int, vp, vp, vp, vp, i32, i64, i32, i32, i32, i32, i32, i32,
                  ctypes.c_float, i32, vp, vp, vp]
    f.restype = ctypes.c_int

    def static(**kw):
        a = dict(B=1, T=128, N=1, HK=2, HV=4, Dk=128, Dv=128, BT=64, cu=None, io=1)
        a.update(kw)
        return f(A, A + 64 * MB, A + 128 * MB, a["io"], A + 192 * MB, A + 200 * MB, None, a["cu"], a["B"], a["T"],
                 a["N"], a["HK"], a["HV"], a["Dk"], a["Dv"], a["BT"], 1.0, 1, A + 256 * MB, A + 384 * MB, None)

    cases = [dict(HK=2, HV=3), dict(HK=0), dict(B=2, N=1), dict(cu=A + 500 * MB, B=2, N=2), dict(Dk=96),
             dict(BT=48), dict(T=-1), dict(io=5), dict(cu=A + 500 * MB, T=1 << 31)]
    for kw in cases:
        want = _prefill(L, **{k: v for k, v in kw.items() if k != "io"}, **({"io": kw["io"]} if "io" in kw else {}))
        assert want != 0, kw
        assert static(**kw) == want, (kw, static(**kw), want)
    assert static(HK=2, HV=3) == 2   # GDN_ERR_SHAPE, as gdn_chunk_prefill


def test_prefill_gated_validation(L):
    def call(**kw):
        a = dict(q=A, k=A + 64 * MB, v=A + 128 * MB, io=1, ga=A + 192 * MB, gb=A + 200 * MB, ab=0, Al=A + 208 * MB,
                 dtb=A + 209 * MB, h0=None, cu=None, B=1, T=128, N=1, HK=2, HV=4, Dk=128, Dv=128, BT=64,
                 o=A + 256 * MB, hT=A + 384 * MB, ws=A + 448 * MB, ws_bytes=1 << 30)
        a.update(kw)
        return L.gdn_chunk_prefill_gated(a["q"], a["k"], a["v"], a["io"], a["ga"], a["gb"], a["ab"], a["Al"], a["dtb"],
                                         a["h0"], a["cu"], a["B"], a["T"], a["N"], a["HK"], a["HV"], a["Dk"], a["Dv"],
                                         a["BT"], 1.0, 1, a["o"], a["hT"], a["ws"], a["ws_bytes"], None)
    assert call(ga=None) == 1                  # NULL gate input
    assert call(Al=None) == 1
    assert call(HV=3) == 2                     # HV % HK
    assert call(Dk=64, Dv=64) == 4             # not a tensor-core shape
    assert call(io=0) == 4                     # fp32 io: the CUDA-core path has no fused gates
    assert call(ab=7) == 4                     # unknown gate dtype
    assert call(ga=A + 192 * MB + 4) == 3      # misaligned
    assert call(o=A + 192 * MB) == 5           # output over a gate input
    assert call(ws_bytes=16) == 6


def test_decode_fused_outgate_validation(L):
    C = 2 * 2 * 128 + 4 * 128
    def call(**kw):
        a = dict(x=A, cw=A + 8 * MB, csi=A + 16 * MB, cso=A + 24 * MB, ga=A + 32 * MB, gb=A + 33 * MB,
                 Al=A + 34 * MB, dtb=A + 35 * MB, st=A + 64 * MB, B=2, HK=2, HV=4, z=A + 40 * MB,
                 nw=A + 41 * MB, eps=1e-6, o=A + 48 * MB)
        a.update(kw)
        return L.gdn_decode_step_fused_outgate(a["x"], 1, a["cw"], a["csi"], a["cso"], 1, a["ga"], a["gb"], 0,
                                               a["Al"], a["dtb"], a["st"], a["B"], a["HK"], a["HV"], 128, 128,
                                               1.0, 1, a["z"], a["nw"], a["eps"], a["o"], None)
    assert call(z=None) == 1
    assert call(nw=None) == 1
    assert call(eps=-1.0) == 2
    assert call(eps=float("nan")) == 2
    assert call(z=A + 40 * MB + 8) == 3
    assert call(o=A + 40 * MB) == 5      # output over z
    assert call(st=A + 41 * MB) == 5     # state over norm_w
    assert call(HV=3) == 2
