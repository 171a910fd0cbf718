"""The C ABI library: it loads, exports every symbol include/gdn.h declares,
and rejects bad arguments on the host before touching a GPU."""
import ctypes
import os
import re

import pytest

import gated_delta_rule_112_b200 as gdn
from gated_delta_rule_112_b200 import build as gbuild

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "gdn.h")


@pytest.fixture(scope="module")
def L():
    gbuild.build()
    return gdn.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gdn_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for must in ("gdn_chunk_fwd", "gdn_chunk_fwd_workspace_size", "gdn_decode_step",
                 "gdn_get_status", "gdn_status_string"):
        assert must in names


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), f"libgdn.so does not export {name}"


def test_checked_variant_exports_the_same_symbols():
    lib = gbuild.build(checked=True)
    C = ctypes.CDLL(lib)
    for name in declared_functions():
        assert hasattr(C, name), f"libgdn_checked.so does not export {name}"
    C.gdn_checked_build.restype = ctypes.c_int
    assert C.gdn_checked_build() == 1


def test_status_strings(L):
    assert L.gdn_status_string(0) == b"GDN_OK"
    assert L.gdn_status_string(5) == b"GDN_ERR_DEVICE_TIMEOUT"
    assert L.gdn_status_string(6) == b"GDN_ERR_DEVICE_BOUNDS"
    assert L.gdn_checked_build() == 0
    assert L.gdn_status_string(99) == b"GDN_ERR_UNKNOWN"


def test_path_selection(L):
    assert L.gdn_chunk_fwd_path(128, 128, 64, gdn.BF16) == gdn.PATH_TCGEN05
    assert L.gdn_chunk_fwd_path(128, 128, 64, gdn.F32) == gdn.PATH_SIMT
    assert L.gdn_chunk_fwd_path(64, 64, 64, gdn.BF16) == gdn.PATH_SIMT
    assert L.gdn_chunk_fwd_path(128, 128, 32, gdn.BF16) == gdn.PATH_SIMT
    assert L.gdn_chunk_fwd_path(256, 128, 64, gdn.BF16) < 0
    assert L.gdn_chunk_fwd_path(128, 128, 48, gdn.BF16) < 0


def test_workspace_size(L):
    ws = L.gdn_chunk_fwd_workspace_size
    tc = ws(4, 4096, 16, 128, 128, 0, 64, gdn.BF16)
    # 4096 (chunk, head) units x (-W 16 KB + (D K)^T 16 KB + T diag(beta) 8 KB +
    # P 8 KB + 512 B of decay factors) plus bookkeeping
    per_unit = 16384 + 16384 + 8192 + 8192 + 512
    assert tc >= 4096 * per_unit
    assert tc < 4096 * per_unit + (1 << 20)
    simt = ws(1, 256, 2, 64, 64, 0, 64, gdn.F32)
    assert 0 < simt < (1 << 16)
    # varlen bound: (T + N (C-1)) / C chunks
    v = ws(1, 1000, 1, 128, 128, 10, 64, gdn.BF16)
    assert v >= ((1000 + 10 * 63) // 64) * (16384 + 16384 + 8192 + 8192 + 512)
    assert ws(0, 10, 1, 128, 128, 0, 64, gdn.BF16) == 0
    assert ws(1, 10, 1, 128, 128, 0, 48, gdn.BF16) == 0


def _chunk_call(L, fn="gdn_chunk_fwd", **kw):
    a = dict(q=1 << 20, k=1 << 20, v=1 << 20, g=1 << 20, beta=1 << 20, s0=None, cu=None, B=1,
             T=64, H=1, dk=128, dv=128, ns=0, chunk=64, dtype=gdn.BF16, o=1 << 20, sN=None,
             ws=1 << 20, wsb=1 << 30, stream=None)
    a.update(kw)
    vp = ctypes.c_void_p
    return getattr(L, fn)(vp(a["q"]), vp(a["k"]), vp(a["v"]), vp(a["g"]), vp(a["beta"]),
                           vp(a["s0"]), vp(a["cu"]), a["B"], a["T"], a["H"], a["dk"], a["dv"],
                           a["ns"], a["chunk"], a["dtype"], vp(a["o"]), vp(a["sN"]),
                           vp(a["ws"]), a["wsb"], vp(a["stream"]))


def test_host_argument_checks_launch_nothing(L):
    # Each of these is rejected before any CUDA call is made.
    assert _chunk_call(L, q=None) == gdn.ERR_INVALID_ARG
    assert _chunk_call(L, o=None) == gdn.ERR_INVALID_ARG
    assert _chunk_call(L, B=0) == gdn.ERR_INVALID_ARG
    assert _chunk_call(L, T=-1) == gdn.ERR_INVALID_ARG
    assert _chunk_call(L, dtype=7) == gdn.ERR_INVALID_ARG
    assert _chunk_call(L, dk=256) == gdn.ERR_UNSUPPORTED
    assert _chunk_call(L, chunk=48) == gdn.ERR_UNSUPPORTED
    assert _chunk_call(L, q=(1 << 20) + 2) == gdn.ERR_INVALID_ARG      # misaligned
    assert _chunk_call(L, ws=None) == gdn.ERR_WORKSPACE
    assert _chunk_call(L, ws=(1 << 20) + 16) == gdn.ERR_WORKSPACE      # not 256-aligned
    assert _chunk_call(L, wsb=100) == gdn.ERR_WORKSPACE
    assert _chunk_call(L, cu=1 << 20, ns=2, B=2) == gdn.ERR_INVALID_ARG  # varlen needs B == 1
    assert _chunk_call(L, ns=3) == gdn.ERR_INVALID_ARG                  # num_seqs without cu


def test_decode_host_checks(L):
    vp = ctypes.c_void_p
    p = vp(1 << 20)

    def call(**kw):
        a = dict(N=2, H=2, dk=128, dv=128, dtype=gdn.BF16, state=p, q=p)
        a.update(kw)
        return L.gdn_decode_step(a["q"], p, p, p, p, a["state"], p, a["N"], a["H"], a["dk"],
                                 a["dv"], a["dtype"], None)
    assert call(state=None) == gdn.ERR_INVALID_ARG
    assert call(q=vp((1 << 20) + 4)) == gdn.ERR_INVALID_ARG
    assert call(N=0) == gdn.ERR_INVALID_ARG
    assert call(dv=130) == gdn.ERR_UNSUPPORTED
    assert call(dv=126) == gdn.ERR_UNSUPPORTED


def test_scan_segments_rule(L):
    seg = L.gdn_chunk_fwd_scan_segments
    BF, F = gdn.BF16, gdn.F32
    # few long chains: split; one chain per SM-wave of short chains: no split
    assert seg(1, 65536, 16, 128, 128, 0, 64, BF, 148) == 9     # long64k: 16 chains x 1024 chunks
    assert seg(4, 4096, 16, 128, 128, 0, 64, BF, 148) == 1      # 64 chains x 64 chunks
    assert seg(1, 64 * 40, 1, 128, 128, 0, 64, BF, 148) > 1
    assert seg(1, 320, 2, 128, 128, 0, 64, BF, 148) == 1        # 5 chunks
    assert seg(1, 65536, 16, 128, 128, 4, 64, BF, 148) == 1     # packed sequences: never
    assert seg(1, 65536, 16, 128, 128, 0, 64, F, 148) == 1      # CUDA-core path: never
    assert seg(1, 65536, 16, 128, 128, 0, 64, BF, 0) == 1       # unknown device
    for sms in (1, 16, 148, 160):
        g = seg(1, 64 * 1000, 3, 128, 128, 0, 64, BF, sms)
        assert 1 <= g <= 16


def test_kda_entry_points_host_checks(L):
    kda = "gdn_kda_chunk_fwd"
    assert _chunk_call(L, fn=kda, q=None) == gdn.ERR_INVALID_ARG
    assert _chunk_call(L, fn=kda, g=(1 << 20) + 2) == gdn.ERR_INVALID_ARG   # misaligned gate
    assert _chunk_call(L, fn=kda, dk=256) == gdn.ERR_UNSUPPORTED
    assert _chunk_call(L, fn=kda, chunk=48) == gdn.ERR_UNSUPPORTED
    assert _chunk_call(L, fn=kda, ws=None) == gdn.ERR_WORKSPACE
    assert _chunk_call(L, fn=kda, wsb=100) == gdn.ERR_WORKSPACE
    # bf16, d = 128, chunk 64: the tensor-core path, whose workspace holds the
    # scalar gate's per-(chunk, head) operand tiles plus Q .* exp(Gamma) (16 KB)
    # and a 1 KB decay record (256 fp32) instead of 512 B
    kws = L.gdn_kda_chunk_fwd_workspace_size(4, 4096, 16, 128, 128, 0, 64, gdn.BF16)
    sws = L.gdn_chunk_fwd_workspace_size(4, 4096, 16, 128, 128, 0, 64, gdn.BF16)
    assert kws == sws + 4096 * (16384 + 512)
    # every other size and dtype: the CUDA-core kernel, chunk table alone
    fws = L.gdn_kda_chunk_fwd_workspace_size(4, 4096, 16, 128, 128, 0, 64, gdn.F32)
    assert fws == L.gdn_chunk_fwd_workspace_size(4, 4096, 16, 128, 128, 0, 64, gdn.F32)
    assert 0 < fws < (1 << 20)
    assert L.gdn_kda_chunk_fwd_workspace_size(1, 10, 1, 128, 128, 0, 48, gdn.BF16) == 0
    vp = ctypes.c_void_p
    p = vp(1 << 20)
    assert L.gdn_kda_decode_step(p, p, p, p, p, None, p, 2, 2, 128, 128, gdn.BF16,
                                 None) == gdn.ERR_INVALID_ARG
    assert L.gdn_kda_decode_step(p, p, p, p, p, p, p, 2, 2, 128, 126, gdn.BF16,
                                 None) == gdn.ERR_UNSUPPORTED


def test_bwd_host_checks(L):
    vp = ctypes.c_void_p
    p = vp(1 << 20)

    def call(**kw):
        a = dict(B=1, T=64, H=1, dk=128, dv=128, ns=0, dtype=gdn.BF16, q=p, ds0=p, ws=p,
                 wsb=1 << 40, cu=None)
        a.update(kw)
        return L.gdn_chunk_bwd(a["q"], p, p, p, p, None, a["cu"], p, None, a["B"], a["T"],
                               a["H"], a["dk"], a["dv"], a["ns"], a["dtype"], p, p, p, p, p,
                               a["ds0"], a["ws"], a["wsb"], None)
    assert call(q=None) == gdn.ERR_INVALID_ARG
    assert call(ds0=None) == gdn.ERR_INVALID_ARG
    assert call(dtype=9) == gdn.ERR_INVALID_ARG
    assert call(dv=126) == gdn.ERR_UNSUPPORTED
    assert call(dk=256) == gdn.ERR_UNSUPPORTED
    assert call(ns=2) == gdn.ERR_INVALID_ARG                  # num_seqs without cu_seqlens
    assert call(ws=None) == gdn.ERR_WORKSPACE
    assert call(wsb=1000) == gdn.ERR_WORKSPACE
    # token-level path: every token's S_{t-1} and S_{t-1} k_t in fp32, plus the control block
    need = L.gdn_chunk_bwd_exact_workspace_size(4, 4096, 16, 128, 128, 0)
    assert need >= 4 * 4096 * 16 * (128 * 128 + 128) * 4
    assert need < 4 * 4096 * 16 * (128 * 128 + 128) * 4 + 4096
    assert L.gdn_chunk_bwd_workspace_size(4, 4096, 16, 128, 128, 0, gdn.F32) == need
    assert L.gdn_chunk_bwd_exact_workspace_size(0, 1, 1, 128, 128, 0) == 0
    assert L.gdn_chunk_bwd_workspace_size(0, 1, 1, 128, 128, 0, gdn.BF16) == 0
    # chunkwise path (bf16, d = 128): the forward's workspace plus two bf16
    # 128 x 128 states per (chunk, head) unit
    tc = L.gdn_chunk_bwd_workspace_size(4, 4096, 16, 128, 128, 0, gdn.BF16)
    fwd = L.gdn_chunk_fwd_workspace_size(4, 4096, 16, 128, 128, 0, 64, gdn.BF16)
    assert tc >= fwd + 4096 * 2 * 128 * 128 * 2
    assert tc < fwd + 4096 * 2 * 128 * 128 * 2 + (1 << 20)


def test_saved_pair_host_checks(L):
    """gdn_chunk_fwd_save / gdn_chunk_bwd_saved: tensor-core path only, and the
    backward's workspace size (checked before anything is launched)."""
    vp = ctypes.c_void_p
    p = vp(1 << 20)

    def fwd(**kw):
        a = dict(B=1, T=64, H=1, dk=128, dv=128, ns=0, dtype=gdn.BF16, o=p, ws=p, wsb=1 << 40)
        a.update(kw)
        return L.gdn_chunk_fwd_save(p, p, p, p, p, None, None, a["B"], a["T"], a["H"], a["dk"],
                                    a["dv"], a["ns"], a["dtype"], a["o"], None, a["ws"],
                                    a["wsb"], None)

    def bwd(**kw):
        a = dict(dk=128, dv=128, dtype=gdn.BF16, wsb=1 << 40)
        a.update(kw)
        return L.gdn_chunk_bwd_saved(p, p, p, p, p, None, None, p, None, 1, 64, 1, a["dk"],
                                     a["dv"], 0, a["dtype"], p, p, p, p, p, p, p, a["wsb"], None)

    assert fwd(dtype=gdn.F32) == gdn.ERR_UNSUPPORTED
    assert fwd(dk=64) == gdn.ERR_UNSUPPORTED
    assert fwd(o=None) == gdn.ERR_INVALID_ARG
    assert fwd(ws=None) == gdn.ERR_WORKSPACE
    need = L.gdn_chunk_bwd_workspace_size(1, 64, 1, 128, 128, 0, gdn.BF16)
    assert need > L.gdn_chunk_fwd_workspace_size(1, 64, 1, 128, 128, 0, 64, gdn.BF16)
    assert fwd(wsb=need - 1) == gdn.ERR_WORKSPACE
    assert bwd(dtype=gdn.F32) == gdn.ERR_UNSUPPORTED
    assert bwd(dk=64) == gdn.ERR_UNSUPPORTED
    assert bwd(wsb=need - 1) == gdn.ERR_WORKSPACE
