"""gdn_chunk_fwd_noalloc: the chunked forward pass for callers that cannot
allocate device memory (it uses scratch built into the library). Its results
must match gdn_chunk_fwd's, call after call, through the C ABI.

Kept in a file of its own that pytest collects last; it must pass both when
run alone in a fresh process and after the rest of the suite.
"""
import ctypes

import pytest
import torch

import gated_delta_rule_112_b200 as gdn
from gated_delta_rule_112_b200.inputs import Workload, make_chunk_inputs
from tests.parity import TOL_BF16, TOL_F32, assert_close, np64, oracle_chunk, rel_l2, to_dev

SCRATCH_BYTES = 64 << 20


def _lib():
    L = gdn.lib()
    vp, ci = ctypes.c_void_p, ctypes.c_int
    L.gdn_chunk_fwd_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, ci, ci,
                                        ci, vp, vp, vp]
    L.gdn_chunk_fwd_noalloc.restype = ci
    return L


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _call(L, d, B, T, H, dk, dv, num_seqs, chunk, dtype, o, fs):
    return L.gdn_chunk_fwd_noalloc(
        _ptr(d["q"]), _ptr(d["k"]), _ptr(d["v"]), _ptr(d["g"]), _ptr(d["beta"]),
        _ptr(d["initial_state"]), _ptr(d["cu_seqlens"]), B, T, H, dk, dv, num_seqs, chunk,
        dtype, _ptr(o), _ptr(fs), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_noalloc_rejects_sizes_beyond_its_scratch():
    # Checked on the host before any launch (the size query reads the current
    # device's SM count, nothing more): B4 H16 T8192 needs far more than 64 MiB.
    L = _lib()
    need = L.gdn_chunk_fwd_workspace_size(4, 8192, 16, 128, 128, 0, 64, gdn.BF16)
    assert need > SCRATCH_BYTES
    p = ctypes.c_void_p(1 << 20)
    rc = L.gdn_chunk_fwd_noalloc(p, p, p, p, p, None, None, 4, 8192, 16, 128, 128, 0, 64,
                                 gdn.BF16, p, None, None)
    assert rc == gdn.ERR_WORKSPACE


CASES = [
    # (workload, tolerance): tensor-core path with a ragged tail and initial
    # state, then the fp32 CUDA-core path on packed sequences.
    (Workload("na_tc", B=2, T=200, H=3, d_k=128, d_v=128, seed=31, random_state=True),
     None, 64, TOL_BF16),
    (Workload("na_simt", B=1, T=0, H=2, d_k=64, d_v=48, dtype=torch.float32, seed=32,
              random_state=True), [70, 1, 33], 32, TOL_F32),
]


@pytest.mark.gpu
@pytest.mark.parametrize("case", range(len(CASES)))
def test_noalloc_matches_chunk_fwd_on_consecutive_calls(case):
    w, lengths, chunk, tol = CASES[case]
    L = _lib()
    for rep in range(2):                      # two calls in a row share the scratch
        inp = make_chunk_inputs(w, seed=w.seed + 100 * rep, lengths=lengths)
        d = to_dev(inp)
        B, T, H = inp["B"], inp["T"], inp["H"]
        N = inp["num_seqs"]
        num_seqs = N if lengths is not None else 0
        o_ref, fs_ref = gdn.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"],
                                      d["initial_state"], d["cu_seqlens"], chunk=chunk)
        o = torch.full_like(o_ref, float("nan"))
        fs = torch.full_like(fs_ref, float("nan"))
        rc = _call(L, d, B, T, H, w.d_k, w.d_v, num_seqs, chunk,
                   gdn.BF16 if w.dtype == torch.bfloat16 else gdn.F32, o, fs)
        assert rc == gdn.OK, gdn.lib().gdn_status_string(rc)
        torch.cuda.synchronize()
        assert rel_l2(np64(o), np64(o_ref)) <= tol
        assert rel_l2(np64(fs), np64(fs_ref)) <= tol
        # and directly against the fp64 oracle on the same inputs
        ro, rfs = oracle_chunk(inp)
        assert_close(f"o (call {rep})", np64(o), ro, tol)
        assert_close(f"final_state (call {rep})", np64(fs), rfs, tol)
