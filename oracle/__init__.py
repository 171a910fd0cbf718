"""CPU fp64 oracle for the gated delta rule -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg may import this package. The CUDA library never links, loads or calls it,
and it imports nothing from the CUDA side (inputs come from the shared seeded
generator module, which holds no arithmetic of the method).

Two independent formulations live here:

* ``chunk_fwd`` / ``decode_step``: the defining token-by-token recurrence in
  plain C (``gdn_oracle.c``), fp64, threaded over (sequence, head). This is
  the oracle the GPU results are compared with.
* ``chunked.chunk_fwd_dense``: the chunkwise WY / UT-transform form in numpy
  (dense inversion of I + A per chunk). It is used to pin the recurrence and
  to give per-chunk intermediates (T, W, U, P) for debugging kernels.
* ``kda_chunk_fwd`` / ``kda_decode_step`` and ``chunked.kda_chunk_fwd_dense``:
  the same two formulations for the channel-wise gate (the Kimi Delta
  Attention variant: g = log alpha has one value per d_k channel).
* ``chunk_bwd``: the gradients of ``chunk_fwd`` by reverse-mode
  differentiation of the token recurrence (C, fp64).

Every function is pinned by ``tests/test_oracle_pins.py``,
``tests/test_oracle_kda_pins.py`` and ``tests/test_oracle_bwd_pins.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn_oracle.c")
_LIB_DIR = os.path.join(_HERE, "_build")
_LIB = os.path.join(_LIB_DIR, "libgdn_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle with gcc (no GPU involved)."""
    os.makedirs(_LIB_DIR, exist_ok=True)
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-shared", "-fPIC", "-pthread",
                               _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        d = ctypes.POINTER(ctypes.c_double)
        i32 = ctypes.POINTER(ctypes.c_int32)
        ci = ctypes.c_int
        lib.gdn_oracle_chunk_fwd.argtypes = [d, d, d, d, d, d, i32, ci, ci, ci, ci, ci, ci,
                                             d, d, ci]
        lib.gdn_oracle_chunk_fwd.restype = ci
        lib.gdn_oracle_decode_step.argtypes = [d, d, d, d, d, d, d, ci, ci, ci, ci, ci]
        lib.gdn_oracle_decode_step.restype = ci
        lib.gdn_oracle_kda_chunk_fwd.argtypes = lib.gdn_oracle_chunk_fwd.argtypes
        lib.gdn_oracle_kda_chunk_fwd.restype = ci
        lib.gdn_oracle_kda_decode_step.argtypes = lib.gdn_oracle_decode_step.argtypes
        lib.gdn_oracle_kda_decode_step.restype = ci
        lib.gdn_oracle_chunk_bwd.argtypes = [d, d, d, d, d, d, i32, ci, ci, ci, ci, ci, ci,
                                             d, d, d, d, d, d, d, d, ci]
        lib.gdn_oracle_chunk_bwd.restype = ci
        _lib = lib
    return _lib


def _f64(x):
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)))


def chunk_fwd(q, k, v, g, beta, initial_state=None, cu_seqlens=None, nthreads=None):
    """Run the fp64 token recurrence over whole sequences.

    q, k: [B,T,H,d_k]; v: [B,T,H,d_v]; g (= log alpha), beta: [B,T,H];
    initial_state: [N,H,d_k,d_v] or None (zeros); cu_seqlens: int [N+1] or None.
    Returns (o [B,T,H,d_v], final_state [N,H,d_k,d_v]) as float64 arrays.
    """
    return _run_chunk("gdn_oracle_chunk_fwd", q, k, v, g, beta, initial_state, cu_seqlens,
                      nthreads, channel=False)


def kda_chunk_fwd(q, k, v, g, beta, initial_state=None, cu_seqlens=None, nthreads=None):
    """The fp64 token recurrence with the channel-wise gate:
    S_t = S_{t-1} diag(alpha_t) (I - beta_t k_t k_t^T) + beta_t v_t k_t^T, o_t = S_t q_t.

    Same layouts as ``chunk_fwd`` except g (= log alpha): [B,T,H,d_k].
    """
    return _run_chunk("gdn_oracle_kda_chunk_fwd", q, k, v, g, beta, initial_state, cu_seqlens,
                      nthreads, channel=True)


def _run_chunk(fn, q, k, v, g, beta, initial_state, cu_seqlens, nthreads, channel):
    q, k, v, g, beta = (_f64(a) for a in (q, k, v, g, beta))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if g.shape != ((B, T, H, dk) if channel else (B, T, H)):
        raise ValueError(f"g has shape {g.shape}")
    cu = None
    N = B
    if cu_seqlens is not None:
        cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int32))
        N = cu.shape[0] - 1
    s0 = None if initial_state is None else _f64(initial_state)
    o = np.zeros((B, T, H, dv), dtype=np.float64)
    fs = np.zeros((N, H, dk, dv), dtype=np.float64)
    rc = getattr(_load(), fn)(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(s0),
        None if cu is None else cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
        B, T, H, dk, dv, N, _ptr(o), _ptr(fs), nthreads or default_threads())
    if rc != 0:
        raise ValueError("oracle rejected the arguments")
    return o, fs


def chunk_bwd(q, k, v, g, beta, d_o, initial_state=None, cu_seqlens=None,
              d_final_state=None, nthreads=None):
    """Gradients of ``chunk_fwd`` (scalar gate) for the loss
    L = sum(d_o * o) + sum(d_final_state * final_state), by reverse-mode
    differentiation of the token recurrence in fp64.

    Returns a dict of float64 arrays: dq, dk [B,T,H,d_k], dv [B,T,H,d_v],
    dg, dbeta [B,T,H], d_initial_state [N,H,d_k,d_v].
    """
    q, k, v, g, beta, d_o = (_f64(a) for a in (q, k, v, g, beta, d_o))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if g.shape != (B, T, H) or d_o.shape != (B, T, H, dv):
        raise ValueError("g or d_o has the wrong shape")
    cu = None
    N = B
    if cu_seqlens is not None:
        cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int32))
        N = cu.shape[0] - 1
    s0 = None if initial_state is None else _f64(initial_state)
    dsN = None if d_final_state is None else _f64(d_final_state)
    out = dict(dq=np.zeros((B, T, H, dk)), dk=np.zeros((B, T, H, dk)),
               dv=np.zeros((B, T, H, dv)), dg=np.zeros((B, T, H)), dbeta=np.zeros((B, T, H)),
               d_initial_state=np.zeros((N, H, dk, dv)))
    rc = _load().gdn_oracle_chunk_bwd(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(s0),
        None if cu is None else cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
        B, T, H, dk, dv, N, _ptr(d_o), _ptr(dsN), _ptr(out["dq"]), _ptr(out["dk"]),
        _ptr(out["dv"]), _ptr(out["dg"]), _ptr(out["dbeta"]), _ptr(out["d_initial_state"]),
        nthreads or default_threads())
    if rc != 0:
        raise ValueError("oracle rejected the arguments")
    return out


def decode_step(q, k, v, g, beta, state, nthreads=None):
    """One recurrent step for every (n, h). Returns (o [N,H,d_v], new_state)."""
    return _run_decode("gdn_oracle_decode_step", q, k, v, g, beta, state, nthreads)


def kda_decode_step(q, k, v, g, beta, state, nthreads=None):
    """One channel-wise-gated step for every (n, h); g: [N,H,d_k]."""
    return _run_decode("gdn_oracle_kda_decode_step", q, k, v, g, beta, state, nthreads)


def _run_decode(fn, q, k, v, g, beta, state, nthreads):
    q, k, v, g, beta = (_f64(a) for a in (q, k, v, g, beta))
    st = _f64(state).copy()
    N, H, dk = q.shape
    dv = v.shape[-1]
    o = np.zeros((N, H, dv), dtype=np.float64)
    rc = getattr(_load(), fn)(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                              _ptr(st), _ptr(o), N, H, dk, dv,
                              nthreads or default_threads())
    if rc != 0:
        raise ValueError("oracle rejected the arguments")
    return o, st
