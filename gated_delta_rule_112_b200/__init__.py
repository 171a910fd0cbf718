"""Gated delta rule forward pass and decode step on B200 (sm_100a).

A thin ctypes binding over ``libgdn.so`` (C ABI in ``include/gdn.h``). This
module only marshals arguments: it allocates outputs and workspace with
PyTorch, passes device pointers and the current CUDA stream, and checks the
returned status. Every step of the computation runs in the library's CUDA
kernels; there is no CPU fallback -- if the library or a GPU is missing, the
calls raise.
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = ["chunk_fwd", "chunk_bwd", "chunk_fwd_save", "chunk_bwd_saved", "decode_step",
           "workspace_size", "chunk_path", "get_status",
           "lib", "GdnError", "BF16", "F32", "PATH_TCGEN05", "PATH_SIMT"]

_HERE = os.path.dirname(os.path.abspath(__file__))
# GDN_LIBRARY selects another build of the same library (e.g. the bounds-checked
# libgdn_checked.so); the default is the in-tree libgdn.so.
LIB_PATH = os.environ.get("GDN_LIBRARY") or os.path.join(_HERE, "libgdn.so")

(OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_WORKSPACE, ERR_CUDA, ERR_DEVICE_TIMEOUT,
 ERR_DEVICE_BOUNDS) = range(7)
BF16, F32 = 0, 1
PATH_TCGEN05, PATH_SIMT = 1, 2

_lib = None


class GdnError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {_status_string(code)} ({code})")


def _status_string(code: int) -> str:
    try:
        return lib().gdn_status_string(code).decode()
    except Exception:  # library missing
        return str(code)


def lib() -> ctypes.CDLL:
    """Load libgdn.so (built in-tree by ``gated_delta_rule_112_b200.build``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libgdn.so not built ({LIB_PATH}); run "
                               "python -m gated_delta_rule_112_b200.build")
        L = ctypes.CDLL(LIB_PATH)
        vp, fp, ip = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p
        ci, sz = ctypes.c_int, ctypes.c_size_t
        chunk_args = [vp, vp, vp, fp, fp, fp, ip, ci, ci, ci, ci, ci, ci, ci, ci, vp, fp, vp,
                      sz, vp]
        L.gdn_chunk_fwd.argtypes = chunk_args
        L.gdn_chunk_fwd.restype = ci
        L.gdn_chunk_fwd_simt.argtypes = chunk_args
        L.gdn_chunk_fwd_simt.restype = ci
        L.gdn_chunk_fwd_workspace_size.argtypes = [ci] * 8
        L.gdn_chunk_fwd_workspace_size.restype = sz
        L.gdn_chunk_fwd_scan_segments.argtypes = [ci] * 9
        L.gdn_chunk_fwd_scan_segments.restype = ci
        L.gdn_selftest_wait_timeout.argtypes = [vp, vp]
        L.gdn_selftest_wait_timeout.restype = ci
        L.gdn_chunk_fwd_path.argtypes = [ci] * 4
        L.gdn_chunk_fwd_path.restype = ci
        L.gdn_decode_step.argtypes = [vp, vp, vp, fp, fp, fp, vp, ci, ci, ci, ci, ci, vp]
        L.gdn_decode_step.restype = ci
        L.gdn_kda_chunk_fwd.argtypes = chunk_args
        L.gdn_kda_chunk_fwd.restype = ci
        L.gdn_kda_chunk_fwd_workspace_size.argtypes = [ci] * 8
        L.gdn_kda_chunk_fwd_workspace_size.restype = sz
        L.gdn_kda_decode_step.argtypes = L.gdn_decode_step.argtypes
        L.gdn_kda_decode_step.restype = ci
        L.gdn_chunk_bwd_workspace_size.argtypes = [ci] * 7
        L.gdn_chunk_bwd_workspace_size.restype = sz
        L.gdn_chunk_bwd_exact_workspace_size.argtypes = [ci] * 6
        L.gdn_chunk_bwd_exact_workspace_size.restype = sz
        L.gdn_chunk_bwd.argtypes = [vp, vp, vp, fp, fp, fp, ip, vp, fp, ci, ci, ci, ci, ci, ci,
                                    ci, fp, fp, fp, fp, fp, fp, vp, sz, vp]
        L.gdn_chunk_bwd.restype = ci
        L.gdn_chunk_bwd_saved.argtypes = L.gdn_chunk_bwd.argtypes
        L.gdn_chunk_bwd_saved.restype = ci
        L.gdn_chunk_fwd_save.argtypes = [vp, vp, vp, fp, fp, fp, ip, ci, ci, ci, ci, ci, ci, ci,
                                         vp, fp, vp, sz, vp]
        L.gdn_chunk_fwd_save.restype = ci
        L.gdn_chunk_bwd_exact.argtypes = [vp, vp, vp, fp, fp, fp, ip, vp, fp, ci, ci, ci, ci, ci, ci,
                                    ci, fp, fp, fp, fp, fp, fp, vp, sz, vp]
        L.gdn_chunk_bwd_exact.restype = ci
        L.gdn_get_status.argtypes = [vp, vp]
        L.gdn_get_status.restype = ci
        L.gdn_set_profile_events.argtypes = [vp, vp, vp, vp]
        L.gdn_set_profile_events.restype = ci
        L.gdn_checked_build.argtypes = []
        L.gdn_checked_build.restype = ci
        L.gdn_status_string.argtypes = [ci]
        L.gdn_status_string.restype = ctypes.c_char_p
        _lib = L
    return _lib


def _dtype_code(t: torch.dtype) -> int:
    if t == torch.bfloat16:
        return BF16
    if t == torch.float32:
        return F32
    raise TypeError(f"unsupported dtype {t}; use bfloat16 or float32")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_ptr(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(code: int, what: str):
    if code != OK:
        raise GdnError(code, what)


def workspace_size(B, T, H, d_k, d_v, num_seqs=0, chunk=64, dtype=torch.bfloat16) -> int:
    return int(lib().gdn_chunk_fwd_workspace_size(B, T, H, d_k, d_v, num_seqs, chunk,
                                                  _dtype_code(dtype)))


def chunk_path(d_k, d_v, chunk=64, dtype=torch.bfloat16) -> int:
    return int(lib().gdn_chunk_fwd_path(d_k, d_v, chunk, _dtype_code(dtype)))


def _require_cuda(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("all tensors must be contiguous CUDA tensors")


def chunk_fwd(q, k, v, g, beta, initial_state=None, cu_seqlens=None, chunk=64,
              output_final_state=True, workspace=None, out=None, force_simt=False,
              stream=None):
    """Chunkwise forward pass. Returns ``(o, final_state or None)``.

    q, k: [B,T,H,d_k]; v: [B,T,H,d_v] (bf16 or fp32, same dtype); g (= log
    alpha), beta: [B,T,H] fp32; initial_state: [N,H,d_k,d_v] fp32 or None;
    cu_seqlens: int32 [N+1] CUDA tensor (packed sequences, B == 1) or None.
    """
    fn = lib().gdn_chunk_fwd_simt if force_simt else lib().gdn_chunk_fwd
    return _chunk_call(fn, "gdn_chunk_fwd", lib().gdn_chunk_fwd_workspace_size, q, k, v, g,
                       beta, initial_state, cu_seqlens, chunk, output_final_state, workspace,
                       out, stream, channel_gate=False)


def kda_workspace_size(B, T, H, d_k, d_v, num_seqs=0, chunk=64, dtype=torch.bfloat16) -> int:
    return int(lib().gdn_kda_chunk_fwd_workspace_size(B, T, H, d_k, d_v, num_seqs, chunk,
                                                      _dtype_code(dtype)))


def kda_chunk_fwd(q, k, v, g, beta, initial_state=None, cu_seqlens=None, chunk=64,
                  output_final_state=True, workspace=None, out=None, stream=None):
    """Chunkwise forward pass with the channel-wise gate: as ``chunk_fwd`` but
    g (= log alpha) is [B,T,H,d_k] fp32. Returns ``(o, final_state or None)``."""
    return _chunk_call(lib().gdn_kda_chunk_fwd, "gdn_kda_chunk_fwd",
                       lib().gdn_kda_chunk_fwd_workspace_size, q, k, v, g, beta, initial_state,
                       cu_seqlens, chunk, output_final_state, workspace, out, stream,
                       channel_gate=True)


def _chunk_call(fn, name, ws_fn, q, k, v, g, beta, initial_state, cu_seqlens, chunk,
                output_final_state, workspace, out, stream, channel_gate):
    _require_cuda(q, k, v, g, beta, initial_state, cu_seqlens)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if tuple(g.shape) != ((B, T, H, dk) if channel_gate else (B, T, H)):
        raise ValueError(f"{name}: g has shape {tuple(g.shape)}")
    num_seqs = 0 if cu_seqlens is None else cu_seqlens.numel() - 1
    N = num_seqs if cu_seqlens is not None else B
    dt = _dtype_code(q.dtype)
    o = torch.empty(B, T, H, dv, dtype=q.dtype, device=q.device) if out is None else out
    fs = (torch.empty(N, H, dk, dv, dtype=torch.float32, device=q.device)
          if output_final_state else None)
    need = int(ws_fn(B, T, H, dk, dv, num_seqs, chunk, dt))
    if need == 0:
        raise GdnError(ERR_INVALID_ARG, name + "_workspace_size")
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    rc = fn(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(initial_state),
            _ptr(cu_seqlens), B, T, H, dk, dv, num_seqs, chunk, dt, _ptr(o), _ptr(fs),
            _ptr(workspace), workspace.numel(), _stream_ptr(stream))
    _check(rc, name)
    return o, fs


def bwd_workspace_size(B, T, H, d_k, d_v, num_seqs=0, dtype=torch.bfloat16,
                       exact=False) -> int:
    """Workspace bytes of ``chunk_bwd`` (exact=False: the path gdn_chunk_bwd
    picks for dtype; exact=True: the token-level fp32 path)."""
    if exact:
        return int(lib().gdn_chunk_bwd_exact_workspace_size(B, T, H, d_k, d_v, num_seqs))
    return int(lib().gdn_chunk_bwd_workspace_size(B, T, H, d_k, d_v, num_seqs,
                                                   _dtype_code(dtype)))


def chunk_bwd(q, k, v, g, beta, d_o, initial_state=None, cu_seqlens=None, d_final_state=None,
              workspace=None, stream=None, exact=False, _saved=False):
    """Gradients of ``chunk_fwd`` (scalar gate) for the loss
    sum(d_o * o) + sum(d_final_state * final_state).

    Inputs as for ``chunk_fwd``, plus d_o [B,T,H,d_v] (same dtype as v) and
    d_final_state [N,H,d_k,d_v] fp32 or None. Returns a dict of fp32 CUDA
    tensors: dq, dk [B,T,H,d_k], dv [B,T,H,d_v], dg, dbeta [B,T,H],
    d_initial_state [N,H,d_k,d_v]. bf16 with d_k = d_v = 128 runs the chunkwise
    tensor-core backward; exact=True (or any other size or dtype) the
    token-level fp32 backward.
    """
    _require_cuda(q, k, v, g, beta, d_o, initial_state, cu_seqlens, d_final_state)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    num_seqs = 0 if cu_seqlens is None else cu_seqlens.numel() - 1
    N = num_seqs if cu_seqlens is not None else B
    dev = q.device
    f32 = dict(dtype=torch.float32, device=dev)
    out = dict(dq=torch.empty(B, T, H, dk, **f32), dk=torch.empty(B, T, H, dk, **f32),
               dv=torch.empty(B, T, H, dv, **f32), dg=torch.empty(B, T, H, **f32),
               dbeta=torch.empty(B, T, H, **f32),
               d_initial_state=torch.empty(N, H, dk, dv, **f32))
    need = bwd_workspace_size(B, T, H, dk, dv, num_seqs, q.dtype, exact)
    if need == 0:
        raise GdnError(ERR_INVALID_ARG, "gdn_chunk_bwd_workspace_size")
    if _saved:
        if workspace is None or workspace.numel() < need:
            raise GdnError(ERR_WORKSPACE, "gdn_chunk_bwd_saved")
    elif workspace is None or workspace.numel() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    fn = (lib().gdn_chunk_bwd_saved if _saved else
          lib().gdn_chunk_bwd_exact if exact else lib().gdn_chunk_bwd)
    name = "gdn_chunk_bwd_saved" if _saved else "gdn_chunk_bwd_exact" if exact else "gdn_chunk_bwd"
    rc = fn(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(initial_state),
            _ptr(cu_seqlens), _ptr(d_o), _ptr(d_final_state), B, T, H, dk, dv,
            num_seqs, _dtype_code(q.dtype), _ptr(out["dq"]), _ptr(out["dk"]),
            _ptr(out["dv"]), _ptr(out["dg"]), _ptr(out["dbeta"]),
            _ptr(out["d_initial_state"]), _ptr(workspace), workspace.numel(),
            _stream_ptr(stream))
    _check(rc, name)
    return out


def chunk_fwd_save(q, k, v, g, beta, initial_state=None, cu_seqlens=None,
                   output_final_state=True, workspace=None, out=None, stream=None):
    """Forward pass of a training step (bf16, d_k = d_v = 128): ``chunk_fwd``
    that also keeps in its workspace what ``chunk_bwd_saved`` needs (the chunk
    map, the prep tiles and every chunk's entering state). Returns ``(o,
    final_state or None, saved)``; hand ``saved`` unchanged to
    ``chunk_bwd_saved`` with the same inputs."""
    _require_cuda(q, k, v, g, beta, initial_state, cu_seqlens)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if tuple(g.shape) != (B, T, H):
        raise ValueError(f"gdn_chunk_fwd_save: g has shape {tuple(g.shape)}")
    num_seqs = 0 if cu_seqlens is None else cu_seqlens.numel() - 1
    N = num_seqs if cu_seqlens is not None else B
    o = torch.empty(B, T, H, dv, dtype=q.dtype, device=q.device) if out is None else out
    fs = (torch.empty(N, H, dk, dv, dtype=torch.float32, device=q.device)
          if output_final_state else None)
    need = bwd_workspace_size(B, T, H, dk, dv, num_seqs, q.dtype)
    if need == 0:
        raise GdnError(ERR_INVALID_ARG, "gdn_chunk_bwd_workspace_size")
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    rc = lib().gdn_chunk_fwd_save(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                                  _ptr(initial_state), _ptr(cu_seqlens), B, T, H, dk, dv,
                                  num_seqs, _dtype_code(q.dtype), _ptr(o), _ptr(fs),
                                  _ptr(workspace), workspace.numel(), _stream_ptr(stream))
    _check(rc, "gdn_chunk_fwd_save")
    return o, fs, workspace


def chunk_bwd_saved(q, k, v, g, beta, d_o, saved, initial_state=None, cu_seqlens=None,
                    d_final_state=None, stream=None):
    """``chunk_bwd`` from the workspace ``saved`` that ``chunk_fwd_save`` filled
    for the same inputs: the forward replay is skipped. Returns the same dict
    of fp32 gradients."""
    return chunk_bwd(q, k, v, g, beta, d_o, initial_state, cu_seqlens, d_final_state,
                     workspace=saved, stream=stream, _saved=True)


def get_status(workspace=None, stream=None) -> int:
    """Synchronise the stream and return the first recorded error code."""
    return int(lib().gdn_get_status(_ptr(workspace), _stream_ptr(stream)))


def decode_step(q, k, v, g, beta, state, out=None, stream=None):
    """One recurrent step, updating ``state`` [N,H,d_k,d_v] fp32 in place.

    q, k: [N,H,d_k]; v: [N,H,d_v]; g, beta: [N,H] fp32. Returns o [N,H,d_v].
    """
    return _decode_call(lib().gdn_decode_step, "gdn_decode_step", q, k, v, g, beta, state,
                        out, stream, channel_gate=False)


def kda_decode_step(q, k, v, g, beta, state, out=None, stream=None):
    """One channel-wise-gated step (g: [N,H,d_k] fp32), ``state`` updated in place."""
    return _decode_call(lib().gdn_kda_decode_step, "gdn_kda_decode_step", q, k, v, g, beta,
                        state, out, stream, channel_gate=True)


def _decode_call(fn, name, q, k, v, g, beta, state, out, stream, channel_gate):
    _require_cuda(q, k, v, g, beta, state)
    N, H, dk = q.shape
    dv = v.shape[-1]
    if tuple(g.shape) != ((N, H, dk) if channel_gate else (N, H)):
        raise ValueError(f"{name}: g has shape {tuple(g.shape)}")
    o = torch.empty(N, H, dv, dtype=q.dtype, device=q.device) if out is None else out
    rc = fn(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(state), _ptr(o), N, H, dk, dv,
            _dtype_code(q.dtype), _stream_ptr(stream))
    _check(rc, name)
    return o
