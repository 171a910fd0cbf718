"""Helpers shared by the GPU parity tests: run the CUDA path and the oracle on
the same seeded bytes and compare with the tolerances the tests state."""
import numpy as np
import torch

import oracle

# Relative L2 thresholds: bf16 inputs (tensor-core path, bf16 operands, fp32
# accumulation) and fp32 inputs (fp32 CUDA-core path).
TOL_BF16 = 5e-3
TOL_F32 = 1e-5

# Every comparison made through assert_close, in order: the test that made it,
# the tensor's name, relative L2, max-abs and the tolerance. conftest.py prints
# them at the end of the session and writes them as JSON when the environment
# variable GDN_PARITY_MARGINS names a file.
RECORDS = []
CURRENT_TEST = {"id": None}


def np64(t):
    return None if t is None else t.detach().float().cpu().double().numpy()


def rel_l2(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(got - ref) / (den if den > 0 else 1.0))


def max_abs(got, ref):
    return float(np.max(np.abs(np.asarray(got, np.float64) - np.asarray(ref, np.float64)))) \
        if np.size(ref) else 0.0


def oracle_chunk(inp, heads=None):
    """Oracle on the inputs dict from make_chunk_inputs (optionally a head subset)."""
    sl = slice(None) if heads is None else heads
    s0 = inp["initial_state"]
    cu = inp["cu_seqlens"]
    return oracle.chunk_fwd(np64(inp["q"][:, :, sl]), np64(inp["k"][:, :, sl]),
                            np64(inp["v"][:, :, sl]), np64(inp["g"][:, :, sl]),
                            np64(inp["beta"][:, :, sl]),
                            None if s0 is None else np64(s0[:, sl]),
                            None if cu is None else cu.numpy())


def to_dev(inp, dev="cuda"):
    out = {}
    for key in ("q", "k", "v", "g", "beta", "initial_state", "cu_seqlens"):
        t = inp[key]
        out[key] = None if t is None else t.to(dev)
    return out


def gpu_chunk(inp, force_simt=False, chunk=None):
    import gated_delta_rule_112_b200 as gdn
    d = to_dev(inp)
    o, fs = gdn.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["initial_state"],
                          d["cu_seqlens"], chunk=chunk or inp["chunk"], force_simt=force_simt)
    torch.cuda.synchronize()
    return o, fs


def assert_close(name, got, ref, tol):
    r = rel_l2(got, ref)
    m = max_abs(got, ref)
    RECORDS.append({"test": CURRENT_TEST["id"], "tensor": name, "rel_l2": r, "max_abs": m,
                    "ref_max_abs": float(np.max(np.abs(ref))) if np.size(ref) else 0.0,
                    "tol": tol, "passed": bool(np.all(np.isfinite(got)) and r <= tol)})
    assert np.all(np.isfinite(got)), f"{name}: non-finite values"
    assert r <= tol, f"{name}: rel-L2 {r:.3e} > {tol:.1e} (max-abs {m:.3e})"
    return r, m
