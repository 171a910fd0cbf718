"""GPU parity of gdn_decode_step against the fp64 oracle (through the C ABI)."""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_112_b200.inputs import make_decode_inputs
from tests.parity import TOL_BF16, TOL_F32, assert_close, np64

pytestmark = pytest.mark.gpu


def run_steps(d, steps, dtype=None):
    import gated_delta_rule_112_b200 as gdn
    st = d["state"].cuda()
    outs = []
    for t in range(steps):
        o = gdn.decode_step(d["q"][t].cuda(), d["k"][t].cuda(), d["v"][t].cuda(),
                            d["g"][t].cuda(), d["beta"][t].cuda(), st)
        outs.append(o.float().cpu())
    torch.cuda.synchronize()
    return outs, st.cpu()


def oracle_steps(d, steps, units=None):
    st = np64(d["state"])
    if units is not None:
        st = st[units[0], units[1]][:, None]
    outs = []
    for t in range(steps):
        q, k, v, g, b = (np64(d[key][t]) for key in ("q", "k", "v", "g", "beta"))
        if units is not None:
            q, k, v, g, b = (x[units[0], units[1]][:, None] for x in (q, k, v, g, b))
        o, st = oracle.decode_step(q, k, v, g, b, st)
        outs.append(o)
    return outs, st


@pytest.mark.parametrize("dtype,dk,dv,tol", [(torch.bfloat16, 128, 128, TOL_BF16),
                                             (torch.float32, 128, 128, TOL_F32),
                                             (torch.float32, 64, 32, TOL_F32),
                                             (torch.bfloat16, 96, 64, TOL_BF16)])
def test_decode_small_chained(dtype, dk, dv, tol):
    from gated_delta_rule_112_b200.inputs import Workload
    w = Workload("t", B=5, T=1, H=3, d_k=dk, d_v=dv, dtype=dtype, random_state=True, seed=7,
                 steps=4)
    d = make_decode_inputs(w)
    got, st = run_steps(d, 4)
    ref, rst = oracle_steps(d, 4)
    for t in range(4):
        assert_close(f"o step {t}", got[t].numpy(), ref[t], tol)
    assert_close("state", st.numpy(), rst, tol)


def test_workload_decode_full_size():
    """The full decode workload (N=256, H=32, d=128, 64 steps), every state and
    every output of every step against the oracle."""
    d = make_decode_inputs("decode")
    steps = d["steps"]
    got, st = run_steps(d, steps)
    ref, rst = oracle_steps(d, steps)
    worst = 0.0
    for t in range(steps):
        r, _ = assert_close(f"o step {t}", got[t].numpy(), ref[t], TOL_BF16)
        worst = max(worst, r)
    assert_close("o all 64 steps", np.stack([g.numpy() for g in got]), np.stack(ref), TOL_BF16)
    assert_close("state after 64 steps", st.numpy(), rst, TOL_BF16)
