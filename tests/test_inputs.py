"""The seeded generator: determinism and the stated distributions."""
import hashlib

import torch

from gated_delta_rule_112_b200.inputs import make_chunk_inputs, make_decode_inputs


def digest(d):
    h = hashlib.sha256()
    for key in ("q", "k", "v", "g", "beta", "initial_state", "cu_seqlens", "state"):
        t = d.get(key)
        if t is not None:
            h.update(t.contiguous().view(torch.uint8).numpy().tobytes())
    return h.hexdigest()


def test_same_seed_same_bytes():
    a = make_chunk_inputs("b4h16t4096", T=128, B=2, H=2)
    b = make_chunk_inputs("b4h16t4096", T=128, B=2, H=2)
    assert digest(a) == digest(b)
    c = make_chunk_inputs("b4h16t4096", T=128, B=2, H=2, seed=99)
    assert digest(a) != digest(c)


def test_distributions():
    d = make_chunk_inputs("b4h16t4096", T=256, B=2, H=4)
    assert d["q"].dtype == torch.bfloat16 and d["g"].dtype == torch.float32
    n = d["k"].float().norm(dim=-1)
    assert torch.allclose(n, torch.ones_like(n), atol=1e-2)
    assert (d["beta"] > 0).all() and (d["beta"] < 1).all()
    assert (d["g"] < 0).all()
    assert d["initial_state"] is None


def test_varlen_lengths_and_cu():
    d = make_chunk_inputs("varlen64", H=2)
    cu = d["cu_seqlens"]
    lens = (cu[1:] - cu[:-1])
    assert cu[0] == 0 and int(cu[-1]) == d["T"] and len(lens) == 64
    assert int(lens.min()) >= 128 and int(lens.max()) <= 2048


def test_decode_inputs():
    d = make_decode_inputs(N=4, H=2, steps=3)
    assert d["state"].shape == (4, 2, 128, 128) and d["q"].shape == (3, 4, 2, 128)
    assert abs(float(d["state"].std()) - 0.02) < 2e-3


def test_beta_up_to_two_workload_draws_the_same_bytes_scaled():
    a = make_chunk_inputs("b4h16t4096", T=128, seed=5)
    b = make_chunk_inputs("b4h16t4096_beta2", T=128)
    assert torch.equal(a["q"], b["q"]) and torch.equal(a["g"], b["g"])
    assert torch.allclose(b["beta"], 2.0 * a["beta"])
    assert float(b["beta"].min()) > 0.0 and float(b["beta"].max()) < 2.0
    assert float(b["beta"].max()) > 1.0
