"""Failure handling on the GPU, without a GPU fault: a bounded device-side
wait that can never complete must give up, be reported as
GDN_ERR_DEVICE_TIMEOUT, and leave the CUDA context usable."""
import pytest
import torch

import gated_delta_rule_112_b200 as gdn
from gated_delta_rule_112_b200.inputs import Workload, make_chunk_inputs
from tests.parity import TOL_BF16, assert_close, gpu_chunk, np64, oracle_chunk

pytestmark = pytest.mark.gpu


def test_bounded_wait_expires_and_is_reported():
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    assert gdn.lib().gdn_selftest_wait_timeout(ws.data_ptr(), stream) == gdn.OK
    assert gdn.get_status(ws) == gdn.ERR_DEVICE_TIMEOUT
    assert gdn.get_status(ws) == gdn.OK          # the error word was cleared
    # the context still works: a normal call matches the oracle
    inp = make_chunk_inputs(Workload("after_timeout", B=1, T=100, H=1, d_k=128, d_v=128,
                                     seed=41), random_state=True)
    o, fs = gpu_chunk(inp)
    ro, rfs = oracle_chunk(inp)
    assert_close("o", np64(o), ro, TOL_BF16)
    assert_close("final_state", np64(fs), rfs, TOL_BF16)


def test_selftest_rejects_a_missing_workspace():
    assert gdn.lib().gdn_selftest_wait_timeout(None, None) == gdn.ERR_WORKSPACE
