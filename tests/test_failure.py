"""Failure detection without a GPU fault: a wait that nothing satisfies gives
up after its bound and reports TRI_ATTN_ERR_TIMEOUT in the status word; the
context stays usable and the next call runs clean. Host-side argument checks
of the diagnostic entry point run without a GPU."""

import ctypes

import pytest
import torch

import triangle_attention_b200 as ta
from helpers import to_device
from tri_inputs import STARTING, make_inputs

TIMEOUT = 5


def test_diagnostic_rejects_bad_workspace():
    lib = ta.lib()
    assert lib.tri_attn_check_wait_timeout(None, 1024, None) == 3
    assert lib.tri_attn_check_wait_timeout(ctypes.c_void_p(4100), 1024, None) == 3
    assert lib.tri_attn_check_wait_timeout(ctypes.c_void_p(4096), 64, None) == 3


@pytest.mark.gpu
def test_unsatisfied_wait_reports_timeout_and_context_survives():
    ws = ta.workspace(256, torch.device("cuda:0"))
    assert ta.check_wait_timeout(ws) == TIMEOUT
    assert ta.STATUS[TIMEOUT] == "device wait timed out"
    # the same word through the query call of the boundary
    assert ta.get_status(ws) == TIMEOUT
    # the same context runs a normal forward and backward afterwards
    g = to_device(make_inputs(136, H=2, c=32, dtype="bf16", seed=3), "cuda:0")
    prob = ta.problem(g["q"], g["mask"], STARTING)
    ws_b = ta.workspace(ta.bwd_workspace_size(prob), g["q"].device)
    out, lse = ta.fwd(g["q"], g["k"], g["v"], g["bias"], g["gate"], g["mask"], STARTING)
    ta.bwd(g["q"], g["k"], g["v"], g["bias"], g["gate"], g["mask"], out, lse, g["dout"],
           STARTING, ws=ws_b)
    assert ta.read_status(ws_b) == 0
    assert ta.get_status(ws_b) == 0
    assert torch.isfinite(lse).all()
