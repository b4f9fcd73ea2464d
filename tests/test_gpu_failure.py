"""Failure reporting on the GPU without any fault: a bounded mbarrier wait is
made to run out (nothing ever arrives on it), the kernel records the timeout in
the workspace status word and returns, the host reads FLCE_ERR_TIMEOUT, and the
context keeps working."""
import ctypes
import time

import pytest
import torch

import flce_inputs as fi
import lm_head_linear_tmem_b200 as flce
from lm_head_linear_tmem_b200 import _native
from tests import _gpu as G

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    lib = _native.load()
    ws = flce.alloc_workspace(64, 64, 512, torch.bfloat16, "cuda")
    ws.zero_()
    st = torch.cuda.current_stream().cuda_stream
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    assert lib.flce_selftest_wait_timeout(ctypes.c_void_p(ws.data_ptr()), 30, ctypes.c_void_p(st)) == 0
    assert flce.status(ws) == 6  # FLCE_ERR_TIMEOUT
    dt = time.perf_counter() - t0
    assert 0.025 <= dt < 5.0
    # the context still works and the next forward clears the status
    inp = fi.make_inputs("tiny")
    f = flce.forward(G.bf16_tensor(inp.hidden_bits), G.bf16_tensor(inp.weight_bits),
                     G.labels_tensor(inp.labels), workspace=ws, check_status=True)
    assert f.num_tokens.item() == 48


def test_selftest_rejects_bad_arguments():
    lib = _native.load()
    assert lib.flce_selftest_wait_timeout(None, 10, None) == 1
    ws = flce.alloc_workspace(64, 64, 512, torch.bfloat16, "cuda")
    assert lib.flce_selftest_wait_timeout(ctypes.c_void_p(ws.data_ptr()), 0, None) == 1
    assert lib.flce_selftest_wait_timeout(ctypes.c_void_p(ws.data_ptr()), 20000, None) == 1
