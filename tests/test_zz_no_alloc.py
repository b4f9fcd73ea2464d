"""flce_forward_noalloc: the forward for callers that cannot allocate device
memory (an op/plugin interface that hands the kernel only its inputs and
outputs, or a program that has reserved all device memory in its own pool).
Its scratch is a static buffer inside the library, so these tests check that
it gives the same results as flce_forward with a caller workspace, on two
calls in a row (the buffer keeps the previous call's contents), and that it
refuses sizes its buffer cannot hold.

Collected last on purpose: it runs after every other GPU test, and also
passes alone in a fresh process.
"""
import numpy as np
import pytest
import torch

import flce_inputs as fi
import lm_head_linear_tmem_b200 as flce
from lm_head_linear_tmem_b200 import _native
from tests import _gpu as G

pytestmark = pytest.mark.gpu
IGN = fi.IGNORE_INDEX
REDUCTION = {"sum": 0, "mean": 1}


def call_noalloc(h, W, y, softcap, reduction, dtype=0):
    lib = _native.load()
    N, H = h.shape
    V = W.shape[0]
    loss = torch.empty((), dtype=torch.float32, device="cuda")
    ntok = torch.empty((), dtype=torch.int64, device="cuda")
    lse = torch.empty(N, dtype=torch.float32, device="cuda")
    status = torch.full((1,), 0x7F, dtype=torch.int32, device="cuda")
    rc = lib.flce_forward_noalloc(h.data_ptr(), W.data_ptr(), y.data_ptr(), N, H, V, IGN,
                                  float(softcap), REDUCTION[reduction], dtype, loss.data_ptr(),
                                  ntok.data_ptr(), lse.data_ptr(), status.data_ptr(),
                                  torch.cuda.current_stream().cuda_stream)
    assert rc == 0, _native.STATUS_NAMES.get(rc, rc)
    torch.cuda.synchronize()
    return loss.item(), int(ntok.item()), lse.cpu().numpy(), int(status.item())


def problems():
    a = G.small_inputs(N=300, H=200, V=1000, seed=21, n_ign=40, w_std=0.2)
    b = fi.make_inputs("v32k_mean")
    return [("ragged_softcap_sum", a, 5.0, "sum"), ("v32k_mean", b, 0.0, "mean")]


@pytest.mark.parametrize("idx", [0, 1])
def test_noalloc_forward_matches_workspace_forward(idx):
    name, inp, softcap, reduction = problems()[idx]
    h = G.bf16_tensor(inp.hidden_bits)
    W = G.bf16_tensor(inp.weight_bits)
    y = G.labels_tensor(inp.labels)
    ref = flce.forward(h, W, y, IGN, softcap, reduction, check_status=True)
    torch.cuda.synchronize()
    ref_loss, ref_ntok, ref_lse = ref.loss.item(), int(ref.num_tokens.item()), ref.lse.cpu().numpy()
    for _ in range(2):  # the second call reuses the buffer left by the first
        loss, ntok, lse, status = call_noalloc(h, W, y, softcap, reduction)
        assert status == 0
        assert ntok == ref_ntok
        G.check_loss(loss, ref_loss)
        assert np.max(np.abs(lse - ref_lse)) <= G.LSE_ATOL


def test_noalloc_reports_bad_labels_and_clears():
    inp = G.small_inputs(N=130, H=64, V=300, seed=22, n_ign=0)
    h = G.bf16_tensor(inp.hidden_bits)
    W = G.bf16_tensor(inp.weight_bits)
    bad = inp.labels.copy()
    bad[3] = 300  # == V
    _, _, _, status = call_noalloc(h, W, G.labels_tensor(bad), 0.0, "sum")
    assert status & 1
    _, _, _, status = call_noalloc(h, W, G.labels_tensor(inp.labels), 0.0, "sum")
    assert status == 0


def test_noalloc_refuses_sizes_beyond_its_buffer():
    lib = _native.load()
    fake = 0x10000  # never dereferenced: the size check comes first
    # N=16384, V=131072 needs 64 MiB of forward scratch, above the buffer
    rc = lib.flce_forward_noalloc(fake, fake, fake, 16384, 4096, 131072, IGN, 0.0, 0, 0, fake,
                                  fake, fake, None, None)
    assert rc == 2  # FLCE_ERR_SHAPE
