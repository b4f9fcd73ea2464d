"""The CUDA path inside a captured CUDA graph and on concurrent streams.

Every call is asynchronous on the caller's stream and allocates nothing, so a
forward + backward step can be captured once and replayed (the inputs updated in
place between replays), and two independent problems with their own workspaces
can run on two streams at once.  Both must give, bit for bit, what eager
sequential calls give."""
import numpy as np
import pytest
import torch

import flce_inputs as fi
import lm_head_linear_tmem_b200 as flce
from lm_head_linear_tmem_b200 import _native
from tests import _gpu as G

pytestmark = pytest.mark.gpu
IGN = fi.IGNORE_INDEX


def _problem(seed, N=4500, H=136, V=9000):
    inp = G.small_inputs(N=N, H=H, V=V, seed=seed, n_ign=N // 10, w_std=0.1)
    return (G.bf16_tensor(inp.hidden_bits), G.bf16_tensor(inp.weight_bits),
            G.labels_tensor(inp.labels))


def _eager(h, W, y, softcap):
    f = flce.forward(h, W, y, IGN, softcap, "sum", check_status=True)
    dh, dw = flce.backward(h, W, y, f.lse, softcap=softcap, check_status=True)
    torch.cuda.synchronize()
    return f.loss.clone(), f.lse.clone(), dh, dw


@pytest.mark.parametrize("softcap,buffers", [(0.0, 1), (3.0, 1), (3.0, 2)])
def test_graph_capture_replays_identically(softcap, buffers):
    h, W, y = _problem(30)
    h2, _, y2 = _problem(31)
    N, H = h.shape
    V = W.shape[0]
    # several chunks, so the capture holds the whole schedule (with two dZ blocks,
    # the chunks' dZ and gradient launches overlap inside the graph)
    with G.chunks(1024, 2048), _native.options(dz_buffers=buffers):
        ref1 = _eager(h, W, y, softcap)
        ref2 = _eager(h2, W, y2, softcap)
        hs, ys = h.clone(), y.clone()  # the graph's static inputs
        ws = flce.alloc_workspace(N, H, V, torch.bfloat16, "cuda")
        lse = torch.empty(N, device="cuda")
        dh = torch.empty(N, H, device="cuda")
        dw = torch.empty(V, H, device="cuda")

        def step():
            f = flce.forward(hs, W, ys, IGN, softcap, "sum", workspace=ws, lse=lse)
            flce.backward(hs, W, ys, lse, softcap=softcap, workspace=ws, d_hidden=dh,
                          d_weight=dw)
            return f.loss

        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):  # warm-up outside the capture
            step()
        torch.cuda.current_stream().wait_stream(side)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            loss = step()
        for hin, yin, ref in ((h, y, ref1), (h2, y2, ref2), (h, y, ref1)):
            hs.copy_(hin)
            ys.copy_(yin)
            graph.replay()
            torch.cuda.synchronize()
            assert flce.status(ws) == 0
            assert torch.equal(loss, ref[0]) and torch.equal(lse, ref[1])
            assert torch.equal(dh, ref[2]) and torch.equal(dw, ref[3])
        del graph


def test_two_streams_at_once():
    probs = [_problem(32), _problem(33, N=3000, H=200, V=7000)]
    refs = [_eager(*p, 0.0) for p in probs]
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    outs = []
    torch.cuda.synchronize()
    for p, s in zip(probs, streams):
        with torch.cuda.stream(s):
            for t in p:
                t.record_stream(s)
            f = flce.forward(*p)
            dh, dw = flce.backward(*p, f.lse)
            outs.append((f.loss, f.lse, dh, dw))
    torch.cuda.synchronize()
    for got, ref in zip(outs, refs):
        for a, b in zip(got, ref):
            assert torch.equal(a, b)


@pytest.mark.parametrize("buffers", [1, 2])
def test_many_steps_back_to_back(buffers):
    """Forty forward + backward steps enqueued without a host synchronisation in
    between (so successive calls' dependent launches overlap on the device, and
    with two dZ blocks the chunks' dZ and gradient launches overlap as well):
    no bounded wait runs out and every step's results are bit-identical."""
    h, W, y = _problem(35, N=3000, H=192, V=7000)
    N, H = h.shape
    V = W.shape[0]
    with G.chunks(1024, 2048), _native.options(dz_buffers=buffers):
        ref = _eager(h, W, y, 2.0)
        ws = flce.alloc_workspace(N, H, V, torch.bfloat16, "cuda")
        outs = []
        for _ in range(40):
            f = flce.forward(h, W, y, IGN, 2.0, "sum", workspace=ws)
            dh, dw = flce.backward(h, W, y, f.lse, softcap=2.0, workspace=ws)
            outs.append((f.loss, f.lse, dh, dw))
        torch.cuda.synchronize()
        assert flce.status(ws) == 0
    for got in outs:
        for a, b in zip(got, ref):
            assert torch.equal(a, b)
