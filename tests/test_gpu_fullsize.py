"""GPU parity at the full workload sizes, in the launch configuration the
benchmark times.

The V=32000 problem is compared in full against the float64 oracle.  For the
larger ones the oracle's full-size values (every row's logsumexp and label
logit, the loss, the counts) were written by tests/golden/make_oracle_fullsize.py,
which calls only the oracle; dHidden is compared on 4096 seeded token rows and
dWeight on 4096 seeded vocabulary rows (the most frequent labels and both ends
among them), which the oracle computes one by one on the host cores.
"""
import os

import numpy as np
import pytest
import torch

import flce_inputs as fi
import lm_head_linear_tmem_b200 as flce
import oracle
from tests import _gpu as G

pytestmark = pytest.mark.gpu
IGN = fi.IGNORE_INDEX
SAMPLE_ROWS = 4096   # dHidden token rows compared at full size
SAMPLE_VOCAB = 4096  # dWeight vocabulary rows compared at full size
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def golden(name):
    path = os.path.join(GOLDEN, f"oracle_{name}.npz")
    if not os.path.exists(path):
        pytest.fail(f"missing {path}: run tests/golden/make_oracle_fullsize.py")
    return np.load(path)


def device_inputs(inp):
    return (G.bf16_tensor(inp.hidden_bits), G.bf16_tensor(inp.weight_bits),
            G.labels_tensor(inp.labels))


def sample_rows(labels, k, seed):
    g = np.random.default_rng(seed)
    N = len(labels)
    rows = set(g.choice(N, size=k, replace=False).tolist())
    rows |= {0, N - 1}
    ign = np.nonzero(labels == IGN)[0]
    if len(ign):
        rows |= set(g.choice(ign, size=min(4, len(ign)), replace=False).tolist())
    return np.array(sorted(rows))


def sample_vocab(labels, V, k, seed):
    g = np.random.default_rng(seed + 1)
    rows = set(g.choice(V, size=k, replace=False).tolist())
    valid = labels[labels != IGN]
    counts = np.bincount(valid, minlength=V)
    rows |= set(np.argsort(counts)[-6:].tolist())  # the most frequent labels
    rows |= {0, V - 1}
    return np.array(sorted(rows))


def test_v32k_mean_full_compare():
    inp = fi.make_inputs("v32k_mean")
    w = inp.workload
    h, W, y = device_inputs(inp)
    f = flce.forward(h, W, y, IGN, w.softcap, w.reduction, check_status=True)
    dh, dw = flce.backward(h, W, y, f.lse, softcap=w.softcap, reduction=w.reduction,
                           check_status=True)
    assert int(f.num_tokens.item()) == 0  # 'mean' returns num_tokens = 0
    H64, W64 = inp.hidden.astype(np.float64), inp.weight.astype(np.float64)
    rf = oracle.forward(H64, W64, inp.labels, IGN, w.softcap, w.reduction)
    G.check_loss(f.loss.item(), rf["loss"])
    G.check_lse(f.lse.cpu().numpy(), rf["lse"], inp.labels, w.V)
    rb = oracle.backward(H64, W64, inp.labels, IGN, w.softcap, w.reduction)
    dh_np, dw_np = dh.cpu().numpy(), dw.cpu().numpy()
    assert np.all(dh_np[inp.labels == IGN] == 0.0)
    assert G.rel_l2(dh_np, rb["d_hidden"]) <= G.GRAD_RL2
    assert G.rel_l2(dw_np, rb["d_weight"]) <= G.GRAD_RL2


def _check_sampled(inp, gold, lse_gpu, dh, dw, g, seed):
    w = inp.workload
    H64, W64 = inp.hidden.astype(np.float64), inp.weight.astype(np.float64)
    G.check_lse(lse_gpu, gold["lse"], inp.labels, w.V)
    ign = inp.labels == IGN
    assert np.all(dh[ign] == 0.0)
    assert np.all(np.isfinite(dh))
    rows = sample_rows(inp.labels, SAMPLE_ROWS, seed)
    ref_dh = oracle.d_hidden_rows(H64, W64, inp.labels, rows, g, IGN, w.softcap)
    assert G.rel_l2(dh[rows], ref_dh) <= G.GRAD_RL2
    vrows = sample_vocab(inp.labels, w.V, SAMPLE_VOCAB, seed)
    ref_dw = oracle.d_weight_rows(H64, W64, inp.labels, vrows, gold["lse"], g, IGN, w.softcap)
    got_dw = dw[vrows]
    assert np.all(np.isfinite(got_dw))
    assert G.rel_l2(got_dw, ref_dw) <= G.GRAD_RL2


@pytest.mark.parametrize("name", ["v131k_zipf", "v256k_softcap"])
def test_fullsize_sampled(name):
    gold = golden(name)
    inp = fi.make_inputs(name)
    w = inp.workload
    h, W, y = device_inputs(inp)
    f = flce.forward(h, W, y, IGN, w.softcap, w.reduction, check_status=True)
    dh, dw = flce.backward(h, W, y, f.lse, softcap=w.softcap, reduction=w.reduction,
                           check_status=True)
    torch.cuda.synchronize()
    assert int(f.num_tokens.item()) == int(gold["num_tokens"])
    G.check_loss(f.loss.item(), float(gold["loss"]))
    dh_np = dh.cpu().numpy()
    del dh
    dw_np = dw.cpu().numpy()
    del dw
    _check_sampled(inp, gold, f.lse.cpu().numpy(), dh_np, dw_np, 1.0, seed=sum(map(ord, name)))


def test_microbatch_token_weighted_scale():
    """4 micro-batches of 4096 tokens, micro-batch 1 all ignored; 'sum' with
    grad_scale = 1 / sum_k n_k; dWeight accumulated over the micro-batches by
    the library (accumulate flag), as a trainer does within one step."""
    gold = golden("microbatch")
    inp = fi.make_inputs("microbatch")
    w = inp.workload
    h, W, y = device_inputs(inp)
    n_tot = int(gold["num_valid"])
    gs = 1.0 / n_tot
    dw_acc = torch.empty(w.V, w.H, dtype=torch.float32, device="cuda")
    dh_all = torch.empty(w.N, w.H, dtype=torch.float32, device="cuda")
    lse_all = torch.empty(w.N, dtype=torch.float32, device="cuda")
    total = 0.0
    ntok = 0
    ws = flce.alloc_workspace(w.N // w.microbatches, w.H, w.V, torch.bfloat16, "cuda")
    slices = inp.microbatch_slices()
    for k, sl in enumerate(slices):
        f = flce.forward(h[sl], W, y[sl], IGN, 0.0, "sum", workspace=ws, lse=lse_all[sl],
                         check_status=True)
        flce.backward(h[sl], W, y[sl], f.lse, grad_scale=gs, workspace=ws, d_hidden=dh_all[sl],
                      d_weight=dw_acc, accumulate_d_weight=(k > 0), check_status=True)
        lk = f.loss.item()
        nk = int(f.num_tokens.item())
        assert nk == int(gold["mb_count"][k])
        G.check_loss(lk, float(gold["mb_loss"][k]))
        if k == w.empty_microbatch:
            assert lk == 0.0 and nk == 0
            assert bool(torch.all(dh_all[sl] == 0))
        total += lk
        ntok += nk
    assert ntok == n_tot
    G.check_loss(total, float(gold["loss"]))
    # the all-ignored micro-batch on its own adds exactly nothing to dWeight
    sl = slices[w.empty_microbatch]
    _, dw_empty = flce.backward(h[sl], W, y[sl], lse_all[sl], grad_scale=gs, workspace=ws,
                                check_status=True)
    assert bool(torch.all(dw_empty == 0))
    del dw_empty
    assert bool(torch.isfinite(dw_acc).all())
    torch.cuda.synchronize()
    _check_sampled(inp, gold, lse_all.cpu().numpy(), dh_all.cpu().numpy(),
                   dw_acc.cpu().numpy(), gs, seed=5)


def test_flat_offsets_beyond_int32():
    """V*H > 2^31: the top vocabulary rows of W and dWeight lie past the int32
    range of flat element offsets.  Half of the valid rows take labels there, so
    the dZ label entries, the dHidden W-row gathers and the dWeight label-term
    sums all touch those rows; lse and the loss are checked on every row,
    dWeight on the top rows (plus a sample) and dHidden on rows labelled in the
    top rows (plus ignored and low-label rows), against the oracle evaluated
    over vocabulary slices."""
    N, H, V = 256, 4096, (1 << 19) + 512  # V*H = 2^31 + 2^21 elements
    w = fi.custom_workload(N, H, V, seed=41, w_std=0.02, ignore_count=16)
    inp = fi.make_inputs(w)
    y = inp.labels.copy()
    valid = np.nonzero(y != IGN)[0]
    rng = np.random.default_rng(7)
    y[valid[::2]] = rng.integers(V - 512, V, size=len(valid[::2]))
    h = G.bf16_tensor(inp.hidden_bits)
    W = G.bf16_tensor(inp.weight_bits)
    yt = G.labels_tensor(y)
    f = flce.forward(h, W, yt, IGN, 0.0, "sum", check_status=True)
    dh, dw = flce.backward(h, W, yt, f.lse, check_status=True)
    torch.cuda.synchronize()
    lse_gpu = f.lse.cpu().numpy()
    top = torch.arange(V - 512, V, device="cuda")
    low = torch.from_numpy(np.sort(rng.choice(V - 512, size=64, replace=False))).cuda()
    vrows = torch.cat([low, top])
    dw_rows = dw[vrows].cpu().numpy()
    dh_np = dh.cpu().numpy()
    loss = f.loss.item()
    del dw, dh, W
    torch.cuda.empty_cache()
    lse_ref = oracle.lse_rows_sliced(inp.hidden, inp.weight, np.arange(N), vocab_slice=65536)
    G.check_lse(lse_gpu, lse_ref, y, V)
    ll = oracle.label_logits(inp.hidden, inp.weight, y, IGN)
    G.check_loss(loss, float(np.sum((lse_ref - ll)[y != IGN])))
    ref_dw = oracle.d_weight_rows(inp.hidden, inp.weight, y, vrows.cpu().numpy(), lse_ref, 1.0,
                                  IGN)
    assert G.rel_l2(dw_rows, ref_dw) <= G.GRAD_RL2
    assert G.rel_l2(dw_rows[64:], ref_dw[64:]) <= G.GRAD_RL2  # the rows past 2^31
    assert np.all(dh_np[y == IGN] == 0.0) and np.all(np.isfinite(dh_np))
    # dHidden rows whose label entry gathers a W row past 2^31 elements, plus a few
    # rows with low labels and ignored rows
    top_rows = np.nonzero(y >= V - 512)[0]
    other = np.nonzero((y < V - 512) & (y != IGN))[0][:16]
    ign_rows = np.nonzero(y == IGN)[0][:4]
    rows = np.sort(np.concatenate([top_rows, other, ign_rows]))
    ref_dh = oracle.d_hidden_rows_sliced(inp.hidden, inp.weight, y, rows, lse_ref[rows], 1.0,
                                         IGN, vocab_slice=65536)
    assert G.rel_l2(dh_np[rows], ref_dh) <= G.GRAD_RL2
    assert G.rel_l2(dh_np[top_rows], ref_dh[np.isin(rows, top_rows)]) <= G.GRAD_RL2
