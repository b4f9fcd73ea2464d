"""GPU parity of the CUDA path (through the C ABI) against the float64 oracle
on small problems that span several tiles, ragged tails and several backward
chunks, plus the edge cases of the method."""
import contextlib

import numpy as np
import pytest
import torch

import flce_inputs as fi
import lm_head_linear_tmem_b200 as flce
import oracle
from lm_head_linear_tmem_b200 import _native
from tests import _gpu as G

pytestmark = pytest.mark.gpu
IGN = fi.IGNORE_INDEX


def run(h, w, y, softcap, reduction, grad_scale=1.0, grad_output=None, ignore_index=IGN):
    f = flce.forward(h, w, y, ignore_index, softcap, reduction, check_status=True)
    dh, dw = flce.backward(h, w, y, f.lse, grad_output=grad_output, grad_scale=grad_scale,
                           ignore_index=ignore_index, softcap=softcap, reduction=reduction,
                           check_status=True)
    torch.cuda.synchronize()
    return dict(loss=f.loss.item(), ntok=int(f.num_tokens.item()), lse=f.lse.cpu().numpy(),
                dh=dh.cpu().numpy(), dw=dw.cpu().numpy(), loss_dtype=f.loss.dtype)


def compare(got, hidden, weight, labels, softcap, reduction, grad_scale=1.0, grad_output=1.0,
            ignore_index=IGN):
    rf = oracle.forward(hidden, weight, labels, ignore_index, softcap, reduction)
    rb = oracle.backward(hidden, weight, labels, ignore_index, softcap, reduction,
                         grad_output=grad_output, grad_scale=grad_scale)
    assert got["loss_dtype"] == torch.float32
    assert got["ntok"] == rf["num_tokens"]
    G.check_loss(got["loss"], rf["loss"])
    G.check_lse(got["lse"], rf["lse"], labels, weight.shape[0], ignore_index)
    ign = labels == ignore_index
    assert np.all(got["dh"][ign] == 0.0), "ignored rows must get exact zero gradient"
    assert np.all(np.isfinite(got["dh"])) and np.all(np.isfinite(got["dw"]))
    assert G.rel_l2(got["dh"], rb["d_hidden"]) <= G.GRAD_RL2
    assert G.rel_l2(got["dw"], rb["d_weight"]) <= G.GRAD_RL2
    return rf, rb


def test_tiny_bf16_tensor_core_path():
    inp = fi.make_inputs("tiny")
    w = inp.workload
    got = run(G.bf16_tensor(inp.hidden_bits), G.bf16_tensor(inp.weight_bits),
              G.labels_tensor(inp.labels), w.softcap, w.reduction)
    compare(got, inp.hidden, inp.weight, inp.labels, w.softcap, w.reduction)


def test_tiny_fp32_cuda_core_path():
    inp = fi.make_inputs("tiny", keep_raw=True)
    w = inp.workload
    got = run(G.f32_tensor(inp.hidden_raw), G.f32_tensor(inp.weight_raw),
              G.labels_tensor(inp.labels), w.softcap, w.reduction)
    rf, rb = compare(got, inp.hidden_raw, inp.weight_raw, inp.labels, w.softcap, w.reduction)
    # fp32 end to end: much tighter than the bf16-operand bar
    assert G.rel_l2(got["dh"], rb["d_hidden"]) <= 1e-5
    assert G.rel_l2(got["dw"], rb["d_weight"]) <= 1e-5


@pytest.mark.parametrize("softcap", [0.0, 5.0])
@pytest.mark.parametrize("reduction", ["sum", "mean"])
def test_ragged_multi_tile(softcap, reduction):
    # N, V not multiples of the 128 x 256 tile; H not a multiple of the 64 K-block
    inp = G.small_inputs(N=300, H=200, V=1000, seed=7, n_ign=60, w_std=0.2)
    go = torch.tensor(0.75, device="cuda")
    got = run(G.bf16_tensor(inp.hidden_bits), G.bf16_tensor(inp.weight_bits),
              G.labels_tensor(inp.labels), softcap, reduction, grad_scale=1.3, grad_output=go)
    compare(got, inp.hidden, inp.weight, inp.labels, softcap, reduction, grad_scale=1.3,
            grad_output=0.75)


SMALL_CHUNKS = (1024, 2048)  # tokens x vocab per backward chunk in the multi-chunk tests


@pytest.mark.parametrize("chunked", [False, True])
@pytest.mark.parametrize("softcap", [0.0, 3.0])
def test_several_backward_chunks(softcap, chunked):
    # default chunks: one chunk; 1024 x 2048 chunks: 5 token x 5 vocab chunks, which
    # exercises the cross-chunk accumulation (dWeight TMA reduce-add, dHidden
    # read-add-write) and the ragged last chunk of each dimension
    inp = G.small_inputs(N=4500, H=136, V=9000, seed=8, n_ign=450, w_std=0.1)
    with G.chunks(*SMALL_CHUNKS) if chunked else contextlib.nullcontext():
        got = run(G.bf16_tensor(inp.hidden_bits), G.bf16_tensor(inp.weight_bits),
                  G.labels_tensor(inp.labels), softcap, "sum", grad_scale=1.0 / 4050)
    compare(got, inp.hidden, inp.weight, inp.labels, softcap, "sum", grad_scale=1.0 / 4050)


def test_all_ignored_gives_zero_not_nan():
    inp = G.small_inputs(N=200, H=64, V=700, seed=9, n_ign=0)
    y = np.full(200, IGN, dtype=np.int64)
    for red in ("sum", "mean"):
        got = run(G.bf16_tensor(inp.hidden_bits), G.bf16_tensor(inp.weight_bits),
                  G.labels_tensor(y), 0.0, red)
        assert got["loss"] == 0.0 and got["ntok"] == 0
        assert np.all(got["dh"] == 0.0) and np.all(got["dw"] == 0.0)
        assert np.all(np.isfinite(got["lse"]))


def test_empty_batch():
    w = torch.zeros(512, 64, dtype=torch.bfloat16, device="cuda")
    h = torch.zeros(0, 64, dtype=torch.bfloat16, device="cuda")
    y = torch.zeros(0, dtype=torch.int64, device="cuda")
    f = flce.forward(h, w, y, check_status=True)
    assert f.loss.item() == 0.0 and f.num_tokens.item() == 0
    dh, dw = flce.backward(h, w, y, f.lse, check_status=True)
    assert dh.shape == (0, 64) and torch.all(dw == 0)


def test_single_token_and_ignore_index_inside_vocab():
    inp = G.small_inputs(N=1, H=64, V=300, seed=10, n_ign=0)
    got = run(G.bf16_tensor(inp.hidden_bits), G.bf16_tensor(inp.weight_bits),
              G.labels_tensor(inp.labels), 0.0, "sum")
    compare(got, inp.hidden, inp.weight, inp.labels, 0.0, "sum")
    # an ignore_index that is a real vocab id: rows with that label are ignored
    inp = G.small_inputs(N=257, H=64, V=300, seed=11, n_ign=0)
    y = inp.labels.copy()
    y[::3] = 7
    got = run(G.bf16_tensor(inp.hidden_bits), G.bf16_tensor(inp.weight_bits),
              G.labels_tensor(y), 0.0, "mean", ignore_index=7)
    compare(got, inp.hidden, inp.weight, y, 0.0, "mean", ignore_index=7)


def test_label_out_of_range_is_reported():
    inp = G.small_inputs(N=130, H=64, V=300, seed=12, n_ign=0)
    y = inp.labels.copy()
    y[5] = 300  # == V
    with pytest.raises(flce.FlceError) as e:
        flce.forward(G.bf16_tensor(inp.hidden_bits), G.bf16_tensor(inp.weight_bits),
                     G.labels_tensor(y), check_status=True)
    assert e.value.status == 3
    # the row is left out of the loss and the count, and its lse is 0, on every
    # forward path
    for compact in (1, 0):
        with _native.options(fwd_compact=compact):
            f = flce.forward(G.bf16_tensor(inp.hidden_bits), G.bf16_tensor(inp.weight_bits),
                             G.labels_tensor(y))
            torch.cuda.synchronize()
        assert int(f.num_tokens.item()) == 129 and f.lse[5].item() == 0.0
    # the backward finds the same label on its own (compacted bf16, uncompacted, fp32)
    # and, like the forward, treats its row as ignored: the gradients equal, bit for
    # bit, those of the labels with that row set to ignore_index
    y_ign = y.copy()
    y_ign[5] = IGN
    for dt in ("bf16", "fp32"):
        if dt == "bf16":
            h, W = G.bf16_tensor(inp.hidden_bits), G.bf16_tensor(inp.weight_bits)
        else:
            h, W = G.f32_tensor(inp.hidden_raw), G.f32_tensor(inp.weight_raw)
        lse = flce.forward(h, W, G.labels_tensor(y_ign), reduction="mean", check_status=True).lse
        for compact in ((1, 0) if dt == "bf16" else (1,)):
            with _native.options(bwd_compact=compact):
                ref = flce.backward(h, W, G.labels_tensor(y_ign), lse, reduction="mean",
                                    check_status=True)
                ws = flce.alloc_workspace(130, 64, 300, h.dtype, "cuda")
                got = flce.backward(h, W, G.labels_tensor(y), lse, reduction="mean",
                                    workspace=ws)
                assert flce.status(ws) == 3
                assert torch.equal(got[0], ref[0]) and torch.equal(got[1], ref[1])
    h, W = G.bf16_tensor(inp.hidden_bits), G.bf16_tensor(inp.weight_bits)
    # the status is cleared by the next forward ...
    f = flce.forward(h, W, G.labels_tensor(inp.labels), check_status=True)
    # ... and by the next backward, also on a workspace never used before
    ws = flce.alloc_workspace(130, 64, 300, torch.bfloat16, "cuda")
    ws.fill_(255)
    flce.backward(h, W, G.labels_tensor(inp.labels), f.lse, workspace=ws, check_status=True)


def bf16_round(a: np.ndarray) -> np.ndarray:
    """The oracle's float64 gradient rounded once to bf16 (nearest even), the
    precision autograd returns gradients of bf16 parameters in."""
    return fi.bf16_to_f32(fi.bf16_round(np.asarray(a, dtype=np.float32))).astype(np.float64)


def test_module_autograd_and_num_tokens_contract():
    """bf16 parameters get bf16 gradients (the fp32 gradient rounded once); they
    are compared with the oracle's gradient rounded once to bf16."""
    inp = G.small_inputs(N=256, H=128, V=640, seed=13, n_ign=40, w_std=0.1)
    h = G.bf16_tensor(inp.hidden_bits).requires_grad_(True)
    w = G.bf16_tensor(inp.weight_bits).requires_grad_(True)
    y = G.labels_tensor(inp.labels)
    n = int((inp.labels != IGN).sum())
    for red in ("sum", "mean"):
        mod = flce.FusedLinearCrossEntropy(ignore_index=IGN, logit_softcapping=2.0, reduction=red)
        loss = mod(h.view(2, 128, 128), y.view(2, 128), w)
        assert loss.dtype == torch.float32
        assert int(mod.num_tokens) == (n if red == "sum" else 0)
        h.grad = None
        w.grad = None
        loss.backward()
        assert h.grad.dtype == torch.bfloat16 and w.grad.dtype == torch.bfloat16
        rb = oracle.backward(inp.hidden, inp.weight, inp.labels, IGN, 2.0, red)
        assert G.rel_l2(h.grad.float().cpu().numpy().reshape(256, 128),
                        bf16_round(rb["d_hidden"])) <= G.GRAD_RL2
        assert G.rel_l2(w.grad.float().cpu().numpy(), bf16_round(rb["d_weight"])) <= G.GRAD_RL2


@pytest.mark.parametrize("buffers", [1, 2])
def test_repeated_calls_are_deterministic(buffers):
    """Every sum has a fixed order: repeated calls agree bit for bit, and one or two
    dZ blocks (which only change which launches overlap) give the same bits."""
    inp = G.small_inputs(N=4200, H=128, V=8500, seed=14, n_ign=100)
    args = (G.bf16_tensor(inp.hidden_bits), G.bf16_tensor(inp.weight_bits),
            G.labels_tensor(inp.labels), 0.0, "sum")
    with G.chunks(*SMALL_CHUNKS):
        a = run(*args)
        with _native.options(dz_buffers=buffers):
            b = run(*args)
    assert a["loss"] == b["loss"]
    assert np.array_equal(a["lse"], b["lse"])
    assert np.array_equal(a["dh"], b["dh"]) and np.array_equal(a["dw"], b["dw"])


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_accumulate_flags(dtype):
    inp = G.small_inputs(N=4200, H=136, V=9000, seed=15, n_ign=300, w_std=0.1)
    if dtype == "bf16":
        h, W = G.bf16_tensor(inp.hidden_bits), G.bf16_tensor(inp.weight_bits)
    else:
        inp = G.small_inputs(N=96, H=64, V=700, seed=15, n_ign=10, w_std=0.1)
        h, W = G.f32_tensor(inp.hidden_raw), G.f32_tensor(inp.weight_raw)
    y = G.labels_tensor(inp.labels)
    with G.chunks(*SMALL_CHUNKS):
        f = flce.forward(h, W, y, check_status=True)
        dh1, dw1 = flce.backward(h, W, y, f.lse, grad_scale=0.5, check_status=True)
        dh2, dw2 = dh1.clone(), dw1.clone()
        flce.backward(h, W, y, f.lse, grad_scale=0.5, d_hidden=dh2, d_weight=dw2,
                      accumulate_d_hidden=True, accumulate_d_weight=True, check_status=True)
        torch.cuda.synchronize()
        assert G.rel_l2(dh2.cpu().numpy(), 2 * dh1.cpu().numpy().astype(np.float64)) <= 1e-6
        assert G.rel_l2(dw2.cpu().numpy(), 2 * dw1.cpu().numpy().astype(np.float64)) <= 1e-6
        # accumulate only dWeight: dHidden is overwritten
        dh3, dw3 = dh1.clone(), dw1.clone()
        flce.backward(h, W, y, f.lse, grad_scale=0.5, d_hidden=dh3, d_weight=dw3,
                      accumulate_d_weight=True, check_status=True)
        assert torch.equal(dh3, dh1)


def test_microbatch_accumulation_matches_full_batch():
    inp = G.small_inputs(N=4400, H=128, V=9000, seed=16, n_ign=400, w_std=0.1)
    h, W, y = (G.bf16_tensor(inp.hidden_bits), G.bf16_tensor(inp.weight_bits),
               G.labels_tensor(inp.labels))
    n = int((inp.labels != IGN).sum())
    with G.chunks(*SMALL_CHUNKS):
        f = flce.forward(h, W, y)
        dh_full, dw_full = flce.backward(h, W, y, f.lse, grad_scale=1.0 / n)
        dw_acc = torch.empty_like(dw_full)
        dh_acc = torch.empty_like(dh_full)
        for k, sl in enumerate([slice(0, 1500), slice(1500, 4400)]):
            fk = flce.forward(h[sl], W, y[sl], check_status=True)
            flce.backward(h[sl], W, y[sl], fk.lse, grad_scale=1.0 / n, d_hidden=dh_acc[sl],
                          d_weight=dw_acc, accumulate_d_weight=(k > 0), check_status=True)
        torch.cuda.synchronize()
    assert G.rel_l2(dw_acc.cpu().numpy(), dw_full.cpu().numpy().astype(np.float64)) <= 1e-5
    assert G.rel_l2(dh_acc.cpu().numpy(), dh_full.cpu().numpy().astype(np.float64)) <= 1e-6


def _label_term_case(case):
    if case == "tiny":
        inp = fi.make_inputs("tiny")
        return inp, inp.workload.softcap, inp.workload.reduction, 1.0
    if case == "softcap_chunks":
        return (G.small_inputs(N=4500, H=136, V=9000, seed=8, n_ign=450, w_std=0.1), 3.0, "sum",
                1.0 / 4050)
    if case == "zipf_runs":  # the most frequent label has 853 rows: runs cross many segments
        w = fi.custom_workload(5000, 256, 1000, seed=21, w_std=0.1, ignore_count=300,
                               labels="zipf1.1")
        return fi.make_inputs(w), 0.0, "mean", 1.0
    inp = G.small_inputs(N=700, H=128, V=512, seed=22, n_ign=50, w_std=0.1)  # one label
    inp.labels[inp.labels != IGN] = 77
    return inp, 2.0, "sum", 1.0


@pytest.mark.parametrize("case", ["tiny", "softcap_chunks", "zipf_runs", "one_label"])
def test_label_term_is_exact(case):
    """dZ reaches the gradient GEMMs in bf16, but the label entry (p - 1)*t', the largest of
    each row, is carried exactly: its rounding residual is added back in fp32 to dHidden
    (a W-row gather) and to dWeight (a sum over each label's rows in a fixed order).  What
    is left is the rounding of the small softmax entries, an order of magnitude below the
    ~1e-3 a bf16 label entry costs on these problems (measured without the residual:
    7e-4 to 1.7e-3)."""
    inp, softcap, red, gs = _label_term_case(case)
    args = (G.bf16_tensor(inp.hidden_bits), G.bf16_tensor(inp.weight_bits),
            G.labels_tensor(inp.labels), softcap, red)
    with G.chunks(*SMALL_CHUNKS) if case in ("softcap_chunks", "zipf_runs") else \
            contextlib.nullcontext():
        got = run(*args, grad_scale=gs)
        again = run(*args, grad_scale=gs)  # the per-label sums have a fixed order
    rb = oracle.backward(inp.hidden, inp.weight, inp.labels, IGN, softcap, red, grad_scale=gs)
    assert G.rel_l2(got["dh"], rb["d_hidden"]) <= 4e-4
    assert G.rel_l2(got["dw"], rb["d_weight"]) <= 4e-4
    assert np.array_equal(got["dh"], again["dh"]) and np.array_equal(got["dw"], again["dw"])


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_bf16_gradient_outputs(dtype):
    """bf16 dHidden / dWeight are the fp32 gradients rounded once to nearest even:
    bf16(g) when overwriting, bf16(float(old) + g) when accumulating."""
    inp = G.small_inputs(N=700, H=136 if dtype == "bf16" else 64, V=1300, seed=23, n_ign=90,
                         w_std=0.1)
    if dtype == "bf16":
        h, W = G.bf16_tensor(inp.hidden_bits), G.bf16_tensor(inp.weight_bits)
    else:
        h, W = G.f32_tensor(inp.hidden_raw), G.f32_tensor(inp.weight_raw)
    y = G.labels_tensor(inp.labels)
    with G.chunks(*SMALL_CHUNKS):
        f = flce.forward(h, W, y, softcap=2.0, check_status=True)
        args = dict(softcap=2.0, grad_scale=0.3, check_status=True)
        dh32, dw32 = flce.backward(h, W, y, f.lse, **args)
        dh16, dw16 = flce.backward(h, W, y, f.lse, grad_dtype=torch.bfloat16, **args)
        assert dh16.dtype == torch.bfloat16 and dw16.dtype == torch.bfloat16
        assert torch.equal(dh16, dh32.to(torch.bfloat16))
        assert torch.equal(dw16, dw32.to(torch.bfloat16))
        assert torch.all(dh16[G.labels_tensor(inp.labels) == IGN] == 0)
        g = torch.Generator(device="cuda").manual_seed(5)
        old_h = torch.randn(dh32.shape, device="cuda", generator=g).to(torch.bfloat16)
        old_w = torch.randn(dw32.shape, device="cuda", generator=g).to(torch.bfloat16)
        acc_h, acc_w = old_h.clone(), old_w.clone()
        flce.backward(h, W, y, f.lse, d_hidden=acc_h, d_weight=acc_w, accumulate_d_hidden=True,
                      accumulate_d_weight=True, **args)
        assert torch.equal(acc_h, (old_h.float() + dh32).to(torch.bfloat16))
        assert torch.equal(acc_w, (old_w.float() + dw32).to(torch.bfloat16))
        # mixed: fp32 dHidden accumulated, bf16 dWeight overwritten
        mix_h, mix_w = dh32.clone(), torch.empty_like(dw16)
        flce.backward(h, W, y, f.lse, d_hidden=mix_h, d_weight=mix_w, accumulate_d_hidden=True,
                      **args)
        assert torch.equal(mix_w, dw16)
        assert G.rel_l2(mix_h.cpu().numpy(), 2 * dh32.cpu().numpy().astype(np.float64)) <= 1e-6


@pytest.mark.parametrize("softcap", [0.0, 30.0])
def test_large_logits_stay_finite(softcap):
    """Logits of several hundred in magnitude (W ~ N(0, 3^2), H=256): the softmax is
    nearly one-hot, exp() of the raw logits would overflow fp32, and the online
    max-subtracted logsumexp must still match the oracle."""
    inp = G.small_inputs(N=300, H=256, V=2000, seed=24, n_ign=30, w_std=3.0)
    got = run(G.bf16_tensor(inp.hidden_bits), G.bf16_tensor(inp.weight_bits),
              G.labels_tensor(inp.labels), softcap, "sum")
    assert np.all(np.isfinite(got["lse"])) and np.isfinite(got["loss"])
    assert np.max(np.abs(got["lse"])) > (100.0 if softcap == 0 else 20.0)
    live = inp.labels != IGN
    rf = oracle.forward(inp.hidden, inp.weight, inp.labels, IGN, softcap, "sum")
    rb = oracle.backward(inp.hidden, inp.weight, inp.labels, IGN, softcap, "sum")
    # lse: fp32 accumulation of K = 256 products errs by at most K * 2^-24 times the
    # sum of their magnitudes (the bound of recursive summation), and the
    # softcap only shrinks it
    absdot = np.abs(inp.hidden.astype(np.float64)) @ np.abs(inp.weight.astype(np.float64)).T
    tol = 256 * 2.0 ** -24 * absdot.max(axis=1) + G.LSE_ATOL
    assert np.all(np.abs(got["lse"] - rf["lse"])[live] <= tol[live])
    assert np.all(got["lse"][~live] == 0.0)
    G.check_loss(got["loss"], rf["loss"])
    assert got["ntok"] == rf["num_tokens"]
    assert np.all(got["dh"][inp.labels == IGN] == 0.0)
    assert G.rel_l2(got["dh"], rb["d_hidden"]) <= G.GRAD_RL2
    assert G.rel_l2(got["dw"], rb["d_weight"]) <= G.GRAD_RL2


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("N,H,V", [(37, 8, 2), (37, 8, 7), (300, 16, 1), (129, 24, 257)])
def test_degenerate_shapes(N, H, V, dtype):
    """The smallest hidden size (H = 8), one- and two-word vocabularies, and a
    vocabulary one past a tile: the tensor maps' boxes extend far past the tensors."""
    inp = G.small_inputs(N=N, H=H, V=V, seed=25 + V, n_ign=N // 5, w_std=0.5)
    if dtype == "bf16":
        h, W = G.bf16_tensor(inp.hidden_bits), G.bf16_tensor(inp.weight_bits)
        hid, wt = inp.hidden, inp.weight
    else:
        h, W = G.f32_tensor(inp.hidden_raw), G.f32_tensor(inp.weight_raw)
        hid, wt = inp.hidden_raw, inp.weight_raw
    got = run(h, W, G.labels_tensor(inp.labels), 0.0, "sum")
    if V == 1:
        # every valid row's loss is lse - L_y = 0 and its gradient 0 - 0; fp32 keeps
        # only rounding-level residue of the log2-domain logsumexp
        rf = oracle.forward(hid, wt, inp.labels, IGN, 0.0, "sum")
        assert got["ntok"] == rf["num_tokens"]
        assert abs(got["loss"]) <= 1e-5 * np.sum(np.abs(rf["lse"]))
        G.check_lse(got["lse"], rf["lse"], inp.labels, V)
        assert np.max(np.abs(got["dh"])) <= 1e-5 and np.max(np.abs(got["dw"])) <= 1e-5
    else:
        compare(got, hid, wt, inp.labels, 0.0, "sum")


@pytest.mark.parametrize("switch", ["cta_group=1", "bwd_fuse=0", "bwd_compact=0", "mn3d=0",
                                    "grad_tile_n=256", "dz_tile_n=512", "dz_tile_n=256",
                                    "fwd_tile_n=256",
                                    "fwd_dynamic=0", "dz_buffers=2", "dz_buffers=2,bwd_fuse=0",
                                    "dz_buffers=2,cta_group=1", "fwd_group_m=3,dz_group_m=2,"
                                    "grad_group_m=1", "fwd_compact=0", "fwd_compact=0,cta_group=1"])
def test_alternative_paths(switch):
    """Each schedule option of the library selects another correct path: single-CTA
    128 x 256 tiles, separate dHidden and dWeight launches, no row compaction (and
    so no exact label term), 2-D views for MN-major operands, 256-column gradient
    and forward tiles, either dZ tile width, round-robin forward tiles, two dZ
    blocks (9 chunks here, so a dZ launch waits on the gradient launches two
    chunks back before it overwrites their block), other raster groups, a
    forward over every row instead of the compacted ones."""
    opts = {kv.split("=")[0]: int(kv.split("=")[1]) for kv in switch.split(",")}
    inp = G.small_inputs(N=2100, H=192, V=4500, seed=26, n_ign=300, w_std=0.1)
    with _native.options(**opts), G.chunks(*SMALL_CHUNKS):
        got = run(G.bf16_tensor(inp.hidden_bits), G.bf16_tensor(inp.weight_bits),
                  G.labels_tensor(inp.labels), 2.0, "mean", grad_scale=0.7)
    compare(got, inp.hidden, inp.weight, inp.labels, 2.0, "mean", grad_scale=0.7)


@pytest.mark.parametrize("softcap", [0.0, 3.0])
@pytest.mark.parametrize("width", [256, 512])
@pytest.mark.parametrize("shape", [(300, 200, 1000), (37, 8, 700), (700, 1000, 1300),
                                   (4500, 136, 9000)])
def test_tile_widths(width, shape, softcap):
    """Every tensor-core GEMM with 256- or 512-column tiles on ragged shapes, with and
    without softcap (each epilogue has a separate softcapped body): the second
    256-column bank of a 512-column tile may lie wholly past the vocabulary
    (forward, dZ) or past H (dHidden, dWeight: H = 8, 136, 200, 1000), and the
    multi-chunk case crosses 5 x 5 backward chunks."""
    N, H, V = shape
    inp = G.small_inputs(N=N, H=H, V=V, seed=31 + N, n_ign=N // 7, w_std=0.1)
    chunked = G.chunks(*SMALL_CHUNKS) if N > 4000 else contextlib.nullcontext()
    with _native.options(fwd_tile_n=width, dz_tile_n=width, grad_tile_n=width), chunked:
        got = run(G.bf16_tensor(inp.hidden_bits), G.bf16_tensor(inp.weight_bits),
                  G.labels_tensor(inp.labels), softcap, "sum", grad_scale=0.5)
    compare(got, inp.hidden, inp.weight, inp.labels, softcap, "sum", grad_scale=0.5)


@pytest.mark.parametrize("softcap", [0.05, 1.0])
def test_small_softcap_saturates(softcap):
    """A softcap well below the logits' spread saturates tanh: most capped logits sit at
    +-softcap and their derivative 1 - tanh^2 vanishes; the rest still carry the
    gradient."""
    inp = G.small_inputs(N=300, H=200, V=1000, seed=28, n_ign=30, w_std=0.2)
    got = run(G.bf16_tensor(inp.hidden_bits), G.bf16_tensor(inp.weight_bits),
              G.labels_tensor(inp.labels), softcap, "mean")
    compare(got, inp.hidden, inp.weight, inp.labels, softcap, "mean")


def test_module_num_label_tokens():
    """NeMo AutoModel linear_ce API, forward(num_label_tokens): the global count of
    non-padding target tokens normalises a 'sum' loss (and so its gradient); it is
    not used by 'mean'; a sharded lm_weight's grad_reduce_group is refused."""
    inp = G.small_inputs(N=256, H=128, V=640, seed=29, n_ign=40, w_std=0.1)
    h = G.bf16_tensor(inp.hidden_bits).requires_grad_(True)
    w = G.bf16_tensor(inp.weight_bits).requires_grad_(True)
    y = G.labels_tensor(inp.labels)
    n_global = 1000  # e.g. this micro-batch is one of several
    mod = flce.FusedLinearCrossEntropy(ignore_index=IGN, reduction="sum")
    loss = mod(h.view(2, 128, 128), y.view(2, 128), w, num_label_tokens=n_global)
    loss.backward()
    rf = oracle.forward(inp.hidden, inp.weight, inp.labels, IGN, 0.0, "sum")
    rb = oracle.backward(inp.hidden, inp.weight, inp.labels, IGN, 0.0, "sum",
                         grad_scale=1.0 / n_global)
    G.check_loss(loss.item(), rf["loss"] / n_global)
    assert int(mod.num_tokens) == rf["num_tokens"]
    assert G.rel_l2(h.grad.float().cpu().numpy().reshape(256, 128),
                    bf16_round(rb["d_hidden"])) <= G.GRAD_RL2
    assert G.rel_l2(w.grad.float().cpu().numpy(), bf16_round(rb["d_weight"])) <= G.GRAD_RL2
    # the count reaches the library as an integer: the same normalisation through the
    # C entry points directly, in fp32 gradients, and the clamp max(n, 1) for n = 0
    hd, Wd = h.detach(), w.detach()
    f = flce.forward(hd, Wd, y, num_label_tokens=n_global, check_status=True)
    G.check_loss(f.loss.item(), rf["loss"] / n_global)
    dh, dw = flce.backward(hd, Wd, y, f.lse, num_label_tokens=n_global, check_status=True)
    assert G.rel_l2(dh.cpu().numpy(), rb["d_hidden"]) <= G.GRAD_RL2
    assert G.rel_l2(dw.cpu().numpy(), rb["d_weight"]) <= G.GRAD_RL2
    f0 = flce.forward(hd, Wd, y, num_label_tokens=0, check_status=True)
    G.check_loss(f0.loss.item(), rf["loss"])
    dh0, _ = flce.backward(hd, Wd, y, f.lse, num_label_tokens=0, check_status=True)
    dh1, _ = flce.backward(hd, Wd, y, f.lse, check_status=True)
    assert torch.equal(dh0, dh1)
    # 'mean' ignores it
    mean = flce.FusedLinearCrossEntropy(ignore_index=IGN, reduction="mean")
    a = mean(h, y, w, num_label_tokens=n_global).item()
    b = mean(h, y, w).item()
    assert a == b
    with pytest.raises(NotImplementedError):
        mod(h, y, w, grad_reduce_group=object())


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_optional_gradients(dtype):
    """A NULL output skips its gradient (a frozen LM head needs no dWeight GEMM); the
    other one is bit-identical to a full backward."""
    if dtype == "bf16":
        inp = G.small_inputs(N=2100, H=192, V=4500, seed=30, n_ign=300, w_std=0.1)
        h, W = G.bf16_tensor(inp.hidden_bits), G.bf16_tensor(inp.weight_bits)
    else:
        inp = G.small_inputs(N=200, H=64, V=700, seed=30, n_ign=20, w_std=0.1)
        h, W = G.f32_tensor(inp.hidden_raw), G.f32_tensor(inp.weight_raw)
    y = G.labels_tensor(inp.labels)
    with G.chunks(*SMALL_CHUNKS):
        f = flce.forward(h, W, y, softcap=3.0, check_status=True)
        args = dict(softcap=3.0, grad_scale=0.4, check_status=True)
        dh, dw = flce.backward(h, W, y, f.lse, **args)
        only_dh, none_w = flce.backward(h, W, y, f.lse, compute_d_weight=False, **args)
        none_h, only_dw = flce.backward(h, W, y, f.lse, compute_d_hidden=False, **args)
        torch.cuda.synchronize()
    assert none_w is None and none_h is None
    assert torch.equal(only_dh, dh) and torch.equal(only_dw, dw)
    if dtype == "bf16":  # autograd with a frozen LM head asks for dHidden alone
        with G.chunks(*SMALL_CHUNKS):
            ref_dh, _ = flce.backward(h, W, y, f.lse, softcap=3.0, compute_d_weight=False,
                                      grad_dtype=torch.bfloat16, check_status=True)
            hh = h.clone().requires_grad_(True)
            loss = flce.FusedLinearCrossEntropy(logit_softcapping=3.0)(hh, y, W)
            loss.backward()
        assert W.grad is None
        # the same fp32 gradient (g = 1) rounded once to bf16: bit for bit
        assert torch.equal(hh.grad, ref_dh)


@pytest.mark.parametrize("softcap,ign_frac", [(0.0, 0.3), (4.0, 0.95), (0.0, 1.0)])
def test_forward_compaction_changes_no_bits(softcap, ign_frac):
    """The forward's GEMM over the compacted rows computes each row's logits and
    logsumexp in the same order as over all rows: lse bit-identical, the count
    identical, the loss equal up to the order of its float64 sum; rows outside
    the loss get lse 0 either way."""
    N = 3000
    inp = G.small_inputs(N=N, H=192, V=5000, seed=33, n_ign=int(ign_frac * N), w_std=0.1)
    args = (G.bf16_tensor(inp.hidden_bits), G.bf16_tensor(inp.weight_bits),
            G.labels_tensor(inp.labels), IGN, softcap, "sum")
    out = []
    for compact in (1, 0):
        with _native.options(fwd_compact=compact):
            f = flce.forward(*args, check_status=True)
            torch.cuda.synchronize()
            out.append((f.loss.item(), int(f.num_tokens.item()), f.lse.cpu().numpy()))
    (la, na, sa), (lb, nb, sb) = out
    assert na == nb == int((inp.labels != IGN).sum())
    assert np.array_equal(sa, sb)
    assert abs(la - lb) <= 1e-6 * max(abs(lb), 1e-30)
    assert np.all(sa[inp.labels == IGN] == 0.0)
    rf = oracle.forward(inp.hidden, inp.weight, inp.labels, IGN, softcap, "sum")
    G.check_loss(la, rf["loss"])
    G.check_lse(sa, rf["lse"], inp.labels, 5000)


def test_two_token_chunks_at_the_default_chunk_size():
    """N = 16384 + 300 rows cross the default 16384-token backward chunk: dWeight is
    stored by the first token chunk and read-add-written by the second, with
    512-column gradient tiles and the compacted passes; compared in full."""
    N = 16384 + 300
    inp = G.small_inputs(N=N, H=256, V=3000, seed=34, n_ign=N // 8, w_std=0.1)
    got = run(G.bf16_tensor(inp.hidden_bits), G.bf16_tensor(inp.weight_bits),
              G.labels_tensor(inp.labels), 0.0, "sum", grad_scale=1.0 / N)
    compare(got, inp.hidden, inp.weight, inp.labels, 0.0, "sum", grad_scale=1.0 / N)


@pytest.mark.parametrize("width", [256, 512])
def test_labels_at_tile_edges(width):
    """Labels on both sides of every 256- and 512-column tile edge, the first and the
    last vocabulary column of a ragged V, and an ignore_index inside the vocabulary
    next to them: the label-logit capture and the label entry of dZ at the edges."""
    V = 1283  # 5 x 256 + 3: the last tile holds 3 columns
    edges = [0, 1, 254, 255, 256, 257, 510, 511, 512, 513, 767, 768, 1023, 1024, 1279, 1280,
             V - 2, V - 1]
    N = 4 * len(edges)
    inp = G.small_inputs(N=N, H=136, V=V, seed=36, n_ign=0, w_std=0.3)
    y = np.array(edges * 4, dtype=np.int64)
    y[::9] = 1100  # the ignore_index below: a real vocabulary id
    with _native.options(fwd_tile_n=width, dz_tile_n=width, grad_tile_n=width):
        got = run(G.bf16_tensor(inp.hidden_bits), G.bf16_tensor(inp.weight_bits),
                  G.labels_tensor(y), 2.5, "sum", ignore_index=1100)
    compare(got, inp.hidden, inp.weight, y, 2.5, "sum", ignore_index=1100)


def test_large_hidden_size():
    """H = 8192 (the hidden size of 70B-class models): 128 K-blocks in the forward
    and dZ GEMMs and 16 column tiles of 512 in dHidden and dWeight."""
    inp = G.small_inputs(N=600, H=8192, V=3000, seed=37, n_ign=60, w_std=0.01)
    got = run(G.bf16_tensor(inp.hidden_bits), G.bf16_tensor(inp.weight_bits),
              G.labels_tensor(inp.labels), 0.0, "mean")
    compare(got, inp.hidden, inp.weight, inp.labels, 0.0, "mean")
