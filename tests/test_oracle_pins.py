"""Pins of the float64 oracle against things other than itself (CPU only).

Closed forms, invariants, a pure-Python brute force with finite-difference
gradients, torch's CPU cross-entropy, and the values the pages print.  The
mutation test at the end plants plausible mistakes in the oracle and checks
that some pin fails for each.
"""
import json
import math
import os

import numpy as np
import pytest
import scipy.special

import oracle
import oracle.flce_ref as ref
import flce_inputs as fi
from tests import _brute

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "pages_facts.json")
IGN = -100


def small_problem(N=6, H=5, V=7, seed=0, w_std=0.5, n_ign=2):
    g = np.random.default_rng(seed)
    h = g.standard_normal((N, H))
    w = g.standard_normal((V, H)) * w_std
    y = g.integers(0, V, N)
    if n_ign:
        y[g.choice(N, n_ign, replace=False)] = IGN
    return h, w, y


# --------------------------------------------------------------------------
# check functions (also used by the mutation test)
# --------------------------------------------------------------------------

def check_zero_weight_closed_form():
    """W = 0: every logit is 0, loss_i = ln V, dH = 0, dW_v = g*sum_i(1/V - [y_i=v]) h_i."""
    h, _, y = small_problem(N=9, H=4, V=6, seed=3, n_ign=3)
    V = 6
    w = np.zeros((V, 4))
    n = int((y != IGN).sum())
    f = oracle.forward(h, w, y, IGN, 0.0, "sum")
    assert f["num_tokens"] == n
    assert abs(f["loss"] - n * math.log(V)) < 1e-12 * max(1, n)
    assert np.allclose(f["lse"], math.log(V), atol=1e-14, rtol=0)
    b = oracle.backward(h, w, y, IGN, 0.0, "sum", grad_output=1.0, grad_scale=0.7)
    assert np.all(b["d_hidden"] == 0.0)
    expect = np.zeros((V, 4))
    for i in range(h.shape[0]):
        if y[i] == IGN:
            continue
        for v in range(V):
            expect[v] += 0.7 * ((1.0 / V) - (1.0 if v == y[i] else 0.0)) * h[i]
    assert np.allclose(b["d_weight"], expect, atol=1e-14, rtol=1e-12)


def check_brute_force(softcap, reduction):
    h, w, y = small_problem(N=4, H=3, V=8, seed=11 + int(softcap), w_std=0.8, n_ign=1)
    f = oracle.forward(h, w, y, IGN, softcap, reduction)
    bl, bn = _brute.loss(h.tolist(), w.tolist(), y.tolist(), IGN, softcap, reduction)
    assert f["num_tokens"] == bn
    assert abs(f["loss"] - bl) <= 1e-12 * max(1.0, abs(bl))
    b = oracle.backward(h, w, y, IGN, softcap, reduction)
    dh, dw = _brute.finite_diff(h.tolist(), w.tolist(), y.tolist(), IGN, softcap, reduction)
    assert np.allclose(b["d_hidden"], np.array(dh), atol=1e-8, rtol=1e-6)
    assert np.allclose(b["d_weight"], np.array(dw), atol=1e-8, rtol=1e-6)


def check_torch_library(softcap, reduction, N=48, H=16, V=40, seed=5):
    """Same problem through torch's CPU F.linear / F.cross_entropy in float64."""
    import torch
    import torch.nn.functional as F
    h, w, y = small_problem(N=N, H=H, V=V, seed=seed, w_std=0.3, n_ign=N // 4)
    th = torch.tensor(h, requires_grad=True)
    tw = torch.tensor(w, requires_grad=True)
    z = F.linear(th, tw)
    if softcap > 0:
        z = softcap * torch.tanh(z / softcap)
    tl = F.cross_entropy(z, torch.tensor(y), ignore_index=IGN, reduction="sum")
    n = int((y != IGN).sum())
    if reduction == "mean":
        tl = tl / max(n, 1)
    tl.backward()
    f = oracle.forward(h, w, y, IGN, softcap, reduction)
    b = oracle.backward(h, w, y, IGN, softcap, reduction)
    assert abs(f["loss"] - tl.item()) <= 1e-12 * max(1.0, abs(tl.item()))
    assert np.allclose(b["d_hidden"], th.grad.numpy(), atol=1e-13, rtol=1e-10)
    assert np.allclose(b["d_weight"], tw.grad.numpy(), atol=1e-13, rtol=1e-10)


def check_grad_rows_sum_to_zero():
    """Without softcap, sum_v dZ_iv = 0 per row, so sum_v dW_v = 0."""
    h, w, y = small_problem(N=10, H=6, V=9, seed=4)
    z, L = ref.capped_logits(h, w, 0.0)
    lse = ref.row_logsumexp(L)
    G = ref.dlogits(z, L, lse, y, y != IGN, 0.0, 1.3)
    assert np.allclose(G.sum(axis=1), 0.0, atol=1e-14)
    b = oracle.backward(h, w, y, IGN, 0.0, "sum")
    assert np.allclose(b["d_weight"].sum(axis=0), 0.0, atol=1e-12)


def check_mean_is_sum_over_n():
    h, w, y = small_problem(N=12, H=5, V=11, seed=8, n_ign=5)
    s = oracle.forward(h, w, y, IGN, 2.0, "sum")
    m = oracle.forward(h, w, y, IGN, 2.0, "mean")
    n = int((y != IGN).sum())
    assert s["num_tokens"] == n and m["num_tokens"] == 0
    assert abs(m["loss"] - s["loss"] / n) < 1e-14 * abs(s["loss"])
    bs = oracle.backward(h, w, y, IGN, 2.0, "sum")
    bm = oracle.backward(h, w, y, IGN, 2.0, "mean")
    assert np.allclose(bm["d_hidden"] * n, bs["d_hidden"], rtol=1e-13, atol=1e-15)
    assert np.allclose(bm["d_weight"] * n, bs["d_weight"], rtol=1e-13, atol=1e-15)


def check_ignored_rows():
    h, w, y = small_problem(N=12, H=5, V=11, seed=9, n_ign=4)
    b = oracle.backward(h, w, y, IGN, 3.0, "sum")
    assert np.all(b["d_hidden"][y == IGN] == 0.0)
    assert np.all(np.abs(b["d_hidden"][y != IGN]).sum(axis=1) > 0)
    # dropping the ignored rows entirely gives the same loss and dW
    keep = y != IGN
    f_all = oracle.forward(h, w, y, IGN, 3.0, "sum")
    f_keep = oracle.forward(h[keep], w, y[keep], IGN, 3.0, "sum")
    assert abs(f_all["loss"] - f_keep["loss"]) < 1e-12 * abs(f_all["loss"])
    b_keep = oracle.backward(h[keep], w, y[keep], IGN, 3.0, "sum")
    assert np.allclose(b["d_weight"], b_keep["d_weight"], rtol=1e-13, atol=1e-15)


def check_all_ignored():
    h, w, _ = small_problem(N=5, H=4, V=6, seed=2, n_ign=0)
    y = np.full(5, IGN)
    for red in ("sum", "mean"):
        f = oracle.forward(h, w, y, IGN, 0.0, red)
        assert f["loss"] == 0.0 and f["num_tokens"] == 0
        b = oracle.backward(h, w, y, IGN, 0.0, red, grad_scale=1.0)
        assert np.all(b["d_hidden"] == 0.0) and np.all(b["d_weight"] == 0.0)
        assert np.all(np.isfinite(f["lse"]))


def check_softcap_limits():
    h, w, y = small_problem(N=8, H=5, V=9, seed=6)
    plain = oracle.forward(h, w, y, IGN, 0.0, "sum")
    huge = oracle.forward(h, w, y, IGN, 1e30, "sum")
    assert abs(plain["loss"] - huge["loss"]) < 1e-12 * abs(plain["loss"])
    bp = oracle.backward(h, w, y, IGN, 0.0, "sum")
    bh = oracle.backward(h, w, y, IGN, 1e30, "sum")
    assert np.allclose(bp["d_hidden"], bh["d_hidden"], rtol=1e-12, atol=1e-15)
    # small logits: s*tanh(z/s) = z - z^3/(3 s^2) + 2 z^5/(15 s^4) - ...
    s = 5.0
    z, L = ref.capped_logits(h * 0.05, w, s)
    series = z - z ** 3 / (3 * s ** 2) + 2 * z ** 5 / (15 * s ** 4)
    assert np.max(np.abs(L - series)) < 1e-9
    assert np.max(np.abs(L - z)) > 1e-7  # the cap really acts


# --------------------------------------------------------------------------
# tests
# --------------------------------------------------------------------------

def test_zero_weight_closed_form():
    check_zero_weight_closed_form()


@pytest.mark.parametrize("softcap", [0.0, 1.5])
@pytest.mark.parametrize("reduction", ["sum", "mean"])
def test_brute_force_tiny(softcap, reduction):
    check_brute_force(softcap, reduction)


@pytest.mark.parametrize("softcap", [0.0, 4.0])
@pytest.mark.parametrize("reduction", ["sum", "mean"])
def test_torch_cpu_cross_entropy(softcap, reduction):
    check_torch_library(softcap, reduction)


def test_grad_rows_sum_to_zero():
    check_grad_rows_sum_to_zero()


def test_mean_is_sum_over_n():
    check_mean_is_sum_over_n()


def test_ignored_rows_zero_and_removable():
    check_ignored_rows()


def test_all_ignored_gives_zero_not_nan():
    check_all_ignored()


def test_softcap_limits():
    check_softcap_limits()


def test_logsumexp_matches_scipy():
    g = np.random.default_rng(1)
    L = g.standard_normal((7, 300)) * 20
    assert np.allclose(ref.row_logsumexp(L), scipy.special.logsumexp(L, axis=1),
                       rtol=1e-15, atol=1e-13)


def test_rejects_bad_arguments():
    h, w, y = small_problem()
    with pytest.raises(ValueError):
        oracle.forward(h, w, y, IGN, -1.0, "sum")
    with pytest.raises(ValueError):
        oracle.forward(h, w, y, IGN, 0.0, "avg")
    y2 = y.copy()
    y2[0] = w.shape[0]
    with pytest.raises(ValueError):
        oracle.forward(h, w, y2, IGN, 0.0, "sum")


def test_microbatch_token_weighted_scale():
    """Split into micro-batches (one all-ignored) with grad_scale = 1/sum n_k.

    The summed micro-batch losses and gradients equal the unsplit batch with
    the same scale (modelscope/twinkle PR #335, item 2: 'sum' uses scale 1.0
    per micro-batch; the trainer divides by the global token count).
    """
    h, w, y = small_problem(N=16, H=5, V=9, seed=12, n_ign=3)
    y[4:8] = IGN  # micro-batch 1 fully ignored
    n_tot = int((y != IGN).sum())
    gs = 1.0 / n_tot
    full_f = oracle.forward(h, w, y, IGN, 0.0, "sum")
    full_b = oracle.backward(h, w, y, IGN, 0.0, "sum", grad_scale=gs)
    loss = 0.0
    ntok = 0
    dW = np.zeros_like(w)
    dH = np.zeros_like(h)
    for k in range(4):
        sl = slice(4 * k, 4 * k + 4)
        f = oracle.forward(h[sl], w, y[sl], IGN, 0.0, "sum")
        b = oracle.backward(h[sl], w, y[sl], IGN, 0.0, "sum", grad_scale=gs)
        loss += f["loss"]
        ntok += f["num_tokens"]
        dW += b["d_weight"]
        dH[sl] = b["d_hidden"]
        if k == 1:
            assert f["loss"] == 0.0 and f["num_tokens"] == 0
    assert ntok == n_tot
    assert abs(loss - full_f["loss"]) < 1e-12 * full_f["loss"]
    assert np.allclose(dW, full_b["d_weight"], rtol=1e-12, atol=1e-16)
    assert np.allclose(dH, full_b["d_hidden"], rtol=1e-12, atol=1e-16)


def test_row_sampled_forms_match_full():
    h, w, y = small_problem(N=20, H=6, V=13, seed=21, n_ign=5)
    for s in (0.0, 2.5):
        f = oracle.forward(h, w, y, IGN, s, "sum")
        b = oracle.backward(h, w, y, IGN, s, "sum", grad_scale=0.5)
        rows = [0, 3, 7, 19]
        assert np.allclose(oracle.lse_rows(h, w, rows, s), f["lse"][rows], rtol=1e-14)
        assert np.allclose(oracle.label_logits(h, w, y, IGN, s), f["label_logit"], rtol=1e-14)
        assert np.allclose(oracle.d_hidden_rows(h, w, y, rows, 0.5, IGN, s),
                           b["d_hidden"][rows], rtol=1e-12, atol=1e-16)
        vr = [0, 5, 12]
        assert np.allclose(oracle.d_weight_rows(h, w, y, vr, f["lse"], 0.5, IGN, s),
                           b["d_weight"][vr], rtol=1e-12, atol=1e-16)


def test_vocab_sliced_forms_match_brute_force_and_full():
    """The vocabulary-sliced lse and dHidden (for weights too large for host
    memory in float64) against the pure-Python brute force with finite
    differences, and against the unsliced forms, with slices that do not divide V
    and labels in every slice."""
    h, w, y = small_problem(N=4, H=3, V=8, seed=31, w_std=0.8, n_ign=1)
    for s in (0.0, 1.5):
        rows = [0, 1, 2, 3]
        lse = oracle.lse_rows_sliced(h, w, rows, s, vocab_slice=3)
        for i in rows:
            L = [s * math.tanh(float(np.dot(h[i], wv)) / s) if s > 0 else float(np.dot(h[i], wv))
                 for wv in w]
            assert abs(lse[i] - math.log(sum(math.exp(v) for v in L))) < 1e-12
        dh_bf, _ = _brute.finite_diff(h.tolist(), w.tolist(), y.tolist(), IGN, s, "sum")
        got = oracle.d_hidden_rows_sliced(h, w, y, rows, lse, 1.0, IGN, s, vocab_slice=3)
        assert np.allclose(got, np.array(dh_bf), atol=1e-7, rtol=1e-6)
    h, w, y = small_problem(N=30, H=6, V=50, seed=32, n_ign=6)
    for s in (0.0, 2.5):
        rows = [0, 4, 9, 29]
        ref_lse = oracle.lse_rows(h, w, rows, s)
        for k in (1, 7, 50, 64):
            lse = oracle.lse_rows_sliced(h, w, rows, s, vocab_slice=k)
            assert np.allclose(lse, ref_lse, rtol=1e-14, atol=0)
            assert np.allclose(oracle.d_hidden_rows_sliced(h, w, y, rows, lse, 0.3, IGN, s,
                                                           vocab_slice=k),
                               oracle.d_hidden_rows(h, w, y, rows, 0.3, IGN, s),
                               rtol=1e-12, atol=1e-16)


# --------------------------------------------------------------------------
# values printed by the pages
# --------------------------------------------------------------------------

def _facts():
    with open(GOLDEN) as fh:
        return json.load(fh)


def test_pages_mtp_label_example():
    facts = _facts()
    ex = facts["mtp_labels_example"]
    ign = facts["ignore_index_default"]["value"]
    labels = np.array(ex["labels"])
    g = np.random.default_rng(0)
    h = g.standard_normal((4, 3))
    w = g.standard_normal((5, 3))
    f = oracle.forward(h, w, labels, ign, 0.0, "sum")
    assert f["num_tokens"] == ex["valid_main_targets"]
    # the roll then the causal shift (position t predicts t+1) leaves only ignored targets
    rolled = np.array(ex["after_first_roll"])
    shifted = rolled[1:]
    f2 = oracle.forward(h[:-1], w, shifted, ign, 0.0, "mean")
    assert int((shifted != ign).sum()) == ex["valid_after_causal_shift"]
    assert f2["loss"] == facts["empty_target_loss"]["value"]
    b2 = oracle.backward(h[:-1], w, shifted, ign, 0.0, "mean")
    assert np.all(b2["d_hidden"] == 0.0) and np.all(b2["d_weight"] == 0.0)


def test_pages_logits_memory_matches_workload_shape():
    facts = _facts()["fp32_logits_bytes"]
    w = fi.WORKLOADS["v131k_zipf"]
    b, s, v = facts["shape"]
    assert (w.N, w.V) == (b * s, v)
    assert w.N * w.V * 4 == facts["bytes"] == 8 * 2 ** 30


def test_pages_bf16_grid_at_36():
    facts = _facts()["bf16_grid_at_loss_36"]
    bits = fi.bf16_round(np.array([facts["value"]], dtype=np.float32))
    here = fi.bf16_to_f32(bits)[0]
    nxt = fi.bf16_to_f32(bits + np.uint16(1))[0]
    assert here == facts["value"]
    assert nxt - here == facts["spacing"]
    # a value one third of the way to the next grid point rounds back to 36
    assert fi.bf16_to_f32(fi.bf16_round(np.array([36.08], np.float32)))[0] == 36.0


def test_bf16_round_ties_to_even():
    # 1 + 2^-8 lies exactly between bf16 neighbours 1 and 1+2^-7: ties to even (1.0)
    x = np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -(1.0 + 2.0 ** -8)], dtype=np.float32)
    got = fi.bf16_to_f32(fi.bf16_round(x))
    assert got.tolist() == [1.0, 1.0 + 2.0 ** -6, -1.0]


# --------------------------------------------------------------------------
# planted mistakes: each mutant of the oracle must fail at least one pin
# --------------------------------------------------------------------------

_ALL_CHECKS = [
    check_zero_weight_closed_form,
    lambda: check_brute_force(0.0, "sum"),
    lambda: check_brute_force(1.5, "mean"),
    lambda: check_torch_library(4.0, "sum"),
    lambda: check_torch_library(0.0, "mean"),
    check_grad_rows_sum_to_zero,
    check_mean_is_sum_over_n,
    check_ignored_rows,
    check_all_ignored,
    check_softcap_limits,
]


def _mutant_no_softcap_derivative(z, L, lse, y, valid, s, g):
    return _orig_dlogits(z, L, lse, y, valid, 0.0, g)


def _mutant_wrong_sign(z, L, lse, y, valid, s, g):
    G = np.exp(L - lse[:, None])
    idx = np.nonzero(valid)[0]
    G[idx, y[idx]] += 1.0
    if s > 0:
        G *= 1.0 - np.tanh(z / s) ** 2
    G[~valid] = 0.0
    return G * g


def _mutant_ignored_not_zeroed(z, L, lse, y, valid, s, g):
    G = np.exp(L - lse[:, None])
    idx = np.nonzero(valid)[0]
    G[idx, y[idx]] -= 1.0
    if s > 0:
        G *= 1.0 - np.tanh(z / s) ** 2
    return G * g


def _mutant_cap_without_scale(h, w, s):
    z = np.asarray(h, np.float64) @ np.asarray(w, np.float64).T
    return (z, np.tanh(z / s)) if s > 0 else (z, z)


def _mutant_lse_no_log(L):
    m = L.max(axis=1)
    return m + np.exp(L - m[:, None]).sum(axis=1) - 1.0


def _mutant_grad_factor_no_mean(n, reduction, go=1.0, gs=1.0):
    return float(go) * float(gs)


_orig_dlogits = ref.dlogits

MUTANTS = {
    "softcap derivative dropped": ("dlogits", _mutant_no_softcap_derivative),
    "onehot sign flipped": ("dlogits", _mutant_wrong_sign),
    "ignored rows keep gradient": ("dlogits", _mutant_ignored_not_zeroed),
    "softcap missing outer scale": ("capped_logits", _mutant_cap_without_scale),
    "logsumexp without log": ("row_logsumexp", _mutant_lse_no_log),
    "mean gradient not divided by n": ("grad_factor", _mutant_grad_factor_no_mean),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name, monkeypatch):
    attr, fn = MUTANTS[name]
    monkeypatch.setattr(ref, attr, fn)
    caught = 0
    for chk in _ALL_CHECKS:
        try:
            chk()
        except AssertionError:
            caught += 1
    assert caught > 0, f"no pin detects the planted mistake: {name}"
