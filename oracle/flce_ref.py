"""Float64 CPU oracle for fused linear cross-entropy (FLCE).

TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only `tests/`, `__graft_entry__.smoke()`
and `bench.py` (its CPU-baseline leg and its `--impl reference` arm) may import
this module.  It shares no code with the CUDA path and imports nothing from the
product package.

What it computes is the plain definition the pages give for the fused op, not
an algorithm replica:

* the fused kernel has "the same semantics" as
  `F.cross_entropy(F.linear(hidden, W), labels)` with the optional softcap
  (modelscope/twinkle PR #335, "Experiment results");
* the softcap is `softcap * tanh(logits / softcap)`, 0 meaning off
  (modelscope/twinkle PR #335, "PR information" item 3; NeMo AutoModel
  `FusedLinearCrossEntropy(ignore_index=-100, logit_softcapping=0,
  reduction='sum')`, "API");
* `lm_weight` has shape `[vocab, hidden]` (NeMo AutoModel, `forward`
  parameters);
* rows whose label equals `ignore_index` contribute nothing and are not
  counted (NeMo AutoModel constructor; Modalities PR #464, "Tests" item 3);
* 'sum' returns `num_tokens` = number of non-ignored tokens, 'mean' returns
  `num_tokens = 0` (modelscope/twinkle PR #335, "PR information" item 1);
* an all-ignored batch gives loss 0 and zero gradients, never NaN, via
  `sum / max(count, 1)` (inclusionAI/Ling-3.1-flash discussion #7, "Why use
  num_items_in_batch for MTP?");
* the evaluation is an independent float64 one on the same bf16-quantised
  values (Modalities PR #464, "Measured" and "Tests" item 2).

The gradient is the textbook derivative of that definition:
`dZ = g * (softmax(L) - onehot(y)) * (softcap > 0 ? 1 - tanh(Z/s)^2 : 1)`,
`dH = dZ W`, `dW = dZ^T H`, with `g = grad_output * grad_scale` and an extra
`1 / max(n, 1)` for 'mean'.  The pages fix the loss and say the gradient into
the LM head must follow it (Modalities PR #464, "Measured"); they print no
gradient formula, so this is the plain calculus of the definition above.

Rows are processed in chunks of tokens only so that a `[chunk, V]` logits
block, never the full `[N, V]`, exists at a time; rows are independent, so the
chunking does not change the arithmetic of any row.
"""
from __future__ import annotations

from typing import Dict, Optional, Sequence

import numpy as np

SUM = "sum"
MEAN = "mean"


def _f64(a: np.ndarray) -> np.ndarray:
    return np.asarray(a, dtype=np.float64)


def _check(hidden: np.ndarray, weight: np.ndarray, labels: np.ndarray,
           ignore_index: int, softcap: float, reduction: str) -> None:
    if hidden.ndim != 2 or weight.ndim != 2 or hidden.shape[1] != weight.shape[1]:
        raise ValueError("hidden must be [N, H] and weight [V, H]")
    if labels.shape != (hidden.shape[0],):
        raise ValueError("labels must be [N]")
    if reduction not in (SUM, MEAN):
        raise ValueError(f"reduction must be 'sum' or 'mean', got {reduction!r}")
    if softcap < 0:
        raise ValueError("softcap must be >= 0 (0 = off)")
    V = weight.shape[0]
    bad = (labels != ignore_index) & ((labels < 0) | (labels >= V))
    if np.any(bad):
        raise ValueError("label outside [0, V) that is not ignore_index")


def capped_logits(h_rows: np.ndarray, weight: np.ndarray, softcap: float):
    """Z = h W^T and L = softcap*tanh(Z/softcap) (L = Z when softcap == 0)."""
    z = _f64(h_rows) @ _f64(weight).T
    if softcap > 0:
        return z, softcap * np.tanh(z / softcap)
    return z, z


def row_logsumexp(L: np.ndarray) -> np.ndarray:
    """lse_i = m_i + log(sum_v exp(L_iv - m_i)), m_i = max_v L_iv."""
    m = L.max(axis=1)
    return m + np.log(np.exp(L - m[:, None]).sum(axis=1))


def forward(hidden: np.ndarray, weight: np.ndarray, labels: np.ndarray,
            ignore_index: int = -100, softcap: float = 0.0, reduction: str = SUM,
            chunk: int = 512) -> Dict[str, object]:
    """Loss, num_tokens and the per-row logsumexp of the FLCE definition.

    Returns a dict with
      loss        float  ('sum': sum of per-token losses; 'mean': sum / max(n,1))
      num_tokens  int    ('sum': n = #non-ignored; 'mean': 0)
      num_valid   int    n, whatever the reduction
      lse         [N] float64 logsumexp of every row (ignored rows included)
      label_logit [N] float64 L[i, y_i] (0 for ignored rows)
      row_loss    [N] float64 lse_i - L[i, y_i] (0 for ignored rows)
    """
    labels = np.asarray(labels, dtype=np.int64)
    _check(hidden, weight, labels, ignore_index, softcap, reduction)
    N = hidden.shape[0]
    valid = labels != ignore_index
    lse = np.zeros(N, dtype=np.float64)
    label_logit = np.zeros(N, dtype=np.float64)
    W = _f64(weight)
    for r0 in range(0, N, chunk):
        r1 = min(N, r0 + chunk)
        _, L = capped_logits(hidden[r0:r1], W, softcap)
        lse[r0:r1] = row_logsumexp(L)
        v = valid[r0:r1]
        idx = np.nonzero(v)[0]
        label_logit[r0 + idx] = L[idx, labels[r0:r1][idx]]
    row_loss = np.where(valid, lse - label_logit, 0.0)
    n = int(valid.sum())
    total = float(row_loss.sum())
    if reduction == SUM:
        loss, num_tokens = total, n
    else:
        loss, num_tokens = total / max(n, 1), 0
    return dict(loss=loss, num_tokens=num_tokens, num_valid=n, lse=lse,
                label_logit=label_logit, row_loss=row_loss)


def grad_factor(num_valid: int, reduction: str, grad_output: float = 1.0,
                grad_scale: float = 1.0) -> float:
    """g = grad_output * grad_scale, times 1/max(n,1) for 'mean'."""
    g = float(grad_output) * float(grad_scale)
    if reduction == MEAN:
        g /= max(int(num_valid), 1)
    return g


def dlogits(z: np.ndarray, L: np.ndarray, lse_rows: np.ndarray, y_rows: np.ndarray,
            valid_rows: np.ndarray, softcap: float, g: float) -> np.ndarray:
    """dLoss/dZ for a block of rows: g*(softmax - onehot)*softcap', 0 on ignored rows."""
    G = np.exp(L - lse_rows[:, None])
    idx = np.nonzero(valid_rows)[0]
    G[idx, y_rows[idx]] -= 1.0
    if softcap > 0:
        G *= 1.0 - np.tanh(z / softcap) ** 2
    G[~valid_rows] = 0.0
    G *= g
    return G


def backward(hidden: np.ndarray, weight: np.ndarray, labels: np.ndarray,
             ignore_index: int = -100, softcap: float = 0.0, reduction: str = SUM,
             grad_output: float = 1.0, grad_scale: float = 1.0,
             chunk: int = 512) -> Dict[str, np.ndarray]:
    """dHidden [N,H] and dWeight [V,H] (float64) of the loss returned by `forward`."""
    labels = np.asarray(labels, dtype=np.int64)
    _check(hidden, weight, labels, ignore_index, softcap, reduction)
    N, H = hidden.shape
    V = weight.shape[0]
    valid = labels != ignore_index
    g = grad_factor(int(valid.sum()), reduction, grad_output, grad_scale)
    W = _f64(weight)
    dH = np.zeros((N, H), dtype=np.float64)
    dW = np.zeros((V, H), dtype=np.float64)
    for r0 in range(0, N, chunk):
        r1 = min(N, r0 + chunk)
        h = _f64(hidden[r0:r1])
        z, L = capped_logits(h, W, softcap)
        lse = row_logsumexp(L)
        G = dlogits(z, L, lse, labels[r0:r1], valid[r0:r1], softcap, g)
        dH[r0:r1] = G @ W
        dW += G.T @ h
    return dict(d_hidden=dH, d_weight=dW, g=g, num_valid=int(valid.sum()))


# ---------------------------------------------------------------------------
# Row-sampled forms for problems too large to evaluate in full on the host.
# Each is the same definition restricted to the requested outputs.
# ---------------------------------------------------------------------------

def label_logits(hidden: np.ndarray, weight: np.ndarray, labels: np.ndarray,
                 ignore_index: int = -100, softcap: float = 0.0) -> np.ndarray:
    """L[i, y_i] for every row (0 on ignored rows), one dot product per row."""
    labels = np.asarray(labels, dtype=np.int64)
    valid = labels != ignore_index
    out = np.zeros(hidden.shape[0], dtype=np.float64)
    idx = np.nonzero(valid)[0]
    z = np.einsum("ij,ij->i", _f64(hidden[idx]), _f64(weight[labels[idx]]))
    out[idx] = softcap * np.tanh(z / softcap) if softcap > 0 else z
    return out


def lse_rows(hidden: np.ndarray, weight: np.ndarray, rows: Sequence[int],
             softcap: float = 0.0, chunk: int = 256) -> np.ndarray:
    """logsumexp of the selected rows only."""
    rows = np.asarray(rows, dtype=np.int64)
    out = np.empty(len(rows), dtype=np.float64)
    W = _f64(weight)
    for a in range(0, len(rows), chunk):
        b = min(len(rows), a + chunk)
        _, L = capped_logits(hidden[rows[a:b]], W, softcap)
        out[a:b] = row_logsumexp(L)
    return out


def d_hidden_rows(hidden: np.ndarray, weight: np.ndarray, labels: np.ndarray,
                  rows: Sequence[int], g: float, ignore_index: int = -100,
                  softcap: float = 0.0, chunk: int = 256) -> np.ndarray:
    """dHidden restricted to the selected token rows."""
    rows = np.asarray(rows, dtype=np.int64)
    labels = np.asarray(labels, dtype=np.int64)
    W = _f64(weight)
    out = np.empty((len(rows), hidden.shape[1]), dtype=np.float64)
    for a in range(0, len(rows), chunk):
        b = min(len(rows), a + chunk)
        r = rows[a:b]
        z, L = capped_logits(hidden[r], W, softcap)
        lse = row_logsumexp(L)
        y = labels[r]
        G = dlogits(z, L, lse, y, y != ignore_index, softcap, g)
        out[a:b] = G @ W
    return out


def d_weight_rows(hidden: np.ndarray, weight: np.ndarray, labels: np.ndarray,
                  vocab_rows: Sequence[int], lse_all: np.ndarray, g: float,
                  ignore_index: int = -100, softcap: float = 0.0) -> np.ndarray:
    """dWeight restricted to the selected vocab rows.

    `lse_all` is the oracle's own logsumexp of every token row (from `forward`
    or `lse_rows`); the column v of dZ needs it for every token.
    """
    vr = np.asarray(vocab_rows, dtype=np.int64)
    labels = np.asarray(labels, dtype=np.int64)
    h = _f64(hidden)
    z = h @ _f64(weight[vr]).T  # [N, len(vr)]
    L = softcap * np.tanh(z / softcap) if softcap > 0 else z
    G = np.exp(L - np.asarray(lse_all, dtype=np.float64)[:, None])
    G -= (labels[:, None] == vr[None, :])
    if softcap > 0:
        G *= 1.0 - np.tanh(z / softcap) ** 2
    G[labels == ignore_index] = 0.0
    G *= g
    return G.T @ h


# ---------------------------------------------------------------------------
# The same definitions with the sums over the vocabulary split into slices, for
# a weight too large to hold on the host in float64 at once.  A logsumexp over
# disjoint column sets combines as lse = log(sum_k exp(lse_k)), and dHidden is a
# sum over vocabulary rows, so slicing changes only the order of the float64
# additions.
# ---------------------------------------------------------------------------

def lse_rows_sliced(hidden: np.ndarray, weight: np.ndarray, rows: Sequence[int],
                    softcap: float = 0.0, vocab_slice: int = 65536) -> np.ndarray:
    """logsumexp of the selected rows, taken over vocabulary slices and combined."""
    V = weight.shape[0]
    parts = [lse_rows(hidden, weight[a:a + vocab_slice], rows, softcap)
             for a in range(0, V, vocab_slice)]
    return np.logaddexp.reduce(np.stack(parts), axis=0)


def d_hidden_rows_sliced(hidden: np.ndarray, weight: np.ndarray, labels: np.ndarray,
                         rows: Sequence[int], lse: np.ndarray, g: float,
                         ignore_index: int = -100, softcap: float = 0.0,
                         vocab_slice: int = 65536) -> np.ndarray:
    """dHidden of the selected rows from their logsumexp `lse` (one value per
    selected row), summed over vocabulary slices."""
    rows = np.asarray(rows, dtype=np.int64)
    labels = np.asarray(labels, dtype=np.int64)
    y = labels[rows]
    valid = y != ignore_index
    lse = np.asarray(lse, dtype=np.float64)
    h = _f64(hidden[rows])
    V = weight.shape[0]
    out = np.zeros((len(rows), hidden.shape[1]), dtype=np.float64)
    for a in range(0, V, vocab_slice):
        Wsl = _f64(weight[a:a + vocab_slice])
        z, L = capped_logits(h, Wsl, softcap)
        G = np.exp(L - lse[:, None])
        here = np.nonzero(valid & (y >= a) & (y < a + Wsl.shape[0]))[0]
        G[here, y[here] - a] -= 1.0
        if softcap > 0:
            G *= 1.0 - np.tanh(z / softcap) ** 2
        G[~valid] = 0.0
        out += G @ Wsl
    return g * out
