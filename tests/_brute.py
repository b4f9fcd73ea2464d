"""Pure-Python brute force of the FLCE loss for tiny problems (no numpy).

Independent of `oracle/`: the loss is evaluated term by term as
-log(exp(L_y) / sum_v exp(L_v)) with `math.exp`/`math.log`, and gradients are
taken by central finite differences of that scalar.  Used only to pin the
oracle on problems with V <= 8, N <= 4, H <= 4.
"""
import math


def _dot(a, b):
    s = 0.0
    for x, y in zip(a, b):
        s += x * y
    return s


def loss(hidden, weight, labels, ignore_index=-100, softcap=0.0, reduction="sum"):
    """(loss, num_tokens) straight from the textbook formula."""
    total = 0.0
    n = 0
    for i, row in enumerate(hidden):
        y = labels[i]
        if y == ignore_index:
            continue
        L = []
        for w in weight:
            z = _dot(row, w)
            L.append(softcap * math.tanh(z / softcap) if softcap > 0 else z)
        denom = 0.0
        for lv in L:
            denom += math.exp(lv)
        total += -math.log(math.exp(L[y]) / denom)
        n += 1
    if reduction == "sum":
        return total, n
    return total / max(n, 1), 0


def finite_diff(hidden, weight, labels, ignore_index=-100, softcap=0.0,
                reduction="sum", eps=1e-6):
    """(dHidden, dWeight) by central differences of `loss` (lists of lists)."""
    def f(h, w):
        return loss(h, w, labels, ignore_index, softcap, reduction)[0]

    h = [list(r) for r in hidden]
    w = [list(r) for r in weight]
    dh = [[0.0] * len(r) for r in h]
    dw = [[0.0] * len(r) for r in w]
    for i in range(len(h)):
        for k in range(len(h[i])):
            old = h[i][k]
            h[i][k] = old + eps
            fp = f(h, w)
            h[i][k] = old - eps
            fm = f(h, w)
            h[i][k] = old
            dh[i][k] = (fp - fm) / (2 * eps)
    for v in range(len(w)):
        for k in range(len(w[v])):
            old = w[v][k]
            w[v][k] = old + eps
            fp = f(h, w)
            w[v][k] = old - eps
            fm = f(h, w)
            w[v][k] = old
            dw[v][k] = (fp - fm) / (2 * eps)
    return dh, dw
