"""Float64 CPU oracle for fused linear cross-entropy.

TEST INFRASTRUCTURE, NOT PRODUCT CODE: only `tests/`, `__graft_entry__.smoke()`
and `bench.py`'s CPU-baseline leg / `--impl reference` arm may import it.  The
CUDA product path never imports, links or executes anything under `oracle/`.

Every function is pinned by `-m "not gpu"` tests against closed forms,
invariants, a pure-Python brute force and torch's CPU cross-entropy; see the
module docstring of `oracle.flce_ref` for the definitions it follows.
"""
from .flce_ref import (  # noqa: F401
    MEAN, SUM, backward, capped_logits, d_hidden_rows, d_hidden_rows_sliced, d_weight_rows,
    dlogits, forward, grad_factor, label_logits, lse_rows, lse_rows_sliced, row_logsumexp,
)
