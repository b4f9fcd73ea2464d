"""Helpers shared by the GPU parity tests (inputs to device, comparisons).

Tolerances come from the contract of this FLCE build:
  num_tokens, ignored-row zeros   bit-exact
  loss                            1e-5 relative
  dHidden, dWeight                2e-3 relative L2
  lse (per row)                   1e-4 absolute: the row's logsumexp is an
                                  fp32 quantity of magnitude <= ~15 here, its
                                  fp32 grid is ~1e-6 and the tensor-core dot
                                  products of K <= 4096 bf16 pairs carry
                                  ~1e-6 of accumulated rounding; 1e-4 leaves a
                                  wide margin while still catching any
                                  dropped tile or wrong column (>= 1e-2).
"""
import numpy as np
import torch

import flce_inputs as fi
from lm_head_linear_tmem_b200 import _native

LOSS_RTOL = 1e-5
GRAD_RL2 = 2e-3
LSE_ATOL = 1e-4


def bf16_tensor(bits: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


def f32_tensor(a: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device)


def labels_tensor(y: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(y, dtype=np.int64)).to(device)


def rel_l2(got: np.ndarray, ref: np.ndarray) -> float:
    den = float(np.linalg.norm(ref))
    num = float(np.linalg.norm(np.asarray(got, np.float64) - ref))
    if den == 0.0:
        return num
    return num / den


def check_lse(got: np.ndarray, ref: np.ndarray, labels: np.ndarray, V: int,
              ignore_index: int = fi.IGNORE_INDEX, atol=LSE_ATOL):
    """Rows in the loss: within `atol` of the oracle's logsumexp.  Rows outside it
    (ignore_index, or a label outside [0, V)): exactly 0, as the library defines
    (their logits are not computed)."""
    labels = np.asarray(labels)
    live = (labels != ignore_index) & (labels >= 0) & (labels < V)
    assert np.all(np.asarray(got)[~live] == 0.0), "rows outside the loss must get lse 0"
    if live.any():
        err = np.abs(np.asarray(got, np.float64)[live] - np.asarray(ref)[live])
        assert np.all(err <= atol), float(np.max(err - atol))


def check_loss(got: float, ref: float):
    if ref == 0.0:
        assert got == 0.0, got
    else:
        assert abs(got - ref) <= LOSS_RTOL * abs(ref), (got, ref, abs(got - ref) / abs(ref))


def small_inputs(N, H, V, seed, n_ign, w_std=0.05):
    """Seeded ad-hoc problem with the workload recipe (bf16-quantised)."""
    w = fi.custom_workload(N, H, V, seed=seed, w_std=w_std, ignore_count=n_ign)
    return fi.make_inputs(w, keep_raw=True)


def chunks(tokens: int, vocab: int):
    """Run the backward with tokens x vocab chunks instead of the default
    16384 x 16384, so that small problems span several chunks along both
    reduced dimensions (library options FLCE_OPT_CHUNK_TOKENS / _VOCAB)."""
    return _native.options(chunk_tokens=tokens, chunk_vocab=vocab)
