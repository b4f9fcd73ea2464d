"""PyTorch binding of the FLCE C ABI (argument marshalling only).

Every arithmetic step of the fused linear cross-entropy runs in the CUDA
library `_flce.so`; this module only checks tensor arguments, allocates the
outputs and the workspace with torch, and passes raw device pointers and the
current CUDA stream.  There is no CPU or PyTorch fallback.

API (names follow the pages):
  forward(hidden, weight, labels, ignore_index=-100, softcap=0.0, reduction='sum',
          loss_scale=1.0, num_label_tokens=None) -> FlceForward(loss, num_tokens, lse)
  backward(hidden, weight, labels, lse, grad_output=None, grad_scale=1.0,
           num_label_tokens=None, ...)
      -> (d_hidden, d_weight), fp32 or bf16, optionally accumulated into given
         buffers, either one skippable
  options(**values), set_option, get_option: the library's process-wide
      settings (schedule switches and limits; see flce_option in flce.h)
  FusedLinearCrossEntropy(ignore_index=-100, logit_softcapping=0, reduction='sum')
      an nn.Module whose forward(hidden_states, labels, lm_weight,
      num_label_tokens=None, grad_reduce_group=None) returns the loss and
      records `num_tokens` ('sum': non-ignored count, 'mean': 0), as the NeMo
      AutoModel linear_ce API and modelscope/twinkle PR #335 specify.
"""
from __future__ import annotations

import ctypes
from typing import NamedTuple, Optional, Tuple

import torch

from . import _native

_DTYPES = {torch.bfloat16: _native.BF16, torch.float32: _native.FP32}
_REDUCTIONS = {"sum": _native.SUM, "mean": _native.MEAN}


class FlceForward(NamedTuple):
    loss: torch.Tensor        # float32 scalar
    num_tokens: torch.Tensor  # int64 scalar ('sum': n, 'mean': 0)
    lse: torch.Tensor         # float32 [N]


def _lib():
    return _native.load()


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(device: torch.device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _prep(hidden: torch.Tensor, weight: torch.Tensor, labels: torch.Tensor):
    if not (hidden.is_cuda and weight.is_cuda and labels.is_cuda):
        raise ValueError("hidden, weight and labels must be CUDA tensors")
    if hidden.device != weight.device or hidden.device != labels.device:
        raise ValueError("hidden, weight and labels must be on one device")
    if hidden.dtype not in _DTYPES or weight.dtype != hidden.dtype:
        raise TypeError("hidden and weight must both be bfloat16 or both float32")
    if weight.dim() != 2:
        raise ValueError("weight must be [vocab, hidden]")
    H = weight.shape[1]
    if hidden.shape[-1] != H:
        raise ValueError("hidden's last dim must equal weight.shape[1]")
    h2 = hidden.reshape(-1, H).contiguous()
    y = labels.reshape(-1)
    if y.dtype != torch.int64:
        y = y.to(torch.int64)
    y = y.contiguous()
    if y.shape[0] != h2.shape[0]:
        raise ValueError("labels must have one entry per token")
    return h2, weight.contiguous(), y


def workspace_bytes(N: int, H: int, V: int, dtype: torch.dtype = torch.bfloat16,
                    flags: int = 0) -> int:
    """Workspace for forward/backward; `flags` as for backward (bf16 gradient
    outputs need fp32 scratch)."""
    return int(_lib().flce_workspace_bytes_ex(N, H, V, _DTYPES[dtype], int(flags)))


def alloc_workspace(N: int, H: int, V: int, dtype: torch.dtype, device,
                    flags: int = 0) -> torch.Tensor:
    n = workspace_bytes(N, H, V, dtype, flags)
    if n == 0:
        raise ValueError("invalid FLCE sizes or flags")
    return torch.empty(n, dtype=torch.uint8, device=device)


def status(workspace: torch.Tensor) -> int:
    """Synchronise and return the asynchronous status recorded in `workspace`."""
    return int(_lib().flce_get_status(ctypes.c_void_p(workspace.data_ptr()),
                                      ctypes.c_void_p(_stream(workspace.device))))


def _count(num_label_tokens: Optional[int]) -> int:
    """The C ABI's encoding of an optional global label-token count (-1: none)."""
    if num_label_tokens is None:
        return -1
    n = int(num_label_tokens)
    if n < 0:
        raise ValueError("num_label_tokens must be >= 0")
    return n


def forward(hidden: torch.Tensor, weight: torch.Tensor, labels: torch.Tensor,
            ignore_index: int = -100, softcap: float = 0.0, reduction: str = "sum",
            workspace: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
            check_status: bool = False, loss_scale: float = 1.0,
            num_label_tokens: Optional[int] = None) -> FlceForward:
    """loss ('sum' or 'mean', times loss_scale), num_tokens and every row's lse.
    With num_label_tokens, a 'sum' loss is normalised by that global count (the
    library divides by max(num_label_tokens, 1))."""
    h2, w, y = _prep(hidden, weight, labels)
    N, H = h2.shape
    V = w.shape[0]
    dev = h2.device
    if workspace is None:
        workspace = alloc_workspace(N, H, V, h2.dtype, dev)
    loss = torch.empty((), dtype=torch.float32, device=dev)
    ntok = torch.empty((), dtype=torch.int64, device=dev)
    if lse is None:
        lse = torch.empty(N, dtype=torch.float32, device=dev)
    st = _lib().flce_forward_ex2(_ptr(h2), _ptr(w), _ptr(y), N, H, V, int(ignore_index),
                                 float(softcap), _REDUCTIONS[reduction], _DTYPES[h2.dtype],
                                 float(loss_scale), _count(num_label_tokens), _ptr(loss),
                                 _ptr(ntok), _ptr(lse), _ptr(workspace), workspace.numel(),
                                 _stream(dev))
    _native.check(st, "flce_forward")
    if check_status:
        _native.check(status(workspace), "flce_forward (device status)")
    return FlceForward(loss, ntok, lse)


def backward(hidden: torch.Tensor, weight: torch.Tensor, labels: torch.Tensor,
             lse: torch.Tensor, grad_output: Optional[torch.Tensor] = None,
             grad_scale: float = 1.0, num_valid: Optional[torch.Tensor] = None,
             num_label_tokens: Optional[int] = None,
             ignore_index: int = -100, softcap: float = 0.0, reduction: str = "sum",
             workspace: Optional[torch.Tensor] = None,
             d_hidden: Optional[torch.Tensor] = None, d_weight: Optional[torch.Tensor] = None,
             accumulate_d_hidden: bool = False, accumulate_d_weight: bool = False,
             grad_dtype: torch.dtype = torch.float32,
             compute_d_hidden: bool = True, compute_d_weight: bool = True,
             check_status: bool = False) -> Tuple[Optional[torch.Tensor], Optional[torch.Tensor]]:
    """dHidden [N, H] and dWeight [V, H], float32 or bfloat16 (the dtype of a
    given d_hidden / d_weight, else `grad_dtype`).  A bf16 gradient is
    computed in fp32 and rounded once.  With accumulate_* the gradient is
    added into the given d_hidden / d_weight instead of overwriting them (e.g.
    over the micro-batches of one optimizer step).  compute_d_weight=False
    (a frozen LM head) or compute_d_hidden=False skips that gradient's GEMM
    and returns None in its place.  num_label_tokens as for forward: the
    gradient of the normalised 'sum' loss."""
    h2, w, y = _prep(hidden, weight, labels)
    N, H = h2.shape
    V = w.shape[0]
    dev = h2.device
    if grad_dtype not in (torch.float32, torch.bfloat16):
        raise TypeError("grad_dtype must be float32 or bfloat16")
    if not (compute_d_hidden or compute_d_weight):
        raise ValueError("nothing to compute: both gradients are switched off")
    if (accumulate_d_hidden and not compute_d_hidden) or (accumulate_d_weight and
                                                          not compute_d_weight):
        raise ValueError("cannot accumulate a gradient that is not computed")
    for name, t, acc, shape in (("d_hidden", d_hidden, accumulate_d_hidden, (N, H)),
                                ("d_weight", d_weight, accumulate_d_weight, (V, H))):
        if acc and t is None:
            raise ValueError(f"accumulating needs an existing {name}")
        if t is not None and (tuple(t.shape) != shape
                              or t.dtype not in (torch.float32, torch.bfloat16)
                              or not t.is_contiguous() or t.device != dev):
            raise ValueError(f"{name} must be a contiguous float32 or bfloat16 {list(shape)} "
                             f"tensor on {dev}")
    if not compute_d_hidden:
        d_hidden = None
    elif d_hidden is None:
        d_hidden = torch.empty((N, H), dtype=grad_dtype, device=dev)
    if not compute_d_weight:
        d_weight = None
    elif d_weight is None:
        d_weight = torch.empty((V, H), dtype=grad_dtype, device=dev)
    flags = ((_native.ACCUMULATE_DHIDDEN if accumulate_d_hidden else 0)
             | (_native.ACCUMULATE_DWEIGHT if accumulate_d_weight else 0)
             | (_native.DHIDDEN_BF16 if d_hidden is not None
                and d_hidden.dtype == torch.bfloat16 else 0)
             | (_native.DWEIGHT_BF16 if d_weight is not None
                and d_weight.dtype == torch.bfloat16 else 0))
    if workspace is None:
        workspace = alloc_workspace(N, H, V, h2.dtype, dev, flags)
    if grad_output is not None:
        grad_output = grad_output.reshape(()).to(device=dev, dtype=torch.float32).contiguous()
    if num_valid is not None:
        num_valid = num_valid.reshape(()).to(device=dev, dtype=torch.int64).contiguous()
    lse = lse.contiguous()
    st = _lib().flce_backward_ex(_ptr(h2), _ptr(w), _ptr(y), _ptr(lse), N, H, V,
                                 int(ignore_index), float(softcap), _REDUCTIONS[reduction],
                                 _DTYPES[h2.dtype], _ptr(grad_output), float(grad_scale),
                                 _count(num_label_tokens), _ptr(num_valid), _ptr(d_hidden),
                                 _ptr(d_weight), flags, _ptr(workspace), workspace.numel(),
                                 _stream(dev))
    _native.check(st, "flce_backward")
    if check_status:
        _native.check(status(workspace), "flce_backward (device status)")
    return d_hidden, d_weight


class _FlceFunction(torch.autograd.Function):
    @staticmethod
    def forward(ctx, hidden, weight, labels, ignore_index, softcap, reduction, grad_scale,
                loss_scale, num_label_tokens):
        out = forward(hidden, weight, labels, ignore_index, softcap, reduction,
                      loss_scale=loss_scale, num_label_tokens=num_label_tokens)
        ctx.save_for_backward(hidden, weight, labels, out.lse)
        # the returned loss is scaled by loss_scale (and normalised by the count,
        # in the library), so is its gradient
        ctx.cfg = (ignore_index, softcap, reduction, grad_scale * loss_scale, num_label_tokens,
                   hidden.shape)
        ctx.mark_non_differentiable(out.num_tokens)
        return out.loss, out.num_tokens

    @staticmethod
    def backward(ctx, grad_loss, _grad_ntok):
        hidden, weight, labels, lse = ctx.saved_tensors
        ignore_index, softcap, reduction, grad_scale, num_label_tokens, hshape = ctx.cfg
        # gradients in the parameters' own dtype (bf16 rounded once from fp32),
        # and only those autograd asks for (a frozen LM head skips dWeight)
        need_dh, need_dw = ctx.needs_input_grad[0], ctx.needs_input_grad[1]
        if not (need_dh or need_dw):
            return (None,) * 9
        dh = (torch.empty(hshape, dtype=hidden.dtype, device=hidden.device)
              .view(-1, hshape[-1]) if need_dh else None)
        dw = torch.empty(weight.shape, dtype=weight.dtype, device=weight.device) \
            if need_dw else None
        backward(hidden, weight, labels, lse, grad_output=grad_loss, grad_scale=grad_scale,
                 num_label_tokens=num_label_tokens, ignore_index=ignore_index, softcap=softcap,
                 reduction=reduction, d_hidden=dh, d_weight=dw, compute_d_hidden=need_dh,
                 compute_d_weight=need_dw)
        return ((dh.view(hshape) if need_dh else None), dw) + (None,) * 7


def fused_linear_cross_entropy(hidden, weight, labels, ignore_index: int = -100,
                               softcap: float = 0.0, reduction: str = "sum",
                               grad_scale: float = 1.0, loss_scale: float = 1.0,
                               num_label_tokens: Optional[int] = None):
    """Differentiable (loss, num_tokens); gradients flow to hidden and weight.
    The loss is multiplied by loss_scale and, for 'sum' with num_label_tokens,
    normalised by that global count (so is its gradient); grad_scale scales the
    gradient alone (a micro-batch's token weighting)."""
    return _FlceFunction.apply(hidden, weight, labels, ignore_index, softcap, reduction,
                               grad_scale, loss_scale, num_label_tokens)


class FusedLinearCrossEntropy(torch.nn.Module):
    """Loss module with the constructor of the NeMo AutoModel linear_ce API."""

    def __init__(self, ignore_index: int = -100, logit_softcapping: float = 0,
                 reduction: str = "sum"):
        super().__init__()
        if reduction not in _REDUCTIONS:
            raise ValueError("reduction must be 'sum' or 'mean'")
        if logit_softcapping < 0:
            raise ValueError("logit_softcapping must be >= 0")
        self.ignore_index = ignore_index
        self.logit_softcapping = float(logit_softcapping)
        self.reduction = reduction
        self.num_tokens: Optional[torch.Tensor] = None

    def forward(self, hidden_states: torch.Tensor, labels: torch.Tensor,
                lm_weight: torch.Tensor, num_label_tokens: Optional[int] = None,
                grad_reduce_group=None, *, grad_scale: float = 1.0) -> torch.Tensor:
        """Loss of hidden_states [..., H] against labels [...] with lm_weight [V, H].

        num_label_tokens: the global number of non-padding target tokens; the
        library divides a 'sum' loss by max(num_label_tokens, 1) (in its fp64
        loss sum) and its gradient with it.  Ignored for 'mean'.
        grad_reduce_group: only None (one GPU, a regular lm_weight tensor).
        grad_scale: scales the gradient alone (micro-batch token weighting)."""
        if grad_reduce_group is not None:
            raise NotImplementedError("a sharded lm_weight (grad_reduce_group) is not "
                                      "supported: this loss runs on one GPU")
        loss, ntok = fused_linear_cross_entropy(hidden_states, lm_weight, labels,
                                                self.ignore_index, self.logit_softcapping,
                                                self.reduction, grad_scale,
                                                num_label_tokens=num_label_tokens)
        self.num_tokens = ntok
        return loss
