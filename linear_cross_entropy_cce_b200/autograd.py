"""torch.autograd drop-in over libcce: the role of the pip package's loss
function ("The loss and the mask ...", part "Cut Your Losses in
Large-Vocabulary Language Models (CCE)": code on PyPI as a drop-in loss).

    loss = linear_cross_entropy(H, E, y)                 # mean over valid rows
    loss.backward()                                      # dH, dE via cce_bwd

The forward runs cce_fwd and keeps lse; the backward turns the upstream
gradient of the reduction into the per-row dloss and runs cce_bwd.  The
reduction over rows (mean / sum) is a single torch reduction of the per-row
losses; every other step runs in libcce's kernels.
"""
from __future__ import annotations

from typing import Optional, Sequence

import torch

from . import cce


class _LinearCrossEntropy(torch.autograd.Function):
    @staticmethod
    def forward(ctx, H, E, y, ignore_index, filter_eps, full_de, vocab_sort, check, segments_meta,
                *seg_E):
        segments = [(b, e, t) for (b, e), t in zip(segments_meta, seg_E)] if segments_meta else None
        V = segments_meta[-1][1] if segments_meta else None
        st = torch.zeros(1, dtype=torch.int32, device=H.device) if check else None
        if vocab_sort:
            loss, lse, colmax = cce.fwd(H, E, y, ignore_index, segments=segments, V=V,
                                        want_colmax=True, status=st)
            perm = cce.vocab_sort(colmax, y, V if segments else E.shape[0], ignore_index,
                                  segments=segments)
        else:
            loss, lse = cce.fwd(H, E, y, ignore_index, segments=segments, V=V, status=st)
            perm = colmax = None
        if check:
            cce.check_status(st, "cce_fwd")
        ctx.save_for_backward(H, E if E is not None else torch.empty(0), y, lse,
                              perm if perm is not None else torch.empty(0),
                              colmax if colmax is not None else torch.empty(0), *seg_E)
        ctx.meta = (ignore_index, filter_eps, full_de, check, segments_meta, E is not None,
                    perm is not None)
        return loss

    @staticmethod
    def backward(ctx, grad_loss):
        H, E, y, lse, perm, colmax, *seg_E = ctx.saved_tensors
        ignore_index, filter_eps, full_de, check, segments_meta, has_E, has_perm = ctx.meta
        segments = [(b, e, t) for (b, e), t in zip(segments_meta, seg_E)] if segments_meta else None
        V = segments_meta[-1][1] if segments_meta else None
        dloss = grad_loss.contiguous().to(torch.float32)
        st = torch.zeros(1, dtype=torch.int32, device=H.device) if check else None
        dH, dE, _ = cce.bwd(H, E if has_E else None, y, lse, dloss, ignore_index, segments=segments,
                            V=V, filter_eps=filter_eps, vocab_perm=perm if has_perm else None,
                            colmax=colmax if has_perm else None, full_de=full_de, status=st)
        if check:
            cce.check_status(st, "cce_bwd")
        dH = dH.to(H.dtype)
        if segments:
            return (dH, None, None, None, None, None, None, None, None,
                    *[g.to(t.dtype) for g, t in zip(dE, seg_E)])
        return (dH, dE.to(E.dtype), None, None, None, None, None, None, None)


def linear_cross_entropy(H: torch.Tensor, E: Optional[torch.Tensor], y: torch.Tensor,
                         ignore_index: int = -100, reduction: str = "mean",
                         filter_eps: float = 2.0 ** -12, full_de: bool = False,
                         vocab_sort: bool = False,
                         segments: Optional[Sequence] = None,
                         check_status: bool = False) -> torch.Tensor:
    """Cross-entropy of the logits H @ E^T (never materialised) against y.

    H [N, D] bf16, E [V, D] bf16 (or `segments` = [(begin, end, E_s), ...] for
    a composite head with dead gaps), y [N] int32 (int64 is converted).
    reduction: "mean" over rows whose target is not ignore_index, "sum", or
    "none" (per-row losses, ignored rows 0).  filter_eps <= 0 disables the
    gradient filter; full_de keeps the classifier gradient unfiltered;
    vocab_sort walks the vocabulary in descending max-logit order in the
    backward and, with the filter on, skips the tiles whose every softmax
    entry the forward's column maxima bound below filter_eps.
    check_status: after each library call, synchronise and raise CCEError if
    a kernel reported a bad target (NaN rows) or a wait that ran out
    (incomplete outputs); off by default because it costs a host sync.
    """
    if y.dtype != torch.int32:
        y = y.to(torch.int32)
    meta = tuple((int(b), int(e)) for b, e, _ in segments) if segments else ()
    seg_E = tuple(t for _, _, t in segments) if segments else ()
    per_row = _LinearCrossEntropy.apply(H, E, y, ignore_index, float(filter_eps), bool(full_de),
                                        bool(vocab_sort), bool(check_status), meta, *seg_E)
    if reduction == "none":
        return per_row
    if reduction == "sum":
        return per_row.sum()
    if reduction == "mean":
        n_valid = (y != ignore_index).sum()
        return per_row.sum() / n_valid
    raise ValueError(f"unknown reduction {reduction!r}")


class _SoftTargetKL(torch.autograd.Function):
    @staticmethod
    def forward(ctx, Hs, Es, Ht, Et, row_mask, filter_eps):
        kl, lse_s, lse_t = cce.kl_fwd(Hs, Es, Ht, Et, row_mask)
        ctx.save_for_backward(Hs, Es, Ht, Et, lse_s, lse_t,
                              row_mask if row_mask is not None else torch.empty(0))
        ctx.meta = (filter_eps, row_mask is not None)
        return kl

    @staticmethod
    def backward(ctx, grad_kl):
        Hs, Es, Ht, Et, lse_s, lse_t, row_mask = ctx.saved_tensors
        filter_eps, has_mask = ctx.meta
        dH, dE = cce.kl_bwd(Hs, Es, Ht, Et, lse_s, lse_t, grad_kl.contiguous().to(torch.float32),
                            row_mask if has_mask else None, filter_eps=filter_eps)
        return dH.to(Hs.dtype), dE.to(Es.dtype), None, None, None, None


def soft_target_kl(Hs: torch.Tensor, Es: torch.Tensor, Ht: torch.Tensor, Et: torch.Tensor,
                   row_mask: Optional[torch.Tensor] = None, reduction: str = "mean",
                   filter_eps: float = 2.0 ** -12) -> torch.Tensor:
    """KL(p_teacher || p_student) per row with p = softmax(H E^T), never
    materialising either softmax.  The teacher (Ht, Et) is a constant target:
    gradients flow to Hs and Es only (pass the same tensor as Es and Et for a
    shared head; only its student use is differentiated).  row_mask [N]
    (nonzero = counted row) is optional; "mean" averages over counted rows.
    filter_eps drops gradient entries where both probabilities are below it."""
    if row_mask is not None and row_mask.dtype != torch.int32:
        row_mask = row_mask.to(torch.int32)
    per_row = _SoftTargetKL.apply(Hs, Es, Ht.detach(), Et.detach(), row_mask, float(filter_eps))
    if reduction == "none":
        return per_row
    if reduction == "sum":
        return per_row.sum()
    if reduction == "mean":
        n = Hs.shape[0] if row_mask is None else int((row_mask != 0).sum())
        return per_row.sum() / n
    raise ValueError(f"unknown reduction {reduction!r}")
