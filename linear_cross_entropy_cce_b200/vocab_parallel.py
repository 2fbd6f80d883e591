"""Vocabulary-parallel cross-entropy: the classifier E split by vocabulary
rows across ranks, one process per GPU.

Each rank holds a contiguous range [v0, v1) of the logical vocabulary (its
part of every segment of the head).  The loss of row i needs only the
correct-token logit and the log-sum-exp over the vocabulary, and the
log-sum-exp composes over disjoint parts by log-add-exp ("Cut Your Losses in
Large-Vocabulary Language Models", first page §Contribution; research-map
entry §Limitations: log-add-exp of partial results).  So:

  forward   cce_fwd_shard on the local shard gives per row the shard's
            log-sum-exp and, where the shard holds the target, the correct
            token logit; one all-gather of these [2, N] values and
            cce_vocab_combine (log-add-exp over shards) give every rank the
            full lse and loss.
  backward  cce_bwd with CCE_VOCAB_SHARD and the full lse gives the shard's
            dE rows (bf16, complete: they depend only on local columns) and
            its share of dH in fp32 (CCE_FP32_DH), which one all-reduce sums
            over ranks before the cast to bf16.

The kernels are those of the single-GPU path plus the combine kernel;
torch.distributed carries the two exchanges.
"""
from typing import List, Optional, Sequence, Tuple

import torch

from . import cce

SegSpec = Tuple[int, int, torch.Tensor]


def shard_ranges(V: int, world: int, align: int = 256) -> List[Tuple[int, int]]:
    """Contiguous ranges of the logical vocabulary [0, V), one per rank, with
    boundaries on multiples of `align` (the last range takes the rest)."""
    if world < 1 or V < 1:
        raise ValueError("need world >= 1 and V >= 1")
    per = -(-V // world)
    per = -(-per // align) * align
    return [(min(V, r * per), min(V, (r + 1) * per)) for r in range(world)]


def shard_segments(segments: Sequence[SegSpec], v0: int, v1: int) -> List[SegSpec]:
    """The parts of a head's segments [(begin, end, E_s)] inside [v0, v1), as
    segments of their own (E rows sliced, no copy)."""
    out = []
    for b, e, E in segments:
        lo, hi = max(int(b), v0), min(int(e), v1)
        if lo < hi:
            out.append((lo, hi, E[lo - int(b):hi - int(b)]))
    return out


def _all_gather(x: torch.Tensor, group) -> torch.Tensor:
    """[R, *x.shape]: every rank's x, gathered into one buffer."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    out = torch.empty((world * x.shape[0],) + tuple(x.shape[1:]), dtype=x.dtype, device=x.device)
    dist.all_gather_into_tensor(out, x.contiguous(), group=group)  # ranks along dim 0
    return out.view((world,) + tuple(x.shape))


def exchange_forward(lse_part: torch.Tensor, zy_part: torch.Tensor, y: torch.Tensor, V: int,
                     head_ranges: Optional[Sequence[Tuple[int, int]]] = None,
                     ignore_index: int = -100, group=None, combine=None):
    """The forward's one exchange: all-gather every rank's [2, N] parts, then
    combine them (cce.vocab_combine; `combine` substitutes another function
    of the same signature, e.g. a host one for CPU process groups).
    head_ranges: the whole head's live [begin, end) ranges (None: [0, V)).
    Returns (loss, lse), the same on every rank."""
    parts = _all_gather(torch.stack([lse_part, zy_part]), group)
    fn = combine if combine is not None else cce.vocab_combine
    return fn(parts, y, V, ignore_index, head_ranges)


def exchange_backward(dH_part: torch.Tensor, group=None) -> torch.Tensor:
    """The backward's one exchange: dH shares summed over ranks (in place)."""
    import torch.distributed as dist
    dist.all_reduce(dH_part, op=dist.ReduceOp.SUM, group=group)
    return dH_part


def shard_forward_parts(H: torch.Tensor, y: torch.Tensor, local: Sequence[SegSpec], V: int,
                        ignore_index: int = -100, want_colmax: bool = False):
    """This rank's (lse part, correct-token logit part[, colmax]).  A rank
    whose range holds no ids (more ranks than 256-aligned ranges) contributes
    -inf to the log-add-exp and a zero logit part, without a launch."""
    if not local:
        n = H.shape[0]
        lse_p = torch.full((n,), float("-inf"), dtype=torch.float32, device=H.device)
        parts = (lse_p, torch.zeros(n, dtype=torch.float32, device=H.device))
        return parts + (torch.empty(0, dtype=torch.float32, device=H.device),) if want_colmax else parts
    out = cce.fwd(H, None, y, ignore_index, segments=list(local), V=V, shard=True,
                  want_colmax=want_colmax)
    parts = (out[1], out[0])
    return parts + (out[2],) if want_colmax else parts


def vp_forward(H: torch.Tensor, y: torch.Tensor, local: Sequence[SegSpec], V: int,
               ignore_index: int = -100, group=None, want_colmax: bool = False,
               head_ranges: Optional[Sequence[Tuple[int, int]]] = None):
    """Forward over this rank's shard plus the exchange; returns (loss, lse)
    for every row (identical on all ranks), and the shard's colmax if asked."""
    parts = shard_forward_parts(H, y, local, V, ignore_index, want_colmax)
    loss, lse = exchange_forward(parts[0], parts[1], y, V, head_ranges, ignore_index, group)
    return (loss, lse, parts[2]) if want_colmax else (loss, lse)


def vp_backward(H: torch.Tensor, y: torch.Tensor, lse: torch.Tensor, dloss: torch.Tensor,
                local: Sequence[SegSpec], V: int, ignore_index: int = -100,
                filter_eps: float = 0.0, vocab_perm: Optional[torch.Tensor] = None,
                colmax: Optional[torch.Tensor] = None, group=None):
    """Backward over this rank's shard with the full lse; returns (dH summed
    over ranks, bf16; this shard's dE per local segment, bf16).  A row with a
    NaN lse (a target no shard holds) gets a NaN dH row and no gradient."""
    bad = torch.isnan(lse) & (y != ignore_index)
    if not local:  # a rank without ids: a zero share of dH, no dE
        dH = torch.zeros(H.shape, dtype=torch.float32, device=H.device)
        exchange_backward(dH, group)
        dH[bad] = float("nan")
        return dH.to(torch.bfloat16), []
    lse_b = torch.where(bad, torch.zeros_like(lse), lse)
    dl = torch.where(bad, torch.zeros_like(dloss), dloss).to(torch.float32).contiguous()
    dH, dEs, _ = cce.bwd(H, None, y, lse_b, dl, ignore_index, segments=list(local), V=V,
                         filter_eps=filter_eps, vocab_perm=vocab_perm, colmax=colmax,
                         fp32_dh=True, shard=True)
    exchange_backward(dH, group)
    dH[bad] = float("nan")
    return dH.to(torch.bfloat16), dEs


class _VocabParallelCE(torch.autograd.Function):
    @staticmethod
    def forward(ctx, H, y, V, ignore_index, filter_eps, group, bounds, head_ranges, *E_local):
        local = [(b, e, t) for (b, e), t in zip(bounds, E_local)]
        loss, lse = vp_forward(H, y, local, V, ignore_index, group, head_ranges=head_ranges)
        ctx.save_for_backward(H, y, lse, *E_local)
        ctx.meta = (V, ignore_index, filter_eps, group, bounds)
        return loss

    @staticmethod
    def backward(ctx, grad_loss):
        H, y, lse, *E_local = ctx.saved_tensors
        V, ignore_index, filter_eps, group, bounds = ctx.meta
        local = [(b, e, t) for (b, e), t in zip(bounds, E_local)]
        dH, dEs = vp_backward(H, y, lse, grad_loss, local, V, ignore_index, filter_eps, group=group)
        return (dH.to(H.dtype), None, None, None, None, None, None, None,
                *[g.to(t.dtype) for g, t in zip(dEs, E_local)])


def vocab_parallel_cross_entropy(H: torch.Tensor, y: torch.Tensor, local: Sequence[SegSpec],
                                 V: int, ignore_index: int = -100, reduction: str = "mean",
                                 filter_eps: float = 2.0 ** -12, group=None,
                                 head_ranges: Optional[Sequence[Tuple[int, int]]] = None
                                 ) -> torch.Tensor:
    """Cross-entropy of H @ E^T against y with E split by vocabulary over the
    ranks of `group`: `local` is this rank's [(begin, end, E_rows)] (see
    shard_segments), `head_ranges` the whole head's live [begin, end) ranges
    (None: one range [0, V)).  Every rank passes the same H and y and gets
    the same loss; dE flows to its own rows only."""
    if y.dtype != torch.int32:
        y = y.to(torch.int32)
    bounds = tuple((int(b), int(e)) for b, e, _ in local)
    head = tuple((int(b), int(e)) for b, e in head_ranges) if head_ranges else None
    per_row = _VocabParallelCE.apply(H, y, V, ignore_index, float(filter_eps), group, bounds, head,
                                     *[t for _, _, t in local])
    if reduction == "none":
        return per_row
    if reduction == "sum":
        return per_row.sum()
    if reduction == "mean":
        return per_row.sum() / (y != ignore_index).sum()
    raise ValueError(f"unknown reduction {reduction!r}")
