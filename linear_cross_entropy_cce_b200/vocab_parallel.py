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
            token logit; one all-gather of these [3, N] values (with an
            ownership count) and a local log-add-exp give every rank the full
            lse and loss.
  backward  cce_bwd with CCE_VOCAB_SHARD and the full lse gives the shard's
            dE rows (complete: they depend only on local columns) and its
            share of dH, which an all-reduce sums over ranks.

The kernels are those of the single-GPU path; torch.distributed carries the
two exchanges.
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


def combine_shards(parts: torch.Tensor, y: torch.Tensor, ignore_index: int = -100):
    """Per-rank parts [R, 3, N] (lse over the shard, correct-token logit or 0,
    1 where the shard holds the target) -> (loss, lse) [N].

    lse = log-add-exp over ranks; loss = lse - the owner's logit.  Ignored
    rows give 0; a target that no shard holds (outside [0, V) or in a dead
    gap of the head) gives NaN, as on one GPU."""
    lse_p, zy_p, own = parts[:, 0], parts[:, 1], parts[:, 2]
    lse = torch.logsumexp(lse_p, dim=0)
    zy = zy_p.sum(dim=0)
    ignored = y == ignore_index
    bad = (~ignored) & (own.sum(dim=0) == 0)
    zero = torch.zeros_like(lse)
    nan = torch.full_like(lse, float("nan"))
    lse = torch.where(ignored, zero, torch.where(bad, nan, lse))
    loss = torch.where(ignored, zero, torch.where(bad, nan, lse - zy))
    return loss, lse


def owned(y: torch.Tensor, local: Sequence[SegSpec]) -> torch.Tensor:
    """1.0 where this shard's segments hold the target, else 0.0."""
    o = torch.zeros(y.shape, dtype=torch.float32, device=y.device)
    for b, e, _ in local:
        o += ((y >= int(b)) & (y < int(e))).to(torch.float32)
    return o


def _all_gather(x: torch.Tensor, group) -> torch.Tensor:
    import torch.distributed as dist
    world = dist.get_world_size(group)
    bufs = [torch.empty_like(x) for _ in range(world)]
    dist.all_gather(bufs, x.contiguous(), group=group)
    return torch.stack(bufs)


def exchange_forward(lse_part: torch.Tensor, zy_part: torch.Tensor, own: torch.Tensor,
                     y: torch.Tensor, ignore_index: int = -100, group=None):
    """The forward's one exchange: all-gather every rank's [3, N] parts, then
    combine_shards locally.  Returns (loss, lse), the same on every rank."""
    return combine_shards(_all_gather(torch.stack([lse_part, zy_part, own]), group), y,
                          ignore_index)


def exchange_backward(dH_part: torch.Tensor, group=None) -> torch.Tensor:
    """The backward's one exchange: dH shares summed over ranks (in place)."""
    import torch.distributed as dist
    dist.all_reduce(dH_part, op=dist.ReduceOp.SUM, group=group)
    return dH_part


def shard_forward_parts(H: torch.Tensor, y: torch.Tensor, local: Sequence[SegSpec], V: int,
                        ignore_index: int = -100, want_colmax: bool = False):
    """This rank's (lse part, correct-token logit part, ownership[, colmax]).
    A rank whose range holds no ids (more ranks than 256-aligned ranges)
    contributes -inf to the log-add-exp and nothing else, without a launch."""
    if not local:
        n = H.shape[0]
        lse_p = torch.full((n,), float("-inf"), dtype=torch.float32, device=H.device)
        zero = torch.zeros(n, dtype=torch.float32, device=H.device)
        parts = (lse_p, zero, zero.clone())
        return parts + (torch.empty(0, dtype=torch.float32, device=H.device),) if want_colmax else parts
    out = cce.fwd(H, None, y, ignore_index, segments=list(local), V=V, shard=True,
                  want_colmax=want_colmax)
    parts = (out[1], out[0], owned(y, local))
    return parts + (out[2],) if want_colmax else parts


def vp_forward(H: torch.Tensor, y: torch.Tensor, local: Sequence[SegSpec], V: int,
               ignore_index: int = -100, group=None, want_colmax: bool = False):
    """Forward over this rank's shard plus the exchange; returns (loss, lse)
    for every row (identical on all ranks), and the shard's colmax if asked."""
    parts = shard_forward_parts(H, y, local, V, ignore_index, want_colmax)
    loss, lse = exchange_forward(parts[0], parts[1], parts[2], y, ignore_index, group)
    return (loss, lse, parts[3]) if want_colmax else (loss, lse)


def vp_backward(H: torch.Tensor, y: torch.Tensor, lse: torch.Tensor, dloss: torch.Tensor,
                local: Sequence[SegSpec], V: int, ignore_index: int = -100,
                filter_eps: float = 0.0, vocab_perm: Optional[torch.Tensor] = None,
                colmax: Optional[torch.Tensor] = None, group=None):
    """Backward over this rank's shard with the full lse; returns (dH summed
    over ranks, this shard's dE per local segment), bf16."""
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
                         fp32_grads=True, shard=True)
    exchange_backward(dH, group)
    dH[bad] = float("nan")
    return dH.to(torch.bfloat16), [d.to(torch.bfloat16) for d in dEs]


class _VocabParallelCE(torch.autograd.Function):
    @staticmethod
    def forward(ctx, H, y, V, ignore_index, filter_eps, group, bounds, *E_local):
        local = [(b, e, t) for (b, e), t in zip(bounds, E_local)]
        loss, lse = vp_forward(H, y, local, V, ignore_index, group)
        ctx.save_for_backward(H, y, lse, *E_local)
        ctx.meta = (V, ignore_index, filter_eps, group, bounds)
        return loss

    @staticmethod
    def backward(ctx, grad_loss):
        H, y, lse, *E_local = ctx.saved_tensors
        V, ignore_index, filter_eps, group, bounds = ctx.meta
        local = [(b, e, t) for (b, e), t in zip(bounds, E_local)]
        dH, dEs = vp_backward(H, y, lse, grad_loss, local, V, ignore_index, filter_eps, group=group)
        return (dH.to(H.dtype), None, None, None, None, None, None,
                *[g.to(t.dtype) for g, t in zip(dEs, E_local)])


def vocab_parallel_cross_entropy(H: torch.Tensor, y: torch.Tensor, local: Sequence[SegSpec],
                                 V: int, ignore_index: int = -100, reduction: str = "mean",
                                 filter_eps: float = 2.0 ** -12, group=None) -> torch.Tensor:
    """Cross-entropy of H @ E^T against y with E split by vocabulary over the
    ranks of `group`: `local` is this rank's [(begin, end, E_rows)] (see
    shard_segments).  Every rank passes the same H and y and gets the same
    loss; dE flows to its own rows only."""
    if y.dtype != torch.int32:
        y = y.to(torch.int32)
    bounds = tuple((int(b), int(e)) for b, e, _ in local)
    per_row = _VocabParallelCE.apply(H, y, V, ignore_index, float(filter_eps), group, bounds,
                                     *[t for _, _, t in local])
    if reduction == "none":
        return per_row
    if reduction == "sum":
        return per_row.sum()
    if reduction == "mean":
        return per_row.sum() / (y != ignore_index).sum()
    raise ValueError(f"unknown reduction {reduction!r}")
