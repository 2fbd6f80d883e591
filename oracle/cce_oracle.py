"""Plain, slow, fp64 CPU oracle for the Cut Cross-Entropy hot path.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call or
execute this module: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.  It shares
no code with the CUDA library (``linear_cross_entropy_cce_b200``) and imports
nothing from it.

Sources (web pages, cited by title and section):
  [LM]  "The loss and the mask: Cut Cross-Entropy + FlexAttention (2 papers)",
        part "Cut Your Losses in Large-Vocabulary Language Models (CCE)":
        §Contribution, §What transfers to us.
  [MAP] "Cut Your Losses in Large-Vocabulary Language Models" (research-map
        entry): §Approach, §Key results, §Limitations.
  [DE]  "The Defensive Edit: Chunking Cross-Entropy Loss After an OOM Wake-Up
        Call": §The OOM: A 12.2 GB Softmax Wall (the soft KL between a
        student and a teacher softmax, computed in position chunks),
        §The Trade-Off Analysis / §Assumptions (Assumption 2).

What it computes.  The cross-entropy of row i is the log-sum-exp of its logits
minus its correct-token logit, the logits being plain dot products
z_ij = <h_i, e_j> ([LM] §Contribution).  The oracle materialises the logits in
row slices (the position-chunked CE of [DE]), which the method itself never
does; that is the point of an oracle.  The backward is the exact gradient of
sum_i dloss_i * loss_i; with gradient filtering on, softmax entries below the
threshold are dropped element by element ([LM] §Contribution; [MAP] §Approach).
A composite head is a list of segments on the logical vocabulary; ids that no
segment covers form the dead gap whose logits are -inf ([LM] §What transfers
to us, third bullet).

Readings where the pages are silent:
  * no bias, temperature or soft-capping on the logits;
  * ignored rows (y == ignore_index) have loss = lse = 0 and zero gradient;
  * a target outside [0, V) or inside the gap yields NaN loss/lse for its row;
  * the filter drops p_ij < filter_eps (strict), decided on the softmax p
    itself, never on the target's one-hot term; filter_eps <= 0 means off.

Inputs are bf16 bit patterns (uint16 arrays), widened exactly to fp64; fp64
arrays are accepted as they are (the finite-difference pin needs them).
Every function below is pinned by the ``-m "not gpu"`` tests in
``tests/test_oracle_pins.py``; none is "parity unpinned".
"""
from __future__ import annotations

import math
from typing import Iterable, List, Sequence, Tuple

import numpy as np

SLICE_ROWS = 512  # rows per materialised slice ([DE]: chunk the positions)


def widen_bf16(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> float64, exactly (bf16 is the top half of fp32)."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def as_f64(x: np.ndarray) -> np.ndarray:
    """fp64 arrays pass through (finite-difference tests); bf16 bits widen."""
    x = np.asarray(x)
    return x if x.dtype == np.float64 else widen_bf16(x)


def _segments_f64(segments) -> List[Tuple[int, int, np.ndarray]]:
    out = []
    for begin, end, E in segments:
        E64 = as_f64(E)
        assert E64.shape[0] == end - begin
        out.append((int(begin), int(end), E64))
    return out


def logits_rows(H64: np.ndarray, segs64, V: int) -> np.ndarray:
    """Logical logit rows z[r, j] = <h_r, e_j>; ids in no segment are -inf.

    [LM] §Contribution (dot-product logits); [LM] §What transfers to us (a
    dead gap contributes -inf).  Written out on the logical vocabulary on
    purpose: the segment composition by log-add-exp is *not* reused here.
    """
    Z = np.full((H64.shape[0], V), -np.inf)
    for begin, end, E64 in segs64:
        Z[:, begin:end] = H64 @ E64.T
    return Z


def logsumexp_rows(Z: np.ndarray) -> np.ndarray:
    """lse_r = m_r + log sum_j exp(z_rj - m_r), m_r the row max (textbook)."""
    m = Z.max(axis=1)
    return m + np.log(np.exp(Z - m[:, None]).sum(axis=1))


def _valid_targets(y: np.ndarray, V: int, ignore_index: int, segs64):
    live = np.zeros(V, dtype=bool)
    for begin, end, _ in segs64:
        live[begin:end] = True
    y = np.asarray(y, dtype=np.int64)
    ignored = y == ignore_index
    in_range = (y >= 0) & (y < V)
    good = np.zeros_like(ignored)
    good[in_range] = live[y[in_range]]
    good &= ~ignored
    bad = ~ignored & ~good
    return ignored, good, bad


def forward(H, segments, y, V: int, ignore_index: int = -100,
            rows: Iterable[int] | None = None,
            slice_rows: int = SLICE_ROWS) -> Tuple[np.ndarray, np.ndarray]:
    """Per-row loss and lse in fp64 for ``rows`` (default: all rows).

    segments: sequence of (vocab_begin, vocab_end, E_bits[end-begin, D]).
    loss_i = lse_i - z_{i, y_i}  ([LM] §Contribution).
    Returns arrays indexed like ``rows``.
    """
    segs64 = _segments_f64(segments)
    y = np.asarray(y, dtype=np.int64)
    rows = np.arange(y.shape[0]) if rows is None else np.asarray(list(rows), dtype=np.int64)
    ignored, good, bad = _valid_targets(y[rows], V, ignore_index, segs64)
    loss = np.zeros(rows.shape[0])
    lse = np.zeros(rows.shape[0])
    for s in range(0, rows.shape[0], slice_rows):
        r = rows[s:s + slice_rows]
        Z = logits_rows(as_f64(H[r]), segs64, V)
        l = logsumexp_rows(Z)
        g = good[s:s + slice_rows]
        zy = np.zeros(r.shape[0])
        zy[g] = Z[np.nonzero(g)[0], y[r][g]]
        loss[s:s + slice_rows] = np.where(g, l - zy, 0.0)
        lse[s:s + slice_rows] = np.where(g, l, 0.0)
    loss[bad] = np.nan
    lse[bad] = np.nan
    return loss, lse


def dlogits(Z: np.ndarray, lse: np.ndarray, y_rows: np.ndarray,
            dloss_rows: np.ndarray, filter_eps: float = 0.0) -> np.ndarray:
    """G = dloss_i * (softmax_ij * keep_ij - [j == y_i]) on a logit slice.

    keep_ij = softmax_ij >= filter_eps when filter_eps > 0 (softmax entries
    below the threshold carry no gradient: [LM] §Contribution, [MAP]
    §Approach); the one-hot term is never filtered.  Rows with y < 0 are
    treated as having no target (callers zero their dloss).
    """
    P = np.exp(Z - lse[:, None])
    if filter_eps > 0.0:
        P = np.where(P >= filter_eps, P, 0.0)
    G = P
    has_t = y_rows >= 0
    G[np.nonzero(has_t)[0], y_rows[has_t]] -= 1.0
    return dloss_rows[:, None] * G


def backward(H, segments, y, V: int, dloss, ignore_index: int = -100,
             filter_eps: float = 0.0, slice_rows: int = SLICE_ROWS, filter_dE: bool = True):
    """Exact gradients of sum_i dloss_i * loss_i w.r.t. H and each E segment.

    Returns (dH[N, D] fp64, [dE_s[n_s, D] fp64 per segment]).  Ignored rows
    get a zero dH row and contribute nothing to dE.  [LM] §Contribution,
    [MAP] §Approach (the method recomputes these blockwise; the oracle just
    forms them slice by slice).  filter_dE=False keeps the classifier
    gradient unfiltered while dH is filtered: the "FullC" variant of [MAP]
    §Key results / §Limitations (full classifier gradient).
    """
    segs64 = _segments_f64(segments)
    y = np.asarray(y, dtype=np.int64)
    N, D = H.shape
    dloss = np.asarray(dloss, dtype=np.float64)
    ignored, good, bad = _valid_targets(y, V, ignore_index, segs64)
    dH = np.zeros((N, D))
    dE = [np.zeros_like(E64) for _, _, E64 in segs64]
    for s in range(0, N, slice_rows):
        r = np.arange(s, min(N, s + slice_rows))
        g = good[r]
        if not g.any():
            continue
        r = r[g]
        H64 = as_f64(H[r])
        Z = logits_rows(H64, segs64, V)
        lse = logsumexp_rows(Z)
        G = dlogits(Z, lse, y[r], dloss[r], filter_eps)
        GE = G if filter_dE else dlogits(Z, lse, y[r], dloss[r], 0.0)
        acc = np.zeros((r.shape[0], D))
        for k, (begin, end, E64) in enumerate(segs64):
            acc += G[:, begin:end] @ E64
            dE[k] += GE[:, begin:end].T @ H64
        dH[r] = acc
    dH[bad] = np.nan
    return dH, dE


def softmax_rows(H, segments, V: int, rows) -> np.ndarray:
    """Softmax over the logical vocabulary for the given rows (gap = 0)."""
    segs64 = _segments_f64(segments)
    Z = logits_rows(as_f64(H[np.asarray(rows)]), segs64, V)
    return np.exp(Z - logsumexp_rows(Z)[:, None])


def dE_columns(H, segments, y, V: int, dloss, cols: Sequence[int],
               ignore_index: int = -100, filter_eps: float = 0.0,
               slice_rows: int = SLICE_ROWS) -> np.ndarray:
    """Rows of dE for a few logical vocab ids (needs every row's lse).

    dE_j = sum_i G_ij h_i; the lse of every valid row comes from the oracle's
    own forward over all rows.  Used for sampled checks at full size.
    """
    segs64 = _segments_f64(segments)
    y = np.asarray(y, dtype=np.int64)
    N, D = H.shape
    cols = np.asarray(cols, dtype=np.int64)
    ignored, good, bad = _valid_targets(y, V, ignore_index, segs64)
    out = np.zeros((cols.shape[0], D))
    dloss = np.asarray(dloss, dtype=np.float64)
    for s in range(0, N, slice_rows):
        r = np.arange(s, min(N, s + slice_rows))
        r = r[good[r]]
        if r.shape[0] == 0:
            continue
        H64 = as_f64(H[r])
        Z = logits_rows(H64, segs64, V)
        lse = logsumexp_rows(Z)
        Zc = Z[:, cols]
        P = np.exp(Zc - lse[:, None])
        if filter_eps > 0.0:
            P = np.where(P >= filter_eps, P, 0.0)
        P -= (y[r][:, None] == cols[None, :])
        out += (dloss[r][:, None] * P).T @ H64
    return out


def full_pass(H, segments, y, V: int, dloss, cols: Sequence[int], ignore_index: int = -100,
              filter_eps: Sequence[float] = (0.0,), slice_rows: int = SLICE_ROWS):
    """One pass over every row for the checks at full size: the per-row loss
    and lse of forward() and, for each threshold in ``filter_eps``, the dE
    rows of dE_columns() for the logical ids ``cols``.

    The same slice arithmetic as those two functions (logits, textbook
    log-sum-exp, loss = lse - z_y; G = dloss (p keep - onehot) on the sampled
    columns, dE_j = sum_i G_ij h_i), done once per slice instead of once per
    function, because at full size each pass is the whole N x V x D product.
    Returns (loss[N], lse[N], {eps: dE_cols[len(cols), D]}).
    """
    segs64 = _segments_f64(segments)
    y = np.asarray(y, dtype=np.int64)
    N, D = H.shape
    cols = np.asarray(cols, dtype=np.int64)
    dloss = np.asarray(dloss, dtype=np.float64)
    ignored, good, bad = _valid_targets(y, V, ignore_index, segs64)
    loss = np.zeros(N)
    lse_all = np.zeros(N)
    out = {float(e): np.zeros((cols.shape[0], D)) for e in filter_eps}
    for s in range(0, N, slice_rows):
        r = np.arange(s, min(N, s + slice_rows))
        r = r[good[r]]
        if r.shape[0] == 0:
            continue
        H64 = as_f64(H[r])
        Z = logits_rows(H64, segs64, V)
        lse = logsumexp_rows(Z)
        loss[r] = lse - Z[np.arange(r.shape[0]), y[r]]
        lse_all[r] = lse
        Pc = np.exp(Z[:, cols] - lse[:, None])
        onehot = y[r][:, None] == cols[None, :]
        for e, acc in out.items():
            P = np.where(Pc >= e, Pc, 0.0) if e > 0.0 else Pc.copy()
            P -= onehot
            acc += (dloss[r][:, None] * P).T @ H64
    loss[bad] = np.nan
    lse_all[bad] = np.nan
    return loss, lse_all, out


def mean_loss(loss: np.ndarray, valid: np.ndarray) -> float:
    """Mean over valid rows, exactly rounded (math.fsum); N_v = 0 gives NaN."""
    n_v = int(np.count_nonzero(valid))
    if n_v == 0:
        return float("nan")
    return math.fsum(np.asarray(loss, dtype=np.float64)[valid].tolist()) / n_v


def kahan_reference(parts: Sequence[np.ndarray]) -> np.ndarray:
    """The exactly rounded element-wise sum of several gradient contributions:
    the value a compensated (Kahan) accumulation of the classifier gradient
    over micro-batches approaches ([MAP] §Limitations, Kahan variants).

    Each element is summed with math.fsum (Shewchuk's exact partials), so the
    result does not depend on the order of the parts and is the fp64 number
    nearest to the true sum, even when the parts cancel.
    """
    stack = np.stack([np.asarray(p, dtype=np.float64) for p in parts])
    flat = stack.reshape(stack.shape[0], -1)
    out = np.fromiter((math.fsum(flat[:, k]) for k in range(flat.shape[1])), dtype=np.float64,
                      count=flat.shape[1])
    return out.reshape(stack.shape[1:])


# ---------------------------------------------------------------------------
# Soft-target KL ([DE] §The OOM: the KL divergence between the student and the
# teacher softmax over the whole vocabulary, computed in position chunks).
# Readings where the page is silent:
#   * direction KL(p_t || p_s): the teacher distribution is the target;
#   * temperature 1, no bias; p_s = softmax(H_s E_s^T), p_t = softmax(H_t E_t^T)
#     (E_s and E_t may be the same head);
#   * the teacher is a constant: gradients flow to H_s and E_s only, and
#     d KL_i / d z_s,ij = p_s,ij - p_t,ij;
#   * rows with row_mask == 0 have KL = 0 and no gradient;
#   * the gradient filter drops entry (i, j) when both p_s,ij and p_t,ij are
#     below filter_eps (its gradient is then below filter_eps in magnitude).

def _kl_rows(Hs, Es64, Ht, Et64, r):
    Zs = as_f64(Hs[r]) @ Es64.T
    Zt = as_f64(Ht[r]) @ Et64.T
    ls = logsumexp_rows(Zs)
    lt = logsumexp_rows(Zt)
    return Zs - ls[:, None], Zt - lt[:, None], ls, lt


def kl_forward(Hs, Es, Ht, Et, row_mask=None, slice_rows: int = SLICE_ROWS):
    """Per row (KL(p_t || p_s), lse_s, lse_t), fp64; masked rows give zeros."""
    N = Hs.shape[0]
    mask = np.ones(N, bool) if row_mask is None else np.asarray(row_mask) != 0
    Es64, Et64 = as_f64(Es), as_f64(Et)
    kl, ls_o, lt_o = np.zeros(N), np.zeros(N), np.zeros(N)
    for s in range(0, N, slice_rows):
        r = np.arange(s, min(N, s + slice_rows))
        r = r[mask[r]]
        if r.shape[0] == 0:
            continue
        log_ps, log_pt, ls, lt = _kl_rows(Hs, Es64, Ht, Et64, r)
        kl[r] = np.sum(np.exp(log_pt) * (log_pt - log_ps), axis=1)
        ls_o[r], lt_o[r] = ls, lt
    return kl, ls_o, lt_o


def kl_backward(Hs, Es, Ht, Et, dloss, row_mask=None, filter_eps: float = 0.0,
                slice_rows: int = SLICE_ROWS):
    """Gradients of sum_i dloss_i KL_i w.r.t. H_s and E_s (fp64)."""
    N, D = Hs.shape
    mask = np.ones(N, bool) if row_mask is None else np.asarray(row_mask) != 0
    Es64, Et64 = as_f64(Es), as_f64(Et)
    dloss = np.asarray(dloss, dtype=np.float64)
    dH = np.zeros((N, D))
    dE = np.zeros_like(Es64)
    for s in range(0, N, slice_rows):
        r = np.arange(s, min(N, s + slice_rows))
        r = r[mask[r]]
        if r.shape[0] == 0:
            continue
        log_ps, log_pt, _, _ = _kl_rows(Hs, Es64, Ht, Et64, r)
        Ps, Pt = np.exp(log_ps), np.exp(log_pt)
        G = Ps - Pt
        if filter_eps > 0.0:
            G = np.where((Ps < filter_eps) & (Pt < filter_eps), 0.0, G)
        G *= dloss[r][:, None]
        dH[r] = G @ Es64
        dE += G.T @ as_f64(Hs[r])
    return dH, dE
