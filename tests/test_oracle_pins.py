"""Pins for the fp64 oracle: each test ties it to something other than itself.

Closed forms, invariants, a library routine (torch fp64 on the CPU), brute
force on tiny inputs and central finite differences.  A dropped term, a wrong
sign or index, or a transposed operand anywhere in the oracle fails at least
one of them (see the "catches" note on each test).
"""
import math

import numpy as np
import pytest
import torch

import oracle
from linear_cross_entropy_cce_b200 import synthetic as syn

IGN = -100


def _small(N=37, D=24, V=53, std=2.0, seed=1, ignore=0.2, segments=None):
    wl = syn.Workload("t", N=N, D=D, V=V, logit_std=std, ignore_frac=ignore,
                      segments=tuple(segments) if segments else (),
                      segment_mix=(0.6, 0.4) if segments else ())
    return syn.make_inputs(wl, seed=seed)


# ---------------------------------------------------------------- closed forms
@pytest.mark.parametrize("V", [7, 4096, 256000])
def test_zero_E_gives_lnV_exactly(V):
    """E = 0: every logit is 0, sum exp = V exactly, loss = lse = ln V bitwise.
    Catches: a missing/extra term in the lse, a wrong max shift."""
    N, D = 5, 8
    H = syn.fp32_to_bf16_bits(np.random.default_rng(0).standard_normal((N, D)).astype(np.float32))
    E = np.zeros((V, D), dtype=np.uint16)
    y = np.array([0, V - 1, 3 % V, IGN, 1], dtype=np.int32)
    loss, lse = oracle.forward(H, [(0, V, E)], y, V, IGN)
    valid = y != IGN
    assert np.all(loss[valid] == np.log(V)) and np.all(lse[valid] == np.log(V))
    assert loss[~valid] == 0 and lse[~valid] == 0


def test_zero_E_composite_counts_only_live_ids():
    """With a dead gap and E = 0 the loss is ln(V_live): the gap adds nothing
    (its logits are -inf).  Catches: a gap filled with 0 instead of -inf."""
    V, D = 40, 4
    segs = [(0, 17, np.zeros((17, D), np.uint16)), (25, 40, np.zeros((15, D), np.uint16))]
    H = np.zeros((3, D), np.uint16)
    y = np.array([0, 30, 16], np.int32)
    loss, lse = oracle.forward(H, segs, y, V, IGN)
    assert np.all(loss == np.log(32.0))


def test_two_class_is_softplus():
    """V = 2: CE reduces to softplus(z_other - z_target) (textbook logistic loss).
    Catches: sign errors, using the wrong logit as the target."""
    rng = np.random.default_rng(3)
    H = rng.standard_normal((9, 3))
    E = rng.standard_normal((2, 3))
    y = rng.integers(0, 2, 9).astype(np.int32)
    loss, _ = oracle.forward(H, [(0, 2, E)], y, 2, IGN)
    Z = H @ E.T
    d = Z[np.arange(9), 1 - y] - Z[np.arange(9), y]
    assert np.allclose(loss, np.log1p(np.exp(d)), rtol=1e-13, atol=1e-15)


def test_identity_head_matches_library_logsumexp():
    """E = I (D = V): logits are H itself, so lse must equal the library's
    scipy.special.logsumexp of H's rows.  Catches: transposed H/E."""
    from scipy.special import logsumexp
    rng = np.random.default_rng(4)
    V = 11
    H = rng.standard_normal((6, V)) * 5
    E = np.eye(V)
    y = rng.integers(0, V, 6).astype(np.int32)
    loss, lse = oracle.forward(H, [(0, V, E)], y, V, IGN)
    assert np.allclose(lse, logsumexp(H, axis=1), rtol=1e-14, atol=0)
    assert np.allclose(loss, lse - H[np.arange(6), y], rtol=1e-13, atol=1e-14)


# ------------------------------------------------------------------ invariants
def test_shift_invariance():
    """Adding c to every logit (extra column h=1, e=c) leaves the loss unchanged.
    Catches: lse without the max term cancelling, a target logit taken from
    the wrong place."""
    x = _small()
    c = syn.fp32_to_bf16_bits(np.array([3.0], np.float32))[0]
    H2 = np.concatenate([x.H, np.full((x.H.shape[0], 1), syn.fp32_to_bf16_bits(np.array([1.0], np.float32))[0], np.uint16)], 1)
    E = x.segments[0][2]
    E2 = np.concatenate([E, np.full((E.shape[0], 1), c, np.uint16)], 1)
    l1, s1 = oracle.forward(x.H, x.segments, x.y, x.wl.V, IGN)
    l2, s2 = oracle.forward(H2, [(0, x.wl.V, E2)], x.y, x.wl.V, IGN)
    v = x.valid
    assert np.allclose(l1[v], l2[v], rtol=1e-12, atol=1e-12)
    assert np.allclose(s2[v] - s1[v], 3.0, rtol=0, atol=1e-12)


def test_dlogit_rows_sum_to_zero():
    """Unfiltered, sum_j dloss*(p_ij - onehot_ij) = 0 for every row.
    Catches: a missing one-hot term, a softmax that does not normalise."""
    x = _small()
    H64 = oracle.widen_bf16(x.H[x.valid])
    Z = oracle.logits_rows(H64, [(0, x.wl.V, oracle.widen_bf16(x.segments[0][2]))], x.wl.V)
    G = oracle.dlogits(Z, oracle.logsumexp_rows(Z), x.y[x.valid].astype(np.int64),
                       np.ones(H64.shape[0]))
    assert np.max(np.abs(G.sum(1))) <= 1e-12


def test_gradient_pairing_identity():
    """<dH, H>_F = <dE, E>_F: both equal sum_ij G_ij z_ij.
    Catches: a transposed operand in either contraction, a wrong row scatter."""
    x = _small(N=64, D=16, V=40, std=3.0)
    dl = x.dloss_mean()
    dH, dE = oracle.backward(x.H, x.segments, x.y, x.wl.V, dl, IGN)
    a = np.sum(dH * oracle.widen_bf16(x.H))
    b = np.sum(dE[0] * oracle.widen_bf16(x.segments[0][2]))
    assert abs(a - b) <= 1e-12 * max(1.0, abs(a))


def test_softmax_rows_sum_to_one_and_gap_is_zero():
    x = _small(N=8, D=8, V=30, segments=[(0, 10), (14, 30)])
    P = oracle.softmax_rows(x.H, x.segments, 30, np.arange(8))
    assert np.allclose(P.sum(1), 1.0, rtol=0, atol=1e-14)
    assert np.all(P[:, 10:14] == 0.0)


# ----------------------------------------------------------- finite differences
def test_central_finite_differences():
    """dH, dE against central differences of sum_i dloss_i loss_i on N=3, D=5,
    V=7 in fp64.  Catches: any sign/index/scale error in the backward."""
    rng = np.random.default_rng(5)
    N, D, V = 3, 5, 7
    H = rng.standard_normal((N, D))
    E = rng.standard_normal((V, D))
    y = np.array([2, 6, 0], np.int32)
    dl = np.array([0.7, -1.3, 0.25])

    def f(Hx, Ex):
        loss, _ = oracle.forward(Hx, [(0, V, Ex)], y, V, IGN)
        return float(np.dot(dl, loss))

    dH, dE = oracle.backward(H, [(0, V, E)], y, V, dl, IGN)
    h = 1e-6
    for arr, grad in ((H, dH), (E, dE[0])):
        num = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            old = arr[idx]
            arr[idx] = old + h
            fp = f(H, E)
            arr[idx] = old - h
            fm = f(H, E)
            arr[idx] = old
            num[idx] = (fp - fm) / (2 * h)
        rel = np.linalg.norm(num - grad) / np.linalg.norm(grad)
        assert rel <= 1e-7, rel


# ------------------------------------------------------------------ brute force
def _brute(H, E, y, dl, eps=0.0):
    N, D = len(H), len(H[0])
    V = len(E)
    loss, dH, dE = [], [[0.0] * D for _ in range(N)], [[0.0] * D for _ in range(V)]
    for i in range(N):
        z = [sum(H[i][d] * E[j][d] for d in range(D)) for j in range(V)]
        m = max(z)
        lse = m + math.log(sum(math.exp(zj - m) for zj in z))
        loss.append(lse - z[y[i]])
        for j in range(V):
            p = math.exp(z[j] - lse)
            if eps > 0 and p < eps:
                p = 0.0
            g = dl[i] * (p - (1.0 if j == y[i] else 0.0))
            for d in range(D):
                dH[i][d] += g * E[j][d]
                dE[j][d] += g * H[i][d]
    return np.array(loss), np.array(dH), np.array(dE)


@pytest.mark.parametrize("eps", [0.0, 0.05])
def test_brute_force_triple_loop(eps):
    """Pure-Python loops on N=4, D=8, V=16, with and without the filter."""
    rng = np.random.default_rng(6)
    H = oracle.widen_bf16(syn.fp32_to_bf16_bits(rng.standard_normal((4, 8)).astype(np.float32)))
    E = oracle.widen_bf16(syn.fp32_to_bf16_bits(rng.standard_normal((16, 8)).astype(np.float32)))
    y = np.array([3, 0, 15, 7], np.int32)
    dl = np.array([0.25, 0.25, -0.5, 1.0])
    bl, bdH, bdE = _brute(H.tolist(), E.tolist(), y.tolist(), dl.tolist(), eps)
    loss, _ = oracle.forward(H, [(0, 16, E)], y, 16, IGN)
    dH, dE = oracle.backward(H, [(0, 16, E)], y, 16, dl, IGN, filter_eps=eps)
    assert np.allclose(loss, bl, rtol=1e-12, atol=1e-12)
    assert np.allclose(dH, bdH, rtol=1e-12, atol=1e-12)
    assert np.allclose(dE[0], bdE, rtol=1e-12, atol=1e-12)


# ------------------------------------------------------------- library routine
def test_matches_torch_cross_entropy_fp64_on_tiny():
    """Tiny workload vs torch.nn.functional.cross_entropy (CPU, fp64,
    reduction='none', ignore_index=-100) and torch.autograd for dH, dE."""
    x = syn.make_inputs(syn.WORKLOADS["tiny"], seed=0)
    V = x.wl.V
    Ht = torch.tensor(oracle.widen_bf16(x.H), requires_grad=True)
    Et = torch.tensor(oracle.widen_bf16(x.segments[0][2]), requires_grad=True)
    yt = torch.tensor(x.y.astype(np.int64))
    ref = torch.nn.functional.cross_entropy(Ht @ Et.T, yt, reduction="none", ignore_index=IGN)
    dl = x.dloss_mean().astype(np.float64)
    (ref * torch.tensor(dl)).sum().backward()
    loss, lse = oracle.forward(x.H, x.segments, x.y, V, IGN)
    assert np.allclose(loss, ref.detach().numpy(), rtol=1e-12, atol=1e-12)
    lse_t = torch.logsumexp(Ht.detach() @ Et.detach().T, 1).numpy()
    assert np.allclose(lse[x.valid], lse_t[x.valid], rtol=1e-13, atol=1e-13)
    dH, dE = oracle.backward(x.H, x.segments, x.y, V, dl, IGN)
    assert np.allclose(dH, Ht.grad.numpy(), rtol=1e-12, atol=1e-14)
    assert np.allclose(dE[0], Et.grad.numpy(), rtol=1e-12, atol=1e-14)
    # mean over valid rows, exactly rounded, equals torch's 'mean' reduction
    m = torch.nn.functional.cross_entropy(Ht.detach() @ Et.detach().T, yt, ignore_index=IGN).item()
    assert abs(oracle.mean_loss(loss, x.valid) - m) <= 1e-13 * abs(m)


# ------------------------------------------------------------ chunking / segments
def test_row_chunking_does_not_change_results():
    """Position-chunked CE summed equals the unchunked CE (rows are independent)."""
    x = _small(N=70, D=16, V=33)
    a = oracle.forward(x.H, x.segments, x.y, 33, IGN, slice_rows=1)
    b = oracle.forward(x.H, x.segments, x.y, 33, IGN, slice_rows=512)
    c = oracle.forward(x.H, x.segments, x.y, 33, IGN, slice_rows=16)
    for u, v in ((a, b), (b, c)):
        assert np.allclose(u[0], v[0], rtol=1e-14, atol=1e-14)
        assert np.allclose(u[1], v[1], rtol=1e-14, atol=1e-14)
    dl = x.dloss_mean()
    g1 = oracle.backward(x.H, x.segments, x.y, 33, dl, IGN, slice_rows=7)
    g2 = oracle.backward(x.H, x.segments, x.y, 33, dl, IGN, slice_rows=512)
    assert np.allclose(g1[0], g2[0], rtol=1e-13, atol=1e-16)
    assert np.allclose(g1[1][0], g2[1][0], rtol=1e-13, atol=1e-16)


def test_vocab_chunked_logaddexp_equals_full_lse():
    """lse over the whole vocabulary equals log-add-exp of per-chunk lse values."""
    x = _small(N=20, D=16, V=301, std=6.0)
    Z = oracle.logits_rows(oracle.widen_bf16(x.H), [(0, 301, oracle.widen_bf16(x.segments[0][2]))], 301)
    full = oracle.logsumexp_rows(Z)
    parts = [oracle.logsumexp_rows(Z[:, a:a + 64]) for a in range(0, 301, 64)]
    comp = parts[0]
    for p in parts[1:]:
        comp = np.logaddexp(comp, p)
    assert np.allclose(comp, full, rtol=1e-13, atol=0)


def test_segmented_with_gap_equals_compact_head():
    """Segments with a -inf gap == one compact head [E_A; E_B] with targets of
    segment B shifted down by the gap width."""
    segs = [(0, 40), (47, 90)]
    x = _small(N=50, D=12, V=90, std=4.0, segments=segs)
    EA, EB = x.segments[0][2], x.segments[1][2]
    compact = [(0, 83, np.concatenate([EA, EB], 0))]
    y2 = x.y.copy()
    y2[x.y >= 47] -= 7
    l1, s1 = oracle.forward(x.H, x.segments, x.y, 90, IGN)
    l2, s2 = oracle.forward(x.H, compact, y2, 83, IGN)
    assert np.allclose(l1, l2, rtol=1e-13, atol=1e-13)
    assert np.allclose(s1, s2, rtol=1e-13, atol=1e-13)
    dl = x.dloss_mean()
    dH1, dE1 = oracle.backward(x.H, x.segments, x.y, 90, dl, IGN)
    dH2, dE2 = oracle.backward(x.H, compact, y2, 83, dl, IGN)
    assert np.allclose(dH1, dH2, rtol=1e-12, atol=1e-15)
    assert np.allclose(np.concatenate(dE1, 0), dE2[0], rtol=1e-12, atol=1e-15)


# ---------------------------------------------------------------- edge cases
def test_ignored_and_bad_targets():
    V, D = 10, 4
    rng = np.random.default_rng(8)
    H = syn.fp32_to_bf16_bits(rng.standard_normal((5, D)).astype(np.float32))
    segs = [(0, 6, syn.fp32_to_bf16_bits(rng.standard_normal((6, D)).astype(np.float32)))]
    y = np.array([IGN, 10, 7, -3, 2], np.int32)   # ignored, out of range, in gap, negative, ok
    loss, lse = oracle.forward(H, segs, y, V, IGN)
    assert loss[0] == 0 and lse[0] == 0
    assert np.all(np.isnan(loss[1:4])) and np.all(np.isnan(lse[1:4]))
    assert np.isfinite(loss[4])
    dH, dE = oracle.backward(H, segs, y, V, np.ones(5), IGN)
    assert np.all(dH[0] == 0) and np.all(np.isnan(dH[1:4])) and np.all(np.isfinite(dH[4]))
    assert math.isnan(oracle.mean_loss(loss, np.zeros(5, bool)))


def test_filter_drops_exactly_the_small_softmax_entries():
    """With filter_eps, dE of a column whose softmax is below eps in every row
    equals the one-hot part only; a column at/above eps keeps its softmax part."""
    x = _small(N=30, D=16, V=64, std=8.0, ignore=0.0)
    eps = 2.0 ** -12
    P = oracle.softmax_rows(x.H, x.segments, 64, np.arange(30))
    dl = x.dloss_mean().astype(np.float64)
    _, dE = oracle.backward(x.H, x.segments, x.y, 64, dl, IGN, filter_eps=eps)
    H64 = oracle.widen_bf16(x.H)
    for j in range(64):
        keep = P[:, j] >= eps
        expect = ((dl * np.where(keep, P[:, j], 0.0) - dl * (x.y == j))[:, None] * H64).sum(0)
        assert np.allclose(dE[0][j], expect, rtol=1e-12, atol=1e-15)


def test_dE_columns_match_backward():
    x = _small(N=40, D=8, V=50, segments=[(0, 20), (26, 50)])
    dl = x.dloss_mean()
    _, dE = oracle.backward(x.H, x.segments, x.y, 50, dl, IGN, filter_eps=1e-3)
    cols = [0, 19, 26, 49]
    got = oracle.dE_columns(x.H, x.segments, x.y, 50, dl, cols, IGN, filter_eps=1e-3, slice_rows=9)
    ref = np.stack([dE[0][0], dE[0][19], dE[1][0], dE[1][23]])
    assert np.allclose(got, ref, rtol=1e-12, atol=1e-16)


def test_full_pass_equals_forward_and_dE_columns():
    """The one-pass helper of the full-size checks reproduces forward() (bit
    for bit: same slice arithmetic) and dE_columns() for each threshold."""
    x = _small(N=70, D=8, V=50, std=6.0, segments=[(0, 20), (26, 50)])
    dl = x.dloss_mean()
    cols = [0, 7, 19, 26, 31, 49]
    loss, lse, dEc = oracle.full_pass(x.H, x.segments, x.y, 50, dl, cols, IGN,
                                      filter_eps=(0.0, 1e-3), slice_rows=16)
    rl, rs = oracle.forward(x.H, x.segments, x.y, 50, IGN, slice_rows=16)
    assert np.array_equal(loss, rl, equal_nan=True) and np.array_equal(lse, rs, equal_nan=True)
    for e in (0.0, 1e-3):
        ref = oracle.dE_columns(x.H, x.segments, x.y, 50, dl, cols, IGN, filter_eps=e, slice_rows=16)
        assert np.allclose(dEc[e], ref, rtol=1e-12, atol=1e-16)
    assert not np.allclose(dEc[0.0], dEc[1e-3], rtol=1e-6, atol=0)


def test_full_classifier_gradient_variant():
    """filter_dE=False ("FullC"): dE equals the unfiltered dE, dH the filtered
    dH; and the filter does change both on this peaky case (so the variant is
    not vacuous)."""
    x = _small(N=40, D=16, V=200, std=10.0, ignore=0.1)
    dl = x.dloss_mean()
    eps = 2.0 ** -12
    fH, fE = oracle.backward(x.H, x.segments, x.y, 200, dl, IGN, filter_eps=eps)
    uH, uE = oracle.backward(x.H, x.segments, x.y, 200, dl, IGN)
    cH, cE = oracle.backward(x.H, x.segments, x.y, 200, dl, IGN, filter_eps=eps, filter_dE=False)
    assert np.array_equal(cH, fH) and np.array_equal(cE[0], uE[0])
    assert not np.allclose(fE[0], uE[0], rtol=1e-9, atol=0) and not np.allclose(fH, uH, rtol=1e-9, atol=0)


# --------------------------------------------------- exact sum of gradient parts
def test_kahan_reference_survives_cancellation():
    """Parts built to cancel: 1e16 + 1 - 1e16 is exactly 1 (a running fp64 sum
    gives 0 or 2); the order of the parts does not matter.
    Catches: a plain left-to-right fp64 accumulation."""
    a = np.array([1e16, 1.0, 3.0, -2.5])
    parts = [a, np.array([1.0, 1e-30, -1e20, 2.5]), np.array([-1e16, -1.0, 1e20, 0.0])]
    want = np.array([1.0, 1e-30, 3.0, 0.0])
    assert np.array_equal(oracle.kahan_reference(parts), want)
    assert np.array_equal(oracle.kahan_reference(parts[::-1]), want)


def test_kahan_reference_is_the_exactly_rounded_rational_sum():
    """Against exact rational arithmetic (fractions.Fraction): the result is
    the fp64 number nearest to the true sum, bit for bit, on parts spanning 60
    binary orders of magnitude with mixed signs.
    Catches: any order-dependent or compensated-but-inexact summation."""
    from fractions import Fraction
    rng = np.random.default_rng(7)
    K, M = 23, 41
    parts = [rng.standard_normal(M) * np.exp2(rng.integers(-30, 30, M)) for _ in range(K)]
    got = oracle.kahan_reference([p.reshape(1, M) for p in parts]).reshape(M)
    for k in range(M):
        exact = sum((Fraction(float(p[k])) for p in parts), Fraction(0))
        assert got[k] == float(exact)  # Fraction -> float rounds to nearest


def test_kahan_reference_keeps_shape_and_closed_form():
    """n copies of 0.1 sum to the double nearest n/10, and shapes survive."""
    parts = [np.full((3, 4), 0.1) for _ in range(10)]
    got = oracle.kahan_reference(parts)
    assert got.shape == (3, 4) and np.all(got == 1.0)  # fsum: 10 x 0.1 == 1.0 exactly rounded
    assert np.all(oracle.kahan_reference([np.full(5, 0.1)] * 3) == 0.30000000000000004)


# ------------------------------------------------------------- soft-target KL
def _kl_inputs(N=29, D=16, V=61, seed=3, std_s=2.0, std_t=3.0, shared=False):
    rng = np.random.default_rng(seed)
    Hs = rng.standard_normal((N, D))
    Ht = rng.standard_normal((N, D))
    Es = rng.standard_normal((V, D)) * std_s / math.sqrt(D)
    Et = Es if shared else rng.standard_normal((V, D)) * std_t / math.sqrt(D)
    return Hs, Es, Ht, Et


def test_kl_matches_torch_kl_div_fp64():
    """torch.nn.functional.kl_div (log targets) on the materialised logits,
    fp64, is an independent implementation of KL(p_t || p_s)."""
    Hs, Es, Ht, Et = _kl_inputs()
    mask = np.ones(len(Hs), np.int32)
    mask[[2, 11]] = 0
    kl, ls, lt = oracle.kl_forward(Hs, Es, Ht, Et, mask)
    zs = torch.from_numpy(Hs @ Es.T)
    zt = torch.from_numpy(Ht @ Et.T)
    ref = torch.nn.functional.kl_div(torch.log_softmax(zs, -1), torch.log_softmax(zt, -1),
                                     reduction="none", log_target=True).sum(-1).numpy()
    on = mask != 0
    assert np.allclose(kl[on], ref[on], rtol=1e-12, atol=1e-14)
    assert np.all(kl[~on] == 0) and np.all(ls[~on] == 0) and np.all(kl[on] >= 0)
    assert np.allclose(ls[on], torch.logsumexp(zs, -1).numpy()[on], rtol=1e-14)
    assert np.allclose(lt[on], torch.logsumexp(zt, -1).numpy()[on], rtol=1e-14)


def test_kl_two_classes_is_bernoulli_kl():
    """V = 2: KL between Bernoulli(q) and Bernoulli(p) in closed form, with
    p = sigmoid of the logit difference."""
    rng = np.random.default_rng(4)
    Hs, Ht = rng.standard_normal((9, 3)), rng.standard_normal((9, 3))
    Es, Et = rng.standard_normal((2, 3)), rng.standard_normal((2, 3))
    kl, _, _ = oracle.kl_forward(Hs, Es, Ht, Et)
    ps = 1.0 / (1.0 + np.exp(-(Hs @ (Es[0] - Es[1]))))
    pt = 1.0 / (1.0 + np.exp(-(Ht @ (Et[0] - Et[1]))))
    ref = pt * np.log(pt / ps) + (1 - pt) * np.log((1 - pt) / (1 - ps))
    assert np.allclose(kl, ref, rtol=1e-10, atol=1e-15)


def test_kl_of_identical_models_is_zero_with_zero_gradient():
    Hs, Es, _, _ = _kl_inputs(shared=True)
    kl, _, _ = oracle.kl_forward(Hs, Es, Hs, Es)
    dH, dE = oracle.kl_backward(Hs, Es, Hs, Es, np.ones(len(Hs)))
    assert np.all(kl == 0) and np.all(dH == 0) and np.all(dE == 0)


def test_kl_gradient_central_differences_and_torch_autograd():
    """d(sum_i dloss_i KL_i)/dH_s and /dE_s: central differences on a tiny
    case, and torch autograd through kl_div with the teacher detached."""
    Hs, Es, Ht, Et = _kl_inputs(N=3, D=4, V=6, seed=8)
    dl = np.array([0.9, -0.4, 1.7])
    dH, dE = oracle.kl_backward(Hs, Es, Ht, Et, dl)

    def f(Hx, Ex):
        return float(np.dot(dl, oracle.kl_forward(Hx, Ex, Ht, Et)[0]))

    h = 1e-6
    for arr, grad in ((Hs, dH), (Es, dE)):
        num = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            old = arr[idx]
            arr[idx] = old + h
            fp = f(Hs, Es)
            arr[idx] = old - h
            fm = f(Hs, Es)
            arr[idx] = old
            num[idx] = (fp - fm) / (2 * h)
        assert np.linalg.norm(num - grad) / np.linalg.norm(grad) <= 1e-7
    Hs, Es, Ht, Et = _kl_inputs(N=17, D=8, V=40, seed=9)
    dl = np.linspace(-1, 2, 17)
    dH, dE = oracle.kl_backward(Hs, Es, Ht, Et, dl)
    tH = torch.tensor(Hs, requires_grad=True)
    tE = torch.tensor(Es, requires_grad=True)
    zt = torch.from_numpy(Ht @ Et.T)
    kl = torch.nn.functional.kl_div(torch.log_softmax(tH @ tE.T, -1), torch.log_softmax(zt, -1),
                                    reduction="none", log_target=True).sum(-1)
    (kl * torch.from_numpy(dl)).sum().backward()
    assert np.allclose(tH.grad.numpy(), dH, rtol=1e-10, atol=1e-13)
    assert np.allclose(tE.grad.numpy(), dE, rtol=1e-10, atol=1e-13)


def test_kl_filter_drops_only_entries_small_in_both():
    """With the filter, dH_s is G E_s where G keeps p_s - p_t unless both are
    below eps: checked against the explicit rule on materialised softmaxes."""
    Hs, Es, Ht, Et = _kl_inputs(N=21, D=12, V=300, seed=10, std_s=6.0, std_t=6.0)
    eps = 2.0 ** -12
    dl = np.full(21, 0.5)
    dH, dE = oracle.kl_backward(Hs, Es, Ht, Et, dl, filter_eps=eps)
    uH, _ = oracle.kl_backward(Hs, Es, Ht, Et, dl)
    Ps = torch.softmax(torch.from_numpy(Hs @ Es.T), -1).numpy()
    Pt = torch.softmax(torch.from_numpy(Ht @ Et.T), -1).numpy()
    drop = (Ps < eps) & (Pt < eps)
    assert drop.any() and (~drop).any()
    G = np.where(drop, 0.0, Ps - Pt) * 0.5
    assert np.allclose(dH, G @ Es, rtol=1e-10, atol=1e-15)
    assert np.allclose(dE, G.T @ Hs, rtol=1e-10, atol=1e-15)
    assert not np.allclose(dH, uH, rtol=1e-12, atol=0)
