"""Soft-target KL (cce_kl_fwd / cce_kl_bwd) against the fp64 oracle."""
import math

import numpy as np
import pytest
import torch

import oracle
from linear_cross_entropy_cce_b200 import synthetic as syn
from _helpers import EPS_BF16, TOL_GRAD, TOL_GRAD_FILTER, TOL_ROW, normwise, to_np

pytestmark = pytest.mark.gpu


def _kl_case(N, D, V, std_s, std_t, shared, seed, masked):
    """Student and teacher rows from two seeded synthetic draws of the same
    shapes (H ~ N(0, 1), E scaled to the logit std); optionally one head."""
    xs = syn.make_inputs(syn.Workload("kls", N=N, D=D, V=V, logit_std=std_s, ignore_frac=0.0),
                         seed=seed)
    xt = syn.make_inputs(syn.Workload("klt", N=N, D=D, V=V, logit_std=std_t, ignore_frac=0.0),
                         seed=seed + 100)
    Es = xs.segments[0][2]
    Et = Es if shared else xt.segments[0][2]
    mask = None
    if masked:
        mask = (np.random.default_rng(seed).random(N) > 0.2).astype(np.int32)
    return xs.H, Es, xt.H, Et, mask


def _up(a):
    from linear_cross_entropy_cce_b200 import cce
    return cce.bf16_from_bits(a, "cuda")


CASES = {
    "separate_heads": dict(N=333, D=200, V=5000, std_s=3.0, std_t=4.0, shared=False, seed=1, masked=True),
    "shared_head": dict(N=300, D=256, V=7001, std_s=2.0, std_t=2.0, shared=True, seed=2, masked=False),
    # peaky distributions: after filtering the sparse (CUDA-core) route runs
    "sparse": dict(N=700, D=192, V=30000, std_s=14.0, std_t=14.0, shared=True, seed=3, masked=True),
    # 11 vocabulary tiles in splits of 2: the last split is one tile with 100
    # valid ids, so the forward's second column half has an empty partial
    "half_tail": dict(N=300, D=256, V=2660, std_s=3.0, std_t=3.0, shared=True, seed=5, masked=True),
}


@pytest.mark.parametrize("case", sorted(CASES))
@pytest.mark.parametrize("eps", [0.0, EPS_BF16])
def test_kl_matches_oracle(case, eps):
    from linear_cross_entropy_cce_b200 import cce
    Hs, Es, Ht, Et, mask = _kl_case(**CASES[case])
    tm = torch.from_numpy(mask).cuda() if mask is not None else None
    Hs_d, Es_d, Ht_d = _up(Hs), _up(Es), _up(Ht)
    Et_d = Es_d if CASES[case]["shared"] else _up(Et)
    kl, ls, lt = cce.kl_fwd(Hs_d, Es_d, Ht_d, Et_d, tm)
    N = Hs.shape[0]
    dl = np.linspace(0.2, 1.0, N) / N
    dH, dE = cce.kl_bwd(Hs_d, Es_d, Ht_d, Et_d, ls, lt, torch.from_numpy(dl).float().cuda(), tm,
                        filter_eps=eps)
    torch.cuda.synchronize()
    rk, rls, rlt = oracle.kl_forward(Hs, Es, Ht, Et, mask)
    assert np.max(np.abs(to_np(kl) - rk)) <= TOL_ROW
    assert np.max(np.abs(to_np(ls) - rls)) <= TOL_ROW
    assert np.max(np.abs(to_np(lt) - rlt)) <= TOL_ROW
    rH, rE = oracle.kl_backward(Hs, Es, Ht, Et, dl, mask, filter_eps=eps)
    tol = TOL_GRAD_FILTER if eps > 0 else TOL_GRAD
    assert normwise(to_np(dH), rH) <= tol
    assert normwise(to_np(dE), rE) <= tol
    if mask is not None:
        off = mask == 0
        assert np.all(to_np(kl)[off] == 0) and np.all(to_np(dH)[off] == 0)


def test_kl_of_identical_models_is_exactly_zero():
    """Teacher = student: the two tiles of every pair are the same products,
    so KL, dH and dE come out exactly 0."""
    from linear_cross_entropy_cce_b200 import cce
    Hs, Es, _, _, _ = _kl_case(N=260, D=128, V=3000, std_s=5.0, std_t=5.0, shared=True, seed=4,
                               masked=False)
    H, E = _up(Hs), _up(Es)
    kl, ls, lt = cce.kl_fwd(H, E, H, E)
    dH, dE = cce.kl_bwd(H, E, H, E, ls, lt, torch.full((260,), 0.5, device="cuda"))
    torch.cuda.synchronize()
    assert torch.equal(ls, lt)
    assert torch.all(kl == 0) and torch.all(dH == 0) and torch.all(dE == 0)


def test_soft_target_kl_autograd():
    from linear_cross_entropy_cce_b200.autograd import soft_target_kl
    Hs, Es, Ht, Et, mask = _kl_case(**CASES["separate_heads"])
    Hl = _up(Hs).requires_grad_(True)
    El = _up(Es).requires_grad_(True)
    tm = torch.from_numpy(mask).cuda()
    loss = soft_target_kl(Hl, El, _up(Ht), _up(Et), row_mask=tm, filter_eps=0.0)
    loss.backward()
    torch.cuda.synchronize()
    rk, _, _ = oracle.kl_forward(Hs, Es, Ht, Et, mask)
    n = int((mask != 0).sum())
    ref = math.fsum(rk.tolist()) / n
    assert abs(loss.item() - ref) <= 1e-4 * abs(ref)
    dl = np.where(mask != 0, 1.0 / n, 0.0)
    rH, rE = oracle.kl_backward(Hs, Es, Ht, Et, dl, mask)
    assert normwise(to_np(Hl.grad), rH) <= TOL_GRAD
    assert normwise(to_np(El.grad), rE) <= TOL_GRAD


def test_kl_full_size_sampled_rows_and_pairing_identity():
    """The 24,576 x 248,320 stand-in workload of bench.py --loss kl: KL, both
    lse and dH on sampled rows (each an independent oracle row); dE through
    sum_i <dH_i, H_s,i> = <dE, E_s> (both equal sum_ij G_ij z_s,ij)."""
    from linear_cross_entropy_cce_b200 import cce
    wl = syn.KL_WORKLOADS["soft_kl_24k_248k"]
    Hs, Ht, E = syn.make_kl_inputs(wl, seed=0)
    a, b, e = _up(Hs), _up(Ht), _up(E)
    kl, ls, lt = cce.kl_fwd(a, e, b, e)
    dl = np.full(wl.N, 1.0 / wl.N)
    dH, dE = cce.kl_bwd(a, e, b, e, ls, lt, torch.from_numpy(dl).float().cuda(),
                        filter_eps=EPS_BF16, fp32_grads=True)
    torch.cuda.synchronize()
    rng = np.random.default_rng(5)
    rows = np.unique(np.concatenate([[0, wl.N - 1], rng.choice(wl.N, 10, replace=False)]))
    E64 = oracle.widen_bf16(E)
    rk, rls, rlt = oracle.kl_forward(Hs[rows], E64, Ht[rows], E64)
    assert np.max(np.abs(to_np(kl)[rows] - rk)) <= TOL_ROW
    assert np.max(np.abs(to_np(ls)[rows] - rls)) <= TOL_ROW
    assert np.max(np.abs(to_np(lt)[rows] - rlt)) <= TOL_ROW
    rH, _ = oracle.kl_backward(Hs[rows], E64, Ht[rows], E64, dl[rows], filter_eps=EPS_BF16)
    assert normwise(to_np(dH)[rows], rH) <= TOL_GRAD_FILTER
    lhs = float(torch.sum(dH.double() * a.double()))
    rhs = float(torch.sum(dE.double() * e.double()))
    assert abs(lhs - rhs) <= 1e-3 * max(abs(lhs), abs(rhs), 1e-12)


@pytest.mark.parametrize("case", ["separate_heads", "sparse"])
def test_kl_filter_criterion_per_element(case):
    """Every entry the KL backward drops has both oracle probabilities below
    eps (its gradient dloss (p_s - p_t) is then below eps in magnitude); every
    entry where either reaches eps (with a margin for fp32 rounding) is kept."""
    from linear_cross_entropy_cce_b200 import cce
    Hs, Es, Ht, Et, mask = _kl_case(**CASES[case])
    tm = torch.from_numpy(mask).cuda() if mask is not None else None
    Hs_d, Es_d, Ht_d = _up(Hs), _up(Es), _up(Ht)
    Et_d = Es_d if CASES[case]["shared"] else _up(Et)
    kl, ls, lt = cce.kl_fwd(Hs_d, Es_d, Ht_d, Et_d, tm)
    N, V = Hs.shape[0], Es.shape[0]
    dl = torch.full((N,), 1.0 / N, dtype=torch.float32, device="cuda")
    _, _, keep = cce.kl_bwd(Hs_d, Es_d, Ht_d, Et_d, ls, lt, dl, tm, filter_eps=EPS_BF16,
                            debug_rows=N)
    torch.cuda.synchronize()
    bits = keep.cpu().numpy().view(np.uint32)
    kept = np.unpackbits(bits.view(np.uint8), bitorder="little").reshape(N, -1)[:, :V].astype(bool)
    rows = np.arange(N) if mask is None else np.nonzero(mask)[0]
    Es64, Et64 = oracle.widen_bf16(Es), oracle.widen_bf16(Et)
    Zs = oracle.widen_bf16(Hs[rows]) @ Es64.T
    Zt = oracle.widen_bf16(Ht[rows]) @ Et64.T
    Ps = np.exp(Zs - oracle.logsumexp_rows(Zs)[:, None])
    Pt = np.exp(Zt - oracle.logsumexp_rows(Zt)[:, None])
    k = kept[rows]
    dropped = ~k
    assert np.all((Ps[dropped] < EPS_BF16) & (Pt[dropped] < EPS_BF16))
    must_keep = (Ps >= EPS_BF16 * 1.001) | (Pt >= EPS_BF16 * 1.001)
    assert np.all(k[must_keep])
    if mask is not None:  # masked rows keep nothing
        assert not kept[mask == 0].any()
    assert dropped.any() and k.any()  # the criterion is exercised both ways


@pytest.mark.parametrize("shared", [True, False])
def test_kl_kahan_accumulation_beats_plain_bf16_and_is_deterministic(shared):
    """The KL backward's classifier gradient accumulated with CCE_KAHAN_DE over
    128 micro-batches (8 batches cycled 16 times): a plain bf16 running sum
    of the oracle's exact parts drifts past the 1e-2 tolerance, while the
    GPU's Kahan pair (s, c) gives s - c within half of it and at least 4x
    closer to the exactly rounded sum; two runs agree bit for bit."""
    from linear_cross_entropy_cce_b200 import cce
    N, D, V, K = 256, 128, 1024, 128
    cases = [_kl_case(N, D, V, 2.0, 3.0, shared, seed=60 + s, masked=False) for s in range(8)]
    Es, Et = cases[0][1], cases[0][3]  # one student head (and teacher head) for every batch
    Es_d = _up(Es)
    Et_d = Es_d if shared else _up(Et)
    dl = np.full(N, 1.0 / N)
    dev = []
    for Hs, _, Ht, _, _ in cases:
        Hs_d, Ht_d = _up(Hs), _up(Ht)
        _, ls, lt = cce.kl_fwd(Hs_d, Es_d, Ht_d, Et_d)
        dev.append((Hs_d, Ht_d, ls, lt))
    dlt = torch.from_numpy(dl).float().cuda()
    finals = []
    for rep in range(2):
        S = torch.zeros((V, D), dtype=torch.bfloat16, device="cuda")
        C = torch.zeros_like(S)
        for k in range(K):
            Hs_d, Ht_d, ls, lt = dev[k % 8]
            cce.kl_bwd(Hs_d, Es_d, Ht_d, Et_d, ls, lt, dlt, kahan=True, dE_out=S, dE_comp=C)
        torch.cuda.synchronize()
        finals.append((S.clone(), C.clone()))
    assert torch.equal(finals[0][0], finals[1][0]) and torch.equal(finals[0][1], finals[1][1])
    parts = [oracle.kl_backward(Hs, Es, Ht, Et, dl)[1] for Hs, _, Ht, _, _ in cases]
    exact = oracle.kahan_reference([parts[k % 8] for k in range(K)])
    plain = np.zeros_like(exact)
    for k in range(K):  # bf16 storage, exact parts, rounded after every add
        plain = oracle.widen_bf16(syn.fp32_to_bf16_bits((plain + parts[k % 8]).astype(np.float32)))
    err_plain = normwise(plain, exact)
    S, C = finals[0]
    err_kahan = normwise(to_np(S) - to_np(C), exact)
    assert err_plain > TOL_GRAD, err_plain
    assert err_kahan <= TOL_GRAD / 2, err_kahan
    assert err_plain >= 4 * err_kahan, (err_plain, err_kahan)


@pytest.mark.parametrize("N,D,V,shared", [(3, 8, 2000000, True), (200000, 16, 6, False)])
@pytest.mark.parametrize("eps", [0.0, EPS_BF16])
def test_kl_extreme_aspect_ratios(N, D, V, shared, eps):
    """A few rows over a very wide head (shared: the CTA-pair G producer over
    7813 tiles) and very many rows over a tiny one (separate heads)."""
    from linear_cross_entropy_cce_b200 import cce
    Hs, Es, Ht, Et, mask = _kl_case(N, D, V, 3.0, 2.0, shared, seed=71, masked=True)
    tm = torch.from_numpy(mask).cuda()
    Hs_d, Es_d, Ht_d = _up(Hs), _up(Es), _up(Ht)
    Et_d = Es_d if shared else _up(Et)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    kl, ls, lt = cce.kl_fwd(Hs_d, Es_d, Ht_d, Et_d, tm, status=st)
    dl = np.full(N, 1.0 / N)
    dH, dE = cce.kl_bwd(Hs_d, Es_d, Ht_d, Et_d, ls, lt, torch.from_numpy(dl).float().cuda(), tm,
                        filter_eps=eps, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    rk, rls, rlt = oracle.kl_forward(Hs, Es, Ht, Et, mask)
    assert np.max(np.abs(to_np(kl) - rk)) <= TOL_ROW
    assert np.max(np.abs(to_np(ls) - rls)) <= TOL_ROW
    assert np.max(np.abs(to_np(lt) - rlt)) <= TOL_ROW
    rH, rE = oracle.kl_backward(Hs, Es, Ht, Et, dl, mask, filter_eps=eps)
    tol = TOL_GRAD_FILTER if eps > 0 else TOL_GRAD
    assert normwise(to_np(dH), rH) <= tol
    assert normwise(to_np(dE), rE) <= tol
