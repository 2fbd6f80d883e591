"""Seeded random combinations of shape and mode against the oracle.

The parity suite pins each mode on hand-picked shapes; here every case draws
its own N, D, V, segment layout (gaps before, between and after segments),
logit scale, ignored fraction and backward mode (filter, vocabulary sort with
the tile skip, FullC, fp32 gradients), so that modes meet shapes no
hand-picked case combines.  The soft-target KL cases draw shapes, the two
logit scales, one or two heads, a row mask, the filter and fp32 gradients
the same way.  Same acceptance tolerances as the parity suite.
"""
import numpy as np
import pytest
import torch

import oracle
from linear_cross_entropy_cce_b200 import cce, synthetic as syn
from _helpers import (EPS_BF16, TOL_GRAD, TOL_GRAD_FILTER, TOL_ROW, normwise, run_bwd, run_fwd,
                      to_np, upload)

pytestmark = pytest.mark.gpu

N_CASES = 20


def _draw(k):
    rng = np.random.default_rng(5000 + k)
    N = int(rng.integers(1, 641))
    D = 8 * int(rng.integers(1, 65))
    V = int(rng.integers(1, 12001))
    nseg = int(rng.choice([1, 1, 2, 3])) if V >= 8 else 1
    segments = ()
    if nseg > 1 or rng.random() < 0.3:
        # 2 nseg distinct cut points: segment s is [c[2s], c[2s+1]), so gaps
        # fall before, between and after the segments
        cuts = np.sort(rng.choice(np.arange(V + 1), size=2 * nseg, replace=False))
        segments = tuple((int(cuts[2 * s]), int(cuts[2 * s + 1])) for s in range(nseg))
    filt = bool(rng.random() < 0.6)
    mode = {
        "filter": filt,
        "sort": filt and bool(rng.random() < 0.5),
        "full_de": filt and bool(rng.random() < 0.3),
        "fp32": bool(rng.random() < 0.25),
    }
    wl = syn.Workload(f"fuzz{k}", N=N, D=D, V=V,
                      logit_std=float(rng.choice([0.5, 2.0, 6.0, 16.0])),
                      ignore_frac=float(rng.choice([0.0, 0.1, 0.5, 1.0])),
                      segments=segments,
                      segment_mix=tuple(float(e - b) for b, e in segments) if segments else ())
    return wl, mode


def _close(got, ref, tol):
    if not np.any(ref):
        return np.max(np.abs(got), initial=0.0) <= 1e-6
    return normwise(got, ref) <= tol


@pytest.mark.parametrize("k", range(N_CASES))
def test_random_case_matches_oracle(k):
    wl, mode = _draw(k)
    x = syn.make_inputs(wl, seed=k)
    H, segs, y = upload(x)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = run_fwd(x, H, segs, y, want_colmax=mode["sort"], status=st)
    loss, lse = out[0], out[1]
    kw = {}
    if mode["sort"]:
        colmax = out[2]
        seg_arg = None if len(segs) == 1 and segs[0][:2] == (0, wl.V) else [s[:2] for s in segs]
        kw["vocab_perm"] = cce.vocab_sort(colmax, y, wl.V, x.ignore_index, segments=seg_arg)
        kw["colmax"] = colmax
    eps = EPS_BF16 if mode["filter"] else 0.0
    dl = x.dloss_mean()
    dH, dEs, _ = run_bwd(x, H, segs, y, lse, torch.from_numpy(dl).cuda(), filter_eps=eps,
                         full_de=mode["full_de"], fp32_grads=mode["fp32"], status=st, **kw)
    torch.cuda.synchronize()
    assert int(st.item()) == 0, (wl, mode)

    rl, rs = oracle.forward(x.H, x.segments, x.y, wl.V, x.ignore_index)
    assert np.max(np.abs(to_np(loss) - rl), initial=0.0) <= TOL_ROW, (wl, mode)
    assert np.max(np.abs(to_np(lse) - rs), initial=0.0) <= TOL_ROW, (wl, mode)
    rH, rE = oracle.backward(x.H, x.segments, x.y, wl.V, dl, x.ignore_index, filter_eps=eps,
                             filter_dE=not mode["full_de"])
    tol = TOL_GRAD_FILTER if mode["filter"] else TOL_GRAD
    assert _close(to_np(dH), rH, tol), (wl, mode, normwise(to_np(dH), rH))
    for g, r in zip(dEs, rE):
        assert _close(to_np(g), r, tol), (wl, mode, normwise(to_np(g), r))
    assert np.all(to_np(dH)[~x.valid] == 0)


# ---- soft-target KL --------------------------------------------------------
N_KL_CASES = 10


def _draw_kl(k):
    rng = np.random.default_rng(7000 + k)
    N = int(rng.integers(1, 513))
    D = 8 * int(rng.integers(1, 49))
    V = int(rng.integers(2, 9001))
    std_s, std_t = (float(v) for v in rng.choice([0.5, 2.0, 6.0, 14.0], size=2))
    shared = bool(rng.random() < 0.5)
    masked = bool(rng.random() < 0.5)
    eps = EPS_BF16 if rng.random() < 0.6 else 0.0
    fp32 = bool(rng.random() < 0.25)
    return N, D, V, std_s, std_t, shared, masked, eps, fp32


@pytest.mark.parametrize("k", range(N_KL_CASES))
def test_random_kl_case_matches_oracle(k):
    N, D, V, std_s, std_t, shared, masked, eps, fp32 = _draw_kl(k)
    xs = syn.make_inputs(syn.Workload("kls", N=N, D=D, V=V, logit_std=std_s, ignore_frac=0.0),
                         seed=k)
    xt = syn.make_inputs(syn.Workload("klt", N=N, D=D, V=V, logit_std=std_t, ignore_frac=0.0),
                         seed=k + 100)
    Hs, Es, Ht = xs.H, xs.segments[0][2], xt.H
    Et = Es if shared else xt.segments[0][2]
    mask = (np.random.default_rng(k).random(N) > 0.3).astype(np.int32) if masked else None
    up = lambda a: cce.bf16_from_bits(a, "cuda")
    Hs_d, Es_d, Ht_d = up(Hs), up(Es), up(Ht)
    Et_d = Es_d if shared else up(Et)
    tm = torch.from_numpy(mask).cuda() if mask is not None else None
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    kl, ls, lt = cce.kl_fwd(Hs_d, Es_d, Ht_d, Et_d, tm, status=st)
    dl = np.linspace(0.2, 1.0, N) / N
    dH, dE = cce.kl_bwd(Hs_d, Es_d, Ht_d, Et_d, ls, lt, torch.from_numpy(dl).float().cuda(), tm,
                        filter_eps=eps, fp32_grads=fp32, status=st)
    torch.cuda.synchronize()
    case = (N, D, V, std_s, std_t, shared, masked, eps, fp32)
    assert int(st.item()) == 0, case
    rk, rls, rlt = oracle.kl_forward(Hs, Es, Ht, Et, mask)
    assert np.max(np.abs(to_np(kl) - rk)) <= TOL_ROW, case
    assert np.max(np.abs(to_np(ls) - rls)) <= TOL_ROW, case
    assert np.max(np.abs(to_np(lt) - rlt)) <= TOL_ROW, case
    rH, rE = oracle.kl_backward(Hs, Es, Ht, Et, dl, mask, filter_eps=eps)
    tol = TOL_GRAD_FILTER if eps > 0 else TOL_GRAD
    assert _close(to_np(dH), rH, tol), (case, normwise(to_np(dH), rH))
    assert _close(to_np(dE), rE, tol), (case, normwise(to_np(dE), rE))
    if mask is not None:
        assert np.all(to_np(kl)[mask == 0] == 0) and np.all(to_np(dH)[mask == 0] == 0)


# ---- vocabulary parallel (shards run one after another on one GPU) ---------
N_VP_CASES = 8


@pytest.mark.parametrize("k", range(N_VP_CASES))
def test_random_vocab_parallel_case_matches_oracle(k):
    from linear_cross_entropy_cce_b200 import vocab_parallel as vp
    wl, _ = _draw(100 + k)
    rng = np.random.default_rng(9000 + k)
    R = int(rng.integers(2, 6))
    eps = EPS_BF16 if rng.random() < 0.5 else 0.0
    # filtered cases sort each shard's vocabulary by its column maxima, as
    # the vocabulary-parallel step of the benchmark does
    sort = eps > 0 and bool(np.random.default_rng(9500 + k).random() < 0.7)
    x = syn.make_inputs(wl, seed=100 + k)
    H, segs, y = upload(x)
    parts, colmaxes = [], []
    shards = [vp.shard_segments(segs, v0, v1) for v0, v1 in vp.shard_ranges(wl.V, R)]
    for local in shards:
        if not local:  # a rank whose range holds no live ids
            parts.append(torch.stack([torch.full((wl.N,), -float("inf"), device="cuda"),
                                      torch.zeros(wl.N, device="cuda")]))
            colmaxes.append(None)
            continue
        out = cce.fwd(H, None, y, x.ignore_index, segments=local, V=wl.V, shard=True,
                      want_colmax=sort)
        parts.append(torch.stack([out[1], out[0]]))
        colmaxes.append(out[2] if sort else None)
    loss, lse = cce.vocab_combine(torch.stack(parts), y, wl.V, x.ignore_index, list(wl.segs()))
    rl, rlse = oracle.forward(x.H, x.segments, x.y, wl.V, x.ignore_index)
    case = (wl, R, eps, sort)
    assert np.max(np.abs(to_np(loss) - rl), initial=0.0) <= TOL_ROW, case
    assert np.max(np.abs(to_np(lse) - rlse), initial=0.0) <= TOL_ROW, case

    dl = x.dloss_mean()
    dlt = torch.from_numpy(dl).cuda()
    dH = torch.zeros((wl.N, wl.D), dtype=torch.float32, device="cuda")
    dE = {}
    for local, cm in zip(shards, colmaxes):
        if not local:
            continue
        perm = (cce.vocab_sort(cm, y, wl.V, x.ignore_index, segments=[s_[:2] for s_ in local])
                if sort else None)
        dH_p, dEs, _ = cce.bwd(H, None, y, lse, dlt, x.ignore_index, segments=local, V=wl.V,
                               filter_eps=eps, vocab_perm=perm, colmax=cm, fp32_dh=True,
                               shard=True)
        dH += dH_p
        for (b, e, _), g in zip(local, dEs):
            dE[(b, e)] = g
    torch.cuda.synchronize()
    rH, rE = oracle.backward(x.H, x.segments, x.y, wl.V, dl, x.ignore_index, filter_eps=eps)
    tol = TOL_GRAD_FILTER if eps > 0 else TOL_GRAD
    assert _close(to_np(dH), rH, tol), (case, normwise(to_np(dH), rH))
    for (b, e, _), r in zip(x.segments, rE):
        got = torch.cat([dE[kk] for kk in sorted(dE) if b <= kk[0] < e]).float().cpu().numpy()
        assert got.shape == r.shape, case
        assert _close(got, r, tol), (case, normwise(got, r))
