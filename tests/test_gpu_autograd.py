"""The torch.autograd drop-in and the full-classifier-gradient variant,
against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from linear_cross_entropy_cce_b200 import synthetic as syn
from _helpers import EPS_BF16, TOL_GRAD, TOL_GRAD_FILTER, TOL_MEAN_REL, TOL_ROW, normwise, to_np, upload

pytestmark = pytest.mark.gpu


def _leaf(t):
    return t.detach().clone().requires_grad_(True)


@pytest.mark.parametrize("reduction", ["mean", "sum", "none"])
def test_autograd_matches_oracle(reduction):
    from linear_cross_entropy_cce_b200.autograd import linear_cross_entropy
    wl = syn.Workload("ag", N=500, D=256, V=7000, logit_std=3.0, ignore_frac=0.1)
    x = syn.make_inputs(wl, seed=3)
    H, segs, y = upload(x)
    Hl, El = _leaf(H), _leaf(segs[0][2])
    loss = linear_cross_entropy(Hl, El, y, reduction=reduction, filter_eps=0.0)
    rng = np.random.default_rng(0)
    if reduction == "none":
        up = rng.standard_normal(wl.N).astype(np.float32)
        loss.backward(torch.from_numpy(up).cuda())
        dl = np.where(x.valid, up, 0).astype(np.float64)
    else:
        loss.backward()
        dl = x.dloss_mean().astype(np.float64) if reduction == "mean" else x.valid.astype(np.float64)
    rl, _ = oracle.forward(x.H, x.segments, x.y, wl.V, x.ignore_index)
    if reduction == "none":
        assert np.max(np.abs(to_np(loss) - rl)) <= TOL_ROW
    elif reduction == "mean":
        ref = oracle.mean_loss(rl, x.valid)
        assert abs(loss.item() - ref) <= TOL_MEAN_REL * abs(ref)
    else:
        assert abs(loss.item() - rl.sum()) <= 1e-5 * abs(rl.sum())
    rH, rE = oracle.backward(x.H, x.segments, x.y, wl.V, dl, x.ignore_index)
    assert Hl.grad.dtype == torch.bfloat16 and El.grad.dtype == torch.bfloat16
    assert normwise(to_np(Hl.grad), rH) <= TOL_GRAD
    assert normwise(to_np(El.grad), rE[0]) <= TOL_GRAD


def test_autograd_segments_sort_and_filter():
    from linear_cross_entropy_cce_b200.autograd import linear_cross_entropy
    wl = syn.Workload("ags", N=600, D=192, V=9000, logit_std=12.0, ignore_frac=0.2,
                      segments=((0, 5000), (5200, 9000)), segment_mix=(0.6, 0.4))
    x = syn.make_inputs(wl, seed=4)
    H, segs, y = upload(x)
    Hl = _leaf(H)
    Es = [_leaf(t) for _, _, t in segs]
    loss = linear_cross_entropy(Hl, None, y, segments=[(b, e, t) for (b, e, _), t in zip(segs, Es)],
                                vocab_sort=True)
    loss.backward()
    rH, rE = oracle.backward(x.H, x.segments, x.y, wl.V, x.dloss_mean(), x.ignore_index,
                             filter_eps=EPS_BF16)
    assert normwise(to_np(Hl.grad), rH) <= TOL_GRAD_FILTER
    for g, r in zip(Es, rE):
        assert normwise(to_np(g.grad), r) <= TOL_GRAD_FILTER


@pytest.mark.parametrize("std", [4.0, 16.0])  # dense chunks / sparse-route chunks
def test_full_classifier_gradient(std):
    from linear_cross_entropy_cce_b200 import cce
    wl = syn.Workload("fullc", N=700, D=256, V=24000, logit_std=std, ignore_frac=0.1)
    x = syn.make_inputs(wl, seed=5)
    H, segs, y = upload(x)
    E = segs[0][2]
    loss, lse = cce.fwd(H, E, y)
    dl = x.dloss_mean()
    dlt = torch.from_numpy(dl).cuda()
    dH, dE, _ = cce.bwd(H, E, y, lse, dlt, filter_eps=EPS_BF16, full_de=True)
    dH_f, _, _ = cce.bwd(H, E, y, lse, dlt, filter_eps=EPS_BF16)   # both filtered
    _, dE_u, _ = cce.bwd(H, E, y, lse, dlt, filter_eps=0.0)        # both full
    torch.cuda.synchronize()
    rH, rE = oracle.backward(x.H, x.segments, x.y, wl.V, dl, x.ignore_index, filter_eps=EPS_BF16,
                             filter_dE=False)
    # dE is the full classifier gradient: the filter-off result, bit for bit
    assert torch.equal(dE.view(torch.int16), dE_u.view(torch.int16))
    assert normwise(to_np(dE), rE[0]) <= TOL_GRAD
    # dH is the filtered input gradient, in dense and sparse-route chunks alike;
    # it takes the same G entries as the default filtered path
    assert normwise(to_np(dH), rH) <= TOL_GRAD_FILTER
    assert normwise(to_np(dH), to_np(dH_f).astype(np.float64)) <= 2e-3


def test_full_classifier_gradient_with_kahan():
    """FullC combined with Kahan accumulation of dE over micro-batches: the
    Kahan path runs every chunk on the dense route, so dH comes from the
    filtered slab and dE from the full one."""
    from linear_cross_entropy_cce_b200 import cce
    wl = syn.Workload("fullck", N=400, D=128, V=5000, logit_std=5.0, ignore_frac=0.1)
    xs = [syn.make_inputs(wl, seed=s) for s in range(3)]
    Eh = xs[0].segments
    Et = cce.bf16_from_bits(Eh[0][2], "cuda")
    out = {}
    for full in (True, False):
        S = torch.zeros((wl.V, wl.D), dtype=torch.bfloat16, device="cuda")
        C = torch.zeros_like(S)
        dHs = []
        for x in xs:
            H = cce.bf16_from_bits(x.H, "cuda")
            y = torch.from_numpy(x.y).cuda()
            _, lse = cce.fwd(H, Et, y)
            dl = torch.from_numpy(x.dloss_mean()).cuda()
            eps = EPS_BF16 if full else 0.0
            dH, _, _ = cce.bwd(H, Et, y, lse, dl, filter_eps=eps, kahan=True, full_de=full,
                               dE_out=S, dE_comp=C)
            dHs.append(dH)
        torch.cuda.synchronize()
        out[full] = (S, C, dHs)
    S, C, dHs = out[True]
    # the full dE parts are the filter-off parts, so the Kahan state matches bit for bit
    assert torch.equal(S, out[False][0]) and torch.equal(C, out[False][1])
    parts = [oracle.backward(x.H, Eh, x.y, wl.V, x.dloss_mean(), -100)[1][0] for x in xs]
    assert normwise(to_np(S) - to_np(C), oracle.kahan_reference(parts)) <= TOL_GRAD
    for x, dH in zip(xs, dHs):
        rH, _ = oracle.backward(x.H, Eh, x.y, wl.V, x.dloss_mean(), -100, filter_eps=EPS_BF16,
                                filter_dE=False)
        assert normwise(to_np(dH), rH) <= TOL_GRAD_FILTER
