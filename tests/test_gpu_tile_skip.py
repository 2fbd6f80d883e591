"""The exact tile skip of the backward (cce_bwd with the forward's colmax):
a 128 x 256 tile whose bound  max colmax - min lse  lies below ln(eps) is not
recomputed.  The skip must not change which softmax entries are kept, and a
skipped tile must contribute exactly its one-hot entries."""
import numpy as np
import pytest
import torch

import oracle
from linear_cross_entropy_cce_b200 import synthetic as syn
from _helpers import EPS_BF16, TOL_GRAD, TOL_GRAD_FILTER, normwise, run_bwd, to_np, upload

pytestmark = pytest.mark.gpu

LOG2E = 1.4426950408889634

# a flat softmax over a wide vocabulary and few rows: most column maxima sit
# below lse + ln(eps), so after the sort the tail tiles can be skipped
WL = syn.Workload("skip", N=300, D=192, V=60000, logit_std=1.0, ignore_frac=0.1)


def _fwd_sort(x):
    from linear_cross_entropy_cce_b200 import cce
    H, segs, y = upload(x)
    loss, lse, colmax = cce.fwd(H, segs[0][2], y, x.ignore_index, want_colmax=True)
    perm = cce.vocab_sort(colmax, y, x.wl.V, x.ignore_index)
    return H, segs, y, lse, colmax, perm


def _skippable_tiles(x, lse, colmax, perm):
    """Tiles the kernel's rule skips, evaluated on the host (compact rows in
    blocks of 128, walk tiles of 256 columns, margin 1/16 in log2 units)."""
    lse = lse.cpu().numpy()[x.valid].astype(np.float32) * np.float32(LOG2E)
    cm = colmax.cpu().numpy()[perm.cpu().numpy()]
    tiles = np.array([cm[t:t + 256].max() for t in range(0, len(cm), 256)], np.float32) * np.float32(LOG2E)
    blk = np.array([lse[b:b + 128].min() for b in range(0, len(lse), 128)], np.float32)
    thr = np.log2(np.float32(EPS_BF16 * (1 - 1 / 256))) - 1 / 16
    return int(((tiles[:, None] - blk[None, :]) < thr).sum()), tiles.size * blk.size


def test_tile_skip_keeps_the_same_entries():
    x = syn.make_inputs(WL, seed=11)
    H, segs, y, lse, colmax, perm = _fwd_sort(x)
    n_skip, n_tiles = _skippable_tiles(x, lse, colmax, perm)
    assert 0 < n_skip < n_tiles, (n_skip, n_tiles)    # the case exercises both paths
    dl = torch.from_numpy(x.dloss_mean()).cuda()
    rows = x.wl.N
    kw = dict(filter_eps=EPS_BF16, vocab_perm=perm, debug_rows=rows)
    dH0, dE0, keep0 = run_bwd(x, H, segs, y, lse, dl, **kw)
    dH1, dE1, keep1 = run_bwd(x, H, segs, y, lse, dl, colmax=colmax, **kw)
    torch.cuda.synchronize()
    assert torch.equal(keep0, keep1)
    rH, rE = oracle.backward(x.H, x.segments, x.y, x.wl.V, x.dloss_mean(), x.ignore_index,
                             filter_eps=EPS_BF16)
    assert normwise(to_np(dH1), rH) <= TOL_GRAD_FILTER
    assert normwise(to_np(dE1[0]), rE[0]) <= TOL_GRAD_FILTER
    assert normwise(to_np(dH1), to_np(dH0)) <= 2e-3
    assert normwise(to_np(dE1[0]), to_np(dE0[0])) <= 2e-3


def test_tile_skip_with_kahan_is_exact():
    """On the dense deterministic (Kahan) route the skip changes no bit."""
    from linear_cross_entropy_cce_b200 import cce
    x = syn.make_inputs(WL, seed=12)
    H, segs, y, lse, colmax, perm = _fwd_sort(x)
    dl = torch.from_numpy(x.dloss_mean()).cuda()
    outs = []
    for cm in (None, colmax):
        S = torch.zeros((x.wl.V, x.wl.D), dtype=torch.bfloat16, device="cuda")
        C = torch.zeros_like(S)
        dH, _, _ = cce.bwd(H, segs[0][2], y, lse, dl, x.ignore_index, filter_eps=EPS_BF16,
                           vocab_perm=perm, colmax=cm, kahan=True, dE_out=S, dE_comp=C)
        outs.append((dH, S, C))
    torch.cuda.synchronize()
    for a, b in zip(outs[0], outs[1]):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))


@pytest.mark.parametrize("segmented", [False, True])
def test_every_tile_skipped_leaves_the_one_hot_gradient(segmented):
    """A colmax far below the true one skips every tile: what remains is the
    one-hot part of G, i.e. the oracle's gradient with every softmax entry
    filtered (filter_eps above any probability)."""
    from linear_cross_entropy_cce_b200 import cce
    if segmented:
        wl = syn.Workload("skip_all_seg", N=260, D=128, V=9000, logit_std=3.0, ignore_frac=0.2,
                          segments=((0, 5000), (5300, 9000)), segment_mix=(0.6, 0.4))
    else:
        wl = syn.Workload("skip_all", N=333, D=200, V=7000, logit_std=3.0, ignore_frac=0.15)
    x = syn.make_inputs(wl, seed=13)
    H, segs, y = upload(x)
    single = not segmented
    if single:
        _, lse, colmax = cce.fwd(H, segs[0][2], y, x.ignore_index, want_colmax=True)
    else:
        _, lse, colmax = cce.fwd(H, None, y, x.ignore_index, segments=segs, V=wl.V, want_colmax=True)
    low = colmax - 1000.0
    dl = torch.from_numpy(x.dloss_mean()).cuda()
    dH, dEs, _ = run_bwd(x, H, segs, y, lse, dl, filter_eps=EPS_BF16, colmax=low)
    torch.cuda.synchronize()
    rH, rE = oracle.backward(x.H, x.segments, x.y, wl.V, x.dloss_mean(), x.ignore_index,
                             filter_eps=2.0)
    assert normwise(to_np(dH), rH) <= TOL_GRAD
    for g, r in zip(dEs, rE):
        assert normwise(to_np(g), r) <= TOL_GRAD
