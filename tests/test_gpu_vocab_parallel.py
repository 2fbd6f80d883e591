"""Vocabulary-parallel kernels (cce_fwd_shard, cce_bwd with CCE_VOCAB_SHARD)
on one GPU: R shards run one after another, their parts are combined as the
ranks would combine them, and the result is checked against the
single-call path and the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from linear_cross_entropy_cce_b200 import synthetic as syn
from linear_cross_entropy_cce_b200 import vocab_parallel as vp
from _helpers import EPS_BF16, TOL_GRAD, TOL_GRAD_FILTER, TOL_ROW, normwise, to_np, upload

pytestmark = pytest.mark.gpu

HEADS = {
    "single": syn.Workload("vp_single", N=600, D=256, V=9000, logit_std=4.0, ignore_frac=0.1),
    "composite": syn.Workload("vp_comp", N=500, D=192, V=8000, logit_std=6.0, ignore_frac=0.3,
                              segments=((0, 4500), (4700, 8000)), segment_mix=(0.7, 0.3)),
}


def _shards(x, segs, R):
    return [vp.shard_segments(segs, v0, v1) for v0, v1 in vp.shard_ranges(x.wl.V, R)]


@pytest.mark.parametrize("R", [2, 3])
@pytest.mark.parametrize("head", ["single", "composite"])
@pytest.mark.parametrize("eps", [0.0, EPS_BF16])
def test_vocab_parallel_matches_oracle(head, R, eps):
    from linear_cross_entropy_cce_b200 import cce
    wl = HEADS[head]
    x = syn.make_inputs(wl, seed=21)
    x.y[7] = wl.V + 5                       # outside the vocabulary: NaN row
    if head == "composite":
        x.y[9] = 4600                       # in the dead gap: no shard holds it
    H, segs, y = upload(x)
    shards = _shards(x, segs, R)
    parts = []
    for local in shards:
        zy_p, lse_p = cce.fwd(H, None, y, x.ignore_index, segments=local, V=wl.V, shard=True)
        parts.append(torch.stack([lse_p, zy_p]))
    loss, lse = cce.vocab_combine(torch.stack(parts), y, wl.V, x.ignore_index, list(wl.segs()))
    torch.cuda.synchronize()
    rl, rlse = oracle.forward(x.H, x.segments, x.y, wl.V, x.ignore_index)
    bad = np.isnan(rl)
    assert bad[7] and np.array_equal(np.isnan(to_np(loss)), bad)
    assert np.max(np.abs(to_np(loss)[~bad] - rl[~bad])) <= TOL_ROW
    assert np.max(np.abs(to_np(lse)[~bad] - rlse[~bad])) <= TOL_ROW

    # backward: each shard with the combined lse, dH shares summed
    dl = x.dloss_mean()
    dl[bad] = 0.0
    lse_b = torch.where(torch.isnan(lse), torch.zeros_like(lse), lse)
    dlt = torch.from_numpy(dl).cuda()
    dH = torch.zeros((wl.N, wl.D), dtype=torch.float32, device="cuda")
    dE = {}
    for local in shards:
        dH_p, dEs, _ = cce.bwd(H, None, y, lse_b, dlt, x.ignore_index, segments=local, V=wl.V,
                               filter_eps=eps, fp32_dh=True, shard=True)
        assert dH_p.dtype == torch.float32 and all(g.dtype == torch.bfloat16 for g in dEs)
        dH += torch.nan_to_num(dH_p, nan=0.0)
        for (b, e, _), g in zip(local, dEs):
            dE[(b, e)] = g
    torch.cuda.synchronize()
    y_ok = np.where(bad, x.ignore_index, x.y)
    rH, rE = oracle.backward(x.H, x.segments, y_ok, wl.V, dl, x.ignore_index, filter_eps=eps)
    tol = TOL_GRAD_FILTER if eps > 0 else TOL_GRAD
    assert normwise(to_np(dH)[~bad], rH[~bad]) <= tol
    for (b, e, _), r in zip(x.segments, rE):
        got = torch.cat([dE[k] for k in sorted(dE) if b <= k[0] < e]).float().cpu().numpy()
        assert got.shape == r.shape
        assert normwise(got, r) <= tol


def test_one_shard_is_the_single_call():
    """R = 1: the shard forward's parts combine to cce_fwd's loss and lse."""
    from linear_cross_entropy_cce_b200 import cce
    wl = HEADS["single"]
    x = syn.make_inputs(wl, seed=22)
    H, segs, y = upload(x)
    loss0, lse0 = cce.fwd(H, segs[0][2], y, x.ignore_index)
    zy_p, lse_p = cce.fwd(H, segs[0][2], y, x.ignore_index, shard=True)
    loss1, lse1 = cce.vocab_combine(torch.stack([lse_p, zy_p])[None], y, wl.V, x.ignore_index)
    torch.cuda.synchronize()
    assert torch.equal(lse0, lse1)
    assert torch.allclose(loss0, loss1, atol=1e-5, rtol=0)


@pytest.mark.parametrize("R", [1, 2, 5])
def test_combine_kernel_matches_oracle_with_empty_shards(R):
    """cce_vocab_combine on shard parts computed by the oracle, with two
    extra ranks that hold no ids (-inf, 0): per-row loss and lse equal the
    oracle's full-vocabulary forward; ignored rows 0; targets in the dead gap
    or outside the vocabulary NaN."""
    from linear_cross_entropy_cce_b200 import cce
    wl = HEADS["composite"]
    x = syn.make_inputs(wl, seed=24)
    x.y[3] = 4600        # dead gap
    x.y[5] = wl.V + 11   # outside the vocabulary
    x.y[6] = -7          # negative, not the ignore index
    segs64 = [(b, e, oracle.widen_bf16(E)) for b, e, E in x.segments]
    Z = oracle.logits_rows(oracle.widen_bf16(x.H), segs64, wl.V)
    parts = []
    for v0, v1 in vp.shard_ranges(wl.V, R) + [(wl.V, wl.V)] * 2:
        cols = np.zeros(wl.V, bool)
        cols[v0:v1] = True
        Zs = np.where(cols[None, :], Z, -np.inf)
        m = Zs.max(axis=1)
        with np.errstate(invalid="ignore", divide="ignore"):
            lse = np.where(np.isfinite(m), m + np.log(np.exp(Zs - np.where(np.isfinite(m), m, 0)[:, None]).sum(1)), -np.inf)
        yc = np.clip(x.y, 0, wl.V - 1)
        held = (x.y >= v0) & (x.y < v1) & np.isfinite(Z[np.arange(wl.N), yc])
        zy = np.where(held, Z[np.arange(wl.N), yc], 0.0)
        parts.append(np.stack([lse, zy]))
    P = torch.from_numpy(np.stack(parts).astype(np.float32)).cuda()
    y = torch.from_numpy(x.y).cuda()
    loss, lse = cce.vocab_combine(P, y, wl.V, x.ignore_index, list(wl.segs()))
    torch.cuda.synchronize()
    rl, rs = oracle.forward(x.H, x.segments, x.y, wl.V, x.ignore_index)
    bad = np.isnan(rl)
    assert bad[3] and bad[5] and bad[6]
    assert np.array_equal(np.isnan(to_np(loss)), bad) and np.array_equal(np.isnan(to_np(lse)), bad)
    ign = x.y == x.ignore_index
    assert np.all(to_np(loss)[ign] == 0) and np.all(to_np(lse)[ign] == 0)
    ok = ~bad & ~ign
    assert np.max(np.abs(to_np(loss)[ok] - rl[ok])) <= TOL_ROW
    assert np.max(np.abs(to_np(lse)[ok] - rs[ok])) <= TOL_ROW


def test_autograd_over_a_one_rank_nccl_group():
    """vocab_parallel_cross_entropy end to end (forward, all-gather,
    backward, all-reduce) on a world-size-1 NCCL group."""
    import datetime
    import socket
    import torch.distributed as dist
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60))
    try:
        wl = HEADS["composite"]
        x = syn.make_inputs(wl, seed=23)
        H, segs, y = upload(x)
        Hl = H.detach().clone().requires_grad_(True)
        local = [(b, e, t.detach().clone().requires_grad_(True)) for b, e, t in segs]
        loss = vp.vocab_parallel_cross_entropy(Hl, y, local, wl.V, x.ignore_index,
                                               head_ranges=list(wl.segs()))
        loss.backward()
        torch.cuda.synchronize()
        rl, _ = oracle.forward(x.H, x.segments, x.y, wl.V, x.ignore_index)
        ref = oracle.mean_loss(rl, x.valid)
        assert abs(loss.item() - ref) <= 1e-5 * abs(ref)
        rH, rE = oracle.backward(x.H, x.segments, x.y, wl.V, x.dloss_mean(), x.ignore_index,
                                 filter_eps=EPS_BF16)
        assert normwise(to_np(Hl.grad), rH) <= TOL_GRAD_FILTER
        for (_, _, t), r in zip(local, rE):
            assert normwise(to_np(t.grad), r) <= TOL_GRAD_FILTER
    finally:
        dist.destroy_process_group()
