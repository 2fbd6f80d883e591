"""Vocabulary-parallel host logic on CPU: shard ranges, the per-row combine
of shard parts, and the two exchanges over world-size-2 gloo ranks.  The
per-shard parts come from the oracle's logits (no GPU); the expected values
from the oracle's full-vocabulary forward and backward."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
from linear_cross_entropy_cce_b200 import synthetic as syn
from linear_cross_entropy_cce_b200 import vocab_parallel as vp

WL = syn.Workload("vp", N=70, D=24, V=1300, logit_std=3.0, ignore_frac=0.15,
                  segments=((0, 700), (760, 1300)), segment_mix=(0.6, 0.4))


def _inputs(seed=0):
    x = syn.make_inputs(WL, seed=seed)
    y = x.y.copy()
    y[3] = 730      # a target in the dead gap: no shard holds it
    y[5] = WL.V + 9  # outside the vocabulary
    return x, y


def _combine_ref(parts, y, V, ignore_index, head_ranges):
    """Host restatement of the combine (the library's is a CUDA kernel, which
    a CPU process group cannot run): lse = log-add-exp of the shards' lse
    parts, loss = lse - sum of their logit parts; ignored rows 0; a target
    outside the head's live ranges NaN."""
    ranges = head_ranges or [(0, V)]
    lse_p, zy_p = parts[:, 0].double(), parts[:, 1].double()
    lse = torch.logsumexp(lse_p, dim=0)
    zy = zy_p.sum(dim=0)
    yl = y.long()
    held = torch.zeros_like(yl, dtype=torch.bool)
    for b, e in ranges:
        held |= (yl >= b) & (yl < e)
    ign = yl == ignore_index
    bad = ~ign & ~held
    nan = torch.full_like(lse, float("nan"))
    zero = torch.zeros_like(lse)
    lse = torch.where(ign, zero, torch.where(bad, nan, lse))
    loss = torch.where(ign, zero, torch.where(bad, nan, lse - zy))
    return loss, lse


HEAD = [(b, e) for b, e in WL.segments]


def _oracle_parts(x, y, v0, v1):
    """Shard [v0, v1): (lse over its live ids, correct-token logit if held,
    1 if held) per row, from the oracle's logits."""
    H64 = oracle.widen_bf16(x.H)
    segs = [(b, e, oracle.widen_bf16(E)) for b, e, E in x.segments]
    local = [(max(b, v0), min(e, v1), E[max(b, v0) - b:min(e, v1) - b])
             for b, e, E in segs if max(b, v0) < min(e, v1)]
    Z = oracle.logits_rows(H64, local, WL.V)
    lse = oracle.logsumexp_rows(Z)
    held = np.array([any(b <= t < e for b, e, _ in local) for t in y])
    zy = np.where(held, Z[np.arange(len(y)), np.clip(y, 0, WL.V - 1)], 0.0)
    ign = y == x.ignore_index
    lse = np.where(ign, 0.0, lse)
    zy = np.where(ign, 0.0, zy)
    return np.stack([lse, zy, held.astype(np.float64)]), Z


def _expected(x, y):
    loss, lse = oracle.forward(x.H, x.segments, y, WL.V, x.ignore_index)
    return loss, lse


def test_shard_ranges_partition_the_vocabulary():
    for V, R in [(256000, 3), (1000, 4), (300, 8), (5, 1)]:
        r = vp.shard_ranges(V, R)
        assert len(r) == R and r[0][0] == 0 and r[-1][1] == V
        assert all(a[1] == b[0] for a, b in zip(r, r[1:]))
        assert all(b % 256 == 0 or b == V for _, b in r)


def test_shard_segments_cut_the_head():
    E = torch.arange(1300 * 2, dtype=torch.float32).view(1300, 2)
    segs = [(0, 700, E[:700]), (760, 1300, E[700:])]
    got = vp.shard_segments(segs, 512, 1024)
    assert [(b, e) for b, e, _ in got] == [(512, 700), (760, 1024)]
    assert torch.equal(got[0][2], E[512:700]) and torch.equal(got[1][2], E[700:964])
    assert vp.shard_segments(segs, 700, 760) == []


@pytest.mark.parametrize("R", [2, 3])
def test_combine_matches_full_oracle(R):
    x, y = _inputs()
    parts = np.stack([_oracle_parts(x, y, v0, v1)[0][:2] for v0, v1 in vp.shard_ranges(WL.V, R)])
    loss, lse = _combine_ref(torch.from_numpy(parts), torch.from_numpy(y), WL.V, x.ignore_index, HEAD)
    rl, rlse = _expected(x, y)
    bad = np.isnan(rl)
    assert bad[3] and bad[5] and np.array_equal(np.isnan(loss.numpy()), bad)
    assert np.allclose(loss.numpy()[~bad], rl[~bad], atol=1e-9, rtol=0)
    assert np.allclose(lse.numpy()[~bad], rlse[~bad], atol=1e-9, rtol=0)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    import datetime
    import sys
    import torch.distributed as dist
    sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=60))
    x, y = _inputs()
    v0, v1 = vp.shard_ranges(WL.V, world)[rank]
    parts, Z = _oracle_parts(x, y, v0, v1)
    t = [torch.from_numpy(p.copy()) for p in parts]
    loss, lse = vp.exchange_forward(t[0], t[1], torch.from_numpy(y), WL.V, HEAD, x.ignore_index,
                                    combine=_combine_ref)
    # this shard's share of dH with the full lse: dloss * (softmax - onehot) over its ids
    lse_full = lse.numpy()
    dl = x.dloss_mean()
    ok = ~np.isnan(lse_full) & (y != x.ignore_index)
    P = np.exp(Z - np.where(ok, lse_full, 0.0)[:, None])
    for i in np.nonzero(ok & (parts[2] > 0))[0]:
        P[i, y[i]] -= 1.0
    G = np.where(ok, dl, 0.0)[:, None] * P
    E_full = np.zeros((WL.V, WL.D))
    for b, e, E in x.segments:
        E_full[b:e] = oracle.widen_bf16(E)
    dH_part = torch.from_numpy(G @ E_full)
    vp.exchange_backward(dH_part)
    out[rank] = (loss.numpy(), lse_full, dH_part.numpy())
    dist.barrier()
    dist.destroy_process_group()


def test_exchanges_world2_gloo():
    world, port = 2, _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn")
        res = dict(out)
    x, y = _inputs()
    rl, rlse = _expected(x, y)
    bad = np.isnan(rl)
    rH, _ = oracle.backward(x.H, x.segments, np.where(bad, x.ignore_index, y), WL.V,
                            np.where(bad, 0.0, x.dloss_mean()), x.ignore_index)
    for r in range(world):
        loss, lse, dH = res[r]
        assert np.array_equal(np.isnan(loss), bad)
        assert np.allclose(loss[~bad], rl[~bad], atol=1e-9, rtol=0)
        assert np.allclose(lse[~bad], rlse[~bad], atol=1e-9, rtol=0)
        assert np.allclose(dH[~bad], rH[~bad], atol=1e-10, rtol=1e-8)


def test_rank_without_ids_contributes_nothing():
    """More ranks than 256-aligned ranges leave some ranks an empty shard:
    their parts are -inf / 0 / 0 (no launch), and the combine is unchanged."""
    ranges = vp.shard_ranges(600, 4)
    assert ranges[-1] == (600, 600)
    H = torch.zeros((6, 8))
    y = torch.tensor([0, 5, -100, 599, 300, 1], dtype=torch.int32)
    lse_p, zy_p = vp.shard_forward_parts(H, y, [], 600)
    assert torch.all(torch.isinf(lse_p) & (lse_p < 0)) and torch.all(zy_p == 0)
    full = torch.tensor([[1.0, 2.0, 0.0, 3.0, 0.5, 1.5], [0.2, 0.1, 0.0, 0.3, 0.4, 0.2]])
    parts = torch.stack([full, torch.stack([lse_p, zy_p])])
    loss, lse = _combine_ref(parts, y, 600, -100, None)
    ref_loss, ref_lse = _combine_ref(full[None], y, 600, -100, None)
    assert torch.equal(loss, ref_loss) and torch.equal(lse, ref_lse)
