"""GPU parity: libcce (through its C ABI) against the fp64 oracle.

Sizes here are ones the oracle finishes in seconds while still spanning
several 128x256 tiles, ragged row/vocabulary/D tails, ignored rows, a
composite head with a dead gap, filtering, the vocabulary sort and the Kahan
path.  Tolerances are the acceptance tolerances (tests/_helpers.py).
"""
import math

import numpy as np
import pytest
import torch

import oracle
from linear_cross_entropy_cce_b200 import synthetic as syn
from _helpers import (EPS_BF16, TOL_GRAD, TOL_GRAD_FILTER, TOL_MEAN_REL, TOL_ROW, normwise,
                      run_bwd, run_fwd, to_np, upload)

pytestmark = pytest.mark.gpu

CASES = {
    "tiny": syn.WORKLOADS["tiny"],
    # ragged everything: N % 128, D % 64 != 0, V % 256 != 0
    "ragged": syn.Workload("ragged", N=333, D=200, V=1000, logit_std=4.0, ignore_frac=0.15),
    "gemma_like_small": syn.scaled(syn.WORKLOADS["gemma2_2b_head"], N=700, D=576, V=5000),
    "phi_like_small": syn.scaled(syn.WORKLOADS["phi35_mini_head"], N=520, D=384, V=3001),
    "composite_small": syn.scaled(syn.WORKLOADS["composite_two_segment"], N=900, D=256, V=6200,
                                  segments=((0, 3800), (3954, 6200))),
    "wide_D": syn.Workload("wide_D", N=260, D=1032, V=2300, logit_std=2.0, ignore_frac=0.0),
    # logit std 40: after filtering nearly every 16-wide slice of G is zero,
    # so most tensor-core steps and whole tiles are skipped
    "peaky": syn.Workload("peaky", N=400, D=320, V=9000, logit_std=40.0, ignore_frac=0.05),
    # filtered G below 1/2048 density: the sparse (CUDA-core) contractions run
    "sparse_g": syn.Workload("sparse_g", N=900, D=264, V=30000, logit_std=16.0, ignore_frac=0.1),
    "sparse_g_segments": syn.Workload("sparse_g_segments", N=700, D=192, V=26000, logit_std=16.0,
                                      ignore_frac=0.3, segments=((0, 15000), (15500, 26000)),
                                      segment_mix=(0.7, 0.3)),
}


@pytest.fixture(scope="module")
def data():
    return {k: syn.make_inputs(wl, seed=0) for k, wl in CASES.items()}


def _fwd_check(x):
    H, segs, y = upload(x)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    loss, lse = run_fwd(x, H, segs, y, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    rl, rs = oracle.forward(x.H, x.segments, x.y, x.wl.V, x.ignore_index)
    gl, gs = to_np(loss), to_np(lse)
    assert np.max(np.abs(gl - rl)) <= TOL_ROW, np.max(np.abs(gl - rl))
    assert np.max(np.abs(gs - rs)) <= TOL_ROW, np.max(np.abs(gs - rs))
    v = x.valid
    m_ref = oracle.mean_loss(rl, v)
    m_got = float(np.sum(gl[v], dtype=np.float64)) / max(1, int(v.sum()))
    # relative 1e-5, with an absolute floor at fp32 resolution for a mean
    # that is exactly 0 (a one-id vocabulary)
    assert abs(m_got - m_ref) <= TOL_MEAN_REL * abs(m_ref) + 1e-6
    assert np.all(gl[~v] == 0) and np.all(gs[~v] == 0)
    return H, segs, y, lse


@pytest.mark.parametrize("case", list(CASES))
def test_forward_matches_oracle(data, case):
    _fwd_check(data[case])


@pytest.mark.parametrize("case", list(CASES))
def test_backward_unfiltered_matches_oracle(data, case):
    x = data[case]
    H, segs, y, lse = _fwd_check(x)
    dl = x.dloss_mean()
    dH, dEs, _ = run_bwd(x, H, segs, y, lse, torch.from_numpy(dl).cuda())
    torch.cuda.synchronize()
    rH, rE = oracle.backward(x.H, x.segments, x.y, x.wl.V, dl, x.ignore_index)
    assert normwise(to_np(dH), rH) <= TOL_GRAD
    for g, r in zip(dEs, rE):
        assert normwise(to_np(g), r) <= TOL_GRAD
    assert np.all(to_np(dH)[~x.valid] == 0)


@pytest.mark.parametrize("case", ["gemma_like_small", "phi_like_small", "composite_small", "ragged",
                                  "peaky", "sparse_g", "sparse_g_segments"])
def test_backward_filtered_matches_oracle_and_criterion(data, case):
    x = data[case]
    H, segs, y, lse = _fwd_check(x)
    dl = x.dloss_mean()
    rows = min(64, x.wl.N)
    dH, dEs, keep = run_bwd(x, H, segs, y, lse, torch.from_numpy(dl).cuda(),
                            filter_eps=EPS_BF16, debug_rows=rows)
    torch.cuda.synchronize()
    rH, rE = oracle.backward(x.H, x.segments, x.y, x.wl.V, dl, x.ignore_index,
                             filter_eps=EPS_BF16)
    assert normwise(to_np(dH), rH) <= TOL_GRAD_FILTER
    for g, r in zip(dEs, rE):
        assert normwise(to_np(g), r) <= TOL_GRAD_FILTER
    # every filtered-out entry has oracle softmax < 2^-12; kept ones >= it
    P = oracle.softmax_rows(x.H, x.segments, x.wl.V, np.arange(rows))
    bits = keep.cpu().numpy().view(np.uint32)
    kept = np.unpackbits(bits.view(np.uint8), bitorder="little").reshape(rows, -1)[:, :x.wl.V]
    live = np.zeros(x.wl.V, bool)
    for b, e, _ in x.segments:
        live[b:e] = True
    valid = x.valid[:rows]
    dropped = (kept == 0) & live[None, :] & valid[:, None]
    assert np.all(P[dropped] < EPS_BF16)
    must_keep = (P >= EPS_BF16 * 1.001) & valid[:, None]
    assert np.all(kept[must_keep] == 1)
    assert np.all(kept[~valid] == 0)


def test_colmax_matches_oracle(data):
    x = data["composite_small"]
    H, segs, y = upload(x)
    loss, lse, colmax = run_fwd(x, H, segs, y, want_colmax=True)
    torch.cuda.synchronize()
    segs64 = [(b, e, oracle.widen_bf16(E)) for b, e, E in x.segments]
    Z = oracle.logits_rows(oracle.widen_bf16(x.H[x.valid]), segs64, x.wl.V)
    ref = np.concatenate([Z[:, b:e].max(0) for b, e, _ in x.segments])
    assert np.max(np.abs(to_np(colmax) - ref)) <= 1e-3


@pytest.mark.parametrize("keyed", ["colmax", "targets"])
def test_vocab_sort_and_permuted_backward(data, keyed):
    x = data["composite_small"]
    from linear_cross_entropy_cce_b200 import cce
    H, segs, y, lse = _fwd_check(x)
    colmax = run_fwd(x, H, segs, y, want_colmax=True)[2] if keyed == "colmax" else None
    perm = cce.vocab_sort(colmax, y, x.wl.V, x.ignore_index, segments=segs)
    torch.cuda.synchronize()
    p = perm.cpu().numpy()
    off = 0
    for b, e, _ in x.segments:
        n = e - b
        seg = p[off:off + n]
        assert np.array_equal(np.sort(seg), np.arange(n))
        key = (to_np(colmax)[off:off + n] if colmax is not None else
               np.bincount(x.y[(x.y >= b) & (x.y < e)] - b, minlength=n).astype(np.float64))
        k = key[seg]
        assert np.all(k[:-1] >= k[1:])
        ties = k[:-1] == k[1:]
        assert np.all(seg[:-1][ties] < seg[1:][ties])
        off += n
    dl = x.dloss_mean()
    dH, dEs, _ = run_bwd(x, H, segs, y, lse, torch.from_numpy(dl).cuda(), vocab_perm=perm,
                         filter_eps=EPS_BF16)
    rH, rE = oracle.backward(x.H, x.segments, x.y, x.wl.V, dl, x.ignore_index,
                             filter_eps=EPS_BF16)
    assert normwise(to_np(dH), rH) <= TOL_GRAD_FILTER
    for g, r in zip(dEs, rE):
        assert normwise(to_np(g), r) <= TOL_GRAD_FILTER


def _bf16_round(a: np.ndarray) -> np.ndarray:
    """fp64 -> the nearest bf16 value (via fp32), as an fp64 array."""
    return oracle.widen_bf16(syn.fp32_to_bf16_bits(a.astype(np.float32)))


def test_kahan_accumulation_beats_plain_bf16_and_is_deterministic():
    """dE accumulated over 128 micro-batches (8 batches cycled 16 times, one
    head): the plain bf16 running sum of the oracle's own parts drifts beyond
    the 1e-2 tolerance, while the GPU's Kahan pair (s, c) gives s - c within
    it and at least 4x closer to the exactly rounded sum; two runs agree bit
    for bit (each element has one owner thread)."""
    from linear_cross_entropy_cce_b200 import cce
    wl = syn.Workload("k", N=256, D=128, V=1024, logit_std=2.0, ignore_frac=0.1)
    xs = [syn.make_inputs(wl, seed=s) for s in range(8)]
    E = xs[0].segments  # the same head for every micro-batch
    K = 128
    Et = cce.bf16_from_bits(E[0][2], "cuda")
    dev = []
    for x in xs:
        H = cce.bf16_from_bits(x.H, "cuda")
        y = torch.from_numpy(x.y).cuda()
        _, lse = cce.fwd(H, Et, y)
        dev.append((H, y, lse, torch.from_numpy(x.dloss_mean()).cuda()))
    finals = []
    for rep in range(2):
        S = torch.zeros((wl.V, wl.D), dtype=torch.bfloat16, device="cuda")
        C = torch.zeros_like(S)
        for k in range(K):
            H, y, lse, dl = dev[k % 8]
            cce.bwd(H, Et, y, lse, dl, kahan=True, dE_out=S, dE_comp=C)
        torch.cuda.synchronize()
        finals.append((S.clone(), C.clone()))
    assert torch.equal(finals[0][0], finals[1][0]) and torch.equal(finals[0][1], finals[1][1])
    parts = [oracle.backward(x.H, E, x.y, wl.V, x.dloss_mean(), -100)[1][0] for x in xs]
    exact = oracle.kahan_reference([parts[k % 8] for k in range(K)])
    plain = np.zeros_like(exact)
    for k in range(K):  # bf16 storage, exact parts, rounded after every add
        plain = _bf16_round(plain + parts[k % 8])
    err_plain = normwise(plain, exact)
    S, C = finals[0]
    err_kahan = normwise(to_np(S) - to_np(C), exact)  # s - c is the compensated value
    assert err_plain > TOL_GRAD, err_plain
    assert err_kahan <= TOL_GRAD / 2, err_kahan
    assert err_plain >= 4 * err_kahan, (err_plain, err_kahan)


def test_fp32_grads(data):
    x = data["ragged"]
    H, segs, y, lse = _fwd_check(x)
    dl = x.dloss_mean()
    dH, dEs, _ = run_bwd(x, H, segs, y, lse, torch.from_numpy(dl).cuda(), fp32_grads=True)
    assert dH.dtype == torch.float32 and dEs[0].dtype == torch.float32
    rH, rE = oracle.backward(x.H, x.segments, x.y, x.wl.V, dl, x.ignore_index)
    assert normwise(to_np(dH), rH) <= TOL_GRAD / 2
    assert normwise(to_np(dEs[0]), rE[0]) <= TOL_GRAD / 2


def test_zero_head_gives_lnV():
    from linear_cross_entropy_cce_b200 import cce
    N, D, V = 300, 64, 5000
    H = torch.randn(N, D, device="cuda").to(torch.bfloat16)
    E = torch.zeros(V, D, device="cuda", dtype=torch.bfloat16)
    y = torch.randint(0, V, (N,), device="cuda", dtype=torch.int32)
    loss, lse = cce.fwd(H, E, y)
    assert torch.max(torch.abs(loss - math.log(V))).item() <= 1e-5
    assert torch.max(torch.abs(lse - math.log(V))).item() <= 1e-5


def test_bad_targets_set_status_and_nan():
    from linear_cross_entropy_cce_b200 import cce
    N, D, V = 200, 64, 700
    H = torch.randn(N, D, device="cuda").to(torch.bfloat16)
    EA = (torch.randn(300, D, device="cuda") * 0.1).to(torch.bfloat16)
    EB = (torch.randn(350, D, device="cuda") * 0.1).to(torch.bfloat16)
    segs = [(0, 300, EA), (350, 700, EB)]
    y = torch.randint(0, 300, (N,), device="cuda", dtype=torch.int32)
    y[3] = 320      # in the gap
    y[7] = 700      # out of range
    y[9] = -100     # ignored
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    loss, lse = cce.fwd(H, None, y, segments=segs, V=V, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & cce.STATUS_BADTARGET
    l = loss.cpu().numpy()
    assert math.isnan(l[3]) and math.isnan(l[7]) and l[9] == 0
    assert np.isfinite(np.delete(l, [3, 7])).all()
    dl = torch.full((N,), 1.0 / N, device="cuda")
    st.zero_()
    dH, dEs, _ = cce.bwd(H, None, y, lse, dl, segments=segs, V=V, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & cce.STATUS_BADTARGET
    d = dH.float().cpu().numpy()
    assert np.isnan(d[3]).all() and np.isnan(d[7]).all() and (d[9] == 0).all()
    assert np.isfinite(np.delete(d, [3, 7], axis=0)).all()
    assert all(torch.isfinite(g.float()).all() for g in dEs)


def test_all_rows_ignored():
    from linear_cross_entropy_cce_b200 import cce
    N, D, V = 130, 64, 600
    H = torch.randn(N, D, device="cuda").to(torch.bfloat16)
    E = torch.randn(V, D, device="cuda").to(torch.bfloat16)
    y = torch.full((N,), -100, device="cuda", dtype=torch.int32)
    loss, lse = cce.fwd(H, E, y)
    dH, dE, _ = cce.bwd(H, E, y, lse, torch.zeros(N, device="cuda"))
    torch.cuda.synchronize()
    assert (loss == 0).all() and (lse == 0).all()
    assert (dH.float() == 0).all() and (dE.float() == 0).all()


@pytest.mark.parametrize("eps", [0.0, EPS_BF16])
def test_segmented_head_equals_compact_head(data, eps):
    """A head with a dead gap equals the compact head [E_A; E_B] with the
    targets past the gap moved down by the gap width: the same logits, the
    gap contributing nothing (GPU against GPU, no oracle)."""
    from linear_cross_entropy_cce_b200 import cce
    x = data["composite_small"]
    H, segs, y = upload(x)
    (a0, a1, EA), (b0, b1, EB) = segs
    gap = b0 - a1
    E_c = torch.cat([EA, EB]).contiguous()
    y_c = torch.where(y >= b0, y - gap, y)
    loss_s, lse_s = run_fwd(x, H, segs, y)
    loss_c, lse_c = cce.fwd(H, E_c, y_c, x.ignore_index)
    dl = torch.from_numpy(x.dloss_mean()).cuda()
    dH_s, dE_s, _ = run_bwd(x, H, segs, y, lse_s, dl, filter_eps=eps, fp32_grads=True)
    dH_c, dE_c, _ = cce.bwd(H, E_c, y_c, lse_c, dl, x.ignore_index, filter_eps=eps,
                            fp32_grads=True)
    torch.cuda.synchronize()
    assert torch.max(torch.abs(lse_s - lse_c)).item() <= 1e-5
    assert torch.max(torch.abs(loss_s - loss_c)).item() <= 1e-5
    # filtered: the two layouts may route a chunk differently (bf16 slab on
    # the dense route, fp32 lists on the sparse one), so bf16-level agreement
    tol = 5e-3 if eps > 0 else 1e-5
    assert normwise(to_np(dH_s), to_np(dH_c)) <= tol
    assert normwise(to_np(dE_s[0]), to_np(dE_c[:a1 - a0])) <= tol
    assert normwise(to_np(dE_s[1]), to_np(dE_c[a1 - a0:])) <= tol


def test_empty_batch():
    """N = 0: every entry point returns at once with empty outputs."""
    from linear_cross_entropy_cce_b200 import cce
    H = torch.empty((0, 64), dtype=torch.bfloat16, device="cuda")
    E = torch.randn(300, 64, device="cuda").to(torch.bfloat16)
    y = torch.empty(0, dtype=torch.int32, device="cuda")
    loss, lse = cce.fwd(H, E, y)
    dH, dE, _ = cce.bwd(H, E, y, lse, torch.empty(0, device="cuda"))
    kl, ls, lt = cce.kl_fwd(H, E, H, E)
    torch.cuda.synchronize()
    assert loss.numel() == 0 and lse.numel() == 0 and dH.shape == (0, 64) and kl.numel() == 0


@pytest.mark.parametrize("N,D,V", [(5, 8, 1), (5, 8, 37), (131, 8, 256), (7, 24, 300)])
@pytest.mark.parametrize("eps", [0.0, EPS_BF16])
def test_degenerate_shapes(N, D, V, eps):
    """The smallest D (8, one 16-byte vector), a one-id vocabulary (loss 0,
    zero gradient), vocabularies below and exactly at one 256-wide tile."""
    wl = syn.Workload(f"deg{N}x{D}x{V}", N=N, D=D, V=V, logit_std=2.0, ignore_frac=0.2)
    x = syn.make_inputs(wl, seed=31)
    H, segs, y, lse = _fwd_check(x)
    dl = x.dloss_mean()
    dH, dEs, _ = run_bwd(x, H, segs, y, lse, torch.from_numpy(dl).cuda(), filter_eps=eps,
                         fp32_grads=True)
    torch.cuda.synchronize()
    rH, rE = oracle.backward(x.H, x.segments, x.y, V, dl, x.ignore_index, filter_eps=eps)
    if V == 1:
        assert np.max(np.abs(to_np(dH))) <= 1e-5 and np.max(np.abs(to_np(dEs[0]))) <= 1e-5
    else:
        tol = TOL_GRAD_FILTER if eps > 0 else TOL_GRAD
        assert normwise(to_np(dH), rH) <= tol
        assert normwise(to_np(dEs[0]), rE[0]) <= tol


def test_mispredicted_chunks_and_mixed_routes():
    """A filtered call whose vocabulary chunks alternate sparse / dense: with
    N = 512 (list capacity 4096 entries per 16384-id chunk), chunks 1 and 3
    hold 256 "hot" ids per row (every row's logit there is about 8 while the
    other ~65k logits are ~N(0, 1), so each hot entry keeps p ~ 3e-3 and the
    chunk holds 131k kept entries), chunks 0 and 2 keep almost nothing but the
    targets.  The backward predicts chunk 1 sparse from chunk 0 and must repair
    it with a second, dense launch; it predicts chunk 2 dense from chunk 1 (the
    slab is written) but takes the sparse route there; chunk 3 is mispredicted
    again.  dH then sums the dense chunks' accumulator with the sparse
    chunks' gathers.  Parity with the oracle, and every hot entry kept."""
    from linear_cross_entropy_cce_b200 import cce
    N, D, V = 512, 64, 4 * 16384
    rng = np.random.default_rng(11)
    H = rng.standard_normal((N, D)).astype(np.float32)
    H[:, 0] = 4.0
    E = (rng.standard_normal((V, D)) / np.sqrt(D)).astype(np.float32)
    E[:, 0] = 0.0
    hot = np.concatenate([np.arange(16384 + 1000, 16384 + 1256), np.arange(3 * 16384 + 77, 3 * 16384 + 333)])
    E[hot] = 0.01 * E[hot]
    E[hot, 0] = 2.0  # logit 8 for every row
    y = rng.integers(0, V, N).astype(np.int32)
    y[::9] = -100
    Hb, Eb = syn.fp32_to_bf16_bits(H), syn.fp32_to_bf16_bits(E)
    Hd, Ed = cce.bf16_from_bits(Hb, "cuda"), cce.bf16_from_bits(Eb, "cuda")
    yd = torch.from_numpy(y).cuda()
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    loss, lse = cce.fwd(Hd, Ed, yd, status=st)
    valid = y != -100
    dl = np.where(valid, 1.0 / valid.sum(), 0.0)
    dH, dE, keep = cce.bwd(Hd, Ed, yd, lse, torch.from_numpy(dl).float().cuda(),
                           filter_eps=EPS_BF16, debug_rows=N, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    rH, rE = oracle.backward(Hb, [(0, V, Eb)], y, V, dl, -100, filter_eps=EPS_BF16)
    assert normwise(to_np(dH), rH) <= TOL_GRAD_FILTER
    assert normwise(to_np(dE), rE[0]) <= TOL_GRAD_FILTER
    bits = keep.cpu().numpy().view(np.uint32)
    kept = np.unpackbits(bits.view(np.uint8), bitorder="little").reshape(N, -1)[:, :V].astype(bool)
    assert kept[np.ix_(valid, hot)].all()
    per_chunk = kept[valid].reshape(-1, 4, 16384).sum(axis=(0, 2))
    assert per_chunk[1] > 4096 and per_chunk[3] > 4096  # dense: beyond the list capacity
    assert per_chunk[0] < 1024 and per_chunk[2] < 1024  # sparse
    # the hot columns' dE rows are the large ones, and they are right
    assert normwise(to_np(dE)[hot], rE[0][hot]) <= TOL_GRAD_FILTER


@pytest.mark.parametrize("eps", [0.0, EPS_BF16])
def test_maximum_segment_count(eps):
    """CCE_MAX_SEGMENTS (8) segments: single-id segments, gaps of one id and
    of thousands, a segment ending at V; peaky logits so that filtered chunks
    take the sparse route, with the vocabulary sort and the tile skip.  The
    backward's workspace is sized for exactly 8 segments (each can add one
    partial chunk to the sparse lists)."""
    from linear_cross_entropy_cce_b200 import cce
    segs = ((0, 1), (5, 6), (100, 3000), (3001, 3002), (4000, 9000), (9100, 9101),
            (12000, 19000), (19999, 20000))
    wl = syn.Workload("max_segs", N=500, D=64, V=20000, logit_std=16.0, ignore_frac=0.1,
                      segments=segs, segment_mix=tuple(float(e - b) for b, e in segs))
    x = syn.make_inputs(wl, seed=41)
    H, dsegs, y = upload(x)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    loss, lse, colmax = run_fwd(x, H, dsegs, y, want_colmax=True, status=st)
    perm = cce.vocab_sort(colmax, y, wl.V, x.ignore_index, segments=list(segs))
    dl = x.dloss_mean()
    assert cce.bwd_workspace_size(wl.N, wl.D, wl.V, 8) > cce.bwd_workspace_size(wl.N, wl.D, wl.V, 1)
    dH, dEs, _ = run_bwd(x, H, dsegs, y, lse, torch.from_numpy(dl).cuda(), filter_eps=eps,
                         vocab_perm=perm if eps > 0 else None, colmax=colmax if eps > 0 else None,
                         status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    rl, rs = oracle.forward(x.H, x.segments, x.y, wl.V, x.ignore_index)
    assert np.max(np.abs(to_np(loss) - rl)) <= TOL_ROW
    assert np.max(np.abs(to_np(lse) - rs)) <= TOL_ROW
    rH, rE = oracle.backward(x.H, x.segments, x.y, wl.V, dl, x.ignore_index, filter_eps=eps)
    tol = TOL_GRAD_FILTER if eps > 0 else TOL_GRAD
    assert normwise(to_np(dH), rH) <= tol
    for g, r in zip(dEs, rE):
        got = to_np(g)
        assert got.shape == r.shape
        if np.any(r):
            assert normwise(got, r) <= tol
        else:
            assert np.max(np.abs(got)) <= 1e-6


@pytest.mark.parametrize("eps", [0.0, EPS_BF16])
def test_maximum_width(eps):
    """D = 65536, the largest row width the library accepts: 1024 K steps per
    tile in the tensor-core kernels and 16 passes over each row in the
    CUDA-core gathers of the sparse route (the filtered case)."""
    wl = syn.Workload("max_D", N=200, D=65536, V=700, logit_std=12.0, ignore_frac=0.1)
    x = syn.make_inputs(wl, seed=43)
    H, segs, y = upload(x)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    loss, lse = run_fwd(x, H, segs, y, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    rl, rs = oracle.forward(x.H, x.segments, x.y, wl.V, x.ignore_index)
    # Each logit is an fp32 sum of D bf16 products; its rounding error grows
    # as sqrt(D) for products of random sign, so the per-row tolerance (set
    # for D <= 4096) scales by sqrt(D / 4096) here.
    tol_row = TOL_ROW * math.sqrt(wl.D / 4096)
    assert np.max(np.abs(to_np(loss) - rl)) <= tol_row, np.max(np.abs(to_np(loss) - rl))
    assert np.max(np.abs(to_np(lse) - rs)) <= tol_row, np.max(np.abs(to_np(lse) - rs))
    dl = x.dloss_mean()
    dH, dEs, _ = run_bwd(x, H, segs, y, lse, torch.from_numpy(dl).cuda(), filter_eps=eps)
    torch.cuda.synchronize()
    rH, rE = oracle.backward(x.H, x.segments, x.y, wl.V, dl, x.ignore_index, filter_eps=eps)
    tol = TOL_GRAD_FILTER if eps > 0 else TOL_GRAD
    assert normwise(to_np(dH), rH) <= tol
    assert normwise(to_np(dEs[0]), rE[0]) <= tol


@pytest.mark.parametrize("N,D,V", [(300000, 16, 5), (3, 8, 3000000)])
@pytest.mark.parametrize("eps", [0.0, EPS_BF16])
def test_extreme_aspect_ratios(N, D, V, eps):
    """Very many rows over a tiny head (row compaction, scans and the row
    gathers at scale: 2344 row blocks) and a handful of rows over a very
    wide head (11719 vocabulary tiles, many backward chunks and list slots)."""
    wl = syn.Workload(f"aspect{N}x{V}", N=N, D=D, V=V, logit_std=3.0, ignore_frac=0.3)
    x = syn.make_inputs(wl, seed=47)
    H, segs, y, lse = _fwd_check(x)
    dl = x.dloss_mean()
    dH, dEs, _ = run_bwd(x, H, segs, y, lse, torch.from_numpy(dl).cuda(), filter_eps=eps)
    torch.cuda.synchronize()
    rH, rE = oracle.backward(x.H, x.segments, x.y, V, dl, x.ignore_index, filter_eps=eps)
    tol = TOL_GRAD_FILTER if eps > 0 else TOL_GRAD
    assert normwise(to_np(dH), rH) <= tol
    assert normwise(to_np(dEs[0]), rE[0]) <= tol
    assert np.all(to_np(dH)[~x.valid] == 0)


@pytest.mark.parametrize("ign", [7, -1])
def test_other_ignore_index_values(ign):
    """ignore_index is any int32: a valid vocabulary id (rows whose target is
    id 7 are then ignored, and id 7 gets no one-hot term) or another negative
    value (rows with -1 ignored).  Compared with the oracle called with the
    same ignore_index."""
    from linear_cross_entropy_cce_b200 import cce
    wl = syn.Workload("ign", N=400, D=64, V=300, logit_std=2.0, ignore_frac=0.0, targets="uniform")
    x = syn.make_inputs(wl, seed=51)
    y = x.y.copy()
    y[:40] = ign           # forty ignored rows
    if ign == 7:
        y[40:45] = 7       # more rows on id 7: ignored too
    Hd = cce.bf16_from_bits(x.H, "cuda")
    Ed = cce.bf16_from_bits(x.segments[0][2], "cuda")
    yd = torch.from_numpy(y).cuda()
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    loss, lse = cce.fwd(Hd, Ed, yd, ign, status=st)
    valid = y != ign
    dl = np.where(valid, 1.0 / valid.sum(), 0.0).astype(np.float32)
    dH, dE, _ = cce.bwd(Hd, Ed, yd, lse, torch.from_numpy(dl).cuda(), ign, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    rl, rs = oracle.forward(x.H, x.segments, y, wl.V, ign)
    assert np.max(np.abs(to_np(loss) - rl)) <= TOL_ROW
    assert np.all(to_np(loss)[~valid] == 0) and np.all(to_np(lse)[~valid] == 0)
    rH, rE = oracle.backward(x.H, x.segments, y, wl.V, dl, ign)
    assert normwise(to_np(dH), rH) <= TOL_GRAD
    assert normwise(to_np(dE), rE[0]) <= TOL_GRAD
    assert np.all(to_np(dH)[~valid] == 0)
