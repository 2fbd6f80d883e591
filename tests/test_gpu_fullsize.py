"""Parity at the full workload sizes, in the configuration bench.py times.

The oracle cannot afford every output at these sizes, so:
  * loss, lse and dH are compared on sampled rows (each oracle row is one
    D x V pass), including the first row, the last row and rows of the last,
    ragged 128-row block;
  * the filter criterion is checked per element on sampled rows;
  * dE is checked through identities that hold at any size:
      <dH, H>_F = <dE, E>_F   (both equal sum_ij G_ij z_ij), and, with
      filtering off, sum_j dE_j = 0 (every row of G sums to zero);
    and against the oracle on sampled vocabulary rows of E (that needs every
    row's lse: one full oracle pass over the workload, seconds to a minute of
    fp64 BLAS on the host).
"""
import numpy as np
import pytest
import torch

import oracle
from linear_cross_entropy_cce_b200 import synthetic as syn
from _helpers import (EPS_BF16, TOL_GRAD, TOL_GRAD_FILTER, TOL_MEAN_REL, TOL_ROW, normwise,
                      run_bwd, run_fwd, to_np, upload)

pytestmark = pytest.mark.gpu

# (filter on, vocabulary sort on): the bench configuration of each workload
MODES = {
    "gemma2_2b_head": (True, True),
    "llama3_8b_head": (False, False),
    "phi35_mini_head": (True, False),
    "composite_two_segment": (True, False),
}


def _sample_rows(x, k=24, seed=1):
    valid = np.nonzero(x.valid)[0]
    rng = np.random.default_rng(seed)
    pick = set(rng.choice(valid, size=min(k, len(valid)), replace=False).tolist())
    pick |= {int(valid[0]), int(valid[-1])}
    pick |= set(valid[valid >= (x.wl.N // 128) * 128][:4].tolist())  # ragged last block
    ign = np.nonzero(~x.valid)[0]
    if len(ign):
        pick.add(int(ign[0]))
    return np.array(sorted(pick))


@pytest.fixture(scope="module", params=list(MODES))
def run(request):
    name = request.param
    x = syn.make_inputs(syn.WORKLOADS[name], seed=0)
    filt, sort = MODES[name]
    from linear_cross_entropy_cce_b200 import cce
    H, segs, y = upload(x)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = run_fwd(x, H, segs, y, want_colmax=sort, status=st)
    loss, lse = out[0], out[1]
    perm = None
    if sort:
        single = len(segs) == 1
        perm = cce.vocab_sort(out[2], y, x.wl.V, x.ignore_index, segments=None if single else segs)
    rows = _sample_rows(x)
    dl = x.dloss_mean()
    eps = EPS_BF16 if filt else 0.0
    dH, dEs, keep = run_bwd(x, H, segs, y, lse, torch.from_numpy(dl).cuda(), filter_eps=eps,
                            vocab_perm=perm, debug_rows=int(rows.max()) + 1, status=st)
    torch.cuda.synchronize()
    res = dict(x=x, filt=filt, eps=eps, rows=rows, status=int(st.item()),
               loss=to_np(loss), lse=to_np(lse), dH=to_np(dH),
               dEs=[g.float().cpu().numpy() for g in dEs],  # fp32 copies (exact for bf16)
               keep=keep.cpu().numpy().view(np.uint32) if keep is not None else None)
    del H, segs, y, dH, dEs, keep, loss, lse
    torch.cuda.empty_cache()
    yield res


def test_forward_sampled_rows(run):
    x, rows = run["x"], run["rows"]
    assert run["status"] == 0
    rl, rs = oracle.forward(x.H, x.segments, x.y, x.wl.V, x.ignore_index, rows=rows)
    gl, gs = run["loss"][rows], run["lse"][rows]
    assert np.max(np.abs(gl - rl)) <= TOL_ROW
    assert np.max(np.abs(gs - rs)) <= TOL_ROW
    v = x.valid[rows]
    assert abs(gl[v].mean() - rl[v].mean()) <= TOL_MEAN_REL * abs(rl[v].mean())
    assert np.all(run["loss"][~x.valid] == 0)


def test_dH_sampled_rows_and_filter_criterion(run):
    x, rows = run["x"], run["rows"]
    dl = x.dloss_mean()
    sub = syn.Inputs(x.wl, x.H[rows], x.segments, x.y[rows])
    rH, _ = oracle.backward(sub.H, x.segments, sub.y, x.wl.V, dl[rows], x.ignore_index,
                            filter_eps=run["eps"])
    tol = TOL_GRAD_FILTER if run["filt"] else TOL_GRAD
    assert normwise(run["dH"][rows], rH) <= tol
    # per-element filter criterion on the sampled rows
    if run["filt"]:
        P = oracle.softmax_rows(x.H, x.segments, x.wl.V, rows)
        bits = run["keep"][rows]
        kept = np.unpackbits(bits.view(np.uint8), bitorder="little").reshape(len(rows), -1)[:, :x.wl.V]
        live = np.zeros(x.wl.V, bool)
        for b, e, _ in x.segments:
            live[b:e] = True
        v = x.valid[rows]
        dropped = (kept == 0) & live[None, :] & v[:, None]
        assert np.all(P[dropped] < EPS_BF16)
        assert np.all(kept[(P >= EPS_BF16 * 1.001) & v[:, None]] == 1)


def _frob_dot(a32, b_bits, chunk=1 << 14):
    """<a, b>_F in fp64, chunked over rows (a fp32, b bf16 bits)."""
    acc = 0.0
    for r in range(0, a32.shape[0], chunk):
        acc += float(np.sum(a32[r:r + chunk].astype(np.float64) * oracle.widen_bf16(b_bits[r:r + chunk])))
    return acc


def test_dE_identities(run):
    x = run["x"]
    lhs = float(np.sum(run["dH"] * oracle.widen_bf16(x.H)))
    rhs = sum(_frob_dot(g, E) for g, (_, _, E) in zip(run["dEs"], x.segments))
    scale = max(abs(lhs), 1e-30)
    assert abs(lhs - rhs) <= 2e-2 * scale + 1e-6, (lhs, rhs)
    if not run["filt"]:
        colsum = sum(g.astype(np.float64).sum(0) for g in run["dEs"])
        fro = np.sqrt(sum(float(np.sum(np.square(g, dtype=np.float64))) for g in run["dEs"]))
        assert np.linalg.norm(colsum) <= 1e-2 * fro


def test_dE_sampled_vocab_rows(run):
    x = run["x"]
    rng = np.random.default_rng(2)
    live = np.concatenate([np.arange(b, e) for b, e, _ in x.segments])
    cols = np.unique(np.concatenate([rng.choice(live, 16, replace=False), x.y[x.valid][:8],
                                     [live[0], live[-1]]])).astype(np.int64)
    ref = oracle.dE_columns(x.H, x.segments, x.y, x.wl.V, x.dloss_mean(), cols,
                            x.ignore_index, filter_eps=run["eps"], slice_rows=1024)
    got = np.zeros_like(ref)
    for k, c in enumerate(cols):  # logical id -> (segment, local row)
        for (b, e, _), g in zip(x.segments, run["dEs"]):
            if b <= c < e:
                got[k] = g[c - b]
    tol = TOL_GRAD_FILTER if run["filt"] else TOL_GRAD
    assert normwise(got, ref) <= tol
