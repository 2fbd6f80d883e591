"""Parity at the full workload sizes, in every mode the benchmarks run them.

Cases: the Gemma-2-2B-shaped head with filtering and the vocabulary sort; the
Llama-3-8B-shaped head with filtering off, with filtering on, and with the
Kahan-compensated dE accumulation (two accumulations into a zeroed bf16 sum
and compensation); the Phi-3.5-mini-shaped head with filtering; the composite
two-segment head with filtering.

The oracle makes one full pass per workload (oracle.full_pass: every row's
loss and lse, and dE on sampled vocabulary rows, which need every row's lse).
With it:
  * loss and lse are compared on EVERY row, and the mean loss over all valid
    rows against the oracle's exactly rounded mean;
  * dH is compared on sampled rows (each oracle dH row is one D x V pass),
    including the first and last valid rows and rows of the last, ragged
    128-row block;
  * the filter criterion is checked per element on the sampled rows;
  * dE is checked on sampled vocabulary rows and through identities that hold
    at any size:  <dH, H>_F = <dE, E>_F  (both equal sum_ij G_ij z_ij) and,
    with filtering off, sum_j dE_j = 0 (every row of G sums to zero);
  * no buffer of the size class of the logits is ever allocated: every
    workspace is below N V 2 / 8 bytes, and the step allocates nothing beyond
    its workspaces and its outputs.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from linear_cross_entropy_cce_b200 import synthetic as syn
from _helpers import (EPS_BF16, TOL_GRAD, TOL_GRAD_FILTER, TOL_MEAN_REL, TOL_ROW, normwise,
                      to_np, upload)

pytestmark = pytest.mark.gpu

# (workload, filter on, vocabulary sort on, Kahan dE)
CASES = {
    "gemma2_2b_head-filter-sort": ("gemma2_2b_head", True, True, False),
    "llama3_8b_head-off": ("llama3_8b_head", False, False, False),
    "llama3_8b_head-filter": ("llama3_8b_head", True, False, False),
    "llama3_8b_head-kahan": ("llama3_8b_head", False, False, True),
    "phi35_mini_head-filter": ("phi35_mini_head", True, False, False),
    "composite_two_segment-filter": ("composite_two_segment", True, False, False),
}
KAHAN_STEPS = 2

_inputs = {}
_oracle = {}


def _workload_inputs(name):
    if name not in _inputs:
        _inputs.clear()  # one workload's inputs in host memory at a time
        _inputs[name] = syn.make_inputs(syn.WORKLOADS[name], seed=0)
    return _inputs[name]


def _sample_cols(x):
    rng = np.random.default_rng(2)
    live = np.concatenate([np.arange(b, e) for b, e, _ in x.segments])
    return np.unique(np.concatenate([rng.choice(live, 16, replace=False), x.y[x.valid][:8],
                                     [live[0], live[-1]]])).astype(np.int64)


def _oracle_full(name, x):
    """One oracle pass per workload: every row's loss/lse, dE columns for
    filtering off and on."""
    if name not in _oracle:
        _oracle.clear()
        cols = _sample_cols(x)
        loss, lse, dEc = oracle.full_pass(x.H, x.segments, x.y, x.wl.V, x.dloss_mean(), cols,
                                          x.ignore_index, filter_eps=(0.0, EPS_BF16),
                                          slice_rows=1024)
        _oracle[name] = dict(cols=cols, loss=loss, lse=lse, dEc=dEc)
    return _oracle[name]


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


def _nbytes(t):
    return 0 if t is None else t.numel() * t.element_size()


@pytest.fixture(scope="module", params=list(CASES))
def run(request):
    name, filt, sort, kahan = CASES[request.param]
    x = _workload_inputs(name)
    from linear_cross_entropy_cce_b200 import cce
    H, segs, y = upload(x)
    single = len(segs) == 1 and segs[0][0] == 0 and segs[0][1] == x.wl.V
    N, D, V = x.wl.N, x.wl.D, x.wl.V
    nseg = 0 if single else len(segs)
    rows = _sample_rows(x)
    dl = torch.from_numpy(x.dloss_mean()).cuda()
    eps = EPS_BF16 if filt else 0.0
    kahan_kw, S, C = {}, None, None
    if kahan:
        S = [torch.zeros_like(s[2]) for s in segs]
        C = [torch.zeros_like(s[2]) for s in segs]
        kahan_kw = dict(kahan=True, dE_out=S[0] if single else S, dE_comp=C[0] if single else C)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    base = torch.cuda.memory_allocated()
    torch.cuda.reset_peak_memory_stats()
    # caller-owned workspaces, so every byte of scratch is accounted for here
    ws_f = torch.empty(cce.fwd_workspace_size(N, D, V, nseg), dtype=torch.uint8, device="cuda")
    ws_b = torch.empty(cce.bwd_workspace_size(N, D, V, nseg, cce.KAHAN_DE if kahan else 0),
                       dtype=torch.uint8, device="cuda")
    ws_s = torch.empty(cce.vocab_sort_workspace_size(N, V, nseg), dtype=torch.uint8, device="cuda")
    seg_kw = {} if single else dict(segments=segs, V=V)
    E0 = segs[0][2] if single else None
    out = cce.fwd(H, E0, y, x.ignore_index, want_colmax=sort, workspace=ws_f, status=st, **seg_kw)
    loss, lse = out[0], out[1]
    perm = cm = None
    if sort:
        cm = out[2]
        perm = cce.vocab_sort(cm, y, V, x.ignore_index, segments=None if single else segs,
                              workspace=ws_s)
    calls = KAHAN_STEPS if kahan else 1
    for _ in range(calls):
        dH, dE, keep = cce.bwd(H, E0, y, lse, dl, x.ignore_index, filter_eps=eps, vocab_perm=perm,
                               colmax=cm, debug_rows=int(rows.max()) + 1 if filt else 0,
                               workspace=ws_b, status=st, **kahan_kw, **seg_kw)
    torch.cuda.synchronize()
    peak = torch.cuda.max_memory_allocated() - base
    dEs = dE if isinstance(dE, list) else [dE]
    # what the step itself allocates besides workspaces: its outputs (the
    # Kahan sum and compensation exist before the step; a second call's dH
    # coexists with the first one's until it is rebound)
    outputs = sum(_nbytes(t) for t in [loss, lse, cm, perm, keep]) + calls * _nbytes(dH)
    if not kahan:
        outputs += sum(_nbytes(t) for t in dEs)
    if kahan:  # s - c / steps: the compensated value of the accumulated gradient
        grads = [(to_np(s_) - to_np(c_)) / KAHAN_STEPS for s_, c_ in zip(S, C)]
    else:
        grads = [g.float().cpu().numpy() for g in dEs]  # fp32 copies (exact for bf16)
    # the same backward with fp32 gradients (CCE_FP32_GRADS), for the
    # inner-product identity: rounded to bf16, a gradient element whose
    # one-hot part (-dloss e_y in dH, -dloss h_i in dE) is exactly
    # representable (dloss = 2^-14 on the Llama-shaped head) swallows every
    # kept softmax contribution below half an ulp of it, so bf16 gradients no
    # longer show the kept part of sum_ij G_ij z_ij, which nearly cancels the
    # one-hot part on the filtered flat-softmax head
    dH32, dE32, _ = cce.bwd(H, E0, y, lse, dl, x.ignore_index, filter_eps=eps, vocab_perm=perm,
                            colmax=cm, fp32_grads=True, **seg_kw)
    torch.cuda.synchronize()
    dH32 = to_np(dH32)
    dE32 = [g.cpu().numpy() for g in (dE32 if isinstance(dE32, list) else [dE32])]
    res = dict(x=x, name=name, filt=filt, eps=eps, rows=rows, status=int(st.item()),
               loss=to_np(loss), lse=to_np(lse), dH=to_np(dH), dH32=dH32, dE32=dE32, dEs=grads,
               keep=keep.cpu().numpy().view(np.uint32) if keep is not None else None,
               ws=[_nbytes(w) for w in (ws_f, ws_b, ws_s)], peak=peak, outputs=outputs)
    del H, segs, y, dH, dE, dEs, keep, loss, lse, out, S, C, ws_f, ws_b, ws_s, cm, perm
    torch.cuda.empty_cache()
    yield res


def test_no_logit_sized_buffer(run):
    """Nothing of the size class of the [N, V] logits is allocated: the
    buffers of the backward's workspace that hold parts of the product (the
    G slab of one vocabulary chunk and the sparse lists,
    cce_bwd_workspace_parts "logits") stay below N V 2 / 8 bytes, an eighth
    of the bf16 logits; the rest of the scratch scales with the inputs (N x D
    rows, chunk x D rows of E), and the step's peak allocation is its
    workspaces plus its outputs (so no hidden allocation exists either)."""
    from linear_cross_entropy_cce_b200 import cce
    x = run["x"]
    wl = x.wl
    bound = wl.N * wl.V * 2 / 8
    nseg = 0 if len(wl.segs()) == 1 else len(wl.segs())
    parts = cce.bwd_workspace_parts(wl.N, wl.D, wl.V, nseg, 0)  # Kahan needs no more scratch
    assert sum(parts.values()) == run["ws"][1]
    assert parts["logits"] < bound, (parts, bound)
    assert run["ws"][0] < bound and run["ws"][2] < bound  # forward and sort scratch
    slack = 8 << 20  # allocator rounding and a few small tensors (dloss, status)
    assert run["peak"] <= sum(run["ws"]) + run["outputs"] + slack, (run["peak"], run["ws"],
                                                                     run["outputs"])


def test_forward_every_row_and_exact_mean(run):
    x = run["x"]
    assert run["status"] == 0
    o = _oracle_full(run["name"], x)
    v = x.valid
    assert np.max(np.abs(run["loss"][v] - o["loss"][v])) <= TOL_ROW
    assert np.max(np.abs(run["lse"][v] - o["lse"][v])) <= TOL_ROW
    assert np.all(run["loss"][~v] == 0) and np.all(run["lse"][~v] == 0)
    m_ref = oracle.mean_loss(o["loss"], v)
    m_got = math.fsum(run["loss"][v].tolist()) / int(v.sum())
    assert abs(m_got - m_ref) <= TOL_MEAN_REL * abs(m_ref), (m_got, m_ref)


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
    """<a, b>_F in fp64, chunked over rows (a fp32 or fp64, b bf16 bits)."""
    acc = 0.0
    for r in range(0, a32.shape[0], chunk):
        acc += float(np.sum(a32[r:r + chunk].astype(np.float64) * oracle.widen_bf16(b_bits[r:r + chunk])))
    return acc


def test_dE_identities(run):
    x = run["x"]
    # both sides from the fp32-gradient pass (see the fixture); the dE of the
    # benchmark configuration is checked on sampled columns and below
    lhs = float(np.sum(run["dH32"] * oracle.widen_bf16(x.H)))
    rhs = sum(_frob_dot(g, E) for g, (_, _, E) in zip(run["dE32"], x.segments))
    scale = max(abs(lhs), 1e-30)
    assert abs(lhs - rhs) <= 2e-2 * scale + 1e-6, (lhs, rhs)
    if not run["filt"]:
        colsum = sum(g.astype(np.float64).sum(0) for g in run["dEs"])
        fro = np.sqrt(sum(float(np.sum(np.square(g, dtype=np.float64))) for g in run["dEs"]))
        assert np.linalg.norm(colsum) <= 1e-2 * fro


def test_dE_sampled_vocab_rows(run):
    x = run["x"]
    o = _oracle_full(run["name"], x)
    cols = o["cols"]
    ref = o["dEc"][run["eps"]]
    got = np.zeros_like(ref)
    for k, c in enumerate(cols):  # logical id -> (segment, local row)
        for (b, e, _), g in zip(x.segments, run["dEs"]):
            if b <= c < e:
                got[k] = g[c - b]
    tol = TOL_GRAD_FILTER if run["filt"] else TOL_GRAD
    assert normwise(got, ref) <= tol
