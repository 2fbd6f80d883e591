"""Guard-byte (canary) checks: every buffer a call writes (outputs, debug
masks, workspace) sits inside a larger allocation whose bytes before and after
it hold a known pattern; after the call those guard bytes must be unchanged.
Shapes are ragged (N, D and V not multiples of any tile) so that the tails of
every kernel's index arithmetic are exercised; the calls go through the C ABI
with caller-owned buffers, as a C user would make them."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from linear_cross_entropy_cce_b200 import cce, synthetic as syn
from _helpers import EPS_BF16, TOL_GRAD, TOL_GRAD_FILTER, normwise, to_np

pytestmark = pytest.mark.gpu

GUARD = 64 << 10  # bytes of pattern on each side (a multiple of 256: keeps alignment)
PATTERN = 0xA5


class Guarded:
    """Buffers carved out of patterned allocations, checked after a call."""

    def __init__(self):
        self.bufs = []

    def alloc(self, shape, dtype, zero=False):
        n = int(np.prod(shape)) * torch.empty(0, dtype=dtype).element_size()
        n_al = (n + 255) // 256 * 256
        raw = torch.full((GUARD + n_al + GUARD,), PATTERN, dtype=torch.uint8, device="cuda")
        mid = raw[GUARD:GUARD + n]
        if zero:
            mid.zero_()
        t = mid.view(dtype).view(shape) if n else torch.empty(shape, dtype=dtype, device="cuda")
        self.bufs.append((raw, n))
        return t

    def check(self):
        torch.cuda.synchronize()
        for raw, n in self.bufs:
            head = raw[:GUARD]
            tail = raw[GUARD + n:]
            assert bool((head == PATTERN).all()), "bytes before a buffer were written"
            assert bool((tail == PATTERN).all()), "bytes after a buffer were written"


def _p(t):
    return None if t is None else t.data_ptr()


def _stream():
    return torch.cuda.current_stream().cuda_stream


def _segarr(segs, dEs=None, comps=None):
    arr = (cce.Segment * len(segs))()
    for k, (b, e, E) in enumerate(segs):
        arr[k].vocab_begin, arr[k].vocab_end, arr[k].E = b, e, E.data_ptr()
        arr[k].dE = dEs[k].data_ptr() if dEs is not None else None
        arr[k].dE_comp = comps[k].data_ptr() if comps is not None else None
    return arr


HEADS = {
    "single": syn.Workload("canary_single", N=333, D=200, V=1000, logit_std=4.0, ignore_frac=0.15),
    "composite": syn.Workload("canary_comp", N=389, D=136, V=2100, logit_std=8.0, ignore_frac=0.2,
                              segments=((0, 1150), (1203, 2100)), segment_mix=(0.6, 0.4)),
}
MODES = {  # (filter_eps, flags, sort)
    "plain": (0.0, 0, False),
    "filter": (EPS_BF16, 0, True),
    "kahan": (0.0, cce.KAHAN_DE, False),
    "fullc": (EPS_BF16, cce.FULL_DE, False),
    "fp32": (EPS_BF16, cce.FP32_GRADS, False),
    "fp32_dh": (0.0, cce.FP32_DH, False),
}


@pytest.mark.parametrize("mode", list(MODES))
@pytest.mark.parametrize("head", list(HEADS))
def test_forward_and_backward_write_only_their_buffers(head, mode):
    L = cce.lib()
    wl = HEADS[head]
    x = syn.make_inputs(wl, seed=31)
    eps, flags, sort = MODES[mode]
    g = Guarded()
    N, D, V = wl.N, wl.D, wl.V
    composite = head == "composite"
    H = g.alloc((N, D), torch.bfloat16)
    H.view(torch.int16).copy_(torch.from_numpy(x.H.view(np.int16)))
    segs = []
    for b, e, E in x.segments:
        t = g.alloc((e - b, D), torch.bfloat16)
        t.view(torch.int16).copy_(torch.from_numpy(E.view(np.int16)))
        segs.append((b, e, t))
    y = g.alloc((N,), torch.int32)
    y.copy_(torch.from_numpy(x.y))
    nseg = len(segs) if composite else 0
    v_live = wl.v_live
    loss, lse = g.alloc((N,), torch.float32), g.alloc((N,), torch.float32)
    colmax = g.alloc((v_live,), torch.float32)
    st = g.alloc((1,), torch.int32, zero=True)
    ws_f = g.alloc((L.cce_fwd_workspace_size(N, D, V, nseg),), torch.uint8)
    E0 = None if composite else segs[0][2]
    arr = _segarr(segs) if composite else None
    rc = L.cce_fwd(_p(H), _p(E0), _p(y), N, D, V, x.ignore_index, arr, nseg, _p(loss), _p(lse),
                   _p(colmax), _p(ws_f), ws_f.numel(), _p(st), _stream())
    assert rc == 0
    perm = None
    if sort:
        perm = g.alloc((v_live,), torch.int32)
        ws_s = g.alloc((L.cce_vocab_sort_workspace_size(N, V, nseg),), torch.uint8)
        rc = L.cce_vocab_sort(_p(colmax), _p(y), N, V, x.ignore_index, arr, nseg, _p(perm),
                              _p(ws_s), ws_s.numel(), _stream())
        assert rc == 0
    fp32_de = bool(flags & cce.FP32_GRADS)
    fp32_dh = fp32_de or bool(flags & cce.FP32_DH)
    dH = g.alloc((N, D), torch.float32 if fp32_dh else torch.bfloat16)
    dEs = [g.alloc((e - b, D), torch.float32 if fp32_de else torch.bfloat16,
                   zero=bool(flags & cce.KAHAN_DE)) for b, e, _ in segs]
    comps = [g.alloc((e - b, D), torch.bfloat16, zero=True) for b, e, _ in segs] \
        if flags & cce.KAHAN_DE else None
    dbg_rows = N
    keep = g.alloc((dbg_rows, (V + 31) // 32), torch.int32) if eps > 0 else None
    dl = g.alloc((N,), torch.float32)
    dl.copy_(torch.from_numpy(x.dloss_mean()))
    ws_b = g.alloc((L.cce_bwd_workspace_size(N, D, V, nseg, flags),), torch.uint8)
    arr_b = _segarr(segs, dEs, comps) if composite else None
    rc = L.cce_bwd(_p(H), _p(E0), _p(y), _p(lse), _p(dl), N, D, V, x.ignore_index, arr_b, nseg,
                   float(eps), _p(perm), _p(colmax) if sort else None, flags, _p(dH),
                   None if composite else _p(dEs[0]),
                   None if (composite or comps is None) else _p(comps[0]),
                   _p(keep), dbg_rows if keep is not None else 0, _p(ws_b), ws_b.numel(), _p(st),
                   _stream())
    assert rc == 0
    g.check()
    assert int(st.item()) == 0
    # and the results are right
    rH, rE = oracle.backward(x.H, x.segments, x.y, V, x.dloss_mean(), x.ignore_index,
                             filter_eps=eps, filter_dE=not (flags & cce.FULL_DE))
    tol = TOL_GRAD_FILTER if eps > 0 else TOL_GRAD
    assert normwise(to_np(dH), rH) <= tol
    for k, r in enumerate(rE):
        got = to_np(dEs[k]) - (to_np(comps[k]) if comps is not None else 0.0)
        assert normwise(got, r) <= tol


@pytest.mark.parametrize("eps", [0.0, EPS_BF16])
def test_soft_target_kl_writes_only_its_buffers(eps):
    L = cce.lib()
    N, D, V = 299, 136, 1700
    rng = np.random.default_rng(4)
    g = Guarded()

    def bf(a):
        t = g.alloc(a.shape, torch.bfloat16)
        t.view(torch.int16).copy_(torch.from_numpy(syn.fp32_to_bf16_bits(a).view(np.int16)))
        return t
    Hs_h = rng.standard_normal((N, D)).astype(np.float32)
    Ht_h = rng.standard_normal((N, D)).astype(np.float32)
    E_h = (rng.standard_normal((V, D)) * 6.0 / np.sqrt(D)).astype(np.float32)
    Hs, Ht, E = bf(Hs_h), bf(Ht_h), bf(E_h)
    mask = g.alloc((N,), torch.int32)
    mask.copy_(torch.from_numpy((np.arange(N) % 7 != 3).astype(np.int32)))
    kl, ls, lt = (g.alloc((N,), torch.float32) for _ in range(3))
    st = g.alloc((1,), torch.int32, zero=True)
    ws_f = g.alloc((L.cce_kl_fwd_workspace_size(N, D, V),), torch.uint8)
    rc = L.cce_kl_fwd(_p(Hs), _p(E), _p(Ht), _p(E), _p(mask), N, D, V, _p(kl), _p(ls), _p(lt),
                      _p(ws_f), ws_f.numel(), _p(st), _stream())
    assert rc == 0
    dl = g.alloc((N,), torch.float32)
    dl.fill_(1.0 / N)
    dH = g.alloc((N, D), torch.bfloat16)
    dE = g.alloc((V, D), torch.bfloat16)
    ws_b = g.alloc((L.cce_kl_bwd_workspace_size(N, D, V, 0),), torch.uint8)
    keep = g.alloc((N, (V + 31) // 32), torch.int32) if eps > 0 else None
    rc = L.cce_kl_bwd(_p(Hs), _p(E), _p(Ht), _p(E), _p(mask), _p(ls), _p(lt), _p(dl), N, D, V,
                      float(eps), 0, _p(dH), _p(dE), None, _p(keep), N if keep is not None else 0,
                      _p(ws_b), ws_b.numel(), _p(st), _stream())
    assert rc == 0
    g.check()
    assert int(st.item()) == 0
    bits = lambda a: syn.fp32_to_bf16_bits(a)  # noqa: E731
    m = mask.cpu().numpy()
    rkl, _, _ = oracle.kl_forward(bits(Hs_h), bits(E_h), bits(Ht_h), bits(E_h), row_mask=m)
    assert np.max(np.abs(to_np(kl) - rkl)) <= 2e-3
    rH, rE = oracle.kl_backward(bits(Hs_h), bits(E_h), bits(Ht_h), bits(E_h), np.full(N, 1.0 / N),
                                row_mask=m, filter_eps=eps)
    tol = TOL_GRAD_FILTER if eps > 0 else TOL_GRAD
    assert normwise(to_np(dH), rH) <= tol and normwise(to_np(dE), rE) <= tol


def test_combine_and_noalloc_forward_write_only_their_buffers():
    L = cce.lib()
    wl = HEADS["composite"]
    x = syn.make_inputs(wl, seed=32)
    g = Guarded()
    N, D, V = wl.N, wl.D, wl.V
    R = 3
    parts = g.alloc((R, 2, N), torch.float32)
    parts.copy_(torch.randn(R, 2, N))
    y = g.alloc((N,), torch.int32)
    y.copy_(torch.from_numpy(x.y))
    loss, lse = g.alloc((N,), torch.float32), g.alloc((N,), torch.float32)
    arr = (cce.Segment * 2)()
    for k, (b, e) in enumerate(wl.segs()):
        arr[k].vocab_begin, arr[k].vocab_end = b, e
    assert L.cce_vocab_combine(_p(parts), R, _p(y), N, V, x.ignore_index, arr, 2, _p(loss),
                               _p(lse), _stream()) == 0
    # the allocation-free forward on the same guarded inputs
    H = g.alloc((N, D), torch.bfloat16)
    H.view(torch.int16).copy_(torch.from_numpy(x.H.view(np.int16)))
    segs = []
    for b, e, E in x.segments:
        t = g.alloc((e - b, D), torch.bfloat16)
        t.view(torch.int16).copy_(torch.from_numpy(E.view(np.int16)))
        segs.append((b, e, t))
    st = g.alloc((1,), torch.int32, zero=True)
    f = L.cce_fwd_noalloc
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                  ctypes.c_int64, ctypes.c_int32, ctypes.POINTER(cce.Segment), ctypes.c_int32,
                  ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                  ctypes.c_void_p]
    colmax = g.alloc((wl.v_live,), torch.float32)
    assert f(_p(H), None, _p(y), N, D, V, x.ignore_index, _segarr(segs), 2, _p(loss), _p(lse),
             _p(colmax), _p(st), _stream()) == 0
    g.check()
    assert int(st.item()) == 0
