"""ctypes binding of libcce (argument marshalling only).

Every step of the computation runs in libcce.so's CUDA kernels; torch is used
for device memory, the current stream and dtype bookkeeping.  There is no CPU
fallback: if the library is missing or no sm_100 GPU is present the calls
raise.
"""
from __future__ import annotations

import ctypes
import os
from typing import List, Optional, Sequence, Tuple

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libcce.so")

CCE_OK, CCE_EINVAL, CCE_EWORKSPACE, CCE_ELAUNCH, CCE_EDEVICE = 0, 1, 2, 3, 4
STATUS_BADTARGET, STATUS_TIMEOUT = 1, 2
KAHAN_DE, FP32_GRADS, FULL_DE, VOCAB_SHARD, FP32_DH = 1, 2, 4, 8, 16
MAX_SEGMENTS = 8

EXPORTS = ("cce_version", "cce_strerror", "cce_fwd_workspace_size", "cce_fwd", "cce_fwd_shard",
           "cce_bwd_workspace_size", "cce_bwd", "cce_vocab_sort_workspace_size",
           "cce_vocab_sort", "cce_launch_count", "cce_timing_enable", "cce_timing_read",
           "cce_kl_fwd_workspace_size", "cce_kl_fwd", "cce_kl_bwd_workspace_size", "cce_kl_bwd",
           "cce_vocab_combine", "cce_fwd_noalloc", "cce_debug_stall",
           "cce_debug_stall_pair", "cce_bwd_workspace_parts")
# kernel classes for cce_timing_enable / cce_timing_read
KC_FWD, KC_G, KC_DE, KC_DH, KC_AUX, KC_SPARSE = 0, 1, 2, 3, 4, 5
KC_NAMES = ("fwd_tile_stream", "bwd_g_producer", "bwd_dE_contraction", "bwd_dH_contraction", "aux",
            "bwd_sparse")


class CCEError(RuntimeError):
    pass


class Segment(ctypes.Structure):
    _fields_ = [("vocab_begin", ctypes.c_int64), ("vocab_end", ctypes.c_int64),
                ("E", ctypes.c_void_p), ("dE", ctypes.c_void_p), ("dE_comp", ctypes.c_void_p)]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libcce.so (built in-tree by ``linear_cross_entropy_cce_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise CCEError(f"libcce.so not found at {LIB_PATH}; build it with "
                       "`python -m linear_cross_entropy_cce_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    i64, i32, u32, vp, sz, fp = (ctypes.c_int64, ctypes.c_int32, ctypes.c_uint32, ctypes.c_void_p,
                                 ctypes.c_size_t, ctypes.c_float)
    L.cce_version.restype = ctypes.c_int
    L.cce_strerror.restype = ctypes.c_char_p
    L.cce_strerror.argtypes = [ctypes.c_int]
    L.cce_fwd_workspace_size.restype = sz
    L.cce_fwd_workspace_size.argtypes = [i64, i64, i64, i32]
    L.cce_fwd.restype = ctypes.c_int
    L.cce_fwd.argtypes = [vp, vp, vp, i64, i64, i64, i32, ctypes.POINTER(Segment), i32,
                          vp, vp, vp, vp, sz, vp, vp]
    L.cce_fwd_shard.restype = ctypes.c_int
    L.cce_fwd_shard.argtypes = L.cce_fwd.argtypes
    L.cce_kl_fwd_workspace_size.restype = sz
    L.cce_kl_fwd_workspace_size.argtypes = [i64, i64, i64]
    L.cce_kl_fwd.restype = ctypes.c_int
    L.cce_kl_fwd.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, vp, vp, vp, vp, sz, vp, vp]
    L.cce_kl_bwd_workspace_size.restype = sz
    L.cce_kl_bwd_workspace_size.argtypes = [i64, i64, i64, u32]
    L.cce_kl_bwd.restype = ctypes.c_int
    L.cce_kl_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i64, i64, i64, fp, u32, vp, vp, vp,
                             vp, i64, vp, sz, vp, vp]
    L.cce_bwd_workspace_size.restype = sz
    L.cce_bwd_workspace_size.argtypes = [i64, i64, i64, i32, u32]
    L.cce_bwd_workspace_parts.restype = ctypes.c_int
    L.cce_bwd_workspace_parts.argtypes = [i64, i64, i64, i32, u32, ctypes.POINTER(sz),
                                          ctypes.POINTER(sz), ctypes.POINTER(sz)]
    L.cce_bwd.restype = ctypes.c_int
    L.cce_bwd.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i32, ctypes.POINTER(Segment), i32,
                          fp, vp, vp, u32, vp, vp, vp, vp, i64, vp, sz, vp, vp]
    L.cce_vocab_sort_workspace_size.restype = sz
    L.cce_vocab_sort_workspace_size.argtypes = [i64, i64, i32]
    L.cce_vocab_sort.restype = ctypes.c_int
    L.cce_vocab_sort.argtypes = [vp, vp, i64, i64, i32, ctypes.POINTER(Segment), i32, vp, vp, sz, vp]
    L.cce_vocab_combine.restype = ctypes.c_int
    L.cce_vocab_combine.argtypes = [vp, i32, vp, i64, i64, i32, ctypes.POINTER(Segment), i32,
                                    vp, vp, vp]
    L.cce_debug_stall.restype = ctypes.c_int
    L.cce_debug_stall.argtypes = [ctypes.c_uint64, vp, vp]
    L.cce_debug_stall_pair.restype = ctypes.c_int
    L.cce_debug_stall_pair.argtypes = [ctypes.c_uint64, vp, vp]
    L.cce_launch_count.restype = ctypes.c_uint64
    L.cce_timing_enable.restype = ctypes.c_int
    L.cce_timing_enable.argtypes = [u32]
    L.cce_timing_read.restype = ctypes.c_int
    L.cce_timing_read.argtypes = [ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_int64), i32]
    _lib = L
    return L


def _check(rc: int, what: str):
    if rc != CCE_OK:
        raise CCEError(f"{what}: {lib().cce_strerror(rc).decode()} (code {rc})")


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream_ptr(device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _require_cuda(*ts: torch.Tensor):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise CCEError("all tensors must be contiguous CUDA tensors")


SegSpec = Tuple[int, int, torch.Tensor]  # (vocab_begin, vocab_end, E_s)


def _expect(t: Optional[torch.Tensor], name: str, dtype, shape):
    """The C ABI takes bare pointers and trusts the sizes it is given, so a
    tensor of the wrong type or shape would be read or written out of
    bounds: refuse it here."""
    if t is None:
        return
    if t.dtype != dtype:
        raise CCEError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise CCEError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _expect_status(st: Optional[torch.Tensor]):
    if st is not None and (st.dtype != torch.int32 or st.numel() < 1):
        raise CCEError("status must be an int32 tensor of at least one element")


def _rows(H: torch.Tensor, name: str = "H") -> Tuple[int, int]:
    if H.dim() != 2 or H.dtype != torch.bfloat16:
        raise CCEError(f"{name} must be a 2-D bfloat16 tensor, got {H.dtype} {tuple(H.shape)}")
    return int(H.shape[0]), int(H.shape[1])


def _check_head(E: Optional[torch.Tensor], segments, D: int):
    """E [V, D] bf16, or each segment's E_s [end - begin, D] bf16."""
    if segments:
        for k, s in enumerate(segments):
            b, e = int(s[0]), int(s[1])
            if e <= b:
                raise CCEError(f"segment {k} is empty or reversed: [{b}, {e})")
            if len(s) > 2:
                _expect(s[2], f"segment {k} E", torch.bfloat16, (e - b, D))
    elif E is None:
        raise CCEError("E is required when no segments are given")
    else:
        _expect(E, "E", torch.bfloat16, (int(E.shape[0]), D))


def _seg_array(segments: Optional[Sequence], dEs=None, comps=None):
    if not segments:
        return None, 0
    arr = (Segment * len(segments))()
    for k, s in enumerate(segments):
        # (begin, end) ranges suffice where no head rows are read (vocab_sort)
        b, e, E = s[0], s[1], (s[2] if len(s) > 2 else None)
        arr[k].vocab_begin, arr[k].vocab_end = int(b), int(e)
        arr[k].E = E.data_ptr() if E is not None else None
        arr[k].dE = dEs[k].data_ptr() if dEs is not None else None
        arr[k].dE_comp = comps[k].data_ptr() if comps is not None else None
    return arr, len(segments)


def fwd_workspace_size(N: int, D: int, V: int, n_segs: int = 0) -> int:
    return int(lib().cce_fwd_workspace_size(N, D, V, n_segs))


def bwd_workspace_size(N: int, D: int, V: int, n_segs: int = 0, flags: int = 0) -> int:
    return int(lib().cce_bwd_workspace_size(N, D, V, n_segs, flags))


def bwd_workspace_parts(N: int, D: int, V: int, n_segs: int = 0, flags: int = 0):
    """{"rows", "vocab", "logits"}: the backward workspace by size class
    (see cce_bwd_workspace_parts)."""
    r, v, l = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    _check(lib().cce_bwd_workspace_parts(N, D, V, n_segs, flags, ctypes.byref(r), ctypes.byref(v),
                                         ctypes.byref(l)), "cce_bwd_workspace_parts")
    return {"rows": r.value, "vocab": v.value, "logits": l.value}


def vocab_sort_workspace_size(N: int, V: int, n_segs: int = 0) -> int:
    return int(lib().cce_vocab_sort_workspace_size(N, V, n_segs))


def _workspace(nbytes: int, device, workspace: Optional[torch.Tensor]) -> torch.Tensor:
    if workspace is not None:
        if workspace.numel() * workspace.element_size() < nbytes:
            raise CCEError("workspace too small")
        return workspace
    return torch.empty(max(nbytes, 16), dtype=torch.uint8, device=device)


def fwd(H: torch.Tensor, E: Optional[torch.Tensor], y: torch.Tensor, ignore_index: int = -100,
        segments: Optional[Sequence[SegSpec]] = None, V: Optional[int] = None,
        want_colmax: bool = False, workspace: Optional[torch.Tensor] = None,
        status: Optional[torch.Tensor] = None, shard: bool = False):
    """Per-row (loss, lse) fp32; optional colmax [V_live].  See cce_fwd.

    shard=True runs cce_fwd_shard instead and returns (zy_part, lse_part)
    in place of (loss, lse): the correct-token logit when this shard holds
    the target (else 0) and the log-sum-exp over this shard."""
    N, D = _rows(H)
    _check_head(E, segments, D)
    if segments:
        V = V if V is not None else int(segments[-1][1])
        v_live = sum(int(e) - int(b) for b, e, *_ in segments)
    else:
        V = int(E.shape[0])
        v_live = V
    _expect(y, "y", torch.int32, (N,))
    _expect_status(status)
    _require_cuda(H, E, y, *[s[2] for s in (segments or [])])
    dev = H.device
    loss = torch.empty(N, dtype=torch.float32, device=dev)
    lse = torch.empty(N, dtype=torch.float32, device=dev)
    colmax = torch.empty(v_live, dtype=torch.float32, device=dev) if want_colmax else None
    segarr, nseg = _seg_array(segments)
    ws = _workspace(fwd_workspace_size(N, D, V, nseg), dev, workspace)
    st = status if status is not None else torch.zeros(1, dtype=torch.int32, device=dev)
    fn = lib().cce_fwd_shard if shard else lib().cce_fwd
    rc = fn(_ptr(H), _ptr(E) if not segments else None, _ptr(y), N, D, V, ignore_index,
            segarr, nseg, _ptr(lse) if shard else _ptr(loss), _ptr(loss) if shard else _ptr(lse),
            _ptr(colmax), _ptr(ws), ws.numel(), _ptr(st), _stream_ptr(dev))
    _check(rc, "cce_fwd_shard" if shard else "cce_fwd")
    if want_colmax:
        return loss, lse, colmax
    return loss, lse


def bwd(H: torch.Tensor, E: Optional[torch.Tensor], y: torch.Tensor, lse: torch.Tensor,
        dloss: torch.Tensor, ignore_index: int = -100,
        segments: Optional[Sequence[SegSpec]] = None, V: Optional[int] = None,
        filter_eps: float = 0.0, vocab_perm: Optional[torch.Tensor] = None,
        colmax: Optional[torch.Tensor] = None, kahan: bool = False, shard: bool = False,
        fp32_grads: bool = False, full_de: bool = False, fp32_dh: bool = False,
        dE_out=None, dE_comp=None, debug_rows: int = 0,
        workspace: Optional[torch.Tensor] = None, status: Optional[torch.Tensor] = None):
    """Gradients (dH, dE) of sum_i dloss_i loss_i.  See cce_bwd.

    dE is one tensor for a single head, a list (one per segment) otherwise.
    With kahan=True, dE_out and dE_comp (bf16, same shape(s)) are required
    and updated in place.  colmax (the forward's, same inputs) enables the
    exact tile skip when filtering.  fp32_dh=True returns dH in fp32 with dE
    in bf16.  Returns (dH, dE, debug_keep or None).
    """
    N, D = _rows(H)
    _check_head(E, segments, D)
    dev = H.device
    gdt = torch.float32 if fp32_grads else torch.bfloat16
    if segments:
        V = V if V is not None else int(segments[-1][1])
        shapes = [(int(e) - int(b), D) for b, e, *_ in segments]
    else:
        V = int(E.shape[0])
        shapes = [(V, D)]
    v_live = sum(r for r, _ in shapes)
    for t, name in ((y, "y"),):
        _expect(t, name, torch.int32, (N,))
    for t, name in ((lse, "lse"), (dloss, "dloss")):
        _expect(t, name, torch.float32, (N,))
    _expect(vocab_perm, "vocab_perm", torch.int32, (v_live,))
    _expect(colmax, "colmax", torch.float32, (v_live,))
    _expect_status(status)
    if dE_out is None:
        if kahan:
            raise CCEError("kahan accumulation needs dE_out and dE_comp")
        dEs = [torch.empty(s, dtype=gdt, device=dev) for s in shapes]
    else:
        dEs = list(dE_out) if isinstance(dE_out, (list, tuple)) else [dE_out]
        if len(dEs) != len(shapes):
            raise CCEError(f"dE_out must hold {len(shapes)} tensor(s), one per segment")
        for k, (t, shp) in enumerate(zip(dEs, shapes)):
            _expect(t, f"dE_out[{k}]", torch.bfloat16 if kahan else gdt, shp)
    comps = None
    if kahan:
        comps = list(dE_comp) if isinstance(dE_comp, (list, tuple)) else [dE_comp]
        if len(comps) != len(shapes):
            raise CCEError(f"dE_comp must hold {len(shapes)} tensor(s), one per segment")
        for k, (t, shp) in enumerate(zip(comps, shapes)):
            _expect(t, f"dE_comp[{k}]", torch.bfloat16, shp)
    _require_cuda(H, E, y, lse, dloss, vocab_perm, colmax, *dEs, *(comps or []))
    dH = torch.empty((N, D), dtype=torch.float32 if fp32_dh else gdt, device=dev)
    flags = ((KAHAN_DE if kahan else 0) | (FP32_GRADS if fp32_grads else 0) |
             (FULL_DE if full_de else 0) | (VOCAB_SHARD if shard else 0) |
             (FP32_DH if fp32_dh else 0))
    words = (V + 31) // 32
    dbg = torch.empty((debug_rows, words), dtype=torch.int32, device=dev) if debug_rows > 0 else None
    segarr, nseg = _seg_array(segments, dEs if segments else None, comps if segments else None)
    ws = _workspace(bwd_workspace_size(N, D, V, nseg, flags), dev, workspace)
    st = status if status is not None else torch.zeros(1, dtype=torch.int32, device=dev)
    rc = lib().cce_bwd(_ptr(H), _ptr(E) if not segments else None, _ptr(y), _ptr(lse), _ptr(dloss),
                       N, D, V, ignore_index, segarr, nseg, float(filter_eps), _ptr(vocab_perm),
                       _ptr(colmax), flags, _ptr(dH), None if segments else dEs[0].data_ptr(),
                       None if (segments or not kahan) else comps[0].data_ptr(),
                       _ptr(dbg), debug_rows, _ptr(ws), ws.numel(), _ptr(st), _stream_ptr(dev))
    _check(rc, "cce_bwd")
    return dH, (dEs if segments else dEs[0]), dbg


def vocab_sort(colmax: Optional[torch.Tensor], y: torch.Tensor, V: int, ignore_index: int = -100,
               segments: Optional[Sequence] = None,
               workspace: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Per-segment permutation of live vocabulary rows by descending key.
    `segments` are (begin, end) ranges, or the (begin, end, E_s) triples of
    fwd / bwd (the head rows themselves are not read)."""
    dev = y.device
    v_live = sum(int(e) - int(b) for b, e, *_ in segments) if segments else V
    if y.dim() != 1:
        raise CCEError("y must be 1-D")
    _expect(y, "y", torch.int32, (y.numel(),))
    _expect(colmax, "colmax", torch.float32, (v_live,))
    _require_cuda(y, colmax)
    perm = torch.empty(v_live, dtype=torch.int32, device=dev)
    segarr, nseg = _seg_array(segments)
    ws = _workspace(vocab_sort_workspace_size(y.numel(), V, nseg), dev, workspace)
    rc = lib().cce_vocab_sort(_ptr(colmax), _ptr(y), y.numel(), V, ignore_index, segarr, nseg,
                              _ptr(perm), _ptr(ws), ws.numel(), _stream_ptr(dev))
    _check(rc, "cce_vocab_sort")
    return perm


def vocab_combine(parts: torch.Tensor, y: torch.Tensor, V: int, ignore_index: int = -100,
                  ranges: Optional[Sequence[Tuple[int, int]]] = None):
    """(loss, lse) [N] from the gathered shard parts [R, 2, N] (lse part,
    correct-token logit part); `ranges` are the whole head's live
    [begin, end) ranges (None: [0, V)).  See cce_vocab_combine."""
    _require_cuda(parts, y)
    R, two, N = parts.shape
    if two != 2 or parts.dtype != torch.float32 or y.dtype != torch.int32 or y.numel() != N:
        raise CCEError("parts must be [R, 2, N] float32 and y [N] int32")
    arr, n = None, 0
    if ranges:
        arr = (Segment * len(ranges))()
        for k, (b, e) in enumerate(ranges):
            arr[k].vocab_begin, arr[k].vocab_end = int(b), int(e)
        n = len(ranges)
    loss = torch.empty(N, dtype=torch.float32, device=parts.device)
    lse = torch.empty(N, dtype=torch.float32, device=parts.device)
    rc = lib().cce_vocab_combine(_ptr(parts), R, _ptr(y), N, V, ignore_index, arr, n, _ptr(loss),
                                 _ptr(lse), _stream_ptr(parts.device))
    _check(rc, "cce_vocab_combine")
    return loss, lse


def check_status(status: torch.Tensor, what: str = "libcce"):
    """Synchronise on the status word's stream and raise CCEError if a kernel
    reported a bad target or a wait that ran out (the outputs of that call are
    then incomplete).  Costs one device-to-host read."""
    v = int(status.item())
    if v & STATUS_TIMEOUT:
        raise CCEError(f"{what}: a kernel wait ran out (CCE_STATUS_TIMEOUT); outputs are incomplete")
    if v & STATUS_BADTARGET:
        raise CCEError(f"{what}: a target outside the vocabulary or in a gap (CCE_STATUS_BADTARGET)")
    return v


def debug_stall(wait_ns: int, status: torch.Tensor, pair: bool = False):
    """Run the bounded-wait diagnostic (see cce_debug_stall; pair=True:
    cce_debug_stall_pair, on one CTA pair)."""
    _require_cuda(status)
    fn = lib().cce_debug_stall_pair if pair else lib().cce_debug_stall
    _check(fn(int(wait_ns), _ptr(status), _stream_ptr(status.device)),
           "cce_debug_stall_pair" if pair else "cce_debug_stall")


def launch_count() -> int:
    """Kernels libcce has enqueued in this process."""
    return int(lib().cce_launch_count())


def timing_enable(class_mask: int):
    _check(lib().cce_timing_enable(class_mask), "cce_timing_enable")


def timing_read():
    """{class name: (summed ms, timed launches)}; clears the record."""
    ms = (ctypes.c_float * 6)()
    n = (ctypes.c_int64 * 6)()
    _check(lib().cce_timing_read(ms, n, 6), "cce_timing_read")
    return {KC_NAMES[i]: (float(ms[i]), int(n[i])) for i in range(6)}


def bf16_from_bits(bits, device) -> torch.Tensor:
    """Upload uint16 bf16 bit patterns (numpy) as a bf16 CUDA tensor."""
    import numpy as np
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.to(device).view(torch.bfloat16)


def _check_kl(Hs, Es, Ht, Et, row_mask) -> Tuple[int, int, int]:
    N, D = _rows(Hs, "Hs")
    if Es is None or Et is None:
        raise CCEError("Es and Et are required")
    V = int(Es.shape[0])
    _expect(Ht, "Ht", torch.bfloat16, (N, D))
    _expect(Es, "Es", torch.bfloat16, (V, D))
    _expect(Et, "Et", torch.bfloat16, (V, D))
    _expect(row_mask, "row_mask", torch.int32, (N,))
    return N, D, V


def kl_fwd(Hs: torch.Tensor, Es: torch.Tensor, Ht: torch.Tensor, Et: torch.Tensor,
           row_mask: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
           status: Optional[torch.Tensor] = None):
    """Per-row (KL(p_t || p_s), lse_s, lse_t) fp32.  See cce_kl_fwd."""
    N, D, V = _check_kl(Hs, Es, Ht, Et, row_mask)
    _expect_status(status)
    _require_cuda(Hs, Es, Ht, Et, row_mask)
    dev = Hs.device
    kl = torch.empty(N, dtype=torch.float32, device=dev)
    ls = torch.empty(N, dtype=torch.float32, device=dev)
    lt = torch.empty(N, dtype=torch.float32, device=dev)
    ws = _workspace(int(lib().cce_kl_fwd_workspace_size(N, D, V)), dev, workspace)
    st = status if status is not None else torch.zeros(1, dtype=torch.int32, device=dev)
    rc = lib().cce_kl_fwd(_ptr(Hs), _ptr(Es), _ptr(Ht), _ptr(Et), _ptr(row_mask), N, D, V,
                          _ptr(kl), _ptr(ls), _ptr(lt), _ptr(ws), ws.numel(), _ptr(st),
                          _stream_ptr(dev))
    _check(rc, "cce_kl_fwd")
    return kl, ls, lt


def kl_bwd(Hs: torch.Tensor, Es: torch.Tensor, Ht: torch.Tensor, Et: torch.Tensor,
           lse_s: torch.Tensor, lse_t: torch.Tensor, dloss: torch.Tensor,
           row_mask: Optional[torch.Tensor] = None, filter_eps: float = 0.0,
           fp32_grads: bool = False, kahan: bool = False, dE_out=None, dE_comp=None,
           debug_rows: int = 0, workspace: Optional[torch.Tensor] = None,
           status: Optional[torch.Tensor] = None):
    """Student gradients (dH, dE) of sum_i dloss_i KL_i.  See cce_kl_bwd.
    With debug_rows > 0 returns (dH, dE, keep bits [debug_rows, ceil(V/32)])."""
    N, D, V = _check_kl(Hs, Es, Ht, Et, row_mask)
    for t, name in ((lse_s, "lse_s"), (lse_t, "lse_t"), (dloss, "dloss")):
        _expect(t, name, torch.float32, (N,))
    _expect_status(status)
    if dE_out is not None:
        _expect(dE_out, "dE_out", torch.bfloat16 if kahan else
                (torch.float32 if fp32_grads else torch.bfloat16), (V, D))
    if kahan:
        _expect(dE_comp, "dE_comp", torch.bfloat16, (V, D))
    _require_cuda(Hs, Es, Ht, Et, lse_s, lse_t, dloss, row_mask, dE_out,
                  dE_comp if kahan else None)
    dev = Hs.device
    gdt = torch.float32 if fp32_grads else torch.bfloat16
    if kahan and (dE_out is None or dE_comp is None):
        raise CCEError("kahan accumulation needs dE_out and dE_comp")
    dE = dE_out if dE_out is not None else torch.empty((V, D), dtype=gdt, device=dev)
    dH = torch.empty((N, D), dtype=gdt, device=dev)
    flags = (KAHAN_DE if kahan else 0) | (FP32_GRADS if fp32_grads else 0)
    ws = _workspace(int(lib().cce_kl_bwd_workspace_size(N, D, V, flags)), dev, workspace)
    st = status if status is not None else torch.zeros(1, dtype=torch.int32, device=dev)
    dbg = (torch.empty((debug_rows, (V + 31) // 32), dtype=torch.int32, device=dev)
           if debug_rows > 0 else None)
    rc = lib().cce_kl_bwd(_ptr(Hs), _ptr(Es), _ptr(Ht), _ptr(Et), _ptr(row_mask), _ptr(lse_s),
                          _ptr(lse_t), _ptr(dloss), N, D, V, float(filter_eps), flags, _ptr(dH),
                          _ptr(dE), _ptr(dE_comp) if kahan else None, _ptr(dbg), debug_rows,
                          _ptr(ws), ws.numel(), _ptr(st), _stream_ptr(dev))
    _check(rc, "cce_kl_bwd")
    if debug_rows > 0:
        return dH, dE, dbg
    return dH, dE
