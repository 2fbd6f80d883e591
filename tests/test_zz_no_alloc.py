"""cce_fwd_noalloc: the forward entry point that allocates nothing.

Some callers cannot call cudaMalloc (a host framework that owns all device
memory and gives plugins no allocation hook, or a C/Fortran program linking
libcce without a device allocator).  For them the forward keeps its scratch
in a fixed array inside the library's device image.  These tests call that
entry point through the C ABI and check it against the workspace-taking
cce_fwd, on two calls in a row with different inputs (the second call must
not see anything the first left in the shared array).  This file is named so
that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

from linear_cross_entropy_cce_b200 import cce, synthetic as syn
from _helpers import TOL_ROW, to_np, upload


def _entry():
    L = cce.lib()
    f = L.cce_fwd_noalloc
    vp, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32
    f.restype = ctypes.c_int
    f.argtypes = [vp, vp, vp, i64, i64, i64, i32, ctypes.POINTER(cce.Segment), i32,
                  vp, vp, vp, vp, vp]
    return f


def test_noalloc_rejects_sizes_beyond_its_scratch():
    # Gemma-2-2B-shaped forward needs far more than the fixed scratch; the
    # size check fails before any device work.
    f = _entry()
    rc = f(16, 16, 16, 8192, 2304, 256000, -100, None, 0, 16, 16, None, 16, None)
    assert rc == cce.CCE_EWORKSPACE


@pytest.mark.gpu
def test_noalloc_forward_matches_workspace_forward_two_calls():
    f = _entry()
    cases = [
        syn.Workload("na1", N=1000, D=512, V=7000, logit_std=4.0, ignore_frac=0.1),
        syn.scaled(syn.WORKLOADS["composite_two_segment"], N=600, D=256, V=5200,
                   segments=((0, 3000), (3100, 5200))),
    ]
    for seed, wl in enumerate(cases):
        x = syn.make_inputs(wl, seed=seed)
        H, segs, y = upload(x)
        single = len(segs) == 1
        if single:
            ref_loss, ref_lse = cce.fwd(H, segs[0][2], y, x.ignore_index)
            arr, nseg = None, 0
        else:
            ref_loss, ref_lse = cce.fwd(H, None, y, x.ignore_index, segments=segs, V=wl.V)
            arr, nseg = cce._seg_array(segs)
        loss = torch.full((wl.N,), float("nan"), device="cuda")
        lse = torch.full((wl.N,), float("nan"), device="cuda")
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        stream = torch.cuda.current_stream().cuda_stream
        rc = f(H.data_ptr(), segs[0][2].data_ptr() if single else None, y.data_ptr(), wl.N, wl.D,
               wl.V, x.ignore_index, arr, nseg, loss.data_ptr(), lse.data_ptr(), None,
               st.data_ptr(), stream)
        assert rc == cce.CCE_OK
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        assert np.max(np.abs(to_np(loss) - to_np(ref_loss))) <= TOL_ROW
        assert np.max(np.abs(to_np(lse) - to_np(ref_lse))) <= TOL_ROW
