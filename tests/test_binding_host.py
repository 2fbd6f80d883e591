"""The binding refuses tensors whose type or shape does not match the sizes it
passes to the C ABI (which trusts them and would read or write out of
bounds).  Everything here fails before any device work, so it runs on CPU
tensors: a call with valid types and shapes gets as far as the CUDA check."""
import pytest
import torch

from linear_cross_entropy_cce_b200 import cce

N, D, V = 6, 16, 40
bf = torch.bfloat16


def _ok():
    return dict(H=torch.zeros(N, D, dtype=bf), E=torch.zeros(V, D, dtype=bf),
                y=torch.zeros(N, dtype=torch.int32), lse=torch.zeros(N),
                dloss=torch.zeros(N))


def _raises(match, fn, *a, **kw):
    with pytest.raises(cce.CCEError, match=match):
        fn(*a, **kw)


def test_valid_arguments_reach_the_cuda_check():
    t = _ok()
    _raises("CUDA", cce.fwd, t["H"], t["E"], t["y"])
    _raises("CUDA", cce.bwd, t["H"], t["E"], t["y"], t["lse"], t["dloss"])
    _raises("CUDA", cce.kl_fwd, t["H"], t["E"], t["H"], t["E"])
    _raises("CUDA", cce.vocab_sort, None, t["y"], V)


def test_forward_arguments():
    t = _ok()
    _raises("bfloat16", cce.fwd, t["H"].float(), t["E"], t["y"])
    _raises("bfloat16", cce.fwd, t["H"][0], t["E"], t["y"])             # 1-D
    _raises(r"E must have shape \(40, 16\)", cce.fwd, t["H"], t["E"][:, :8].contiguous(), t["y"])
    _raises("E must be torch.bfloat16", cce.fwd, t["H"], t["E"].half(), t["y"])
    _raises("y must be torch.int32", cce.fwd, t["H"], t["E"], t["y"].long())
    _raises(r"y must have shape \(6,\)", cce.fwd, t["H"], t["E"], t["y"][:5])
    _raises("status", cce.fwd, t["H"], t["E"], t["y"], status=torch.zeros(1))
    _raises("required", cce.fwd, t["H"], None, t["y"])
    segs = [(0, 10, torch.zeros(10, D, dtype=bf)), (20, 40, torch.zeros(19, D, dtype=bf))]
    _raises(r"segment 1 E must have shape \(20, 16\)", cce.fwd, t["H"], None, t["y"],
            segments=segs, V=V)
    _raises("empty or reversed", cce.fwd, t["H"], None, t["y"],
            segments=[(5, 5, torch.zeros(0, D, dtype=bf))], V=V)


def test_backward_arguments():
    t = _ok()
    H, E, y, lse, dl = t["H"], t["E"], t["y"], t["lse"], t["dloss"]
    _raises(r"lse must have shape", cce.bwd, H, E, y, lse[:3], dl)
    _raises("dloss must be torch.float32", cce.bwd, H, E, y, lse, dl.half())
    _raises(r"vocab_perm must have shape \(40,\)", cce.bwd, H, E, y, lse, dl,
            vocab_perm=torch.zeros(39, dtype=torch.int32))
    _raises("colmax must be torch.float32", cce.bwd, H, E, y, lse, dl,
            colmax=torch.zeros(V, dtype=bf))
    _raises(r"dE_out\[0\] must have shape", cce.bwd, H, E, y, lse, dl,
            dE_out=torch.zeros(V - 1, D, dtype=bf))
    _raises(r"dE_out\[0\] must be torch.float32", cce.bwd, H, E, y, lse, dl, fp32_grads=True,
            dE_out=torch.zeros(V, D, dtype=bf))
    _raises(r"dE_comp\[0\] must be torch.bfloat16", cce.bwd, H, E, y, lse, dl, kahan=True,
            dE_out=torch.zeros(V, D, dtype=bf), dE_comp=torch.zeros(V, D))
    _raises("one per segment", cce.bwd, H, None, y, lse, dl, V=V,
            segments=[(0, 10, torch.zeros(10, D, dtype=bf)), (20, 40, torch.zeros(20, D, dtype=bf))],
            dE_out=[torch.zeros(10, D, dtype=bf)])


def test_kl_and_sort_arguments():
    t = _ok()
    H, E = t["H"], t["E"]
    _raises(r"Ht must have shape \(6, 16\)", cce.kl_fwd, H, E, H[:5].contiguous(), E)
    _raises("Et must be torch.bfloat16", cce.kl_fwd, H, E, H, E.float())
    _raises("row_mask must be torch.int32", cce.kl_fwd, H, E, H, E,
            row_mask=torch.ones(N, dtype=torch.int64))
    _raises(r"lse_t must have shape", cce.kl_bwd, H, E, H, E, t["lse"], t["lse"][:2], t["dloss"])
    _raises(r"dE_out must have shape \(40, 16\)", cce.kl_bwd, H, E, H, E, t["lse"], t["lse"],
            t["dloss"], dE_out=torch.zeros(V, 8, dtype=bf))
    _raises(r"colmax must have shape \(40,\)", cce.vocab_sort, torch.zeros(V + 1), t["y"], V)
    _raises(r"colmax must have shape \(30,\)", cce.vocab_sort, torch.zeros(V), t["y"], V,
            segments=[(0, 10), (20, 40)])
