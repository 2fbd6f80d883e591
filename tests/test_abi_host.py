"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every symbol include/cce.h declares, and rejects bad arguments before any
device work (no compute call is made here)."""
import ctypes
import json
import os
import re

import pytest

from linear_cross_entropy_cce_b200 import cce

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "cce.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(cce_[a-z_0-9]+)\s*\(", src)))


def test_library_loads_and_exports_every_declared_symbol():
    L = cce.lib()
    names = _declared()
    assert set(names) >= set(cce.EXPORTS)
    for n in names:
        assert hasattr(L, n), n
    assert L.cce_version() >= 10000


def test_strerror_covers_codes():
    L = cce.lib()
    for c in range(5):
        assert L.cce_strerror(c)
    assert b"unknown" in L.cce_strerror(99)


def test_workspace_sizes_and_invalid_sizes():
    L = cce.lib()
    assert L.cce_fwd_workspace_size(256, 256, 4096, 0) > 0
    assert L.cce_fwd_workspace_size(256, 250, 4096, 0) == 0      # D % 8 != 0
    assert L.cce_fwd_workspace_size(-1, 256, 4096, 0) == 0
    assert L.cce_fwd_workspace_size(256, 256, 0, 0) == 0
    assert L.cce_fwd_workspace_size(256, 256, 4096, 9) == 0      # too many segments
    assert L.cce_bwd_workspace_size(256, 256, 4096, 0, 0) > 0
    # CCE_FULL_DE adds one more bf16 slab of G (the full one, read by dE only)
    plain, full = L.cce_bwd_workspace_size(256, 256, 4096, 0, 0), L.cce_bwd_workspace_size(256, 256, 4096, 0, 4)
    assert full - plain >= 256 * 4096 * 2
    assert L.cce_bwd_workspace_size(256, 256, 4096, 0, 1) == plain   # Kahan needs no scratch
    assert L.cce_vocab_sort_workspace_size(256, 4096, 0) > 0


def test_size_limits_are_enforced():
    L = cce.lib()
    top = 2 ** 31 - 257
    assert L.cce_fwd_workspace_size(1, 8, top, 0) > 0
    assert L.cce_fwd_workspace_size(1, 8, top + 1, 0) == 0
    assert L.cce_fwd_workspace_size(top + 1, 8, 16, 0) == 0
    assert L.cce_fwd_workspace_size(1, 65536, 16, 0) > 0
    assert L.cce_fwd_workspace_size(1, 65544, 16, 0) == 0
    assert L.cce_bwd_workspace_size(1, 8, top + 1, 0, 0) == 0
    assert L.cce_bwd_workspace_size(1, 65544, 16, 0, 0) == 0
    assert _null_fwd(V=top + 1) == cce.CCE_EINVAL
    assert _null_fwd(N=top + 1) == cce.CCE_EINVAL
    assert _null_fwd(D=65544) == cce.CCE_EINVAL


def test_workspace_is_far_below_materialised_logits():
    """The page on chunking CE after an OOM prints 12.2 GB for one bf16
    softmax over 24,576 positions x 248,320 vocabulary; the research-map
    entry prints 24000 MB of loss memory for Gemma 2 (2B).  libcce's scratch
    for those shapes stays a small fraction of it: its largest buffer, the
    bf16 G slab of one vocabulary chunk, is capped at 512 MiB, nothing is
    N x V."""
    g = json.load(open(os.path.join(ROOT, "tests", "golden", "pages_memory.json")))
    for case in g["cases"]:
        N, D, V, nseg = case["N"], case["D"], case["V"], case["n_segs"]
        assert abs(N * V * case["bytes_per_elt"] - case["page_bytes"]) <= case["rel_tol"] * case["page_bytes"]
        ws = max(cce.fwd_workspace_size(N, D, V, nseg), cce.bwd_workspace_size(N, D, V, nseg))
        assert ws < 0.10 * case["page_bytes"], (case["name"], ws)


def _null_fwd(**kw):
    L = cce.lib()
    a = dict(H=16, E=16, y=16, N=4, D=8, V=10, ign=-100, segs=None, nseg=0, loss=16, lse=16,
             colmax=None, ws=16, wsb=1 << 30, st=16, stream=None)
    a.update(kw)
    return L.cce_fwd(a["H"], a["E"], a["y"], a["N"], a["D"], a["V"], a["ign"], a["segs"],
                     a["nseg"], a["loss"], a["lse"], a["colmax"], a["ws"], a["wsb"], a["st"],
                     a["stream"])


def test_fwd_rejects_bad_arguments_on_host():
    # None of these reaches the device: validation fails first.
    assert _null_fwd(D=12) == cce.CCE_EINVAL
    assert _null_fwd(H=None) == cce.CCE_EINVAL
    assert _null_fwd(E=None) == cce.CCE_EINVAL
    assert _null_fwd(H=18) == cce.CCE_EINVAL                    # misaligned
    assert _null_fwd(ws=None) == cce.CCE_EWORKSPACE
    assert _null_fwd(wsb=8) == cce.CCE_EWORKSPACE
    assert _null_fwd(N=0) == cce.CCE_OK                          # nothing to do


def test_segment_table_validation():
    seg = (cce.Segment * 2)()
    seg[0].vocab_begin, seg[0].vocab_end, seg[0].E = 0, 6, 16
    seg[1].vocab_begin, seg[1].vocab_end, seg[1].E = 4, 10, 32  # overlaps
    assert _null_fwd(E=None, segs=seg, nseg=2) == cce.CCE_EINVAL
    seg[1].vocab_begin = 7
    seg[1].vocab_end = 11                                       # beyond V
    assert _null_fwd(E=None, segs=seg, nseg=2) == cce.CCE_EINVAL
    seg[1].vocab_end = 10
    assert _null_fwd(E=16, segs=seg, nseg=2) == cce.CCE_EINVAL   # E and segs both given
    seg[1].E = None
    assert _null_fwd(E=None, segs=seg, nseg=2) == cce.CCE_EINVAL
    seg[1].E = 32
    assert _null_fwd(E=None, segs=seg, nseg=2, ws=None) == cce.CCE_EWORKSPACE


def test_bwd_rejects_bad_flags_and_missing_kahan_buffer():
    L = cce.lib()

    def call(flags=0, dE=16, comp=None):
        return L.cce_bwd(16, 16, 16, 16, 16, 4, 8, 10, -100, None, 0, 0.0, None, None, flags,
                         16, dE, comp, None, 0, 16, 1 << 30, 16, None)
    assert call(flags=32) == cce.CCE_EINVAL                      # unknown flag bit
    assert call(flags=cce.KAHAN_DE) == cce.CCE_EINVAL           # no compensation buffer
    assert call(flags=cce.KAHAN_DE | cce.FP32_GRADS, comp=16) == cce.CCE_EINVAL
    assert call(dE=None) == cce.CCE_EINVAL


def test_bwd_workspace_follows_the_segment_count():
    # each segment may add one partial vocabulary chunk to the sparse lists,
    # so the size grows with n_segs, and a call with more segments than the
    # workspace was sized for is refused before anything reaches the device
    L = cce.lib()
    sizes = [cce.bwd_workspace_size(4, 8, 10, n) for n in (0, 1, 2, 8)]
    assert sizes[0] == sizes[1] < sizes[2] < sizes[3]
    seg = (cce.Segment * 2)()
    seg[0].vocab_begin, seg[0].vocab_end, seg[0].E, seg[0].dE = 0, 6, 16, 16
    seg[1].vocab_begin, seg[1].vocab_end, seg[1].E, seg[1].dE = 6, 10, 32, 32
    rc = L.cce_bwd(16, None, 16, 16, 16, 4, 8, 10, -100, seg, 2, 0.0, None, None, 0,
                   16, None, None, None, 0, 16, sizes[1], 16, None)
    assert rc == cce.CCE_EWORKSPACE


def test_vocab_combine_rejects_bad_arguments_on_host():
    L = cce.lib()
    EINVAL = cce.CCE_EINVAL

    def comb(parts=16, R=2, y=16, N=4, V=10, segs=None, nseg=0, loss=16, lse=16):
        return L.cce_vocab_combine(parts, R, y, N, V, -100, segs, nseg, loss, lse, None)
    assert comb(R=0) == EINVAL and comb(R=5000) == EINVAL
    assert comb(N=-1) == EINVAL and comb(V=0) == EINVAL
    assert comb(parts=None) == EINVAL and comb(y=None) == EINVAL
    assert comb(loss=None) == EINVAL and comb(lse=None) == EINVAL
    assert comb(N=0, parts=None) == cce.CCE_OK  # nothing to do: no launch
    seg = (cce.Segment * 2)()
    seg[0].vocab_begin, seg[0].vocab_end = 0, 6
    seg[1].vocab_begin, seg[1].vocab_end = 5, 10  # overlapping ranges
    assert comb(segs=seg, nseg=2) == EINVAL
    seg[1].vocab_begin, seg[1].vocab_end = 7, 11  # beyond V
    assert comb(segs=seg, nseg=2) == EINVAL
    assert comb(segs=seg, nseg=9) == EINVAL


def test_kl_and_shard_entry_points_reject_bad_arguments_on_host():
    L = cce.lib()
    EINVAL = cce.CCE_EINVAL
    # cce_kl_fwd(Hs, Es, Ht, Et, row_mask, N, D, V, kl, lse_s, lse_t, ws, wsb, status, stream)
    ok = dict(Hs=16, Es=16, Ht=16, Et=16, N=4, D=8, V=10)

    def kl_fwd(**kw):
        a = dict(ok, **kw)
        return L.cce_kl_fwd(a["Hs"], a["Es"], a["Ht"], a["Et"], None, a["N"], a["D"], a["V"],
                            16, 16, 16, 16, 1 << 30, 16, None)
    assert kl_fwd(Hs=None) == EINVAL
    assert kl_fwd(Et=None) == EINVAL
    assert kl_fwd(Ht=24) == EINVAL          # not 16-byte aligned
    assert kl_fwd(D=12) == EINVAL           # D % 8 != 0
    assert kl_fwd(N=0) == cce.CCE_OK        # nothing to do

    # cce_kl_bwd(Hs, Es, Ht, Et, mask, lse_s, lse_t, dloss, N, D, V, eps, flags, dH, dE, dE_comp,
    #            debug_keep, debug_rows, ws, wsb, status, stream)
    def kl_bwd(flags=0, Ht=16, dbg_rows=0):
        return L.cce_kl_bwd(16, 16, Ht, 16, None, 16, 16, 16, 4, 8, 10, 0.0, flags, 16, 16, None,
                            16 if dbg_rows else None, dbg_rows, 16, 1 << 30, 16, None)
    assert kl_bwd(flags=cce.FULL_DE) == EINVAL
    assert kl_bwd(flags=cce.VOCAB_SHARD) == EINVAL
    assert kl_bwd(Ht=None) == EINVAL
    assert kl_bwd(dbg_rows=5) == EINVAL  # more debug rows than rows
    assert L.cce_kl_bwd_workspace_size(256, 256, 4096, 0) > L.cce_bwd_workspace_size(256, 256, 4096, 0, 0)
    assert L.cce_kl_fwd_workspace_size(256, 250, 4096) == 0

    # cce_fwd_shard: the cce_fwd argument checks
    assert L.cce_fwd_shard(None, 16, 16, 4, 8, 10, -100, None, 0, 16, 16, None, 16, 1 << 30, 16,
                           None) == EINVAL
    assert L.cce_fwd_shard(16, 16, 16, 4, 8, 10, -100, None, 0, None, 16, None, 16, 1 << 30, 16,
                           None) == EINVAL


def test_plain_c_consumer(tmp_path):
    """tests/c_abi_check.c: a C99 program that includes only include/cce.h and
    links libcce.so checks the host-side contract."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    cce.lib()  # built
    libdir = os.path.join(ROOT, "linear_cross_entropy_cce_b200")
    exe = str(tmp_path / "c_abi_check")
    subprocess.run([gcc, "-std=c99", "-Wall", "-Werror", "-D_DEFAULT_SOURCE",
                    "-I", os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "c_abi_check.c"),
                    "-L", libdir, "-lcce", "-Wl,-rpath," + libdir, "-o", exe], check=True)
    out = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, out.stderr
    assert "c abi ok" in out.stdout


def test_workspace_plan_invariants_over_random_shapes():
    """For seeded random shapes, segment counts and flags: the three size
    classes add up to the workspace size, the size grows with n_segs, and on
    heads whose bf16 logits exceed 512 MiB (N V 2 / 8 >= 64 MiB) the
    logits-class buffers stay below an eighth of them (no buffer of the
    logits' size)."""
    import numpy as np
    rng = np.random.default_rng(2024)
    for _ in range(300):
        N = int(rng.integers(1, 1 << 16))
        D = 8 * int(rng.integers(1, 1025))
        V = int(rng.integers(1, 1 << 19))
        nseg = int(rng.integers(0, 9))
        flags = int(rng.choice([0, cce.KAHAN_DE, cce.FULL_DE, cce.FP32_GRADS]))
        total = cce.bwd_workspace_size(N, D, V, nseg, flags)
        parts = cce.bwd_workspace_parts(N, D, V, nseg, flags)
        assert total > 0 and sum(parts.values()) == total, (N, D, V, nseg, flags)
        assert cce.bwd_workspace_size(N, D, V, min(8, nseg + 1), flags) >= total
        bound = N * V * 2 / 8
        if bound >= 64 * 2 ** 20:
            assert parts["logits"] < bound, (N, D, V, nseg, flags, parts["logits"], bound)
        # the forward's and the sort's scratch never shrink with more segments either
        more = min(8, nseg + 1)
        assert cce.fwd_workspace_size(N, D, V, more) >= cce.fwd_workspace_size(N, D, V, nseg) > 0
        assert cce.vocab_sort_workspace_size(N, V, more) >= cce.vocab_sort_workspace_size(N, V, nseg) > 0
