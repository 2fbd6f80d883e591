"""Seeded synthetic inputs for the fused classifier + cross-entropy workloads.

This module only draws random data: it holds none of the loss arithmetic and
imports neither the CUDA library binding nor the oracle, so both sides of the
parity tests consume the very same bf16 bit patterns from here.

Recipe (one ``numpy.random.SeedSequence(seed)``, spawned into independent
streams for H, E, the vocabulary permutation, the targets and the ignore mask):
  * H ~ N(0, 1) and E ~ N(0, (logit_std / sqrt(D))^2), drawn in fp32 and
    rounded to bf16 with round-to-nearest-even, so a logit <h, e> has a
    standard deviation of about ``logit_std``;
  * targets follow a Zipf law truncated to the vocabulary,
    P(rank k) proportional to k^-s for k = 1..n (s = 1.1), mapped through a
    random permutation of the vocabulary, or are uniform;
  * exactly round(ignore_frac * N) rows, chosen at random, get ignore_index;
  * a composite head draws each valid target from segment A or B with the
    stated mixture, Zipf within the segment over its own permutation.
Large matrices are generated in fixed blocks of 2^22 elements, each from its
own spawned stream, so the result does not depend on the thread count.
"""
from __future__ import annotations

import concurrent.futures as _cf
import os
from dataclasses import dataclass, field
from typing import List, Optional, Sequence, Tuple

import numpy as np

IGNORE_INDEX = -100
_BLOCK = 1 << 22


@dataclass(frozen=True)
class Workload:
    name: str
    N: int
    D: int
    V: int                      # logical vocabulary size
    logit_std: float
    ignore_frac: float
    targets: str = "zipf"       # "zipf" | "uniform"
    zipf_s: float = 1.1
    # live segments [begin, end) on the logical vocabulary; default one [0, V)
    segments: Tuple[Tuple[int, int], ...] = ()
    # probability of drawing a valid target from each segment
    segment_mix: Tuple[float, ...] = ()

    def segs(self) -> Tuple[Tuple[int, int], ...]:
        return self.segments if self.segments else ((0, self.V),)

    @property
    def n_ignore(self) -> int:
        return int(round(self.ignore_frac * self.N))

    @property
    def n_valid(self) -> int:
        return self.N - self.n_ignore

    @property
    def v_live(self) -> int:
        return sum(e - b for b, e in self.segs())


WORKLOADS = {
    "tiny": Workload("tiny", N=256, D=256, V=4096, logit_std=1.0, ignore_frac=0.10),
    "gemma2_2b_head": Workload("gemma2_2b_head", N=8192, D=2304, V=256000,
                               logit_std=8.0, ignore_frac=0.05),
    "llama3_8b_head": Workload("llama3_8b_head", N=16384, D=4096, V=128256,
                               logit_std=1.0, ignore_frac=0.0),
    "phi35_mini_head": Workload("phi35_mini_head", N=16384, D=3072, V=32064,
                                logit_std=4.0, ignore_frac=0.20, targets="uniform"),
    "composite_two_segment": Workload(
        "composite_two_segment", N=24576, D=2048, V=248320, logit_std=6.0,
        ignore_frac=0.50, segments=((0, 151936), (153090, 248320)),
        segment_mix=(0.7, 0.3)),
    # the Llama-3-8B-shaped head at half the rows: sized for kernel captures
    # (a few GB on the device; H_c still larger than L2)
    "llama3_8b_head_8k": Workload("llama3_8b_head_8k", N=8192, D=4096, V=128256,
                                  logit_std=1.0, ignore_frac=0.0),
}


def scaled(wl: Workload, N: int, D: int, V: int, name: Optional[str] = None,
           segments: Optional[Sequence[Tuple[int, int]]] = None) -> Workload:
    """The same value recipe at another size (for small parity cases)."""
    return Workload(name or f"{wl.name}@{N}x{D}x{V}", N=N, D=D, V=V,
                    logit_std=wl.logit_std, ignore_frac=wl.ignore_frac,
                    targets=wl.targets, zipf_s=wl.zipf_s,
                    segments=tuple(segments) if segments is not None else (),
                    segment_mix=wl.segment_mix if segments is not None else ())


def fp32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest, ties to even); returns uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


def _normal_bf16(ss: np.random.SeedSequence, shape, std: float,
                 threads: Optional[int] = None) -> np.ndarray:
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16)
    nblk = (n + _BLOCK - 1) // _BLOCK
    children = ss.spawn(nblk)

    def fill(b):
        lo, hi = b * _BLOCK, min(n, (b + 1) * _BLOCK)
        g = np.random.Generator(np.random.SFC64(children[b]))
        x = g.standard_normal(hi - lo, dtype=np.float32)
        if std != 1.0:
            x *= np.float32(std)
        out[lo:hi] = fp32_to_bf16_bits(x)

    threads = threads or min(16, len(os.sched_getaffinity(0)))
    if nblk == 1 or threads == 1:
        for b in range(nblk):
            fill(b)
    else:
        with _cf.ThreadPoolExecutor(threads) as ex:
            list(ex.map(fill, range(nblk)))
    return out.reshape(shape)


def zipf_ranks(rng: np.random.Generator, n_items: int, size: int, s: float) -> np.ndarray:
    """Ranks 0..n_items-1 with P(rank k) proportional to (k+1)^-s (truncated)."""
    w = np.arange(1, n_items + 1, dtype=np.float64) ** (-s)
    cdf = np.cumsum(w)
    cdf /= cdf[-1]
    u = rng.random(size)
    return np.minimum(np.searchsorted(cdf, u, side="right"), n_items - 1)


@dataclass
class Inputs:
    wl: Workload
    H: np.ndarray                       # uint16 [N, D] (bf16 bits)
    segments: List[Tuple[int, int, np.ndarray]]  # (begin, end, E bits [n_s, D])
    y: np.ndarray                       # int32 [N]
    ignore_index: int = IGNORE_INDEX

    @property
    def valid(self) -> np.ndarray:
        return self.y != self.ignore_index

    @property
    def n_valid(self) -> int:
        return int(np.count_nonzero(self.valid))

    def dloss_mean(self) -> np.ndarray:
        """Upstream gradient of the mean loss: 1/N_v on valid rows, else 0."""
        nv = max(1, self.n_valid)
        return np.where(self.valid, np.float32(1.0 / nv), np.float32(0.0)).astype(np.float32)


def make_inputs(wl: Workload, seed: int = 0, threads: Optional[int] = None) -> Inputs:
    ss_H, ss_E, ss_perm, ss_y, ss_ign = np.random.SeedSequence(seed).spawn(5)
    N, D = wl.N, wl.D
    H = _normal_bf16(ss_H, (N, D), 1.0, threads)
    e_std = wl.logit_std / np.sqrt(D)
    segs = []
    for (b, e), ss in zip(wl.segs(), ss_E.spawn(len(wl.segs()))):
        segs.append((b, e, _normal_bf16(ss, (e - b, D), e_std, threads)))
    # valid rows and targets
    r_ign = np.random.Generator(np.random.PCG64(ss_ign))
    ignore = np.zeros(N, dtype=bool)
    ignore[r_ign.permutation(N)[:wl.n_ignore]] = True
    r_perm = np.random.Generator(np.random.PCG64(ss_perm))
    r_y = np.random.Generator(np.random.PCG64(ss_y))
    seg_list = wl.segs()
    perms = [r_perm.permutation(e - b) for b, e in seg_list]
    mix = wl.segment_mix if wl.segment_mix else (1.0,)
    which = r_y.choice(len(seg_list), size=N, p=np.asarray(mix) / np.sum(mix)) \
        if len(seg_list) > 1 else np.zeros(N, dtype=np.int64)
    y = np.empty(N, dtype=np.int64)
    for k, (b, e) in enumerate(seg_list):
        sel = which == k
        cnt = int(np.count_nonzero(sel))
        if wl.targets == "uniform":
            local = r_y.integers(0, e - b, size=cnt)
        else:
            local = perms[k][zipf_ranks(r_y, e - b, cnt, wl.zipf_s)]
        y[sel] = b + local
    y[ignore] = IGNORE_INDEX
    return Inputs(wl, H, segs, y.astype(np.int32))


# ---- soft-target KL workload ------------------------------------------------
# The page on chunking the loss after an OOM trains with a soft KL term
# between a student and a teacher softmax at 24,576 positions over a 248,320
# vocabulary.  Stand-in inputs of that shape: student and teacher rows
# H ~ N(0, 1) drawn independently, one shared head E ~ N(0, logit_std/sqrt(D)).
@dataclass(frozen=True)
class KLWorkload:
    name: str
    N: int
    D: int
    V: int
    logit_std: float


KL_WORKLOADS = {
    "soft_kl_24k_248k": KLWorkload("soft_kl_24k_248k", N=24576, D=2048, V=248320, logit_std=6.0),
    "soft_kl_small": KLWorkload("soft_kl_small", N=512, D=256, V=8192, logit_std=6.0),
    # kernel captures: E (268 MB) larger than L2, about 1 GB on the device
    "soft_kl_8k_64k": KLWorkload("soft_kl_8k_64k", N=8192, D=2048, V=65536, logit_std=6.0),
}


def make_kl_inputs(wl: KLWorkload, seed: int = 0, threads: Optional[int] = None):
    """(Hs, Ht, E) as bf16 bit patterns for a soft-target KL workload."""
    ss_s, ss_t, ss_e = np.random.SeedSequence(seed).spawn(3)
    Hs = _normal_bf16(ss_s, (wl.N, wl.D), 1.0, threads)
    Ht = _normal_bf16(ss_t, (wl.N, wl.D), 1.0, threads)
    E = _normal_bf16(ss_e, (wl.V, wl.D), wl.logit_std / np.sqrt(wl.D), threads)
    return Hs, Ht, E
