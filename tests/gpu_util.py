"""Helpers for the GPU parity tests: seeded workloads packed by the CPU
oracle, numpy <-> torch transfers, and sampled-row oracle checks."""
from __future__ import annotations

import functools

import numpy as np
import torch

import oracle as orc
import synth

DEV = torch.device("cuda", 0)


def to_dev(a: np.ndarray) -> torch.Tensor:
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).to(DEV).view(torch.bfloat16)
    return torch.from_numpy(a).to(DEV)


def bits(t: torch.Tensor) -> np.ndarray:
    """bf16 device tensor -> uint16 numpy bit patterns."""
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


@functools.lru_cache(maxsize=8)
def packed_weights(fmt: str, E: int, N: int, K: int, std: float, seed: int):
    """Seeded N(0, std^2) expert weights packed by the oracle, and the bf16
    weights the oracle decodes from them."""
    w = synth.normal((E, N, K), seed, std)
    if fmt == "nf4":
        codes, scale = orc.nf4_pack(w)
        wdec = orc.nf4_decode(codes, scale, K, bf16=True)
    else:
        codes, scale = orc.mxfp4_pack(w)
        wdec = orc.mxfp4_decode(codes, scale, bf16=True)
    del w
    return codes, scale, wdec


def sample_rows(off: np.ndarray, n: int, seed: int) -> np.ndarray:
    """Rows worth checking: first/last row of the largest, smallest and some
    random non-empty experts, rows at 256-row tile edges, plus random rows."""
    rng = np.random.default_rng(seed)
    cnt = np.diff(off)
    live = np.nonzero(cnt)[0]
    picks = set()
    for e in [live[np.argmax(cnt[live])], live[np.argmin(cnt[live])],
              *rng.choice(live, size=min(4, len(live)), replace=False)]:
        a, b = int(off[e]), int(off[e + 1])
        for r in (a, b - 1, a + 127, a + 128, a + 255, a + 256, a + 257):
            if a <= r < b:
                picks.add(r)
    P = int(off[-1])
    picks.update(int(v) for v in rng.integers(0, P, size=max(0, n - len(picks))))
    return np.array(sorted(picks), np.int64)
