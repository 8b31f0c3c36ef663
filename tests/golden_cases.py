"""Loads the fixtures under tests/golden/: the pages' printed worked
examples and the hand-derived grouped-matmul cases (each file states its
source).  Builds the packed bytes, scales, activations and routing those
files describe; holds none of the method's arithmetic."""
from __future__ import annotations

import json
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def load(name: str) -> dict:
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _runs(runs, n):
    out = []
    for v, c in runs:
        out += [v] * c
    assert len(out) == n, (len(out), n)
    return out


def _x_row(desc: str, K: int) -> np.ndarray:
    if desc.startswith("k for"):
        return np.arange(K, dtype=np.float32)
    return np.full(K, float(desc.split()[0]), np.float32)


def hand_case(fmt: str):
    """-> dict with codes, scale, x (fp32, exact in bf16), offsets,
    row_to_token and the expected out (fp64), from hand_worked.json."""
    c = load("hand_worked.json")[fmt]
    E, N, K, T = c["E"], c["N"], c["K"], c["T"]
    nbytes = K // 2
    codes = np.zeros((E, N, nbytes), np.uint8)
    for e in range(E):
        for n in range(N):
            codes[e, n] = _runs(c["bytes"][f"e{e}r{n}"], nbytes)
    if fmt == "mxfp4":
        codes = codes.reshape(E, N, K // 32, 16)
        scale = np.array(c["scales"], np.uint8).reshape(E, N, K // 32)
    else:
        scale = np.array(c["absmax"], np.float32).reshape(E, N, K // 64)
    x = np.stack([_x_row(c["x"][f"t{t}"], K) for t in range(T)])
    return {"codes": codes, "scale": scale, "x": x,
            "offsets": np.array(c["expert_offsets"], np.int32),
            "row_to_token": np.array(c["row_to_token"], np.int32),
            "out": np.array(c["out"], np.float64), "K": K}
