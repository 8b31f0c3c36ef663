"""Seeded synthetic inputs: weights, activations and routing.

This module holds only random draws and routing structure (which routed row
goes to which expert).  It holds none of the packing, decoding or matmul
arithmetic, so both the GPU path and the CPU oracle can take their inputs
from it.  The source pages measure on Qwen3-30B-A3B- and gpt-oss-class MoE
layers with real checkpoints and real text; none of that is available here,
so these generators stand in for them with the same expert shapes.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np


def normal(shape, seed: int, std: float = 1.0) -> np.ndarray:
    """fp32 N(0, std^2) draws from numpy's PCG64 stream `seed`."""
    rng = np.random.default_rng(seed)
    out = rng.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        out *= np.float32(std)
    return out


def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 activations to bf16 (torch's cast) and return the uint16
    bit patterns the C ABI takes."""
    import torch

    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16).copy()


def route_uniform_topk(T: int, E: int, k: int, seed: int) -> np.ndarray:
    """Each of T tokens picks k distinct experts uniformly at random -> [T,k]."""
    rng = np.random.default_rng(seed)
    keys = rng.random((T, E))
    return np.argsort(keys, axis=1, kind="stable")[:, :k].astype(np.int32)


def route_softmax_topk(T: int, E: int, k: int, seed: int,
                       bias_std: float = 2.0, n_masked: int = 8) -> np.ndarray:
    """Skewed router: logits g[t,e] = N(0,1) + b_e with b_e = bias_std*N(0,1);
    the n_masked experts with the lowest b_e are masked out (they receive
    no rows); softmax over experts, then the top-k experts per token."""
    rng = np.random.default_rng(seed)
    b = bias_std * rng.standard_normal(E)
    g = rng.standard_normal((T, E)) + b[None, :]
    if n_masked:
        g[:, np.argsort(b, kind="stable")[:n_masked]] = -np.inf
    g = g - g.max(axis=1, keepdims=True)
    prob = np.exp(g)
    prob /= prob.sum(axis=1, keepdims=True)
    return np.argsort(-prob, axis=1, kind="stable")[:, :k].astype(np.int32)


def sort_routes(ids: np.ndarray, E: int):
    """Expert-sorted routed rows from per-token expert choices ids[T,k].

    Rows are ordered by (expert, token) -- a stable sort -- and row p of the
    result is token row_to_token[p] routed to expert e, where
    offsets[e] <= p < offsets[e+1].  Returns (offsets [E+1] int32,
    row_to_token [P] int32)."""
    T, k = ids.shape
    tok = np.repeat(np.arange(T, dtype=np.int64), k)
    exp = ids.reshape(-1).astype(np.int64)
    order = np.lexsort((tok, exp))
    counts = np.bincount(exp, minlength=E)
    offsets = np.zeros(E + 1, np.int32)
    offsets[1:] = np.cumsum(counts)
    return offsets, tok[order].astype(np.int32)


@dataclass(frozen=True)
class Layer:
    """One grouped projection: E experts of weight [N, K], P routed rows."""
    name: str
    fmt: str          # "nf4" or "mxfp4"
    E: int
    N: int
    K: int
    w_std: float


# The five workloads the build is measured and checked on.
TINY = Layer("tiny_nf4", "nf4", 8, 256, 512, 1.0)
QWEN_GATE_UP = Layer("qwen3_30b_a3b_gate_up", "nf4", 128, 1536, 2048, 0.02)
QWEN_DOWN = Layer("qwen3_30b_a3b_down", "nf4", 128, 2048, 768, 0.02)
GPTOSS_GATE_UP = Layer("gpt_oss_20b_gate_up", "mxfp4", 32, 5760, 2880, 0.02)
GPTOSS_DOWN = Layer("gpt_oss_20b_down", "mxfp4", 32, 2880, 2880, 0.02)


def tiny_routing(seed: int = 0):
    """64 tokens, top-2 uniform over 8 experts -> 128 routed rows."""
    return sort_routes(route_uniform_topk(64, 8, 2, seed), 8)


def decode_routing(E: int, k: int, seed: int, experts=None):
    """One token routed to k distinct experts (one row per expert)."""
    if experts is None:
        experts = route_uniform_topk(1, E, k, seed)[0]
    return sort_routes(np.asarray(experts, np.int32).reshape(1, k), E)


def prefill_routing(T: int = 4096, E: int = 128, k: int = 8, seed: int = 0):
    """Qwen3-30B-A3B-shaped prefill: softmax-of-Gaussian-logits top-8 with
    skewed counts and some zero-row experts."""
    return sort_routes(route_softmax_topk(T, E, k, seed), E)


def uniform_routing(T: int, E: int, k: int, seed: int = 0):
    return sort_routes(route_uniform_topk(T, E, k, seed), E)
