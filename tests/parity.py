"""Parity helpers shared by the tests: the tolerance the grouped matmuls
must meet against the oracle, and checks that a comparison is not vacuous."""
from __future__ import annotations

import numpy as np


def bf16_bits_to_f64(h) -> np.ndarray:
    h = np.ascontiguousarray(h, dtype=np.uint16)
    return (h.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def bf16_ulp(v) -> np.ndarray:
    """Spacing of bf16 numbers at |v| (8 significant bits; subnormal floor)."""
    a = np.abs(np.asarray(v, np.float64))
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -126)))
    return np.exp2(e - 7)


def row_tolerance(oracle_f64: np.ndarray, rel: float = 1e-2) -> np.ndarray:
    """|gpu - oracle| <= rel * rms(oracle row) + 1 bf16 ulp(oracle value),
    elementwise; rows are the last axis."""
    o = np.asarray(oracle_f64, np.float64)
    rms = np.sqrt(np.mean(o * o, axis=-1, keepdims=True)) if o.shape[-1] else 0.0
    return rel * rms + bf16_ulp(o)


def check_rows(gpu_bf16_bits, oracle_f64, rel: float = 1e-2):
    """Returns (ok, worst normalised error, number of elements compared).
    Raises if nothing was compared (an empty comparison is not a pass)."""
    g = bf16_bits_to_f64(gpu_bf16_bits)
    o = np.asarray(oracle_f64, np.float64)
    assert g.shape == o.shape, (g.shape, o.shape)
    if o.size == 0:
        raise AssertionError("empty comparison")
    tol = row_tolerance(o, rel)
    err = np.abs(g - o)
    bad = ~(err <= tol)  # NaN counts as bad
    worst = float(np.max(err / tol))
    return (not bool(bad.any())), worst, int(o.size)


def assert_rows_close(gpu_bf16_bits, oracle_f64, rel: float = 1e-2, what=""):
    ok, worst, n = check_rows(gpu_bf16_bits, oracle_f64, rel)
    assert ok, f"{what}: {n} elements, worst |err|/tol = {worst:.3g} (> 1)"
    return worst


def assert_rows_exact_operands(gpu_bf16_bits, oracle_f64, rel_acc=1e-4, what=""):
    """Stricter check for paths whose bf16 operands equal the oracle's decoded
    weights exactly: the only differences left are fp32 accumulation order
    (bounded here by rel_acc * rms(row)) and the final rounding to bf16
    (half an ulp of the value).  A weight decoded even 2^-9 off would move
    outputs by ~1e-3 * rms and fail."""
    g = bf16_bits_to_f64(gpu_bf16_bits)
    o = np.asarray(oracle_f64, np.float64)
    assert g.shape == o.shape and o.size > 0
    rms = np.sqrt(np.mean(o * o, axis=-1, keepdims=True))
    bound = 0.5 * np.maximum(bf16_ulp(o), bf16_ulp(g)) + rel_acc * rms
    err = np.abs(g - o)
    ratio = float(np.max(err / bound))
    assert np.all(err <= bound), f"{what}: worst |err|/bound = {ratio:.3g}"
    return ratio


def swiglu_tolerance(gu_bf16_bits, rel: float = 1e-2) -> np.ndarray:
    """Per-element tolerance of h = bf16(silu(gate) * up) computed from a
    gate_up output that is itself only fixed within the matmul tolerance:
    that tolerance (rel * rms(gate_up row) + 1 ulp, which also covers a bf16
    rounding of gate or up that lands one ulp away) propagated through
    silu(g) * u to second order, plus one bf16 ulp of h.  gu [P, 2I] holds the
    oracle's gate (columns [0, I)) and up ([I, 2I)) values."""
    gu = bf16_bits_to_f64(gu_bf16_bits)
    tol = row_tolerance(gu, rel)
    I = gu.shape[-1] // 2
    g, u, tg, tu = gu[..., :I], gu[..., I:], tol[..., :I], tol[..., I:]
    sig = 1.0 / (1.0 + np.exp(-g))
    silu = g * sig
    dsilu = sig * (1.0 + g * (1.0 - sig))
    # first order, plus the second-order terms (cross term silu'(g) dg du and
    # the curvature of silu, |silu''| <= 1/2) that matter near g, u ~ 0
    return (np.abs(dsilu * u) * tg + np.abs(silu) * tu + np.abs(dsilu) * tg * tu
            + 0.25 * tg * tg * (np.abs(u) + tu) + bf16_ulp(silu * u))


def assert_close_to(gpu_bf16_bits, oracle_f64, tol, what=""):
    """|gpu - oracle| <= tol elementwise (a non-empty comparison)."""
    g = bf16_bits_to_f64(gpu_bf16_bits)
    o = np.asarray(oracle_f64, np.float64)
    assert g.shape == o.shape and o.size > 0, (g.shape, o.shape)
    err = np.abs(g - o)
    worst = float(np.max(err / tol))
    assert np.all(err <= tol), f"{what}: {o.size} elements, worst |err|/tol = {worst:.3g}"
    return worst
