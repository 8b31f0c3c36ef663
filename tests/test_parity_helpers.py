"""The tolerance helpers the GPU tests use, checked on CPU: the SwiGLU
tolerance is the matmul tolerance of gate and up carried through
silu(g) * u, so it must accept exactly that perturbation and reject a
clearly larger one."""
import numpy as np

import oracle as orc
from parity import bf16_bits_to_f64, row_tolerance, swiglu_tolerance


def _h(g, u):
    return g / (1.0 + np.exp(-g)) * u


def test_swiglu_tolerance_covers_the_propagated_matmul_tolerance():
    rng = np.random.default_rng(0)
    gu = orc.f64_to_bf16(rng.standard_normal((4, 512)) * 3.0)
    g64 = bf16_bits_to_f64(gu)
    tol_gu = row_tolerance(g64)
    I = 256
    g, u = g64[:, :I], g64[:, I:]
    tol = swiglu_tolerance(gu)
    h = _h(g, u)
    # gate and up moved by (just under) their own matmul tolerance, in the
    # direction that moves h the most: inside the SwiGLU tolerance
    sg = np.sign((1 / (1 + np.exp(-g))) * (1 + g * (1 - 1 / (1 + np.exp(-g)))) * u)
    su = np.sign(g / (1 + np.exp(-g)))
    hp = _h(g + 0.99 * sg * tol_gu[:, :I], u + 0.99 * su * tol_gu[:, I:])
    assert np.all(np.abs(hp - h) <= tol * 1.05)
    # five times the matmul tolerance on gate alone is rejected somewhere
    hb = _h(g + 5 * sg * tol_gu[:, :I], u)
    assert np.any(np.abs(hb - h) > tol)


def test_swiglu_tolerance_is_a_few_percent_of_the_row():
    rng = np.random.default_rng(1)
    gu = orc.f64_to_bf16(rng.standard_normal((8, 1536)))
    g64 = bf16_bits_to_f64(gu)
    h = _h(g64[:, :768], g64[:, 768:])
    rms = np.sqrt(np.mean(h * h, axis=1, keepdims=True))
    ratio = np.median(swiglu_tolerance(gu) / rms)
    assert 0.005 < ratio < 0.05, ratio
