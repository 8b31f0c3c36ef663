"""Fused expert pass (gate_up -> SwiGLU -> down, NF4 and MXFP4) against the
CPU oracle's steps: the grouped gate_up matmul (bf16 out), the SwiGLU
combine (bf16 h) and the grouped down matmul over the same expert-sorted
rows.  Each step is held to its own tolerance:
  h    against the oracle's h, within the matmul tolerance of gate and up
       (1e-2 * rms(gate_up row) + 1 bf16 ulp) propagated through
       silu(g) * u, plus one bf16 ulp of h (parity.swiglu_tolerance);
  out  against the oracle's down matmul of the GPU's own h, within the
       matmul tolerance 1e-2 * rms(row) + 1 bf16 ulp.
A one-ulp flip of a rounded gate value moves h by silu'(g) * u * ulp(g),
which the plain matmul tolerance on h does not cover."""
import numpy as np
import pytest
import torch

import oracle as orc
import synth
from parity import (assert_close_to, assert_rows_close, bf16_bits_to_f64, check_rows,
                    swiglu_tolerance)

pytestmark = pytest.mark.gpu

gbw = pytest.importorskip("grouped_bit_weight_b200")
from gpu_util import bits, packed_weights, sample_rows, to_dev  # noqa: E402

FUSED = {"nf4": lambda *a, **k: gbw.gnf4_grouped_expert_mlp(*a, **k),
         "mxfp4": lambda *a, **k: gbw.gmxfp4_grouped_expert_mlp(*a, **k)}


def _run(fmt, x, gu, dn, off, r2t, mode):
    out, h = FUSED[fmt](to_dev(x), to_dev(gu[0]), to_dev(gu[1]), to_dev(dn[0]), to_dev(dn[1]),
                        to_dev(off), None if r2t is None else to_dev(r2t), mode=mode)
    torch.cuda.synchronize()
    assert gbw.device_status() == 0
    return bits(out), bits(h)


def _check(got, h, gu_ref, wdn, off, what):
    """h against the oracle's SwiGLU of its gate_up; out against the
    oracle's down matmul of the GPU's h."""
    href = orc.swiglu(gu_ref)
    assert_close_to(h, bf16_bits_to_f64(href), swiglu_tolerance(gu_ref), what=what + " h")
    _, ref = orc.grouped_forward(h, wdn, off, None, want_f64=True)
    return assert_rows_close(got, ref, what=what + " out")


def _full_check(fmt, E, H, I, std, off, r2t, T, mode, seed):
    gu = packed_weights(fmt, E, 2 * I, H, std, seed)
    dn = packed_weights(fmt, E, H, I, std, seed + 1)
    x = synth.to_bf16_bits(synth.normal((T, H), seed + 2))
    got, h = _run(fmt, x, gu, dn, off, r2t, mode)
    gu_ref = orc.grouped_forward(x, gu[2], off, r2t)
    return _check(got, h, gu_ref, dn[2], off, f"fused {fmt} {mode} E{E} H{H} I{I}")


@pytest.mark.parametrize("fmt", ["nf4", "mxfp4"])
@pytest.mark.parametrize("mode", ["auto", "gemm", "gemv"])
def test_fused_tiny(fmt, mode):
    """64 tokens, top-2 of 8 experts (128 routed rows), H=512, I=256."""
    off, r2t = synth.tiny_routing(0)
    _full_check(fmt, 8, 512, 256, 0.05, off, r2t, 64, mode, seed=61)


@pytest.mark.parametrize("fmt", ["nf4", "mxfp4"])
def test_fused_ragged(fmt):
    """Empty experts, one expert over three 256-row tiles with a ragged
    tail, H=320 and I=192 (odd numbers of 64-wide tiles), gathered and
    identity rows."""
    E, H, I = 5, 320, 192
    counts = np.array([0, 601, 1, 0, 37], np.int32)
    off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    P = int(off[-1])
    r2t = np.random.default_rng(62).integers(0, 300, P).astype(np.int32)
    _full_check(fmt, E, H, I, 0.05, off, r2t, 300, "auto", seed=63)
    _full_check(fmt, E, H, I, 0.05, off, None, P, "gemm", seed=64)


def test_fused_qwen_decode():
    """Qwen3-30B-A3B expert MLP, one token routed to 8 of 128 experts:
    gate_up [128, 1536, 2048], down [128, 2048, 768]."""
    GU, DN = synth.QWEN_GATE_UP, synth.QWEN_DOWN
    off, r2t = synth.decode_routing(GU.E, 8, seed=3)
    gu = packed_weights("nf4", GU.E, GU.N, GU.K, GU.w_std, 1)
    dn = packed_weights("nf4", DN.E, DN.N, DN.K, DN.w_std, 1)
    x = synth.to_bf16_bits(synth.normal((1, GU.K), 65))
    got, h = _run("nf4", x, gu, dn, off, r2t, "auto")
    _check(got, h, orc.grouped_forward(x, gu[2], off, r2t), dn[2], off, "qwen decode fused")


def test_fused_gptoss_decode():
    """gpt-oss-20b expert MLP in MXFP4, one token to 4 of 32 experts:
    gate_up [32, 5760, 2880], down [32, 2880, 2880]."""
    GU, DN = synth.GPTOSS_GATE_UP, synth.GPTOSS_DOWN
    off, r2t = synth.decode_routing(GU.E, 4, seed=6)
    gu = packed_weights("mxfp4", GU.E, GU.N, GU.K, GU.w_std, 1)
    dn = packed_weights("mxfp4", DN.E, DN.N, DN.K, DN.w_std, 1)
    x = synth.to_bf16_bits(synth.normal((1, GU.K), 66))
    got, h = _run("mxfp4", x, gu, dn, off, r2t, "auto")
    _check(got, h, orc.grouped_forward(x, gu[2], off, r2t), dn[2], off, "gpt-oss decode fused")


def test_fused_qwen_prefill_sampled():
    """Qwen3-30B-A3B prefill (4096 tokens, skewed top-8 routing with empty
    experts, 32768 routed rows); sampled rows checked: the oracle's gate_up
    for those rows (all 1536 columns, rounded to bf16), its SwiGLU, then its
    down matmul for the same rows."""
    GU, DN = synth.QWEN_GATE_UP, synth.QWEN_DOWN
    off, r2t = synth.prefill_routing()
    gu = packed_weights("nf4", GU.E, GU.N, GU.K, GU.w_std, 1)
    dn = packed_weights("nf4", DN.E, DN.N, DN.K, DN.w_std, 1)
    x = synth.to_bf16_bits(synth.normal((4096, GU.K), 67))
    got, h = _run("nf4", x, gu, dn, off, r2t, "auto")
    rows = sample_rows(off, 48, 68)
    sp = np.repeat(rows, GU.N)
    sn = np.tile(np.arange(GU.N), len(rows))
    gu_rows = orc.f64_to_bf16(orc.grouped_forward_sampled(x, gu[2], off, r2t, sp, sn))
    experts = np.searchsorted(off, rows, side="right") - 1
    off_r = np.searchsorted(experts, np.arange(GU.E + 1), side="left").astype(np.int32)
    _check(got[rows], h[rows], gu_rows.reshape(len(rows), GU.N), dn[2], off_r,
           "qwen prefill fused (sampled)")


def test_fused_corrupted_gate_code_is_detected():
    """Positive control: one flipped gate code of a routed row's expert must
    push that row past the tolerance."""
    E, H, I = 2, 512, 128
    off, r2t = synth.uniform_routing(6, E, 1, seed=69)
    gu = packed_weights("nf4", E, 2 * I, H, 0.05, 70)
    dn = packed_weights("nf4", E, H, I, 0.05, 71)
    x = synth.to_bf16_bits(synth.normal((6, H), 72))
    _, ref = orc.grouped_forward(orc.swiglu(orc.grouped_forward(x, gu[2], off, r2t)), dn[2], off,
                                 None, want_f64=True)
    e0 = int(np.searchsorted(off, 0, side="right") - 1)
    bad = gu[0].copy()
    bad[e0, :I] ^= 0x88   # flip the sign bit of every gate code of expert e0
    got, _ = _run("nf4", x, (bad, gu[1]), dn, off, r2t, "auto")
    ok, worst, n = check_rows(got, ref)
    assert n > 0 and not ok, worst
