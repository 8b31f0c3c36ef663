"""Grouped 4-bit activation gradient (NF4 and MXFP4) against the CPU oracle."""
import numpy as np
import pytest

import oracle as orc
import synth
from parity import assert_rows_close, assert_rows_exact_operands

pytestmark = pytest.mark.gpu

gbw = pytest.importorskip("grouped_bit_weight_b200")
from gpu_util import bits, packed_weights, sample_rows, to_dev  # noqa: E402


DGRAD = {"nf4": lambda *a: gbw.gnf4_grouped_dgrad(*a),
         "mxfp4": lambda *a: gbw.gmxfp4_grouped_dgrad(*a)}


def _dgrad(dy, codes, scale, off, fmt="nf4"):
    import torch
    dx = DGRAD[fmt](to_dev(dy), to_dev(codes), to_dev(scale), to_dev(off))
    torch.cuda.synchronize()
    assert gbw.device_status() == 0
    return bits(dx)


@pytest.mark.parametrize("fmt", ["nf4", "mxfp4"])
def test_tiny_dgrad(fmt):
    off, _ = synth.tiny_routing(0)
    codes, scale, wdec = packed_weights(fmt, 8, 256, 512, 1.0, 1)
    P = int(off[-1])
    dy = synth.to_bf16_bits(synth.normal((P, 256), 3, std=1e-2))
    _, ref = orc.grouped_dgrad(dy, wdec, off, want_f64=True)
    got = _dgrad(dy, codes, scale, off, fmt)
    assert_rows_close(got, ref, what=f"tiny {fmt} dgrad")
    assert_rows_exact_operands(got, ref, what=f"tiny {fmt} dgrad")


@pytest.mark.parametrize("fmt", ["nf4", "mxfp4"])
def test_dgrad_ragged_edges(fmt):
    """Empty experts, a 2-tile expert with a ragged tail (300 rows: one
    256-row tile over both accumulator halves, then 44 rows), a 5-row
    expert, K = 320 (the last output tile is 64 wide), N = 192."""
    E, N, K = 4, 192, 320
    counts = np.array([0, 300, 5, 0], np.int32)
    off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    codes, scale, wdec = packed_weights(fmt, E, N, K, 1.0, 2)
    dy = synth.to_bf16_bits(synth.normal((int(off[-1]), N), 4, std=1e-2))
    _, ref = orc.grouped_dgrad(dy, wdec, off, want_f64=True)
    got = _dgrad(dy, codes, scale, off, fmt)
    assert_rows_close(got, ref, what=f"ragged {fmt} dgrad")
    assert_rows_exact_operands(got, ref, what=f"ragged {fmt} dgrad")


@pytest.mark.parametrize("layer", [synth.QWEN_GATE_UP, synth.QWEN_DOWN])
def test_dgrad_full_size(layer):
    """Training dgrad on the Qwen3-30B-A3B prefill routing: dY [32768, N]
    N(0, 1e-2); sampled rows checked."""
    off, _ = synth.prefill_routing()
    codes, scale, wdec = packed_weights("nf4", layer.E, layer.N, layer.K, layer.w_std, 21)
    P = int(off[-1])
    dy = synth.to_bf16_bits(synth.normal((P, layer.N), 22, std=1e-2))
    got = _dgrad(dy, codes, scale, off)
    rows = sample_rows(off, 32, 23)
    sp = np.repeat(rows, layer.K)
    sk = np.tile(np.arange(layer.K), len(rows))
    ref = orc.grouped_dgrad_sampled(dy, wdec, off, sp, sk).reshape(len(rows), layer.K)
    assert_rows_close(got[rows], ref, what=f"{layer.name} dgrad")
    assert_rows_exact_operands(got[rows], ref, what=f"{layer.name} dgrad")


@pytest.mark.parametrize("layer", [synth.GPTOSS_GATE_UP, synth.GPTOSS_DOWN])
def test_mxfp4_dgrad_full_size(layer):
    """MXFP4 training dgrad at gpt-oss-20b expert shapes, 2048 tokens top-4
    of 32 (P = 8192); sampled rows checked."""
    off, _ = synth.uniform_routing(2048, layer.E, 4, seed=7)
    codes, scale, wdec = packed_weights("mxfp4", layer.E, layer.N, layer.K, layer.w_std, 31)
    P = int(off[-1])
    dy = synth.to_bf16_bits(synth.normal((P, layer.N), 32, std=1e-2))
    got = _dgrad(dy, codes, scale, off, "mxfp4")
    rows = sample_rows(off, 24, 33)
    sp = np.repeat(rows, layer.K)
    sk = np.tile(np.arange(layer.K), len(rows))
    ref = orc.grouped_dgrad_sampled(dy, wdec, off, sp, sk).reshape(len(rows), layer.K)
    assert_rows_close(got[rows], ref, what=f"{layer.name} mxfp4 dgrad")
    assert_rows_exact_operands(got[rows], ref, what=f"{layer.name} mxfp4 dgrad")


def test_dgrad_repeatable():
    """Repeated dgrad launches give identical bits (no pipeline races)."""
    import torch
    L = synth.QWEN_GATE_UP
    off, _ = synth.prefill_routing()
    P = int(off[-1])
    gen = torch.Generator(device="cuda")
    gen.manual_seed(41)
    codes = torch.empty((L.E, L.N, L.K // 2), dtype=torch.uint8, device="cuda")
    sc = torch.empty((L.E, L.N, L.K // 64), dtype=torch.float32, device="cuda")
    for e in range(L.E):
        c, s = gbw.gnf4_quantize(torch.randn((L.N, L.K), generator=gen, device="cuda") * L.w_std)
        codes[e].copy_(c)
        sc[e].copy_(s)
    dy = (torch.randn((P, L.N), generator=gen, device="cuda") * 1e-2).to(torch.bfloat16)
    d_off = to_dev(off)
    ref = gbw.gnf4_grouped_dgrad(dy, codes, sc, d_off)
    for _ in range(4):
        got = gbw.gnf4_grouped_dgrad(dy, codes, sc, d_off)
        torch.cuda.synchronize()
        assert torch.equal(got.view(torch.int16), ref.view(torch.int16))
    assert gbw.device_status() == 0
