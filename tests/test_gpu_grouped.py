"""Grouped forward (tensor-core GEMM and bandwidth GEMV, NF4 and MXFP4)
against the CPU oracle on the five workloads, their edge cases and the
device error word.  Tolerance (stated for the method): per element
|gpu - oracle| <= 1e-2 * rms(oracle row) + 1 bf16 ulp, fp32 accumulation."""
import ctypes as C

import numpy as np
import pytest
import torch

import oracle as orc
import synth
from parity import assert_rows_close, assert_rows_exact_operands, check_rows

pytestmark = pytest.mark.gpu

gbw = pytest.importorskip("grouped_bit_weight_b200")
from gpu_util import bits, packed_weights, sample_rows, to_dev  # noqa: E402

FWD = {"nf4": lambda *a, **k: gbw.gnf4_grouped_gemm(*a, **k),
       "mxfp4": lambda *a, **k: gbw.gmxfp4_grouped_gemm(*a, **k)}


def _run(fmt, x, codes, scale, off, r2t, mode):
    out = FWD[fmt](to_dev(x), to_dev(codes), to_dev(scale), to_dev(off),
                   None if r2t is None else to_dev(r2t), mode=mode)
    torch.cuda.synchronize()
    assert gbw.device_status() == 0
    return bits(out)


def _full_check(fmt, E, N, K, std, off, r2t, T, mode, seed=0, rel=1e-2):
    codes, scale, wdec = packed_weights(fmt, E, N, K, std, seed + 1)
    x = synth.to_bf16_bits(synth.normal((T, K), seed + 2))
    _, ref = orc.grouped_forward(x, wdec, off, r2t, want_f64=True)
    got = _run(fmt, x, codes, scale, off, r2t, mode)
    what = f"{fmt} {mode} E{E} N{N} K{K}"
    worst = assert_rows_close(got, ref, rel=rel, what=what)
    P = int(off[-1])
    if mode == "gemm" or (mode == "auto" and P > 4 * E):
        assert_rows_exact_operands(got, ref, what=what)
    return worst


@pytest.mark.parametrize("fmt", ["nf4", "mxfp4"])
@pytest.mark.parametrize("mode", ["gemm", "gemv", "auto"])
def test_tiny_config(fmt, mode):
    """64 tokens, top-2 of 8 experts, N=256, K=512 (weights N(0,1))."""
    off, r2t = synth.tiny_routing(0)
    _full_check(fmt, 8, 256, 512, 1.0, off, r2t, 64, mode)


@pytest.mark.parametrize("layer", [synth.QWEN_GATE_UP, synth.QWEN_DOWN])
@pytest.mark.parametrize("mode", ["auto", "gemm"])
def test_qwen_decode(layer, mode):
    """Qwen3-30B-A3B decode: one token routed to 8 of 128 experts."""
    off, r2t = synth.decode_routing(layer.E, 8, seed=3)
    T = 1 if layer is synth.QWEN_GATE_UP else 8
    if T == 8:  # down projection: one distinct activation row per routed row
        r2t = None
    _full_check("nf4", layer.E, layer.N, layer.K, layer.w_std, off, r2t, T, mode)


@pytest.mark.parametrize("fmt", ["nf4", "mxfp4"])
def test_gemv_experts_with_several_rows(fmt):
    """Experts with 2-8 routed rows next to single-row and empty ones: the
    GEMV reads each active expert's weights once and serves all its rows
    (forced, and picked by AUTO since P <= 4 E)."""
    E, N, K = 8, 512, 1024
    counts = np.array([2, 8, 1, 1, 3, 0, 5, 1], np.int32)
    off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    P = int(off[-1])
    r2t = np.random.default_rng(90).integers(0, 12, P).astype(np.int32)
    _full_check(fmt, E, N, K, 1.0, off, r2t, 12, "gemv", seed=91)
    _full_check(fmt, E, N, K, 1.0, off, None, P, "auto", seed=92)


@pytest.mark.parametrize("layer", [synth.QWEN_GATE_UP, synth.QWEN_DOWN])
def test_qwen_decode_batch(layer):
    """A decode batch of 4 tokens, top-8 of 128 experts: 32 routed rows,
    some experts with 2-3 of them; AUTO takes the GEMV (P <= 4 E)."""
    off, r2t = synth.uniform_routing(4, layer.E, 8, seed=93)
    assert np.diff(off).max() >= 2
    if layer is synth.QWEN_GATE_UP:
        _full_check("nf4", layer.E, layer.N, layer.K, layer.w_std, off, r2t, 4, "auto")
    else:
        _full_check("nf4", layer.E, layer.N, layer.K, layer.w_std, off, None, 32, "auto")


def _sampled_check(fmt, layer, off, r2t, T, mode, nrows, seed):
    codes, scale, wdec = packed_weights(fmt, layer.E, layer.N, layer.K, layer.w_std, seed + 1)
    x = synth.to_bf16_bits(synth.normal((T, layer.K), seed + 2))
    got = _run(fmt, x, codes, scale, off, r2t, mode)
    rows = sample_rows(off, nrows, seed)
    sp = np.repeat(rows, layer.N)
    sn = np.tile(np.arange(layer.N), len(rows))
    ref = orc.grouped_forward_sampled(x, wdec, off, r2t, sp, sn).reshape(len(rows), layer.N)
    worst = assert_rows_close(got[rows], ref, what=f"{layer.name} sampled")
    assert_rows_exact_operands(got[rows], ref, what=f"{layer.name} sampled")
    return worst


@pytest.mark.parametrize("layer", [synth.QWEN_GATE_UP, synth.QWEN_DOWN])
def test_qwen_prefill_full_size(layer):
    """Qwen3-30B-A3B prefill: 4096 tokens, top-8 of 128 with skewed counts
    and zero-row experts -> 32768 routed rows; sampled rows checked."""
    off, r2t = synth.prefill_routing()
    assert (np.diff(off) == 0).sum() >= 8
    if layer is synth.QWEN_GATE_UP:
        _sampled_check("nf4", layer, off, r2t, 4096, "auto", 48, 4)
    else:
        _sampled_check("nf4", layer, off, None, int(off[-1]), "auto", 48, 5)


@pytest.mark.parametrize("layer", [synth.GPTOSS_GATE_UP, synth.GPTOSS_DOWN])
@pytest.mark.parametrize("mode", ["auto", "gemm"])
def test_gptoss_batch1(layer, mode):
    """gpt-oss-20b MXFP4, one token routed to 4 of 32 experts."""
    off, r2t = synth.decode_routing(layer.E, 4, seed=6)
    _full_check("mxfp4", layer.E, layer.N, layer.K, layer.w_std, off, r2t, 1, mode)


@pytest.mark.parametrize("layer", [synth.GPTOSS_GATE_UP, synth.GPTOSS_DOWN])
def test_gptoss_batch2048_full_size(layer):
    off, r2t = synth.uniform_routing(2048, layer.E, 4, seed=7)
    _sampled_check("mxfp4", layer, off, r2t, 2048, "auto", 40, 7)


@pytest.mark.parametrize("fmt", ["nf4", "mxfp4"])
@pytest.mark.parametrize("mode", ["gemm", "gemv"])
def test_ragged_edges(fmt, mode):
    """Empty experts, one expert spanning 3 token tiles with a ragged tail,
    rows not a multiple of 4 or 16, N not a multiple of 128, K = 320."""
    E, N, K = 5, 200, 320
    counts = np.array([0, 601, 1, 0, 37], np.int32)
    off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    P = int(off[-1])
    r2t = np.random.default_rng(8).integers(0, 300, P).astype(np.int32)
    _full_check(fmt, E, N, K, 1.0, off, r2t, 300, mode, seed=9)
    _full_check(fmt, E, N, K, 1.0, off, None, P, mode, seed=10)


@pytest.mark.parametrize("K", [32, 352, 2912])
@pytest.mark.parametrize("mode", ["gemm", "auto"])
def test_mxfp4_k_tail_on_tensor_cores(K, mode):
    """MXFP4 with K % 64 == 32: the tensor-core GEMM runs its last 64-wide
    stage half full (AUTO takes the GEMM here too, P > 4 E).  Ragged experts
    over several token and weight tiles, gathered and identity rows, held to
    the exact-operand bound."""
    E, N = 5, 200
    counts = np.array([0, 601, 1, 0, 37], np.int32)
    off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    P = int(off[-1])
    r2t = np.random.default_rng(K).integers(0, 300, P).astype(np.int32)
    _full_check("mxfp4", E, N, K, 1.0, off, r2t, 300, mode, seed=K + 1)
    _full_check("mxfp4", E, N, K, 1.0, off, None, P, mode, seed=K + 2)


def test_single_expert_and_empty_batch():
    off = np.array([0, 130], np.int32)
    _full_check("nf4", 1, 64, 128, 1.0, off, None, 130, "gemm", seed=11)
    _full_check("nf4", 1, 64, 128, 1.0, off, None, 130, "gemv", seed=11)
    codes, scale, _ = packed_weights("nf4", 2, 64, 128, 1.0, 12)
    x = to_dev(synth.to_bf16_bits(synth.normal((4, 128), 1)))
    out = gbw.gnf4_grouped_gemm(x, to_dev(codes), to_dev(scale),
                                to_dev(np.zeros(3, np.int32)),
                                to_dev(np.zeros(0, np.int32)))
    assert out.shape == (0, 64)


def test_raw_c_abi_call():
    """The same grouped NF4 GEMM through ctypes with plain device pointers."""
    E, N, K = 4, 128, 256
    off, r2t = synth.uniform_routing(20, E, 2, seed=13)
    codes, scale, wdec = packed_weights("nf4", E, N, K, 1.0, 14)
    x = synth.to_bf16_bits(synth.normal((20, K), 15))
    P = int(off[-1])
    dx, dc, ds, do, dr = map(to_dev, (x, codes, scale, off, r2t))
    out = torch.empty((P, N), dtype=torch.bfloat16, device=dx.device)
    st = gbw.lib.gnf4_grouped_gemm(C.c_void_p(dx.data_ptr()), 20, K,
                                   C.c_void_p(dc.data_ptr()), C.c_void_p(ds.data_ptr()),
                                   E, N, C.c_void_p(do.data_ptr()), C.c_void_p(dr.data_ptr()),
                                   P, C.c_void_p(out.data_ptr()), gbw.MODE_GEMM,
                                   C.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0
    torch.cuda.synchronize()
    _, ref = orc.grouped_forward(x, wdec, off, r2t, want_f64=True)
    assert_rows_close(bits(out), ref, what="raw C ABI")


@pytest.mark.parametrize("mode", ["gemm", "gemv"])
def test_bad_offsets_and_tokens_raise_device_error(mode):
    """Decreasing / oversized offsets and out-of-range token ids are clamped
    in the kernels (nothing is read or written outside the buffers) and
    reported in the device error word."""
    E, N, K = 3, 64, 128
    codes, scale, _ = packed_weights("nf4", E, N, K, 1.0, 16)
    x = to_dev(synth.to_bf16_bits(synth.normal((10, K), 1)))
    bad_off = to_dev(np.array([0, 7, 3, 99], np.int32))   # P = 10
    r2t = to_dev(np.arange(10, dtype=np.int32))
    gbw.device_status(clear=True)
    gbw.gnf4_grouped_gemm(x, to_dev(codes), to_dev(scale), bad_off, r2t, mode=mode)
    assert gbw.device_status() & gbw.DEVERR_OFFSETS
    good_off = to_dev(np.array([0, 3, 6, 10], np.int32))
    bad_tok = to_dev(np.array([0, 1, 2, 3, 4, 5, 6, 7, 8, 1000], np.int32))
    gbw.gnf4_grouped_gemm(x, to_dev(codes), to_dev(scale), good_off, bad_tok, mode=mode)
    assert gbw.device_status() & gbw.DEVERR_TOKEN
    assert gbw.device_status() == 0  # cleared


@pytest.mark.parametrize("mode", ["gemm", "gemv"])
def test_corrupted_nibble_is_detected(mode):
    """Positive control: the GPU run on weights with one flipped code must
    fail the tolerance against the oracle of the intact weights."""
    E, N, K = 2, 64, 2048
    off, r2t = synth.uniform_routing(6, E, 1, seed=17)
    codes, scale, wdec = packed_weights("nf4", E, N, K, 1.0, 18)
    x = synth.to_bf16_bits(synth.normal((6, K), 19))
    _, ref = orc.grouped_forward(x, wdec, off, r2t, want_f64=True)
    e0 = int(np.searchsorted(off, 0, side="right") - 1)
    xf = orc.bf16_to_f32(x)[r2t[0]].astype(np.float64)
    wf = orc.nf4_decode(codes, scale, K)[e0, 0].astype(np.float64)
    k = int(np.argmax(np.abs(xf * wf)))
    bad = codes.copy()
    byte = int(bad[e0, 0, k // 2])
    q = (byte >> 4) if k % 2 == 0 else byte & 15
    bad[e0, 0, k // 2] = (((15 - q) << 4) | (byte & 15)) if k % 2 == 0 else ((byte & 0xF0) | (15 - q))
    got = _run("nf4", x, bad, scale, off, r2t, mode)
    ok, worst, n = check_rows(got, ref)
    assert n > 0 and not ok, worst
    assert check_rows(_run("nf4", x, codes, scale, off, r2t, mode), ref)[0]


def _device_layer(fmt, L, seed):
    gen = torch.Generator(device="cuda")
    gen.manual_seed(seed)
    if fmt == "mxfp4":
        codes = torch.empty((L.E, L.N, L.K // 32, 16), dtype=torch.uint8, device="cuda")
        sc = torch.empty((L.E, L.N, L.K // 32), dtype=torch.uint8, device="cuda")
        for e in range(L.E):
            c, s = gbw.gmxfp4_quantize(torch.randn((L.N, L.K), generator=gen, device="cuda") * L.w_std)
            codes[e].copy_(c)
            sc[e].copy_(s)
    else:
        codes = torch.empty((L.E, L.N, L.K // 2), dtype=torch.uint8, device="cuda")
        sc = torch.empty((L.E, L.N, L.K // 64), dtype=torch.float32, device="cuda")
        for e in range(L.E):
            c, s = gbw.gnf4_quantize(torch.randn((L.N, L.K), generator=gen, device="cuda") * L.w_std)
            codes[e].copy_(c)
            sc[e].copy_(s)
    return codes, sc, gen


@pytest.mark.parametrize("fmt,layer,tokens", [("mxfp4", synth.GPTOSS_GATE_UP, 2048),
                                               ("mxfp4", synth.GPTOSS_DOWN, 2048),
                                               ("nf4", synth.QWEN_GATE_UP, 4096)])
def test_repeatable_and_path_independent(fmt, layer, tokens):
    """The tensor-core path is deterministic: repeated launches give the same
    bits, and gathering rows through row_to_token gives exactly the bits of
    running on the pre-gathered rows (same decode, same MMA order).  A race
    in the pipeline shows up here long before it exceeds the tolerance."""
    if tokens == 4096:
        off, r2t = synth.prefill_routing()
    else:
        off, r2t = synth.uniform_routing(tokens, layer.E, 4, seed=7)
    codes, sc, gen = _device_layer(fmt, layer, 31)
    x = torch.randn((tokens, layer.K), generator=gen, device="cuda").to(torch.bfloat16)
    d_off, d_r2t = to_dev(off), to_dev(r2t)
    xg = x[d_r2t.long()].contiguous()
    fn = FWD[fmt]
    ref = fn(xg, codes, sc, d_off, None, mode="gemm")
    for _ in range(3):
        a = fn(x, codes, sc, d_off, d_r2t, mode="gemm")
        b = fn(xg, codes, sc, d_off, None, mode="gemm")
        torch.cuda.synchronize()
        assert torch.equal(a.view(torch.int16), ref.view(torch.int16))
        assert torch.equal(b.view(torch.int16), ref.view(torch.int16))
    assert gbw.device_status() == 0


@pytest.mark.parametrize("fmt", ["nf4", "mxfp4"])
def test_overlap_prev_chain_reads_x_after_the_previous_kernel(fmt):
    """Programmatic dependent launch: with overlap_prev=True the GEMV may read
    weights and routing while the kernel before it still runs, but x only
    after it.  Here each call's x is the previous call's output, so reading
    x early would use stale values; 50 chained launches must give exactly
    the bits of the same calls run one at a time."""
    E, N, K = 4, 512, 512
    codes, scale, _ = packed_weights(fmt, E, N, K, 0.05, 51)
    off = np.array([0, 2, 4, 6, 8], np.int32)  # 8 routed rows, 2 per expert
    fn = FWD[fmt]
    dc, ds, do = to_dev(codes), to_dev(scale), to_dev(off)
    x0 = to_dev(synth.to_bf16_bits(synth.normal((8, K), 52)))

    def chain(overlap, sync_each):
        x = x0
        for _ in range(50):
            x = fn(x, dc, ds, do, None, mode="gemv", overlap_prev=overlap)
            if sync_each:
                torch.cuda.synchronize()
        torch.cuda.synchronize()
        return bits(x)

    ref = chain(False, True)
    got = chain(True, False)
    assert gbw.device_status() == 0
    assert np.array_equal(got, ref)
    assert np.any(ref != 0)  # the chain did not decay to all zeros
