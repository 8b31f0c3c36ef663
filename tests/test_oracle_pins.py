"""Pins the CPU oracle to facts that do not come from the oracle itself:
numbers the source pages print, the QLoRA and OCP MX definitions, closed
forms, library routines and brute force.  CPU only."""
from __future__ import annotations

import numpy as np
import pytest
import torch
from scipy.stats import norm

import oracle as orc
import synth
from parity import bf16_bits_to_f64, check_rows

# OCP MX v1.0, FP4 E2M1: the eight magnitudes, codes 0..7.
OCP_E2M1 = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


# ----------------------------------------------------------------- bf16

def test_f32_to_bf16_matches_torch_cast():
    rng = np.random.default_rng(1)
    bits = rng.integers(0, 2**32, size=20000, dtype=np.uint64).astype(np.uint32)
    vals = bits.view(np.float32)
    vals = vals[np.isfinite(vals)]
    specials = np.array([0.0, -0.0, 1.0, 1.00390625, 1.005859375, 3.0e38,
                         3.4e38, 1e-40, -1e-45, np.inf, -np.inf], np.float32)
    vals = np.concatenate([vals, specials])
    want = torch.from_numpy(vals).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = orc.f32_to_bf16(vals)
    assert np.array_equal(got, want)


def _bf16_value(h):
    return float(bf16_bits_to_f64(np.array([h], np.uint16))[0])


def test_f64_to_bf16_is_nearest_with_ties_to_even():
    rng = np.random.default_rng(2)
    xs = list(rng.standard_normal(3000) * np.exp2(rng.integers(-140, 120, 3000)))
    # exact midpoints between neighbouring bf16 values (ties)
    xs += [1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -(2.0 + 2.0 ** -7), 2.0 ** -134,
           3 * 2.0 ** -134]
    for x in xs:
        h = int(orc.f64_to_bf16(np.array([x]))[0])
        v = _bf16_value(h)
        up = _bf16_value((h + 1) & 0xFFFF) if (h & 0x7FFF) != 0x7F7F else np.inf
        dn = _bf16_value(h - 1) if (h & 0x7FFF) != 0 else -v
        # no representable value strictly closer than the chosen one
        assert abs(x - v) <= abs(x - up) and abs(x - v) <= abs(x - dn), x
        if abs(x - v) in (abs(x - up), abs(x - dn)) and abs(x - v) > 0:
            assert h % 2 == 0, x  # tie -> even last bit


def test_f64_to_bf16_avoids_double_rounding():
    # 1 + 2^-8 + 2^-30 is above the midpoint of (1, 1+2^-7): must round up.
    # Rounding to fp32 first would land exactly on the midpoint and go even.
    x = 1.0 + 2.0 ** -8 + 2.0 ** -30
    assert orc.f64_to_bf16(np.array([x]))[0] == 0x3F81


# ------------------------------------------------------------------ NF4

def test_nf4_codebook_is_the_qlora_table():
    c = orc.nf4_codebook().astype(np.float64)
    assert c[0] == -1.0 and c[15] == 1.0 and c[7] == 0.0
    assert np.all(np.diff(c) > 0)
    # QLoRA's construction: normal quantiles, 8 positive and 7 negative, plus 0,
    # scaled by the largest.  The published fp32 table matches it to ~2e-7.
    off = 1 - 0.5 * (1 / 32 + 1 / 30)
    pos = norm.ppf(np.linspace(off, 0.5, 9)[:-1])
    neg = -norm.ppf(np.linspace(off, 0.5, 8)[:-1])
    v = np.sort(np.concatenate([pos, [0.0], neg]))
    v = v / v.max()
    assert np.max(np.abs(v - c)) < 2e-7


def test_nf4_page_example_roundtrip():
    """pypi page, example 1: w = randn(256, 512); packed [256,256] u8 and
    absmax [256,8] fp32; rel-err ~0.09; re-pack of the decoded weights is
    byte-identical."""
    w = synth.normal((256, 512), seed=0)
    packed, absmax = orc.nf4_pack(w)
    assert packed.shape == (256, 256) and packed.dtype == np.uint8
    assert absmax.shape == (256, 8) and absmax.dtype == np.float32
    wq = orc.nf4_decode(packed, absmax, 512)
    rel = np.linalg.norm(wq - w) / np.linalg.norm(w)
    assert round(float(rel), 2) == 0.09, rel
    p2, a2 = orc.nf4_pack(wq)
    assert np.array_equal(p2, packed) and np.array_equal(a2, absmax)


def test_nf4_nibble_order_and_endpoints():
    # High nibble = even k (bitsandbytes layout): byte 0x0F -> (-a, +a).
    a = np.float32(2.5)
    packed = np.full((1, 32), 0x0F, np.uint8)
    w = orc.nf4_decode(packed, np.array([[a]], np.float32), 64)
    assert np.all(w[0, 0::2] == -a) and np.all(w[0, 1::2] == a)
    packed[:] = 0x7F
    w = orc.nf4_decode(packed, np.array([[a]], np.float32), 64)
    assert np.all(w[0, 0::2] == 0.0) and np.all(w[0, 1::2] == a)


def test_nf4_decode_exhaustive_closed_form():
    c = orc.nf4_codebook()
    scales = np.array([1.0, 0.037, 3.9e-3, 1234.5, 2.0 ** -120], np.float32)
    allbytes = np.arange(256, dtype=np.uint8)
    packed = np.tile(allbytes, (len(scales), 1)).reshape(len(scales) * 8, 32)
    absmax = np.repeat(scales, 8).reshape(-1, 1)
    w = orc.nf4_decode(packed, absmax, 64).reshape(len(scales), 512)
    wb = orc.nf4_decode(packed, absmax, 64, bf16=True).reshape(len(scales), 512)
    for i, s in enumerate(scales):
        hi = c[allbytes >> 4] * s
        lo = c[allbytes & 15] * s
        want = np.stack([hi, lo], axis=1).reshape(-1).astype(np.float32)
        assert np.array_equal(w[i], want)
        wt = torch.from_numpy(want).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        assert np.array_equal(wb[i], wt)


def test_nf4_pack_exact_codes_and_blocks():
    rng = np.random.default_rng(3)
    c = orc.nf4_codebook()
    q = rng.integers(0, 16, size=(4, 128))
    q[:, 0] = 15  # each 64-block holds an endpoint, so its absmax is a
    q[:, 64] = 0
    a = np.array([[0.5, 2.0], [1.0, 8.0], [0.25, 0.125], [4.0, 1.0]], np.float32)
    w = (c[q] * np.repeat(a, 64, axis=1)).astype(np.float32)
    packed, absmax = orc.nf4_pack(w)
    assert np.array_equal(absmax, a)
    got = np.stack([packed >> 4, packed & 15], axis=-1).reshape(4, 128)
    assert np.array_equal(got, q)


def test_nf4_pack_zero_block_ties_and_errors():
    w = np.zeros((2, 64), np.float32)
    w[1, 5] = -3.0
    packed, absmax = orc.nf4_pack(w)
    assert absmax[0, 0] == 0 and np.all(packed[0] == 0x77)
    assert absmax[1, 0] == 3.0 and (packed[1, 2] & 15) == 0  # k=5: low nibble
    # a value exactly halfway between two codes takes the lower code
    c = orc.nf4_codebook().astype(np.float64)
    for i in range(15):
        mid = np.float32((c[i] + c[i + 1]) / 2)
        if abs(np.float64(mid) - c[i]) != abs(c[i + 1] - np.float64(mid)):
            continue  # midpoint not representable in fp32
        blk = np.zeros((1, 64), np.float32)
        blk[0, 0] = 1.0
        blk[0, 2] = mid
        p, _ = orc.nf4_pack(blk)
        assert (p[0, 1] >> 4) == i
    with pytest.raises(orc.OracleError):
        orc.nf4_pack(np.full((1, 64), np.nan, np.float32))
    with pytest.raises(orc.OracleError):
        orc.nf4_pack(np.zeros((1, 32), np.float32))


# ---------------------------------------------------------------- MXFP4

def test_mxfp4_page_example_roundtrip():
    """pypi page, example 2: w = randn(128, 256); blocks [128,8,16] u8,
    scales [128,8] u8 (e8m0); rel-err ~0.12."""
    w = synth.normal((128, 256), seed=0)
    blocks, scales = orc.mxfp4_pack(w)
    assert blocks.shape == (128, 8, 16) and blocks.dtype == np.uint8
    assert scales.shape == (128, 8) and scales.dtype == np.uint8
    wq = orc.mxfp4_decode(blocks, scales)
    rel = np.linalg.norm(wq - w) / np.linalg.norm(w)
    assert round(float(rel), 2) == 0.12, rel
    b2, s2 = orc.mxfp4_pack(wq)  # derived invariant: re-pack is idempotent
    assert np.array_equal(b2, blocks) and np.array_equal(s2, scales)


def test_mxfp4_decode_matches_ocp_table():
    codes = np.arange(16)
    byte = (codes | (codes << 4)).astype(np.uint8)  # both nibbles = code
    for s, f in [(127, 1.0), (130, 8.0), (120, 2.0 ** -7), (1, 2.0 ** -126)]:
        blocks = np.zeros((1, 1, 16), np.uint8)
        blocks[0, 0, :] = byte
        w = orc.mxfp4_decode(blocks, np.array([[s]], np.uint8))[0]
        want = np.array([(-1) ** (c >> 3) * OCP_E2M1[c & 7] * f for c in codes],
                        np.float64)
        assert np.array_equal(w[0::2].astype(np.float64), want), s
        assert np.array_equal(w[1::2].astype(np.float64), want), s
    w = orc.mxfp4_decode(np.zeros((1, 1, 16), np.uint8) + 0x22,
                         np.array([[255]], np.uint8))
    assert np.all(np.isnan(w))


def test_mxfp4_pack_scale_rule_nibbles_and_ties():
    blk = np.zeros((1, 32), np.float32)
    blk[0, 0] = 6.0
    blk[0, 1] = 0.5
    b, s = orc.mxfp4_pack(blk)
    # amax 6 -> X = floor(log2 6) - 2 = 0 -> byte 127; even k in the LOW nibble
    assert s[0, 0] == 127 and b[0, 0, 0] == (7 | (1 << 4))
    # ties go to the even code: 0.25->0, 0.75->1.0, 1.25->1.0, 1.75->2,
    # 2.5->2, 3.5->4, 5->4; past 6 saturates; sign kept
    vals = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 7.9, -0.75, -5.0]
    want = [0, 2, 2, 4, 4, 6, 6, 7, 8 | 2, 8 | 6]
    blk = np.zeros((1, 32), np.float32)
    blk[0, 31] = 7.9  # amax 7.9 -> X = 0 as well
    blk[0, :len(vals)] = vals
    b, s = orc.mxfp4_pack(blk)
    assert s[0, 0] == 127
    codes = np.stack([b[0, 0] & 15, b[0, 0] >> 4], axis=-1).reshape(-1)
    assert list(codes[:len(vals)]) == want
    # scale tracks the block maximum: amax = 1 -> X = -2 -> byte 125
    blk = np.full((1, 32), 0.25, np.float32)
    blk[0, 3] = 1.0
    b, s = orc.mxfp4_pack(blk)
    assert s[0, 0] == 125
    # all-zero block: byte 0, codes 0
    b, s = orc.mxfp4_pack(np.zeros((1, 32), np.float32))
    assert s[0, 0] == 0 and np.all(b == 0)
    with pytest.raises(orc.OracleError):
        orc.mxfp4_pack(np.zeros((1, 48), np.float32))


# ------------------------------------------------------- grouped matmuls

def _tiny_problem(seed=0, E=4, N=24, K=128, T=10, k=2, fmt="nf4"):
    ids = synth.route_uniform_topk(T, E, k, seed)
    off, r2t = synth.sort_routes(ids, E)
    w = synth.normal((E, N, K), seed + 1)
    if fmt == "nf4":
        p, a = orc.nf4_pack(w)
        wd = orc.nf4_decode(p, a, K, bf16=True)
    else:
        b, s = orc.mxfp4_pack(w)
        wd = orc.mxfp4_decode(b, s, bf16=True)
    x = synth.to_bf16_bits(synth.normal((T, K), seed + 2))
    return x, wd, off, r2t


@pytest.mark.parametrize("fmt", ["nf4", "mxfp4"])
def test_grouped_forward_equals_per_expert_matmul(fmt):
    x, wd, off, r2t = _tiny_problem(fmt=fmt)
    out, o64 = orc.grouped_forward(x, wd, off, r2t, want_f64=True)
    xf = bf16_bits_to_f64(x)
    wf = bf16_bits_to_f64(wd)
    want = np.zeros_like(o64)
    for e in range(wd.shape[0]):
        rows = slice(off[e], off[e + 1])
        want[rows] = xf[r2t[rows]] @ wf[e].T
    assert np.allclose(o64, want, rtol=1e-12, atol=1e-12)
    assert np.array_equal(out, orc.f64_to_bf16(o64))


def test_grouped_forward_empty_experts_and_empty_batch():
    x, wd, _, _ = _tiny_problem()
    E = wd.shape[0]
    off = np.array([0, 0, 3, 3, 5], np.int32)  # experts 0 and 2 get no rows
    r2t = np.array([4, 1, 7, 0, 9], np.int32)
    out, o64 = orc.grouped_forward(x, wd, off, r2t, want_f64=True)
    xf, wf = bf16_bits_to_f64(x), bf16_bits_to_f64(wd)
    assert np.allclose(o64[:3], xf[r2t[:3]] @ wf[1].T)
    assert np.allclose(o64[3:], xf[r2t[3:]] @ wf[3].T)
    z = orc.grouped_forward(x, wd, np.zeros(E + 1, np.int32), np.zeros(0, np.int32))
    assert z.shape == (0, wd.shape[1])
    with pytest.raises(orc.OracleError):
        orc.grouped_forward(x, wd, np.array([0, 3, 2, 4, 5], np.int32), r2t)


def test_grouped_forward_expert_relabelling_invariance():
    x, wd, off, r2t = _tiny_problem(E=5)
    out = orc.grouped_forward(x, wd, off, r2t)
    perm = np.array([3, 0, 4, 1, 2])  # new expert i holds old expert perm[i]
    counts = np.diff(off)
    new_off = np.concatenate([[0], np.cumsum(counts[perm])]).astype(np.int32)
    new_r2t = np.concatenate([r2t[off[e]:off[e + 1]] for e in perm])
    out2 = orc.grouped_forward(x, wd[perm], new_off, new_r2t)
    old_rows = np.concatenate([np.arange(off[e], off[e + 1]) for e in perm])
    assert np.array_equal(out2, out[old_rows])


@pytest.mark.parametrize("fmt", ["nf4", "mxfp4"])
def test_grouped_dgrad_brute_force_and_adjoint(fmt):
    x, wd, off, r2t = _tiny_problem(fmt=fmt, T=12)
    P = int(off[-1])
    N, K = wd.shape[1], wd.shape[2]
    dy = synth.to_bf16_bits(synth.normal((P, N), 9, std=1e-2))
    dx, d64 = orc.grouped_dgrad(dy, wd, off, want_f64=True)
    dyf, wf = bf16_bits_to_f64(dy), bf16_bits_to_f64(wd)
    want = np.zeros((P, K))
    for e in range(wd.shape[0]):
        rows = slice(off[e], off[e + 1])
        want[rows] = dyf[rows] @ wf[e]
    assert np.allclose(d64, want, rtol=1e-12, atol=1e-14)
    assert np.array_equal(dx, orc.f64_to_bf16(d64))
    # adjoint identity <dy, X W^T> = <dy W, X> with X the gathered rows
    xs = x[r2t]
    _, fwd = orc.grouped_forward(xs, wd, off, None, want_f64=True)
    lhs = float(np.sum(dyf * fwd))
    rhs = float(np.sum(d64 * bf16_bits_to_f64(xs)))
    assert abs(lhs - rhs) <= 1e-10 * (abs(lhs) + 1e-30) + 1e-15


def test_sampled_evaluations_agree_with_full():
    x, wd, off, r2t = _tiny_problem(T=16)
    _, o64 = orc.grouped_forward(x, wd, off, r2t, want_f64=True)
    P, N = o64.shape
    rng = np.random.default_rng(5)
    sp, sn = rng.integers(0, P, 50), rng.integers(0, N, 50)
    s = orc.grouped_forward_sampled(x, wd, off, r2t, sp, sn)
    assert np.array_equal(s, o64[sp, sn])
    dy = synth.to_bf16_bits(synth.normal((P, N), 4))
    _, d64 = orc.grouped_dgrad(dy, wd, off, want_f64=True)
    sk = rng.integers(0, wd.shape[2], 50)
    s = orc.grouped_dgrad_sampled(dy, wd, off, sp, sk)
    assert np.array_equal(s, d64[sp, sk])


def test_parity_check_has_teeth():
    """Positive control: one corrupted nibble in the packed weights must make
    the row-tolerance comparison fail (a gate that cannot fail proves
    nothing)."""
    E, N, K, T = 2, 16, 2048, 6
    ids = synth.route_uniform_topk(T, E, 1, 0)
    off, r2t = synth.sort_routes(ids, E)
    w = synth.normal((E, N, K), 1)
    p, a = orc.nf4_pack(w)
    x = synth.to_bf16_bits(synth.normal((T, K), 2))
    good = orc.grouped_forward(x, orc.nf4_decode(p, a, K, bf16=True), off, r2t)
    _, ref = orc.grouped_forward(x, orc.nf4_decode(p, a, K, bf16=True), off, r2t,
                                 want_f64=True)
    assert check_rows(good, ref)[0]
    # corrupt the nibble of row 0's largest product: code q -> 15 - q
    e0 = int(np.searchsorted(off, 0, side="right") - 1)  # expert of row 0
    xf = bf16_bits_to_f64(x)[r2t[0]]
    wf = orc.nf4_decode(p, a, K)[e0]
    kk = int(np.argmax(np.abs(xf * wf[0])))
    bad = p.copy()
    byte = int(bad[e0, 0, kk // 2])
    q = (byte >> 4) if kk % 2 == 0 else (byte & 15)
    q2 = 15 - q
    bad[e0, 0, kk // 2] = ((q2 << 4) | (byte & 15)) if kk % 2 == 0 else ((byte & 0xF0) | q2)
    corrupt = orc.grouped_forward(x, orc.nf4_decode(bad, a, K, bf16=True), off, r2t)
    ok, worst, n = check_rows(corrupt, ref)
    assert n > 0 and not ok, worst
    with pytest.raises(AssertionError):
        check_rows(np.zeros((0, 4), np.uint16), np.zeros((0, 4)))


# ------------------------------------------------------ golden fixtures

def test_page_examples_fixture():
    """The packers' printed worked examples (tests/golden/page_examples.json:
    'grouped-nf4-gemm 0.43.0', 'Try the packers and byte checks on CPU',
    examples 1 and 2): shapes, dtypes, the rounded relative error and the
    byte-identical re-pack, on this repository's own N(0,1) draws."""
    from golden_cases import load
    g = load("page_examples.json")
    n = g["nf4"]
    w = synth.normal(tuple(n["w_shape"]), seed=0)
    p, a = orc.nf4_pack(w)
    assert list(p.shape) == n["packed_shape"] and p.dtype == np.dtype(n["packed_dtype"])
    assert list(a.shape) == n["absmax_shape"] and a.dtype == np.dtype(n["absmax_dtype"])
    wq = orc.nf4_decode(p, a, n["w_shape"][1])
    rel = np.linalg.norm(wq - w) / np.linalg.norm(w)
    assert round(float(rel), n["rel_err_digits"]) == n["rel_err_printed"], rel
    assert np.array_equal(orc.nf4_pack(wq)[0], p) == n["repack_identical"]
    m = g["mxfp4"]
    w = synth.normal(tuple(m["w_shape"]), seed=0)
    b, s = orc.mxfp4_pack(w)
    assert list(b.shape) == m["blocks_shape"] and b.dtype == np.dtype(m["blocks_dtype"])
    assert list(s.shape) == m["scales_shape"] and s.dtype == np.dtype(m["scales_dtype"])
    wq = orc.mxfp4_decode(b, s)
    rel = np.linalg.norm(wq - w) / np.linalg.norm(w)
    assert round(float(rel), m["rel_err_digits"]) == m["rel_err_printed"], rel


@pytest.mark.parametrize("fmt", ["nf4", "mxfp4"])
def test_hand_worked_grouped_matmul(fmt):
    """tests/golden/hand_worked.json: bytes, scales, activations and routing
    chosen so every product and sum is exact, with the outputs derived by
    hand.  A flipped nibble order, a wrong sign bit, a scale off by one
    power of two or a routing slip changes at least one of them."""
    from golden_cases import hand_case
    c = hand_case(fmt)
    if fmt == "nf4":
        wd = orc.nf4_decode(c["codes"], c["scale"], c["K"], bf16=True)
    else:
        wd = orc.mxfp4_decode(c["codes"], c["scale"], bf16=True)
    x = orc.f32_to_bf16(c["x"])
    out, o64 = orc.grouped_forward(x, wd, c["offsets"], c["row_to_token"], want_f64=True)
    assert np.array_equal(o64, c["out"])
    assert np.array_equal(bf16_bits_to_f64(out), c["out"])


# ------------------------------------------------------- SwiGLU, fused pass

def _bf16_bits(a64):
    """fp64 -> bf16 bits with one rounding, by the oracle's f64_to_bf16,
    which test_f64_to_bf16_is_nearest_with_ties_to_even pins by brute force
    (torch's fp64 -> bf16 cast rounds twice, through fp32, so it cannot serve
    as the reference here)."""
    a = np.array(a64, np.float64)
    return orc.f64_to_bf16(a.ravel()).reshape(a.shape)


def test_swiglu_closed_forms():
    """silu(0) = 0, silu(1) = 1 / (1 + e^-1), silu(-1) = -e^-1 / (1 + e^-1);
    up = 0 gives 0; a large gate passes up through (silu(20) = 20 to bf16);
    gate columns come first, up columns second."""
    e1 = np.exp(-1.0)
    gate = np.array([0.0, 1.0, -1.0, 3.0, 20.0, 1.0], np.float64)
    up = np.array([5.0, 1.0, 1.0, 0.0, 0.5, 2.0], np.float64)
    gu = _bf16_bits(np.concatenate([gate, up])[None, :])
    h = bf16_bits_to_f64(orc.swiglu(gu))[0]
    want = [0.0, 1.0 / (1.0 + e1), -e1 / (1.0 + e1), 0.0, 10.0, 2.0 / (1.0 + e1)]
    got_bits = orc.swiglu(gu)[0]
    assert np.array_equal(got_bits[[1, 2, 5]], _bf16_bits(np.array(want)[[1, 2, 5]]))
    assert h[0] == 0.0 and h[3] == 0.0 and h[4] == 10.0
    # swapping the halves changes the result: the layout is [gate | up]
    swapped = _bf16_bits(np.concatenate([up, gate])[None, :])
    assert not np.array_equal(orc.swiglu(swapped), orc.swiglu(gu))


def test_swiglu_matches_torch_silu_in_fp64():
    """Random bf16 gate/up values: h = bf16(silu(g) * u) with torch's silu in
    fp64 (a library routine) and one rounding."""
    rng = np.random.default_rng(11)
    P, I = 37, 96
    g = _bf16_bits(rng.standard_normal((P, I)) * 4)
    u = _bf16_bits(rng.standard_normal((P, I)))
    gu = np.concatenate([g, u], axis=1)
    g64 = torch.from_numpy(bf16_bits_to_f64(g))
    u64 = torch.from_numpy(bf16_bits_to_f64(u))
    want = _bf16_bits((torch.nn.functional.silu(g64) * u64).numpy())
    assert np.array_equal(orc.swiglu(gu), want)


def test_fused_expert_brute_force():
    """Fused pass on tiny shapes against an independent torch fp64 evaluation
    with bf16 rounding at the two stated points (gate_up output, h); an
    identity down projection returns h itself."""
    rng = np.random.default_rng(12)
    E, H, I, T = 3, 32, 16, 10
    counts = np.array([4, 0, 7], np.int32)
    off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    P = int(off[-1])
    r2t = rng.integers(0, T, size=P).astype(np.int32)
    x = _bf16_bits(rng.standard_normal((T, H)))
    wgu = _bf16_bits(rng.standard_normal((E, 2 * I, H)) * 0.3)
    wd = _bf16_bits(rng.standard_normal((E, H, I)) * 0.3)
    got = orc.fused_expert(x, wgu, wd, off, r2t)
    x64 = bf16_bits_to_f64(x)
    want = np.zeros((P, H), np.uint16)
    for e in range(E):
        for p in range(off[e], off[e + 1]):
            gu = _bf16_bits(bf16_bits_to_f64(wgu[e]) @ x64[r2t[p]])
            g = torch.from_numpy(bf16_bits_to_f64(gu[:I]))
            u = torch.from_numpy(bf16_bits_to_f64(gu[I:]))
            h = _bf16_bits((torch.nn.functional.silu(g) * u).numpy())
            want[p] = _bf16_bits(bf16_bits_to_f64(wd[e]) @ bf16_bits_to_f64(h))
    assert np.array_equal(got, want)
    # identity down projection (H = I): the pass returns the SwiGLU output
    eye = _bf16_bits(np.array(np.broadcast_to(np.eye(I), (E, I, I))))
    wgu_i = wgu[:, :, :I]
    x_i = x[:, :I]
    h_only = orc.swiglu(orc.grouped_forward(x_i, wgu_i, off, r2t))
    assert np.array_equal(orc.fused_expert(x_i, wgu_i, eye, off, r2t), h_only)
