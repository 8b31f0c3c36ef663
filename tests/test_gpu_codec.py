"""GPU decode and packers against the CPU oracle: decode bit-exact, packers
byte-identical (through the C ABI via the thin binding)."""
import numpy as np
import pytest
import torch

import oracle as orc
import synth

pytestmark = pytest.mark.gpu

gbw = pytest.importorskip("grouped_bit_weight_b200")
from gpu_util import bits, packed_weights, to_dev  # noqa: E402


def _same_bits_nan_aware(a, b):
    a = np.asarray(a, np.uint16)
    b = np.asarray(b, np.uint16)
    nan_a = ((a & 0x7F80) == 0x7F80) & ((a & 0x7F) != 0)
    nan_b = ((b & 0x7F80) == 0x7F80) & ((b & 0x7F) != 0)
    return bool(np.array_equal(nan_a, nan_b) and np.array_equal(a[~nan_a], b[~nan_b]))


@pytest.mark.parametrize("shape,std", [((8, 256, 512), 1.0),
                                       ((128, 1536, 2048), 0.02),
                                       ((128, 2048, 768), 0.02)])
def test_nf4_dequant_bit_exact(shape, std):
    codes, scale, wdec = packed_weights("nf4", *shape, std, 11)
    got = gbw.gnf4_dequant(to_dev(codes), to_dev(scale))
    assert got.shape == shape
    assert np.array_equal(bits(got), wdec)


@pytest.mark.parametrize("shape", [(4, 5760, 2880), (4, 2880, 2880), (3, 64, 96)])
def test_mxfp4_dequant_bit_exact(shape):
    codes, scale, wdec = packed_weights("mxfp4", *shape, 0.02, 12)
    got = gbw.gmxfp4_dequant(to_dev(codes), to_dev(scale))
    assert _same_bits_nan_aware(bits(got), wdec)


def test_mxfp4_dequant_every_code_and_extreme_scales():
    # every byte value under every scale byte, including 0, 1, 253..255
    sc = np.arange(256, dtype=np.uint8).reshape(256, 1).repeat(16, axis=1)  # [256 rows, 16 blocks]
    blocks = np.tile(np.arange(256, dtype=np.uint8).reshape(16, 16), (256, 1, 1))
    got = gbw.gmxfp4_dequant(to_dev(blocks), to_dev(sc))
    want = orc.mxfp4_decode(blocks, sc, bf16=True)
    assert _same_bits_nan_aware(bits(got), want)


def test_nf4_dequant_every_byte_and_scale():
    rng = np.random.default_rng(5)
    a = np.concatenate([np.float32([0.0, 1.0, 2.0 ** -126, 2.0 ** -140, 3.0e38]),
                        rng.standard_normal(59).astype(np.float32) ** 3])
    packed = np.tile(np.arange(256, dtype=np.uint8), (len(a), 8))  # K = 4096
    absmax = np.repeat(a[:, None], 64, axis=1).astype(np.float32)
    got = gbw.gnf4_dequant(to_dev(packed), to_dev(absmax))
    want = orc.nf4_decode(packed, absmax, 4096, bf16=True)
    assert _same_bits_nan_aware(bits(got), want)


@pytest.mark.parametrize("std", [1.0, 0.02])
def test_nf4_quantize_matches_cpu_packer(std):
    w = synth.normal((64, 2048), 21, std)
    w[0, :64] = 0.0                             # all-zero block
    w[1, :64] = np.linspace(-1, 1, 64, dtype=np.float32)
    w[2, :] *= np.float32(1e-30)                # tiny values
    w[3, 5] = np.float32(3e38)
    p_ref, a_ref = orc.nf4_pack(w)
    p, a = gbw.gnf4_quantize(to_dev(w))
    assert np.array_equal(p.cpu().numpy(), p_ref)
    assert np.array_equal(a.cpu().numpy(), a_ref)


@pytest.mark.parametrize("std", [1.0, 0.02])
def test_mxfp4_quantize_matches_cpu_packer(std):
    w = synth.normal((64, 2880), 22, std)
    w[0, :32] = 0.0
    w[1, :32] = np.float32([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0] * 4)
    w[2, :] *= np.float32(1e-40)                # subnormal inputs
    w[3, 7] = np.float32(3e38)
    w[4, :32] = -0.0
    b_ref, s_ref = orc.mxfp4_pack(w)
    b, s = gbw.gmxfp4_quantize(to_dev(w))
    assert np.array_equal(b.cpu().numpy(), b_ref)
    assert np.array_equal(s.cpu().numpy(), s_ref)
