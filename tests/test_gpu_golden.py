"""The hand-derived grouped-matmul cases of tests/golden/hand_worked.json on
the GPU, through both paths: every output is exact in bf16, so the tensor
core GEMM and the bandwidth GEMV must reproduce it bit for bit.  The MXFP4
case has K = 32: on the GEMM that is one half-full 64-wide stage."""
import numpy as np
import pytest

from golden_cases import hand_case
from parity import bf16_bits_to_f64

pytestmark = pytest.mark.gpu

gbw = pytest.importorskip("grouped_bit_weight_b200")
from gpu_util import bits, to_dev  # noqa: E402
import synth  # noqa: E402


@pytest.mark.parametrize("fmt", ["nf4", "mxfp4"])
@pytest.mark.parametrize("mode", ["gemm", "gemv"])
def test_hand_worked_cases_exact(fmt, mode):
    import torch
    c = hand_case(fmt)
    fn = gbw.gnf4_grouped_gemm if fmt == "nf4" else gbw.gmxfp4_grouped_gemm
    # the library takes N % 8 == 0: pad each expert with rows whose codes all
    # decode to zero (NF4 code 7, MXFP4 code 0), which must come out as 0
    codes, scale = c["codes"], c["scale"]
    E, N = codes.shape[:2]
    pad = 8 - N
    zero = 0x77 if fmt == "nf4" else 0x00
    codes = np.concatenate([codes, np.full((E, pad) + codes.shape[2:], zero, np.uint8)], axis=1)
    scale = np.concatenate([scale, np.repeat(scale[:, :1], pad, axis=1)], axis=1)
    x = to_dev(synth.to_bf16_bits(c["x"]))
    out = fn(x, to_dev(codes), to_dev(scale), to_dev(c["offsets"]),
             to_dev(c["row_to_token"]), mode=mode)
    torch.cuda.synchronize()
    assert gbw.device_status() == 0
    got = bf16_bits_to_f64(bits(out))
    assert np.array_equal(got[:, :N], c["out"])
    assert np.all(got[:, N:] == 0)
