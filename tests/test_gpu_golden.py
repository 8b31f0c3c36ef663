"""The hand-derived grouped-matmul cases of tests/golden/hand_worked.json on
the GPU, through both paths: every output is exact in bf16, so the tensor
core GEMM and the bandwidth GEMV must reproduce it bit for bit."""
import numpy as np
import pytest

from golden_cases import hand_case
from parity import bf16_bits_to_f64

pytestmark = pytest.mark.gpu

gbw = pytest.importorskip("grouped_bit_weight_b200")
from gpu_util import bits, to_dev  # noqa: E402
from grouped_bit_weight_b200 import synth  # noqa: E402


@pytest.mark.parametrize("fmt", ["nf4", "mxfp4"])
@pytest.mark.parametrize("mode", ["gemm", "gemv"])
def test_hand_worked_cases_exact(fmt, mode):
    import torch
    c = hand_case(fmt)
    if mode == "gemm" and c["K"] % 64:
        pytest.skip("the tensor-core path needs K % 64 == 0")
    fn = gbw.gnf4_grouped_gemm if fmt == "nf4" else gbw.gmxfp4_grouped_gemm
    x = to_dev(synth.to_bf16_bits(c["x"]))
    out = fn(x, to_dev(c["codes"]), to_dev(c["scale"]), to_dev(c["offsets"]),
             to_dev(c["row_to_token"]), mode=mode)
    torch.cuda.synchronize()
    assert gbw.device_status() == 0
    assert np.array_equal(bf16_bits_to_f64(bits(out)), c["out"])
