"""The Python binding checks every size the C ABI cannot see (it receives
bare pointers): scale and packed-weight element counts and caller-supplied
output shapes.  A mismatch raises ValueError before anything reaches the
library, so these run on CPU tensors."""
import pytest
import torch

gbw = pytest.importorskip("grouped_bit_weight_b200")

E, N, K, P = 2, 64, 128, 6


def _fwd_args(fmt, **over):
    a = dict(x=torch.zeros((P, K), dtype=torch.bfloat16),
             w=torch.zeros((E, N, K // 2), dtype=torch.uint8),
             s=(torch.zeros((E, N, K // 64), dtype=torch.float32) if fmt == "nf4"
                else torch.zeros((E, N, K // 32), dtype=torch.uint8)),
             off=torch.zeros(E + 1, dtype=torch.int32))
    a.update(over)
    return a


@pytest.mark.parametrize("fmt", ["nf4", "mxfp4"])
def test_forward_rejects_short_scales_and_weights(fmt):
    fn = gbw.gnf4_grouped_gemm if fmt == "nf4" else gbw.gmxfp4_grouped_gemm
    sdt = torch.float32 if fmt == "nf4" else torch.uint8
    sdiv = 64 if fmt == "nf4" else 32
    a = _fwd_args(fmt, s=torch.zeros((E, N, K // sdiv - 1), dtype=sdt))
    with pytest.raises(ValueError, match="scales"):
        fn(a["x"], a["w"], a["s"], a["off"])
    a = _fwd_args(fmt, w=torch.zeros((E, N, K // 2 - 16), dtype=torch.uint8))
    with pytest.raises(ValueError, match="packed weights"):
        fn(a["x"], a["w"], a["s"], a["off"])
    a = _fwd_args(fmt, off=torch.zeros(E, dtype=torch.int32))
    with pytest.raises(ValueError, match="expert_offsets"):
        fn(a["x"], a["w"], a["s"], a["off"])
    a = _fwd_args(fmt)
    with pytest.raises(ValueError, match="out must be"):
        fn(a["x"], a["w"], a["s"], a["off"], out=torch.zeros((P, N - 8), dtype=torch.bfloat16))
    # sizes right, but not on a GPU: still refused before the library
    with pytest.raises(ValueError, match="CUDA tensor"):
        fn(a["x"], a["w"], a["s"], a["off"])


@pytest.mark.parametrize("fmt", ["nf4", "mxfp4"])
def test_dgrad_rejects_bad_sizes_and_out(fmt):
    fn = gbw.gnf4_grouped_dgrad if fmt == "nf4" else gbw.gmxfp4_grouped_dgrad
    sdt = torch.float32 if fmt == "nf4" else torch.uint8
    sdiv = 64 if fmt == "nf4" else 32
    dy = torch.zeros((P, N), dtype=torch.bfloat16)
    w = torch.zeros((E, N, K // 2), dtype=torch.uint8)
    s = torch.zeros((E, N, K // sdiv), dtype=sdt)
    off = torch.zeros(E + 1, dtype=torch.int32)
    with pytest.raises(ValueError, match="scales"):
        fn(dy, w, torch.zeros((E, N, K // sdiv - 1), dtype=sdt), off)
    with pytest.raises(ValueError, match="dx must be"):
        fn(dy, w, s, off, out=torch.zeros((P, K - 8), dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="packed rows"):
        fn(dy, torch.zeros((E, N + 8, K // 2), dtype=torch.uint8), s, off)
    with pytest.raises(ValueError, match="CUDA tensor"):
        fn(dy, w, s, off)


def test_dequant_rejects_bad_sizes_and_out():
    w = torch.zeros((E, N, K // 2), dtype=torch.uint8)
    with pytest.raises(ValueError, match="scales"):
        gbw.gnf4_dequant(w, torch.zeros((E, N, K // 64 - 1), dtype=torch.float32))
    with pytest.raises(ValueError, match="out"):
        gbw.gnf4_dequant(w, torch.zeros((E, N, K // 64), dtype=torch.float32),
                         out=torch.zeros((E, N, K - 1), dtype=torch.bfloat16))
    b = torch.zeros((E, N, K // 32, 16), dtype=torch.uint8)
    with pytest.raises(ValueError, match="scales"):
        gbw.gmxfp4_dequant(b, torch.zeros((E, N, K // 32 + 1), dtype=torch.uint8))
    with pytest.raises(ValueError, match="out"):
        gbw.gmxfp4_dequant(b, torch.zeros((E, N, K // 32), dtype=torch.uint8),
                           out=torch.zeros((E * N * K + 8,), dtype=torch.bfloat16))
