"""The C-ABI library loads without a GPU, exports every entry point that
include/gbw.h declares, and rejects bad host arguments before touching CUDA."""
import ctypes as C
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    text = open(os.path.join(ROOT, "include", "gbw.h")).read()
    return re.findall(r"GBW_API\s+[\w\s\*]+?\b(\w+)\s*\(", text)


def test_header_declares_the_entry_points():
    names = set(_declared())
    for n in ["gnf4_grouped_gemm", "gmxfp4_grouped_gemm", "gnf4_grouped_dgrad",
              "gmxfp4_grouped_dgrad", "gnf4_grouped_expert_mlp",
              "gmxfp4_grouped_expert_mlp", "gnf4_dequant", "gmxfp4_dequant", "gnf4_quantize",
              "gmxfp4_quantize", "gbw_device_status", "gbw_status_string",
              "gbw_version"]:
        assert n in names, n


def test_library_exports_every_declared_symbol():
    import grouped_bit_weight_b200 as gbw
    for name in _declared():
        assert hasattr(gbw.lib, name), name
        assert name in gbw.EXPORTS, name
    assert gbw.lib.gbw_version() >= 100


def _call(fn, **kw):
    import grouped_bit_weight_b200 as gbw
    a = dict(x=16, T=4, K=128, w=16, s=16, E=2, N=64, off=16, r2t=None, P=4,
             out=16, mode=0)
    a.update(kw)
    f = getattr(gbw.lib, fn)
    return f(C.c_void_p(a["x"]), a["T"], a["K"], C.c_void_p(a["w"]),
             C.c_void_p(a["s"]), a["E"], a["N"], C.c_void_p(a["off"]),
             None if a["r2t"] is None else C.c_void_p(a["r2t"]), a["P"],
             C.c_void_p(a["out"]), a["mode"], None)


@pytest.mark.parametrize("fn", ["gnf4_grouped_gemm", "gmxfp4_grouped_gemm"])
def test_host_validation_needs_no_gpu(fn):
    SHAPE, NULL, ALIGN = 2, 1, 3
    assert _call(fn, K=100) == SHAPE          # K not a multiple of 32/64
    assert _call(fn, N=60) == SHAPE           # N % 8
    assert _call(fn, E=0) == SHAPE
    assert _call(fn, P=-1) == SHAPE
    assert _call(fn, mode=7) == SHAPE
    assert _call(fn, mode=0x200) == SHAPE     # unknown flag bit
    assert _call(fn, E=1025) == SHAPE         # more experts than the kernels hold
    assert _call(fn, T=2, P=4) == SHAPE       # identity rows need T >= P
    assert _call(fn, off=0) == NULL
    assert _call(fn, w=0) == NULL
    assert _call(fn, x=0) == NULL
    assert _call(fn, x=24) == ALIGN           # not 16-byte aligned
    assert _call(fn, out=8) == ALIGN
    if fn == "gnf4_grouped_gemm":
        assert _call(fn, s=18) == ALIGN       # absmax needs 4-byte alignment
    else:
        assert _call(fn, s=17) == ALIGN       # e8m0 scales need 2-byte alignment
    if fn == "gnf4_grouped_gemm":
        assert _call(fn, K=96) == SHAPE
    else:
        assert _call(fn, K=80, mode=1) == SHAPE  # MXFP4 needs K % 32


def test_dgrad_and_codec_validation():
    import grouped_bit_weight_b200 as gbw
    L = gbw.lib
    p = C.c_void_p(16)
    assert L.gnf4_grouped_dgrad(p, 4, 60, p, p, 1, 128, p, p, None) == 2
    assert L.gnf4_grouped_dgrad(p, 4, 64, p, p, 1, 96, p, p, None) == 2
    assert L.gnf4_grouped_dgrad(None, 4, 64, p, p, 1, 128, p, p, None) == 1
    assert L.gmxfp4_grouped_dgrad(p, 4, 60, p, p, 1, 128, p, p, None) == 2
    assert L.gmxfp4_grouped_dgrad(p, 4, 64, p, p, 1, 96, p, p, None) == 2
    assert L.gmxfp4_grouped_dgrad(None, 4, 64, p, p, 1, 128, p, p, None) == 1
    assert L.gmxfp4_grouped_dgrad(p, 4, 64, p, C.c_void_p(17), 1, 128, p, p, None) == 3
    assert L.gnf4_dequant(p, p, 4, 96, p, None) == 2
    assert L.gmxfp4_dequant(p, p, 4, 48, p, None) == 2
    assert L.gnf4_quantize(None, 4, 64, p, p, None) == 1
    assert L.gmxfp4_quantize(C.c_void_p(8), 4, 64, p, p, None) == 3
    assert L.gnf4_dequant(p, p, 4, 96, p, None) == 2
    assert b"K % 64" in L.gbw_status_string(2)  # text of the last error


@pytest.mark.parametrize("fn", ["gnf4_grouped_expert_mlp", "gmxfp4_grouped_expert_mlp"])
def test_fused_pass_host_validation(fn):
    import grouped_bit_weight_b200 as gbw
    f = getattr(gbw.lib, fn)
    SHAPE, NULL, ALIGN = 2, 1, 3

    def call(**kw):
        a = dict(x=16, T=8, H=256, gu=16, gs=16, dn=16, ds=16, E=2, I=128, off=16,
                 r2t=None, P=8, h=16, out=16, mode=0)
        a.update(kw)
        v = lambda k: None if a[k] is None else C.c_void_p(a[k])
        return f(v("x"), a["T"], a["H"], v("gu"), v("gs"), v("dn"), v("ds"), a["E"], a["I"],
                 v("off"), v("r2t"), a["P"], v("h"), v("out"), a["mode"], None)
    assert call(H=320 + 32) == SHAPE      # H % 64
    assert call(I=96) == SHAPE            # I % 64
    assert call(E=0) == SHAPE
    assert call(mode=0x100) == SHAPE      # no flags on the fused pass
    assert call(T=4, P=8) == SHAPE        # identity rows need T >= P
    assert call(h=0) == NULL
    assert call(dn=0) == NULL
    assert call(h=24) == ALIGN
    assert call(gs=17) == ALIGN
