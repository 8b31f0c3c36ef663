"""ctypes front end of the CPU oracle (oracle.c).

TEST INFRASTRUCTURE ONLY: imported by tests/, by __graft_entry__.smoke() and
by bench.py's cpu_baseline / reference leg.  The product package never
imports it.  Arrays are numpy; bf16 values travel as uint16 bit patterns.
"""
from __future__ import annotations

import ctypes as C
import os
import sys

import numpy as np

sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
import build as _build  # noqa: E402

_lib = C.CDLL(_build.build())

_P = C.c_void_p
_I64 = C.c_int64
_I32 = C.c_int32


def _sig(name, res, *args):
    f = getattr(_lib, name)
    f.restype = res
    f.argtypes = list(args)
    return f


_sig("orc_f32_to_bf16", C.c_uint16, C.c_float)
_sig("orc_f64_to_bf16", C.c_uint16, C.c_double)
_sig("orc_nf4_codebook", None, _P)
_sig("orc_nf4_pack", C.c_int, _P, _I64, _I64, _P, _P)
_sig("orc_nf4_decode_f32", None, _P, _P, _I64, _I64, _P)
_sig("orc_nf4_decode_bf16", None, _P, _P, _I64, _I64, _P)
_sig("orc_mxfp4_pack", C.c_int, _P, _I64, _I64, _P, _P)
_sig("orc_mxfp4_decode_f32", None, _P, _P, _I64, _I64, _P)
_sig("orc_mxfp4_decode_bf16", None, _P, _P, _I64, _I64, _P)
_sig("orc_grouped_forward", C.c_int, _P, _I64, _I64, _P, _I32, _I64, _P, _P,
     _I64, _P, _P)
_sig("orc_grouped_forward_sampled", C.c_int, _P, _I64, _I64, _P, _I32, _I64,
     _P, _P, _I64, _P, _P, _I64, _P)
_sig("orc_grouped_dgrad", C.c_int, _P, _I64, _I64, _P, _I32, _I64, _P, _P, _P)
_sig("orc_grouped_dgrad_sampled", C.c_int, _P, _I64, _I64, _P, _I32, _I64, _P,
     _P, _P, _I64, _P)
_sig("orc_swiglu", C.c_int, _P, _I64, _I64, _P)
_sig("orc_num_threads", C.c_int)
_sig("orc_set_num_threads", None, C.c_int)


class OracleError(RuntimeError):
    pass


def _ptr(a):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _check(rc, what):
    if rc != 0:
        raise OracleError(f"{what} failed with code {rc}")


def num_threads() -> int:
    return _lib.orc_num_threads()


def set_num_threads(n: int) -> None:
    _lib.orc_set_num_threads(int(n))


# ---- bf16 -------------------------------------------------------------

def f32_to_bf16(a) -> np.ndarray:
    a = _c(a, np.float32)
    return np.array([_lib.orc_f32_to_bf16(float(v)) for v in a.ravel()],
                    dtype=np.uint16).reshape(a.shape)


def f64_to_bf16(a) -> np.ndarray:
    a = _c(a, np.float64)
    return np.array([_lib.orc_f64_to_bf16(float(v)) for v in a.ravel()],
                    dtype=np.uint16).reshape(a.shape)


def bf16_to_f32(h) -> np.ndarray:
    h = _c(h, np.uint16)
    return (h.astype(np.uint32) << 16).view(np.float32)


# ---- NF4 --------------------------------------------------------------

def nf4_codebook() -> np.ndarray:
    out = np.zeros(16, np.float32)
    _lib.orc_nf4_codebook(_ptr(out))
    return out


def nf4_pack(w):
    """w[..., N, K] fp32 -> (packed [..., N, K/2] u8, absmax [..., N, K/64] f32)."""
    w = _c(w, np.float32)
    K = w.shape[-1]
    rows = w.size // K if K else 0
    packed = np.zeros(w.shape[:-1] + (K // 2,), np.uint8)
    absmax = np.zeros(w.shape[:-1] + (K // 64,), np.float32)
    _check(_lib.orc_nf4_pack(_ptr(w), rows, K, _ptr(packed), _ptr(absmax)),
           "nf4_pack")
    return packed, absmax


def nf4_decode(packed, absmax, K, bf16=False):
    packed = _c(packed, np.uint8)
    absmax = _c(absmax, np.float32)
    rows = packed.size // (K // 2) if K else 0
    shape = packed.shape[:-1] + (K,)
    if bf16:
        out = np.zeros(shape, np.uint16)
        _lib.orc_nf4_decode_bf16(_ptr(packed), _ptr(absmax), rows, K, _ptr(out))
    else:
        out = np.zeros(shape, np.float32)
        _lib.orc_nf4_decode_f32(_ptr(packed), _ptr(absmax), rows, K, _ptr(out))
    return out


# ---- MXFP4 ------------------------------------------------------------

def mxfp4_pack(w):
    """w[..., K] fp32 -> (blocks [..., K/32, 16] u8, scales [..., K/32] u8)."""
    w = _c(w, np.float32)
    K = w.shape[-1]
    rows = w.size // K if K else 0
    blocks = np.zeros(w.shape[:-1] + (K // 32, 16), np.uint8)
    scales = np.zeros(w.shape[:-1] + (K // 32,), np.uint8)
    _check(_lib.orc_mxfp4_pack(_ptr(w), rows, K, _ptr(blocks), _ptr(scales)),
           "mxfp4_pack")
    return blocks, scales


def mxfp4_decode(blocks, scales, bf16=False):
    blocks = _c(blocks, np.uint8)
    scales = _c(scales, np.uint8)
    K = blocks.shape[-2] * 32
    rows = scales.size // (K // 32) if K else 0
    shape = blocks.shape[:-2] + (K,)
    if bf16:
        out = np.zeros(shape, np.uint16)
        _lib.orc_mxfp4_decode_bf16(_ptr(blocks), _ptr(scales), rows, K, _ptr(out))
    else:
        out = np.zeros(shape, np.float32)
        _lib.orc_mxfp4_decode_f32(_ptr(blocks), _ptr(scales), rows, K, _ptr(out))
    return out


# ---- grouped matmuls -----------------------------------------------------

def grouped_forward(x_bf16, wdec_bf16, offsets, row_to_token=None,
                    want_f64=False):
    """x [T,K] bf16 bits, wdec [E,N,K] bf16 bits, offsets [E+1] -> out [P,N]."""
    x = _c(x_bf16, np.uint16)
    w = _c(wdec_bf16, np.uint16)
    off = _c(offsets, np.int32)
    T, K = x.shape
    E, N, K2 = w.shape
    assert K == K2 and off.shape == (E + 1,)
    P = int(off[-1])
    r2t = None if row_to_token is None else _c(row_to_token, np.int32)
    out = np.zeros((P, N), np.uint16)
    o64 = np.zeros((P, N), np.float64) if want_f64 else None
    _check(_lib.orc_grouped_forward(_ptr(x), T, K, _ptr(w), E, N, _ptr(off),
                                    _ptr(r2t), P, _ptr(out), _ptr(o64)),
           "grouped_forward")
    return (out, o64) if want_f64 else out


def grouped_forward_sampled(x_bf16, wdec_bf16, offsets, row_to_token, sp, sn):
    x = _c(x_bf16, np.uint16)
    w = _c(wdec_bf16, np.uint16)
    off = _c(offsets, np.int32)
    T, K = x.shape
    E, N, _ = w.shape
    P = int(off[-1])
    r2t = None if row_to_token is None else _c(row_to_token, np.int32)
    sp = _c(sp, np.int64)
    sn = _c(sn, np.int64)
    out = np.zeros(sp.shape, np.float64)
    _check(_lib.orc_grouped_forward_sampled(_ptr(x), T, K, _ptr(w), E, N,
                                            _ptr(off), _ptr(r2t), P, _ptr(sp),
                                            _ptr(sn), sp.size, _ptr(out)),
           "grouped_forward_sampled")
    return out


def grouped_dgrad(dy_bf16, wdec_bf16, offsets, want_f64=False):
    """dy [P,N] bf16 bits, wdec [E,N,K] bf16 bits -> dx [P,K]."""
    dy = _c(dy_bf16, np.uint16)
    w = _c(wdec_bf16, np.uint16)
    off = _c(offsets, np.int32)
    P, N = dy.shape
    E, N2, K = w.shape
    assert N == N2
    dx = np.zeros((P, K), np.uint16)
    d64 = np.zeros((P, K), np.float64) if want_f64 else None
    _check(_lib.orc_grouped_dgrad(_ptr(dy), P, N, _ptr(w), E, K, _ptr(off),
                                  _ptr(dx), _ptr(d64)), "grouped_dgrad")
    return (dx, d64) if want_f64 else dx


def grouped_dgrad_sampled(dy_bf16, wdec_bf16, offsets, sp, sk):
    dy = _c(dy_bf16, np.uint16)
    w = _c(wdec_bf16, np.uint16)
    off = _c(offsets, np.int32)
    P, N = dy.shape
    E, _, K = w.shape
    sp = _c(sp, np.int64)
    sk = _c(sk, np.int64)
    out = np.zeros(sp.shape, np.float64)
    _check(_lib.orc_grouped_dgrad_sampled(_ptr(dy), P, N, _ptr(w), E, K,
                                          _ptr(off), _ptr(sp), _ptr(sk),
                                          sp.size, _ptr(out)),
           "grouped_dgrad_sampled")
    return out


def swiglu(gu_bf16):
    """SwiGLU combine of a fused gate_up output: gu [P, 2I] bf16 bits ->
    h [P, I] bf16 bits, h = silu(gate) * up with gate = columns [0, I) and
    up = columns [I, 2I) (the reading oracle.c states)."""
    gu = _c(gu_bf16, np.uint16)
    P, I2 = gu.shape
    if I2 % 2:
        raise OracleError("swiglu: gate_up width must be even")
    h = np.empty((P, I2 // 2), np.uint16)
    _check(_lib.orc_swiglu(_ptr(gu), P, I2 // 2, _ptr(h)), "swiglu")
    return h


def fused_expert(x_bf16, w_gate_up_bf16, w_down_bf16, offsets, row_to_token=None):
    """One fused expert pass per routed row: the grouped gate_up matmul (bf16
    out), the SwiGLU combine (bf16 h), then the grouped down matmul over the
    same expert-sorted rows.  w_gate_up [E, 2I, H], w_down [E, H, I]."""
    gu = grouped_forward(x_bf16, w_gate_up_bf16, offsets, row_to_token)
    h = swiglu(gu)
    return grouped_forward(h, w_down_bf16, offsets, None)

