"""grouped_bit_weight_b200 -- grouped 4-bit (NF4 / MXFP4) MoE matmuls on B200.

A thin Python front end over the C ABI of libgbw.so (include/gbw.h).  The
functions below only check arguments and pass torch tensors' device pointers
and the current CUDA stream to the library; every step of the computation
runs in the library's sm_100a kernels.  There is no CPU fallback: importing
this package fails if libgbw.so is missing, and every call raises on a
non-sm_100 device.
"""
from __future__ import annotations

import ctypes as C
import os

import torch

__all__ = [
    "lib", "GbwError", "gnf4_grouped_gemm", "gmxfp4_grouped_gemm",
    "gnf4_grouped_dgrad", "gmxfp4_grouped_dgrad", "gnf4_dequant", "gmxfp4_dequant", "gnf4_quantize",
    "gmxfp4_quantize", "device_status", "MODE_AUTO", "MODE_GEMM", "MODE_GEMV",
    "DEVERR_OFFSETS", "DEVERR_TOKEN", "DEVERR_TIMEOUT", "FLAG_OVERLAP_PREV",
    "EXPORTS",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgbw.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -m "
        "grouped_bit_weight_b200.build` (nvcc, sm_100a). There is no fallback.")

lib = C.CDLL(LIB_PATH)

MODE_AUTO, MODE_GEMM, MODE_GEMV = 0, 1, 2
FLAG_OVERLAP_PREV = 0x100
DEVERR_OFFSETS, DEVERR_TOKEN, DEVERR_TIMEOUT = 1, 2, 4
_STATUS = {0: "GBW_OK", 1: "GBW_ERR_NULL", 2: "GBW_ERR_SHAPE",
           3: "GBW_ERR_ALIGN", 4: "GBW_ERR_ARCH", 5: "GBW_ERR_LAUNCH",
           6: "GBW_ERR_DEVICE"}

_P, _I64, _I32 = C.c_void_p, C.c_int64, C.c_int32

# name -> (restype, argtypes); mirrors include/gbw.h
EXPORTS = {
    "gnf4_grouped_gemm": (C.c_int, [_P, _I64, _I64, _P, _P, _I32, _I64, _P, _P, _I64, _P, _I32, _P]),
    "gmxfp4_grouped_gemm": (C.c_int, [_P, _I64, _I64, _P, _P, _I32, _I64, _P, _P, _I64, _P, _I32, _P]),
    "gnf4_grouped_dgrad": (C.c_int, [_P, _I64, _I64, _P, _P, _I32, _I64, _P, _P, _P]),
    "gmxfp4_grouped_dgrad": (C.c_int, [_P, _I64, _I64, _P, _P, _I32, _I64, _P, _P, _P]),
    "gnf4_dequant": (C.c_int, [_P, _P, _I64, _I64, _P, _P]),
    "gmxfp4_dequant": (C.c_int, [_P, _P, _I64, _I64, _P, _P]),
    "gnf4_quantize": (C.c_int, [_P, _I64, _I64, _P, _P, _P]),
    "gmxfp4_quantize": (C.c_int, [_P, _I64, _I64, _P, _P, _P]),
    "gbw_device_status": (C.c_int, [_P, C.POINTER(C.c_int32), _I32]),
    "gbw_status_string": (C.c_char_p, [C.c_int]),
    "gbw_version": (C.c_int32, []),
}
for _name, (_res, _args) in EXPORTS.items():
    _f = getattr(lib, _name)
    _f.restype = _res
    _f.argtypes = _args


class GbwError(RuntimeError):
    def __init__(self, status: int, where: str):
        msg = lib.gbw_status_string(status).decode()
        super().__init__(f"{where}: {_STATUS.get(status, status)}: {msg}")
        self.status = status


def _check(status: int, where: str) -> None:
    if status != 0:
        raise GbwError(status, where)


def _ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _stream(dev) -> C.c_void_p:
    return C.c_void_p(torch.cuda.current_stream(dev).cuda_stream)


def _need(t, name, dtype, device=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


_MODES = {"auto": MODE_AUTO, "gemm": MODE_GEMM, "gemv": MODE_GEMV}


def _grouped(fn, where, x, w, scale, scale_dtype, expert_offsets, row_to_token,
             out, mode, K_div, overlap_prev=False):
    _need(x, "x", torch.bfloat16)
    dev = x.device
    _need(w, "packed weights", torch.uint8, dev)
    _need(scale, "scales", scale_dtype, dev)
    _need(expert_offsets, "expert_offsets", torch.int32, dev)
    T, K = x.shape
    E, N = w.shape[0], w.shape[1]
    if w.numel() != E * N * (K // 2) or K % K_div:
        raise ValueError(f"{where}: weights do not match x's K={K}")
    if expert_offsets.numel() != E + 1:
        raise ValueError(f"{where}: expert_offsets needs E+1={E + 1} entries")
    if row_to_token is not None:
        _need(row_to_token, "row_to_token", torch.int32, dev)
        P = row_to_token.numel()
    else:
        P = T
    if out is None:
        out = torch.empty((P, N), dtype=torch.bfloat16, device=dev)
    _need(out, "out", torch.bfloat16, dev)
    if tuple(out.shape) != (P, N):
        raise ValueError(f"{where}: out must be [{P}, {N}]")
    m = _MODES[mode] if isinstance(mode, str) else int(mode)
    if overlap_prev:
        m |= FLAG_OVERLAP_PREV
    with torch.cuda.device(dev):
        _check(fn(_ptr(x), T, K, _ptr(w), _ptr(scale), E, N, _ptr(expert_offsets),
                  _ptr(row_to_token), P, _ptr(out), m, _stream(dev)), where)
    return out


def gnf4_grouped_gemm(x, packed, absmax, expert_offsets, row_to_token=None,
                      out=None, mode="auto", overlap_prev=False):
    """out[P, N] = x[row_to_token] @ W_e^T per expert; NF4 weights
    packed [E, N, K/2] uint8 (high nibble = even k), absmax [E, N, K/64] fp32.
    P = len(row_to_token), or x's rows when row_to_token is None.
    overlap_prev=True promises that packed, absmax, expert_offsets and
    row_to_token are not written by the kernel launched just before this
    call on the stream (GBW_FLAG_OVERLAP_PREV)."""
    return _grouped(lib.gnf4_grouped_gemm, "gnf4_grouped_gemm", x, packed,
                    absmax, torch.float32, expert_offsets, row_to_token, out,
                    mode, 64, overlap_prev)


def gmxfp4_grouped_gemm(x, blocks, scales, expert_offsets, row_to_token=None,
                        out=None, mode="auto", overlap_prev=False):
    """MXFP4 variant: blocks [E, N, K/32, 16] uint8 (low nibble = even k),
    scales [E, N, K/32] uint8 (e8m0)."""
    return _grouped(lib.gmxfp4_grouped_gemm, "gmxfp4_grouped_gemm", x, blocks,
                    scales, torch.uint8, expert_offsets, row_to_token, out,
                    mode, 32, overlap_prev)


def gnf4_grouped_dgrad(dy, packed, absmax, expert_offsets, out=None):
    """dx[P, K] = dy[P, N] @ W_e per expert (the activation gradient of
    gnf4_grouped_gemm, rows in the same expert-sorted order)."""
    _need(dy, "dy", torch.bfloat16)
    dev = dy.device
    _need(packed, "packed", torch.uint8, dev)
    _need(absmax, "absmax", torch.float32, dev)
    _need(expert_offsets, "expert_offsets", torch.int32, dev)
    P, N = dy.shape
    E = packed.shape[0]
    K = packed.shape[-1] * 2
    if packed.shape[1] != N:
        raise ValueError("gnf4_grouped_dgrad: packed rows must equal dy's N")
    if out is None:
        out = torch.empty((P, K), dtype=torch.bfloat16, device=dev)
    _need(out, "dx", torch.bfloat16, dev)
    with torch.cuda.device(dev):
        _check(lib.gnf4_grouped_dgrad(_ptr(dy), P, N, _ptr(packed), _ptr(absmax),
                                      E, K, _ptr(expert_offsets), _ptr(out),
                                      _stream(dev)), "gnf4_grouped_dgrad")
    return out


def gmxfp4_grouped_dgrad(dy, blocks, scales, expert_offsets, out=None):
    """dx[P, K] = dy[P, N] @ W_e per expert for MXFP4 weights (blocks
    [E, N, K/32, 16] uint8, scales [E, N, K/32] uint8 e8m0)."""
    _need(dy, "dy", torch.bfloat16)
    dev = dy.device
    _need(blocks, "blocks", torch.uint8, dev)
    _need(scales, "scales", torch.uint8, dev)
    _need(expert_offsets, "expert_offsets", torch.int32, dev)
    P, N = dy.shape
    E = blocks.shape[0]
    K = blocks.shape[2] * 32 if blocks.dim() == 4 else blocks.shape[-1] * 2
    if blocks.shape[1] != N:
        raise ValueError("gmxfp4_grouped_dgrad: blocks rows must equal dy's N")
    if out is None:
        out = torch.empty((P, K), dtype=torch.bfloat16, device=dev)
    _need(out, "dx", torch.bfloat16, dev)
    with torch.cuda.device(dev):
        _check(lib.gmxfp4_grouped_dgrad(_ptr(dy), P, N, _ptr(blocks), _ptr(scales),
                                        E, K, _ptr(expert_offsets), _ptr(out),
                                        _stream(dev)), "gmxfp4_grouped_dgrad")
    return out


def gnf4_dequant(packed, absmax, out=None):
    """bf16 weights [..., K] decoded from NF4 (bit-exact)."""
    _need(packed, "packed", torch.uint8)
    dev = packed.device
    _need(absmax, "absmax", torch.float32, dev)
    K = packed.shape[-1] * 2
    rows = packed.numel() // max(K // 2, 1)
    if out is None:
        out = torch.empty(packed.shape[:-1] + (K,), dtype=torch.bfloat16, device=dev)
    _need(out, "out", torch.bfloat16, dev)
    with torch.cuda.device(dev):
        _check(lib.gnf4_dequant(_ptr(packed), _ptr(absmax), rows, K, _ptr(out),
                                _stream(dev)), "gnf4_dequant")
    return out


def gmxfp4_dequant(blocks, scales, out=None):
    """bf16 weights [..., K] decoded from MXFP4 blocks [..., K/32, 16]."""
    _need(blocks, "blocks", torch.uint8)
    dev = blocks.device
    _need(scales, "scales", torch.uint8, dev)
    K = blocks.shape[-2] * 32
    rows = blocks.numel() // max(K // 2, 1)
    if out is None:
        out = torch.empty(blocks.shape[:-2] + (K,), dtype=torch.bfloat16, device=dev)
    _need(out, "out", torch.bfloat16, dev)
    with torch.cuda.device(dev):
        _check(lib.gmxfp4_dequant(_ptr(blocks), _ptr(scales), rows, K, _ptr(out),
                                  _stream(dev)), "gmxfp4_dequant")
    return out


def gnf4_quantize(w):
    """fp32 [..., K] -> (packed [..., K/2] uint8, absmax [..., K/64] fp32)."""
    _need(w, "w", torch.float32)
    K = w.shape[-1]
    rows = w.numel() // max(K, 1)
    packed = torch.empty(w.shape[:-1] + (K // 2,), dtype=torch.uint8, device=w.device)
    absmax = torch.empty(w.shape[:-1] + (K // 64,), dtype=torch.float32, device=w.device)
    with torch.cuda.device(w.device):
        _check(lib.gnf4_quantize(_ptr(w), rows, K, _ptr(packed), _ptr(absmax),
                                 _stream(w.device)), "gnf4_quantize")
    return packed, absmax


def gmxfp4_quantize(w):
    """fp32 [..., K] -> (blocks [..., K/32, 16] uint8, scales [..., K/32] uint8)."""
    _need(w, "w", torch.float32)
    K = w.shape[-1]
    rows = w.numel() // max(K, 1)
    blocks = torch.empty(w.shape[:-1] + (K // 32, 16), dtype=torch.uint8, device=w.device)
    scales = torch.empty(w.shape[:-1] + (K // 32,), dtype=torch.uint8, device=w.device)
    with torch.cuda.device(w.device):
        _check(lib.gmxfp4_quantize(_ptr(w), rows, K, _ptr(blocks), _ptr(scales),
                                   _stream(w.device)), "gmxfp4_quantize")
    return blocks, scales


def device_status(device=None, clear=True) -> int:
    """The GBW_DEVERR_* bits the library's kernels raised on `device`
    (synchronises the current stream); clears them when `clear`."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    v = C.c_int32(0)
    with torch.cuda.device(dev):
        st = lib.gbw_device_status(_stream(dev), C.byref(v), 1 if clear else 0)
    if st not in (0, 6):
        _check(st, "gbw_device_status")
    return int(v.value)
