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
    "gnf4_grouped_dgrad", "gmxfp4_grouped_dgrad", "gnf4_grouped_expert_mlp",
    "gmxfp4_grouped_expert_mlp", "gnf4_grouped_expert_mlp_noalloc", "gnf4_dequant",
    "gmxfp4_dequant", "gnf4_quantize",
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
    "gnf4_grouped_expert_mlp": (C.c_int, [_P, _I64, _I64, _P, _P, _P, _P, _I32, _I64, _P, _P, _I64, _P, _P, _I32, _P]),
    "gmxfp4_grouped_expert_mlp": (C.c_int, [_P, _I64, _I64, _P, _P, _P, _P, _I32, _I64, _P, _P, _I64, _P, _P, _I32, _P]),
    "gnf4_grouped_expert_mlp_noalloc": (C.c_int, [_P, _I64, _I64, _P, _P, _P, _P, _I32, _I64, _P, _P, _I64, _P, _I32, _P]),
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


def _need(t, name, dtype):
    """Type, dtype and layout of one argument (the device is checked by
    _on_device once every size has been checked)."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _numel(t, name, n, where):
    if t.numel() != n:
        raise ValueError(f"{where}: {name} has {t.numel()} elements, needs {n}")


def _on_device(where, **tensors):
    """Every tensor is a CUDA tensor on one device; returns that device."""
    dev = None
    for name, t in tensors.items():
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError(f"{where}: {name} must be a CUDA tensor")
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError(f"{where}: {name} is on {t.device}, expected {dev}")
    return dev


_MODES = {"auto": MODE_AUTO, "gemm": MODE_GEMM, "gemv": MODE_GEMV}


def _grouped(fn, where, x, w, scale, scale_dtype, expert_offsets, row_to_token,
             out, mode, K_div, overlap_prev=False):
    _need(x, "x", torch.bfloat16)
    _need(w, "packed weights", torch.uint8)
    _need(scale, "scales", scale_dtype)
    _need(expert_offsets, "expert_offsets", torch.int32)
    if x.dim() != 2 or w.dim() < 3:
        raise ValueError(f"{where}: x must be [T, K] and the weights [E, N, ...]")
    T, K = x.shape
    E, N = w.shape[0], w.shape[1]
    if K % K_div:
        raise ValueError(f"{where}: K={K} must be a multiple of {K_div}")
    _numel(w, "packed weights", E * N * (K // 2), where)
    _numel(scale, "scales", E * N * (K // (64 if K_div == 64 else 32)), where)
    _numel(expert_offsets, "expert_offsets", E + 1, where)
    if row_to_token is not None:
        _need(row_to_token, "row_to_token", torch.int32)
        P = row_to_token.numel()
    else:
        P = T
    if out is not None:
        _need(out, "out", torch.bfloat16)
        if tuple(out.shape) != (P, N):
            raise ValueError(f"{where}: out must be [{P}, {N}]")
    dev = _on_device(where, x=x, w=w, scale=scale, expert_offsets=expert_offsets,
                     row_to_token=row_to_token, out=out)
    if out is None:
        out = torch.empty((P, N), dtype=torch.bfloat16, device=dev)
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


def _dgrad(fn, where, dy, w, scale, scale_dtype, K, sdiv, expert_offsets, out):
    _need(dy, "dy", torch.bfloat16)
    _need(w, "packed weights", torch.uint8)
    _need(scale, "scales", scale_dtype)
    _need(expert_offsets, "expert_offsets", torch.int32)
    if dy.dim() != 2 or w.dim() < 3:
        raise ValueError(f"{where}: dy must be [P, N] and the weights [E, N, ...]")
    P, N = dy.shape
    E = w.shape[0]
    if w.shape[1] != N:
        raise ValueError(f"{where}: packed rows must equal dy's N={N}")
    _numel(w, "packed weights", E * N * (K // 2), where)
    _numel(scale, "scales", E * N * (K // sdiv), where)
    _numel(expert_offsets, "expert_offsets", E + 1, where)
    if out is not None:
        _need(out, "dx", torch.bfloat16)
        if tuple(out.shape) != (P, K):
            raise ValueError(f"{where}: dx must be [{P}, {K}]")
    dev = _on_device(where, dy=dy, w=w, scale=scale, expert_offsets=expert_offsets, out=out)
    if out is None:
        out = torch.empty((P, K), dtype=torch.bfloat16, device=dev)
    with torch.cuda.device(dev):
        _check(fn(_ptr(dy), P, N, _ptr(w), _ptr(scale), E, K, _ptr(expert_offsets),
                  _ptr(out), _stream(dev)), where)
    return out


def gnf4_grouped_dgrad(dy, packed, absmax, expert_offsets, out=None):
    """dx[P, K] = dy[P, N] @ W_e per expert (the activation gradient of
    gnf4_grouped_gemm, rows in the same expert-sorted order); packed
    [E, N, K/2] uint8, absmax [E, N, K/64] fp32."""
    K = packed.shape[-1] * 2 if isinstance(packed, torch.Tensor) else 0
    return _dgrad(lib.gnf4_grouped_dgrad, "gnf4_grouped_dgrad", dy, packed, absmax,
                  torch.float32, K, 64, expert_offsets, out)


def gmxfp4_grouped_dgrad(dy, blocks, scales, expert_offsets, out=None):
    """dx[P, K] = dy[P, N] @ W_e per expert for MXFP4 weights (blocks
    [E, N, K/32, 16] or [E, N, K/2] uint8, scales [E, N, K/32] uint8 e8m0)."""
    K = 0
    if isinstance(blocks, torch.Tensor):
        K = blocks.shape[2] * 32 if blocks.dim() == 4 else blocks.shape[-1] * 2
    return _dgrad(lib.gmxfp4_grouped_dgrad, "gmxfp4_grouped_dgrad", dy, blocks, scales,
                  torch.uint8, K, 32, expert_offsets, out)


def _expert_mlp(fn, where, x, gu, gu_scale, dn, dn_scale, scale_dtype, sdiv,
                expert_offsets, row_to_token, h, out, mode):
    _need(x, "x", torch.bfloat16)
    for name, t in (("gate_up weights", gu), ("down weights", dn)):
        _need(t, name, torch.uint8)
    for name, t in (("gate_up scales", gu_scale), ("down scales", dn_scale)):
        _need(t, name, scale_dtype)
    _need(expert_offsets, "expert_offsets", torch.int32)
    if x.dim() != 2 or gu.dim() < 3 or dn.dim() < 3:
        raise ValueError(f"{where}: x must be [T, H] and the weights [E, rows, ...]")
    T, H = x.shape
    E, I2 = gu.shape[0], gu.shape[1]
    I = I2 // 2
    if I2 % 2 or dn.shape[0] != E or dn.shape[1] != H:
        raise ValueError(f"{where}: gate_up must be [E, 2I, ...] and down [E, H={H}, ...]")
    _numel(gu, "gate_up weights", E * I2 * (H // 2), where)
    _numel(gu_scale, "gate_up scales", E * I2 * (H // sdiv), where)
    _numel(dn, "down weights", E * H * (I // 2), where)
    _numel(dn_scale, "down scales", E * H * (I // sdiv), where)
    _numel(expert_offsets, "expert_offsets", E + 1, where)
    if row_to_token is not None:
        _need(row_to_token, "row_to_token", torch.int32)
        P = row_to_token.numel()
    else:
        P = T
    if h is not None:
        _need(h, "h", torch.bfloat16)
        if tuple(h.shape) != (P, I):
            raise ValueError(f"{where}: h must be [{P}, {I}]")
    if out is not None:
        _need(out, "out", torch.bfloat16)
        if tuple(out.shape) != (P, H):
            raise ValueError(f"{where}: out must be [{P}, {H}]")
    dev = _on_device(where, x=x, gu=gu, gu_scale=gu_scale, dn=dn, dn_scale=dn_scale,
                     expert_offsets=expert_offsets, row_to_token=row_to_token, h=h, out=out)
    if h is None:
        h = torch.empty((P, I), dtype=torch.bfloat16, device=dev)
    if out is None:
        out = torch.empty((P, H), dtype=torch.bfloat16, device=dev)
    m = _MODES[mode] if isinstance(mode, str) else int(mode)
    with torch.cuda.device(dev):
        _check(fn(_ptr(x), T, H, _ptr(gu), _ptr(gu_scale), _ptr(dn), _ptr(dn_scale), E, I,
                  _ptr(expert_offsets), _ptr(row_to_token), P, _ptr(h), _ptr(out), m,
                  _stream(dev)), where)
    return out, h


def gnf4_grouped_expert_mlp(x, gu_packed, gu_absmax, dn_packed, dn_absmax, expert_offsets,
                            row_to_token=None, h=None, out=None, mode="auto"):
    """Fused expert pass: gate_up [E, 2I, H/2] (gate rows then up rows),
    h = silu(gate) * up [P, I] (workspace, returned), down [E, H, I/2] ->
    out [P, H].  Returns (out, h).  mode "auto": both projections on the
    bandwidth GEMV when P <= 4 * E, else both on the tensor cores."""
    return _expert_mlp(lib.gnf4_grouped_expert_mlp, "gnf4_grouped_expert_mlp", x, gu_packed,
                       gu_absmax, dn_packed, dn_absmax, torch.float32, 64, expert_offsets,
                       row_to_token, h, out, mode)


def gmxfp4_grouped_expert_mlp(x, gu_blocks, gu_scales, dn_blocks, dn_scales, expert_offsets,
                              row_to_token=None, h=None, out=None, mode="auto"):
    """MXFP4 fused expert pass (blocks [E, rows, K/32, 16], e8m0 scales
    [E, rows, K/32]).  Returns (out, h)."""
    return _expert_mlp(lib.gmxfp4_grouped_expert_mlp, "gmxfp4_grouped_expert_mlp", x, gu_blocks,
                       gu_scales, dn_blocks, dn_scales, torch.uint8, 32, expert_offsets,
                       row_to_token, h, out, mode)


def gnf4_grouped_expert_mlp_noalloc(x, gu_packed, gu_absmax, dn_packed, dn_absmax,
                                    expert_offsets, row_to_token=None, out=None, mode="auto"):
    """gnf4_grouped_expert_mlp for callers that cannot supply device memory
    for h: the library keeps h in its own fixed 4 MiB array (P * I <=
    2,097,152).  Calls that may overlap on the GPU share that array and must
    be ordered.  Returns out [P, H] (allocated here when not given; pass
    `out` to allocate nothing at all)."""
    where = "gnf4_grouped_expert_mlp_noalloc"
    _need(x, "x", torch.bfloat16)
    _need(expert_offsets, "expert_offsets", torch.int32)
    T, H = x.shape
    E, I = gu_packed.shape[0], gu_packed.shape[1] // 2
    _numel(gu_packed, "gate_up weights", E * 2 * I * (H // 2), where)
    _numel(gu_absmax, "gate_up scales", E * 2 * I * (H // 64), where)
    _numel(dn_packed, "down weights", E * H * (I // 2), where)
    _numel(dn_absmax, "down scales", E * H * (I // 64), where)
    _numel(expert_offsets, "expert_offsets", E + 1, where)
    P = row_to_token.numel() if row_to_token is not None else T
    if out is not None:
        _need(out, "out", torch.bfloat16)
        if tuple(out.shape) != (P, H):
            raise ValueError(f"{where}: out must be [{P}, {H}]")
    dev = _on_device(where, x=x, gu=gu_packed, gs=gu_absmax, dn=dn_packed, ds=dn_absmax,
                     expert_offsets=expert_offsets, row_to_token=row_to_token, out=out)
    if out is None:
        out = torch.empty((P, H), dtype=torch.bfloat16, device=dev)
    m = _MODES[mode] if isinstance(mode, str) else int(mode)
    with torch.cuda.device(dev):
        _check(lib.gnf4_grouped_expert_mlp_noalloc(
            _ptr(x), T, H, _ptr(gu_packed), _ptr(gu_absmax), _ptr(dn_packed), _ptr(dn_absmax),
            E, I, _ptr(expert_offsets), _ptr(row_to_token), P, _ptr(out), m, _stream(dev)), where)
    return out


def _dequant(fn, where, w, scale, scale_dtype, K, sdiv, out_shape, out):
    _need(w, "packed weights", torch.uint8)
    _need(scale, "scales", scale_dtype)
    if K <= 0 or K % sdiv:
        raise ValueError(f"{where}: K={K} must be a positive multiple of {sdiv}")
    rows = w.numel() // (K // 2)
    _numel(w, "packed weights", rows * (K // 2), where)
    _numel(scale, "scales", rows * (K // sdiv), where)
    if out is not None:
        _need(out, "out", torch.bfloat16)
        _numel(out, "out", rows * K, where)
    dev = _on_device(where, w=w, scale=scale, out=out)
    if out is None:
        out = torch.empty(out_shape, dtype=torch.bfloat16, device=dev)
    with torch.cuda.device(dev):
        _check(fn(_ptr(w), _ptr(scale), rows, K, _ptr(out), _stream(dev)), where)
    return out


def gnf4_dequant(packed, absmax, out=None):
    """bf16 weights [..., K] decoded from NF4 packed [..., K/2] and absmax
    [..., K/64] (bit-exact)."""
    K = packed.shape[-1] * 2
    return _dequant(lib.gnf4_dequant, "gnf4_dequant", packed, absmax, torch.float32,
                    K, 64, packed.shape[:-1] + (K,), out)


def gmxfp4_dequant(blocks, scales, out=None):
    """bf16 weights [..., K] decoded from MXFP4 blocks [..., K/32, 16] and
    scales [..., K/32]."""
    K = blocks.shape[-2] * 32 if blocks.dim() >= 2 else 0
    return _dequant(lib.gmxfp4_dequant, "gmxfp4_dequant", blocks, scales, torch.uint8,
                    K, 32, blocks.shape[:-2] + (K,), out)


def gnf4_quantize(w):
    """fp32 [..., K] -> (packed [..., K/2] uint8, absmax [..., K/64] fp32)."""
    _need(w, "w", torch.float32)
    dev = _on_device("gnf4_quantize", w=w)
    K = w.shape[-1]
    rows = w.numel() // max(K, 1)
    packed = torch.empty(w.shape[:-1] + (K // 2,), dtype=torch.uint8, device=dev)
    absmax = torch.empty(w.shape[:-1] + (K // 64,), dtype=torch.float32, device=dev)
    with torch.cuda.device(dev):
        _check(lib.gnf4_quantize(_ptr(w), rows, K, _ptr(packed), _ptr(absmax),
                                 _stream(dev)), "gnf4_quantize")
    return packed, absmax


def gmxfp4_quantize(w):
    """fp32 [..., K] -> (blocks [..., K/32, 16] uint8, scales [..., K/32] uint8)."""
    _need(w, "w", torch.float32)
    dev = _on_device("gmxfp4_quantize", w=w)
    K = w.shape[-1]
    rows = w.numel() // max(K, 1)
    blocks = torch.empty(w.shape[:-1] + (K // 32, 16), dtype=torch.uint8, device=dev)
    scales = torch.empty(w.shape[:-1] + (K // 32,), dtype=torch.uint8, device=dev)
    with torch.cuda.device(dev):
        _check(lib.gmxfp4_quantize(_ptr(w), rows, K, _ptr(blocks), _ptr(scales),
                                   _stream(dev)), "gmxfp4_quantize")
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
