"""Fused smooth-rotate-MXFP4 quantisation for B200 (sm_100a): Python binding.

This module only marshals arguments into the C ABI of ``libmxq.so`` (declared in
``include/mxq.h``).  Every step of the path runs in the library's CUDA kernels:
the per-channel smoothing, the 32x32 block rotation, the scale and code
decisions and the packing.  There is no CPU or PyTorch fallback.  If the
library is missing or the device is not supported, the calls raise.

The method is the online step of DuQuant++ (jsqmd.com/news/928156, §2.1, §2.3,
§3.3).  Each 32-element group of an activation row is divided per channel by Λ,
multiplied by one shared orthogonal 32x32 matrix R̂, and quantised to MXFP4.
MXFP4 here means one E8M0 scale per group and E2M1 codes, two per byte, the
even column in the low nibble.
"""
from __future__ import annotations

import ctypes
import os
import re
from typing import Optional, Tuple

import torch

__all__ = [
    "MxqError", "smooth_rotate_quantize", "smooth_rotate_quantize_mma", "smooth_rotate_quantize_nvfp4",
    "smooth_rotate_quantize_nvfp4_mma", "smooth_rotate_f32",
    "weight_rotate_quantize", "rotate_quantize_block", "rotate_block_f32", "scales_to_mma_layout",
    "mxfp4_gemm", "nvfp4_scales_to_mma_layout", "nvfp4_gemm", "dequantize", "quant_error", "rotation_search",
    "sync_check", "selftest_bounded_wait",
    "status_string", "version", "lib", "LIB_PATH", "HEADER_PATH", "declared_symbols",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmxq.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "mxq.h")

MXQ_OK = 0
_STATUS_NAMES = {0: "MXQ_OK", 1: "MXQ_ERR_INVALID_ARG", 2: "MXQ_ERR_UNSUPPORTED", 3: "MXQ_ERR_CUDA",
                 4: "MXQ_ERR_TIMEOUT"}


class MxqError(RuntimeError):
    """A libmxq call returned a status other than MXQ_OK."""

    def __init__(self, status: int, where: str, detail: str = ""):
        self.status = status
        super().__init__(f"{where}: {_STATUS_NAMES.get(status, status)}" + (f" ({detail})" if detail else ""))


_lib = None


def lib() -> ctypes.CDLL:
    """Load libmxq.so (once).  Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise MxqError(3, "load", f"{LIB_PATH} is missing; build it with "
                                      "`python -m mxfp4_block_rotation_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I64, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
        L.mxq_smooth_rotate_quantize.argtypes = [P, I64, I64, P, P, P, P, P]
        L.mxq_smooth_rotate_quantize.restype = I
        L.mxq_smooth_rotate_quantize_mma.argtypes = [P, I64, I64, P, P, P, P, P]
        L.mxq_smooth_rotate_quantize_mma.restype = I
        L.mxq_smooth_rotate_quantize_nvfp4_mma.argtypes = [P, I64, I64, P, P, P, P, P, P]
        L.mxq_smooth_rotate_quantize_nvfp4_mma.restype = I
        L.mxq_smooth_rotate_f32.argtypes = [P, I64, I64, P, P, P, P]
        L.mxq_smooth_rotate_f32.restype = I
        L.mxq_rotate_quantize_block.argtypes = [P, I64, I64, I, P, P, P, P, P]
        L.mxq_rotate_quantize_block.restype = I
        L.mxq_rotate_block_f32.argtypes = [P, I64, I64, I, P, P, P, P]
        L.mxq_rotate_block_f32.restype = I
        L.mxq_weight_rotate_quantize.argtypes = [P, I64, I64, P, P, P, P, P]
        L.mxq_weight_rotate_quantize.restype = I
        L.mxq_smooth_rotate_quantize_nvfp4.argtypes = [P, I64, I64, P, P, P, P, P, P]
        L.mxq_smooth_rotate_quantize_nvfp4.restype = I
        L.mxq_mxfp4_gemm.argtypes = [P, P, P, P, I64, I64, I64, P, I, P]
        L.mxq_scales_mma_bytes.argtypes = [I64, I64]
        L.mxq_scales_mma_bytes.restype = ctypes.c_size_t
        L.mxq_scales_to_mma_layout.argtypes = [P, I64, I64, P, P]
        L.mxq_nvfp4_scales_mma_bytes.argtypes = [I64, I64]
        L.mxq_nvfp4_scales_mma_bytes.restype = ctypes.c_size_t
        L.mxq_nvfp4_scales_to_mma_layout.argtypes = [P, I64, I64, P, P]
        L.mxq_nvfp4_scales_to_mma_layout.restype = I
        L.mxq_nvfp4_gemm.argtypes = [P, P, P, P, P, P, I64, I64, I64, P, I, P]
        L.mxq_nvfp4_gemm.restype = I
        L.mxq_scales_to_mma_layout.restype = I
        L.mxq_mxfp4_gemm.restype = I
        L.mxq_dequantize.argtypes = [P, P, I64, I64, P, P, P, P]
        L.mxq_dequantize.restype = I
        L.mxq_selftest_bounded_wait.argtypes = [ctypes.c_uint32, P, P]
        L.mxq_selftest_bounded_wait.restype = I
        L.mxq_quant_error_workspace_bytes.argtypes = [I64, I64, I]
        L.mxq_quant_error_workspace_bytes.restype = ctypes.c_size_t
        L.mxq_quant_error.argtypes = [P, I64, I64, P, P, P, P, P, ctypes.c_size_t, P]
        L.mxq_quant_error.restype = I
        L.mxq_quant_error_noalloc.argtypes = [P, I64, I64, P, P, P, P, P]
        L.mxq_quant_error_noalloc.restype = I
        L.mxq_rotation_search_workspace_bytes.argtypes = [I64, I64, I]
        L.mxq_rotation_search_workspace_bytes.restype = ctypes.c_size_t
        L.mxq_rotation_search.argtypes = [P, I64, I64, P, I, I, P, P, P, P, P, P, P, ctypes.c_size_t, P]
        L.mxq_rotation_search.restype = I
        L.mxq_sync_check.argtypes = [P]
        L.mxq_sync_check.restype = I
        L.mxq_status_string.argtypes = [I]
        L.mxq_status_string.restype = ctypes.c_char_p
        L.mxq_last_cuda_error.argtypes = []
        L.mxq_last_cuda_error.restype = ctypes.c_char_p
        L.mxq_version.argtypes = []
        L.mxq_version.restype = I
        _lib = L
    return _lib


def declared_symbols() -> list[str]:
    """Names of the functions include/mxq.h declares."""
    with open(HEADER_PATH) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mxq_[a-z0-9_]+)\s*\(", text)))


def status_string(status: int) -> str:
    return lib().mxq_status_string(int(status)).decode()


def version() -> int:
    return int(lib().mxq_version())


def _check(status: int, where: str) -> None:
    if status != MXQ_OK:
        raise MxqError(status, where, lib().mxq_last_cuda_error().decode())


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device: torch.device, stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream))


def _need(t: torch.Tensor, name: str, dtype: torch.dtype, device: torch.device) -> None:
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.device != device:
        raise ValueError(f"{name} must be on {device}, got {t.device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _inputs(x, rhat, lam):
    if x.dim() != 2:
        raise ValueError("x must be 2-D [rows, cols]")
    dev = x.device
    if dev.type != "cuda":
        raise ValueError("x must be a CUDA tensor (this library has no CPU path)")
    _need(x, "x", torch.bfloat16, dev)
    _need(rhat, "rhat", torch.bfloat16, dev)
    if tuple(rhat.shape) != (32, 32):
        raise ValueError("rhat must be [32, 32]")
    if lam is not None:
        _need(lam, "lam", torch.float32, dev)
        if tuple(lam.shape) != (x.shape[1],):
            raise ValueError("lam must be [cols]")
    return dev


def smooth_rotate_quantize(x: torch.Tensor, rhat: torch.Tensor, lam: Optional[torch.Tensor] = None, *,
                           codes: Optional[torch.Tensor] = None, scales: Optional[torch.Tensor] = None,
                           stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """MXFP4(X · Λ⁻¹ · R̂) -> (codes uint8 [rows, cols/2], scales uint8 [rows, cols/32])."""
    dev = _inputs(x, rhat, lam)
    rows, cols = x.shape
    if codes is None:
        codes = torch.empty((rows, cols // 2), dtype=torch.uint8, device=dev)
    if scales is None:
        scales = torch.empty((rows, cols // 32), dtype=torch.uint8, device=dev)
    _need(codes, "codes", torch.uint8, dev)
    _need(scales, "scales", torch.uint8, dev)
    st = lib().mxq_smooth_rotate_quantize(_ptr(x), rows, cols, _ptr(rhat), _ptr(lam), _ptr(codes),
                                          _ptr(scales), _stream(dev, stream))
    _check(st, "mxq_smooth_rotate_quantize")
    return codes, scales


def smooth_rotate_quantize_mma(x: torch.Tensor, rhat: torch.Tensor, lam: Optional[torch.Tensor] = None, *,
                               codes: Optional[torch.Tensor] = None, sf: Optional[torch.Tensor] = None,
                               stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """MXFP4(X · Λ⁻¹ · R̂) -> (codes uint8 [rows, cols/2], scales in the block-scaled MMA layout: flat
    uint8 of mxq_scales_mma_bytes(rows, cols)), ready for mxfp4_gemm with no layout pass."""
    dev = _inputs(x, rhat, lam)
    rows, cols = x.shape
    n = int(lib().mxq_scales_mma_bytes(rows, cols))
    if codes is None:
        codes = torch.empty((rows, cols // 2), dtype=torch.uint8, device=dev)
    if sf is None:
        sf = torch.empty(n, dtype=torch.uint8, device=dev)
    _need(codes, "codes", torch.uint8, dev)
    _need(sf, "sf", torch.uint8, dev)
    if sf.numel() < n:
        raise ValueError(f"sf needs {n} bytes")
    st = lib().mxq_smooth_rotate_quantize_mma(_ptr(x), rows, cols, _ptr(rhat), _ptr(lam), _ptr(codes), _ptr(sf),
                                              _stream(dev, stream))
    _check(st, "mxq_smooth_rotate_quantize_mma")
    return codes, sf


def smooth_rotate_quantize_nvfp4_mma(x: torch.Tensor, rhat: torch.Tensor, tensor_scale: torch.Tensor,
                                     lam: Optional[torch.Tensor] = None, *, codes: Optional[torch.Tensor] = None,
                                     sf: Optional[torch.Tensor] = None,
                                     stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """NVFP4(X · Λ⁻¹ · R̂) -> (codes uint8 [rows, cols/2], E4M3 scales in the block-scaled MMA layout:
    flat uint8 of mxq_nvfp4_scales_mma_bytes(rows, cols)), ready for nvfp4_gemm with no layout pass."""
    dev = _inputs(x, rhat, lam)
    _need(tensor_scale, "tensor_scale", torch.float32, dev)
    if tensor_scale.numel() != 1:
        raise ValueError("tensor_scale must hold one float")
    rows, cols = x.shape
    n = int(lib().mxq_nvfp4_scales_mma_bytes(rows, cols))
    if codes is None:
        codes = torch.empty((rows, cols // 2), dtype=torch.uint8, device=dev)
    if sf is None:
        sf = torch.empty(n, dtype=torch.uint8, device=dev)
    _need(codes, "codes", torch.uint8, dev)
    _need(sf, "sf", torch.uint8, dev)
    if sf.numel() < n:
        raise ValueError(f"sf needs {n} bytes")
    st = lib().mxq_smooth_rotate_quantize_nvfp4_mma(_ptr(x), rows, cols, _ptr(rhat), _ptr(lam), _ptr(tensor_scale),
                                                    _ptr(codes), _ptr(sf), _stream(dev, stream))
    _check(st, "mxq_smooth_rotate_quantize_nvfp4_mma")
    return codes, sf


def smooth_rotate_quantize_nvfp4(x: torch.Tensor, rhat: torch.Tensor, tensor_scale: torch.Tensor,
                                 lam: Optional[torch.Tensor] = None, *, codes: Optional[torch.Tensor] = None,
                                 scales: Optional[torch.Tensor] = None,
                                 stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """NVFP4(X · Λ⁻¹ · R̂) -> (codes uint8 [rows, cols/2], E4M3 scales uint8 [rows, cols/16]).

    tensor_scale: fp32 [1] on the device (the per-tensor scale s_t)."""
    dev = _inputs(x, rhat, lam)
    _need(tensor_scale, "tensor_scale", torch.float32, dev)
    if tensor_scale.numel() != 1:
        raise ValueError("tensor_scale must hold one float")
    rows, cols = x.shape
    if codes is None:
        codes = torch.empty((rows, cols // 2), dtype=torch.uint8, device=dev)
    if scales is None:
        scales = torch.empty((rows, cols // 16), dtype=torch.uint8, device=dev)
    _need(codes, "codes", torch.uint8, dev)
    _need(scales, "scales", torch.uint8, dev)
    st = lib().mxq_smooth_rotate_quantize_nvfp4(_ptr(x), rows, cols, _ptr(rhat), _ptr(lam), _ptr(tensor_scale),
                                                _ptr(codes), _ptr(scales), _stream(dev, stream))
    _check(st, "mxq_smooth_rotate_quantize_nvfp4")
    return codes, scales


def smooth_rotate_f32(x: torch.Tensor, rhat: torch.Tensor, lam: Optional[torch.Tensor] = None, *,
                      out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """X · Λ⁻¹ · R̂ in fp32 [rows, cols] (the values the quantiser decides on)."""
    dev = _inputs(x, rhat, lam)
    rows, cols = x.shape
    if out is None:
        out = torch.empty((rows, cols), dtype=torch.float32, device=dev)
    _need(out, "out", torch.float32, dev)
    st = lib().mxq_smooth_rotate_f32(_ptr(x), rows, cols, _ptr(rhat), _ptr(lam), _ptr(out),
                                     _stream(dev, stream))
    _check(st, "mxq_smooth_rotate_f32")
    return out


def weight_rotate_quantize(wt: torch.Tensor, rhat: torch.Tensor, lam: Optional[torch.Tensor] = None, *,
                           codes: Optional[torch.Tensor] = None, scales: Optional[torch.Tensor] = None,
                           stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """MXFP4(Wᵀ · Λ · R̂): the absorbed weights, W given transposed as wt [n_out, k_in] bf16."""
    dev = _inputs(wt, rhat, lam)
    rows, cols = wt.shape
    if codes is None:
        codes = torch.empty((rows, cols // 2), dtype=torch.uint8, device=dev)
    if scales is None:
        scales = torch.empty((rows, cols // 32), dtype=torch.uint8, device=dev)
    _need(codes, "codes", torch.uint8, dev)
    _need(scales, "scales", torch.uint8, dev)
    st = lib().mxq_weight_rotate_quantize(_ptr(wt), rows, cols, _ptr(rhat), _ptr(lam), _ptr(codes), _ptr(scales),
                                          _stream(dev, stream))
    _check(st, "mxq_weight_rotate_quantize")
    return codes, scales


def scales_to_mma_layout(scales: torch.Tensor, *, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Row-major E8M0 scales [rows, K/32] -> the block-scaled MMA's 512-byte atoms (flat uint8)."""
    dev = scales.device
    if dev.type != "cuda":
        raise ValueError("scales must be a CUDA tensor (this library has no CPU path)")
    _need(scales, "scales", torch.uint8, dev)
    rows, G = scales.shape
    n = int(lib().mxq_scales_mma_bytes(rows, G * 32))
    if out is None:
        out = torch.empty(n, dtype=torch.uint8, device=dev)
    _need(out, "out", torch.uint8, dev)
    if out.numel() < n:
        raise ValueError(f"out needs {n} bytes")
    st = lib().mxq_scales_to_mma_layout(_ptr(scales), rows, G * 32, _ptr(out), _stream(dev, stream))
    _check(st, "mxq_scales_to_mma_layout")
    return out


def mxfp4_gemm(a_codes: torch.Tensor, a_scales: torch.Tensor, b_codes: torch.Tensor, b_scales: torch.Tensor, *,
               out_dtype: torch.dtype = torch.float32, out: Optional[torch.Tensor] = None,
               stream=None) -> torch.Tensor:
    """Y = deq(A) · deq(B)ᵀ on the block-scaled tensor cores; A [M, K/2] codes, B [N, K/2] codes.

    Scales may be row-major ([M, K/32], [N, K/32]: converted here by the layout kernel) or
    already in the MMA layout (flat uint8 of mxq_scales_mma_bytes)."""
    dev = a_codes.device
    if dev.type != "cuda":
        raise ValueError("operands must be CUDA tensors (this library has no CPU path)")
    for t, name in ((a_codes, "a_codes"), (a_scales, "a_scales"), (b_codes, "b_codes"), (b_scales, "b_scales")):
        _need(t, name, torch.uint8, dev)
    M, K = a_codes.shape[0], a_codes.shape[1] * 2
    N = b_codes.shape[0]
    if b_codes.shape[1] * 2 != K:
        raise ValueError("operand shapes disagree")
    if a_scales.dim() == 2:
        if tuple(a_scales.shape) != (M, K // 32):
            raise ValueError("a_scales must be [M, K/32]")
        a_scales = scales_to_mma_layout(a_scales, stream=stream) if M and K else a_scales
    if b_scales.dim() == 2:
        if tuple(b_scales.shape) != (N, K // 32):
            raise ValueError("b_scales must be [N, K/32]")
        b_scales = scales_to_mma_layout(b_scales, stream=stream) if N and K else b_scales
    if out is not None:
        out_dtype = out.dtype
    if out_dtype not in (torch.float32, torch.bfloat16):
        raise ValueError("out_dtype must be float32 or bfloat16")
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=dev)
    _need(out, "out", out_dtype, dev)
    st = lib().mxq_mxfp4_gemm(_ptr(a_codes), _ptr(a_scales), _ptr(b_codes), _ptr(b_scales), M, N, K, _ptr(out),
                              int(out_dtype == torch.bfloat16), _stream(dev, stream))
    _check(st, "mxq_mxfp4_gemm")
    return out


def nvfp4_scales_to_mma_layout(scales: torch.Tensor, *, out: Optional[torch.Tensor] = None,
                               stream=None) -> torch.Tensor:
    """Row-major E4M3 scales [rows, K/16] -> the block-scaled MMA's 512-byte atoms (flat uint8)."""
    dev = scales.device
    if dev.type != "cuda":
        raise ValueError("scales must be a CUDA tensor (this library has no CPU path)")
    _need(scales, "scales", torch.uint8, dev)
    rows, nb = scales.shape
    n = int(lib().mxq_nvfp4_scales_mma_bytes(rows, nb * 16))
    if out is None:
        out = torch.empty(n, dtype=torch.uint8, device=dev)
    _need(out, "out", torch.uint8, dev)
    if out.numel() < n:
        raise ValueError(f"out needs {n} bytes")
    st = lib().mxq_nvfp4_scales_to_mma_layout(_ptr(scales), rows, nb * 16, _ptr(out), _stream(dev, stream))
    _check(st, "mxq_nvfp4_scales_to_mma_layout")
    return out


def nvfp4_gemm(a_codes: torch.Tensor, a_scales: torch.Tensor, a_tscale: torch.Tensor, b_codes: torch.Tensor,
               b_scales: torch.Tensor, b_tscale: torch.Tensor, *, out_dtype: torch.dtype = torch.float32,
               out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Y = deq(A) · deq(B)ᵀ for NVFP4 operands (E4M3 per 16 k; fp32 tensor scales a_tscale, b_tscale of
    one element each, on the device).  Scales row-major ([rows, K/16]) or already in the MMA layout."""
    dev = a_codes.device
    if dev.type != "cuda":
        raise ValueError("operands must be CUDA tensors (this library has no CPU path)")
    for t, name in ((a_codes, "a_codes"), (a_scales, "a_scales"), (b_codes, "b_codes"), (b_scales, "b_scales")):
        _need(t, name, torch.uint8, dev)
    for t, name in ((a_tscale, "a_tscale"), (b_tscale, "b_tscale")):
        _need(t, name, torch.float32, dev)
        if t.numel() != 1:
            raise ValueError(f"{name} must hold one float")
    M, K = a_codes.shape[0], a_codes.shape[1] * 2
    N = b_codes.shape[0]
    if b_codes.shape[1] * 2 != K:
        raise ValueError("operand shapes disagree")
    if a_scales.dim() == 2:
        if tuple(a_scales.shape) != (M, K // 16):
            raise ValueError("a_scales must be [M, K/16]")
        a_scales = nvfp4_scales_to_mma_layout(a_scales, stream=stream) if M and K else a_scales
    if b_scales.dim() == 2:
        if tuple(b_scales.shape) != (N, K // 16):
            raise ValueError("b_scales must be [N, K/16]")
        b_scales = nvfp4_scales_to_mma_layout(b_scales, stream=stream) if N and K else b_scales
    if out is not None:
        out_dtype = out.dtype
    if out_dtype not in (torch.float32, torch.bfloat16):
        raise ValueError("out_dtype must be float32 or bfloat16")
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=dev)
    _need(out, "out", out_dtype, dev)
    st = lib().mxq_nvfp4_gemm(_ptr(a_codes), _ptr(a_scales), _ptr(a_tscale), _ptr(b_codes), _ptr(b_scales),
                              _ptr(b_tscale), M, N, K, _ptr(out), int(out_dtype == torch.bfloat16),
                              _stream(dev, stream))
    _check(st, "mxq_nvfp4_gemm")
    return out


def _block_inputs(x, r, lam):
    if x.dim() != 2:
        raise ValueError("x must be 2-D [rows, cols]")
    dev = x.device
    if dev.type != "cuda":
        raise ValueError("x must be a CUDA tensor (this library has no CPU path)")
    _need(x, "x", torch.bfloat16, dev)
    _need(r, "r", torch.bfloat16, dev)
    if r.dim() != 2 or r.shape[0] != r.shape[1]:
        raise ValueError("r must be square [block, block]")
    if lam is not None:
        _need(lam, "lam", torch.float32, dev)
        if tuple(lam.shape) != (x.shape[1],):
            raise ValueError("lam must be [cols]")
    return dev, int(r.shape[0])


def rotate_quantize_block(x: torch.Tensor, r: torch.Tensor, lam: Optional[torch.Tensor] = None, *,
                          codes: Optional[torch.Tensor] = None, scales: Optional[torch.Tensor] = None,
                          stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """MXFP4 of X · Λ⁻¹ rotated in blocks of B = r.shape[0] columns (16, 32, 64 or 128), 32-column groups."""
    dev, blk = _block_inputs(x, r, lam)
    rows, cols = x.shape
    if codes is None:
        codes = torch.empty((rows, cols // 2), dtype=torch.uint8, device=dev)
    if scales is None:
        scales = torch.empty((rows, cols // 32), dtype=torch.uint8, device=dev)
    _need(codes, "codes", torch.uint8, dev)
    _need(scales, "scales", torch.uint8, dev)
    st = lib().mxq_rotate_quantize_block(_ptr(x), rows, cols, blk, _ptr(r), _ptr(lam), _ptr(codes), _ptr(scales),
                                         _stream(dev, stream))
    _check(st, "mxq_rotate_quantize_block")
    return codes, scales


def rotate_block_f32(x: torch.Tensor, r: torch.Tensor, lam: Optional[torch.Tensor] = None, *,
                     out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """X · Λ⁻¹ rotated in blocks of B = r.shape[0] columns, in fp32 [rows, cols]."""
    dev, blk = _block_inputs(x, r, lam)
    rows, cols = x.shape
    if out is None:
        out = torch.empty((rows, cols), dtype=torch.float32, device=dev)
    _need(out, "out", torch.float32, dev)
    st = lib().mxq_rotate_block_f32(_ptr(x), rows, cols, blk, _ptr(r), _ptr(lam), _ptr(out), _stream(dev, stream))
    _check(st, "mxq_rotate_block_f32")
    return out


def dequantize(codes: torch.Tensor, scales: torch.Tensor, rhat: Optional[torch.Tensor] = None,
               lam: Optional[torch.Tensor] = None, *, out: Optional[torch.Tensor] = None,
               stream=None) -> torch.Tensor:
    """bf16 [rows, cols] from MXFP4 codes/scales; with rhat (and lam) the transform is undone."""
    if codes.dim() != 2 or scales.dim() != 2:
        raise ValueError("codes and scales must be 2-D")
    dev = codes.device
    if dev.type != "cuda":
        raise ValueError("codes must be a CUDA tensor (this library has no CPU path)")
    rows, half = codes.shape
    cols = half * 2
    _need(codes, "codes", torch.uint8, dev)
    _need(scales, "scales", torch.uint8, dev)
    if tuple(scales.shape) != (rows, cols // 32):
        raise ValueError("scales must be [rows, cols/32]")
    if rhat is not None:
        _need(rhat, "rhat", torch.bfloat16, dev)
    if lam is not None:
        _need(lam, "lam", torch.float32, dev)
    if out is None:
        out = torch.empty((rows, cols), dtype=torch.bfloat16, device=dev)
    _need(out, "out", torch.bfloat16, dev)
    st = lib().mxq_dequantize(_ptr(codes), _ptr(scales), rows, cols, _ptr(rhat), _ptr(lam), _ptr(out),
                              _stream(dev, stream))
    _check(st, "mxq_dequantize")
    return out


def quant_error(x: torch.Tensor, rhat: torch.Tensor, lam: Optional[torch.Tensor] = None, *,
                per_group: bool = True, workspace: Optional[torch.Tensor] = None, stream=None):
    """Per-group MXFP4 error ||Q(y) - y|| / ||y|| (fp32 [rows, cols/32], or None) and its mean (a 0-d
    float64 device tensor).  `workspace` (uint8, device) is allocated here when not given."""
    dev = _inputs(x, rhat, lam)
    rows, cols = x.shape
    need = int(lib().mxq_quant_error_workspace_bytes(rows, cols, int(lam is not None)))
    if workspace is None:
        workspace = torch.empty(max(need, 8), dtype=torch.uint8, device=dev)
    _need(workspace, "workspace", torch.uint8, dev)
    err = torch.empty((rows, cols // 32), dtype=torch.float32, device=dev) if per_group else None
    mean = torch.empty((), dtype=torch.float64, device=dev)
    st = lib().mxq_quant_error(_ptr(x), rows, cols, _ptr(rhat), _ptr(lam), _ptr(err), _ptr(mean),
                               _ptr(workspace), workspace.numel(), _stream(dev, stream))
    _check(st, "mxq_quant_error")
    return err, mean


def rotation_search(x: torch.Tensor, lam: Optional[torch.Tensor] = None, *, max_steps: int = 128,
                    n_angle: int = 32, workspace: Optional[torch.Tensor] = None, stream=None) -> dict:
    """The outlier-aware greedy Givens search for the shared rotation (DuQuant++ write-up, §3.2).

    Returns device tensors: R (float64 [32, 32]), rhat (R in bf16, the hot path's input),
    trace (int32 [max_steps, 3]: d, j, angle per step; rows past `steps` unwritten),
    linf (float64 [max_steps + 1]), steps (int32 0-d) and group (int64 0-d).
    `workspace` (uint8, device) is allocated here when not given.  Nothing is synchronised.
    """
    if x.dim() != 2:
        raise ValueError("x must be 2-D [rows, cols]")
    dev = x.device
    if dev.type != "cuda":
        raise ValueError("x must be a CUDA tensor (this library has no CPU path)")
    _need(x, "x", torch.bfloat16, dev)
    if lam is not None:
        _need(lam, "lam", torch.float32, dev)
        if tuple(lam.shape) != (x.shape[1],):
            raise ValueError("lam must be [cols]")
    rows, cols = x.shape
    need = int(lib().mxq_rotation_search_workspace_bytes(rows, cols, int(n_angle)))
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    _need(workspace, "workspace", torch.uint8, dev)
    out = {
        "R": torch.empty((32, 32), dtype=torch.float64, device=dev),
        "rhat": torch.empty((32, 32), dtype=torch.bfloat16, device=dev),
        "trace": torch.zeros((max(int(max_steps), 1), 3), dtype=torch.int32, device=dev),
        "linf": torch.zeros(int(max_steps) + 1, dtype=torch.float64, device=dev),
        "steps": torch.empty((), dtype=torch.int32, device=dev),
        "group": torch.empty((), dtype=torch.int64, device=dev),
    }
    st = lib().mxq_rotation_search(_ptr(x), rows, cols, _ptr(lam), int(max_steps), int(n_angle), _ptr(out["R"]),
                                   _ptr(out["rhat"]), _ptr(out["trace"]), _ptr(out["linf"]), _ptr(out["steps"]),
                                   _ptr(out["group"]), _ptr(workspace), workspace.numel(), _stream(dev, stream))
    _check(st, "mxq_rotation_search")
    return out


def selftest_bounded_wait(timeout_ms: int = 50, device=None, stream=None) -> int:
    """Run the bounded-wait diagnostic kernel; returns its result code (2 = wait ran out as designed)."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    res = torch.zeros(1, dtype=torch.int32, device=dev)
    _check(lib().mxq_selftest_bounded_wait(int(timeout_ms), _ptr(res), _stream(dev, stream)),
           "mxq_selftest_bounded_wait")
    return int(res.item())


def sync_check(stream=None, device=None) -> None:
    """Synchronise the stream and raise if a kernel's bounded wait ran out or the stream failed."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    _check(lib().mxq_sync_check(_stream(dev, stream)), "mxq_sync_check")
