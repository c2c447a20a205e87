"""ctypes binding of libhyb (include/hyb.h): the same entry points, same names.

Argument marshalling only: tensors become device pointers, shapes become the
C sizes, the current torch stream becomes the cudaStream_t.  Every step of the
layer runs in libhyb's CUDA kernels; there is no CPU fallback.  A non-OK status
raises HybError carrying the code.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libhyb.so")

HYB_OK, HYB_ERR_INVALID_ARG, HYB_ERR_UNSUPPORTED, HYB_ERR_WORKSPACE = 0, 1, 2, 3
HYB_ERR_CUDA, HYB_ERR_TIMEOUT, HYB_ERR_DEVICE_CHECK = 4, 5, 6
HYB_DTYPE_F32, HYB_DTYPE_BF16 = 0, 1
HYB_INDEX_FLAT, HYB_INDEX_HISA = 0, 1
HYB_ATTN_PREFILL, HYB_ATTN_DECODE = 0, 1
HYB_ATTN_REAL_KV = 2   # flag OR-ed into the attention mode

_c_int, _c_size, _c_ptr, _c_float = ctypes.c_int, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_float

# name -> (restype, argtypes); must match include/hyb.h
SIGNATURES = {
    "hyb_status_string": (ctypes.c_char_p, [_c_int]),
    "hyb_abi_version": (_c_int, []),
    "hyb_kernel_launches": (ctypes.c_ulonglong, []),
    "hyb_get_device_status": (_c_int, [_c_ptr, ctypes.POINTER(_c_int)]),
    "hyb_compress": (_c_int, [_c_int, _c_int, _c_int, _c_int, _c_int, _c_ptr, _c_ptr, _c_ptr, _c_ptr,
                              _c_ptr, _c_int, _c_int, _c_int, _c_int, _c_ptr, _c_ptr, _c_ptr, _c_int,
                              _c_ptr]),
    "hyb_block_reps": (_c_int, [_c_int, _c_int, _c_int, _c_ptr, _c_int, _c_int, _c_int, _c_int, _c_ptr,
                                _c_int, _c_ptr]),
    "hyb_compress_pc": (_c_int, [_c_int, _c_int, _c_int, _c_int, _c_int, _c_ptr, _c_ptr, _c_ptr, _c_ptr, _c_ptr,
                                 _c_ptr, _c_ptr, _c_int, _c_int, _c_int, _c_int, _c_ptr, _c_ptr, _c_ptr, _c_int,
                                 _c_ptr]),
    "hyb_decode_append": (_c_int, [_c_int, _c_int, _c_int, _c_int, _c_ptr, _c_ptr, _c_ptr, _c_ptr, _c_ptr,
                                   _c_ptr, _c_ptr, _c_ptr, _c_ptr, _c_int, _c_ptr, _c_int, _c_int, _c_ptr,
                                   _c_ptr, _c_ptr, _c_int, _c_ptr, _c_int, _c_ptr, _c_ptr, _c_int, _c_int,
                                   _c_ptr, _c_int, _c_ptr]),
    "hyb_index_topk_workspace_size": (_c_size, [_c_int] * 10),
    "hyb_index_topk": (_c_int, [_c_int, _c_int, _c_int, _c_int, _c_ptr, _c_ptr, _c_ptr, _c_int, _c_int,
                                _c_int, _c_int, _c_int, _c_ptr, _c_int, _c_int, _c_int, _c_int, _c_ptr,
                                _c_ptr, _c_size, _c_ptr]),
    "hyb_index_topk_noalloc": (_c_int, [_c_int, _c_int, _c_int, _c_int, _c_ptr, _c_ptr, _c_ptr, _c_int, _c_int,
                                        _c_int, _c_int, _c_ptr, _c_ptr]),
    "hyb_attn_fwd_wait_test": (_c_int, [_c_int, _c_int, _c_int, _c_int, _c_int, _c_ptr, _c_ptr, _c_ptr, _c_ptr,
                                        _c_int, _c_int, _c_int, _c_ptr, _c_int, _c_ptr, _c_ptr, _c_int, _c_int,
                                        _c_float, _c_ptr, _c_ptr, _c_int, _c_ptr, _c_size, _c_ptr,
                                        ctypes.c_ulonglong, _c_int]),
    "hyb_attn_fwd_workspace_size": (_c_size, [_c_int] * 9),
    "hyb_attn_fwd": (_c_int, [_c_int, _c_int, _c_int, _c_int, _c_int, _c_ptr, _c_ptr, _c_ptr, _c_ptr,
                              _c_int, _c_int, _c_int, _c_ptr, _c_int, _c_ptr, _c_ptr, _c_int, _c_int,
                              _c_float, _c_ptr, _c_ptr, _c_int, _c_ptr, _c_size, _c_ptr]),
}

_lib: Optional[ctypes.CDLL] = None


class HybError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn}: {status_string(status)}")


def lib() -> ctypes.CDLL:
    """Loads libhyb.so (built in-tree by sparse_attention_hyb_b200.build); raises if absent."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m sparse_attention_hyb_b200.build` (there is no CPU fallback)")
        l = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(l, name)
            f.restype, f.argtypes = res, args
        _lib = l
    return _lib


def status_string(status: int) -> str:
    return lib().hyb_status_string(status).decode()


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return HYB_DTYPE_F32
    if t.dtype == torch.bfloat16:
        return HYB_DTYPE_BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libhyb takes device tensors only")
    if not t.is_contiguous():
        raise ValueError("libhyb takes contiguous tensors only")
    return t.data_ptr()


def _expect(t: Optional[torch.Tensor], shape, dtype, name: str):
    """Raises unless `t` has exactly this shape and dtype: the kernels write and
    read these tensors at the sizes the other arguments imply."""
    if t is None:
        raise ValueError(f"{name} is required")
    if tuple(t.shape) != tuple(shape) or t.dtype != dtype:
        raise ValueError(f"{name}: expected {tuple(shape)} {dtype}, got {tuple(t.shape)} {t.dtype}")


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _check(fn: str, status: int):
    if status != HYB_OK:
        raise HybError(fn, status)


def hyb_abi_version() -> int:
    return lib().hyb_abi_version()


def hyb_kernel_launches() -> int:
    return lib().hyb_kernel_launches()


def hyb_get_device_status(stream=None) -> int:
    out = _c_int(0)
    _check("hyb_get_device_status", lib().hyb_get_device_status(_stream(stream), ctypes.byref(out)))
    return out.value


def hyb_compress(xk, xv, xi, logits, bias, r: int, overlap: bool, j_begin: int, j_end: int,
                 kc, vc, ic, stream=None):
    """S1 on [B, L, D] raw tensors into [B, nc_cap, D] caches (see include/hyb.h)."""
    B, L, D = xk.shape
    dI = xi.shape[2] if xi is not None else 0
    st = lib().hyb_compress(_dtype_code(xk), B, L, D, dI, _ptr(xk), _ptr(xv), _ptr(xi), _ptr(logits),
                            _ptr(bias), r, int(bool(overlap)), j_begin, j_end, _ptr(kc), _ptr(vc),
                            _ptr(ic), kc.shape[1], _stream(stream))
    _check("hyb_compress", st)


def hyb_compress_pc(xk, xv, xi, z_kv, bias_kv, z_i, bias_i, r: int, overlap: bool, j_begin: int, j_end: int,
                    kc, vc, ic, stream=None):
    """S1 with per-channel weights: z_kv [B, L, D], bias_kv [span, D], z_i [B, L, dI],
    bias_i [span, dI] fp32 (see include/hyb.h)."""
    B, L, D = xk.shape
    dI = xi.shape[2] if xi is not None else 0
    st = lib().hyb_compress_pc(_dtype_code(xk), B, L, D, dI, _ptr(xk), _ptr(xv), _ptr(xi), _ptr(z_kv), _ptr(bias_kv),
                               _ptr(z_i), _ptr(bias_i), r, int(bool(overlap)), j_begin, j_end, _ptr(kc), _ptr(vc),
                               _ptr(ic), kc.shape[1], _stream(stream))
    _check("hyb_compress_pc", st)


def hyb_block_reps(ic, block: int, g_begin: int, g_end: int, reps, stream=None):
    B, nc_cap, dI = ic.shape
    st = lib().hyb_block_reps(_dtype_code(ic), B, dI, _ptr(ic), nc_cap, block, g_begin, g_end, _ptr(reps),
                              reps.shape[1], _stream(stream))
    _check("hyb_block_reps", st)


def hyb_decode_append(xk_new, xv_new, xi_new, z_new, pos, kw, vw, iw, zw,
                      bias_csa=None, r_csa: int = 0, overlap: bool = True, kc=None, vc=None, ic=None,
                      bias_hca=None, r_hca: int = 0, kc_hca=None, vc_hca=None, block: int = 0, reps=None,
                      stream=None):
    """Fused decode-step state update (see include/hyb.h): xk_new/xv_new [B, D],
    xi_new [B, dI] or None, z_new [B] fp32, pos [B] int32; rings kw/vw [B, ring, D],
    iw [B, ring, dI], zw [B, ring]; caches as in hyb_compress / hyb_block_reps."""
    B, D = xk_new.shape
    dI = xi_new.shape[1] if xi_new is not None else 0
    st = lib().hyb_decode_append(
        _dtype_code(xk_new), B, D, dI, _ptr(xk_new), _ptr(xv_new), _ptr(xi_new), _ptr(z_new), _ptr(pos),
        _ptr(kw), _ptr(vw), _ptr(iw), _ptr(zw), kw.shape[1], _ptr(bias_csa), r_csa, int(bool(overlap)),
        _ptr(kc), _ptr(vc), _ptr(ic), kc.shape[1] if kc is not None else 0, _ptr(bias_hca), r_hca, _ptr(kc_hca),
        _ptr(vc_hca), kc_hca.shape[1] if kc_hca is not None else 0, block, _ptr(reps),
        reps.shape[1] if reps is not None else 0, _stream(stream))
    _check("hyb_decode_append", st)


def hyb_index_topk_workspace_size(dtype: int, batch: int, T: int, nc: int, dI: int, k: int, mode: int,
                                  block: int = 0, top_m: int = 0, q_chunk: int = 0) -> int:
    return lib().hyb_index_topk_workspace_size(dtype, batch, T, nc, dI, k, mode, block, top_m, q_chunk)


def hyb_index_topk(qi, q_pos, ic, nc: int, r: int, k: int, mode: int, reps, block: int, top_m: int,
                   q_chunk: int, idx, ws, stream=None):
    B, T, dI = qi.shape
    _expect(q_pos, (B, T), torch.int32, "q_pos")
    _expect(idx, (B, T, k), torch.int32, "idx")
    ws_bytes = ws.numel() * ws.element_size() if ws is not None else 0
    st = lib().hyb_index_topk(_dtype_code(qi), B, T, dI, _ptr(qi), _ptr(q_pos), _ptr(ic), nc, ic.shape[1],
                              r, k, mode, _ptr(reps), reps.shape[1] if reps is not None else 0, block,
                              top_m, q_chunk, _ptr(idx), _ptr(ws), ws_bytes, _stream(stream))
    _check("hyb_index_topk", st)


def hyb_index_topk_noalloc(qi, q_pos, ic, nc: int, r: int, k: int, idx, stream=None):
    """Flat indexer whose scratch is a fixed array inside libhyb (no workspace argument)."""
    B, T, dI = qi.shape
    _expect(q_pos, (B, T), torch.int32, "q_pos")
    _expect(idx, (B, T, k), torch.int32, "idx")
    st = lib().hyb_index_topk_noalloc(_dtype_code(qi), B, T, dI, _ptr(qi), _ptr(q_pos), _ptr(ic), nc, ic.shape[1],
                                      r, k, _ptr(idx), _stream(stream))
    _check("hyb_index_topk_noalloc", st)


def hyb_attn_fwd_workspace_size(dtype: int, batch: int, T: int, H: int, D: int, k: int, nc: int, W: int,
                                mode: int) -> int:
    return lib().hyb_attn_fwd_workspace_size(dtype, batch, T, H, D, k, nc, W, mode)


def hyb_attn_fwd(q, q_pos, kc, vc, nc: int, r: int, idx, k: int, kw, vw, W: int, scale: float, o, lse,
                 mode: int, ws, stream=None):
    B, T, H, D = q.shape
    _expect(q_pos, (B, T), torch.int32, "q_pos")
    if idx is not None:
        _expect(idx, (B, T, k), torch.int32, "idx")
    _expect(o, (B, T, H, D), q.dtype, "o")
    if lse is not None:
        _expect(lse, (B, T, H), torch.float32, "lse")
    ws_bytes = ws.numel() * ws.element_size() if ws is not None else 0
    st = lib().hyb_attn_fwd(_dtype_code(q), B, T, H, D, _ptr(q), _ptr(q_pos), _ptr(kc), _ptr(vc), nc,
                            kc.shape[1] if kc is not None else 0, r, _ptr(idx), k, _ptr(kw), _ptr(vw),
                            kw.shape[1], W, float(scale), _ptr(o), _ptr(lse), mode, _ptr(ws), ws_bytes,
                            _stream(stream))
    _check("hyb_attn_fwd", st)


def hyb_attn_fwd_wait_test(q, q_pos, kc, vc, nc: int, r: int, idx, k: int, kw, vw, W: int, scale: float, o, lse,
                           mode: int, ws, wait_ns: int, drop_arrival: bool, stream=None):
    """Test hook of the bounded device waits (see include/hyb.h): hyb_attn_fwd with
    every wait limited to wait_ns, optionally withholding one K-tile arrival."""
    B, T, H, D = q.shape
    _expect(q_pos, (B, T), torch.int32, "q_pos")
    if idx is not None:
        _expect(idx, (B, T, k), torch.int32, "idx")
    _expect(o, (B, T, H, D), q.dtype, "o")
    if lse is not None:
        _expect(lse, (B, T, H), torch.float32, "lse")
    ws_bytes = ws.numel() * ws.element_size() if ws is not None else 0
    st = lib().hyb_attn_fwd_wait_test(_dtype_code(q), B, T, H, D, _ptr(q), _ptr(q_pos), _ptr(kc), _ptr(vc), nc,
                                      kc.shape[1] if kc is not None else 0, r, _ptr(idx), k, _ptr(kw), _ptr(vw),
                                      kw.shape[1], W, float(scale), _ptr(o), _ptr(lse), mode, _ptr(ws), ws_bytes,
                                      _stream(stream), int(wait_ns), int(bool(drop_arrival)))
    _check("hyb_attn_fwd_wait_test", st)
