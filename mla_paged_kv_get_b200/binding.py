"""ctypes binding of the C ABI in ``include/mla_b200.h``.

Argument marshalling only: every step of the decode runs in the CUDA library
(``libmla_b200.so``).  PyTorch supplies device memory and the current stream.
There is no CPU or PyTorch fallback: if the library cannot be loaded, every
call raises.

Public calls mirror the pages' API (cnblogs "DeepSeek 开源记-第1天-FlashMLA",
§6.2 基本使用):

    tile_md, num_splits = get_metadata(cache_seqlens, s_q * h_q // h_kv, h_kv)
    out, lse = decode_paged(q, k_cache, block_table, cache_seqlens, dv,
                            tile_md, num_splits, causal=causal)
"""

from __future__ import annotations

import ctypes
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_NAME = "libmla_b200.so"
_lib = None

HEAD_DIM = 576
VALUE_DIM = 512
PAGE_SIZE = 64
MD_WORDS = 8

MLA_OK = 0
MLA_ERR_TIMEOUT = -5
MLA_ERR_BAD_INPUT = -6


class MLAError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {status_string(code)} ({code})")


def library_path() -> str:
    return os.path.join(_HERE, _LIB_NAME)


def load_library() -> ctypes.CDLL:
    """Load ``libmla_b200.so`` (built by ``mla_paged_kv_get_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    path = library_path()
    if not os.path.exists(path):
        raise RuntimeError(f"CUDA library not built: {path} is missing "
                           "(run `python -m mla_paged_kv_get_b200.build`)")
    lib = ctypes.CDLL(path)
    vp, i32p, ci, cf, csz = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    lib.mla_status_string.argtypes = [ci]
    lib.mla_status_string.restype = ctypes.c_char_p
    lib.mla_device_sm_count.argtypes = []
    lib.mla_device_sm_count.restype = ci
    lib.mla_rows_per_block.argtypes = [ci]
    lib.mla_rows_per_block.restype = ci
    lib.mla_num_parts.argtypes = [ci, ci, ci]
    lib.mla_num_parts.restype = ci
    lib.mla_get_metadata.argtypes = [i32p, ci, ci, ci, ci, i32p, i32p, ctypes.POINTER(ci), vp]
    lib.mla_get_metadata.restype = ci
    lib.mla_workspace_bytes.argtypes = [ci, ci, ci, ci, ci]
    lib.mla_workspace_bytes.restype = csz
    dec = [vp, vp, ci, i32p, ci, i32p, ci, ci, ci, ci, ci, ci, i32p, i32p, ci, ci, cf, vp, csz, vp, vp, i32p]
    lib.mla_decode_paged.argtypes = dec + [vp]
    lib.mla_decode_paged.restype = ci
    lib.mla_decode_paged_ex.argtypes = dec + [ci, ctypes.c_ulonglong, vp]
    lib.mla_decode_paged_ex.restype = ci
    lib.mla_combine.argtypes = [i32p, vp, csz, ci, ci, ci, ci, ci, vp, vp, vp]
    lib.mla_decode_paged_typed.argtypes = [ci] + dec + [ci, ctypes.c_ulonglong, vp]
    lib.mla_decode_paged_typed.restype = ci
    lib.mla_combine_typed.argtypes = [ci, i32p, vp, csz, ci, ci, ci, ci, ci, vp, vp, vp]
    lib.mla_combine_typed.restype = ci
    lib.mla_combine.restype = ci
    _lib = lib
    return lib


def status_string(code: int) -> str:
    try:
        return load_library().mla_status_string(int(code)).decode()
    except Exception:  # library missing: still give a readable message
        return f"status {code}"


def _check(code: int, where: str) -> None:
    if code != MLA_OK:
        raise MLAError(code, where)


def _stream_handle(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


# element types of q / k_cache / out and their codes in the C ABI (MLA_DTYPE_*)
DTYPES = {torch.bfloat16: 0, torch.float16: 1}


def _ptr(t: torch.Tensor | None) -> ctypes.c_void_p:
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _need(t: torch.Tensor, name: str, dtype, device=None) -> None:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def num_parts(rows_per_kv: int, h_kv: int, num_sms: int | None = None) -> int:
    lib = load_library()
    if num_sms is None:
        num_sms = lib.mla_device_sm_count()
        _check(min(num_sms, 0), "mla_device_sm_count")
    g = lib.mla_num_parts(rows_per_kv, h_kv, num_sms)
    _check(min(g, 0), "mla_num_parts")
    return g


def workspace_bytes(batch: int, rows_per_kv: int, h_kv: int, num_parts_: int, dv: int = VALUE_DIM) -> int:
    return int(load_library().mla_workspace_bytes(batch, rows_per_kv, h_kv, dv, num_parts_))


def get_metadata(cache_seqlens: torch.Tensor, rows_per_kv: int, h_kv: int, num_sms: int | None = None,
                 stream=None):
    """Tile-scheduler table ``[G, 8]`` and ``num_splits`` ``[B + 1]`` (int32, device)."""
    lib = load_library()
    _need(cache_seqlens, "cache_seqlens", torch.int32)
    B = cache_seqlens.numel()
    G = num_parts(rows_per_kv, h_kv, num_sms)
    tile_md = torch.empty((G, MD_WORDS), dtype=torch.int32, device=cache_seqlens.device)
    num_splits = torch.empty((B + 1,), dtype=torch.int32, device=cache_seqlens.device)
    got = ctypes.c_int(0)
    _check(lib.mla_get_metadata(_ptr(cache_seqlens), B, rows_per_kv, h_kv, int(num_sms or 0), _ptr(tile_md),
                                _ptr(num_splits), ctypes.byref(got), _stream_handle(stream)),
           "mla_get_metadata")
    assert got.value == G
    return tile_md, num_splits


def decode_paged(q: torch.Tensor, k_cache: torch.Tensor, block_table: torch.Tensor, cache_seqlens: torch.Tensor,
                 dv: int, tile_md: torch.Tensor, num_splits: torch.Tensor, causal: bool = False,
                 softmax_scale: float | None = None, workspace: torch.Tensor | None = None,
                 out: torch.Tensor | None = None, lse: torch.Tensor | None = None,
                 status: torch.Tensor | None = None, debug_flags: int = 0, timeout_ns: int = 0, stream=None):
    """MLA decode over the paged cache; returns ``(out [B,s_q,h_q,dv], lse [B,s_q,h_q] fp32)``.

    q and k_cache are both bf16 or both fp16; out has their type."""
    lib = load_library()
    if q.dtype not in DTYPES:
        raise ValueError(f"q must be bf16 or fp16, got {q.dtype}")
    _need(q, "q", q.dtype)
    _need(k_cache, "k_cache", q.dtype)
    _need(block_table, "block_table", torch.int32)
    _need(cache_seqlens, "cache_seqlens", torch.int32)
    _need(tile_md, "tile_md", torch.int32)
    _need(num_splits, "num_splits", torch.int32)
    if q.dim() != 4 or k_cache.dim() != 4 or block_table.dim() != 2:
        raise ValueError("q must be [B, s_q, h_q, d], k_cache [pages, 64, h_kv, d], block_table [B, max_pages]")
    B, s_q, h_q, d = q.shape
    num_pages, page, h_kv, d2 = k_cache.shape
    if page != PAGE_SIZE or d2 != d:
        raise ValueError("k_cache must be [pages, 64, h_kv, d] with the same d as q")
    G = tile_md.shape[0]
    R = s_q * h_q // h_kv
    if softmax_scale is None:
        softmax_scale = d ** -0.5
    if workspace is None:
        workspace = torch.empty((workspace_bytes(B, R, h_kv, G, dv),), dtype=torch.uint8, device=q.device)
    if out is None:
        out = torch.empty((B, s_q, h_q, dv), dtype=q.dtype, device=q.device)
    _need(out, "out", q.dtype)
    if lse is None:
        lse = torch.empty((B, s_q, h_q), dtype=torch.float32, device=q.device)
    code = lib.mla_decode_paged_typed(
        DTYPES[q.dtype], _ptr(q), _ptr(k_cache), num_pages, _ptr(block_table), block_table.shape[1], _ptr(cache_seqlens),
        B, s_q, h_q, h_kv, d, dv, _ptr(tile_md), _ptr(num_splits), G, int(bool(causal)), float(softmax_scale),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(out), _ptr(lse), _ptr(status),
        int(debug_flags), int(timeout_ns), _stream_handle(stream))
    _check(code, "mla_decode_paged")
    return out, lse


def mla_decode(q, k_cache, block_table, cache_seqlens, causal=False, softmax_scale=None, num_sms=None):
    """Metadata + decode in one call (what a decoding step does for one layer)."""
    B, s_q, h_q, _ = q.shape
    h_kv = k_cache.shape[2]
    tile_md, num_splits = get_metadata(cache_seqlens, s_q * h_q // h_kv, h_kv, num_sms)
    return decode_paged(q, k_cache, block_table, cache_seqlens, VALUE_DIM, tile_md, num_splits,
                        causal=causal, softmax_scale=softmax_scale)


def default_scale(d: int = HEAD_DIM) -> float:
    return 1.0 / math.sqrt(d)
