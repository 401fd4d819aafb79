"""Absorbed-form MLA decode on B200 (sm_100a): Python binding of the C ABI.

This module only marshals arguments: it checks dtypes, shapes and devices,
allocates outputs and scratch with torch when the caller does not pass them,
and calls the entry points of ``libmla_decode_b200.so`` (declared in
``include/mla_decode.h``) with raw device pointers and the current CUDA
stream.  Every step of the computation runs in that library's kernels; there
is no fallback path.  If the library is missing, importing works but every
call raises ``MLAError`` with the command that builds it.

    sched, splits = decode_metadata(cache_seqlens, s_q, H)   # once per step
    out, lse = decode(q, kv_cache, block_table, cache_seqlens, scale,
                      sched_meta=sched, num_splits=splits)     # per layer
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIBRARY = os.path.join(_HERE, "libmla_decode_b200.so")

D_QK = 576
D_V = 512
PAGE = 64

MLA_OK = 0
STATUS_NAMES = {
    0: "MLA_OK", 1: "MLA_ERR_INVALID_ARG", 2: "MLA_ERR_MISALIGNED",
    3: "MLA_ERR_UNSUPPORTED_SHAPE", 4: "MLA_ERR_WORKSPACE_TOO_SMALL",
    5: "MLA_ERR_CUDA", 6: "MLA_ERR_DEVICE_CHECK",
}
DEVERR_BLOCK_TABLE = 1
DEVERR_SEQLEN = 2
DEVERR_SCHEDULE = 4
DEVERR_TIMEOUT = 8

EXPORTED = (
    "mla_sched_meta_ints", "mla_decode_workspace_size", "mla_decode_metadata",
    "mla_decode", "mla_decode_attention", "mla_decode_combine", "mla_decode_static_workspace",
    "mla_merge_states", "mla_decode_fp8", "mla_decode_attention_fp8", "mla_get_device_error",
    "mla_status_string", "mla_last_error_message", "mla_debug_stall_cta",
    "mla_decode_naive", "mla_decode_naive_workspace_size",
)


class MLAError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str = ""):
        self.status = status
        name = STATUS_NAMES.get(status, f"status {status}")
        super().__init__(f"{where}: {name}" + (f" ({detail})" if detail else ""))


_lib: Optional[ctypes.CDLL] = None


def library_path() -> str:
    return LIBRARY


def load_library(path: str = LIBRARY) -> ctypes.CDLL:
    """Load the shared library and declare the C signatures (no GPU needed)."""
    global _lib
    if _lib is not None and path == LIBRARY:
        return _lib
    if not os.path.exists(path):
        raise MLAError(5, "load_library",
                       f"{path} is missing; build it with `python -m decode_attention_latent_b200.build`")
    lib = ctypes.CDLL(path)
    i32p, vp, sz = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t
    ci, cu16p = ctypes.c_int, ctypes.c_void_p
    lib.mla_sched_meta_ints.argtypes = [ci]
    lib.mla_sched_meta_ints.restype = sz
    lib.mla_decode_workspace_size.argtypes = [ci, ci, ci, ci]
    lib.mla_decode_workspace_size.restype = sz
    lib.mla_decode_metadata.argtypes = [i32p, ci, ci, ci, ci, i32p, i32p, vp]
    lib.mla_decode_metadata.restype = ci
    lib.mla_decode.argtypes = [cu16p, cu16p, i32p, i32p, ci, ci, ci, ctypes.c_int64, ci,
                               ctypes.c_float, ci, i32p, i32p, vp, sz, cu16p, vp, vp]
    lib.mla_decode.restype = ci
    lib.mla_decode_attention.argtypes = lib.mla_decode.argtypes
    lib.mla_decode_attention.restype = ci
    lib.mla_decode_static_workspace.argtypes = [cu16p, cu16p, i32p, i32p, ci, ci, ci, ctypes.c_int64, ci,
                                                ctypes.c_float, ci, i32p, i32p, cu16p, vp, vp]
    lib.mla_decode_static_workspace.restype = ci
    lib.mla_decode_combine.argtypes = [i32p, i32p, vp, sz, ci, ci, ci, ci, cu16p, vp, vp]
    lib.mla_decode_combine.restype = ci
    lib.mla_decode_fp8.argtypes = [cu16p, vp, vp, i32p, i32p, ci, ci, ci, ctypes.c_int64, ci,
                                   ctypes.c_float, ci, i32p, i32p, vp, sz, cu16p, vp, vp]
    lib.mla_decode_fp8.restype = ci
    lib.mla_decode_attention_fp8.argtypes = lib.mla_decode_fp8.argtypes
    lib.mla_decode_attention_fp8.restype = ci
    lib.mla_merge_states.argtypes = [cu16p, vp, ci, ctypes.c_int64, cu16p, vp, vp]
    lib.mla_merge_states.restype = ci
    lib.mla_get_device_error.argtypes = [i32p, ctypes.POINTER(ctypes.c_int32), vp]
    lib.mla_get_device_error.restype = ci
    lib.mla_status_string.argtypes = [ci]
    lib.mla_status_string.restype = ctypes.c_char_p
    lib.mla_last_error_message.argtypes = []
    lib.mla_last_error_message.restype = ctypes.c_char_p
    lib.mla_debug_stall_cta.argtypes = [ci]
    lib.mla_debug_stall_cta.restype = None
    lib.mla_decode_naive_workspace_size.argtypes = [ci, ci, ci, ci, ci]
    lib.mla_decode_naive_workspace_size.restype = sz
    lib.mla_decode_naive.argtypes = [cu16p, cu16p, cu16p, cu16p, i32p, i32p, ci, ci, ci, ctypes.c_int64, ci,
                                     ctypes.c_float, ci, vp, sz, i32p, cu16p, vp, vp]
    lib.mla_decode_naive.restype = ci
    if path == LIBRARY:
        _lib = lib
    return lib


def _check(rc: int, where: str):
    if rc != MLA_OK:
        detail = load_library().mla_last_error_message().decode(errors="replace")
        raise MLAError(rc, where, detail)


def _stream_handle(stream: Optional[torch.cuda.Stream], device: torch.device) -> ctypes.c_void_p:
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return ctypes.c_void_p(s.cuda_stream)


def _require(t: torch.Tensor, name: str, dtype: torch.dtype, device: torch.device, shape=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.device != device:
        raise ValueError(f"{name} must be on {device}, got {t.device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def num_sms(device: Optional[torch.device] = None) -> int:
    """Streaming-multiprocessor count of the device (148 on B200)."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    return torch.cuda.get_device_properties(dev).multi_processor_count


def sched_meta_ints(n_sms: int) -> int:
    return int(load_library().mla_sched_meta_ints(int(n_sms)))


def workspace_size(B: int, s_q: int, H: int, n_sms: int) -> int:
    n = int(load_library().mla_decode_workspace_size(int(B), int(s_q), int(H), int(n_sms)))
    if n == 0:
        raise MLAError(3, "workspace_size", f"B={B} s_q={s_q} H={H} num_sms={n_sms}")
    return n


def decode_metadata(cache_seqlens: torch.Tensor, s_q: int, H: int, num_sms_: Optional[int] = None,
                    sched_meta: Optional[torch.Tensor] = None, num_splits: Optional[torch.Tensor] = None,
                    stream: Optional[torch.cuda.Stream] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Split-KV schedule for one decode step (``mla_decode_metadata``)."""
    dev = cache_seqlens.device
    B = cache_seqlens.shape[0]
    _require(cache_seqlens, "cache_seqlens", torch.int32, dev, (B,))
    n = num_sms(dev) if num_sms_ is None else int(num_sms_)
    lib = load_library()
    if sched_meta is None:
        sched_meta = torch.empty(sched_meta_ints(n), dtype=torch.int32, device=dev)
    if num_splits is None:
        num_splits = torch.empty(B + 1, dtype=torch.int32, device=dev)
    _require(sched_meta, "sched_meta", torch.int32, dev, (sched_meta_ints(n),))
    _require(num_splits, "num_splits", torch.int32, dev, (B + 1,))
    rc = lib.mla_decode_metadata(ctypes.c_void_p(cache_seqlens.data_ptr()), B, int(s_q), int(H), n,
                                 ctypes.c_void_p(sched_meta.data_ptr()), ctypes.c_void_p(num_splits.data_ptr()),
                                 _stream_handle(stream, dev))
    _check(rc, "mla_decode_metadata")
    return sched_meta, num_splits


def decode(q: torch.Tensor, kv_cache: torch.Tensor, block_table: torch.Tensor, cache_seqlens: torch.Tensor,
           softmax_scale: float, *, sched_meta: Optional[torch.Tensor] = None,
           num_splits: Optional[torch.Tensor] = None, num_sms_: Optional[int] = None,
           workspace: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
           lse: Optional[torch.Tensor] = None, stream: Optional[torch.cuda.Stream] = None,
           combine: bool = True) -> Tuple[torch.Tensor, torch.Tensor]:
    """Absorbed-form MLA decode (``mla_decode``: the attention kernel, then the
    combine kernel): returns (out bf16 [B,s_q,H,512], lse fp32 [B,s_q,H]).
    Builds the schedule with ``decode_metadata`` when ``sched_meta`` is None.
    With ``combine=False`` only the attention kernel runs
    (``mla_decode_attention``), leaving split sequences as pieces in
    ``workspace``; the caller then runs ``decode_combine``."""
    dev = q.device
    if dev.type != "cuda":
        raise ValueError("q must be a CUDA tensor")
    if q.dim() != 4 or q.shape[-1] != D_QK:
        raise ValueError(f"q must be [B, s_q, H, {D_QK}]")
    B, s_q, H, _ = q.shape
    _require(q, "q", torch.bfloat16, dev)
    if kv_cache.dim() != 3 or tuple(kv_cache.shape[1:]) != (PAGE, D_QK):
        raise ValueError(f"kv_cache must be [num_blocks, {PAGE}, {D_QK}]")
    _require(kv_cache, "kv_cache", torch.bfloat16, dev)
    if block_table.dim() != 2 or block_table.shape[0] != B:
        raise ValueError("block_table must be [B, max_blocks]")
    _require(block_table, "block_table", torch.int32, dev)
    _require(cache_seqlens, "cache_seqlens", torch.int32, dev, (B,))
    n = num_sms(dev) if num_sms_ is None else int(num_sms_)
    if sched_meta is None or num_splits is None:
        sched_meta, num_splits = decode_metadata(cache_seqlens, s_q, H, n, stream=stream)
    ws_bytes = workspace_size(B, s_q, H, n)
    if workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    _require(workspace, "workspace", torch.uint8, dev)
    if out is None:
        out = torch.empty(B, s_q, H, D_V, dtype=torch.bfloat16, device=dev)
    if lse is None:
        lse = torch.empty(B, s_q, H, dtype=torch.float32, device=dev)
    _require(out, "out", torch.bfloat16, dev, (B, s_q, H, D_V))
    _require(lse, "lse", torch.float32, dev, (B, s_q, H))
    lib = load_library()
    fn = lib.mla_decode if combine else lib.mla_decode_attention
    rc = fn(
        ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(kv_cache.data_ptr()),
        ctypes.c_void_p(block_table.data_ptr()), ctypes.c_void_p(cache_seqlens.data_ptr()),
        B, s_q, H, kv_cache.shape[0], block_table.shape[1], float(softmax_scale), n,
        ctypes.c_void_p(sched_meta.data_ptr()), ctypes.c_void_p(num_splits.data_ptr()),
        ctypes.c_void_p(workspace.data_ptr()), workspace.numel(),
        ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(lse.data_ptr()), _stream_handle(stream, dev))
    _check(rc, "mla_decode" if combine else "mla_decode_attention")
    return out, lse


def decode_combine(num_splits: torch.Tensor, sched_meta: torch.Tensor, workspace: torch.Tensor, B: int,
                   s_q: int, H: int, out: torch.Tensor, lse: torch.Tensor, num_sms_: Optional[int] = None,
                   stream: Optional[torch.cuda.Stream] = None):
    """The combine kernel alone (``mla_decode_combine``)."""
    dev = out.device
    n = num_sms(dev) if num_sms_ is None else int(num_sms_)
    rc = load_library().mla_decode_combine(
        ctypes.c_void_p(num_splits.data_ptr()), ctypes.c_void_p(sched_meta.data_ptr()),
        ctypes.c_void_p(workspace.data_ptr()), workspace.numel(), int(B), int(s_q), int(H), n,
        ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(lse.data_ptr()), _stream_handle(stream, dev))
    _check(rc, "mla_decode_combine")


def decode_fp8(q: torch.Tensor, kv_codes: torch.Tensor, kv_scale: torch.Tensor, block_table: torch.Tensor,
               cache_seqlens: torch.Tensor, softmax_scale: float, *, sched_meta: Optional[torch.Tensor] = None,
               num_splits: Optional[torch.Tensor] = None, num_sms_: Optional[int] = None,
               workspace: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
               lse: Optional[torch.Tensor] = None, stream: Optional[torch.cuda.Stream] = None,
               combine: bool = True) -> Tuple[torch.Tensor, torch.Tensor]:
    """MLA decode over an FP8 cache (``mla_decode_fp8``): ``kv_codes`` uint8
    [num_blocks, 64, 576] e4m3 codes, ``kv_scale`` fp32 [num_blocks, 64], one
    scale per cached token.  16 or 32 query columns: H = 16 with s_q = 1 or
    2, or H = 32 with s_q = 1."""
    dev = q.device
    if dev.type != "cuda":
        raise ValueError("q must be a CUDA tensor")
    if q.dim() != 4 or q.shape[-1] != D_QK:
        raise ValueError(f"q must be [B, s_q, H, {D_QK}]")
    B, s_q, H, _ = q.shape
    _require(q, "q", torch.bfloat16, dev)
    if kv_codes.dim() != 3 or tuple(kv_codes.shape[1:]) != (PAGE, D_QK):
        raise ValueError(f"kv_codes must be [num_blocks, {PAGE}, {D_QK}]")
    _require(kv_codes, "kv_codes", torch.uint8, dev)
    _require(kv_scale, "kv_scale", torch.float32, dev, (kv_codes.shape[0], PAGE))
    if block_table.dim() != 2 or block_table.shape[0] != B:
        raise ValueError("block_table must be [B, max_blocks]")
    _require(block_table, "block_table", torch.int32, dev)
    _require(cache_seqlens, "cache_seqlens", torch.int32, dev, (B,))
    n = num_sms(dev) if num_sms_ is None else int(num_sms_)
    if sched_meta is None or num_splits is None:
        sched_meta, num_splits = decode_metadata(cache_seqlens, s_q, H, n, stream=stream)
    ws_bytes = workspace_size(B, s_q, H, n)
    if workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    if out is None:
        out = torch.empty(B, s_q, H, D_V, dtype=torch.bfloat16, device=dev)
    if lse is None:
        lse = torch.empty(B, s_q, H, dtype=torch.float32, device=dev)
    _require(out, "out", torch.bfloat16, dev, (B, s_q, H, D_V))
    _require(lse, "lse", torch.float32, dev, (B, s_q, H))
    lib = load_library()
    fn = lib.mla_decode_fp8 if combine else lib.mla_decode_attention_fp8
    rc = fn(
        ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(kv_codes.data_ptr()), ctypes.c_void_p(kv_scale.data_ptr()),
        ctypes.c_void_p(block_table.data_ptr()), ctypes.c_void_p(cache_seqlens.data_ptr()),
        B, s_q, H, kv_codes.shape[0], block_table.shape[1], float(softmax_scale), n,
        ctypes.c_void_p(sched_meta.data_ptr()), ctypes.c_void_p(num_splits.data_ptr()),
        ctypes.c_void_p(workspace.data_ptr()), workspace.numel(),
        ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(lse.data_ptr()), _stream_handle(stream, dev))
    _check(rc, "mla_decode_fp8" if combine else "mla_decode_attention_fp8")
    return out, lse


D_NAIVE = 128  # decompressed key / value width of the non-absorbed form


def decode_naive(q: torch.Tensor, kv_cache: torch.Tensor, w_uk: torch.Tensor, w_uv: torch.Tensor,
                 block_table: torch.Tensor, cache_seqlens: torch.Tensor, softmax_scale: float, *,
                 num_sms_: Optional[int] = None, workspace: Optional[torch.Tensor] = None,
                 error_word: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
                 lse: Optional[torch.Tensor] = None,
                 stream: Optional[torch.cuda.Stream] = None) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """Non-absorbed form (``mla_decode_naive``): ``q`` bf16 [B, s_q, H, 192]
    (128 key columns, then 64 rope), the latent cache of ``decode``, ``w_uk``
    / ``w_uv`` bf16 [H, 128, 512].  Returns (out bf16 [B, s_q, H, 128], lse
    fp32 [B, s_q, H], the device error word int32 [1])."""
    dev = q.device
    if dev.type != "cuda":
        raise ValueError("q must be a CUDA tensor")
    if q.dim() != 4 or q.shape[-1] != D_NAIVE + D_QK - D_V:
        raise ValueError("q must be [B, s_q, H, 192]")
    B, s_q, H, _ = q.shape
    _require(q, "q", torch.bfloat16, dev)
    if kv_cache.dim() != 3 or tuple(kv_cache.shape[1:]) != (PAGE, D_QK):
        raise ValueError(f"kv_cache must be [num_blocks, {PAGE}, {D_QK}]")
    _require(kv_cache, "kv_cache", torch.bfloat16, dev)
    _require(w_uk, "w_uk", torch.bfloat16, dev, (H, D_NAIVE, D_V))
    _require(w_uv, "w_uv", torch.bfloat16, dev, (H, D_NAIVE, D_V))
    if block_table.dim() != 2 or block_table.shape[0] != B:
        raise ValueError("block_table must be [B, max_blocks]")
    _require(block_table, "block_table", torch.int32, dev)
    _require(cache_seqlens, "cache_seqlens", torch.int32, dev, (B,))
    n = num_sms(dev) if num_sms_ is None else int(num_sms_)
    lib = load_library()
    ws_bytes = int(lib.mla_decode_naive_workspace_size(B, s_q, H, block_table.shape[1], n))
    if ws_bytes == 0:
        raise MLAError(3, "mla_decode_naive_workspace_size", f"B={B} s_q={s_q} H={H}")
    if workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    if error_word is None:
        error_word = torch.zeros(1, dtype=torch.int32, device=dev)
    if out is None:
        out = torch.empty(B, s_q, H, D_NAIVE, dtype=torch.bfloat16, device=dev)
    if lse is None:
        lse = torch.empty(B, s_q, H, dtype=torch.float32, device=dev)
    _require(workspace, "workspace", torch.uint8, dev)
    _require(error_word, "error_word", torch.int32, dev, (1,))
    _require(out, "out", torch.bfloat16, dev, (B, s_q, H, D_NAIVE))
    _require(lse, "lse", torch.float32, dev, (B, s_q, H))
    rc = lib.mla_decode_naive(
        ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(kv_cache.data_ptr()), ctypes.c_void_p(w_uk.data_ptr()),
        ctypes.c_void_p(w_uv.data_ptr()), ctypes.c_void_p(block_table.data_ptr()),
        ctypes.c_void_p(cache_seqlens.data_ptr()), B, s_q, H, kv_cache.shape[0], block_table.shape[1],
        float(softmax_scale), n, ctypes.c_void_p(workspace.data_ptr()), workspace.numel(),
        ctypes.c_void_p(error_word.data_ptr()), ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(lse.data_ptr()),
        _stream_handle(stream, dev))
    _check(rc, "mla_decode_naive")
    return out, lse, error_word


def merge_states(out_parts: torch.Tensor, lse_parts: torch.Tensor, *, out: Optional[torch.Tensor] = None,
                 lse: Optional[torch.Tensor] = None,
                 stream: Optional[torch.cuda.Stream] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Merge W partial states (``mla_merge_states``): ``out_parts`` bf16
    [W, ..., 512] and ``lse_parts`` fp32 [W, ...] -> (out bf16 [..., 512],
    lse fp32 [...])."""
    dev = out_parts.device
    if dev.type != "cuda":
        raise ValueError("out_parts must be a CUDA tensor")
    if out_parts.dim() < 2 or out_parts.shape[-1] != D_V:
        raise ValueError(f"out_parts must be [W, ..., {D_V}]")
    W = out_parts.shape[0]
    row_shape = tuple(out_parts.shape[1:-1])
    _require(out_parts, "out_parts", torch.bfloat16, dev)
    _require(lse_parts, "lse_parts", torch.float32, dev, (W,) + row_shape)
    if out is None:
        out = torch.empty(row_shape + (D_V,), dtype=torch.bfloat16, device=dev)
    if lse is None:
        lse = torch.empty(row_shape, dtype=torch.float32, device=dev)
    _require(out, "out", torch.bfloat16, dev, row_shape + (D_V,))
    _require(lse, "lse", torch.float32, dev, row_shape)
    rows = lse.numel()
    rc = load_library().mla_merge_states(
        ctypes.c_void_p(out_parts.data_ptr()), ctypes.c_void_p(lse_parts.data_ptr()), int(W), int(rows),
        ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(lse.data_ptr()), _stream_handle(stream, dev))
    _check(rc, "mla_merge_states")
    return out, lse


def debug_stall_cta(cta: int) -> None:
    """Test hook (``mla_debug_stall_cta``): CTA ``cta`` of the next decode
    launches never loads its first chunk, so its bounded waits run out; -1
    turns it off."""
    load_library().mla_debug_stall_cta(int(cta))


def get_device_error(sched_meta: torch.Tensor, stream: Optional[torch.cuda.Stream] = None) -> int:
    """Synchronise the stream and return the device error word (0 = clean)."""
    code = ctypes.c_int32(0)
    rc = load_library().mla_get_device_error(ctypes.c_void_p(sched_meta.data_ptr()), ctypes.byref(code),
                                             _stream_handle(stream, sched_meta.device))
    if rc not in (MLA_OK, 6):
        _check(rc, "mla_get_device_error")
    return int(code.value)


def status_string(status: int) -> str:
    return load_library().mla_status_string(int(status)).decode()
