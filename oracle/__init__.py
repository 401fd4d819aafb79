"""fp64 CPU oracle for absorbed-form MLA decode (test infrastructure only).

This package is the correctness reference for the GPU library.  Only the test
suite, the smoke check and the benchmark's CPU-baseline leg may import it; the
product package never does, and it imports nothing from the product package.

The arithmetic lives in ``mla_oracle.c`` (plain C, IEEE double, OpenMP over
independent output rows); this module only builds that file and marshals
arrays.  See the header of ``mla_oracle.c`` for the definition it follows and
the pages it cites.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "mla_oracle.c")
LIBRARY = os.path.join(_HERE, "libmla_oracle.so")

D_QK = 576
D_V = 512
PAGE = 64


def compile_oracle(source: str = SOURCE, output: str = LIBRARY) -> str:
    """Compile the oracle with gcc (no fast-math: IEEE semantics are kept)."""
    cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
           "-o", output, source, "-lm"]
    subprocess.run(cmd, check=True)
    return output


def _needs_build(source: str, output: str) -> bool:
    return (not os.path.exists(output)
            or os.path.getmtime(output) < os.path.getmtime(source))


class Oracle:
    """ctypes front end for one compiled copy of the oracle."""

    def __init__(self, library: str = LIBRARY, source: str = SOURCE):
        if _needs_build(source, library):
            compile_oracle(source, library)
        self.path = library
        self.lib = ctypes.CDLL(library)
        i32p = ctypes.POINTER(ctypes.c_int32)
        i64p = ctypes.POINTER(ctypes.c_int64)
        u16p = ctypes.POINTER(ctypes.c_uint16)
        f64p = ctypes.POINTER(ctypes.c_double)
        common = [u16p, u16p, i32p, i32p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                  ctypes.c_int64, ctypes.c_int, ctypes.c_double]
        for name in ("mla_oracle_direct", "mla_oracle_transposed"):
            fn = getattr(self.lib, name)
            fn.argtypes = common + [i32p, ctypes.c_int, f64p, f64p]
            fn.restype = ctypes.c_int
        self.lib.mla_oracle_online.argtypes = common + [ctypes.c_int, i32p, ctypes.c_int, f64p, f64p]
        self.lib.mla_oracle_online.restype = ctypes.c_int
        self.lib.mla_oracle_split_merge.argtypes = common + [ctypes.c_int, i64p, f64p, f64p]
        self.lib.mla_oracle_split_merge.restype = ctypes.c_int
        self.lib.mla_oracle_e4m3_to_double.argtypes = [ctypes.c_uint8]
        self.lib.mla_oracle_e4m3_to_double.restype = ctypes.c_double
        self.lib.mla_oracle_direct_fp8.argtypes = [u16p, ctypes.POINTER(ctypes.c_uint8), ctypes.POINTER(ctypes.c_float),
                                                   i32p, i32p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                   ctypes.c_int64, ctypes.c_int, ctypes.c_double, f64p, f64p]
        self.lib.mla_oracle_direct_fp8.restype = ctypes.c_int
        self.lib.mla_oracle_merge_states.argtypes = [f64p, f64p, ctypes.c_int, ctypes.c_int64, f64p, f64p]
        self.lib.mla_oracle_merge_states.restype = ctypes.c_int
        self.lib.mla_oracle_naive.argtypes = [u16p, u16p, u16p, u16p, i32p, i32p, ctypes.c_int, ctypes.c_int,
                                               ctypes.c_int, ctypes.c_int64, ctypes.c_int, ctypes.c_double, i32p,
                                               ctypes.c_int, f64p, f64p]
        self.lib.mla_oracle_naive.restype = ctypes.c_int
        self.lib.mla_oracle_threads.argtypes = []
        self.lib.mla_oracle_threads.restype = ctypes.c_int

    # -- marshalling -------------------------------------------------------
    @staticmethod
    def _bits(t) -> np.ndarray:
        """bf16 torch tensor (or uint16 array) -> contiguous uint16 bit array."""
        if isinstance(t, np.ndarray):
            assert t.dtype == np.uint16
            return np.ascontiguousarray(t)
        import torch
        assert t.dtype == torch.bfloat16, t.dtype
        return np.ascontiguousarray(t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))

    @staticmethod
    def _i32(t) -> np.ndarray:
        if isinstance(t, np.ndarray):
            return np.ascontiguousarray(t, dtype=np.int32)
        return np.ascontiguousarray(t.detach().cpu().numpy().astype(np.int32))

    def _common(self, q, kv_cache, block_table, cache_seqlens, scale):
        qb, kb = self._bits(q), self._bits(kv_cache)
        bt, sl = self._i32(block_table), self._i32(cache_seqlens)
        B, s_q, H, dq = qb.shape
        assert dq == D_QK and kb.shape[1:] == (PAGE, D_QK)
        assert bt.ndim == 2 and bt.shape[0] == B and sl.shape == (B,)
        keep = (qb, kb, bt, sl)
        args = [qb.ctypes.data_as(ctypes.POINTER(ctypes.c_uint16)),
                kb.ctypes.data_as(ctypes.POINTER(ctypes.c_uint16)),
                bt.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
                sl.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
                B, s_q, H, kb.shape[0], bt.shape[1], float(scale)]
        return keep, args, (B, s_q, H)

    @staticmethod
    def _outputs(B, s_q, H):
        out = np.full((B, s_q, H, D_V), np.nan, dtype=np.float64)
        lse = np.full((B, s_q, H), np.nan, dtype=np.float64)
        return out, lse

    @staticmethod
    def _seq_list(seqs: Optional[Sequence[int]]):
        if seqs is None:
            return None, ctypes.POINTER(ctypes.c_int32)(), 0
        arr = np.ascontiguousarray(np.asarray(seqs, dtype=np.int32))
        return arr, arr.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), len(arr)

    @staticmethod
    def _check(rc: int, name: str):
        if rc != 0:
            raise ValueError(f"{name} failed with code {rc} "
                             "(-1 bad argument, -2 block table entry outside the cache, -3 out of memory)")

    # -- the four forms ----------------------------------------------------
    def direct(self, q, kv_cache, block_table, cache_seqlens, scale, seqs=None):
        """out[B,s_q,H,512] and lse[B,s_q,H] in float64; rows of sequences not
        in ``seqs`` (when given) are left as NaN."""
        keep, args, (B, s_q, H) = self._common(q, kv_cache, block_table, cache_seqlens, scale)
        out, lse = self._outputs(B, s_q, H)
        arr, ptr, n = self._seq_list(seqs)
        rc = self.lib.mla_oracle_direct(*args, ptr, n, _f64(out), _f64(lse))
        self._check(rc, "mla_oracle_direct")
        return out, lse

    def transposed(self, q, kv_cache, block_table, cache_seqlens, scale, seqs=None):
        keep, args, (B, s_q, H) = self._common(q, kv_cache, block_table, cache_seqlens, scale)
        out, lse = self._outputs(B, s_q, H)
        arr, ptr, n = self._seq_list(seqs)
        rc = self.lib.mla_oracle_transposed(*args, ptr, n, _f64(out), _f64(lse))
        self._check(rc, "mla_oracle_transposed")
        return out, lse

    def online(self, q, kv_cache, block_table, cache_seqlens, scale, tile, seqs=None):
        keep, args, (B, s_q, H) = self._common(q, kv_cache, block_table, cache_seqlens, scale)
        out, lse = self._outputs(B, s_q, H)
        arr, ptr, n = self._seq_list(seqs)
        rc = self.lib.mla_oracle_online(*args, int(tile), ptr, n, _f64(out), _f64(lse))
        self._check(rc, "mla_oracle_online")
        return out, lse

    def split_merge(self, q, kv_cache, block_table, cache_seqlens, scale, bounds):
        """``bounds``: int array [B, n_splits + 1] of token boundaries."""
        keep, args, (B, s_q, H) = self._common(q, kv_cache, block_table, cache_seqlens, scale)
        bd = np.ascontiguousarray(np.asarray(bounds, dtype=np.int64))
        assert bd.ndim == 2 and bd.shape[0] == B
        out, lse = self._outputs(B, s_q, H)
        rc = self.lib.mla_oracle_split_merge(*args, bd.shape[1] - 1,
                                             bd.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
                                             _f64(out), _f64(lse))
        self._check(rc, "mla_oracle_split_merge")
        return out, lse

    def merge_states(self, out_parts, lse_parts):
        """Merge W partial states: ``out_parts`` [W, ..., 512], ``lse_parts``
        [W, ...] (any float dtype, widened exactly to fp64).  Returns fp64
        (out [..., 512], lse [...])."""
        o = np.ascontiguousarray(_as_f64(out_parts))
        l = np.ascontiguousarray(_as_f64(lse_parts))
        W = o.shape[0]
        assert o.shape[-1] == 512 and l.shape == o.shape[:-1] and W >= 1
        rows = int(np.prod(l.shape[1:], dtype=np.int64))
        out = np.zeros(l.shape[1:] + (512,), dtype=np.float64)
        lse = np.zeros(l.shape[1:], dtype=np.float64)
        rc = self.lib.mla_oracle_merge_states(_f64(o), _f64(l), W, rows, _f64(out), _f64(lse))
        self._check(rc, "mla_oracle_merge_states")
        return out, lse

    def e4m3(self, codes) -> np.ndarray:
        """Values of e4m3 codes (any integer array), in fp64."""
        c = np.asarray(codes, dtype=np.uint8)
        return np.array([self.lib.mla_oracle_e4m3_to_double(int(x)) for x in c.ravel()]).reshape(c.shape)

    def direct_fp8(self, q, kv_codes, kv_scale, block_table, cache_seqlens, scale):
        """The definition over an e4m3 cache: ``kv_codes`` uint8 [num_blocks, 64,
        576], ``kv_scale`` fp32 [num_blocks, 64] (one scale per cached token)."""
        qb = self._bits(q)
        B, s_q, H, _ = qb.shape
        codes = np.ascontiguousarray(np.asarray(kv_codes.cpu() if hasattr(kv_codes, "cpu") else kv_codes,
                                                dtype=np.uint8))
        ks = np.ascontiguousarray(np.asarray(kv_scale.cpu() if hasattr(kv_scale, "cpu") else kv_scale,
                                             dtype=np.float32))
        assert codes.ndim == 3 and codes.shape[1:] == (64, 576) and ks.shape == codes.shape[:2]
        bt = self._i32(block_table)
        sl = self._i32(cache_seqlens)
        out, lse = self._outputs(B, s_q, H)
        rc = self.lib.mla_oracle_direct_fp8(
            qb.ctypes.data_as(ctypes.POINTER(ctypes.c_uint16)), codes.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8)),
            ks.ctypes.data_as(ctypes.POINTER(ctypes.c_float)), bt.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
            sl.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), B, s_q, H, codes.shape[0], bt.shape[1],
            float(scale), _f64(out), _f64(lse))
        self._check(rc, "mla_oracle_direct_fp8")
        return out, lse

    def naive(self, q, kv_cache, w_uk, w_uv, block_table, cache_seqlens, scale, seqs=None):
        """The non-absorbed form: ``q`` bf16 [B, s_q, H, 192] (128 key columns,
        then 64 rope), ``w_uk`` / ``w_uv`` bf16 [H, 128, 512].  Returns fp64 out
        [B, s_q, H, 128] and lse [B, s_q, H]; rows of sequences not in ``seqs``
        (when given) are left as NaN."""
        qb = self._bits(q)
        B, s_q, H, dq = qb.shape
        assert dq == 192
        kv = self._bits(kv_cache)
        wk = self._bits(w_uk)
        wv = self._bits(w_uv)
        assert wk.shape == (H, 128, 512) and wv.shape == (H, 128, 512)
        assert kv.ndim == 3 and kv.shape[1:] == (64, 576)
        bt = self._i32(block_table)
        sl = self._i32(cache_seqlens)
        out = np.full((B, s_q, H, 128), np.nan)
        lse = np.full((B, s_q, H), np.nan)
        arr, ptr, n = self._seq_list(seqs)
        u16 = ctypes.POINTER(ctypes.c_uint16)
        rc = self.lib.mla_oracle_naive(
            qb.ctypes.data_as(u16), kv.ctypes.data_as(u16), wk.ctypes.data_as(u16), wv.ctypes.data_as(u16),
            bt.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), sl.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
            B, s_q, H, kv.shape[0], bt.shape[1], float(scale), ptr, n, _f64(out), _f64(lse))
        self._check(rc, "mla_oracle_naive")
        return out, lse

    def threads(self) -> int:
        return int(self.lib.mla_oracle_threads())


def _as_f64(t) -> np.ndarray:
    if hasattr(t, "detach"):  # a torch tensor (bf16 has no numpy dtype: widen through fp32, exactly)
        t = t.detach().to("cpu").float().numpy()
    return np.asarray(t, dtype=np.float64)


def _f64(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


_default: Optional[Oracle] = None


def default() -> Oracle:
    """The oracle built from this directory's source (compiled on first use)."""
    global _default
    if _default is None:
        _default = Oracle()
    return _default
