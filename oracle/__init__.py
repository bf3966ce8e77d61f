"""Double-precision CPU oracle for the paged KV-cache hot path.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import this package; the product package
``paged_kv_cache_409_b200`` never does, and this package never imports the
product.  The arithmetic lives in ``pagedkv_oracle.c`` (plain C, double);
this module only builds it with gcc and marshals arrays into it.

What each function follows is stated in the C file's header: the block /
block-table data model and block-wise attention of the vLLM case-study page
("vLLM 与 PagedAttention", section 二), copy-on-write and chunked prefill of the
vLLM guide page ("指南").  The attention formula itself is not printed on the
pages; the oracle evaluates plain scaled dot-product attention.

Arrays are numpy; bf16 storage travels as its uint16 bit pattern.  Use
:func:`storage` to turn a CPU torch tensor into such an array.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "pagedkv_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")

F32, F16, BF16, E4M3 = 0, 1, 2, 3


def compile_source(src: str, out: str) -> str:
    """gcc -O2 one C source of the oracle into a shared library at ``out``."""
    tmp = out + f".tmp{os.getpid()}"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-o", tmp, src, "-lm"])
    os.replace(tmp, out)
    return out


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/liboracle.so`` (if stale)."""
    stale = (not os.path.exists(_LIB_PATH)) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(SOURCE)
    if force or stale:
        compile_source(SOURCE, _LIB_PATH)
    return _LIB_PATH


def storage(t) -> tuple:
    """(numpy storage array, dtype code) of a CPU torch tensor (uint8 = E4M3 codes)."""
    import torch
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.float32:
        return t.numpy(), F32
    if t.dtype == torch.float16:
        return t.numpy(), F16
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16), BF16
    if t.dtype in (torch.uint8, torch.float8_e4m3fn):   # pools of E4M3 codes
        return t.view(torch.uint8).numpy(), E4M3
    raise TypeError(f"unsupported oracle dtype {t.dtype}")


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _check(rc: int, what: str):
    if rc != 0:
        raise ValueError(f"oracle {what}: invalid argument or table entry")


class Oracle:
    """The oracle's C functions from one compiled library."""

    def __init__(self, path: str):
        lib = ctypes.CDLL(path)
        P, I, L, D = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_double
        lib.oracle_num_threads.argtypes = [I]
        lib.oracle_num_threads.restype = I
        lib.oracle_to_double.argtypes = [P, P, L, I]
        lib.oracle_blocks_needed.argtypes = [L, I]
        lib.oracle_blocks_needed.restype = L
        lib.oracle_slot_for_position.argtypes = [P, L, I]
        lib.oracle_slot_for_position.restype = L
        lib.oracle_reshape_and_cache.argtypes = [P, P, P, P, P, L, I, I, I, L, I]
        lib.oracle_copy_blocks.argtypes = [P, P, I, P, L, L, L]
        lib.oracle_paged_attention_decode.argtypes = [P, P, P, P, I, P, P, D, L, I, I, I, I, I, L]
        lib.oracle_paged_attention_prefill_chunk.argtypes = [P, P, P, P, I, P, P, P, I, D, I, I, I, I, I, L, P]
        lib.oracle_e4m3_encode.argtypes = [P, P, L]
        lib.oracle_reshape_and_cache_fp8.argtypes = [P, P, P, P, P, L, I, I, I, L, I, D, D]
        lib.oracle_paged_attention_decode_kv.argtypes = [P, P, I, P, P, I, D, D, P, P, D, L, I, I, I, I, I, L]
        lib.oracle_paged_attention_prefill_chunk_kv.argtypes = [P, P, I, P, P, I, D, D, P, P, P, I, D, I, I, I, I,
                                                                I, L, P]
        for f in (lib.oracle_to_double, lib.oracle_reshape_and_cache, lib.oracle_copy_blocks,
                  lib.oracle_paged_attention_decode, lib.oracle_paged_attention_prefill_chunk,
                  lib.oracle_e4m3_encode, lib.oracle_reshape_and_cache_fp8, lib.oracle_paged_attention_decode_kv,
                  lib.oracle_paged_attention_prefill_chunk_kv):
            f.restype = ctypes.c_int
        self.lib = lib
        self.path = path

    def num_threads(self, n: int = 0) -> int:
        """Host threads the attention functions use (n > 0 sets it); 1 without OpenMP."""
        return int(self.lib.oracle_num_threads(int(n)))

    def to_double(self, a: np.ndarray, dtype: int) -> np.ndarray:
        a = np.ascontiguousarray(a)
        out = np.empty(a.shape, dtype=np.float64)
        _check(self.lib.oracle_to_double(_ptr(out), _ptr(a), a.size, dtype), "to_double")
        return out

    def blocks_needed(self, num_tokens: int, block_size: int) -> int:
        return int(self.lib.oracle_blocks_needed(int(num_tokens), block_size))

    def slot_for_position(self, block_table_row, pos: int, block_size: int) -> int:
        row = np.ascontiguousarray(block_table_row, dtype=np.int32)
        return int(self.lib.oracle_slot_for_position(_ptr(row), int(pos), block_size))

    def reshape_and_cache(self, key, value, key_cache, value_cache, slot_mapping, dtype):
        """In place on the numpy pools ``[NB, B, Hkv, D]``."""
        T, Hkv, D = key.shape
        NB, B = key_cache.shape[:2]
        sm = np.ascontiguousarray(slot_mapping, dtype=np.int64)
        rc = self.lib.oracle_reshape_and_cache(_ptr(np.ascontiguousarray(key)), _ptr(np.ascontiguousarray(value)),
                                               _ptr(key_cache), _ptr(value_cache), _ptr(sm), T, Hkv, D, B, NB,
                                               dtype)
        _check(rc, "reshape_and_cache")

    def copy_blocks(self, key_caches, value_caches, src_dst_pairs):
        """In place on every numpy pool of the two lists."""
        L = len(key_caches)
        NB = key_caches[0].shape[0]
        kp = (ctypes.c_void_p * L)(*[c.ctypes.data for c in key_caches])
        vp = (ctypes.c_void_p * L)(*[c.ctypes.data for c in value_caches])
        pairs = np.ascontiguousarray(src_dst_pairs, dtype=np.int64).reshape(-1, 2)
        block_bytes = key_caches[0].nbytes // NB
        rc = self.lib.oracle_copy_blocks(kp, vp, L, _ptr(pairs), pairs.shape[0], block_bytes, NB)
        _check(rc, "copy_blocks")

    def paged_attention_decode(self, query, key_cache, value_cache, block_tables, context_lens, scale, dtype):
        """float64 ``[S, Hq, D]``."""
        S, Hq, D = query.shape
        NB, B, Hkv, D2 = key_cache.shape
        assert D2 == D
        bt = np.ascontiguousarray(block_tables, dtype=np.int32).reshape(S, -1)
        cl = np.ascontiguousarray(context_lens, dtype=np.int32)
        out = np.zeros((S, Hq, D), dtype=np.float64)
        rc = self.lib.oracle_paged_attention_decode(
            _ptr(out), _ptr(np.ascontiguousarray(query)), _ptr(key_cache), _ptr(value_cache), dtype, _ptr(bt),
            _ptr(cl), float(scale), S, Hq, Hkv, D, B, bt.shape[1], NB)
        _check(rc, "paged_attention_decode")
        return out

    def paged_attention_prefill_chunk(self, query, key_cache, value_cache, block_tables, seq_lens,
                                      query_start_loc, scale, dtype, row_select=None):
        """float64 ``[total_q_tokens, Hq, D]``; rows not selected stay NaN."""
        Tq, Hq, D = query.shape
        NB, B, Hkv, _ = key_cache.shape
        sl = np.ascontiguousarray(seq_lens, dtype=np.int32)
        bt = np.ascontiguousarray(block_tables, dtype=np.int32).reshape(len(sl), -1)
        qsl = np.ascontiguousarray(query_start_loc, dtype=np.int32)
        out = np.full((Tq, Hq, D), np.nan, dtype=np.float64)
        sel = None
        if row_select is not None:
            sel = np.ascontiguousarray(row_select, dtype=np.uint8)
            assert sel.shape == (Tq,)
        rc = self.lib.oracle_paged_attention_prefill_chunk(
            _ptr(out), _ptr(np.ascontiguousarray(query)), _ptr(key_cache), _ptr(value_cache), dtype, _ptr(bt),
            _ptr(sl), _ptr(qsl), len(sl), float(scale), Hq, Hkv, D, B, bt.shape[1], NB,
            _ptr(sel) if sel is not None else None)
        _check(rc, "paged_attention_prefill_chunk")
        return out


    # ---------------------------------------------------------------- FP8 (E4M3) pools
    def e4m3_encode(self, x) -> np.ndarray:
        """uint8 E4M3 codes of float64 values (nearest, ties to even, clamp at 448)."""
        x = np.ascontiguousarray(x, dtype=np.float64)
        out = np.empty(x.shape, dtype=np.uint8)
        _check(self.lib.oracle_e4m3_encode(_ptr(out), _ptr(x), x.size), "e4m3_encode")
        return out

    def reshape_and_cache_fp8(self, key, value, key_cache, value_cache, slot_mapping, src_dtype, k_scale, v_scale):
        """In place on uint8 pools ``[NB, B, Hkv, D]``: codes of key / k_scale and value / v_scale."""
        T, Hkv, D = key.shape
        NB, B = key_cache.shape[:2]
        assert key_cache.dtype == np.uint8 and value_cache.dtype == np.uint8
        sm = np.ascontiguousarray(slot_mapping, dtype=np.int64)
        rc = self.lib.oracle_reshape_and_cache_fp8(_ptr(np.ascontiguousarray(key)), _ptr(np.ascontiguousarray(value)),
                                                   _ptr(key_cache), _ptr(value_cache), _ptr(sm), T, Hkv, D, B, NB,
                                                   src_dtype, float(k_scale), float(v_scale))
        _check(rc, "reshape_and_cache_fp8")

    def paged_attention_decode_kv(self, query, q_dtype, key_cache, value_cache, kv_dtype, k_scale, v_scale,
                                  block_tables, context_lens, scale):
        """Decode with the pools in their own type and scales: float64 ``[S, Hq, D]``."""
        S, Hq, D = query.shape
        NB, B, Hkv, D2 = key_cache.shape
        assert D2 == D
        bt = np.ascontiguousarray(block_tables, dtype=np.int32).reshape(S, -1)
        cl = np.ascontiguousarray(context_lens, dtype=np.int32)
        out = np.zeros((S, Hq, D), dtype=np.float64)
        rc = self.lib.oracle_paged_attention_decode_kv(
            _ptr(out), _ptr(np.ascontiguousarray(query)), q_dtype, _ptr(key_cache), _ptr(value_cache), kv_dtype,
            float(k_scale), float(v_scale), _ptr(bt), _ptr(cl), float(scale), S, Hq, Hkv, D, B, bt.shape[1], NB)
        _check(rc, "paged_attention_decode_kv")
        return out

    def paged_attention_prefill_chunk_kv(self, query, q_dtype, key_cache, value_cache, kv_dtype, k_scale, v_scale,
                                         block_tables, seq_lens, query_start_loc, scale, row_select=None):
        """Chunked prefill with the pools in their own type and scales."""
        Tq, Hq, D = query.shape
        NB, B, Hkv, _ = key_cache.shape
        sl = np.ascontiguousarray(seq_lens, dtype=np.int32)
        bt = np.ascontiguousarray(block_tables, dtype=np.int32).reshape(len(sl), -1)
        qsl = np.ascontiguousarray(query_start_loc, dtype=np.int32)
        out = np.full((Tq, Hq, D), np.nan, dtype=np.float64)
        sel = None
        if row_select is not None:
            sel = np.ascontiguousarray(row_select, dtype=np.uint8)
            assert sel.shape == (Tq,)
        rc = self.lib.oracle_paged_attention_prefill_chunk_kv(
            _ptr(out), _ptr(np.ascontiguousarray(query)), q_dtype, _ptr(key_cache), _ptr(value_cache), kv_dtype,
            float(k_scale), float(v_scale), _ptr(bt), _ptr(sl), _ptr(qsl), len(sl), float(scale), Hq, Hkv, D, B,
            bt.shape[1], NB, _ptr(sel) if sel is not None else None)
        _check(rc, "paged_attention_prefill_chunk_kv")
        return out


_default = None


def get() -> Oracle:
    """The oracle built from ``pagedkv_oracle.c``."""
    global _default
    if _default is None:
        _default = Oracle(build())
    return _default
