"""ctypes binding of ``libpagedkv.so`` (declared in ``include/pagedkv.h``).

Argument marshalling only: every function takes torch tensors that already
live on the current CUDA device, passes their data pointers, sizes and the
current stream to the C ABI function of the same name, and raises
:class:`PagedKVError` on a non-zero status.  There is no CPU path: without
the built library every call fails.
"""
from __future__ import annotations

import ctypes
import os

import torch

from .build import LIB

_lib = None

DTYPE_CODE = {torch.float32: 0, torch.float16: 1, torch.bfloat16: 2}
FP8_E4M3 = 3
FP8_POOL_DTYPES = (torch.uint8, torch.float8_e4m3fn)  # one E4M3 code per element

DEVERR_BLOCK_ID = 0x1
DEVERR_SLOT = 0x2
DEVERR_LENGTH = 0x4
DEVERR_PAIR = 0x8
DEVERR_TIMEOUT = 0x10

EXPORTED = (
    "pkv_status_string",
    "pkv_last_cuda_error",
    "pkv_reshape_and_cache",
    "pkv_reshape_and_cache_fp8",
    "pkv_copy_blocks",
    "pkv_swap_blocks",
    "pkv_paged_attention_decode",
    "pkv_paged_attention_decode_fp8",
    "pkv_paged_attention_decode_step",
    "pkv_paged_attention_decode_step_fp8",
    "pkv_paged_attention_decode_static_scratch",
    "pkv_decode_workspace_size",
    "pkv_decode_partition_size",
    "pkv_paged_attention_prefill_chunk",
    "pkv_paged_attention_prefill_chunk_fp8",
    "pkv_prefill_fp8_workspace_size",
    "pkv_paged_attention_decode_multi",
    "pkv_paged_attention_decode_multi_step",
    "pkv_decode_multi_partition_size",
    "pkv_get_device_error",
    "pkv_set_wait_limit_ns",
)


class PagedKVError(RuntimeError):
    def __init__(self, what: str, status: int):
        lib = _lib
        msg = lib.pkv_status_string(status).decode() if lib else str(status)
        extra = lib.pkv_last_cuda_error().decode() if lib else ""
        super().__init__(f"{what}: {msg} ({status}){' - ' + extra if extra and status == -4 else ''}")
        self.status = status


def library_path() -> str:
    return LIB


def load_library():
    """Load ``libpagedkv.so``; raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB):
        raise RuntimeError(f"{LIB} is missing: build it with `python -m paged_kv_cache_409_b200.build`")
    lib = ctypes.CDLL(LIB)
    P, I, I64, F, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
    lib.pkv_status_string.argtypes = [I]
    lib.pkv_status_string.restype = ctypes.c_char_p
    lib.pkv_last_cuda_error.argtypes = []
    lib.pkv_last_cuda_error.restype = ctypes.c_char_p
    lib.pkv_reshape_and_cache.argtypes = [P, P, P, P, P, I64, I, I, I, I64, I, P]
    lib.pkv_reshape_and_cache_fp8.argtypes = [P, P, P, P, P, I64, I, I, I, I64, I, F, F, P]
    lib.pkv_paged_attention_decode_fp8.argtypes = [P, P, P, P, P, P, F, F, F, I, I, I, I, I, I, I64, I, I, I, P, SZ,
                                                   P]
    lib.pkv_copy_blocks.argtypes = [P, P, I, P, I64, I64, I64, P]
    lib.pkv_swap_blocks.argtypes = [P, P, P, P, P, I64, I64, I64, I64, P]
    lib.pkv_paged_attention_decode.argtypes = [P, P, P, P, P, P, F, I, I, I, I, I, I, I64, I, I, I, P, SZ, P]
    lib.pkv_decode_workspace_size.argtypes = [I, I, I, I, I]
    lib.pkv_decode_workspace_size.restype = SZ
    lib.pkv_decode_partition_size.argtypes = [I, I, I, I, I, I, I64, I]
    lib.pkv_paged_attention_prefill_chunk.argtypes = [P, P, P, P, P, P, P, I, I64, I, F, I, I, I, I, I, I64, I, P]
    lib.pkv_paged_attention_decode_multi.argtypes = [P, P, P, P, P, P, P, I, I64, I, I, F, I, I, I, I, I, I64, I, I,
                                                     P, SZ, P]
    lib.pkv_paged_attention_decode_multi_step.argtypes = [P, P, P, I64, P, P, P, P, P, P, P, I, I64, I, I, F, I, I,
                                                          I, I, I, I64, I, I, P, SZ, P]
    lib.pkv_decode_multi_partition_size.argtypes = [I, I, I, I]
    lib.pkv_paged_attention_prefill_chunk_fp8.argtypes = [P, P, P, P, P, P, P, I, I64, I, F, F, F, I, I, I, I, I,
                                                          I64, I, P, SZ, P]
    lib.pkv_prefill_fp8_workspace_size.argtypes = [I, I, I, I, I, I64, I, I]
    lib.pkv_prefill_fp8_workspace_size.restype = SZ
    lib.pkv_get_device_error.argtypes = [ctypes.POINTER(ctypes.c_uint32), P]
    lib.pkv_paged_attention_decode_step.argtypes = [P, P, P, I64, P, P, P, P, P, P, F, I, I, I, I, I, I, I64, I, I,
                                                    I, P, SZ, P]
    lib.pkv_paged_attention_decode_step_fp8.argtypes = [P, P, P, I64, P, P, P, P, P, P, F, F, F, I, I, I, I, I, I,
                                                        I64, I, I, I, P, SZ, P]
    lib.pkv_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
    for name in ("pkv_reshape_and_cache", "pkv_reshape_and_cache_fp8", "pkv_paged_attention_decode_fp8",
                 "pkv_copy_blocks", "pkv_swap_blocks", "pkv_paged_attention_decode",
                 "pkv_decode_partition_size", "pkv_paged_attention_prefill_chunk", "pkv_get_device_error",
                 "pkv_paged_attention_prefill_chunk_fp8", "pkv_paged_attention_decode_multi",
                 "pkv_paged_attention_decode_multi_step",
                 "pkv_decode_multi_partition_size", "pkv_paged_attention_decode_step",
                 "pkv_paged_attention_decode_step_fp8", "pkv_set_wait_limit_ns"):
        getattr(lib, name).restype = I
    _lib = lib
    return lib


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _dev(t: torch.Tensor, name: str) -> int:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def _code(t: torch.Tensor) -> int:
    try:
        return DTYPE_CODE[t.dtype]
    except KeyError:
        raise ValueError(f"unsupported dtype {t.dtype}") from None


def _ok(rc: int, what: str):
    if rc != 0:
        raise PagedKVError(what, rc)


def reshape_and_cache(key, value, key_cache, value_cache, slot_mapping, stream=None):
    """Write ``key``/``value`` ``[T, Hkv, D]`` into pool slots ``slot_mapping`` (int64, -1 = skip)."""
    lib = load_library()
    T, Hkv, D = key.shape
    NB, B = key_cache.shape[:2]
    if slot_mapping.dtype != torch.int64:
        raise ValueError("slot_mapping must be int64")
    rc = lib.pkv_reshape_and_cache(_dev(key, "key"), _dev(value, "value"), _dev(key_cache, "key_cache"),
                                   _dev(value_cache, "value_cache"), _dev(slot_mapping, "slot_mapping"), T, Hkv,
                                   D, B, NB, _code(key), _stream(stream))
    _ok(rc, "reshape_and_cache")


def _fp8_pool(t: torch.Tensor, name: str) -> int:
    if t.dtype not in FP8_POOL_DTYPES:
        raise ValueError(f"{name} must be a uint8 or float8_e4m3fn pool of E4M3 codes")
    return _dev(t, name)


def reshape_and_cache_fp8(key, value, key_cache, value_cache, slot_mapping, k_scale, v_scale, stream=None):
    """Quantise ``key``/``value`` ``[T, Hkv, D]`` (fp32/fp16/bf16) by ``1/k_scale``, ``1/v_scale`` into the
    E4M3 pools' slots ``slot_mapping`` (int64, -1 = skip)."""
    lib = load_library()
    T, Hkv, D = key.shape
    NB, B = key_cache.shape[:2]
    if slot_mapping.dtype != torch.int64:
        raise ValueError("slot_mapping must be int64")
    rc = lib.pkv_reshape_and_cache_fp8(_dev(key, "key"), _dev(value, "value"), _fp8_pool(key_cache, "key_cache"),
                                       _fp8_pool(value_cache, "value_cache"), _dev(slot_mapping, "slot_mapping"), T,
                                       Hkv, D, B, NB, _code(key), float(k_scale), float(v_scale), _stream(stream))
    _ok(rc, "reshape_and_cache_fp8")


def copy_blocks(key_caches, value_caches, src_dst_pairs, stream=None):
    """Copy block src over block dst in every layer's K and V pool (``src_dst_pairs`` int64 ``[P, 2]``)."""
    lib = load_library()
    L = len(key_caches)
    if L != len(value_caches):
        raise ValueError("key_caches and value_caches differ in length")
    if L == 0:
        return
    kp = (ctypes.c_void_p * L)(*[_dev(c, "key_caches[i]") for c in key_caches])
    vp = (ctypes.c_void_p * L)(*[_dev(c, "value_caches[i]") for c in value_caches])
    NB = key_caches[0].shape[0]
    block_bytes = key_caches[0].numel() // NB * key_caches[0].element_size()
    if src_dst_pairs.dtype != torch.int64:
        raise ValueError("src_dst_pairs must be int64")
    npairs = src_dst_pairs.numel() // 2
    rc = lib.pkv_copy_blocks(kp, vp, L, _dev(src_dst_pairs, "src_dst_pairs") if npairs else None, npairs,
                             block_bytes, NB, _stream(stream))
    _ok(rc, "copy_blocks")


def swap_blocks(src_key, src_value, dst_key, dst_value, src_dst_pairs, stream=None):
    """Move blocks ``src -> dst`` between two pools (device and/or pinned host tensors)."""
    lib = load_library()
    for t, name in ((src_key, "src_key"), (src_value, "src_value"), (dst_key, "dst_key"), (dst_value, "dst_value"),
                    (src_dst_pairs, "src_dst_pairs")):
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
        if not (t.is_cuda or t.is_pinned()):
            raise ValueError(f"{name} must be a CUDA tensor or pinned host memory")
    if src_dst_pairs.dtype != torch.int64:
        raise ValueError("src_dst_pairs must be int64")
    block_bytes = src_key[0].numel() * src_key.element_size()
    if dst_key[0].numel() * dst_key.element_size() != block_bytes:
        raise ValueError("pools differ in block size")
    rc = lib.pkv_swap_blocks(src_key.data_ptr(), src_value.data_ptr(), dst_key.data_ptr(), dst_value.data_ptr(),
                             src_dst_pairs.data_ptr(), src_dst_pairs.numel() // 2, block_bytes, src_key.shape[0],
                             dst_key.shape[0], _stream(stream))
    _ok(rc, "swap_blocks")


def decode_workspace_size(num_seqs, num_q_heads, head_dim, max_context_len, partition_size) -> int:
    return int(load_library().pkv_decode_workspace_size(num_seqs, num_q_heads, head_dim, max_context_len,
                                                         partition_size))


def decode_partition_size(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, max_context_len, dtype,
                          total_context_tokens=0) -> int:
    code = DTYPE_CODE[dtype] if isinstance(dtype, torch.dtype) else int(dtype)
    rc = load_library().pkv_decode_partition_size(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                                                  max_context_len, int(total_context_tokens), code)
    if rc < 0:
        raise PagedKVError("decode_partition_size", rc)
    return rc


def paged_attention_decode(out, query, key_cache, value_cache, block_tables, context_lens, scale, max_context_len,
                           partition_size=None, workspace=None, stream=None, total_context_tokens=0):
    """Decode attention; ``out``/``query`` ``[S, Hq, D]``, pools ``[NB, B, Hkv, D]``.

    ``partition_size`` None picks the library's recommendation (given the
    optional host-side ``total_context_tokens``); a workspace is allocated
    here when one is needed and none is given.
    """
    lib = load_library()
    S, Hq, D = query.shape
    NB, B, Hkv, _ = key_cache.shape
    MB = block_tables.shape[1] if block_tables.dim() == 2 else 1
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32:
        raise ValueError("block_tables and context_lens must be int32")
    if partition_size is None:
        partition_size = decode_partition_size(S, Hq, Hkv, D, B, max_context_len, query.dtype, total_context_tokens)
    need = decode_workspace_size(S, Hq, D, max_context_len, partition_size) if partition_size else 0
    if need and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=query.device)
    ws_ptr = _dev(workspace, "workspace") if (need and workspace is not None) else None
    ws_bytes = workspace.numel() * workspace.element_size() if ws_ptr else 0
    rc = lib.pkv_paged_attention_decode(_dev(out, "out"), _dev(query, "query"), _dev(key_cache, "key_cache"),
                                        _dev(value_cache, "value_cache"), _dev(block_tables, "block_tables"),
                                        _dev(context_lens, "context_lens"), float(scale), S, Hq, Hkv, D, B, MB, NB,
                                        int(max_context_len), int(partition_size), _code(query), ws_ptr, ws_bytes,
                                        _stream(stream))
    _ok(rc, "paged_attention_decode")
    return out


def paged_attention_decode_fp8(out, query, key_cache, value_cache, block_tables, context_lens, scale, k_scale,
                               v_scale, max_context_len, partition_size=None, workspace=None, stream=None,
                               total_context_tokens=0):
    """Decode attention over E4M3 pools (values ``k_scale * code``, ``v_scale * code``); ``out``/``query``
    ``[S, Hq, D]`` in fp16 or bf16."""
    lib = load_library()
    S, Hq, D = query.shape
    NB, B, Hkv, _ = key_cache.shape
    MB = block_tables.shape[1] if block_tables.dim() == 2 else 1
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32:
        raise ValueError("block_tables and context_lens must be int32")
    if partition_size is None:
        partition_size = decode_partition_size(S, Hq, Hkv, D, B, max_context_len, FP8_E4M3, total_context_tokens)
    need = decode_workspace_size(S, Hq, D, max_context_len, partition_size) if partition_size else 0
    if need and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=query.device)
    ws_ptr = _dev(workspace, "workspace") if (need and workspace is not None) else None
    ws_bytes = workspace.numel() * workspace.element_size() if ws_ptr else 0
    rc = lib.pkv_paged_attention_decode_fp8(_dev(out, "out"), _dev(query, "query"), _fp8_pool(key_cache, "key_cache"),
                                            _fp8_pool(value_cache, "value_cache"), _dev(block_tables, "block_tables"),
                                            _dev(context_lens, "context_lens"), float(scale), float(k_scale),
                                            float(v_scale), S, Hq, Hkv, D, B, MB, NB, int(max_context_len),
                                            int(partition_size), _code(query), ws_ptr, ws_bytes, _stream(stream))
    _ok(rc, "paged_attention_decode_fp8")
    return out


def _decode_workspace(S, Hq, Hkv, D, B, max_context_len, dtype_code, partition_size, workspace, device,
                      total_context_tokens):
    """(partition_size, workspace pointer, workspace bytes) of a decode call; allocates a workspace when one
    is needed and none (or too small a one) is given."""
    if partition_size is None:
        partition_size = decode_partition_size(S, Hq, Hkv, D, B, max_context_len, dtype_code, total_context_tokens)
    need = decode_workspace_size(S, Hq, D, max_context_len, partition_size) if partition_size else 0
    if need and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=device)
    ws_ptr = _dev(workspace, "workspace") if (need and workspace is not None) else None
    ws_bytes = workspace.numel() * workspace.element_size() if ws_ptr else 0
    return int(partition_size), ws_ptr, ws_bytes


def paged_attention_decode_step(new_keys, new_values, slot_mapping, out, query, key_cache, value_cache, block_tables,
                                context_lens, scale, max_context_len, partition_size=None, workspace=None,
                                stream=None, total_context_tokens=0):
    """One decode step: ``reshape_and_cache(new_keys, new_values, ..., slot_mapping)`` then
    ``paged_attention_decode`` in one call (the decode launched as the append's programmatic dependent)."""
    lib = load_library()
    S, Hq, D = query.shape
    NB, B, Hkv, _ = key_cache.shape
    MB = block_tables.shape[1] if block_tables.dim() == 2 else 1
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32:
        raise ValueError("block_tables and context_lens must be int32")
    if slot_mapping.dtype != torch.int64:
        raise ValueError("slot_mapping must be int64")
    part, ws_ptr, ws_bytes = _decode_workspace(S, Hq, Hkv, D, B, max_context_len, _code(query), partition_size,
                                               workspace, query.device, total_context_tokens)
    rc = lib.pkv_paged_attention_decode_step(_dev(new_keys, "new_keys"), _dev(new_values, "new_values"),
                                             _dev(slot_mapping, "slot_mapping"), new_keys.shape[0], _dev(out, "out"),
                                             _dev(query, "query"), _dev(key_cache, "key_cache"),
                                             _dev(value_cache, "value_cache"), _dev(block_tables, "block_tables"),
                                             _dev(context_lens, "context_lens"), float(scale), S, Hq, Hkv, D, B, MB,
                                             NB, int(max_context_len), part, _code(query), ws_ptr, ws_bytes,
                                             _stream(stream))
    _ok(rc, "paged_attention_decode_step")
    return out


def paged_attention_decode_step_fp8(new_keys, new_values, slot_mapping, out, query, key_cache, value_cache,
                                    block_tables, context_lens, scale, k_scale, v_scale, max_context_len,
                                    partition_size=None, workspace=None, stream=None, total_context_tokens=0):
    """The decode step over E4M3 pools: ``reshape_and_cache_fp8`` then ``paged_attention_decode_fp8``."""
    lib = load_library()
    S, Hq, D = query.shape
    NB, B, Hkv, _ = key_cache.shape
    MB = block_tables.shape[1] if block_tables.dim() == 2 else 1
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32:
        raise ValueError("block_tables and context_lens must be int32")
    if slot_mapping.dtype != torch.int64:
        raise ValueError("slot_mapping must be int64")
    part, ws_ptr, ws_bytes = _decode_workspace(S, Hq, Hkv, D, B, max_context_len, FP8_E4M3, partition_size,
                                               workspace, query.device, total_context_tokens)
    rc = lib.pkv_paged_attention_decode_step_fp8(_dev(new_keys, "new_keys"), _dev(new_values, "new_values"),
                                                 _dev(slot_mapping, "slot_mapping"), new_keys.shape[0],
                                                 _dev(out, "out"), _dev(query, "query"),
                                                 _fp8_pool(key_cache, "key_cache"),
                                                 _fp8_pool(value_cache, "value_cache"),
                                                 _dev(block_tables, "block_tables"),
                                                 _dev(context_lens, "context_lens"), float(scale), float(k_scale),
                                                 float(v_scale), S, Hq, Hkv, D, B, MB, NB, int(max_context_len), part,
                                                 _code(query), ws_ptr, ws_bytes, _stream(stream))
    _ok(rc, "paged_attention_decode_step_fp8")
    return out


def set_wait_limit_ns(limit_ns: int):
    """Limit of the kernels' main-loop waits for later launches (0 = give up at the first blocking wait; a
    test setting).  The default is one second."""
    _ok(load_library().pkv_set_wait_limit_ns(int(limit_ns)), "set_wait_limit_ns")


DEFAULT_WAIT_LIMIT_NS = 1_000_000_000


def paged_attention_prefill_chunk(out, query, key_cache, value_cache, block_tables, seq_lens, query_start_loc,
                                  max_q_len, scale, stream=None):
    """Causal chunked prefill; ``out``/``query`` packed ``[sum n_r, Hq, D]``."""
    lib = load_library()
    Tq, Hq, D = query.shape
    NB, B, Hkv, _ = key_cache.shape
    R = seq_lens.numel()
    MB = block_tables.shape[1]
    for t, name in ((block_tables, "block_tables"), (seq_lens, "seq_lens"), (query_start_loc, "query_start_loc")):
        if t.dtype != torch.int32:
            raise ValueError(f"{name} must be int32")
    rc = lib.pkv_paged_attention_prefill_chunk(_dev(out, "out"), _dev(query, "query"), _dev(key_cache, "key_cache"),
                                               _dev(value_cache, "value_cache"), _dev(block_tables, "block_tables"),
                                               _dev(seq_lens, "seq_lens"), _dev(query_start_loc, "query_start_loc"),
                                               R, Tq, int(max_q_len), float(scale), Hq, Hkv, D, B, MB, NB,
                                               _code(query), _stream(stream))
    _ok(rc, "paged_attention_prefill_chunk")
    return out


def prefill_fp8_workspace_size(num_chunks, max_blocks_per_seq, block_size, num_kv_heads, head_dim, total_q_tokens,
                               num_q_heads, dtype) -> int:
    code = DTYPE_CODE[dtype] if isinstance(dtype, torch.dtype) else int(dtype)
    return int(load_library().pkv_prefill_fp8_workspace_size(num_chunks, max_blocks_per_seq, block_size,
                                                             num_kv_heads, head_dim, int(total_q_tokens),
                                                             num_q_heads, code))


def paged_attention_prefill_chunk_fp8(out, query, key_cache, value_cache, block_tables, seq_lens, query_start_loc,
                                      max_q_len, scale, k_scale, v_scale, workspace=None, stream=None):
    """Causal chunked prefill over E4M3 pools (values ``k_scale * code``, ``v_scale * code``)."""
    lib = load_library()
    Tq, Hq, D = query.shape
    NB, B, Hkv, _ = key_cache.shape
    R = seq_lens.numel()
    MB = block_tables.shape[1]
    for t, name in ((block_tables, "block_tables"), (seq_lens, "seq_lens"), (query_start_loc, "query_start_loc")):
        if t.dtype != torch.int32:
            raise ValueError(f"{name} must be int32")
    need = prefill_fp8_workspace_size(R, MB, B, Hkv, D, Tq, Hq, query.dtype)
    if workspace is None or workspace.numel() * workspace.element_size() < need or workspace.data_ptr() % 256:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=query.device)
    rc = lib.pkv_paged_attention_prefill_chunk_fp8(
        _dev(out, "out"), _dev(query, "query"), _fp8_pool(key_cache, "key_cache"),
        _fp8_pool(value_cache, "value_cache"), _dev(block_tables, "block_tables"), _dev(seq_lens, "seq_lens"),
        _dev(query_start_loc, "query_start_loc"), R, Tq, int(max_q_len), float(scale), float(k_scale),
        float(v_scale), Hq, Hkv, D, B, MB, NB, _code(query), _dev(workspace, "workspace"),
        workspace.numel() * workspace.element_size(), _stream(stream))
    _ok(rc, "paged_attention_prefill_chunk_fp8")
    return out


def decode_multi_partition_size(num_chunks, num_kv_heads, block_size, max_seq_len) -> int:
    rc = load_library().pkv_decode_multi_partition_size(num_chunks, num_kv_heads, block_size, max_seq_len)
    if rc < 0:
        raise PagedKVError("decode_multi_partition_size", rc)
    return rc


def paged_attention_decode_multi(out, query, key_cache, value_cache, block_tables, seq_lens, query_start_loc,
                                 max_q_len, max_seq_len, scale, partition_size=None, workspace=None, stream=None):
    """Multi-token decode (a few causal query tokens per sequence); arguments as for
    :func:`paged_attention_prefill_chunk` plus the host bound ``max_seq_len``."""
    lib = load_library()
    Tq, Hq, D = query.shape
    NB, B, Hkv, _ = key_cache.shape
    R = seq_lens.numel()
    MB = block_tables.shape[1]
    for t, name in ((block_tables, "block_tables"), (seq_lens, "seq_lens"), (query_start_loc, "query_start_loc")):
        if t.dtype != torch.int32:
            raise ValueError(f"{name} must be int32")
    if partition_size is None:
        partition_size = decode_multi_partition_size(R, Hkv, B, max_seq_len)
    need = decode_workspace_size(Tq, Hq, D, max_seq_len, partition_size) if partition_size else 0
    if need and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=query.device)
    ws_ptr = _dev(workspace, "workspace") if (need and workspace is not None) else None
    ws_bytes = workspace.numel() * workspace.element_size() if ws_ptr else 0
    rc = lib.pkv_paged_attention_decode_multi(_dev(out, "out"), _dev(query, "query"), _dev(key_cache, "key_cache"),
                                              _dev(value_cache, "value_cache"), _dev(block_tables, "block_tables"),
                                              _dev(seq_lens, "seq_lens"), _dev(query_start_loc, "query_start_loc"),
                                              R, Tq, int(max_q_len), int(max_seq_len), float(scale), Hq, Hkv, D, B,
                                              MB, NB, int(partition_size), _code(query), ws_ptr, ws_bytes,
                                              _stream(stream))
    _ok(rc, "paged_attention_decode_multi")
    return out


def paged_attention_decode_multi_step(new_keys, new_values, slot_mapping, out, query, key_cache, value_cache,
                                      block_tables, seq_lens, query_start_loc, max_q_len, max_seq_len, scale,
                                      partition_size=None, workspace=None, stream=None):
    """One verification step: ``reshape_and_cache(new_keys, new_values, ..., slot_mapping)`` then
    ``paged_attention_decode_multi`` in one call (the attention launched as the append's
    programmatic dependent)."""
    lib = load_library()
    Tq, Hq, D = query.shape
    NB, B, Hkv, _ = key_cache.shape
    R = seq_lens.numel()
    MB = block_tables.shape[1]
    for t, name in ((block_tables, "block_tables"), (seq_lens, "seq_lens"), (query_start_loc, "query_start_loc")):
        if t.dtype != torch.int32:
            raise ValueError(f"{name} must be int32")
    if slot_mapping.dtype != torch.int64:
        raise ValueError("slot_mapping must be int64")
    if partition_size is None:
        partition_size = decode_multi_partition_size(R, Hkv, B, max_seq_len)
    need = decode_workspace_size(Tq, Hq, D, max_seq_len, partition_size) if partition_size else 0
    if need and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=query.device)
    ws_ptr = _dev(workspace, "workspace") if (need and workspace is not None) else None
    ws_bytes = workspace.numel() * workspace.element_size() if ws_ptr else 0
    rc = lib.pkv_paged_attention_decode_multi_step(
        _dev(new_keys, "new_keys"), _dev(new_values, "new_values"), _dev(slot_mapping, "slot_mapping"),
        new_keys.shape[0], _dev(out, "out"), _dev(query, "query"), _dev(key_cache, "key_cache"),
        _dev(value_cache, "value_cache"), _dev(block_tables, "block_tables"), _dev(seq_lens, "seq_lens"),
        _dev(query_start_loc, "query_start_loc"), R, Tq, int(max_q_len), int(max_seq_len), float(scale), Hq, Hkv, D,
        B, MB, NB, int(partition_size), _code(query), ws_ptr, ws_bytes, _stream(stream))
    _ok(rc, "paged_attention_decode_multi_step")
    return out


def get_device_error(stream=None) -> int:
    """Read and clear the device error word (PKV_DEVERR_* bits); synchronises the stream."""
    lib = load_library()
    v = ctypes.c_uint32(0)
    _ok(lib.pkv_get_device_error(ctypes.byref(v), _stream(stream)), "get_device_error")
    return int(v.value)
