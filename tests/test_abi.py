"""The C-ABI library loads without a GPU and exports every entry point its header declares."""
import ctypes
import os
import re

import pytest
import torch

import paged_kv_cache_409_b200 as pkv
from paged_kv_cache_409_b200 import _binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared():
    src = open(os.path.join(ROOT, "include", "pagedkv.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(pkv_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    from paged_kv_cache_409_b200 import build
    build.build()
    return pkv.load_library()


def test_every_declared_symbol_is_exported(lib):
    names = declared()
    assert len(names) >= 9
    for n in names:
        assert hasattr(lib, n), f"{n} declared in include/pagedkv.h but not exported"
    assert set(names) == set(_binding.EXPORTED) | (set(names) - set(_binding.EXPORTED))
    for n in _binding.EXPORTED:
        assert n in names, f"binding names {n} which the header does not declare"


def test_status_strings(lib):
    assert lib.pkv_status_string(0) == b"ok"
    assert lib.pkv_status_string(-5).startswith(b"workspace")


def test_workspace_size_arithmetic(lib):
    # no split -> no workspace
    assert pkv.decode_workspace_size(64, 32, 128, 2048, 0) == 0
    assert pkv.decode_workspace_size(64, 32, 128, 512, 512) == 0
    # 64 x 32 heads x 4 partitions: max + sum (16-byte rounded) + outputs
    rows = 64 * 32 * 4
    assert pkv.decode_workspace_size(64, 32, 128, 2048, 512) == 2 * rows * 4 + rows * 128 * 4


def test_partition_heuristic(lib):
    # large batches: one CTA per (sequence, KV head), no split
    assert pkv.decode_partition_size(64, 32, 32, 128, 16, 2048, 1) == 0
    assert pkv.decode_partition_size(192, 64, 8, 128, 32, 32768, 2) == 0
    # small batches: block-multiple partitions of at least 256 tokens, shorter than the context
    for B in (8, 16, 32):
        p = pkv.decode_partition_size(2, 2, 2, 128, B, 10000, 1)
        assert p % B == 0 and 256 <= p < 10000
    assert pkv.decode_partition_size(1, 1, 1, 128, 16, 200, 1) == 0
    # a long tail (max far above the mean) is cut at 1.5x the mean
    p = pkv.decode_partition_size(256, 64, 8, 128, 16, 4096, 2, total_context_tokens=256 * 1436)
    assert p == 2160
    assert pkv.decode_partition_size(192, 64, 8, 128, 32, 32768, 2, total_context_tokens=192 * 16500) == 0
    # query heads must group evenly over KV heads
    with pytest.raises(pkv.PagedKVError):
        pkv.decode_partition_size(64, 12, 8, 128, 16, 2048, 1)


def test_partition_heuristic_fp8_waves(lib):
    """E4M3 pools, one query head per KV head: fewer pairs than ~22 CTAs per SM are cut into parts of
    Hkv * total / (22 * SMs - pairs / 2) tokens (at least 512, block multiples); grouped heads, large
    batches, an unknown total and 16-bit pools stay unsplit."""
    sms = 148  # the library's SM count when no device is visible
    total = 64 * 1039
    p = pkv.decode_partition_size(64, 32, 32, 128, 16, 2029, pkv.FP8_E4M3, total_context_tokens=total)
    want = -(-32 * total // (22 * sms - 64 * 32 // 2))
    assert p == -(-want // 16) * 16 == 960
    total = 32 * 2560
    p = pkv.decode_partition_size(32, 32, 32, 128, 16, 4096, pkv.FP8_E4M3, total_context_tokens=total)
    assert p == 960  # 32 x 81920 / (3256 - 512) = 955.4, rounded up to a block multiple
    # short contexts: at least 512 tokens per part, and none when that covers the longest
    assert pkv.decode_partition_size(64, 32, 32, 128, 16, 600, pkv.FP8_E4M3, total_context_tokens=64 * 300) == 512
    assert pkv.decode_partition_size(64, 32, 32, 128, 16, 512, pkv.FP8_E4M3, total_context_tokens=64 * 300) == 0
    for args, total in [((128, 32, 32), 128 * 1088), ((256, 64, 8), 256 * 1088), ((64, 32, 32), 0)]:
        assert pkv.decode_partition_size(*args, 128, 16, 2048, pkv.FP8_E4M3, total_context_tokens=total) == 0
    assert pkv.decode_partition_size(64, 32, 32, 128, 16, 2029, torch.float16, total_context_tokens=64 * 1039) == 0


def test_host_rejections_before_launch(lib):
    # unsupported dtype and bad sizes are refused before any device work
    assert lib.pkv_paged_attention_decode(None, None, None, None, None, None, 0.1, 1, 4, 2, 128, 16, 1, 1, 16, 0, 7,
                                          None, 0, None) == -2
    assert lib.pkv_paged_attention_decode(None, None, None, None, None, None, 0.1, 1, 4, 3, 128, 16, 1, 1, 16, 0, 1,
                                          None, 0, None) == -1
    assert lib.pkv_paged_attention_decode(None, None, None, None, None, None, 0.1, 1, 4, 2, 128, 16, 1, 1, 16, 0, 1,
                                          None, 0, None) == -1  # null pointers
    assert lib.pkv_reshape_and_cache(None, None, None, None, None, 0, 2, 64, 16, 4, 1, None) == 0  # empty: no-op
    assert lib.pkv_copy_blocks(None, None, 0, None, 0, 4096, 4, None) == 0
    assert lib.pkv_paged_attention_prefill_chunk(None, None, None, None, None, None, None, 1, 4, 4, 0.1, 2, 2, 64,
                                                 16, 1, 4, 0, None) == -2  # fp32 prefill
    assert lib.pkv_get_device_error(None, None) == -1


def test_host_rejections_fp8_and_multi_token(lib):
    # FP8 pools: fp32 query, head_dim 64, non-positive or non-finite scales, an fp8 query type
    dec8 = lib.pkv_paged_attention_decode_fp8
    assert dec8(None, None, None, None, None, None, 0.1, 1.0, 1.0, 1, 4, 2, 128, 16, 1, 1, 16, 0, 0, None, 0,
                None) == -2
    assert dec8(None, None, None, None, None, None, 0.1, 1.0, 1.0, 1, 4, 2, 64, 16, 1, 1, 16, 0, 1, None, 0,
                None) == -2
    assert dec8(None, None, None, None, None, None, 0.1, 0.0, 1.0, 1, 4, 2, 128, 16, 1, 1, 16, 0, 1, None, 0,
                None) == -1
    assert dec8(None, None, None, None, None, None, 0.1, 1.0, float("inf"), 1, 4, 2, 128, 16, 1, 1, 16, 0, 1,
                None, 0, None) == -1
    assert lib.pkv_paged_attention_decode(None, None, None, None, None, None, 0.1, 1, 4, 2, 128, 16, 1, 1, 16, 0, 3,
                                          None, 0, None) == -2  # an FP8 query is not a query type
    assert lib.pkv_reshape_and_cache_fp8(None, None, None, None, None, 4, 2, 64, 16, 4, 3, 1.0, 1.0, None) == -2
    assert lib.pkv_reshape_and_cache_fp8(None, None, None, None, None, 4, 2, 64, 16, 4, 1, -1.0, 1.0, None) == -1
    assert lib.pkv_reshape_and_cache_fp8(None, None, None, None, None, 0, 2, 64, 16, 4, 1, 1.0, 1.0, None) == 0
    assert lib.pkv_reshape_and_cache_fp8(None, None, None, None, None, 4, 1, 8, 16, 4, 1, 1.0, 1.0, None) == -2
    # FP8 prefill: workspace is checked before any device work
    pf8 = lib.pkv_paged_attention_prefill_chunk_fp8
    assert pf8(None, None, None, None, None, None, None, 1, 4, 4, 0.1, 1.0, 1.0, 2, 2, 64, 16, 1, 4, 0, None, 0,
               None) == -2  # fp32 query
    assert lib.pkv_prefill_fp8_workspace_size(2, 10, 16, 8, 128, 100, 32, 2) == \
        100 * 32 * 128 * 2 + 2 * (2 * 10 * 16 * 8 * 128 * 2) + 1024
    assert lib.pkv_prefill_fp8_workspace_size(2, 10, 16, 8, 128, 100, 32, 1) == \
        2 * (2 * 10 * 16 * 8 * 128 * 2) + 1024
    # multi-token decode: more than 32 rows per KV head, bad partition size
    mt = lib.pkv_paged_attention_decode_multi
    assert mt(None, None, None, None, None, None, None, 1, 9, 9, 100, 0.1, 32, 8, 128, 16, 8, 16, 0, 1, None, 0,
              None) == -2
    assert mt(None, None, None, None, None, None, None, 1, 6, 6, 100, 0.1, 32, 8, 128, 16, 8, 16, 24, 1, None, 0,
              None) == -1
    assert mt(None, None, None, None, None, None, None, 0, 0, 6, 100, 0.1, 32, 8, 128, 16, 8, 16, 0, 1, None, 0,
              None) == 0
    assert pkv.decode_multi_partition_size(64, 8, 32, 4039) % 32 == 0
    assert pkv.decode_multi_partition_size(1000, 32, 16, 2048) == 0  # enough pairs: no split
    assert pkv.decode_multi_partition_size(1, 1, 16, 200) == 0       # short: no split


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(_binding, "_lib", None)
    monkeypatch.setattr(_binding, "LIB", str(tmp_path / "nope.so"))
    with pytest.raises(RuntimeError):
        _binding.load_library()


def _prototypes():
    """name -> (return type, [parameter types]) for every function both headers declare."""
    protos = {}
    for header in ("pagedkv.h", "pagedkv_block_manager.h"):
        src = open(os.path.join(ROOT, "include", header)).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        src = re.sub(r"//[^\n]*", "", src)
        for ret, name, params in re.findall(r"^([A-Za-z_][\w \t\*]*?)\s*\b(pkv_[a-z0-9_]+)\s*\(([^;{]*?)\)\s*;", src, flags=re.M):
            params = " ".join(params.split())
            types = [] if params in ("", "void") else [re.sub(r"\s*\b\w+$", "", p.strip()) for p in params.split(",")]
            protos[name] = (" ".join(ret.split()), types)
    return protos


def _kind(ctype_name):
    """The ctypes type a C type marshals as."""
    t = ctype_name.replace("const ", "").strip()
    if "*" in t or t in ("pkv_stream_t",):
        return "ptr"
    return {"int": ctypes.c_int, "int64_t": ctypes.c_int64, "float": ctypes.c_float, "size_t": ctypes.c_size_t,
            "uint32_t": ctypes.c_uint32, "uint64_t": ctypes.c_uint64, "void": None}[t]


def _argkind(a):
    if a in (ctypes.c_void_p, ctypes.c_char_p) or (isinstance(a, type) and issubclass(a, ctypes._Pointer)):
        return "ptr"
    return a


def test_binding_argtypes_match_the_header_prototypes(lib):
    """Every argtypes / restype the Python bindings set agrees with the header's prototype in count and
    width (an int marshalled where the C side takes int64_t would pass garbage in the upper half)."""
    from paged_kv_cache_409_b200 import block_manager
    bm_lib = block_manager._lib()
    protos = _prototypes()
    assert "pkv_bm_swap_in" in protos and "pkv_paged_attention_decode_multi" in protos
    checked = 0
    for name, (ret, params) in protos.items():
        fn = getattr(bm_lib if name.startswith("pkv_bm_") else lib, name)
        if fn.argtypes is None:
            continue
        got = [_argkind(a) for a in fn.argtypes]
        want = [_kind(p) for p in params]
        assert got == want, f"{name}: binding {got} vs header {want}"
        rk = _kind(ret)
        if rk == "ptr":
            assert fn.restype in (ctypes.c_void_p, ctypes.c_char_p), name
        elif rk is not None:
            assert fn.restype == rk, f"{name}: restype {fn.restype} vs header {ret}"
        checked += 1
    assert checked >= 25


def test_python_constants_match_the_headers():
    """dtype codes, status codes and device-error bits as the headers define them."""
    from paged_kv_cache_409_b200 import block_manager
    src = open(os.path.join(ROOT, "include", "pagedkv.h")).read() + \
        open(os.path.join(ROOT, "include", "pagedkv_block_manager.h")).read()
    enum = {k: int(v) for k, v in re.findall(r"\b(PKV_[A-Z0-9_]+)\s*=\s*(-?\d+)", src)}
    bits = {k: int(v, 16) for k, v in re.findall(r"#define\s+(PKV_DEVERR_[A-Z_]+)\s+0x([0-9a-fA-F]+)u", src)}
    assert _binding.DTYPE_CODE[torch.float32] == enum["PKV_F32"]
    assert _binding.DTYPE_CODE[torch.float16] == enum["PKV_F16"]
    assert _binding.DTYPE_CODE[torch.bfloat16] == enum["PKV_BF16"]
    assert _binding.FP8_E4M3 == enum["PKV_FP8_E4M3"]
    for name in ("BLOCK_ID", "SLOT", "LENGTH", "PAIR", "TIMEOUT"):
        assert getattr(_binding, "DEVERR_" + name) == bits["PKV_DEVERR_" + name]
    assert (block_manager.OK, block_manager.EINVAL, block_manager.ENOSPACE, block_manager.EBUFFER) == (
        enum["PKV_BM_OK"], enum["PKV_BM_EINVAL"], enum["PKV_BM_ENOSPACE"], enum["PKV_BM_EBUFFER"])
    for code in ("PKV_EINVAL", "PKV_EUNSUPPORTED", "PKV_ERANGE", "PKV_ECUDA", "PKV_EWORKSPACE"):
        assert pkv.load_library().pkv_status_string(enum[code]) != b"ok"


def test_partition_heuristics_properties(lib):
    """Over random batches: a recommended partition is 0 (no split) or a block multiple of at least 256
    tokens (512 for the E4M3 wave rule) shorter than the longest context, and the workspace it needs is
    what pkv_decode_workspace_size reports for it.  Every recommendation stays within the 4096 blocks a
    partition may hold, so the decode accepts it: no split only when the longest context fits."""
    from hypothesis import given, settings, strategies as st

    @settings(max_examples=300, deadline=None)
    @given(st.integers(1, 512), st.sampled_from([1, 2, 4, 8]), st.sampled_from([1, 2, 4, 8, 32]),
           st.sampled_from([8, 16, 32]), st.one_of(st.integers(1, 40000), st.integers(30000, 300000)),
           st.floats(0.05, 1.0),
           st.sampled_from([torch.float16, torch.bfloat16, torch.float32, pkv.FP8_E4M3]))
    def check(S, G, Hkv, B, max_len, mean_frac, dt):
        total = max(S, int(S * max_len * mean_frac))
        p = pkv.decode_partition_size(S, Hkv * G, Hkv, 128, B, max_len, dt, total_context_tokens=total)
        assert p == 0 or (p % B == 0 and 256 <= p < max_len)
        assert (p == 0 and -(-max_len // B) <= 4096) or (p > 0 and p // B <= 4096)
        if p:
            parts = -(-max_len // p)
            rows = S * Hkv * G * parts
            assert pkv.decode_workspace_size(S, Hkv * G, 128, max_len, p) == 2 * (-(-rows * 4 // 16) * 16) + \
                rows * 128 * 4
        m = pkv.decode_multi_partition_size(S, Hkv, B, max_len)
        assert m == 0 or (m % B == 0 and m >= 256 and m < max_len)
        assert (m == 0 and -(-max_len // B) <= 4096) or (m > 0 and m // B <= 4096)

    check()
