"""The Python binding passes every argument to the C ABI in the place the header gives it (no GPU).

A stand-in library is generated from include/pagedkv.h: each entry point records its arguments by
position and returns 0.  The binding is pointed at it, with CPU tensors standing in for device ones, and
each call's recorded arguments are checked by the header's parameter names against the tensors' shapes
and pointers."""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest
import torch

import paged_kv_cache_409_b200 as pkv
from paged_kv_cache_409_b200 import _binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _header_functions():
    src = open(os.path.join(ROOT, "include", "pagedkv.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    out = []
    for ret, name, params in re.findall(r"^([A-Za-z_][\w \t\*]*?)\s*\b(pkv_[a-z0-9_]+)\s*\(([^;{]*?)\)\s*;", src, flags=re.M):
        params = " ".join(params.split())
        plist = [] if params in ("", "void") else [p.strip() for p in params.split(",")]
        names = [re.search(r"(\w+)$", p).group(1) for p in plist]
        out.append((" ".join(ret.split()), name, plist, names))
    return out


@pytest.fixture()
def mock(tmp_path, monkeypatch):
    funcs = _header_functions()
    lines = ['#include <stdint.h>', '#include "pagedkv.h"', 'double rec_vals[64]; int rec_n; char rec_name[64];',
             'static void rec_begin(const char* n) { int i = 0; for (; n[i] && i < 63; ++i) rec_name[i] = n[i];'
             ' rec_name[i] = 0; rec_n = 0; }',
             'static void rec(double v) { if (rec_n < 64) rec_vals[rec_n++] = v; }']
    for ret, name, plist, names in funcs:
        body = [f'rec_begin("{name}");']
        for p, n in zip(plist, names):
            body.append(f"rec((double)(uintptr_t){n});" if ("*" in p or "pkv_stream_t" in p) else f"rec((double){n});")
        body.append('return "ok";' if "char" in ret else "return 0;")
        lines.append(f"{ret} {name}({', '.join(plist) or 'void'}) {{ {' '.join(body)} }}")
    src = tmp_path / "mock.c"
    src.write_text("\n".join(lines) + "\n")
    so = tmp_path / "libmock.so"
    subprocess.check_call(["gcc", "-O0", "-std=c11", "-Wall", "-Werror", "-fPIC", "-shared",
                           "-I", os.path.join(ROOT, "include"), "-o", str(so), str(src)])
    monkeypatch.setattr(_binding, "LIB", str(so))
    monkeypatch.setattr(_binding, "_lib", None)
    monkeypatch.setattr(_binding, "_dev", lambda t, name: t.data_ptr())
    monkeypatch.setattr(_binding, "_stream", lambda s: 0 if s is None else int(s))
    names = {name: pnames for _, name, _, pnames in funcs}

    class Recorder:
        def last(self):
            lib = _binding.load_library()
            fname = (ctypes.c_char * 64).in_dll(lib, "rec_name").value.decode()
            n = ctypes.c_int.in_dll(lib, "rec_n").value
            vals = list((ctypes.c_double * 64).in_dll(lib, "rec_vals"))[:n]
            return fname, dict(zip(names[fname], vals))

    return Recorder()


def f32(x):
    return float(np.float32(x))


def test_decode_arguments(mock):
    S, Hq, Hkv, D, B, NB, MB = 3, 8, 2, 64, 16, 37, 5
    q = torch.zeros(S, Hq, D, dtype=torch.bfloat16)
    out = torch.zeros_like(q)
    kc, vc = torch.zeros(NB, B, Hkv, D, dtype=torch.bfloat16), torch.zeros(NB, B, Hkv, D, dtype=torch.bfloat16)
    bt, cl = torch.zeros(S, MB, dtype=torch.int32), torch.zeros(S, dtype=torch.int32)
    pkv.paged_attention_decode(out, q, kc, vc, bt, cl, 0.3, 71, partition_size=0, stream=5)
    name, a = mock.last()
    assert name == "pkv_paged_attention_decode"
    assert a == {"out": out.data_ptr(), "query": q.data_ptr(), "key_cache": kc.data_ptr(),
                 "value_cache": vc.data_ptr(), "block_tables": bt.data_ptr(), "context_lens": cl.data_ptr(),
                 "scale": f32(0.3), "num_seqs": S, "num_q_heads": Hq, "num_kv_heads": Hkv, "head_dim": D,
                 "block_size": B, "max_blocks_per_seq": MB, "num_blocks": NB, "max_context_len": 71,
                 "partition_size": 0, "dtype": 2, "workspace": 0, "workspace_bytes": 0, "stream": 5}


def test_decode_fp8_and_multi_arguments(mock):
    S, Hq, Hkv, D, B, NB, MB = 4, 16, 4, 128, 32, 19, 3
    q = torch.zeros(S, Hq, D, dtype=torch.float16)
    out = torch.zeros_like(q)
    kc, vc = torch.zeros(NB, B, Hkv, D, dtype=torch.uint8), torch.zeros(NB, B, Hkv, D, dtype=torch.uint8)
    bt, cl = torch.zeros(S, MB, dtype=torch.int32), torch.zeros(S, dtype=torch.int32)
    pkv.paged_attention_decode_fp8(out, q, kc, vc, bt, cl, 0.1, 0.02, 0.03, 90, partition_size=0)
    name, a = mock.last()
    assert name == "pkv_paged_attention_decode_fp8"
    assert (a["scale"], a["k_scale"], a["v_scale"]) == (f32(0.1), f32(0.02), f32(0.03))
    assert (a["num_seqs"], a["num_q_heads"], a["num_kv_heads"], a["head_dim"], a["block_size"],
            a["max_blocks_per_seq"], a["num_blocks"], a["max_context_len"], a["dtype"]) == (S, Hq, Hkv, D, B, MB,
                                                                                            NB, 90, 1)
    assert (a["key_cache"], a["value_cache"], a["out"], a["query"]) == (kc.data_ptr(), vc.data_ptr(),
                                                                        out.data_ptr(), q.data_ptr())
    # multi-token: 3 chunks, 7 packed query tokens
    R, Tq = 3, 7
    q = torch.zeros(Tq, Hq, D, dtype=torch.float16)
    out = torch.zeros_like(q)
    kc16 = torch.zeros(NB, B, Hkv, D, dtype=torch.float16)
    bt, sl = torch.zeros(R, MB, dtype=torch.int32), torch.zeros(R, dtype=torch.int32)
    qsl = torch.zeros(R + 1, dtype=torch.int32)
    pkv.paged_attention_decode_multi(out, q, kc16, kc16, bt, sl, qsl, 4, 80, 0.2, partition_size=0)
    name, a = mock.last()
    assert name == "pkv_paged_attention_decode_multi"
    assert (a["num_chunks"], a["total_q_tokens"], a["max_q_len"], a["max_seq_len"], a["scale"], a["num_q_heads"],
            a["num_kv_heads"], a["head_dim"], a["block_size"], a["max_blocks_per_seq"], a["num_blocks"],
            a["partition_size"], a["dtype"]) == (R, Tq, 4, 80, f32(0.2), Hq, Hkv, D, B, MB, NB, 0, 1)
    assert (a["block_tables"], a["seq_lens"], a["query_start_loc"]) == (bt.data_ptr(), sl.data_ptr(),
                                                                         qsl.data_ptr())


def test_prefill_arguments(mock):
    R, Tq, Hq, Hkv, D, B, NB, MB = 2, 9, 8, 2, 128, 16, 23, 6
    q = torch.zeros(Tq, Hq, D, dtype=torch.bfloat16)
    out = torch.zeros_like(q)
    kc = torch.zeros(NB, B, Hkv, D, dtype=torch.bfloat16)
    bt, sl, qsl = torch.zeros(R, MB, dtype=torch.int32), torch.zeros(R, dtype=torch.int32), \
        torch.zeros(R + 1, dtype=torch.int32)
    pkv.paged_attention_prefill_chunk(out, q, kc, kc, bt, sl, qsl, 5, 0.7)
    name, a = mock.last()
    assert name == "pkv_paged_attention_prefill_chunk"
    assert (a["num_chunks"], a["total_q_tokens"], a["max_q_len"], a["scale"], a["num_q_heads"], a["num_kv_heads"],
            a["head_dim"], a["block_size"], a["max_blocks_per_seq"], a["num_blocks"], a["dtype"]) == (
        R, Tq, 5, f32(0.7), Hq, Hkv, D, B, MB, NB, 2)
    k8 = torch.zeros(NB, B, Hkv, D, dtype=torch.uint8)
    pkv.paged_attention_prefill_chunk_fp8(out, q, k8, k8, bt, sl, qsl, 5, 0.7, 0.5, 0.25)
    name, a = mock.last()
    assert name == "pkv_paged_attention_prefill_chunk_fp8"
    assert (a["k_scale"], a["v_scale"], a["num_chunks"], a["total_q_tokens"], a["num_blocks"]) == (
        0.5, 0.25, R, Tq, NB)
    assert a["workspace"] != 0 and a["workspace_bytes"] >= 256


def test_index_calls_arguments(mock):
    T, Hkv, D, B, NB = 5, 4, 64, 16, 11
    k, v = torch.zeros(T, Hkv, D, dtype=torch.float16), torch.zeros(T, Hkv, D, dtype=torch.float16)
    kc, vc = torch.zeros(NB, B, Hkv, D, dtype=torch.float16), torch.zeros(NB, B, Hkv, D, dtype=torch.float16)
    sm = torch.zeros(T, dtype=torch.int64)
    pkv.reshape_and_cache(k, v, kc, vc, sm)
    name, a = mock.last()
    assert name == "pkv_reshape_and_cache"
    assert (a["key"], a["value"], a["key_cache"], a["value_cache"], a["slot_mapping"]) == (
        k.data_ptr(), v.data_ptr(), kc.data_ptr(), vc.data_ptr(), sm.data_ptr())
    assert (a["num_tokens"], a["num_kv_heads"], a["head_dim"], a["block_size"], a["num_blocks"], a["dtype"]) == (
        T, Hkv, D, B, NB, 1)
    k8 = torch.zeros(NB, B, Hkv, D, dtype=torch.uint8)
    pkv.reshape_and_cache_fp8(k, v, k8, k8, sm, 0.5, 2.0)
    name, a = mock.last()
    assert name == "pkv_reshape_and_cache_fp8"
    assert (a["num_tokens"], a["num_kv_heads"], a["head_dim"], a["block_size"], a["num_blocks"], a["src_dtype"],
            a["k_scale"], a["v_scale"]) == (T, Hkv, D, B, NB, 1, 0.5, 2.0)
    pairs = torch.zeros(3, 2, dtype=torch.int64)
    pkv.copy_blocks([kc, kc], [vc, vc], pairs)
    name, a = mock.last()
    assert name == "pkv_copy_blocks"
    assert (a["num_layers"], a["num_pairs"], a["block_bytes"], a["num_blocks"], a["src_dst_pairs"]) == (
        2, 3, B * Hkv * D * 2, NB, pairs.data_ptr())


def test_size_queries_arguments(mock):
    assert pkv.decode_workspace_size(3, 8, 64, 100, 32) == 0
    name, a = mock.last()
    assert name == "pkv_decode_workspace_size" and a == {"num_seqs": 3, "num_q_heads": 8, "head_dim": 64,
                                                         "max_context_len": 100, "partition_size": 32}
    pkv.decode_partition_size(3, 8, 2, 64, 16, 100, torch.float16, total_context_tokens=250)
    name, a = mock.last()
    assert name == "pkv_decode_partition_size" and a == {
        "num_seqs": 3, "num_q_heads": 8, "num_kv_heads": 2, "head_dim": 64, "block_size": 16,
        "max_context_len": 100, "total_context_tokens": 250, "dtype": 1}
    pkv.decode_multi_partition_size(4, 2, 16, 300)
    name, a = mock.last()
    assert name == "pkv_decode_multi_partition_size" and a == {"num_chunks": 4, "num_kv_heads": 2,
                                                               "block_size": 16, "max_seq_len": 300}
    pkv.prefill_fp8_workspace_size(2, 6, 16, 2, 128, 9, 8, torch.bfloat16)
    name, a = mock.last()
    assert name == "pkv_prefill_fp8_workspace_size" and a == {
        "num_chunks": 2, "max_blocks_per_seq": 6, "block_size": 16, "num_kv_heads": 2, "head_dim": 128,
        "total_q_tokens": 9, "num_q_heads": 8, "dtype": 2}


def test_decode_step_arguments(mock):
    S, Hq, Hkv, D, B, NB, MB = 5, 8, 8, 128, 16, 23, 4
    q = torch.zeros(S, Hq, D, dtype=torch.float16)
    out = torch.zeros_like(q)
    kc, vc = torch.zeros(NB, B, Hkv, D, dtype=torch.float16), torch.zeros(NB, B, Hkv, D, dtype=torch.float16)
    bt, cl = torch.zeros(S, MB, dtype=torch.int32), torch.zeros(S, dtype=torch.int32)
    kn, vn = torch.zeros(S, Hkv, D, dtype=torch.float16), torch.zeros(S, Hkv, D, dtype=torch.float16)
    sm = torch.zeros(S, dtype=torch.int64)
    pkv.paged_attention_decode_step(kn, vn, sm, out, q, kc, vc, bt, cl, 0.4, 60, partition_size=0, stream=9)
    name, a = mock.last()
    assert name == "pkv_paged_attention_decode_step"
    assert a == {"new_keys": kn.data_ptr(), "new_values": vn.data_ptr(), "slot_mapping": sm.data_ptr(),
                 "num_new_tokens": S, "out": out.data_ptr(), "query": q.data_ptr(), "key_cache": kc.data_ptr(),
                 "value_cache": vc.data_ptr(), "block_tables": bt.data_ptr(), "context_lens": cl.data_ptr(),
                 "scale": f32(0.4), "num_seqs": S, "num_q_heads": Hq, "num_kv_heads": Hkv, "head_dim": D,
                 "block_size": B, "max_blocks_per_seq": MB, "num_blocks": NB, "max_context_len": 60,
                 "partition_size": 0, "dtype": 1, "workspace": 0, "workspace_bytes": 0, "stream": 9}
    kc8, vc8 = torch.zeros(NB, B, Hkv, D, dtype=torch.uint8), torch.zeros(NB, B, Hkv, D, dtype=torch.uint8)
    pkv.paged_attention_decode_step_fp8(kn, vn, sm, out, q, kc8, vc8, bt, cl, 0.4, 0.5, 0.25, 60, partition_size=0)
    name, a = mock.last()
    assert name == "pkv_paged_attention_decode_step_fp8"
    assert (a["k_scale"], a["v_scale"], a["key_cache"], a["value_cache"], a["num_new_tokens"], a["dtype"]) == (
        0.5, 0.25, kc8.data_ptr(), vc8.data_ptr(), S, 1)
    pkv.set_wait_limit_ns(1234)
    name, a = mock.last()
    assert name == "pkv_set_wait_limit_ns" and a == {"limit_ns": 1234}
