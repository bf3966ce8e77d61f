"""Decode through the entry point that allocates nothing.

Callers that cannot allocate device memory at the call site (inside another
framework's allocator, a plugin handed only one operation's tensors, a serving
loop that must not touch the allocator between steps) use
``pkv_paged_attention_decode_static_scratch``: the split-K scratch is the
library's own device array instead of a caller workspace.  This test calls it
through the C ABI and checks it against ``pkv_paged_attention_decode`` with an
ordinary workspace and against the CPU oracle, on two calls in a row with
different inputs, checks that an oversized request is refused, and that a bad
argument gets the status the workspace entry point gives.  The file is named
to run last.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_409_b200 as pkv
from paged_kv_cache_409_b200 import workloads
from parity_helpers import TOL, assert_close, gpu_tables, to_device

pytestmark = pytest.mark.gpu

EINVAL, EWORKSPACE = -1, -5
SCRATCH_BYTES = 32 << 20


def _entry():
    lib = pkv.load_library()
    f = lib.pkv_paged_attention_decode_static_scratch
    P, I, I64, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float
    f.argtypes = [P, P, P, P, P, P, F, I, I, I, I, I, I, I64, I, I, I, P]
    f.restype = I
    return f


def _call(f, out, w, q, bt, cl, part):
    return f(out.data_ptr(), q.data_ptr(), w.key_caches[0].data_ptr(), w.value_caches[0].data_ptr(),
             bt.data_ptr(), cl.data_ptr(), w.scale, w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim,
             w.block_size, bt.shape[1], w.num_blocks, w.max_context_len, part,
             pkv._binding.DTYPE_CODE[q.dtype], torch.cuda.current_stream().cuda_stream)


def _close(a, b, dtype):
    atol, rtol = TOL[dtype]
    x, y = a.double(), b.double()
    assert torch.isfinite(x).all()
    assert ((x - y).abs() <= atol + rtol * y.abs()).all()


@pytest.mark.parametrize("dtype,Hq,Hkv", [(torch.float16, 8, 8), (torch.bfloat16, 16, 2)])
def test_static_scratch_matches_workspace_decode_twice(dtype, Hq, Hkv):
    f = _entry()
    w = workloads.decode_workload("ns", [700, 1, 129, 2000, 64, 1500], Hq, Hkv, 128, 16, dtype, seed=31)
    kn, code = oracle.storage(w.key_caches[0].clone())  # host snapshots for the oracle, before any GPU work
    vn, _ = oracle.storage(w.value_caches[0].clone())
    w = to_device(w)
    bt, cl, _ = gpu_tables(w)
    part = 256  # several partitions per sequence: the scratch is used
    assert 0 < pkv.decode_workspace_size(w.num_seqs, Hq, 128, w.max_context_len, part) <= SCRATCH_BYTES
    g = torch.Generator(device="cuda").manual_seed(5)
    for call in range(2):  # the second call reuses the scratch the first one left behind
        q = torch.randn(w.queries[0].shape, generator=g, device="cuda").to(dtype)
        ref = torch.empty_like(q)
        pkv.paged_attention_decode(ref, q, w.key_caches[0], w.value_caches[0], bt, cl, w.scale, w.max_context_len,
                                   partition_size=part)
        out = torch.full_like(q, float("nan"))
        qh = q.cpu()
        assert _call(f, out, w, q, bt, cl, part) == 0, f"call {call}"
        torch.cuda.synchronize()
        _close(out, ref, dtype)
        want = oracle.get().paged_attention_decode(oracle.storage(qh)[0], kn, vn, w.block_tables, w.context_lens,
                                                   w.scale, code)
        assert_close(out, want, dtype, f"static-scratch call {call} vs oracle")
    assert pkv.get_device_error() == 0


def test_static_scratch_refuses_oversized_request():
    f = _entry()
    w = to_device(workloads.decode_workload("big", [4096] * 4, 64, 8, 128, 16, torch.bfloat16, seed=32))
    bt, cl, _ = gpu_tables(w)
    # 512 sequences x 64 heads x 256 partitions would need far more than the array holds
    big = torch.empty(512, 64, 128, dtype=torch.bfloat16, device="cuda")
    need = pkv.decode_workspace_size(512, 64, 128, 4096, 16)
    assert need > SCRATCH_BYTES
    rc = f(big.data_ptr(), big.data_ptr(), w.key_caches[0].data_ptr(), w.value_caches[0].data_ptr(), bt.data_ptr(),
           cl.data_ptr(), w.scale, 512, 64, 8, 128, 16, bt.shape[1], w.num_blocks, 4096, 16, 2,
           torch.cuda.current_stream().cuda_stream)
    assert rc == EWORKSPACE
    # no split needs no scratch at all
    out = torch.empty_like(w.queries[0])
    assert _call(f, out, w, w.queries[0], bt, cl, 0) == 0
    ref = torch.empty_like(out)
    pkv.paged_attention_decode(ref, w.queries[0], w.key_caches[0], w.value_caches[0], bt, cl, w.scale,
                               w.max_context_len, partition_size=0)
    torch.cuda.synchronize()
    _close(out, ref, torch.bfloat16)


def test_static_scratch_bad_argument_gets_the_workspace_calls_status():
    """A partition_size that is not a multiple of block_size is an invalid argument for both decode entry
    points, even when the request would also be too large for the library's array."""
    f = _entry()
    lib = pkv.load_library()
    g = lib.pkv_paged_attention_decode
    w = to_device(workloads.decode_workload("bad", [64] * 2, 64, 8, 128, 16, torch.bfloat16, seed=33))
    bt, cl, _ = gpu_tables(w)
    big = torch.empty(512, 64, 128, dtype=torch.bfloat16, device="cuda")
    args = (big.data_ptr(), big.data_ptr(), w.key_caches[0].data_ptr(), w.value_caches[0].data_ptr(),
            bt.data_ptr(), cl.data_ptr(), w.scale, 512, 64, 8, 128, 16, bt.shape[1], w.num_blocks, 4096, 24, 2)
    assert pkv.decode_workspace_size(512, 64, 128, 4096, 24) > SCRATCH_BYTES
    stream = torch.cuda.current_stream().cuda_stream
    assert g(*args, None, 0, stream) == EINVAL
    assert f(*args, stream) == EINVAL
