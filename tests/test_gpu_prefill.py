"""Chunked prefill on the tcgen05 path against the CPU oracle."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_409_b200 as pkv
from paged_kv_cache_409_b200 import workloads
from parity_helpers import assert_close, compact_tables, snapshot_blocks

pytestmark = pytest.mark.gpu


def run_prefill(m, row_select=None):
    """Append every chunk token, then prefill; returns (gpu out, oracle out)."""
    dec = m.decode
    kc, vc = dec.key_caches[0], dec.value_caches[0]
    pre_k, pre_v = kc.clone(), vc.clone()
    dev = "cuda"
    S = dec.num_seqs
    ck, cv = m.append_keys[S:], m.append_values[S:]
    cslots = m.append_slots[S:]
    kd, vd = pre_k.to(dev), pre_v.to(dev)
    pkv.reshape_and_cache(ck.to(dev), cv.to(dev), kd, vd, torch.from_numpy(cslots).to(dev))
    out = torch.empty_like(m.chunk_query, device=dev)
    pkv.paged_attention_prefill_chunk(out, m.chunk_query.to(dev), kd, vd, torch.from_numpy(m.chunk_tables).to(dev),
                                      torch.from_numpy(m.seq_lens).to(dev),
                                      torch.from_numpy(m.query_start_loc).to(dev), int(m.chunk_lens.max()),
                                      dec.scale)
    torch.cuda.synchronize()
    assert pkv.get_device_error() == 0
    # oracle on host snapshots
    used, bt = compact_tables(m.chunk_tables, m.seq_lens, dec.block_size)
    kn, code = oracle.storage(snapshot_blocks(pre_k, used))
    vn, _ = oracle.storage(snapshot_blocks(pre_v, used))
    kn, vn = kn.copy(), vn.copy()
    B = dec.block_size
    remap = {int(b): i for i, b in enumerate(used)}
    slots = np.array([remap[int(s) // B] * B + int(s) % B for s in cslots], dtype=np.int64)
    orc = oracle.get()
    orc.reshape_and_cache(oracle.storage(ck)[0], oracle.storage(cv)[0], kn, vn, slots, code)
    ref = orc.paged_attention_prefill_chunk(oracle.storage(m.chunk_query)[0], kn, vn, bt, m.seq_lens,
                                            m.query_start_loc, dec.scale, code, row_select=row_select)
    return out, ref


CASES = [
    # dtype, D, B, Hq, Hkv, c0s, ns
    (torch.bfloat16, 128, 32, 32, 8, [0, 300], [512, 77]),
    (torch.float16, 128, 16, 8, 8, [5, 0, 129], [1, 130, 128]),
    (torch.bfloat16, 64, 8, 16, 2, [1000, 0], [33, 257]),
    (torch.float16, 64, 16, 4, 2, [17], [300]),
    (torch.bfloat16, 128, 16, 16, 2, [255, 64], [200, 16]),
    (torch.float16, 128, 32, 8, 4, [0], [1]),
    # the first tile of a pair needs one key tile fewer than the second (c0 = 90: rows up to 121 and 153)
    (torch.bfloat16, 128, 32, 32, 8, [90, 7], [64, 100]),
    # more chunks than the longest-first ordering handles: the plain launch order
    (torch.float16, 64, 16, 8, 1, [7 * i for i in range(70)], [1 + i % 3 for i in range(70)]),
    # chunks of equal length (ties in the longest-first order)
    (torch.bfloat16, 128, 16, 16, 4, [200, 200, 200], [40, 40, 40]),
]


@pytest.mark.parametrize("case", CASES, ids=[f"case{i}" for i in range(len(CASES))])
def test_prefill_matches_oracle(case):
    dtype, D, B, Hq, Hkv, c0s, ns = case
    m = workloads.mixed_workload("p", [], c0s, ns, Hq, Hkv, D, B, dtype, seed=sum(c0s) + sum(ns) + D + B,
                                 poison=True)
    out, ref = run_prefill(m)
    assert_close(out, ref, dtype, f"prefill {case}")


def test_prefill_row_equals_decode_of_prefix():
    """A chunk from position 0: row i equals decode over the first i + 1 tokens (tensor-core vs CUDA-core path)."""
    n, Hq, Hkv, D, B = 200, 8, 2, 128, 16
    m = workloads.mixed_workload("x", [], [0], [n], Hq, Hkv, D, B, torch.bfloat16, seed=9)
    dev = "cuda"
    kc, vc = m.decode.key_caches[0].to(dev), m.decode.value_caches[0].to(dev)
    pkv.reshape_and_cache(m.append_keys.to(dev), m.append_values.to(dev), kc, vc,
                          torch.from_numpy(m.append_slots).to(dev))
    q = m.chunk_query.to(dev)
    bt = torch.from_numpy(m.chunk_tables).to(dev)
    out = torch.empty_like(q)
    pkv.paged_attention_prefill_chunk(out, q, kc, vc, bt, torch.from_numpy(m.seq_lens).to(dev),
                                      torch.from_numpy(m.query_start_loc).to(dev), n, m.decode.scale)
    dec = torch.empty_like(q)
    lens = torch.arange(1, n + 1, dtype=torch.int32, device=dev)
    pkv.paged_attention_decode(dec, q, kc, vc, bt.expand(n, -1).contiguous(), lens, m.decode.scale, n,
                               partition_size=0)
    diff = (out.float() - dec.float()).abs()
    assert diff.max().item() < 2e-3 + 1e-2 * dec.float().abs().max().item()


def test_prefill_rejects_fp32():
    q = torch.zeros(4, 2, 64, device="cuda")
    kc = torch.zeros(2, 16, 2, 64, device="cuda")
    i32 = torch.zeros(2, dtype=torch.int32, device="cuda")
    with pytest.raises(pkv.PagedKVError) as e:
        pkv.paged_attention_prefill_chunk(torch.empty_like(q), q, kc, kc, i32.view(1, 2), i32[:1] + 4,
                                          torch.tensor([0, 4], dtype=torch.int32, device="cuda"), 4, 0.1)
    assert e.value.status == -2
