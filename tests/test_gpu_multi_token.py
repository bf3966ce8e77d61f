"""Multi-token decode (speculative verification): every sequence appends a few
draft tokens and each of them attends causally over the whole cache -- the
chunked-prefill call with short chunks over long prior contexts."""
import numpy as np
import pytest
import torch

import paged_kv_cache_409_b200 as pkv
from paged_kv_cache_409_b200 import workloads
from parity_helpers import assert_close, oracle_prefill_chunks

pytestmark = pytest.mark.gpu


def run_gpu(m, dev="cuda"):
    """Append every draft token, then the causal attention of all of them."""
    kc, vc = m.decode.key_caches[0].to(dev), m.decode.value_caches[0].to(dev)
    pkv.reshape_and_cache(m.append_keys.to(dev), m.append_values.to(dev), kc, vc,
                          torch.from_numpy(m.append_slots).to(dev))
    out = torch.empty_like(m.chunk_query, device=dev)
    pkv.paged_attention_prefill_chunk(out, m.chunk_query.to(dev), kc, vc, torch.from_numpy(m.chunk_tables).to(dev),
                                      torch.from_numpy(m.seq_lens).to(dev),
                                      torch.from_numpy(m.query_start_loc).to(dev), int(m.chunk_lens.max()),
                                      m.decode.scale)
    return out, kc, vc


CASES = [
    # dtype, D, B, Hq, Hkv, c0s, ns
    (torch.bfloat16, 128, 32, 32, 8, [0, 31, 32, 1000, 4093], [2, 3, 6, 5, 4]),
    (torch.float16, 128, 16, 8, 2, [15, 16, 17, 700], [6, 6, 2, 3]),
    (torch.bfloat16, 64, 8, 16, 16, [1, 63, 300], [2, 4, 6]),
    (torch.float16, 64, 32, 8, 1, [129, 2048], [5, 2]),
]


@pytest.mark.parametrize("case", CASES, ids=[f"case{i}" for i in range(len(CASES))])
def test_multi_token_matches_oracle(case):
    dtype, D, B, Hq, Hkv, c0s, ns = case
    m = workloads.mixed_workload("mt", [], c0s, ns, Hq, Hkv, D, B, dtype, seed=7 + sum(c0s) + D, poison=True)
    pre_k, pre_v = m.decode.key_caches[0].clone(), m.decode.value_caches[0].clone()
    out, _, _ = run_gpu(m)
    torch.cuda.synchronize()
    assert pkv.get_device_error() == 0
    ref = oracle_prefill_chunks(m, pre_k, pre_v)
    assert_close(out, ref, dtype, f"multi-token {case}")


def test_multi_token_full_size_sampled():
    """The 64-sequence bf16 batch (drafts of 2..6 tokens, contexts 256..4096):
    every row of six sampled sequences against the oracle."""
    m = workloads.multi_token_decode_bf16(poison=True)
    pre_k, pre_v = m.decode.key_caches[0].clone(), m.decode.value_caches[0].clone()
    out, _, _ = run_gpu(m)
    torch.cuda.synchronize()
    assert pkv.get_device_error() == 0
    chunks = np.array([0, 9, 21, 40, 52, 63])
    ref = oracle_prefill_chunks(m, pre_k, pre_v, chunks)
    qsl = m.query_start_loc
    rows = np.concatenate([np.arange(qsl[r], qsl[r + 1]) for r in chunks])
    assert_close(out[torch.from_numpy(rows).cuda()], ref, torch.bfloat16, "multi-token 64 sequences")


def test_multi_token_rows_equal_single_token_decode():
    """Draft token i of a sequence sees exactly the first c0 + i + 1 tokens:
    its row equals the one-token decode over that prefix (tensor-core prefill
    path against the decode path, every row of the full-size batch)."""
    m = workloads.multi_token_decode_bf16()
    out, kc, vc = run_gpu(m)
    R = len(m.chunk_lens)
    seq = np.repeat(np.arange(R), m.chunk_lens)
    pos = np.concatenate([m.chunk_c0[r] + np.arange(m.chunk_lens[r]) for r in range(R)])
    bt = torch.from_numpy(m.chunk_tables[seq]).cuda()
    lens = torch.from_numpy((pos + 1).astype(np.int32)).cuda()
    dec = torch.empty_like(out)
    q = m.chunk_query.cuda()
    pkv.paged_attention_decode(dec, q, kc, vc, bt, lens, m.decode.scale, int(pos.max()) + 1)
    torch.cuda.synchronize()
    assert pkv.get_device_error() == 0
    d = dec.double().cpu().numpy()
    assert_close(out, d, torch.bfloat16, "prefill rows vs decode")
