"""Multi-token decode (speculative verification): every sequence appends a few
draft tokens and each of them attends causally over the whole cache.  Both
calls that compute it are checked: the chunked-prefill call and the multi-token
decode call (keys on the M side of the tcgen05 MMAs, persistent CTAs, split-K
partitions merged by a second kernel)."""
import numpy as np
import pytest
import torch

import paged_kv_cache_409_b200 as pkv
from paged_kv_cache_409_b200 import workloads
from parity_helpers import assert_close, oracle_prefill_chunks

pytestmark = pytest.mark.gpu


def run_gpu(m, dev="cuda", call="prefill", partition_size=None):
    """Append every draft token, then the causal attention of all of them."""
    kc, vc = m.decode.key_caches[0].to(dev), m.decode.value_caches[0].to(dev)
    pkv.reshape_and_cache(m.append_keys.to(dev), m.append_values.to(dev), kc, vc,
                          torch.from_numpy(m.append_slots).to(dev))
    out = torch.empty_like(m.chunk_query, device=dev)
    args = (out, m.chunk_query.to(dev), kc, vc, torch.from_numpy(m.chunk_tables).to(dev),
            torch.from_numpy(m.seq_lens).to(dev), torch.from_numpy(m.query_start_loc).to(dev),
            int(m.chunk_lens.max()))
    if call == "prefill":
        pkv.paged_attention_prefill_chunk(*args, m.decode.scale)
    else:
        pkv.paged_attention_decode_multi(*args, int(m.seq_lens.max()), m.decode.scale, partition_size=partition_size)
    return out, kc, vc


CASES = [
    # dtype, D, B, Hq, Hkv, c0s, ns
    (torch.bfloat16, 128, 32, 32, 8, [0, 31, 32, 1000, 4093], [2, 3, 6, 5, 4]),
    (torch.float16, 128, 16, 8, 2, [15, 16, 17, 700], [6, 6, 2, 3]),
    (torch.bfloat16, 64, 8, 16, 16, [1, 63, 300], [2, 4, 6]),
    (torch.float16, 64, 32, 8, 1, [129, 2048], [4, 2]),
]


@pytest.mark.parametrize("call", ["prefill", "multi"])
@pytest.mark.parametrize("case", CASES, ids=[f"case{i}" for i in range(len(CASES))])
def test_multi_token_matches_oracle(case, call):
    dtype, D, B, Hq, Hkv, c0s, ns = case
    m = workloads.mixed_workload("mt", [], c0s, ns, Hq, Hkv, D, B, dtype, seed=7 + sum(c0s) + D, poison=True)
    pre_k, pre_v = m.decode.key_caches[0].clone(), m.decode.value_caches[0].clone()
    ref = oracle_prefill_chunks(m, pre_k, pre_v)
    parts = [None] if call == "prefill" else [0, B, 4 * B, None]
    for part in parts:
        out, _, _ = run_gpu(m, call=call, partition_size=part)
        torch.cuda.synchronize()
        assert pkv.get_device_error() == 0
        assert_close(out, ref, dtype, f"multi-token {call} {case} partition {part}")


# up to 32 rows per KV head (n * G): G 4 and 8 with long drafts, and one head per KV head with 16-token drafts
ROW_CASES = [
    (torch.bfloat16, 128, 16, 32, 8, [40, 1000, 3], [8, 5, 7]),
    (torch.float16, 64, 32, 16, 16, [100, 31], [16, 9]),
    (torch.bfloat16, 128, 8, 64, 8, [77, 500], [4, 3]),
]


@pytest.mark.parametrize("case", ROW_CASES, ids=[f"rows{i}" for i in range(len(ROW_CASES))])
def test_multi_token_row_groups(case):
    dtype, D, B, Hq, Hkv, c0s, ns = case
    m = workloads.mixed_workload("mtr", [], c0s, ns, Hq, Hkv, D, B, dtype, seed=3 + sum(ns), poison=True)
    pre_k, pre_v = m.decode.key_caches[0].clone(), m.decode.value_caches[0].clone()
    ref = oracle_prefill_chunks(m, pre_k, pre_v)
    for part in (0, 2 * B):
        out, _, _ = run_gpu(m, call="multi", partition_size=part)
        torch.cuda.synchronize()
        assert pkv.get_device_error() == 0
        assert_close(out, ref, dtype, f"multi-token rows {case} partition {part}")


def test_multi_token_many_chunks_and_partitions():
    """More chunks than the longest-first schedule takes (partition-major item
    order), and partitions of one, two and three 128-key tiles and of a
    size that leaves a partial tile at every partition end."""
    R = 150
    rng = np.random.default_rng(11)
    c0s = rng.integers(0, 700, size=R).tolist()
    ns = rng.integers(1, 9, size=R).tolist()
    m = workloads.mixed_workload("mtm", [], c0s, ns, 16, 4, 128, 16, torch.float16, seed=12, poison=True)
    pre_k, pre_v = m.decode.key_caches[0].clone(), m.decode.value_caches[0].clone()
    ref = oracle_prefill_chunks(m, pre_k, pre_v)
    for part in (None, 0, 128, 256, 384, 80):
        out, _, _ = run_gpu(m, call="multi", partition_size=part)
        torch.cuda.synchronize()
        assert pkv.get_device_error() == 0
        assert_close(out, ref, torch.float16, f"{R} chunks, partition {part}")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_multi_token_rescales_mid_partition(dtype):
    """Queries scaled up 24x: scores spread over tens of units in the log2
    domain, so a row's running maximum keeps growing by more than 2^8 after
    the first key tile and the accumulated O is rescaled in tensor memory."""
    m = workloads.mixed_workload("mts", [], [900, 2500, 130, 1700], [4, 2, 6, 3], 32, 8, 128, 32, dtype, seed=21,
                                 poison=True)
    m.chunk_query.mul_(24.0)
    pre_k, pre_v = m.decode.key_caches[0].clone(), m.decode.value_caches[0].clone()
    ref = oracle_prefill_chunks(m, pre_k, pre_v)
    for part in (0, 512, None):
        out, _, _ = run_gpu(m, call="multi", partition_size=part)
        torch.cuda.synchronize()
        assert pkv.get_device_error() == 0
        assert_close(out, ref, dtype, f"large scores, partition {part}")


@pytest.mark.parametrize("case", [CASES[0], CASES[3], ROW_CASES[0]], ids=["case0", "case3", "rows0"])
def test_multi_token_step_call(case):
    """The one-call step (append, then the attention launched as its programmatic
    dependent) writes the same pools and the same rows as the two calls, and
    matches the oracle, with and without partitions."""
    dtype, D, B, Hq, Hkv, c0s, ns = case
    m = workloads.mixed_workload("mtst", [], c0s, ns, Hq, Hkv, D, B, dtype, seed=31 + sum(ns), poison=True)
    pre_k, pre_v = m.decode.key_caches[0].clone(), m.decode.value_caches[0].clone()
    ref = oracle_prefill_chunks(m, pre_k, pre_v)
    dev = "cuda"
    for part in (0, 2 * B):
        two, k2, v2 = run_gpu(m, call="multi", partition_size=part)
        kc, vc = pre_k.to(dev), pre_v.to(dev)
        one = torch.empty_like(m.chunk_query, device=dev)
        pkv.paged_attention_decode_multi_step(
            m.append_keys.to(dev), m.append_values.to(dev), torch.from_numpy(m.append_slots).to(dev), one,
            m.chunk_query.to(dev), kc, vc, torch.from_numpy(m.chunk_tables).to(dev),
            torch.from_numpy(m.seq_lens).to(dev), torch.from_numpy(m.query_start_loc).to(dev),
            int(m.chunk_lens.max()), int(m.seq_lens.max()), m.decode.scale, partition_size=part)
        torch.cuda.synchronize()
        assert pkv.get_device_error() == 0
        # bit patterns: the poisoned free slots hold NaNs
        assert torch.equal(kc.view(torch.int16), k2.view(torch.int16))
        assert torch.equal(vc.view(torch.int16), v2.view(torch.int16))
        assert torch.equal(one.view(torch.int16), two.view(torch.int16)), \
            f"step call differs from the two calls, partition {part}"
        assert_close(one, ref, dtype, f"multi-token step call {case} partition {part}")


def test_multi_token_step_refused_changes_nothing():
    """A step the attention call refuses (9 tokens x 4 heads = 36 rows per KV head) returns before the
    append: the pools keep their bytes."""
    dev = "cuda"
    q = torch.zeros(9, 32, 128, device=dev, dtype=torch.float16)
    kc = torch.zeros(4, 16, 8, 128, device=dev, dtype=torch.float16)
    vc = torch.zeros_like(kc)
    nk = torch.ones(9, 8, 128, device=dev, dtype=torch.float16)
    slots = torch.arange(9, dtype=torch.int64, device=dev)
    bt = torch.zeros(1, 4, dtype=torch.int32, device=dev)
    sl = torch.tensor([20], dtype=torch.int32, device=dev)
    qsl = torch.tensor([0, 9], dtype=torch.int32, device=dev)
    with pytest.raises(pkv.PagedKVError) as e:
        pkv.paged_attention_decode_multi_step(nk, nk, slots, torch.empty_like(q), q, kc, vc, bt, sl, qsl, 9, 20, 0.1)
    assert e.value.status == -2
    torch.cuda.synchronize()
    assert not kc.any() and not vc.any()


def test_multi_token_step_without_new_tokens_is_the_attention_call():
    """No draft rows to append: the step is the attention call alone (launched without the dependency)."""
    dtype, D, B, Hq, Hkv, c0s, ns = CASES[1]
    m = workloads.mixed_workload("mt0", [], c0s, ns, Hq, Hkv, D, B, dtype, seed=41, poison=True)
    dev = "cuda"
    two, kc, vc = run_gpu(m, call="multi", partition_size=0)  # appends, then attends
    one = torch.empty_like(two)
    empty_kv = torch.empty(0, Hkv, D, dtype=dtype, device=dev)
    pkv.paged_attention_decode_multi_step(
        empty_kv, empty_kv, torch.empty(0, dtype=torch.int64, device=dev), one, m.chunk_query.to(dev), kc, vc,
        torch.from_numpy(m.chunk_tables).to(dev), torch.from_numpy(m.seq_lens).to(dev),
        torch.from_numpy(m.query_start_loc).to(dev), int(m.chunk_lens.max()), int(m.seq_lens.max()),
        m.decode.scale, partition_size=0)
    torch.cuda.synchronize()
    assert pkv.get_device_error() == 0
    assert torch.equal(one.view(torch.int16), two.view(torch.int16))


def test_multi_token_call_rejects_too_many_rows():
    q = torch.zeros(9, 32, 128, device="cuda", dtype=torch.float16)  # 9 tokens x G 4 = 36 rows > 32
    kc = torch.zeros(4, 16, 8, 128, device="cuda", dtype=torch.float16)
    bt = torch.zeros(1, 4, dtype=torch.int32, device="cuda")
    sl = torch.tensor([20], dtype=torch.int32, device="cuda")
    qsl = torch.tensor([0, 9], dtype=torch.int32, device="cuda")
    with pytest.raises(pkv.PagedKVError) as e:
        pkv.paged_attention_decode_multi(torch.empty_like(q), q, kc, kc, bt, sl, qsl, 9, 20, 0.1)
    assert e.value.status == -2


@pytest.mark.parametrize("call", ["prefill", "multi"])
def test_multi_token_full_size_sampled(call):
    """The 64-sequence bf16 batch (drafts of 2..6 tokens, contexts 256..4096) in the
    launch configuration the benchmark times: every row of six sampled sequences
    against the oracle."""
    m = workloads.multi_token_decode_bf16(poison=True)
    pre_k, pre_v = m.decode.key_caches[0].clone(), m.decode.value_caches[0].clone()
    out, _, _ = run_gpu(m, call=call)
    torch.cuda.synchronize()
    assert pkv.get_device_error() == 0
    chunks = np.array([0, 9, 21, 40, 52, 63])
    ref = oracle_prefill_chunks(m, pre_k, pre_v, chunks)
    qsl = m.query_start_loc
    rows = np.concatenate([np.arange(qsl[r], qsl[r + 1]) for r in chunks])
    assert_close(out[torch.from_numpy(rows).cuda()], ref, torch.bfloat16, f"multi-token 64 sequences ({call})")


@pytest.mark.parametrize("call", ["prefill", "multi"])
def test_multi_token_rows_equal_single_token_decode(call):
    """Draft token i of a sequence sees exactly the first c0 + i + 1 tokens:
    its row equals the one-token decode over that prefix (every row of the
    full-size batch, against the single-token decode path)."""
    m = workloads.multi_token_decode_bf16()
    out, kc, vc = run_gpu(m, call=call)
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
