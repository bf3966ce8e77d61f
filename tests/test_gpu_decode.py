"""Decode attention (and the append before it) on the GPU against the CPU oracle."""
import numpy as np
import pytest
import torch

import paged_kv_cache_409_b200 as pkv
from paged_kv_cache_409_b200 import workloads
from parity_helpers import assert_close, bits, gpu_decode_step, gpu_tables, oracle_decode_step, to_device

pytestmark = pytest.mark.gpu

DT = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


def ragged_lens(B):
    # single token, block edges, a ragged tail, several partitions
    return [1, B - 1, B, B + 1, 3 * B + 5, 37, 300]


CASES = []
for dt in ("f32", "f16", "bf16"):
    for D in (64, 128):
        for B in (8, 16, 32):
            for G in (1, 8) if (D + B) % 3 else (2, 4):
                CASES.append((dt, D, B, G))


@pytest.mark.parametrize("dt,D,B,G", CASES)
def test_decode_matches_oracle(dt, D, B, G):
    w = workloads.decode_workload("sweep", ragged_lens(B), 2 * G, 2, D, B, DT[dt], seed=D * 131 + B * 7 + G,
                                  poison=True)
    pre_k, pre_v = w.key_caches[0].clone(), w.value_caches[0].clone()
    ref, k_after, v_after, used = oracle_decode_step(w, pre_k=pre_k, pre_v=pre_v)
    to_device(w)
    for part in (0, B, 4 * B):
        kc0, vc0 = pre_k.cuda(), pre_v.cuda()
        w.key_caches[0], w.value_caches[0] = kc0, vc0
        out = gpu_decode_step(w, partition_size=part)
        torch.cuda.synchronize()
        assert pkv.get_device_error() == 0
        assert_close(out, ref, DT[dt], f"{dt} D{D} B{B} G{G} partition {part}")
    # the append is bit-exact on the blocks in use
    got_k = w.key_caches[0][torch.from_numpy(used).cuda()]
    got_v = w.value_caches[0][torch.from_numpy(used).cuda()]
    assert np.array_equal(bits(got_k), k_after.view(bits(got_k).dtype))
    assert np.array_equal(bits(got_v), v_after.view(bits(got_v).dtype))


def test_tiny_decode_f32_config():
    """4 sequences, context {1,17,33,100}, 4 heads, d 64, block 16, 32-block pool, fp32: max-abs 1e-5."""
    w = workloads.tiny_decode_f32()
    ref, _, _, _ = oracle_decode_step(w)
    to_device(w)
    out = gpu_decode_step(w)
    err = assert_close(out, ref, torch.float32, "tiny fp32")
    assert err <= 1e-5


def test_one_token_context_returns_v_exactly_fp32():
    w = workloads.decode_workload("one", [1, 1, 1], 4, 4, 64, 16, torch.float32, seed=5)
    to_device(w)
    out = gpu_decode_step(w)
    # the appended token is the only key: output == its V row, bit for bit
    exp = w.new_values[0].repeat_interleave(1, dim=1)
    assert torch.equal(out, exp)


def test_zero_context_gives_zeros():
    w = workloads.decode_workload("z", [3, 5], 4, 2, 128, 16, torch.float16, seed=6)
    to_device(w)
    bt, cl, _ = gpu_tables(w)
    cl.zero_()
    out = torch.full_like(w.queries[0], 7.0)
    pkv.paged_attention_decode(out, w.queries[0], w.key_caches[0], w.value_caches[0], bt, cl, w.scale, 5)
    assert torch.count_nonzero(out) == 0


def test_placement_permutation_is_bit_identical():
    """Moving physical blocks and rewriting tables changes no bit of the output."""
    w = workloads.decode_workload("perm", [50, 333, 17, 1024], 16, 2, 128, 16, torch.bfloat16, seed=7)
    to_device(w)
    bt, cl, sm = gpu_tables(w)
    pkv.reshape_and_cache(w.new_keys[0], w.new_values[0], w.key_caches[0], w.value_caches[0], sm)
    out1 = torch.empty_like(w.queries[0])
    pkv.paged_attention_decode(out1, w.queries[0], w.key_caches[0], w.value_caches[0], bt, cl, w.scale,
                               w.max_context_len, partition_size=256)
    perm = torch.randperm(w.num_blocks, generator=torch.Generator().manual_seed(1)).cuda()
    kc2, vc2 = torch.empty_like(w.key_caches[0]), torch.empty_like(w.value_caches[0])
    kc2[perm] = w.key_caches[0]
    vc2[perm] = w.value_caches[0]
    bt2 = torch.where(bt >= 0, perm[bt.clamp(min=0).long()].int(), bt)
    out2 = torch.empty_like(out1)
    pkv.paged_attention_decode(out2, w.queries[0], kc2, vc2, bt2, cl, w.scale, w.max_context_len,
                               partition_size=256)
    assert torch.equal(out1, out2)


def test_split_k_partitions_agree():
    w = workloads.decode_workload("split", [4000, 2500, 129], 8, 8, 128, 16, torch.float16, seed=8)
    ref, _, _, _ = oracle_decode_step(w)
    to_device(w)
    bt, cl, sm = gpu_tables(w)
    pkv.reshape_and_cache(w.new_keys[0], w.new_values[0], w.key_caches[0], w.value_caches[0], sm)
    outs = []
    for part in (0, 16, 64, 256, 4096):
        out = torch.empty_like(w.queries[0])
        pkv.paged_attention_decode(out, w.queries[0], w.key_caches[0], w.value_caches[0], bt, cl, w.scale,
                                   w.max_context_len, partition_size=part)
        assert_close(out, ref, torch.float16, f"partition {part}")
        outs.append(out.float())
    for o in outs[1:]:
        assert (o - outs[0]).abs().max().item() < 2e-3


def test_empty_batch_is_a_no_op():
    kc = torch.zeros(4, 16, 2, 64, dtype=torch.float16, device="cuda")
    q = torch.zeros(0, 2, 64, dtype=torch.float16, device="cuda")
    bt = torch.zeros(0, 1, dtype=torch.int32, device="cuda")
    cl = torch.zeros(0, dtype=torch.int32, device="cuda")
    pkv.paged_attention_decode(torch.empty_like(q), q, kc, kc, bt, cl, 0.1, 0)
    torch.cuda.synchronize()
