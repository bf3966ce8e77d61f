"""The five named workloads at full size, in the launch configuration the benchmark times.

Small ones are compared element by element everywhere; large ones on sampled
sequences / query rows, which the oracle computes one by one.
"""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_409_b200 as pkv
from paged_kv_cache_409_b200 import workloads
from parity_helpers import (assert_close, bits, compact_tables, gpu_tables, oracle_decode_step,
                            snapshot_blocks)

pytestmark = pytest.mark.gpu


def test_llama7b_decode_f16_full():
    w = workloads.llama7b_decode_f16(device="cuda")
    pre_k, pre_v = w.key_caches[0].cpu(), w.value_caches[0].cpu()
    bt, cl, sm = gpu_tables(w)
    pkv.reshape_and_cache(w.new_keys[0], w.new_values[0], w.key_caches[0], w.value_caches[0], sm)
    out = torch.empty_like(w.queries[0])
    pkv.paged_attention_decode(out, w.queries[0], w.key_caches[0], w.value_caches[0], bt, cl, w.scale,
                               w.max_context_len)
    torch.cuda.synchronize()
    assert pkv.get_device_error() == 0
    ref, k_after, v_after, used = oracle_decode_step(w, pre_k=pre_k, pre_v=pre_v)
    assert_close(out, ref, torch.float16, "llama7b decode")
    got = w.key_caches[0][torch.from_numpy(used).cuda()]
    assert np.array_equal(bits(got), k_after.view(np.int16))


def test_gqa70b_decode_bf16_sampled_layers():
    w = workloads.gqa70b_decode_bf16(device="cuda", num_layers=2)
    S = w.num_seqs
    order = np.argsort(w.context_lens)
    sample = np.unique(np.concatenate([order[:3], order[-5:], np.arange(0, S, 37)]))
    pre = [(w.key_caches[l].cpu(), w.value_caches[l].cpu()) for l in range(2)]
    bt, cl, sm = gpu_tables(w)
    outs = []
    for l in range(2):
        pkv.reshape_and_cache(w.new_keys[l], w.new_values[l], w.key_caches[l], w.value_caches[l], sm)
        out = torch.empty_like(w.queries[l])
        pkv.paged_attention_decode(out, w.queries[l], w.key_caches[l], w.value_caches[l], bt, cl, w.scale,
                                   w.max_context_len)
        outs.append(out)
    torch.cuda.synchronize()
    assert pkv.get_device_error() == 0
    for l in range(2):
        ref, _, _, _ = oracle_decode_step(w, seqs=sample, layer=l, pre_k=pre[l][0], pre_v=pre[l][1])
        assert_close(outs[l][torch.from_numpy(sample).cuda()], ref, torch.bfloat16, f"gqa70b layer {l}")


def test_shared_prefix_cow_full():
    sp = workloads.shared_prefix_decode_f16(device="cuda", poison=True)
    st = sp.step
    kc, vc = st.key_caches[0], st.value_caches[0]
    pre_k, pre_v = kc.cpu(), vc.cpu()
    # phase A: copy-on-write of the partial shared block, then each sequence's private tokens
    pkv.copy_blocks([kc], [vc], torch.from_numpy(sp.cow_pairs).cuda())
    pkv.reshape_and_cache(sp.private_keys, sp.private_values, kc, vc, torch.from_numpy(sp.private_slots).cuda())
    # phase B: the decode step
    bt, cl, sm = gpu_tables(st)
    pkv.reshape_and_cache(st.new_keys[0], st.new_values[0], kc, vc, sm)
    out = torch.empty_like(st.queries[0])
    pkv.paged_attention_decode(out, st.queries[0], kc, vc, bt, cl, st.scale, st.max_context_len)
    torch.cuda.synchronize()
    assert pkv.get_device_error() == 0
    # oracle: the same three steps on host copies of the whole pool
    orc = oracle.get()
    kn, code = oracle.storage(pre_k)
    vn, _ = oracle.storage(pre_v)
    kn, vn = kn.copy(), vn.copy()
    orc.copy_blocks([kn], [vn], sp.cow_pairs)
    orc.reshape_and_cache(oracle.storage(sp.private_keys)[0], oracle.storage(sp.private_values)[0], kn, vn,
                          sp.private_slots, code)
    orc.reshape_and_cache(oracle.storage(st.new_keys[0])[0], oracle.storage(st.new_values[0])[0], kn, vn,
                          st.slot_mapping, code)
    assert np.array_equal(bits(kc), kn.view(np.int16))
    assert np.array_equal(bits(vc), vn.view(np.int16))
    ref = orc.paged_attention_decode(oracle.storage(st.queries[0])[0], kn, vn, st.block_tables, st.context_lens,
                                     st.scale, code)
    assert_close(out, ref, torch.float16, "shared prefix decode")


def test_mixed_step_bf16_sampled():
    m = workloads.mixed_step_bf16(device="cuda")
    dec = m.decode
    kc, vc = dec.key_caches[0], dec.value_caches[0]
    S = dec.num_seqs
    order = np.argsort(dec.context_lens)
    dsample = np.unique(np.concatenate([order[:2], order[-4:], np.arange(5, S, 29)]))
    # host snapshots of the blocks the checks read, before the step
    dused, dbt = compact_tables(dec.block_tables[dsample], dec.context_lens[dsample], dec.block_size)
    cused, cbt = compact_tables(m.chunk_tables, m.seq_lens, dec.block_size)
    dk, dv = snapshot_blocks(kc, dused), snapshot_blocks(vc, dused)
    ck, cv = snapshot_blocks(kc, cused), snapshot_blocks(vc, cused)
    # the step: append everything, prefill the chunks, decode the rest
    pkv.reshape_and_cache(m.append_keys, m.append_values, kc, vc, torch.from_numpy(m.append_slots).cuda())
    pout = torch.empty_like(m.chunk_query)
    pkv.paged_attention_prefill_chunk(pout, m.chunk_query, kc, vc, torch.from_numpy(m.chunk_tables).cuda(),
                                      torch.from_numpy(m.seq_lens).cuda(),
                                      torch.from_numpy(m.query_start_loc).cuda(), int(m.chunk_lens.max()),
                                      dec.scale)
    bt, cl, _ = gpu_tables(dec)
    dout = torch.empty_like(dec.queries[0])
    pkv.paged_attention_decode(dout, dec.queries[0], kc, vc, bt, cl, dec.scale, dec.max_context_len)
    torch.cuda.synchronize()
    assert pkv.get_device_error() == 0
    orc = oracle.get()
    B = dec.block_size
    # decode sample
    kn, code = oracle.storage(dk)
    vn, _ = oracle.storage(dv)
    kn, vn = kn.copy(), vn.copy()
    remap = {int(b): i for i, b in enumerate(dused)}
    sl = np.array([remap[int(s) // B] * B + int(s) % B for s in dec.slot_mapping[dsample]], dtype=np.int64)
    idx = torch.from_numpy(dsample).cuda()
    orc.reshape_and_cache(oracle.storage(m.append_keys[idx])[0], oracle.storage(m.append_values[idx])[0], kn, vn,
                          sl, code)
    ref = orc.paged_attention_decode(oracle.storage(dec.queries[0][idx])[0], kn, vn, dbt,
                                     dec.context_lens[dsample], dec.scale, code)
    assert_close(dout[idx], ref, torch.bfloat16, "mixed decode sample")
    # prefill sample rows: first / last rows of each chunk and around 128-row tile edges
    kn, _ = oracle.storage(ck)
    vn, _ = oracle.storage(cv)
    kn, vn = kn.copy(), vn.copy()
    remap = {int(b): i for i, b in enumerate(cused)}
    cs = m.append_slots[S:]
    sl = np.array([remap[int(s) // B] * B + int(s) % B for s in cs], dtype=np.int64)
    orc.reshape_and_cache(oracle.storage(m.append_keys[S:])[0], oracle.storage(m.append_values[S:])[0], kn, vn, sl,
                          code)
    sel = np.zeros(int(m.query_start_loc[-1]), dtype=np.uint8)
    for r in range(len(m.chunk_lens)):
        q0, n = int(m.query_start_loc[r]), int(m.chunk_lens[r])
        for i in (0, 1, 31, 32, 33, 127, 128, 255, 256, 300, n - 2, n - 1):
            if 0 <= i < n:
                sel[q0 + i] = 1
    ref = orc.paged_attention_prefill_chunk(oracle.storage(m.chunk_query)[0], kn, vn, cbt, m.seq_lens,
                                            m.query_start_loc, dec.scale, code, row_select=sel)
    rows = np.nonzero(sel)[0]
    assert_close(pout[torch.from_numpy(rows).cuda()], ref[rows], torch.bfloat16, "mixed prefill sample")
