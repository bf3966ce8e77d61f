"""The bounded waits' give-up path, run on purpose: with the main-loop wait limit at 0 every kernel's first
wait that would block gives up, sets PKV_DEVERR_TIMEOUT, waits for its own copies and MMAs, releases its
tensor memory and returns.  The device stays usable: with the limit restored, the same calls in the same
process match the oracle."""
import numpy as np
import pytest
import torch

import paged_kv_cache_409_b200 as pkv
from paged_kv_cache_409_b200 import workloads
from parity_helpers import (assert_close, gpu_tables, oracle_decode_step, oracle_prefill_chunks,
                            to_device)

pytestmark = pytest.mark.gpu


def flush_l2():
    """Write a buffer twice the L2's size: the next kernel's K/V come from HBM, so
    its first bulk copies are still in flight when its waits start."""
    torch.empty(256 << 20, dtype=torch.uint8, device="cuda").fill_(1)


def run_decode(w, pre_k, pre_v, part, flush=False):
    w.key_caches[0], w.value_caches[0] = pre_k.cuda(), pre_v.cuda()
    bt, cl, sm = gpu_tables(w, "cuda")
    kc, vc = w.key_caches[0], w.value_caches[0]
    out = torch.empty_like(w.queries[0])
    if w.fp8:
        ks, vs = w.extra["k_scale"], w.extra["v_scale"]
        pkv.reshape_and_cache_fp8(w.new_keys[0], w.new_values[0], kc, vc, sm, ks, vs)
        if flush:
            flush_l2()
        pkv.paged_attention_decode_fp8(out, w.queries[0], kc, vc, bt, cl, w.scale, ks, vs, w.max_context_len,
                                       partition_size=part)
    else:
        pkv.reshape_and_cache(w.new_keys[0], w.new_values[0], kc, vc, sm)
        if flush:
            flush_l2()
        pkv.paged_attention_decode(out, w.queries[0], kc, vc, bt, cl, w.scale, w.max_context_len, partition_size=part)
    return out


def run_prefill(m, pre_k, pre_v, flush=False):
    dev = "cuda"
    kc, vc = pre_k.to(dev), pre_v.to(dev)
    pkv.reshape_and_cache(m.append_keys.to(dev), m.append_values.to(dev), kc, vc,
                          torch.from_numpy(m.append_slots).to(dev))
    q = m.chunk_query.to(dev)
    out = torch.empty_like(q)
    if flush:
        flush_l2()
    pkv.paged_attention_prefill_chunk(out, q, kc, vc, torch.from_numpy(m.chunk_tables).to(dev),
                                      torch.from_numpy(m.seq_lens).to(dev),
                                      torch.from_numpy(m.query_start_loc).to(dev), int(m.chunk_lens.max()),
                                      m.decode.scale)
    return out


def run_multi(m, pre_k, pre_v, part, flush=False):
    dev = "cuda"
    kc, vc = pre_k.to(dev), pre_v.to(dev)
    pkv.reshape_and_cache(m.append_keys.to(dev), m.append_values.to(dev), kc, vc,
                          torch.from_numpy(m.append_slots).to(dev))
    q = m.chunk_query.to(dev)
    out = torch.empty_like(q)
    if flush:
        flush_l2()
    pkv.paged_attention_decode_multi(out, q, kc, vc, torch.from_numpy(m.chunk_tables).to(dev),
                                     torch.from_numpy(m.seq_lens).to(dev),
                                     torch.from_numpy(m.query_start_loc).to(dev), int(m.chunk_lens.max()),
                                     int(m.seq_lens.max()), m.decode.scale, partition_size=part)
    return out


def test_main_loop_waits_give_up_then_the_device_still_matches_the_oracle():
    TIMEOUT = pkv._binding.DEVERR_TIMEOUT
    assert pkv.get_device_error() == 0
    cases = []
    for dt, G, fp8 in ((torch.float32, 1, False), (torch.float16, 1, False), (torch.bfloat16, 8, False),
                       (torch.float16, 4, True)):
        w = workloads.decode_workload("wl", [1, 40, 700, 1500], 2 * G, 2, 128 if fp8 or dt != torch.float32 else 64,
                                      16, dt, seed=60 + G, fp8_scales=(0.05, 0.04) if fp8 else None)
        pre_k, pre_v = w.key_caches[0].clone(), w.value_caches[0].clone()
        ref = oracle_decode_step(w, pre_k=pre_k, pre_v=pre_v)[0]
        to_device(w)
        cases.append(("decode", dt, lambda flush=False, w=w, a=pre_k, b=pre_v: run_decode(w, a, b, 256, flush), ref))
    m = workloads.mixed_workload("wlp", [], [0, 300, 1000], [200, 64, 129], 32, 8, 128, 32, torch.bfloat16, seed=66)
    pk, pv = m.decode.key_caches[0].clone(), m.decode.value_caches[0].clone()
    cases.append(("prefill", torch.bfloat16, lambda flush=False: run_prefill(m, pk, pv, flush),
                  oracle_prefill_chunks(m, pk, pv)))
    mt = workloads.mixed_workload("wlm", [], [500, 3000, 40], [3, 4, 2], 32, 8, 128, 32, torch.float16, seed=67)
    mk, mv = mt.decode.key_caches[0].clone(), mt.decode.value_caches[0].clone()
    cases.append(("multi", torch.float16, lambda flush=False: run_multi(mt, mk, mv, 256, flush),
                  oracle_prefill_chunks(mt, mk, mv)))
    try:
        pkv.set_wait_limit_ns(0)
        for name, _, fn, _ in cases:
            fn(flush=True)
            torch.cuda.synchronize()
            assert pkv.get_device_error() & TIMEOUT, f"{name}: no wait gave up"
    finally:
        pkv.set_wait_limit_ns(pkv.DEFAULT_WAIT_LIMIT_NS)
    for name, dt, fn, ref in cases:
        out = fn()
        torch.cuda.synchronize()
        assert pkv.get_device_error() == 0, name
        assert_close(out, ref, dt, f"{name} after the forced give-up")
