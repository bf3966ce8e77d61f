"""The one-call decode step (append, then decode launched as the append's programmatic dependent) against
the oracle, against the two separate calls bit for bit, inside a CUDA graph, and refused without side
effects."""
import numpy as np
import pytest
import torch

import paged_kv_cache_409_b200 as pkv
from paged_kv_cache_409_b200 import workloads
from parity_helpers import assert_close, bits, gpu_decode_step, gpu_tables, oracle_decode_step, to_device

pytestmark = pytest.mark.gpu

DT = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


def step_call(w, bt, cl, sm, out, part, ws=None):
    kc, vc = w.key_caches[0], w.value_caches[0]
    if w.fp8:
        pkv.paged_attention_decode_step_fp8(w.new_keys[0], w.new_values[0], sm, out, w.queries[0], kc, vc, bt, cl,
                                            w.scale, w.extra["k_scale"], w.extra["v_scale"], w.max_context_len,
                                            partition_size=part, workspace=ws)
    else:
        pkv.paged_attention_decode_step(w.new_keys[0], w.new_values[0], sm, out, w.queries[0], kc, vc, bt, cl,
                                        w.scale, w.max_context_len, partition_size=part, workspace=ws)
    return out


@pytest.mark.parametrize("dt,D,B,G", [("f32", 64, 16, 1), ("f16", 128, 16, 1), ("bf16", 128, 32, 4),
                                      ("f16", 64, 8, 8), ("bf16", 128, 16, 2)])
def test_step_matches_oracle_and_separate_calls(dt, D, B, G):
    lens = [1, B - 1, B, B + 1, 3 * B + 5, 37, 300, 1500]
    w = workloads.decode_workload("step", lens, 2 * G, 2, D, B, DT[dt], seed=D + B + G, poison=True)
    pre_k, pre_v = w.key_caches[0].clone(), w.value_caches[0].clone()
    ref, k_after, v_after, used = oracle_decode_step(w, pre_k=pre_k, pre_v=pre_v)
    to_device(w)
    bt, cl, sm = gpu_tables(w)
    for part in (0, 4 * B):
        w.key_caches[0], w.value_caches[0] = pre_k.cuda(), pre_v.cuda()
        out = step_call(w, bt, cl, sm, torch.empty_like(w.queries[0]), part)
        torch.cuda.synchronize()
        assert pkv.get_device_error() == 0
        assert_close(out, ref, DT[dt], f"step {dt} D{D} B{B} G{G} partition {part}")
        got_k = w.key_caches[0][torch.from_numpy(used).cuda()]
        assert np.array_equal(bits(got_k), k_after.view(bits(got_k).dtype))
        # the same two kernels launched one after the other: the same bits
        w.key_caches[0], w.value_caches[0] = pre_k.cuda(), pre_v.cuda()
        sep = gpu_decode_step(w, partition_size=part)
        assert torch.equal(out.view(torch.int16 if out.element_size() == 2 else torch.int32),
                           sep.view(torch.int16 if sep.element_size() == 2 else torch.int32))


@pytest.mark.parametrize("G", [1, 8])
def test_fp8_step_matches_oracle(G):
    w = workloads.decode_workload("step8", [1, 15, 16, 17, 700, 2100], 2 * G, 2, 128, 16, torch.float16, seed=90 + G,
                                  fp8_scales=(0.05, 0.04))
    pre_k, pre_v = w.key_caches[0].clone(), w.value_caches[0].clone()
    ref, k_after, _, used = oracle_decode_step(w, pre_k=pre_k, pre_v=pre_v)
    to_device(w)
    bt, cl, sm = gpu_tables(w)
    for part in (0, 256):
        w.key_caches[0], w.value_caches[0] = pre_k.cuda(), pre_v.cuda()
        out = step_call(w, bt, cl, sm, torch.empty_like(w.queries[0]), part)
        torch.cuda.synchronize()
        assert pkv.get_device_error() == 0
        assert_close(out, ref, torch.float16, f"fp8 step G{G} partition {part}")
        got = w.key_caches[0][torch.from_numpy(used).cuda()].cpu().numpy()
        assert np.array_equal(got, k_after)


def test_step_in_a_cuda_graph_matches_oracle():
    dtype = torch.bfloat16
    w = workloads.decode_workload("stepgraph", [300, 17, 1000, 64, 2049], 16, 2, 128, 16, dtype, seed=44)
    pre_k, pre_v = w.key_caches[0].clone(), w.value_caches[0].clone()
    to_device(w)
    bt, cl, sm = gpu_tables(w)
    q, nk, nv = w.queries[0].clone(), w.new_keys[0].clone(), w.new_values[0].clone()
    out = torch.empty_like(q)
    ws = torch.empty(1 << 20, dtype=torch.uint8, device="cuda")

    def step():
        pkv.paged_attention_decode_step(nk, nv, sm, out, q, w.key_caches[0], w.value_caches[0], bt, cl, w.scale,
                                        w.max_context_len, partition_size=256, workspace=ws)

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        step()
    torch.cuda.current_stream().wait_stream(s)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    gen = torch.Generator(device="cuda").manual_seed(8)
    for it in range(3):
        for t in (q, nk, nv):
            t.copy_(torch.randn(t.shape, generator=gen, device="cuda").to(dtype))
        graph.replay()
        torch.cuda.synchronize()
        w.queries[0], w.new_keys[0], w.new_values[0] = q.clone(), nk.clone(), nv.clone()
        ref, _, _, _ = oracle_decode_step(w, pre_k=pre_k, pre_v=pre_v)
        assert_close(out, ref, dtype, f"graph replay {it}")
    assert pkv.get_device_error() == 0


def test_refused_step_changes_nothing():
    w = to_device(workloads.decode_workload("refuse", [100, 900], 8, 8, 128, 16, torch.float16, seed=45))
    bt, cl, sm = gpu_tables(w)
    before = w.key_caches[0].clone()
    tiny = torch.empty(16, dtype=torch.uint8, device="cuda")
    lib = pkv.load_library()
    out = torch.empty_like(w.queries[0])
    rc = lib.pkv_paged_attention_decode_step(
        w.new_keys[0].data_ptr(), w.new_values[0].data_ptr(), sm.data_ptr(), 2, out.data_ptr(),
        w.queries[0].data_ptr(), w.key_caches[0].data_ptr(), w.value_caches[0].data_ptr(), bt.data_ptr(),
        cl.data_ptr(), w.scale, 2, 8, 8, 128, 16, bt.shape[1], w.num_blocks, w.max_context_len, 64, 1,
        tiny.data_ptr(), 16, torch.cuda.current_stream().cuda_stream)
    assert rc == -5  # workspace too small: refused before the append ran
    torch.cuda.synchronize()
    assert torch.equal(w.key_caches[0], before)
