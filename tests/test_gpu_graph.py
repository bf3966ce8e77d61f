"""A decode step (append + attend) captured once in a CUDA graph and replayed on new inputs."""
import numpy as np
import pytest
import torch

import paged_kv_cache_409_b200 as pkv
from paged_kv_cache_409_b200 import workloads
from parity_helpers import assert_close, gpu_tables, oracle_decode_step, to_device

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype,Hq,Hkv", [(torch.float16, 8, 8), (torch.bfloat16, 16, 2)])
def test_graph_replay_matches_oracle(dtype, Hq, Hkv):
    w = workloads.decode_workload("graph", [300, 17, 1000, 64], Hq, Hkv, 128, 16, dtype, seed=41)
    pre_k, pre_v = w.key_caches[0].clone(), w.value_caches[0].clone()
    to_device(w)
    bt, cl, sm = gpu_tables(w)
    q, nk, nv = w.queries[0].clone(), w.new_keys[0].clone(), w.new_values[0].clone()
    out = torch.empty_like(q)
    ws = torch.empty(1 << 20, dtype=torch.uint8, device="cuda")

    def step():
        pkv.reshape_and_cache(nk, nv, w.key_caches[0], w.value_caches[0], sm)
        pkv.paged_attention_decode(out, q, w.key_caches[0], w.value_caches[0], bt, cl, w.scale, w.max_context_len,
                                   partition_size=256, workspace=ws)

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        step()                      # first call outside capture: one-time set-up
    torch.cuda.current_stream().wait_stream(s)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    gen = torch.Generator(device="cuda").manual_seed(7)
    for it in range(3):
        for t in (q, nk, nv):
            t.copy_(torch.randn(t.shape, generator=gen, device="cuda").to(dtype))
        graph.replay()
        torch.cuda.synchronize()
        w.queries[0], w.new_keys[0], w.new_values[0] = q.clone(), nk.clone(), nv.clone()
        ref, _, _, _ = oracle_decode_step(w, pre_k=pre_k, pre_v=pre_v)
        assert_close(out, ref, dtype, f"replay {it}")
    assert pkv.get_device_error() == 0
