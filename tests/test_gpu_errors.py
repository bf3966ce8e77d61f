"""Host-detected argument errors and device-detected table errors (no fault, no hang: kernels skip and flag)."""
import pytest
import torch

import paged_kv_cache_409_b200 as pkv
from paged_kv_cache_409_b200 import workloads
from parity_helpers import gpu_tables, to_device

pytestmark = pytest.mark.gpu

EINVAL, EUNSUPPORTED, EWORKSPACE = -1, -2, -5


def small():
    w = to_device(workloads.decode_workload("e", [20, 40], 4, 2, 64, 16, torch.float16, seed=2))
    bt, cl, sm = gpu_tables(w)
    return w, bt, cl, sm


def test_unsupported_head_dim_and_group():
    w, bt, cl, _ = small()
    q = torch.zeros(2, 4, 96, dtype=torch.float16, device="cuda")
    kc = torch.zeros(w.num_blocks, 16, 2, 96, dtype=torch.float16, device="cuda")
    with pytest.raises(pkv.PagedKVError) as e:
        pkv.paged_attention_decode(torch.empty_like(q), q, kc, kc, bt, cl, 0.1, 40)
    assert e.value.status == EUNSUPPORTED
    q3 = torch.zeros(2, 6, 64, dtype=torch.float16, device="cuda")  # group 3
    with pytest.raises(pkv.PagedKVError) as e:
        pkv.paged_attention_decode(torch.empty_like(q3), q3, w.key_caches[0], w.value_caches[0], bt, cl, 0.1, 40)
    assert e.value.status == EUNSUPPORTED


def test_misaligned_pointer_rejected():
    w, bt, cl, _ = small()
    flat = torch.zeros(2 * 4 * 64 + 1, dtype=torch.float16, device="cuda")
    q = flat[1:].view(2, 4, 64)  # 2-byte offset
    with pytest.raises(pkv.PagedKVError) as e:
        pkv.paged_attention_decode(torch.empty(2, 4, 64, dtype=torch.float16, device="cuda"), q, w.key_caches[0],
                                   w.value_caches[0], bt, cl, 0.1, 40)
    assert e.value.status == EINVAL


def test_workspace_too_small():
    w, bt, cl, _ = small()
    ws = torch.empty(16, dtype=torch.uint8, device="cuda")
    lib = pkv.load_library()
    q, out = w.queries[0], torch.empty_like(w.queries[0])
    rc = lib.pkv_paged_attention_decode(out.data_ptr(), q.data_ptr(), w.key_caches[0].data_ptr(),
                                        w.value_caches[0].data_ptr(), bt.data_ptr(), cl.data_ptr(), 0.1, 2, 4, 2, 64,
                                        16, bt.shape[1], w.num_blocks, 40, 16, 1, ws.data_ptr(), 16,
                                        torch.cuda.current_stream().cuda_stream)
    assert rc == EWORKSPACE


def test_bad_block_id_is_flagged_not_faulted():
    w, bt, cl, _ = small()
    bt[1, 1] = w.num_blocks + 1000
    out = torch.empty_like(w.queries[0])
    pkv.paged_attention_decode(out, w.queries[0], w.key_caches[0], w.value_caches[0], bt, cl, w.scale, 40)
    assert pkv.get_device_error() & pkv._binding.DEVERR_BLOCK_ID
    assert pkv.get_device_error() == 0  # reading clears it


@pytest.mark.parametrize("B", [8, 16])
def test_bad_block_id_in_an_e4m3_unit_is_flagged_not_faulted(B):
    """E4M3 pools with 8 heads per KV head group blocks into 32-token steps: a bad id in the first
    block of a step or inside one is skipped and flagged, and the other sequences' rows are unchanged."""
    w = to_device(workloads.decode_workload("e8", [100, 200, 90], 16, 2, 128, B, torch.float16, seed=4,
                                            fp8_scales=(0.05, 0.05)))
    bt, cl, _ = gpu_tables(w)
    ks, vs = w.extra["k_scale"], w.extra["v_scale"]
    ref = torch.empty_like(w.queries[0])
    pkv.paged_attention_decode_fp8(ref, w.queries[0], w.key_caches[0], w.value_caches[0], bt, cl, w.scale, ks, vs,
                                   200, partition_size=0)
    torch.cuda.synchronize()
    assert pkv.get_device_error() == 0
    for col in (0, 1, 3):  # first block of a unit, inside one, inside a later one
        bad = bt.clone()
        bad[1, col] = w.num_blocks + 77
        out = torch.empty_like(ref)
        pkv.paged_attention_decode_fp8(out, w.queries[0], w.key_caches[0], w.value_caches[0], bad, cl, w.scale, ks,
                                       vs, 200, partition_size=0)
        assert pkv.get_device_error() & pkv._binding.DEVERR_BLOCK_ID
        assert torch.equal(out[0], ref[0]) and torch.equal(out[2], ref[2])


def test_context_beyond_table_is_flagged():
    w, bt, cl, _ = small()
    cl[0] = bt.shape[1] * 16 + 5
    out = torch.empty_like(w.queries[0])
    pkv.paged_attention_decode(out, w.queries[0], w.key_caches[0], w.value_caches[0], bt, cl, w.scale,
                               int(cl.max()))
    assert pkv.get_device_error() & pkv._binding.DEVERR_LENGTH


def test_bad_slot_and_pair_are_flagged():
    w, bt, cl, sm = small()
    sm[0] = w.num_blocks * 16 + 3
    pkv.reshape_and_cache(w.new_keys[0], w.new_values[0], w.key_caches[0], w.value_caches[0], sm)
    assert pkv.get_device_error() & pkv._binding.DEVERR_SLOT
    pairs = torch.tensor([[0, w.num_blocks]], dtype=torch.int64, device="cuda")
    pkv.copy_blocks(w.key_caches, w.value_caches, pairs)
    assert pkv.get_device_error() & pkv._binding.DEVERR_PAIR


def test_prefill_chunk_longer_than_sequence_is_flagged():
    m = workloads.mixed_workload("bad", [], [10], [64], 8, 8, 128, 16, torch.bfloat16, seed=3)
    dev = "cuda"
    kc, vc = m.decode.key_caches[0].to(dev), m.decode.value_caches[0].to(dev)
    q = m.chunk_query.to(dev)
    sl = torch.tensor([32], dtype=torch.int32, device=dev)  # fewer tokens than the chunk itself
    pkv.paged_attention_prefill_chunk(torch.empty_like(q), q, kc, vc, torch.from_numpy(m.chunk_tables).to(dev), sl,
                                      torch.from_numpy(m.query_start_loc).to(dev), 64, m.decode.scale)
    assert pkv.get_device_error() & pkv._binding.DEVERR_LENGTH
