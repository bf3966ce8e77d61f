"""Host-side block arithmetic and the synthetic workloads (no GPU)."""
import numpy as np
import pytest
import torch

from oracle_pins import golden
from paged_kv_cache_409_b200 import paging, workloads


def test_blocks_needed_matches_pages_examples():
    for e in golden()["blocks_needed"]:
        assert paging.blocks_needed(e["tokens"], e["block_size"]) == e["blocks"], e["source"]


def test_slot_mapping_matches_block_table_example():
    ex = golden()["block_table_example"]
    bt = np.array([ex["block_table"]], dtype=np.int32)
    got = paging.slot_mapping(bt, np.zeros(len(ex["positions"]), np.int64), ex["positions"], ex["block_size"])
    assert got.tolist() == ex["slots"]


def test_slot_mapping_agrees_with_oracle(orc):
    rng = np.random.default_rng(5)
    for B in (8, 16, 32):
        bt = rng.permutation(200).astype(np.int32)[:60].reshape(3, 20)
        seq = rng.integers(0, 3, size=50)
        pos = rng.integers(0, 20 * B, size=50)
        got = paging.slot_mapping(bt, seq, pos, B)
        want = [orc.slot_for_position(bt[s], p, B) for s, p in zip(seq, pos)]
        assert got.tolist() == want


def test_slot_mapping_rejects_unassigned_blocks():
    bt = np.array([[3, -1]], dtype=np.int32)
    with pytest.raises(ValueError):
        paging.slot_mapping(bt, [0], [20], 16)
    with pytest.raises(ValueError):
        paging.slot_mapping(bt, [0], [40], 16)


def test_kv_bytes_per_token_matches_tutorial_figure():
    g = golden()["kv_bytes_per_token"]
    w = workloads.decode_workload("one", [1], 32, 32, 128, 16, torch.float16, seed=0, num_blocks=1)
    assert w.kv_bytes() * g["layers"] == g["bytes"]
    assert g["bytes"] * g["per_request_tokens"] == g["per_request_bytes"]


def _check_tables(bt, lens, B, nb, shared_ok=False):
    used = []
    for s, n in enumerate(lens):
        need = (int(n) + B - 1) // B
        row = bt[s]
        assert np.all(row[:need] >= 0) and np.all(row[:need] < nb)
        assert np.all(row[need:] == -1)
        # internal fragmentation: fewer than one block of unused slots per sequence
        assert need * B - int(n) < B
        used.extend(row[:need].tolist())
    if not shared_ok:
        assert len(used) == len(set(used)), "a physical block is owned twice"


def test_tiny_workload_shape():
    w = workloads.tiny_decode_f32()
    assert w.num_blocks == 32 and w.context_lens.tolist() == [1, 17, 33, 100]
    assert sum((int(n) + 15) // 16 for n in w.context_lens) == 13
    _check_tables(w.block_tables, w.context_lens, 16, 32)
    assert w.scale == np.float32(0.125)


def test_llama7b_workload_pool_and_tables():
    w = workloads.llama7b_decode_f16(num_seqs=16)
    assert w.context_lens.min() >= 128 and w.context_lens.max() <= 2048
    in_use = int(sum((int(n) + 15) // 16 for n in w.context_lens))
    assert w.num_blocks == in_use + (in_use + 9) // 10
    _check_tables(w.block_tables, w.context_lens, 16, w.num_blocks)
    last = w.context_lens - 1
    expect = [w.block_tables[s, p // 16] * 16 + p % 16 for s, p in enumerate(last)]
    assert w.slot_mapping.tolist() == expect


def test_gqa_lognormal_lengths():
    w = workloads.gqa70b_decode_bf16(num_seqs=512, num_layers=1)
    assert w.context_lens.min() >= 16 and w.context_lens.max() <= 4096
    assert 900 <= np.median(w.context_lens) <= 1150
    assert w.num_q_heads == 64 and w.num_kv_heads == 8


def test_shared_prefix_workload_structure():
    sp = workloads.shared_prefix_decode_f16(num_seqs=8)
    st = sp.step
    assert len(sp.prefix_blocks) == 94 and sp.prefix_len == 1500
    assert np.all(sp.tables_before_cow[:, :94] == sp.prefix_blocks)
    assert np.all(st.block_tables[:, :93] == sp.prefix_blocks[:93])
    assert np.all(sp.cow_pairs[:, 0] == sp.prefix_blocks[93])
    assert np.array_equal(st.block_tables[:, 93], sp.cow_pairs[:, 1])
    assert len(set(sp.cow_pairs[:, 1].tolist())) == len(sp.cow_pairs)
    assert np.all((sp.private_lens >= 8) & (sp.private_lens <= 64))
    assert np.array_equal(st.context_lens, 1500 + sp.private_lens + 1)
    _check_tables(st.block_tables, st.context_lens, 16, st.num_blocks, shared_ok=True)


def test_mixed_workload_structure():
    m = workloads.mixed_step_bf16(num_decode=6, num_chunks=3, chunk_len=40, decode_hi=4000, c0_hi=300)
    assert m.query_start_loc.tolist() == [0, 40, 80, 120]
    assert np.array_equal(m.seq_lens, m.chunk_c0 + 40)
    assert len(m.append_slots) == 6 + 120 and len(set(m.append_slots.tolist())) == 126
    _check_tables(m.chunk_tables, m.seq_lens, 32, m.decode.num_blocks)
    _check_tables(m.decode.block_tables, m.decode.context_lens, 32, m.decode.num_blocks)
    assert not set(m.decode.block_tables[m.decode.block_tables >= 0].tolist()) & \
        set(m.chunk_tables[m.chunk_tables >= 0].tolist())


def test_poison_marks_only_dead_slots():
    w = workloads.decode_workload("p", [5, 20], 2, 2, 8, 8, torch.float32, seed=3, poison=True)
    kc = w.key_caches[0].view(-1, 2 * 8)
    live = workloads.live_slots(w.block_tables, w.context_lens, 8)
    dead = np.setdiff1d(np.arange(kc.shape[0]), live)
    assert torch.isfinite(kc[torch.from_numpy(live)]).all()
    assert torch.isnan(kc[torch.from_numpy(dead)]).all()


def test_fp8_workload_codes():
    """E4M3 pools hold finite codes of N(0,1)/scale in live slots and the NaN code 0x7F in dead ones."""
    w = workloads.decode_workload("f8", [5, 33, 70], 8, 2, 128, 16, torch.float16, seed=3, poison=True,
                                  fp8_scales=(0.02, 0.03))
    assert w.fp8 and w.key_caches[0].dtype == torch.uint8
    assert w.extra["k_scale"] == float(np.float32(0.02)) and w.extra["v_scale"] == float(np.float32(0.03))
    live = workloads.live_slots(w.block_tables, w.context_lens, w.block_size)
    rows = w.key_caches[0].view(-1, 2 * 128)
    mask = np.zeros(rows.shape[0], dtype=bool)
    mask[live] = True
    codes_live = rows[torch.from_numpy(mask)].numpy()
    assert not np.isin(codes_live, [0x7F, 0xFF]).any()           # no NaN codes where tokens live
    assert (rows[torch.from_numpy(~mask)].numpy() == 0x7F).all()  # dead slots poisoned
    vals = torch.from_numpy(codes_live).view(torch.float8_e4m3fn).float() * 0.02
    assert abs(vals.std().item() - 1.0) < 0.1                     # N(0,1) after the scale
    assert w.kv_bytes() == 2 * int(w.context_lens.sum()) * 2 * 128  # one byte per element


def test_build_tracks_every_included_file(tmp_path, monkeypatch):
    """The library is rebuilt when any file it is compiled from changes: every local #include reachable
    from the sources is among the build's dependencies, and a library older than one of them is stale."""
    import os
    import re
    from paged_kv_cache_409_b200 import build
    deps = {os.path.basename(d) for d in build.depends()}
    todo, seen = list(build.SOURCES), set()
    while todo:
        f = todo.pop()
        if f in seen:
            continue
        seen.add(f)
        path = os.path.join(build.CSRC if os.path.exists(os.path.join(build.CSRC, f)) else build.INCLUDE, f)
        todo += re.findall(r'#include\s+"([^"]+)"', open(path).read())
    assert seen <= deps, seen - deps
    newest = max(os.path.getmtime(d) for d in build.depends())
    lib = tmp_path / "lib.so"
    lib.write_bytes(b"")
    monkeypatch.setattr(build, "LIB", str(lib))
    os.utime(lib, (newest - 10, newest - 10))
    assert build.stale()
    os.utime(lib, (newest + 10, newest + 10))
    assert not build.stale()
