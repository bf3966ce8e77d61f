"""Shared pieces of the GPU parity tests: run a workload through the CUDA
library and through the CPU oracle on the same seeded inputs.

Inputs for the oracle are always snapshots taken BEFORE the CUDA path runs
(or host copies of generator output); nothing the kernels write feeds the
oracle.  Sampled checks on large pools copy only the blocks the sampled
sequences use and renumber them densely -- the oracle's own pins show that
physical placement does not change its result.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import paged_kv_cache_409_b200 as pkv

TOL = {torch.float32: (1e-5, 0.0), torch.float16: (2e-3, 1e-2), torch.bfloat16: (2e-3, 1e-2)}


def assert_close(gpu: torch.Tensor, ref: np.ndarray, dtype, what=""):
    """|gpu - ref| <= atol + rtol |ref| element-wise (fp32: max-abs 1e-5)."""
    atol, rtol = TOL[dtype]
    g = gpu.detach().float().cpu().double().numpy()
    assert g.shape == ref.shape, (g.shape, ref.shape)
    assert np.all(np.isfinite(g)), f"{what}: non-finite output"
    err = np.abs(g - ref)
    bound = atol + rtol * np.abs(ref)
    bad = err > bound
    if bad.any():
        i = np.unravel_index(np.argmax(err - bound), err.shape)
        raise AssertionError(f"{what}: {bad.sum()} of {bad.size} elements out of tolerance; worst at {i}: "
                             f"gpu {g[i]!r} ref {ref[i]!r} (atol {atol}, rtol {rtol})")
    return float(err.max())


def bits(t: torch.Tensor) -> np.ndarray:
    """Raw element bits of a tensor, for bit-exact comparisons (NaN payloads included)."""
    t = t.detach().cpu().contiguous()
    if t.element_size() == 4:
        return t.view(torch.int32).numpy()
    return t.view(torch.int16).numpy()


def snapshot_blocks(cache: torch.Tensor, ids: np.ndarray) -> torch.Tensor:
    """Host copy of the listed physical blocks of a pool."""
    return cache[torch.from_numpy(ids.astype(np.int64)).to(cache.device)].cpu().clone()


def compact_tables(tables: np.ndarray, lens, block_size: int):
    """Blocks used by these sequences, and their tables renumbered densely."""
    need = [(int(n) + block_size - 1) // block_size for n in lens]
    used = np.unique(np.concatenate([tables[i, :k] for i, k in enumerate(need)] + [np.zeros(0, np.int32)]))
    remap = {int(b): i for i, b in enumerate(used)}
    out = np.full_like(tables, -1)
    for i, k in enumerate(need):
        out[i, :k] = [remap[int(b)] for b in tables[i, :k]]
    return used.astype(np.int64), out.astype(np.int32)


def oracle_decode_step(w, seqs=None, layer=0, pre_k=None, pre_v=None):
    """Oracle of append-then-attend for sequences ``seqs`` of a DecodeWorkload.

    ``pre_k``/``pre_v``: host snapshots of the whole pools taken before the
    CUDA path ran (else the workload's own pools, which must still be
    untouched).  Returns (out float64 [len(seqs), Hq, D], k_after, v_after,
    used block ids) where *_after are the compacted pools after the append.
    """
    S = w.num_seqs
    seqs = np.arange(S) if seqs is None else np.asarray(seqs)
    lens = w.context_lens[seqs]
    used, bt = compact_tables(w.block_tables[seqs], lens, w.block_size)
    src_k = pre_k if pre_k is not None else w.key_caches[layer]
    src_v = pre_v if pre_v is not None else w.value_caches[layer]
    kc, code = oracle.storage(snapshot_blocks(src_k, used))
    vc, _ = oracle.storage(snapshot_blocks(src_v, used))
    kc, vc = kc.copy(), vc.copy()
    nk, _ = oracle.storage(w.new_keys[layer][torch.from_numpy(seqs).to(w.new_keys[layer].device)])
    nv, _ = oracle.storage(w.new_values[layer][torch.from_numpy(seqs).to(w.new_values[layer].device)])
    B = w.block_size
    remap = {int(b): i for i, b in enumerate(used)}
    slots = np.array([remap[int(s) // B] * B + int(s) % B for s in w.slot_mapping[seqs]], dtype=np.int64)
    orc = oracle.get()
    q, qcode = oracle.storage(w.queries[layer][torch.from_numpy(seqs).to(w.queries[layer].device)])
    if w.fp8:
        ks, vs = w.extra["k_scale"], w.extra["v_scale"]
        orc.reshape_and_cache_fp8(nk, nv, kc, vc, slots, qcode, ks, vs)
        out = orc.paged_attention_decode_kv(q, qcode, kc, vc, oracle.E4M3, ks, vs, bt, lens, w.scale)
    else:
        orc.reshape_and_cache(nk, nv, kc, vc, slots, code)
        out = orc.paged_attention_decode(q, kc, vc, bt, lens, w.scale, code)
    return out, kc, vc, used


def gpu_tables(w, device="cuda"):
    bt = torch.from_numpy(w.block_tables).to(device)
    cl = torch.from_numpy(w.context_lens.astype(np.int32)).to(device)
    sm = torch.from_numpy(w.slot_mapping.astype(np.int64)).to(device)
    return bt, cl, sm


def to_device(w, device="cuda"):
    """Move a CPU-generated DecodeWorkload's tensors to the GPU (in place)."""
    for name in ("key_caches", "value_caches", "queries", "new_keys", "new_values"):
        setattr(w, name, [t.to(device) for t in getattr(w, name)])
    return w


def gpu_decode_step(w, layer=0, partition_size=None, out=None, tables=None):
    """reshape_and_cache then paged_attention_decode on the GPU."""
    bt, cl, sm = tables if tables is not None else gpu_tables(w, w.queries[layer].device)
    kc, vc = w.key_caches[layer], w.value_caches[layer]
    if out is None:
        out = torch.empty_like(w.queries[layer])
    if w.fp8:
        ks, vs = w.extra["k_scale"], w.extra["v_scale"]
        pkv.reshape_and_cache_fp8(w.new_keys[layer], w.new_values[layer], kc, vc, sm, ks, vs)
        pkv.paged_attention_decode_fp8(out, w.queries[layer], kc, vc, bt, cl, w.scale, ks, vs, w.max_context_len,
                                       partition_size=partition_size)
        return out
    pkv.reshape_and_cache(w.new_keys[layer], w.new_values[layer], kc, vc, sm)
    pkv.paged_attention_decode(out, w.queries[layer], kc, vc, bt, cl, w.scale, w.max_context_len,
                               partition_size=partition_size)
    return out


def oracle_prefill_chunks(m, pre_k, pre_v, chunks=None, row_select=None):
    """Oracle of append-then-prefill for chunks ``chunks`` of a MixedWorkload.

    ``pre_k``/``pre_v`` are host snapshots of the pools taken before the CUDA
    path ran.  Only the blocks of the selected chunks are copied (renumbered
    densely).  Returns float64 [sum of the selected chunk lengths, Hq, D].
    """
    R = len(m.chunk_lens)
    chunks = np.arange(R) if chunks is None else np.asarray(chunks)
    S = m.decode.num_seqs
    B = m.decode.block_size
    lens = m.seq_lens[chunks]
    used, bt = compact_tables(m.chunk_tables[chunks], lens, B)
    kn, code = oracle.storage(snapshot_blocks(pre_k, used))
    vn, _ = oracle.storage(snapshot_blocks(pre_v, used))
    kn, vn = kn.copy(), vn.copy()
    remap = {int(b): i for i, b in enumerate(used)}
    qsl = m.query_start_loc
    rows = np.concatenate([np.arange(qsl[r], qsl[r + 1]) for r in chunks]).astype(np.int64)
    src = S + rows  # the chunk tokens follow the decode tokens in append_*
    cslots = m.append_slots[src]
    slots = np.array([remap[int(x) // B] * B + int(x) % B for x in cslots], dtype=np.int64)
    orc = oracle.get()
    idx = torch.from_numpy(src)
    ak, acode = oracle.storage(m.append_keys.cpu()[idx])
    av, _ = oracle.storage(m.append_values.cpu()[idx])
    n = m.chunk_lens[chunks].astype(np.int64)
    new_qsl = np.concatenate([[0], np.cumsum(n)]).astype(np.int32)
    q, qcode = oracle.storage(m.chunk_query.cpu()[torch.from_numpy(rows)])
    if m.decode.fp8:
        ks, vs = m.decode.extra["k_scale"], m.decode.extra["v_scale"]
        orc.reshape_and_cache_fp8(ak, av, kn, vn, slots, acode, ks, vs)
        return orc.paged_attention_prefill_chunk_kv(q, qcode, kn, vn, oracle.E4M3, ks, vs, bt, lens, new_qsl,
                                                    m.decode.scale, row_select=row_select)
    orc.reshape_and_cache(ak, av, kn, vn, slots, code)
    return orc.paged_attention_prefill_chunk(q, kn, vn, bt, lens, new_qsl, m.decode.scale, code,
                                             row_select=row_select)
