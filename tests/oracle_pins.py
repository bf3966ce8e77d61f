"""Pins of the CPU oracle against things other than itself.

Each ``pin_*`` takes an :class:`oracle.Oracle` and raises ``AssertionError``
when the oracle disagrees with what the pages or the mathematics fix:

* library routines on contiguous data (``torch.nn.functional.
  scaled_dot_product_attention`` in float64, numpy fancy indexing, numpy /
  torch element conversion);
* closed forms (one-token context, zero query, equal keys, two-token logistic
  weights, a dominant score, per-head constant values);
* invariants of the paging data model (physical block placement and shared
  prefix blocks do not change the result);
* the worked index examples printed on the pages (``golden/``).

They live in a plain module so that ``test_oracle_mutants.py`` can run the
same pins against deliberately broken copies of the oracle.
"""
from __future__ import annotations

import json
import os

import numpy as np
import torch
import torch.nn.functional as F

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "index_examples.json")


def golden():
    with open(GOLDEN) as f:
        return json.load(f)


# ---------------------------------------------------------------------------
# input construction: dense per-sequence K/V scattered into a pool
# ---------------------------------------------------------------------------

def scatter_pool(dense_k, dense_v, lens, block_size, num_blocks, rng, fill=np.nan):
    """Place dense [S, Lmax, Hkv, D] K/V into a randomly placed fp32 pool.

    Returns (key_cache, value_cache, block_tables); unused slots hold ``fill``.
    """
    S, Lmax, Hkv, D = dense_k.shape
    need = [(int(n) + block_size - 1) // block_size for n in lens]
    mb = max(max(need), 1)
    perm = rng.permutation(num_blocks)
    bt = np.full((S, mb), -1, dtype=np.int32)
    k = 0
    for s, nb in enumerate(need):
        bt[s, :nb] = perm[k:k + nb]
        k += nb
    kc = np.full((num_blocks * block_size, Hkv, D), fill, dtype=np.float32)
    vc = np.full((num_blocks * block_size, Hkv, D), fill, dtype=np.float32)
    for s in range(S):
        for pos in range(int(lens[s])):
            slot = bt[s, pos // block_size] * block_size + pos % block_size
            kc[slot] = dense_k[s, pos]
            vc[slot] = dense_v[s, pos]
    return (kc.reshape(num_blocks, block_size, Hkv, D), vc.reshape(num_blocks, block_size, Hkv, D), bt)


def sdpa_reference(q, k, v, scale, mask=None):
    """float64 torch SDPA; q [Hq, Lq, D], k/v [Hq, Lk, D]."""
    qt, kt, vt = (torch.from_numpy(np.asarray(x, dtype=np.float64)) for x in (q, k, v))
    m = None if mask is None else torch.from_numpy(mask)
    return F.scaled_dot_product_attention(qt, kt, vt, attn_mask=m, scale=float(scale)).numpy()


def _case(rng, lens, Hq=4, Hkv=2, D=8, B=4, extra_blocks=3):
    S, Lmax = len(lens), max(max(lens), 1)
    dk = rng.standard_normal((S, Lmax, Hkv, D)).astype(np.float32)
    dv = rng.standard_normal((S, Lmax, Hkv, D)).astype(np.float32)
    q = rng.standard_normal((S, Hq, D)).astype(np.float32)
    nb = sum((n + B - 1) // B for n in lens) + extra_blocks
    kc, vc, bt = scatter_pool(dk, dv, lens, B, nb, rng)
    return q, dk, dv, kc, vc, bt


# ---------------------------------------------------------------------------
# pins
# ---------------------------------------------------------------------------

def pin_decode_matches_sdpa(orc: oracle.Oracle):
    """Paged decode == SDPA over the contiguous K/V (GQA, ragged, many blocks)."""
    rng = np.random.default_rng(11)
    lens = [1, 7, 13, 4]
    Hq, Hkv, D, B = 4, 2, 8, 4
    q, dk, dv, kc, vc, bt = _case(rng, lens, Hq, Hkv, D, B)
    scale = 0.37
    out = orc.paged_attention_decode(q, kc, vc, bt, np.array(lens), scale, oracle.F32)
    G = Hq // Hkv
    for s, n in enumerate(lens):
        k = np.repeat(dk[s, :n].transpose(1, 0, 2), G, axis=0)   # [Hq, n, D]
        v = np.repeat(dv[s, :n].transpose(1, 0, 2), G, axis=0)
        ref = sdpa_reference(q[s][:, None, :], k, v, scale)[:, 0, :]
        np.testing.assert_allclose(out[s], ref, rtol=0, atol=1e-12)


def pin_prefill_matches_masked_sdpa(orc: oracle.Oracle):
    """Chunked prefill == SDPA with the causal mask key <= c0 + i."""
    rng = np.random.default_rng(12)
    c0s, ns = [5, 0, 11], [6, 9, 1]
    lens = [c + n for c, n in zip(c0s, ns)]
    Hq, Hkv, D, B = 4, 2, 8, 4
    _, dk, dv, kc, vc, bt = _case(rng, lens, Hq, Hkv, D, B)
    qsl = np.concatenate([[0], np.cumsum(ns)]).astype(np.int32)
    q = rng.standard_normal((int(qsl[-1]), Hq, D)).astype(np.float32)
    scale = 0.29
    out = orc.paged_attention_prefill_chunk(q, kc, vc, bt, np.array(lens), qsl, scale, oracle.F32)
    G = Hq // Hkv
    for r, (c0, n) in enumerate(zip(c0s, ns)):
        L = c0 + n
        k = np.repeat(dk[r, :L].transpose(1, 0, 2), G, axis=0)
        v = np.repeat(dv[r, :L].transpose(1, 0, 2), G, axis=0)
        mask = np.arange(L)[None, :] <= (c0 + np.arange(n))[:, None]
        ref = sdpa_reference(q[qsl[r]:qsl[r + 1]].transpose(1, 0, 2), k, v, scale, mask)  # [Hq, n, D]
        np.testing.assert_allclose(out[qsl[r]:qsl[r + 1]], ref.transpose(1, 0, 2), rtol=0, atol=1e-12)


def pin_placement_invariance(orc: oracle.Oracle):
    """Moving physical blocks and rewriting the table consistently changes nothing."""
    rng = np.random.default_rng(13)
    lens = [9, 16, 3]
    q, _, _, kc, vc, bt = _case(rng, lens, 4, 4, 8, 4, extra_blocks=5)
    out = orc.paged_attention_decode(q, kc, vc, bt, np.array(lens), 0.5, oracle.F32)
    nb = kc.shape[0]
    perm = rng.permutation(nb)
    kc2, vc2 = np.empty_like(kc), np.empty_like(vc)
    kc2[perm] = kc
    vc2[perm] = vc
    bt2 = np.where(bt >= 0, perm[np.maximum(bt, 0)], -1).astype(np.int32)
    out2 = orc.paged_attention_decode(q, kc2, vc2, bt2, np.array(lens), 0.5, oracle.F32)
    assert np.array_equal(out, out2)


def pin_shared_prefix_equals_private_copies(orc: oracle.Oracle):
    """Tables that share prefix blocks give what private copies of them give."""
    rng = np.random.default_rng(14)
    B, Hkv, D, S = 4, 2, 8, 3
    prefix_blocks, lens = 3, [14, 13, 16]
    nb = 40
    kc = rng.standard_normal((nb, B, Hkv, D)).astype(np.float32)
    vc = rng.standard_normal((nb, B, Hkv, D)).astype(np.float32)
    q = rng.standard_normal((S, 4, D)).astype(np.float32)
    shared = np.array([0, 1, 2])
    bt_shared = np.full((S, 4), -1, np.int32)
    bt_private = np.full((S, 4), -1, np.int32)
    nxt = 3
    for s in range(S):
        bt_shared[s, :prefix_blocks] = shared
        copies = np.arange(nxt, nxt + prefix_blocks)
        kc[copies], vc[copies] = kc[shared], vc[shared]
        bt_private[s, :prefix_blocks] = copies
        nxt += prefix_blocks
        tail = nxt
        bt_shared[s, prefix_blocks] = tail
        bt_private[s, prefix_blocks] = tail
        nxt += 1
    a = orc.paged_attention_decode(q, kc, vc, bt_shared, np.array(lens), 0.4, oracle.F32)
    b = orc.paged_attention_decode(q, kc, vc, bt_private, np.array(lens), 0.4, oracle.F32)
    assert np.array_equal(a, b)


def pin_one_token_returns_v(orc: oracle.Oracle):
    """Context of one token: softmax weight 1, out = V_0 exactly."""
    rng = np.random.default_rng(15)
    q, _, dv, kc, vc, bt = _case(rng, [1, 1], 4, 2, 8, 4)
    out = orc.paged_attention_decode(q, kc, vc, bt, np.array([1, 1]), 0.7, oracle.F32)
    for s in range(2):
        assert np.array_equal(out[s], np.repeat(dv[s, 0], 2, axis=0).astype(np.float64))


def pin_zero_query_gives_mean_of_v(orc: oracle.Oracle):
    rng = np.random.default_rng(16)
    lens = [5, 12]
    q, _, dv, kc, vc, bt = _case(rng, lens, 2, 2, 8, 4)
    out = orc.paged_attention_decode(np.zeros_like(q), kc, vc, bt, np.array(lens), 1.3, oracle.F32)
    for s, n in enumerate(lens):
        np.testing.assert_allclose(out[s], dv[s, :n].astype(np.float64).mean(axis=0), rtol=0, atol=1e-13)


def pin_equal_keys_give_mean_of_v(orc: oracle.Oracle):
    rng = np.random.default_rng(17)
    lens = [9]
    q, dk, dv, _, _, _ = _case(rng, lens, 2, 2, 8, 4)
    dk[:] = dk[:, :1]
    kc, vc, bt = scatter_pool(dk, dv, lens, 4, 6, rng)
    out = orc.paged_attention_decode(q, kc, vc, bt, np.array(lens), 0.9, oracle.F32)
    np.testing.assert_allclose(out[0], dv[0, :9].astype(np.float64).mean(axis=0), rtol=0, atol=1e-13)


def pin_dominant_score_selects_its_v(orc: oracle.Oracle):
    """A huge scale sends all weight to the arg-max key."""
    rng = np.random.default_rng(18)
    lens = [11]
    q, dk, dv, kc, vc, bt = _case(rng, lens, 1, 1, 8, 4)
    scores = dk[0, :11, 0].astype(np.float64) @ q[0, 0].astype(np.float64)
    top2 = np.sort(scores)[-2:]
    scale = 4000.0 / max(top2[1] - top2[0], 1e-3)
    out = orc.paged_attention_decode(q, kc, vc, bt, np.array(lens), scale, oracle.F32)
    np.testing.assert_allclose(out[0, 0], dv[0, int(np.argmax(scores)), 0], rtol=0, atol=1e-12)


def pin_two_tokens_logistic(orc: oracle.Oracle):
    """n = 2: out = sigma(x0 - x1) V0 + sigma(x1 - x0) V1."""
    rng = np.random.default_rng(19)
    q, dk, dv, kc, vc, bt = _case(rng, [2], 2, 2, 8, 4)
    scale = 0.61
    out = orc.paged_attention_decode(q, kc, vc, bt, np.array([2]), scale, oracle.F32)
    for h in range(2):
        x = scale * (dk[0, :2, h].astype(np.float64) @ q[0, h].astype(np.float64))
        w0 = 1.0 / (1.0 + np.exp(x[1] - x[0]))
        w1 = 1.0 / (1.0 + np.exp(x[0] - x[1]))
        ref = w0 * dv[0, 0, h] + w1 * dv[0, 1, h]
        np.testing.assert_allclose(out[0, h], ref, rtol=0, atol=1e-14)


def pin_empty_context_is_zero(orc: oracle.Oracle):
    rng = np.random.default_rng(20)
    q, _, _, kc, vc, bt = _case(rng, [0, 3], 2, 2, 8, 4)
    out = orc.paged_attention_decode(q, kc, vc, bt, np.array([0, 3]), 0.5, oracle.F32)
    assert np.all(out[0] == 0.0) and np.all(np.isfinite(out[1]))


def pin_group_head_mapping(orc: oracle.Oracle):
    """Query head h reads KV head h // G: with V constant g on KV head g, out[h] = h // G."""
    rng = np.random.default_rng(21)
    Hq, Hkv, D, B = 8, 2, 8, 4
    lens = [10]
    q, dk, dv, _, _, _ = _case(rng, lens, Hq, Hkv, D, B)
    for g in range(Hkv):
        dv[:, :, g, :] = float(g + 1)
    kc, vc, bt = scatter_pool(dk, dv, lens, B, 5, rng)
    out = orc.paged_attention_decode(q, kc, vc, bt, np.array(lens), 0.5, oracle.F32)
    for h in range(Hq):
        np.testing.assert_allclose(out[0, h], h // (Hq // Hkv) + 1.0, rtol=0, atol=1e-13)


def pin_prefill_rows_equal_decode_of_prefix(orc: oracle.Oracle):
    """A chunk starting at position 0: row i == decode over the first i + 1 tokens."""
    rng = np.random.default_rng(22)
    n = 10
    _, _, _, kc, vc, bt = _case(rng, [n], 4, 2, 8, 4)
    q = rng.standard_normal((n, 4, 8)).astype(np.float32)
    pre = orc.paged_attention_prefill_chunk(q, kc, vc, bt, np.array([n]), np.array([0, n]), 0.45, oracle.F32)
    for i in range(n):
        dec = orc.paged_attention_decode(q[i:i + 1], kc, vc, bt, np.array([i + 1]), 0.45, oracle.F32)
        np.testing.assert_allclose(pre[i], dec[0], rtol=0, atol=1e-14)


def pin_storage_dtypes_decode_exactly(orc: oracle.Oracle):
    """fp16 / bf16 elements decode to the values numpy / torch give them."""
    bits = np.arange(1 << 16, dtype=np.uint16)
    half = orc.to_double(bits.view(np.float16), oracle.F16)
    np.testing.assert_array_equal(half, bits.view(np.float16).astype(np.float64))
    bf = orc.to_double(bits, oracle.BF16)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(bf, ref)
    f32 = np.random.default_rng(23).standard_normal(100).astype(np.float32)
    np.testing.assert_array_equal(orc.to_double(f32, oracle.F32), f32.astype(np.float64))


def pin_reshape_and_cache_matches_indexing(orc: oracle.Oracle):
    """Token t lands in row slot_mapping[t] of the flattened pool; -1 is skipped; nothing else moves."""
    rng = np.random.default_rng(24)
    NB, B, Hkv, D, T = 7, 4, 3, 8, 9
    kc = rng.standard_normal((NB, B, Hkv, D)).astype(np.float16)
    vc = rng.standard_normal((NB, B, Hkv, D)).astype(np.float16)
    k = rng.standard_normal((T, Hkv, D)).astype(np.float16)
    v = rng.standard_normal((T, Hkv, D)).astype(np.float16)
    slots = rng.choice(NB * B, size=T, replace=False).astype(np.int64)
    slots[[2, 5]] = -1
    ek, ev = kc.copy(), vc.copy()
    ok = slots >= 0
    ek.reshape(NB * B, Hkv, D)[slots[ok]] = k[ok]
    ev.reshape(NB * B, Hkv, D)[slots[ok]] = v[ok]
    orc.reshape_and_cache(k, v, kc, vc, slots, oracle.F16)
    assert np.array_equal(kc.view(np.uint16), ek.view(np.uint16))
    assert np.array_equal(vc.view(np.uint16), ev.view(np.uint16))


def pin_copy_blocks_matches_indexing(orc: oracle.Oracle):
    rng = np.random.default_rng(25)
    NB, B, Hkv, D = 10, 4, 2, 8
    layers = [rng.standard_normal((NB, B, Hkv, D)).astype(np.float32) for _ in range(4)]
    pairs = np.array([[1, 6], [1, 7], [3, 9], [0, 8]], dtype=np.int64)
    expect = [c.copy() for c in layers]
    for c in expect:
        c[pairs[:, 1]] = c[pairs[:, 0]]
    kcs, vcs = layers[:2], layers[2:]
    orc.copy_blocks(kcs, vcs, pairs)
    for got, want in zip(layers, expect):
        assert np.array_equal(got, want)


def pin_index_examples(orc: oracle.Oracle):
    g = golden()
    for e in g["blocks_needed"]:
        assert orc.blocks_needed(e["tokens"], e["block_size"]) == e["blocks"], e["source"]
    ex = g["block_table_example"]
    row = np.array(ex["block_table"], dtype=np.int32)
    for pos, slot in zip(ex["positions"], ex["slots"]):
        assert orc.slot_for_position(row, pos, ex["block_size"]) == slot, (pos, ex["source"])
    h = g["hundredth_token"]
    table = np.arange(16, dtype=np.int32)
    slot = orc.slot_for_position(table, h["position"], h["block_size"])
    assert (slot // h["block_size"], slot % h["block_size"]) == (h["logical_block"], h["offset"])


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
