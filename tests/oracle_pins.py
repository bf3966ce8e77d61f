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


# ---------------------------------------------------------------------------
# FP8 (E4M3) pools
# ---------------------------------------------------------------------------

def _torch_e4m3_values(codes: np.ndarray) -> np.ndarray:
    return torch.from_numpy(codes.astype(np.uint8)).view(torch.float8_e4m3fn).to(torch.float64).numpy()


def _torch_e4m3_codes(x32: np.ndarray) -> np.ndarray:
    """torch's float32 -> float8_e4m3fn cast (round to nearest even; only used for |x| <= 448)."""
    return torch.from_numpy(np.ascontiguousarray(x32, dtype=np.float32)).to(torch.float8_e4m3fn).view(
        torch.uint8).numpy()


def pin_e4m3_decodes_like_torch(orc: oracle.Oracle):
    """Every one of the 256 codes decodes to torch's float8_e4m3fn value (NaN where torch has NaN)."""
    codes = np.arange(256, dtype=np.uint8)
    got = orc.to_double(codes, oracle.E4M3)
    ref = _torch_e4m3_values(codes)
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(got[ok], ref[ok])
    assert np.array_equal(np.signbit(got[ok]), np.signbit(ref[ok]))


def pin_e4m3_closed_forms(orc: oracle.Oracle):
    """Values fixed by the format: bias 7, 3 mantissa bits, subnormals, 448 max, S.1111.111 NaN."""
    want = {0x38: 1.0, 0x39: 1.125, 0x40: 2.0, 0x7E: 448.0, 0x08: 2.0 ** -6, 0x07: 7 * 2.0 ** -9,
            0x01: 2.0 ** -9, 0x00: 0.0, 0xB8: -1.0, 0xFE: -448.0, 0x30: 0.5, 0x77: 240.0}
    codes = np.array(list(want), dtype=np.uint8)
    got = orc.to_double(codes, oracle.E4M3)
    np.testing.assert_array_equal(got, np.array(list(want.values())))
    nan = orc.to_double(np.array([0x7F, 0xFF], dtype=np.uint8), oracle.E4M3)
    assert np.isnan(nan).all()
    neg0 = orc.to_double(np.array([0x80], dtype=np.uint8), oracle.E4M3)
    assert neg0[0] == 0.0 and np.signbit(neg0[0])


def pin_e4m3_encode_rounding(orc: oracle.Oracle):
    """Encoding: every finite code round-trips; in range it equals torch's round-to-nearest-even cast;
    exact midpoints go to the even code; beyond 448 it saturates; the sign survives rounding to zero."""
    codes = np.arange(256, dtype=np.uint8)
    vals = orc.to_double(codes, oracle.E4M3)
    fin = ~np.isnan(vals)
    back = orc.e4m3_encode(vals[fin])
    assert np.array_equal(back, codes[fin])
    # every finite fp16 value within range, and random fp32 values
    h = np.arange(1 << 16, dtype=np.uint16).view(np.float16).astype(np.float32)
    h = h[np.isfinite(h) & (np.abs(h) <= 448)]
    r = (np.random.default_rng(31).standard_normal(20000) * np.exp2(np.random.default_rng(32).integers(
        -12, 9, 20000))).astype(np.float32)
    r = r[np.abs(r) <= 448]
    for x in (h, r):
        assert np.array_equal(orc.e4m3_encode(x.astype(np.float64)), _torch_e4m3_codes(x))
    # midpoints of adjacent non-negative codes: ties to the even code
    pos = vals[:0x7F]
    mids = (pos[:-1] + pos[1:]) / 2
    got = orc.e4m3_encode(mids)
    lo = np.arange(0x7E, dtype=np.uint8)
    want = np.where(lo % 2 == 0, lo, lo + 1).astype(np.uint8)
    assert np.array_equal(got, want)
    assert orc.e4m3_encode(np.array([1.0625]))[0] == 0x38 and orc.e4m3_encode(np.array([1.1875]))[0] == 0x3A
    sat = orc.e4m3_encode(np.array([448.0, 449.0, 464.0, 1e30, np.inf, -500.0, -np.inf]))
    assert list(sat) == [0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0xFE]
    special = orc.e4m3_encode(np.array([np.nan, -0.0, -1e-9, 1e-9, 2.0 ** -10, 2.0 ** -10 * 1.0001]))
    assert list(special) == [0x7F, 0x80, 0x80, 0x00, 0x00, 0x01]


def pin_fp8_reshape_quantises_each_element(orc: oracle.Oracle):
    """FP8 append: slot t gets the codes of key[t] / k_scale (value / v_scale); -1 skipped; nothing else moves.
    Power-of-two scales keep x / scale exact in fp32, so torch's cast gives the expected codes."""
    rng = np.random.default_rng(33)
    NB, B, Hkv, D, T = 6, 4, 2, 16, 7
    kc = rng.integers(0, 256, (NB, B, Hkv, D), dtype=np.uint8)
    vc = rng.integers(0, 256, (NB, B, Hkv, D), dtype=np.uint8)
    k = (rng.standard_normal((T, Hkv, D)) * 3).astype(np.float16)
    v = (rng.standard_normal((T, Hkv, D)) * 300).astype(np.float16)   # some beyond 448 * v_scale
    k_scale, v_scale = 2.0 ** -4, 0.5
    slots = rng.choice(NB * B, size=T, replace=False).astype(np.int64)
    slots[3] = -1
    ek, ev = kc.copy(), vc.copy()
    ok = slots >= 0
    qk = np.clip(k.astype(np.float32) / np.float32(k_scale), -448, 448)
    qv = np.clip(v.astype(np.float32) / np.float32(v_scale), -448, 448)
    ek.reshape(NB * B, Hkv, D)[slots[ok]] = _torch_e4m3_codes(qk[ok])
    ev.reshape(NB * B, Hkv, D)[slots[ok]] = _torch_e4m3_codes(qv[ok])
    orc.reshape_and_cache_fp8(k, v, kc, vc, slots, oracle.F16, k_scale, v_scale)
    assert np.array_equal(kc, ek)
    assert np.array_equal(vc, ev)


def _fp8_case(rng, lens, Hq, Hkv, D, B, extra_blocks=2):
    """Random codes in randomly placed pools (no NaN codes in used slots)."""
    S = len(lens)
    need = [(n + B - 1) // B for n in lens]
    nb = sum(need) + extra_blocks
    kc = rng.integers(0, 0x7F, (nb, B, Hkv, D), dtype=np.uint8) | (rng.integers(0, 2, (nb, B, Hkv, D),
                                                                               dtype=np.uint8) << 7)
    vc = rng.integers(0, 0x7F, (nb, B, Hkv, D), dtype=np.uint8) | (rng.integers(0, 2, (nb, B, Hkv, D),
                                                                               dtype=np.uint8) << 7)
    perm = rng.permutation(nb)
    bt = np.full((S, max(need)), -1, dtype=np.int32)
    k = 0
    for s, m in enumerate(need):
        bt[s, :m] = perm[k:k + m]
        k += m
    return kc.astype(np.uint8), vc.astype(np.uint8), bt


def _dense(cache, bt, s, n, B):
    rows = [cache[bt[s, j // B], j % B] for j in range(n)]  # [n, Hkv, D]
    return np.stack(rows)


def pin_fp8_decode_matches_sdpa_on_dequantised(orc: oracle.Oracle):
    """Decode over E4M3 pools == SDPA over k_scale * torch(codes), v_scale * torch(codes)."""
    rng = np.random.default_rng(34)
    lens = [1, 9, 20]
    Hq, Hkv, D, B = 4, 2, 8, 4
    kc, vc, bt = _fp8_case(rng, lens, Hq, Hkv, D, B)
    q = rng.standard_normal((len(lens), Hq, D)).astype(np.float32)
    k_scale, v_scale, scale = 0.013, 2.5, 0.4
    out = orc.paged_attention_decode_kv(q, oracle.F32, kc, vc, oracle.E4M3, k_scale, v_scale, bt, np.array(lens),
                                        scale)
    G = Hq // Hkv
    for s, n in enumerate(lens):
        k = k_scale * _torch_e4m3_values(_dense(kc, bt, s, n, B))
        v = v_scale * _torch_e4m3_values(_dense(vc, bt, s, n, B))
        k = np.repeat(k.transpose(1, 0, 2), G, axis=0)
        v = np.repeat(v.transpose(1, 0, 2), G, axis=0)
        ref = sdpa_reference(q[s][:, None, :], k, v, scale)[:, 0, :]
        np.testing.assert_allclose(out[s], ref, rtol=0, atol=1e-12 * max(1.0, np.abs(ref).max()))


def pin_fp8_prefill_matches_masked_sdpa(orc: oracle.Oracle):
    """Chunked prefill over E4M3 pools == causal SDPA over the dequantised K/V."""
    rng = np.random.default_rng(35)
    c0s, ns = [3, 0], [5, 7]
    lens = [c + n for c, n in zip(c0s, ns)]
    Hq, Hkv, D, B = 4, 4, 8, 4
    kc, vc, bt = _fp8_case(rng, lens, Hq, Hkv, D, B)
    qsl = np.concatenate([[0], np.cumsum(ns)]).astype(np.int32)
    q = rng.standard_normal((int(qsl[-1]), Hq, D)).astype(np.float16)
    k_scale, v_scale, scale = 0.02, 0.7, 0.3
    out = orc.paged_attention_prefill_chunk_kv(q, oracle.F16, kc, vc, oracle.E4M3, k_scale, v_scale, bt,
                                               np.array(lens), qsl, scale)
    for r, (c0, n) in enumerate(zip(c0s, ns)):
        L = c0 + n
        k = (k_scale * _torch_e4m3_values(_dense(kc, bt, r, L, B))).transpose(1, 0, 2)
        v = (v_scale * _torch_e4m3_values(_dense(vc, bt, r, L, B))).transpose(1, 0, 2)
        mask = np.arange(L)[None, :] <= (c0 + np.arange(n))[:, None]
        ref = sdpa_reference(q[qsl[r]:qsl[r + 1]].astype(np.float64).transpose(1, 0, 2), k, v, scale, mask)
        np.testing.assert_allclose(out[qsl[r]:qsl[r + 1]], ref.transpose(1, 0, 2), rtol=0, atol=1e-12)


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
