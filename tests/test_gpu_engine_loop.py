"""Decode steps driven by the host block manager on the GPU, checked against the oracle.

Requests share a system prompt through the prefix cache (the second request
prefills only its own tokens and attends to K/V the first one wrote), one
request is forked mid-generation (its first append copies the shared partial
block), and every step the manager's slots, copy-on-write pairs and tables
drive reshape_and_cache, copy_blocks and paged_attention_decode.  A host
mirror of the pools runs the same operations through the oracle.
"""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_409_b200 as pkv
from paged_kv_cache_409_b200.block_manager import BlockManager
from parity_helpers import assert_close

pytestmark = pytest.mark.gpu

B, Hq, Hkv, D, NB, VOCAB = 16, 8, 2, 128, 256, 512
DT = torch.float16


def kv_of(tokens, positions, table):
    """K or V rows of tokens at positions: a fixed per-token vector, scaled by position."""
    t = torch.as_tensor(np.asarray(tokens), dtype=torch.long)
    p = torch.as_tensor(np.asarray(positions), dtype=torch.float32)
    return (table[t] * (1.0 + 0.05 * (p % 11)).view(-1, 1, 1)).to(DT)


@pytest.mark.parametrize("pools", ["fp16", "e4m3"])
def test_block_manager_drives_decode_steps(pools):
    fp8 = pools == "e4m3"
    KS, VS = 0.0131, 0.0157  # E4M3 pool scales
    rng = np.random.default_rng(21)
    g = torch.Generator().manual_seed(21)
    ek = torch.randn(VOCAB, Hkv, D, generator=g)
    ev = torch.randn(VOCAB, Hkv, D, generator=g)
    bm = BlockManager(NB, B, prefix_caching=True)
    pool_dt = torch.uint8 if fp8 else DT
    kc = torch.zeros(NB, B, Hkv, D, dtype=pool_dt, device="cuda")
    vc = torch.zeros_like(kc)
    kn = np.zeros((NB, B, Hkv, D), dtype=np.uint8 if fp8 else np.float16)  # host mirror for the oracle
    vn = np.zeros_like(kn)
    orc = oracle.get()
    tokens = {}

    def write(sid, start, toks, slots):
        pos = np.arange(start, start + len(toks))
        k, v = kv_of(toks, pos, ek), kv_of(toks, pos, ev)
        sl = torch.from_numpy(np.asarray(slots, dtype=np.int64))
        if fp8:
            pkv.reshape_and_cache_fp8(k.cuda(), v.cuda(), kc, vc, sl.cuda(), KS, VS)
            orc.reshape_and_cache_fp8(k.numpy(), v.numpy(), kn, vn, sl.numpy(), oracle.F16,
                                      float(np.float32(KS)), float(np.float32(VS)))
        else:
            pkv.reshape_and_cache(k.cuda(), v.cuda(), kc, vc, sl.cuda())
            orc.reshape_and_cache(k.numpy(), v.numpy(), kn, vn, sl.numpy(), oracle.F16)

    system = rng.integers(0, VOCAB, 40).tolist()
    prompts = {0: system + rng.integers(0, VOCAB, 5).tolist(), 1: system + rng.integers(0, VOCAB, 7).tolist(),
               2: rng.integers(0, VOCAB, 23).tolist()}
    for sid, pr in prompts.items():
        cached = bm.add_sequence(sid, pr)
        assert cached == (32 if sid == 1 else 0)   # two full blocks of the system prompt
        write(sid, cached, pr[cached:], bm.slots(sid, cached, len(pr) - cached))
        tokens[sid] = list(pr)
    live = [0, 1, 2]
    cows = 0
    for step in range(20):
        if step == 5:
            bm.fork(0, 3)
            tokens[3] = list(tokens[0])
            live.append(3)
        new = rng.integers(0, VOCAB, len(live))
        slots, pairs = bm.append_batch(live, new)
        if len(pairs):
            cows += len(pairs)
            pkv.copy_blocks([kc], [vc], torch.from_numpy(pairs).cuda())
            orc.copy_blocks([kn], [vn], pairs)
        for i, sid in enumerate(live):
            write(sid, len(tokens[sid]), [int(new[i])], [slots[i]])
            tokens[sid].append(int(new[i]))
        lens = np.array([bm.num_tokens(s) for s in live], dtype=np.int32)
        mb = int(-(-lens.max() // B))
        bt = bm.tables(live, mb)
        q = torch.randn(len(live), Hq, D, generator=g).to(DT)
        out = torch.empty(len(live), Hq, D, dtype=DT, device="cuda")
        scale = float(np.float32(D ** -0.5))
        if fp8:
            pkv.paged_attention_decode_fp8(out, q.cuda(), kc, vc, torch.from_numpy(bt).cuda(),
                                           torch.from_numpy(lens).cuda(), scale, KS, VS, int(lens.max()))
            ref = orc.paged_attention_decode_kv(q.numpy(), oracle.F16, kn, vn, oracle.E4M3, float(np.float32(KS)),
                                                float(np.float32(VS)), bt, lens, scale)
        else:
            pkv.paged_attention_decode(out, q.cuda(), kc, vc, torch.from_numpy(bt).cuda(),
                                       torch.from_numpy(lens).cuda(), scale, int(lens.max()))
            ref = orc.paged_attention_decode(q.numpy(), kn, vn, bt, lens, scale, oracle.F16)
        assert_close(out, ref, DT, f"step {step}")
    assert cows == 1                                 # the fork's first append copied the shared partial block
    assert pkv.get_device_error() == 0
    assert np.array_equal(kc.cpu().numpy().view(np.uint8), kn.view(np.uint8))


def test_preemption_by_swap_keeps_decode_exact():
    """Sequence 1 is pre-empted at step 4: the block manager hands out host blocks, swap_blocks moves its
    K/V to a page-locked host pool, and its device blocks go back to the free stack, where sequence 0's
    next block comes from.  At step 10 it resumes into new device blocks.  Every step's decode of the
    resident sequences, and the pools at the end, match the oracle's host mirror."""
    NBs, NH = 16, 8
    rng = np.random.default_rng(31)
    g = torch.Generator().manual_seed(31)
    ek = torch.randn(VOCAB, Hkv, D, generator=g)
    ev = torch.randn(VOCAB, Hkv, D, generator=g)
    bm = BlockManager(NBs, B, prefix_caching=False, num_host_blocks=NH)
    kc = torch.zeros(NBs, B, Hkv, D, dtype=DT, device="cuda")
    vc = torch.zeros_like(kc)
    hk = torch.zeros(NH, B, Hkv, D, dtype=DT).pin_memory()
    hv = torch.zeros(NH, B, Hkv, D, dtype=DT).pin_memory()
    kn, vn = np.zeros((NBs, B, Hkv, D), np.float16), np.zeros((NBs, B, Hkv, D), np.float16)
    hkn, hvn = np.zeros((NH, B, Hkv, D), np.float16), np.zeros((NH, B, Hkv, D), np.float16)
    orc = oracle.get()
    tokens = {}

    def write(start, toks, slots):
        pos = np.arange(start, start + len(toks))
        k, v = kv_of(toks, pos, ek), kv_of(toks, pos, ev)
        sl = torch.from_numpy(np.asarray(slots, dtype=np.int64))
        pkv.reshape_and_cache(k.cuda(), v.cuda(), kc, vc, sl.cuda())
        orc.reshape_and_cache(k.numpy(), v.numpy(), kn, vn, sl.numpy(), oracle.F16)

    for sid, n in ((0, 40), (1, 30), (2, 50)):
        pr = rng.integers(0, VOCAB, n).tolist()
        bm.add_sequence(sid, pr)
        write(0, pr, bm.slots(sid, 0, n))
        tokens[sid] = pr
    live = [0, 1, 2]
    reused = False
    for step in range(16):
        if step == 4:
            pairs = bm.swap_out(1)
            freed = set(pairs[:, 0].tolist())
            pkv.swap_blocks(kc, vc, hk, hv, torch.from_numpy(pairs).cuda())
            hkn[pairs[:, 1]], hvn[pairs[:, 1]] = kn[pairs[:, 0]], vn[pairs[:, 0]]
            live.remove(1)
        if step == 10:
            pairs = bm.swap_in(1)
            pkv.swap_blocks(hk, hv, kc, vc, torch.from_numpy(pairs).pin_memory())
            kn[pairs[:, 1]], vn[pairs[:, 1]] = hkn[pairs[:, 0]], hvn[pairs[:, 0]]
            live = [0, 1, 2]
        new = rng.integers(0, VOCAB, len(live))
        slots, cow = bm.append_batch(live, new)
        assert len(cow) == 0
        for i, sid in enumerate(live):
            write(len(tokens[sid]), [int(new[i])], [slots[i]])
            tokens[sid].append(int(new[i]))
        if 4 <= step < 10:
            reused |= bool(freed & {int(b) for b in bm.block_table(0)})
        lens = np.array([bm.num_tokens(s) for s in live], dtype=np.int32)
        bt = bm.tables(live, int(-(-lens.max() // B)))
        q = torch.randn(len(live), Hq, D, generator=g).to(DT)
        out = torch.empty(len(live), Hq, D, dtype=DT, device="cuda")
        scale = float(np.float32(D ** -0.5))
        pkv.paged_attention_decode(out, q.cuda(), kc, vc, torch.from_numpy(bt).cuda(), torch.from_numpy(lens).cuda(),
                                   scale, int(lens.max()))
        ref = orc.paged_attention_decode(q.numpy(), kn, vn, bt, lens, scale, oracle.F16)
        assert_close(out, ref, DT, f"step {step}")
    assert reused                                     # sequence 0 wrote into a block sequence 1 had released
    torch.cuda.synchronize()
    assert pkv.get_device_error() == 0
    assert np.array_equal(kc.cpu().numpy().view(np.uint16), kn.view(np.uint16))
    assert np.array_equal(vc.cpu().numpy().view(np.uint16), vn.view(np.uint16))
