"""Host block manager (C++, in libpagedkv.so) against the pages' statements and
against a plain model of the same policy, operation by operation (no GPU)."""
import numpy as np
import pytest

from oracle.block_manager_model import BlockManagerModel, NoSpace
from oracle_pins import golden
from paged_kv_cache_409_b200.block_manager import BlockManager, BlockManagerError, NoSpaceError


@pytest.fixture(autouse=True)
def _built():
    from paged_kv_cache_409_b200 import build
    build.build()


def test_on_demand_allocation_matches_pages_examples():
    g = golden()
    for e in g["blocks_needed"]:
        bm = BlockManager(64, e["block_size"], prefix_caching=False)
        bm.add_sequence(1, np.arange(e["tokens"]))
        assert len(bm.block_table(1)) == e["blocks"], e["source"]
    # generation one token at a time: the 7th block is only taken once the
    # sequence passes 96 tokens; at the 100th token 7 blocks are held
    bm = BlockManager(64, 16, prefix_caching=False)
    bm.add_sequence(1, [])
    held = []
    for t in range(100):
        bm.append(1, [t])
        held.append(len(bm.block_table(1)))
    assert held[95] == 6 and held[96] == 7 and held[99] == 7


def test_fragmentation_below_one_block():
    rng = np.random.default_rng(3)
    bm = BlockManager(4096, 16)
    for s in range(50):
        n = int(rng.integers(0, 400))
        bm.add_sequence(s, rng.integers(0, 1000, n))
        assert len(bm.block_table(s)) * 16 - n < 16


def test_slots_follow_the_block_table():
    bm = BlockManager(100, 16)
    bm.add_sequence(7, np.arange(40))
    bt = bm.block_table(7)
    slots = bm.slots(7, 0, 40)
    assert slots.tolist() == [bt[p // 16] * 16 + p % 16 for p in range(40)]
    s, pairs = bm.append(7, [1, 2, 3])
    assert s.tolist() == [bt[2] * 16 + 8, bt[2] * 16 + 9, bt[2] * 16 + 10] and len(pairs) == 0


def test_prefix_caching_reuses_the_system_prompt():
    """Case-study page, section 四: a 1500-token system prompt prefilled once is
    reused by later requests, which prefill only their own query."""
    rng = np.random.default_rng(4)
    system = rng.integers(0, 32000, 1500)
    bm = BlockManager(1000, 16)
    assert bm.add_sequence(1, np.concatenate([system, rng.integers(0, 32000, 8)])) == 0
    cached = bm.add_sequence(2, np.concatenate([system, rng.integers(0, 32000, 8)]))
    assert cached == 93 * 16                     # every full block of the shared prefix
    assert cached / 1508 >= 0.80                 # the page's "80-95% of prefill saved" at least
    assert bm.block_table(1)[:93].tolist() == bm.block_table(2)[:93].tolist()
    assert bm.block_table(1)[93] != bm.block_table(2)[93]   # the partial block is private
    assert bm.stats()["hits"] == 93


def test_cached_blocks_survive_free_and_evict_lru_first():
    bm = BlockManager(8, 4)
    bm.add_sequence(1, [1, 2, 3, 4, 5, 6, 7, 8])        # two full blocks: 0, 1 (cached)
    bm.free(1)
    st = bm.stats()
    assert st["free"] == 6 and st["evictable"] == 2 and st["cached"] == 2
    assert bm.add_sequence(2, [1, 2, 3, 4, 9]) == 4      # first block hits the cache
    assert bm.block_table(2)[0] == 0
    bm.free(2)
    bm.add_sequence(3, list(range(100, 128)))            # 7 blocks: all free ones, then an eviction
    assert bm.stats()["evictions"] >= 1


def test_fork_then_append_copies_the_shared_partial_block():
    bm = BlockManager(32, 16)
    bm.add_sequence(1, np.arange(20))                    # blocks: 1 full + 1 partial
    bm.fork(1, 2)
    last = bm.block_table(1)[1]
    assert bm.ref_count(last) == 2
    slots, pairs = bm.append(2, [99])
    assert len(pairs) == 1 and pairs[0, 0] == last
    new = bm.block_table(2)[1]
    assert pairs[0, 1] == new and new != last
    assert slots[0] == new * 16 + 4
    assert bm.ref_count(last) == 1 and bm.block_table(1)[1] == last
    assert bm.block_table(2)[0] == bm.block_table(1)[0]  # the full block stays shared


def test_out_of_space_changes_nothing():
    bm = BlockManager(4, 4)
    bm.add_sequence(1, range(12))
    before = (bm.stats(), bm.block_table(1).tolist())
    with pytest.raises(NoSpaceError):
        bm.add_sequence(2, range(100, 108))
    with pytest.raises(NoSpaceError):
        bm.append(1, range(5))
    assert (bm.stats(), bm.block_table(1).tolist()) == before


def _run_both(ops, num_blocks, B, caching):
    cpp, model = BlockManager(num_blocks, B, caching), BlockManagerModel(num_blocks, B, caching)
    for op in ops:
        kind = op[0]
        try:
            if kind == "add":
                a = cpp.add_sequence(op[1], op[2])
            elif kind == "append":
                s, p = cpp.append(op[1], op[2])
                a = (s.tolist(), [tuple(x) for x in p.tolist()])
            elif kind == "fork":
                a = cpp.fork(op[1], op[2])
            else:
                a = cpp.free(op[1])
        except NoSpaceError:
            a = "nospace"
        try:
            if kind == "add":
                b = model.add_sequence(op[1], op[2])
            elif kind == "append":
                b = model.append(op[1], op[2])
            elif kind == "fork":
                b = model.fork(op[1], op[2])
            else:
                b = model.free(op[1])
        except NoSpace:
            b = "nospace"
        assert a == b, (op, a, b)
        assert cpp.stats() == model.stats(), op
        for sid in model.seqs:
            assert cpp.block_table(sid).tolist() == model.block_table(sid), (op, sid)
            assert cpp.num_tokens(sid) == model.seqs[sid]["n"]


@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("caching", [True, False])
def test_matches_plain_model_on_random_operations(seed, caching):
    rng = np.random.default_rng(100 + seed)
    B = int(rng.choice([4, 8, 16]))
    prefixes = [rng.integers(0, 50, int(rng.integers(0, 6 * B))).tolist() for _ in range(3)]
    live, next_id, ops = [], 0, []
    for _ in range(400):
        r = rng.random()
        if r < 0.3 or not live:
            toks = prefixes[int(rng.integers(0, 3))] + rng.integers(0, 50, int(rng.integers(0, 3 * B))).tolist()
            ops.append(("add", next_id, toks))
            live.append(next_id)
            next_id += 1
        elif r < 0.7:
            ops.append(("append", live[int(rng.integers(0, len(live)))],
                        rng.integers(0, 50, int(rng.integers(1, 2 * B))).tolist()))
        elif r < 0.8:
            ops.append(("fork", live[int(rng.integers(0, len(live)))], next_id))
            live.append(next_id)
            next_id += 1
        else:
            sid = live.pop(int(rng.integers(0, len(live))))
            ops.append(("free", sid))
    # replay against both, dropping ops on sequences a failed add never created
    cpp_live = set()
    filtered = []
    model = BlockManagerModel(40, B, caching)
    for op in ops:
        if op[0] in ("append", "free", "fork") and op[1] not in cpp_live:
            continue
        filtered.append(op)
        try:
            if op[0] == "add":
                model.add_sequence(op[1], op[2])
                cpp_live.add(op[1])
            elif op[0] == "append":
                model.append(op[1], op[2])
            elif op[0] == "fork":
                model.fork(op[1], op[2])
                cpp_live.add(op[2])
            else:
                model.free(op[1])
                cpp_live.discard(op[1])
        except NoSpace:
            pass
    _run_both(filtered, 40, B, caching)


def test_append_batch_equals_one_by_one():
    rng = np.random.default_rng(9)
    a, b = BlockManager(200, 8), BlockManager(200, 8)
    for bm in (a, b):
        for s in range(6):
            bm.add_sequence(s, np.arange(5 * s + 3))
        bm.fork(2, 10)
    ids = np.array([0, 1, 2, 3, 4, 5, 10])
    for step in range(12):
        toks = rng.integers(0, 99, ids.size)
        sb, pb = b.append_batch(ids, toks)
        sa, pa = [], []
        for sid, t in zip(ids, toks):
            s1, p1 = a.append(sid, [t])
            sa += s1.tolist()
            pa += [tuple(x) for x in p1.tolist()]
        assert sb.tolist() == sa and [tuple(x) for x in pb.tolist()] == pa
    assert a.stats() == b.stats()


# ----------------------------------------------------------------------------- swapping

def test_swap_out_and_in_moves_the_table_through_the_host_pool():
    bm = BlockManager(16, 4, num_host_blocks=8)
    bm.add_sequence(1, range(10))                        # 3 blocks: 0, 1, 2
    bm.add_sequence(2, range(100, 105))                  # 2 blocks: 3, 4
    table = bm.block_table(1).tolist()
    out = bm.swap_out(1)
    assert out.tolist() == [[b, h] for b, h in zip(table, [0, 1, 2])]
    st = bm.stats()
    assert st["swapped"] == 1 and st["free_host"] == 5 and st["sequences"] == 2
    assert bm.num_tokens(1) == 10
    # the released device blocks are handed out again (the two cached full blocks wait in the LRU list)
    bm.append(2, range(7))
    back = bm.swap_in(1)
    assert back[:, 0].tolist() == [0, 1, 2]
    assert bm.block_table(1).tolist() == back[:, 1].tolist()
    assert bm.stats()["free_host"] == 8 and bm.stats()["swapped"] == 0
    slots, pairs = bm.append(1, [5, 6])                  # resident again: appends continue at position 10
    assert slots.tolist() == [back[2, 1] * 4 + 2, back[2, 1] * 4 + 3] and len(pairs) == 0


def test_swapped_sequence_only_swaps_in_frees_or_counts():
    bm = BlockManager(16, 4, num_host_blocks=4)
    bm.add_sequence(1, range(6))
    bm.swap_out(1)
    for call in (lambda: bm.append(1, [1]), lambda: bm.fork(1, 2), lambda: bm.slots(1, 0, 1),
                 lambda: bm.block_table(1), lambda: bm.swap_out(1)):
        with pytest.raises(BlockManagerError) as e:
            call()
        assert not isinstance(e.value, NoSpaceError)
    assert bm._l.pkv_bm_set_host_blocks(bm._h, 8) < 0     # no resizing of the host pool while a sequence is out
    assert bm.num_tokens(1) == 6
    bm.free(1)                                            # returns its host blocks
    assert bm.stats()["free_host"] == 4 and bm.stats()["sequences"] == 0
    with pytest.raises(BlockManagerError):
        bm.swap_in(1)


def test_swap_without_room_changes_nothing():
    bm = BlockManager(6, 4, num_host_blocks=2)
    bm.add_sequence(1, range(12))                         # 3 blocks, host pool holds 2
    before = (bm.stats(), bm.block_table(1).tolist())
    with pytest.raises(NoSpaceError):
        bm.swap_out(1)
    assert (bm.stats(), bm.block_table(1).tolist()) == before
    bm2 = BlockManager(4, 4, prefix_caching=False, num_host_blocks=4)
    bm2.add_sequence(1, range(12))
    bm2.swap_out(1)
    bm2.add_sequence(2, range(100, 110))                  # 3 of the 4 device blocks
    before = bm2.stats()
    with pytest.raises(NoSpaceError):
        bm2.swap_in(1)
    assert bm2.stats() == before


@pytest.mark.parametrize("seed", range(4))
@pytest.mark.parametrize("caching", [True, False])
def test_swap_matches_plain_model_on_random_operations(seed, caching):
    """Random traces with pre-emption: every op is drawn valid for the model's current state, applied to both,
    and the outputs (slots, CoW pairs, swap pairs), counters and resident tables compared after each."""
    rng = np.random.default_rng(300 + seed)
    B = int(rng.choice([4, 8]))
    NB, NH = 64, 64
    cpp, model = BlockManager(NB, B, caching, num_host_blocks=NH), BlockManagerModel(NB, B, caching, NH)
    prefixes = [rng.integers(0, 30, int(rng.integers(0, 4 * B))).tolist() for _ in range(2)]
    next_id = 0
    swaps = 0
    for _ in range(500):
        resident = [s for s in model.seqs if not model.swapped(s)]
        out = [s for s in model.seqs if model.swapped(s)]
        r = rng.random()
        if r < 0.2 or not model.seqs:
            toks = prefixes[int(rng.integers(0, 2))] + rng.integers(0, 30, int(rng.integers(0, 2 * B))).tolist()
            op = ("add", next_id, toks)
            next_id += 1
        elif r < 0.5 and resident:
            op = ("append", resident[int(rng.integers(0, len(resident)))],
                  rng.integers(0, 30, int(rng.integers(1, B + 2))).tolist())
        elif r < 0.6 and resident:
            op = ("fork", resident[int(rng.integers(0, len(resident)))], next_id)
            next_id += 1
        elif r < 0.72 and resident:
            k = 1 if rng.random() < 0.5 else int(rng.integers(1, len(resident) + 1))
            op = ("swap_out", [int(x) for x in rng.choice(resident, size=k, replace=False)])
        elif r < 0.84 and out:
            k = 1 if rng.random() < 0.5 else int(rng.integers(1, len(out) + 1))
            op = ("swap_in", [int(x) for x in rng.choice(out, size=k, replace=False)])
        else:
            ids = list(model.seqs)
            op = ("free", ids[int(rng.integers(0, len(ids)))])
        results = []
        for side in (cpp, model):
            try:
                if op[0] == "add":
                    v = side.add_sequence(op[1], op[2])
                elif op[0] == "append":
                    s, p = side.append(op[1], op[2])
                    v = (list(map(int, s)), [tuple(map(int, x)) for x in p])
                elif op[0] == "fork":
                    v = side.fork(op[1], op[2])
                elif op[0] in ("swap_out", "swap_in"):
                    v = [tuple(map(int, x)) for x in getattr(side, op[0])(op[1])]
                else:
                    v = side.free(op[1])
            except (NoSpaceError, NoSpace):
                v = "nospace"
            results.append(v)
        assert results[0] == results[1], (op, results)
        swaps += op[0].startswith("swap") and results[0] != "nospace"
        assert cpp.stats() == model.stats(), op
        for sid in model.seqs:
            assert cpp.num_tokens(sid) == model.seqs[sid]["n"]
            if not model.swapped(sid):
                assert cpp.block_table(sid).tolist() == model.block_table(sid), (op, sid)
    assert swaps >= 30


def test_swapped_kv_survives_reuse_of_its_device_blocks():
    """A host mirror of the pools: every token's K row is a function of (position, token) written at its
    slot; CoW pairs copy blocks, swap pairs move them to a host pool and back.  After every step each
    resident sequence's rows, gathered through its table, must equal what was written -- across
    pre-emptions whose device blocks other sequences took meanwhile."""
    rng = np.random.default_rng(77)
    B, NB, NH, W = 4, 24, 16, 3
    bm = BlockManager(NB, B, num_host_blocks=NH)
    dev = np.full((NB * B, W), -1.0)
    host = np.full((NH * B, W), -1.0)
    row = lambda pos, tok: np.array([pos, tok, 1000.0 * pos + tok])
    tokens = {}

    def write(slots, start, toks):
        for i, (sl, t) in enumerate(zip(slots, toks)):
            dev[sl] = row(start + i, t)

    def move(src, dst, pairs):
        for a, b in pairs:
            dst[b * B:(b + 1) * B] = src[a * B:(a + 1) * B]

    system = rng.integers(0, 20, 9).tolist()
    next_id, preempted = 0, 0
    swapped_set = set()
    for step in range(400):
        live = [s for s in tokens if s not in swapped_set]
        r = rng.random()
        try:
            if r < 0.15 or not tokens:
                toks = system + rng.integers(0, 20, int(rng.integers(0, 6))).tolist()
                cached = bm.add_sequence(next_id, toks)
                write(bm.slots(next_id, cached, len(toks) - cached), cached, toks[cached:])
                tokens[next_id] = toks
                next_id += 1
            elif r < 0.55 and live:
                sid = live[int(rng.integers(0, len(live)))]
                t = int(rng.integers(0, 20))
                slots, pairs = bm.append(sid, [t])
                move(dev, dev, pairs)
                write(slots, len(tokens[sid]), [t])
                tokens[sid].append(t)
            elif r < 0.65 and live:
                sid = live[int(rng.integers(0, len(live)))]
                bm.fork(sid, next_id)
                tokens[next_id] = list(tokens[sid])
                next_id += 1
            elif r < 0.8 and live:
                group = [int(x) for x in rng.choice(live, size=int(rng.integers(1, min(3, len(live)) + 1)),
                                                    replace=False)]
                move(dev, host, bm.swap_out(group))
                swapped_set.update(group)
                preempted += 1
            elif r < 0.92 and swapped_set:
                out = sorted(swapped_set)
                group = [int(x) for x in rng.choice(out, size=int(rng.integers(1, min(3, len(out)) + 1)),
                                                    replace=False)]
                move(host, dev, bm.swap_in(group))
                swapped_set.difference_update(group)
            else:
                sid = list(tokens)[int(rng.integers(0, len(tokens)))]
                bm.free(sid)
                del tokens[sid]
                swapped_set.discard(sid)
        except NoSpaceError:
            pass
        for sid, toks in tokens.items():
            if sid in swapped_set:
                continue
            got = dev[bm.slots(sid, 0, len(toks))] if toks else np.zeros((0, W))
            want = np.array([row(p, t) for p, t in enumerate(toks)]).reshape(-1, W)
            assert np.array_equal(got, want), (step, sid)
    assert preempted >= 20


def test_group_swap_keeps_shared_blocks_shared():
    """Two samples of one request (a fork) share their prompt blocks: swapped out together, each shared block
    crosses to the host once; swapped in together, both tables point at one device copy again, and the
    shared partial last block is still copied on the first divergent append."""
    bm = BlockManager(32, 4, prefix_caching=False, num_host_blocks=16)
    bm.add_sequence(1, range(10))                          # blocks 0, 1 full, 2 partial
    bm.fork(1, 2)
    bm.append(2, [50, 51])                                 # CoW of block 2; sample 2 diverges
    t1, t2 = bm.block_table(1).tolist(), bm.block_table(2).tolist()
    assert t1[:2] == t2[:2] and t1[2] != t2[2]
    out = bm.swap_out([1, 2])
    assert out[:, 0].tolist() == [t1[0], t1[1], t1[2], t2[2]]      # distinct blocks, first appearance
    assert bm.stats()["free_host"] == 12 and bm.stats()["swapped"] == 2
    back = bm.swap_in([2, 1])
    assert len(back) == 4 and set(back[:, 0].tolist()) == set(out[:, 1].tolist())
    n1, n2 = bm.block_table(1).tolist(), bm.block_table(2).tolist()
    assert n1[:2] == n2[:2] and n1[2] != n2[2]
    assert bm.ref_count(n1[0]) == 2 and bm.ref_count(n1[2]) == 1 and bm.ref_count(n2[2]) == 1
    assert bm.stats()["free_host"] == 16
    bm.fork(1, 3)                                          # a new sample shares the restored partial block
    slots, pairs = bm.append(3, [9])
    assert len(pairs) == 1 and pairs[0, 0] == n1[2]


def test_group_swap_in_part_of_a_group():
    """Swapping in one sample of a swapped-out pair copies the shared blocks for it; the host copies stay
    for the other sample until it is swapped in or freed."""
    bm = BlockManager(32, 4, prefix_caching=False, num_host_blocks=8)
    bm.add_sequence(1, range(8))                           # two full blocks
    bm.fork(1, 2)
    out = bm.swap_out([1, 2])
    assert len(out) == 2 and bm.stats()["free_host"] == 6
    a = bm.swap_in(1)
    assert a[:, 0].tolist() == out[:, 1].tolist() and bm.stats()["free_host"] == 6
    bm.free(2)                                             # drops the last host references
    assert bm.stats()["free_host"] == 8
    with pytest.raises(BlockManagerError):
        bm.swap_out([1, 1])                                # repeated id


def test_swap_in_then_swap_out_in_one_step_reuses_a_host_block_in_call_order():
    """Swap-in returns its host blocks to the host free stack at once, so a swap-out made right after it
    may target one of them.  Applying each call's copies in the order of the calls (swap-in's host ->
    device first) keeps both sequences' K/V intact; the reverse order would overwrite A's saved rows."""
    B, NB, NH = 4, 8, 2
    bm = BlockManager(NB, B, prefix_caching=False, num_host_blocks=NH)
    dev = np.full((NB * B, 2), -1.0)
    host = np.full((NH * B, 2), -1.0)

    def move(src, dst, pairs):
        for a, b in pairs:
            dst[b * B:(b + 1) * B] = src[a * B:(a + 1) * B]

    for sid in (1, 2):
        bm.add_sequence(sid, [sid] * 6)                    # two blocks each, the second partial
        for p, sl in enumerate(bm.slots(sid, 0, 6)):
            dev[sl] = (sid, p)
    move(dev, host, bm.swap_out(1))                        # A = 1 fills the whole host pool
    pin = bm.swap_in(1)                                    # A's host blocks are free again ...
    pout = bm.swap_out(2)                                  # ... and B = 2 is saved into them
    assert set(pin[:, 0].tolist()) & set(pout[:, 1].tolist())
    move(host, dev, pin)                                   # call order: A's copies in first
    move(dev, host, pout)
    assert np.array_equal(dev[bm.slots(1, 0, 6)], np.array([(1.0, p) for p in range(6)]))
    move(host, dev, bm.swap_in(2))
    assert np.array_equal(dev[bm.slots(2, 0, 6)], np.array([(2.0, p) for p in range(6)]))
