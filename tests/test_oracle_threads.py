"""The oracle's attention functions share (sequence, KV head) pairs out over host threads: the result must be
bit-identical whatever the thread count, since every output row is still computed by one thread in order."""
import numpy as np

import oracle


def _pools(rng, NB, B, Hkv, D):
    return rng.standard_normal((NB, B, Hkv, D)).astype(np.float32), rng.standard_normal((NB, B, Hkv, D)).astype(
        np.float32)


def test_decode_and_prefill_do_not_depend_on_the_thread_count():
    orc = oracle.get()
    rng = np.random.default_rng(11)
    S, Hq, Hkv, D, B, NB = 6, 8, 2, 16, 4, 40
    kc, vc = _pools(rng, NB, B, Hkv, D)
    lens = np.array([0, 1, 5, 17, 23, 30], dtype=np.int32)
    bt = np.stack([rng.permutation(NB)[:8] for _ in range(S)]).astype(np.int32)
    q = rng.standard_normal((S, Hq, D)).astype(np.float32)
    qsl = np.array([0, 0, 1, 4, 9, 13, 20], dtype=np.int32)
    pq = rng.standard_normal((20, Hq, D)).astype(np.float32)
    before = orc.num_threads()
    try:
        outs = []
        for n in (1, 3, max(2, before)):
            assert orc.num_threads(n) == n or orc.num_threads() == 1  # a build without OpenMP runs one thread
            outs.append((orc.paged_attention_decode(q, kc, vc, bt, lens, 0.25, oracle.F32),
                         orc.paged_attention_prefill_chunk(pq, kc, vc, bt, lens, qsl, 0.25, oracle.F32)))
    finally:
        orc.num_threads(before)
    for d, p in outs[1:]:
        assert np.array_equal(d.view(np.int64), outs[0][0].view(np.int64))
        assert np.array_equal(p.view(np.int64), outs[0][1].view(np.int64))
