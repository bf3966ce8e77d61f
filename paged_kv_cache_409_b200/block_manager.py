"""Host block manager of the paged KV-cache pool (ctypes binding of the C++
manager in ``libpagedkv.so``, declared in ``include/pagedkv_block_manager.h``).

It hands out blocks on demand, keeps per-sequence block tables, shares blocks
between forked sequences and between requests with a common prefix (hash-chain
prefix cache with LRU eviction), and reports the copy-on-write pairs that
``copy_blocks`` must run before a shared partial block is written.
"""
from __future__ import annotations

import ctypes

import numpy as np

from ._binding import load_library

OK, EINVAL, ENOSPACE, EBUFFER = 0, -1, -6, -7


class BlockManagerError(RuntimeError):
    def __init__(self, what, status):
        super().__init__(f"{what}: status {status}")
        self.status = status


class NoSpaceError(BlockManagerError):
    pass


_bound = False


def _lib():
    global _bound
    lib = load_library()
    if not _bound:
        P, I, I64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
        lib.pkv_bm_create.argtypes = [I64, I, I]
        lib.pkv_bm_create.restype = P
        lib.pkv_bm_destroy.argtypes = [P]
        lib.pkv_bm_destroy.restype = None
        lib.pkv_bm_add_sequence.argtypes = [P, I64, P, I64, P]
        lib.pkv_bm_append.argtypes = [P, I64, P, I64, P, P, I64, P]
        lib.pkv_bm_append_batch.argtypes = [P, P, P, I64, P, P, I64, P, P]
        lib.pkv_bm_fork.argtypes = [P, I64, I64]
        lib.pkv_bm_free.argtypes = [P, I64]
        lib.pkv_bm_slots.argtypes = [P, I64, I64, I64, P]
        lib.pkv_bm_block_table.argtypes = [P, I64, P, I64, P]
        lib.pkv_bm_num_tokens.argtypes = [P, I64]
        lib.pkv_bm_num_tokens.restype = I64
        lib.pkv_bm_stats.argtypes = [P, P, I]
        lib.pkv_bm_ref_count.argtypes = [P, I64]
        lib.pkv_bm_set_host_blocks.argtypes = [P, I64]
        lib.pkv_bm_swap_out.argtypes = [P, I64, P, I64, P]
        lib.pkv_bm_swap_in.argtypes = [P, I64, P, I64, P]
        lib.pkv_bm_swap_out_group.argtypes = [P, P, I64, P, I64, P]
        lib.pkv_bm_swap_in_group.argtypes = [P, P, I64, P, I64, P]
        for f in (lib.pkv_bm_add_sequence, lib.pkv_bm_append, lib.pkv_bm_append_batch, lib.pkv_bm_fork,
                  lib.pkv_bm_free, lib.pkv_bm_slots, lib.pkv_bm_block_table, lib.pkv_bm_stats, lib.pkv_bm_ref_count,
                  lib.pkv_bm_set_host_blocks, lib.pkv_bm_swap_out, lib.pkv_bm_swap_in, lib.pkv_bm_swap_out_group,
                  lib.pkv_bm_swap_in_group):
            f.restype = I
        _bound = True
    return lib


def _check(rc, what):
    if rc == ENOSPACE:
        raise NoSpaceError(what, rc)
    if rc < 0:
        raise BlockManagerError(what, rc)
    return rc


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


class BlockManager:
    """One pool of ``num_blocks`` blocks of ``block_size`` tokens (and, for
    swapping, a host pool of ``num_host_blocks`` blocks)."""

    STATS = ("free", "evictable", "cached", "hits", "evictions", "cow_copies", "sequences", "free_host", "swapped")

    def __init__(self, num_blocks: int, block_size: int, prefix_caching: bool = True, num_host_blocks: int = 0):
        self._l = _lib()
        self._h = self._l.pkv_bm_create(int(num_blocks), int(block_size), 1 if prefix_caching else 0)
        if not self._h:
            raise BlockManagerError("pkv_bm_create", EINVAL)
        self.num_blocks, self.block_size = int(num_blocks), int(block_size)
        if num_host_blocks:
            _check(self._l.pkv_bm_set_host_blocks(self._h, int(num_host_blocks)), "set_host_blocks")

    def close(self):
        if self._h:
            self._l.pkv_bm_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def add_sequence(self, seq_id: int, tokens) -> int:
        """Register a prompt; returns how many leading tokens were already cached."""
        t = np.ascontiguousarray(tokens, dtype=np.int32)
        cached = ctypes.c_int64(0)
        _check(self._l.pkv_bm_add_sequence(self._h, int(seq_id), _ptr(t), t.size, ctypes.byref(cached)),
               "add_sequence")
        return int(cached.value)

    def append(self, seq_id: int, tokens):
        """Append tokens; returns (slots int64 [n], cow_pairs int64 [k, 2])."""
        t = np.ascontiguousarray(tokens, dtype=np.int32)
        slots = np.empty(max(t.size, 1), dtype=np.int64)
        pairs = np.empty((1, 2), dtype=np.int64)
        n = ctypes.c_int64(0)
        _check(self._l.pkv_bm_append(self._h, int(seq_id), _ptr(t), t.size, _ptr(slots), _ptr(pairs), 1,
                                     ctypes.byref(n)), "append")
        return slots[:t.size], pairs[:n.value]

    def append_batch(self, seq_ids, tokens):
        """One token per sequence; returns (slots int64 [n], cow_pairs int64 [k, 2])."""
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        t = np.ascontiguousarray(tokens, dtype=np.int32)
        assert ids.shape == t.shape
        slots = np.empty(max(ids.size, 1), dtype=np.int64)
        pairs = np.empty((max(ids.size, 1), 2), dtype=np.int64)
        npairs, done = ctypes.c_int64(0), ctypes.c_int64(0)
        rc = self._l.pkv_bm_append_batch(self._h, _ptr(ids), _ptr(t), ids.size, _ptr(slots), _ptr(pairs), ids.size,
                                         ctypes.byref(npairs), ctypes.byref(done))
        _check(rc, f"append_batch (done {done.value} of {ids.size})")
        return slots[:ids.size], pairs[:npairs.value]

    def fork(self, parent: int, child: int):
        _check(self._l.pkv_bm_fork(self._h, int(parent), int(child)), "fork")

    def free(self, seq_id: int):
        _check(self._l.pkv_bm_free(self._h, int(seq_id)), "free")

    def _swap(self, fn, seq_ids, what):
        ids = np.atleast_1d(np.asarray(seq_ids, dtype=np.int64))
        # a sequence of n tokens holds ceil(n / block_size) blocks, resident or not
        cap = 1
        for s in ids.tolist():
            cap += -(-_check(int(self._l.pkv_bm_num_tokens(self._h, int(s))), what) // self.block_size)
        pairs = np.empty((cap, 2), dtype=np.int64)
        k = ctypes.c_int64(0)
        _check(fn(self._h, _ptr(ids), ids.size, _ptr(pairs), cap, ctypes.byref(k)), what)
        return pairs[:k.value]

    def swap_out(self, seq_ids) -> np.ndarray:
        """Pre-empt one sequence, or several together (blocks they share cross once); returns the
        (device block, host block) pairs int64 [k, 2], one per distinct block."""
        return self._swap(self._l.pkv_bm_swap_out_group, seq_ids, "swap_out")

    def swap_in(self, seq_ids) -> np.ndarray:
        """Resume swapped-out sequences (shared blocks shared again); returns the (host block, device block)
        pairs int64 [k, 2], one per distinct block."""
        return self._swap(self._l.pkv_bm_swap_in_group, seq_ids, "swap_in")

    def slots(self, seq_id: int, start: int, count: int) -> np.ndarray:
        out = np.empty(max(count, 1), dtype=np.int64)
        _check(self._l.pkv_bm_slots(self._h, int(seq_id), int(start), int(count), _ptr(out)), "slots")
        return out[:count]

    def block_table(self, seq_id: int, max_blocks: int = None) -> np.ndarray:
        n = ctypes.c_int64(0)
        if max_blocks is None:
            self._l.pkv_bm_block_table(self._h, int(seq_id), None, 0, ctypes.byref(n))
            max_blocks = n.value
        out = np.empty(max(max_blocks, 1), dtype=np.int32)
        _check(self._l.pkv_bm_block_table(self._h, int(seq_id), _ptr(out), int(max_blocks), ctypes.byref(n)),
               "block_table")
        return out[:max_blocks]

    def num_tokens(self, seq_id: int) -> int:
        return _check(int(self._l.pkv_bm_num_tokens(self._h, int(seq_id))), "num_tokens")

    def stats(self) -> dict:
        out = np.zeros(len(self.STATS), dtype=np.int64)
        self._l.pkv_bm_stats(self._h, _ptr(out), len(self.STATS))
        return dict(zip(self.STATS, out.tolist()))

    def ref_count(self, block: int) -> int:
        return _check(self._l.pkv_bm_ref_count(self._h, int(block)), "ref_count")

    def tables(self, seq_ids, max_blocks: int) -> np.ndarray:
        """int32 [len(seq_ids), max_blocks] block tables for a decode launch."""
        return np.stack([self.block_table(s, max_blocks) for s in seq_ids]) if len(seq_ids) else \
            np.zeros((0, max_blocks), np.int32)
