"""Plain model of the host block manager's policy (test infrastructure).

It restates, with Python lists and dicts, the policy written in
``include/pagedkv_block_manager.h``: a free stack with block 0 on top, blocks
taken on demand, reference counts, copy-on-write of a shared partial last
block, a prefix cache of full blocks keyed by their exact content chain
(parent block's key, token ids) -- no hashing -- whose unreferenced blocks sit
in an LRU list, oldest evicted first, and swapping of whole sequences to a
host pool with its own free stack.  The data model it follows is that of the
vLLM case-study page ("vLLM 与 PagedAttention", sections 二 and 四) and the
298.name page's ``PagedKVCache`` sketch.  The tests compare the C++ manager to
this model operation by operation.
"""
from __future__ import annotations


class NoSpace(Exception):
    pass


class BlockManagerModel:
    def __init__(self, num_blocks, block_size, prefix_caching=True, num_host_blocks=0):
        self.B = block_size
        self.prefix_caching = prefix_caching
        self.free_stack = list(range(num_blocks - 1, -1, -1))  # block 0 on top (end of the list)
        self.ref = [0] * num_blocks
        self.key_of = [None] * num_blocks
        self.cache = {}
        self.lru = []  # oldest first
        self.seqs = {}
        self.hits = self.evictions = self.cows = 0
        self.host_free = list(range(num_host_blocks - 1, -1, -1))  # host block 0 on top
        self.host_ref = [0] * num_host_blocks

    # -- blocks
    def _take(self):
        if self.free_stack:
            b = self.free_stack.pop()
        elif self.lru:
            b = self.lru.pop(0)
            del self.cache[self.key_of[b]]
            self.key_of[b] = None
            self.evictions += 1
        else:
            raise NoSpace()
        self.ref[b] = 1
        return b

    def _release(self, b):
        self.ref[b] -= 1
        if self.ref[b] == 0:
            (self.lru if self.key_of[b] is not None else self.free_stack).append(b)

    def _register_full(self, seq, b, toks):
        key = (seq["last_key"], tuple(toks))
        if self.prefix_caching and self.key_of[b] is None and key not in self.cache:
            self.cache[key] = b
            self.key_of[b] = key
        seq["last_key"] = key

    def _available(self):
        return len(self.free_stack) + len(self.lru)

    # -- operations
    def add_sequence(self, sid, tokens):
        tokens = list(tokens)
        assert sid not in self.seqs
        B = self.B
        full, need = len(tokens) // B, -(-len(tokens) // B)
        hits, parent = [], None
        if self.prefix_caching:
            for i in range(full):
                key = (parent, tuple(tokens[i * B:(i + 1) * B]))
                if key not in self.cache:
                    break
                hits.append(self.cache[key])
                parent = key
        if need - len(hits) > self._available() - sum(1 for b in hits if b in self.lru):
            raise NoSpace()
        seq = {"blocks": [], "last_key": parent, "tail": [], "n": len(tokens)}
        for b in hits:
            if self.ref[b] == 0 and b in self.lru:
                self.lru.remove(b)
            self.ref[b] += 1
            seq["blocks"].append(b)
        self.hits += len(hits)
        for i in range(len(hits), need):
            b = self._take()
            seq["blocks"].append(b)
            if i < full:
                self._register_full(seq, b, tokens[i * B:(i + 1) * B])
        seq["tail"] = tokens[full * B:]
        self.seqs[sid] = seq
        return len(hits) * B

    def append(self, sid, tokens):
        seq, B = self.seqs[sid], self.B
        tokens = list(tokens)
        off0 = seq["n"] % B
        cow = bool(tokens) and off0 != 0 and self.ref[seq["blocks"][-1]] > 1
        new_blocks = -(-(off0 + len(tokens)) // B) - (1 if off0 else 0)
        if new_blocks + (1 if cow else 0) > self._available():
            raise NoSpace()
        pairs = []
        if cow:
            src = seq["blocks"][-1]
            dst = self._take()
            self._release(src)
            seq["blocks"][-1] = dst
            pairs.append((src, dst))
            self.cows += 1
        slots = []
        for t in tokens:
            if seq["n"] % B == 0:
                seq["blocks"].append(self._take())
            slots.append(seq["blocks"][-1] * B + seq["n"] % B)
            seq["tail"].append(t)
            seq["n"] += 1
            if seq["n"] % B == 0:
                self._register_full(seq, seq["blocks"][-1], seq["tail"])
                seq["tail"] = []
        return slots, pairs

    def fork(self, parent, child):
        p = self.seqs[parent]
        self.seqs[child] = {"blocks": list(p["blocks"]), "last_key": p["last_key"], "tail": list(p["tail"]),
                            "n": p["n"]}
        for b in p["blocks"]:
            self.ref[b] += 1

    def _drop_host(self, seq):
        for h in reversed(seq.pop("host")):
            self.host_ref[h] -= 1
            if self.host_ref[h] == 0:
                self.host_free.append(h)

    def free(self, sid):
        seq = self.seqs.pop(sid)
        if "host" in seq:
            self._drop_host(seq)
        for b in reversed(seq["blocks"]):
            self._release(b)

    # -- swapping (pre-empted sequences' blocks move to the host pool and back; a group's shared blocks once)
    @staticmethod
    def _group(sids):
        sids = [sids] if isinstance(sids, int) else [int(s) for s in sids]
        assert sids and len(set(sids)) == len(sids)
        return sids

    @staticmethod
    def _distinct(lists):
        out = []
        for lst in lists:
            for x in lst:
                if x not in out:
                    out.append(x)
        return out

    def swap_out(self, sids):
        seqs = [self.seqs[s] for s in self._group(sids)]
        assert all("host" not in q for q in seqs)
        distinct = self._distinct(q["blocks"] for q in seqs)
        if len(distinct) > len(self.host_free):
            raise NoSpace()
        to_host = {}
        for b in distinct:
            to_host[b] = self.host_free.pop()
        for q in seqs:
            q["host"] = [to_host[b] for b in q["blocks"]]
            for h in q["host"]:
                self.host_ref[h] += 1
            for b in reversed(q["blocks"]):
                self._release(b)
            q["blocks"] = []
        return [(b, to_host[b]) for b in distinct]

    def swap_in(self, sids):
        seqs = [self.seqs[s] for s in self._group(sids)]
        assert all("host" in q for q in seqs)
        distinct = self._distinct(q["host"] for q in seqs)
        if len(distinct) > self._available():
            raise NoSpace()
        to_dev = {}
        for h in distinct:
            d = self._take()
            self.ref[d] = 0          # counted below, one per table entry
            to_dev[h] = d
        for q in seqs:
            q["blocks"] = [to_dev[h] for h in q["host"]]
            for d in q["blocks"]:
                self.ref[d] += 1
            self._drop_host(q)
        return [(h, to_dev[h]) for h in distinct]

    def swapped(self, sid):
        return "host" in self.seqs[sid]

    def block_table(self, sid):
        return list(self.seqs[sid]["blocks"])

    def stats(self):
        return {"free": len(self.free_stack), "evictable": len(self.lru), "cached": len(self.cache),
                "hits": self.hits, "evictions": self.evictions, "cow_copies": self.cows, "sequences": len(self.seqs),
                "free_host": len(self.host_free), "swapped": sum(1 for s in self.seqs.values() if "host" in s)}
