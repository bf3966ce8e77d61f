"""Seeded synthetic workloads for the paged KV-cache path.

This module only draws inputs: context lengths, block placement, and N(0, 1)
query / key / value contents.  It holds none of the attention arithmetic; the
one index computation it needs (turning positions into physical slots) comes
from :mod:`paging`.  The same workload object feeds the CUDA library and the
CPU oracle in the tests.

Shapes follow the models named on the pages: the Llama-2-7B figures of the
tutorial page ("4.1 核心原理", 32 layers x 4096 hidden = 32 heads x d 128) and
the 70B example of the guide page ("KV Cache 是什么", L=80, H=64, D=128), here
with 8 KV heads (grouped-query attention).  Block size 16 is the pages'
default ("PagedAttention 的解法"; "--block-size" advice on the tutorial page,
which also recommends 32 for long generations).

Recipes (all integers drawn inclusive, ``numpy.random.default_rng(seed)``):
  * block placement: the pool holds ceil(1.1 x blocks in use) blocks unless a
    size is given; sequences take, in order, the first blocks of one seeded
    permutation of the pool, so logically adjacent blocks are scattered;
  * tensor contents: ``torch.randn`` from a ``torch.Generator`` seeded with
    the same seed, generated in fp32 on the target device and rounded to the
    storage dtype (round-to-nearest-even);
  * unused table entries are -1; with ``poison=True`` every pool slot that
    holds no live token is filled with NaN, so a kernel that reads one shows
    it in its output.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import List, Optional

import numpy as np
import torch

from . import paging

DTYPES = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}
DTYPE_NAMES = {v: k for k, v in DTYPES.items()}


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def fill_normal(t: torch.Tensor, gen: torch.Generator, chunk: int = 1 << 26) -> torch.Tensor:
    """Fill ``t`` with N(0, 1) drawn in fp32 and rounded to ``t.dtype``."""
    flat = t.view(-1)
    for i in range(0, flat.numel(), chunk):
        n = min(chunk, flat.numel() - i)
        flat[i:i + n] = torch.randn(n, generator=gen, device=t.device, dtype=torch.float32).to(t.dtype)
    return t


def randn(shape, dtype, gen, device) -> torch.Tensor:
    return fill_normal(torch.empty(shape, dtype=dtype, device=device), gen)


def randn_e4m3(shape, scale: float, gen, device, chunk: int = 1 << 26) -> torch.Tensor:
    """uint8 E4M3 codes of N(0, 1) values drawn in fp32 and divided by ``scale``
    (torch's float8_e4m3fn cast, magnitudes clamped to 448 first)."""
    out = torch.empty(shape, dtype=torch.uint8, device=device)
    flat = out.view(-1)
    for i in range(0, flat.numel(), chunk):
        n = min(chunk, flat.numel() - i)
        x = torch.randn(n, generator=gen, device=device, dtype=torch.float32) / scale
        flat[i:i + n] = x.clamp_(-448.0, 448.0).to(torch.float8_e4m3fn).view(torch.uint8)
    return out


def pool_size(blocks_in_use: int, free_fraction: float = 0.1) -> int:
    """Pool of the blocks in use plus ``free_fraction`` free blocks (rounded up)."""
    tenths = int(round(free_fraction * 10))
    return blocks_in_use + (blocks_in_use * tenths + 9) // 10


def place_blocks(rng, blocks_per_seq, num_blocks: int, max_blocks_per_seq: Optional[int] = None):
    """Scatter each sequence's logical blocks over the pool.

    Returns int32 ``[num_seqs, max_blocks_per_seq]`` tables (-1 = unused) and
    the permutation tail of free block ids.
    """
    blocks_per_seq = [int(b) for b in blocks_per_seq]
    total = sum(blocks_per_seq)
    if total > num_blocks:
        raise ValueError("pool too small")
    mb = max_blocks_per_seq or max(1, max(blocks_per_seq, default=1))
    perm = rng.permutation(num_blocks).astype(np.int32)
    bt = np.full((len(blocks_per_seq), mb), -1, dtype=np.int32)
    k = 0
    for s, nb in enumerate(blocks_per_seq):
        bt[s, :nb] = perm[k:k + nb]
        k += nb
    return bt, perm[k:]


def live_slots(block_tables: np.ndarray, lens, block_size: int) -> np.ndarray:
    """Slots of positions [0, lens[s]) of every sequence."""
    seq = np.repeat(np.arange(len(lens), dtype=np.int64), np.asarray(lens, dtype=np.int64))
    pos = np.concatenate([np.arange(int(n), dtype=np.int64) for n in lens]) if len(lens) else np.zeros(0, np.int64)
    return paging.slot_mapping(block_tables, seq, pos, block_size)


def poison_pool(cache: torch.Tensor, keep_slots: np.ndarray):
    """Set every slot of ``cache`` ([NB, B, Hkv, D]) outside ``keep_slots`` to NaN
    (code 0x7F in a uint8 E4M3 pool)."""
    nb, b = cache.shape[:2]
    mask = torch.ones(nb * b, dtype=torch.bool)
    mask[torch.from_numpy(np.asarray(keep_slots, dtype=np.int64))] = False
    rows = cache.view(nb * b, -1)
    rows[mask.to(cache.device)] = 0x7F if cache.dtype == torch.uint8 else float("nan")


@dataclass
class DecodeWorkload:
    """One decode step: append one token per sequence, then attend.

    ``context_lens`` count the appended token; its K/V go to position
    ``context_lens - 1`` through ``slot_mapping``.  Layer ``l`` has its own
    pools, query and new K/V; block tables are shared by all layers.
    """
    name: str
    num_seqs: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    dtype: torch.dtype
    scale: float
    num_blocks: int
    context_lens: np.ndarray
    block_tables: np.ndarray
    slot_mapping: np.ndarray
    key_caches: List[torch.Tensor]
    value_caches: List[torch.Tensor]
    queries: List[torch.Tensor]
    new_keys: List[torch.Tensor]
    new_values: List[torch.Tensor]
    extra: dict = field(default_factory=dict)

    @property
    def num_layers(self):
        return len(self.key_caches)

    @property
    def max_blocks_per_seq(self):
        return self.block_tables.shape[1]

    @property
    def max_context_len(self):
        return int(self.context_lens.max()) if len(self.context_lens) else 0

    @property
    def fp8(self) -> bool:
        """Pools of uint8 E4M3 codes (scales in ``extra``) instead of ``dtype`` elements."""
        return self.key_caches[0].dtype == torch.uint8

    def kv_bytes(self) -> int:
        """Bytes of K and V the attention must read once: sum_s 2 c_s Hkv D T, all layers."""
        t = self.key_caches[0].element_size()
        return int(2 * int(self.context_lens.astype(np.int64).sum()) * self.num_kv_heads * self.head_dim * t
                   * self.num_layers)


def decode_workload(name, context_lens, num_q_heads, num_kv_heads, head_dim, block_size, dtype, *,
                    seed, device="cpu", num_blocks=None, num_layers=1, poison=False,
                    max_blocks_per_seq=None, scale=None, fp8_scales=None) -> DecodeWorkload:
    """``fp8_scales=(k_scale, v_scale)`` makes the pools uint8 E4M3 codes of
    N(0, 1) / scale; queries and new tokens stay in ``dtype``."""
    rng = np.random.default_rng(seed)
    gen = _gen(seed, device)
    lens = np.asarray(context_lens, dtype=np.int32)
    S = len(lens)
    bps = paging.blocks_needed(lens, block_size) if S else np.zeros(0, np.int64)
    in_use = int(np.sum(bps))
    nb = num_blocks if num_blocks is not None else pool_size(max(in_use, 1))
    bt, _ = place_blocks(rng, bps, nb, max_blocks_per_seq)
    slots = paging.slot_mapping(bt, np.arange(S), lens.astype(np.int64) - 1, block_size) if S else \
        np.zeros(0, np.int64)
    kc, vc, qs, nk, nv = [], [], [], [], []
    for _ in range(num_layers):
        if fp8_scales is None:
            kc.append(randn((nb, block_size, num_kv_heads, head_dim), dtype, gen, device))
            vc.append(randn((nb, block_size, num_kv_heads, head_dim), dtype, gen, device))
        else:
            kc.append(randn_e4m3((nb, block_size, num_kv_heads, head_dim), fp8_scales[0], gen, device))
            vc.append(randn_e4m3((nb, block_size, num_kv_heads, head_dim), fp8_scales[1], gen, device))
        qs.append(randn((S, num_q_heads, head_dim), dtype, gen, device))
        nk.append(randn((S, num_kv_heads, head_dim), dtype, gen, device))
        nv.append(randn((S, num_kv_heads, head_dim), dtype, gen, device))
    if poison:
        keep = live_slots(bt, lens, block_size)
        for c in kc + vc:
            poison_pool(c, keep)
    sc = float(np.float32(1.0 / math.sqrt(head_dim))) if scale is None else float(np.float32(scale))
    extra = {} if fp8_scales is None else {"k_scale": float(np.float32(fp8_scales[0])),
                                           "v_scale": float(np.float32(fp8_scales[1]))}
    return DecodeWorkload(name, S, num_q_heads, num_kv_heads, head_dim, block_size, dtype, sc, nb, lens, bt,
                          slots, kc, vc, qs, nk, nv, extra)


# --------------------------------------------------------------------------
# The five named workloads.
# --------------------------------------------------------------------------

def tiny_decode_f32(device="cpu", poison=False):
    """4 sequences, context {1,17,33,100}, 4 heads, d 64, block 16, pool of 32 blocks, fp32."""
    return decode_workload("tiny_decode_f32", [1, 17, 33, 100], 4, 4, 64, 16, torch.float32, seed=1001,
                           device=device, num_blocks=32, poison=poison)


def llama7b_decode_f16(device="cpu", num_seqs=64, poison=False, seed=1002):
    """64 sequences, context U[128, 2048], 32 heads = 32 KV heads, d 128, block 16, fp16."""
    rng = np.random.default_rng(seed)
    lens = rng.integers(128, 2048 + 1, size=num_seqs)
    return decode_workload("llama7b_decode_f16", lens, 32, 32, 128, 16, torch.float16, seed=seed,
                           device=device, poison=poison)


# FP8 pools: a scale that maps 4 standard deviations of N(0, 1) to E4M3's 448
# for K, and a different one for V, neither a power of two.
FP8_K_SCALE = 4.0 / 448.0
FP8_V_SCALE = 5.0 / 448.0


def llama7b_decode_fp8(device="cpu", num_seqs=64, poison=False, seed=1002):
    """The llama7b batch (64 sequences, context U[128, 2048], 32 = 32 KV heads,
    d 128, block 16) with FP8 E4M3 pools and an fp16 query."""
    rng = np.random.default_rng(seed)
    lens = rng.integers(128, 2048 + 1, size=num_seqs)
    return decode_workload("llama7b_decode_fp8", lens, 32, 32, 128, 16, torch.float16, seed=seed, device=device,
                           poison=poison, fp8_scales=(FP8_K_SCALE, FP8_V_SCALE))


def gqa70b_decode_fp8(device="cpu", num_seqs=256, num_layers=80, poison=False, seed=1003):
    """The gqa70b batch (256 sequences, lognormal context, 64 q heads over 8 KV
    heads, d 128, block 16, 80 layers) with FP8 E4M3 pools and a bf16 query."""
    rng = np.random.default_rng(seed)
    lens = np.clip(np.rint(np.exp(rng.normal(math.log(1024.0), 1.0, size=num_seqs))), 16, 4096).astype(np.int64)
    return decode_workload("gqa70b_decode_fp8", lens, 64, 8, 128, 16, torch.bfloat16, seed=seed, device=device,
                           num_layers=num_layers, poison=poison, fp8_scales=(FP8_K_SCALE, FP8_V_SCALE))


def gqa70b_decode_bf16(device="cpu", num_seqs=256, num_layers=80, poison=False, seed=1003):
    """256 sequences, lognormal context (median 1024, sigma 1, clipped to [16, 4096]),
    64 query heads over 8 KV heads, d 128, block 16, bf16, 80 layer caches."""
    rng = np.random.default_rng(seed)
    lens = np.clip(np.rint(np.exp(rng.normal(math.log(1024.0), 1.0, size=num_seqs))), 16, 4096).astype(np.int64)
    return decode_workload("gqa70b_decode_bf16", lens, 64, 8, 128, 16, torch.bfloat16, seed=seed,
                           device=device, num_layers=num_layers, poison=poison)


@dataclass
class SharedPrefixWorkload:
    """Shared-prefix decode with copy-on-write.

    Setup: every table points at the same ``prefix_blocks`` physical blocks
    (the last one partial).  ``cow_pairs`` copy the partial shared block to a
    private block per sequence, after which ``tables_after_cow`` replace the
    shared id of that logical block; ``private_*`` are the tokens each
    sequence wrote after the prefix.  The decode step then appends one token
    per sequence (``step``, a :class:`DecodeWorkload` over the final tables).
    """
    prefix_len: int
    prefix_blocks: np.ndarray
    private_lens: np.ndarray
    tables_before_cow: np.ndarray
    cow_pairs: np.ndarray
    private_keys: torch.Tensor
    private_values: torch.Tensor
    private_slots: np.ndarray
    step: DecodeWorkload


def shared_prefix_decode_f16(device="cpu", num_seqs=128, prefix_len=1500, private_lo=8, private_hi=64,
                             poison=False, seed=1004, num_q_heads=32, num_kv_heads=32, head_dim=128,
                             block_size=16):
    """128 sequences sharing a 1500-token prefix (94 blocks, last partial) plus
    U{8..64} private tokens each; 32 heads, d 128, block 16, fp16."""
    rng = np.random.default_rng(seed)
    gen = _gen(seed, device)
    dtype = torch.float16
    B = block_size
    priv = rng.integers(private_lo, private_hi + 1, size=num_seqs)
    final_lens = prefix_len + priv + 1                       # + the token appended by the step
    n_prefix_blocks = paging.blocks_needed(prefix_len, B)
    last_shared = n_prefix_blocks - 1                        # logical index of the partial block
    partial = prefix_len % B != 0
    total_blocks = paging.blocks_needed(final_lens, B)
    # private blocks: the CoW copy of the partial block (if any) and the blocks past the prefix
    private_blocks = total_blocks - n_prefix_blocks + (1 if partial else 0)
    nb = pool_size(int(n_prefix_blocks + private_blocks.sum()))
    perm = rng.permutation(nb).astype(np.int32)
    prefix_ids = perm[:n_prefix_blocks]
    k = n_prefix_blocks
    mb = int(total_blocks.max())
    before = np.full((num_seqs, mb), -1, dtype=np.int32)
    after = np.full((num_seqs, mb), -1, dtype=np.int32)
    pairs = []
    for s in range(num_seqs):
        before[s, :n_prefix_blocks] = prefix_ids
        after[s, :n_prefix_blocks] = prefix_ids
        rest = int(total_blocks[s] - n_prefix_blocks)
        if partial:
            cow = perm[k]
            k += 1
            pairs.append((int(prefix_ids[last_shared]), int(cow)))
            after[s, last_shared] = cow
            before[s, n_prefix_blocks:n_prefix_blocks + rest] = perm[k:k + rest]
            after[s, n_prefix_blocks:n_prefix_blocks + rest] = perm[k:k + rest]
        else:
            before[s, n_prefix_blocks:n_prefix_blocks + rest] = perm[k:k + rest]
            after[s, n_prefix_blocks:n_prefix_blocks + rest] = perm[k:k + rest]
        k += rest
    Hkv, D = num_kv_heads, head_dim
    kc = randn((nb, B, Hkv, D), dtype, gen, device)
    vc = randn((nb, B, Hkv, D), dtype, gen, device)
    seq = np.repeat(np.arange(num_seqs), priv)
    pos = np.concatenate([prefix_len + np.arange(p) for p in priv])
    pslots = paging.slot_mapping(after, seq, pos, B)
    pk = randn((int(priv.sum()), Hkv, D), dtype, gen, device)
    pv = randn((int(priv.sum()), Hkv, D), dtype, gen, device)
    q = randn((num_seqs, num_q_heads, D), dtype, gen, device)
    nk = randn((num_seqs, Hkv, D), dtype, gen, device)
    nv = randn((num_seqs, Hkv, D), dtype, gen, device)
    if poison:
        # live before the step: the shared prefix plus each sequence's private tokens
        keep = np.concatenate([live_slots(before[:1], [prefix_len], B), pslots])
        for c in (kc, vc):
            poison_pool(c, keep)
    step_slots = paging.slot_mapping(after, np.arange(num_seqs), final_lens - 1, B)
    step = DecodeWorkload("shared_prefix_decode_f16", num_seqs, num_q_heads, Hkv, D, B, dtype,
                          float(np.float32(1.0 / math.sqrt(D))), nb, final_lens.astype(np.int32), after,
                          step_slots, [kc], [vc], [q], [nk], [nv])
    return SharedPrefixWorkload(prefix_len, prefix_ids, priv.astype(np.int32), before,
                                np.asarray(pairs, dtype=np.int64).reshape(-1, 2), pk, pv, pslots, step)


@dataclass
class MixedWorkload:
    """Continuous-batching step: decode sequences plus chunked-prefill chunks
    over one pool.  ``append_*`` hold every token the step writes (decode
    tokens first, then each chunk's tokens in order)."""
    decode: DecodeWorkload
    chunk_lens: np.ndarray          # n_r
    chunk_c0: np.ndarray            # prior context c0_r
    chunk_tables: np.ndarray        # [R, MB]
    chunk_query: torch.Tensor       # [sum n_r, Hq, D]
    query_start_loc: np.ndarray     # [R + 1]
    seq_lens: np.ndarray            # c0_r + n_r
    append_keys: torch.Tensor
    append_values: torch.Tensor
    append_slots: np.ndarray


def mixed_workload(name, decode_lens, chunk_c0, chunk_lens, num_q_heads, num_kv_heads, head_dim, block_size,
                   dtype, *, seed, device="cpu", poison=False, fp8_scales=None):
    """``fp8_scales=(k_scale, v_scale)`` makes the pools uint8 E4M3 codes of
    N(0, 1) / scale; queries and appended tokens stay in ``dtype``."""
    rng = np.random.default_rng(seed)
    gen = _gen(seed, device)
    B = block_size
    dl = np.asarray(decode_lens, dtype=np.int64)
    c0 = np.asarray(chunk_c0, dtype=np.int64)
    n = np.asarray(chunk_lens, dtype=np.int64)
    sl = c0 + n
    S, R = len(dl), len(c0)
    bps = np.concatenate([paging.blocks_needed(dl, B), paging.blocks_needed(sl, B)]).astype(np.int64)
    nb = pool_size(int(bps.sum()))
    bt_all, _ = place_blocks(rng, bps, nb)
    dbt, cbt = bt_all[:S].copy(), bt_all[S:].copy()
    Hkv, D = num_kv_heads, head_dim
    if fp8_scales is None:
        kc = randn((nb, B, Hkv, D), dtype, gen, device)
        vc = randn((nb, B, Hkv, D), dtype, gen, device)
    else:
        kc = randn_e4m3((nb, B, Hkv, D), fp8_scales[0], gen, device)
        vc = randn_e4m3((nb, B, Hkv, D), fp8_scales[1], gen, device)
    dq = randn((S, num_q_heads, D), dtype, gen, device)
    cq = randn((int(n.sum()), num_q_heads, D), dtype, gen, device)
    ak = randn((S + int(n.sum()), Hkv, D), dtype, gen, device)
    av = randn((S + int(n.sum()), Hkv, D), dtype, gen, device)
    dslots = paging.slot_mapping(dbt, np.arange(S), dl - 1, B)
    cseq = np.repeat(np.arange(R), n)
    cpos = np.concatenate([c0[r] + np.arange(n[r]) for r in range(R)]) if R else np.zeros(0, np.int64)
    cslots = paging.slot_mapping(cbt, cseq, cpos, B) if R else np.zeros(0, np.int64)
    if poison:
        keep = np.concatenate([live_slots(dbt, dl, B), live_slots(cbt, sl, B)])
        for c in (kc, vc):
            poison_pool(c, keep)
    qsl = np.concatenate([[0], np.cumsum(n)]).astype(np.int32)
    extra = {} if fp8_scales is None else {"k_scale": float(np.float32(fp8_scales[0])),
                                           "v_scale": float(np.float32(fp8_scales[1]))}
    dec = DecodeWorkload(name, S, num_q_heads, Hkv, D, B, dtype, float(np.float32(1.0 / math.sqrt(D))), nb,
                         dl.astype(np.int32), dbt, dslots, [kc], [vc], [dq], [ak[:S]], [av[:S]], extra)
    return MixedWorkload(dec, n.astype(np.int32), c0.astype(np.int32), cbt, cq, qsl, sl.astype(np.int32), ak, av,
                         np.concatenate([dslots, cslots]).astype(np.int64))


def _mixed_lengths(seed, num_decode, num_chunks, decode_lo, decode_hi, c0_hi, full_decode=192):
    """Decode context lengths, then the chunks' prior contexts c0, from one
    stream.  The lengths are drawn for at least the full 192-sequence batch and
    cut to num_decode, so a smaller decode batch (a profiling case) keeps the
    same chunks."""
    rng = np.random.default_rng(seed)
    dl = rng.integers(decode_lo, decode_hi + 1, size=max(num_decode, full_decode))[:num_decode]
    c0 = rng.integers(0, c0_hi + 1, size=num_chunks)
    return dl, c0


def mixed_step_bf16(device="cpu", num_decode=192, num_chunks=4, chunk_len=512, poison=False, seed=1005,
                    decode_lo=256, decode_hi=32768, c0_hi=8192):
    """192 decode sequences (context U[256, 32768]) plus 4 prefill chunks of 512
    tokens over prior context U[0, 8192]; 32 q heads over 8 KV heads, d 128,
    block 32, bf16."""
    dl, c0 = _mixed_lengths(seed, num_decode, num_chunks, decode_lo, decode_hi, c0_hi)
    n = np.full(num_chunks, chunk_len)
    return mixed_workload("mixed_step_bf16", dl, c0, n, 32, 8, 128, 32, torch.bfloat16, seed=seed, device=device,
                          poison=poison)


def mixed_step_fp8(device="cpu", num_decode=192, num_chunks=4, chunk_len=512, poison=False, seed=1005,
                   decode_lo=256, decode_hi=32768, c0_hi=8192):
    """The mixed step (192 decode sequences + 4 prefill chunks of 512, 32 q
    heads over 8 KV heads, d 128, block 32, bf16 queries) on E4M3 pools."""
    dl, c0 = _mixed_lengths(seed, num_decode, num_chunks, decode_lo, decode_hi, c0_hi)
    n = np.full(num_chunks, chunk_len)
    return mixed_workload("mixed_step_fp8", dl, c0, n, 32, 8, 128, 32, torch.bfloat16, seed=seed, device=device,
                          poison=poison, fp8_scales=(FP8_K_SCALE, FP8_V_SCALE))


def multi_token_decode_bf16(device="cpu", num_seqs=64, draft_lo=2, draft_hi=6, c0_lo=256, c0_hi=4096,
                            poison=False, seed=1006):
    """Multi-token decode (speculative verification): each of 64 sequences
    appends n ~ U{2..6} draft tokens after a context of U[256, 4096] tokens and
    attends causally over the whole cache; 32 q heads over 8 KV heads, d 128,
    block 32, bf16."""
    rng = np.random.default_rng(seed)
    c0 = rng.integers(c0_lo, c0_hi + 1, size=num_seqs)
    n = rng.integers(draft_lo, draft_hi + 1, size=num_seqs)
    return mixed_workload("multi_token_decode_bf16", [], c0, n, 32, 8, 128, 32, torch.bfloat16, seed=seed,
                          device=device, poison=poison)


CONFIGS = {
    "tiny_decode_f32": tiny_decode_f32,
    "llama7b_decode_f16": llama7b_decode_f16,
    "gqa70b_decode_bf16": gqa70b_decode_bf16,
    "shared_prefix_decode_f16": shared_prefix_decode_f16,
    "mixed_step_bf16": mixed_step_bf16,
    "multi_token_decode_bf16": multi_token_decode_bf16,
    "llama7b_decode_fp8": llama7b_decode_fp8,
    "mixed_step_fp8": mixed_step_fp8,
    "gqa70b_decode_fp8": gqa70b_decode_fp8,
}
