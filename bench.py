"""Benchmark of the paged KV-cache decode step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--config NAME]

Default workload: the Llama-2-7B-shaped single-layer decode batch (64
sequences, 32 heads = 32 KV heads, head_dim 128, block 16, context U[128,
2048], fp16).  One step = reshape_and_cache of the 64 new tokens, then
paged decode attention (decode kernel + log-sum-exp merge) over all 64
sequences, on inputs already resident in HBM (the pools, 1.25 GB each, are
far larger than the 126 MB L2).  The step's launches are captured once in a
CUDA graph and replayed (``--no-graph`` launches them one by one).  The timed
region of exactly ``--steps`` steps is repeated until at least
``--min-timed-ms`` have been timed; ``ms_per_step`` is the median region's
time per step.  The decode-call duration for the roofline comes from a second
graph that holds only the step's decode calls, replayed the same way.
``value`` = decode tokens (sequences) per second over all ranks; multi-GPU
runs are independent replicas (weak scaling, no collective on the data path).

Other ``--config`` values time the remaining named workloads for the
report: gqa70b_decode_bf16 (80 layers per step), shared_prefix_decode_f16,
mixed_step_bf16 (append + chunked prefill + decode).

``--impl reference`` times the CPU oracle (double precision, all host cores)
on a bounded sample of the same workload: there is no runnable reference
implementation of this path.  That arm loads only the oracle, never the CUDA
library.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

L2_BYTES = 126e6  # B200 L2
METRIC = "paged decode attention tokens/s and KV GB/s as % of B200 HBM peak (1 GPU)"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return FALLBACK_PEAKS, "fallback"


# ----------------------------------------------------------------------------- workloads as timed steps

class DecodeStep:
    """reshape_and_cache + paged_attention_decode over every layer of a DecodeWorkload.

    ``library=False`` (the oracle's arm) builds only the workload's figures and
    never loads the CUDA library."""

    def __init__(self, w, layers_per_step=None, library=True):
        self.w = w
        dev = w.queries[0].device
        self.bt = torch.from_numpy(w.block_tables).to(dev)
        self.cl = torch.from_numpy(w.context_lens.astype(np.int32)).to(dev)
        self.sm = torch.from_numpy(w.slot_mapping.astype(np.int64)).to(dev)
        self.layers = layers_per_step or w.num_layers
        self.units_per_step = self.layers  # decode calls per step
        self.outs = [torch.empty_like(q) for q in w.queries]
        self.part, self.parts = 0, 1
        if library:
            import paged_kv_cache_409_b200 as pkv
            self.pkv = pkv
            self.part = pkv.decode_partition_size(w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim,
                                                  w.block_size, w.max_context_len, 3 if w.fp8 else w.dtype,
                                                  int(w.context_lens.astype(np.int64).sum()))
            need = pkv.decode_workspace_size(w.num_seqs, w.num_q_heads, w.head_dim, w.max_context_len, self.part)
            self.ws = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
            self.parts = -(-w.max_context_len // self.part) if self.part else 1
        t = w.queries[0].element_size()
        tkv = w.key_caches[0].element_size()
        self.kv_bytes = 2 * int(w.context_lens.astype(np.int64).sum()) * w.num_kv_heads * w.head_dim * tkv
        nblocks = int(((w.context_lens.astype(np.int64) + w.block_size - 1) // w.block_size).sum())
        # algorithmic bytes of one decode call: K/V once, q, out, block ids, lengths
        self.decode_bytes = self.kv_bytes + 2 * w.queries[0].numel() * t + 4 * nblocks + 4 * w.num_seqs
        self.tokens = w.num_seqs  # one generated token per sequence per step
        # K/V bytes of the distinct physical blocks a step reads (shared blocks once)
        used = [w.block_tables[s, :-(-int(c) // w.block_size)] for s, c in enumerate(w.context_lens)]
        distinct = np.unique(np.concatenate(used)).size if used else 0
        self.unique_kv_bytes = 2 * distinct * w.block_size * w.num_kv_heads * w.head_dim * tkv * self.layers

    def l2_note(self):
        """How the timed steps stand to the 126 MB L2."""
        if self.unique_kv_bytes >= 2 * L2_BYTES:
            return "inputs larger than L2 (K/V pools %.2f GB per layer)" % (
                2 * self.w.key_caches[0].numel() * self.w.key_caches[0].element_size() / 1e9)
        return ("distinct K/V blocks read per step %.3f GB, under twice the 126 MB L2: what one step reads "
                "(the shared prefix above all) may stay cached for the next unless --flush-l2"
                % (self.unique_kv_bytes / 1e9))

    def launches_per_step(self):
        return self.layers * (2 + (1 if self.parts > 1 else 0))

    def e2e_plan(self):
        w = self.w
        pairs = []
        for i in range(self.layers):
            l = i % w.num_layers
            pairs += [(w.queries[l], pinned(w.queries[l])), (w.new_keys[l], pinned(w.new_keys[l])),
                      (w.new_values[l], pinned(w.new_values[l]))]
        pairs += [(self.bt, pinned(self.bt)), (self.cl, pinned(self.cl)), (self.sm, pinned(self.sm))]
        outs = [(self.outs[i % w.num_layers], pinned(self.outs[i % w.num_layers])) for i in range(self.layers)]
        return E2EPlan(self, pairs, outs)

    def append(self, l):
        w = self.w
        if w.fp8:
            self.pkv.reshape_and_cache_fp8(w.new_keys[l], w.new_values[l], w.key_caches[l], w.value_caches[l],
                                           self.sm, w.extra["k_scale"], w.extra["v_scale"])
        else:
            self.pkv.reshape_and_cache(w.new_keys[l], w.new_values[l], w.key_caches[l], w.value_caches[l], self.sm)

    def attend(self, l):
        w = self.w
        if w.fp8:
            self.pkv.paged_attention_decode_fp8(self.outs[l], w.queries[l], w.key_caches[l], w.value_caches[l],
                                                self.bt, self.cl, w.scale, w.extra["k_scale"], w.extra["v_scale"],
                                                w.max_context_len, partition_size=self.part, workspace=self.ws)
        else:
            self.pkv.paged_attention_decode(self.outs[l], w.queries[l], w.key_caches[l], w.value_caches[l], self.bt,
                                            self.cl, w.scale, w.max_context_len, partition_size=self.part,
                                            workspace=self.ws)

    def step_call(self, l):
        """The layer's append + decode as one library call (the decode launched as the append's
        programmatic dependent)."""
        w = self.w
        if w.fp8:
            self.pkv.paged_attention_decode_step_fp8(w.new_keys[l], w.new_values[l], self.sm, self.outs[l],
                                                     w.queries[l], w.key_caches[l], w.value_caches[l], self.bt,
                                                     self.cl, w.scale, w.extra["k_scale"], w.extra["v_scale"],
                                                     w.max_context_len, partition_size=self.part, workspace=self.ws)
        else:
            self.pkv.paged_attention_decode_step(w.new_keys[l], w.new_values[l], self.sm, self.outs[l],
                                                 w.queries[l], w.key_caches[l], w.value_caches[l], self.bt, self.cl,
                                                 w.scale, w.max_context_len, partition_size=self.part,
                                                 workspace=self.ws)

    def run(self, timer=None, step=0):
        for i in range(self.layers):
            l = (step * self.layers + i) % self.w.num_layers
            if timer:  # separate calls, so that events can bracket the decode
                self.append(l)
                timer.begin()
                self.attend(l)
                timer.end()
            else:
                self.step_call(l)

    def run_units(self, step=0):
        """The step's decode calls alone (the roofline's unit), in the step's layer order."""
        for i in range(self.layers):
            self.attend((step * self.layers + i) % self.w.num_layers)


class E2EPlan:
    """Per step: copy the step's inputs from pinned host memory, run the step
    through the public API, copy its result back to pinned host memory.

    The inputs travel packed: every input tensor sits at a 256-byte aligned
    offset of one pinned host buffer, so a step's inputs cross PCIe in one
    host-to-device copy (the bytes reported include the alignment padding).
    Two device copies of the packed buffer alternate between steps, so the
    inputs of step i + 1 cross on one side stream and the result of step i on
    another while step i (or i + 1) computes on the launching stream.  Each
    step's tensors are bound to typed views of its set with ``Tensor.set_``,
    which every reference the step holds sees; the step's kernels run in
    order on one stream as before."""

    def __init__(self, step, pairs, outs):
        self.step, self.pairs, self.outs = step, pairs, outs  # pairs: (device dst, pinned src)
        offs, total = [], 0
        for _, src in pairs:
            offs.append(total)
            total += -(-src.numel() * src.element_size() // 256) * 256
        self.h2d = total
        self.d2h = sum(dst.numel() * dst.element_size() for _, dst in outs)
        # the device-timed steps' results (every step recomputes the same ones)
        self.expect = [dst.clone() for _, dst in outs]
        self.host = torch.empty(max(total, 256), dtype=torch.uint8).pin_memory()
        for (_, src), o in zip(pairs, offs):
            n = src.numel() * src.element_size()
            if n:
                self.host[o:o + n].copy_(src.contiguous().reshape(-1).view(torch.uint8))
        dev = pairs[0][0].device
        self.packed = [torch.empty(max(total, 256), dtype=torch.uint8, device=dev) for _ in range(2)]
        self.ins = [[buf[o:o + d.numel() * d.element_size()].view(d.dtype).view(d.shape)
                     for (d, _), o in zip(pairs, offs)] for buf in self.packed]
        self.res = [[torch.empty_like(d) for d, _ in outs] for _ in range(2)]
        self.up, self.down = torch.cuda.Stream(), torch.cuda.Stream()
        ev = lambda: [torch.cuda.Event(), torch.cuda.Event()]
        self.ready, self.done, self.copied = ev(), ev(), ev()

    def start(self):
        """Order both copy streams after everything issued so far (the start event)."""
        cur = torch.cuda.current_stream()
        self.up.wait_stream(cur)
        self.down.wait_stream(cur)

    def finish(self):
        """Make the launching stream wait for the last result copy."""
        torch.cuda.current_stream().wait_stream(self.down)

    def matches(self):
        """Whether the results copied back equal the device-timed steps' bit for bit (after a sync)."""
        return all(torch.equal(dst.view(torch.uint8), ref.view(torch.uint8))
                   for (_, dst), ref in zip(self.outs, self.expect))

    def run(self, i):
        s, cur = i % 2, torch.cuda.current_stream()
        self.up.wait_event(self.done[s])            # step i - 2 has finished reading set s
        with torch.cuda.stream(self.up):
            self.packed[s].copy_(self.host, non_blocking=True)  # every input of the step, one copy
            self.ready[s].record()
        cur.wait_event(self.ready[s])
        cur.wait_event(self.copied[s])               # the result of step i - 2 has left set s
        for buf, (dst, _) in zip(self.ins[s], self.pairs):
            dst.set_(buf)
        for buf, (src, _) in zip(self.res[s], self.outs):
            src.set_(buf)
        self.step.run(step=i)
        self.done[s].record(cur)
        self.down.wait_event(self.done[s])
        with torch.cuda.stream(self.down):
            for src, dst in self.outs:
                dst.copy_(src, non_blocking=True)
            self.copied[s].record()


def pinned(t):
    return t.detach().cpu().pin_memory()


class MixedStep(DecodeStep):
    """Continuous-batching step: append all tokens, chunked prefill, decode."""

    def __init__(self, m, library=True):
        super().__init__(m.decode, library=library)
        self.m = m
        dev = m.decode.queries[0].device
        self.aslots = torch.from_numpy(m.append_slots).to(dev)
        self.cbt = torch.from_numpy(m.chunk_tables).to(dev)
        self.csl = torch.from_numpy(m.seq_lens).to(dev)
        self.qsl = torch.from_numpy(m.query_start_loc).to(dev)
        self.pout = torch.empty_like(m.chunk_query)
        self.prefill_tokens = int(m.chunk_lens.sum())
        Hq, D = m.chunk_query.shape[1:]
        n, c0 = m.chunk_lens.astype(np.int64), m.chunk_c0.astype(np.int64)
        self.prefill_flops = int(4 * D * Hq * np.sum(n * c0 + n * (n + 1) // 2))
        self.pws = None
        if m.decode.fp8 and library:
            w = m.decode
            need = self.pkv.prefill_fp8_workspace_size(len(n), m.chunk_tables.shape[1], w.block_size,
                                                       w.num_kv_heads, D, m.chunk_query.shape[0], Hq, w.dtype)
            self.pws = torch.empty(need, dtype=torch.uint8, device=dev)

    def launches_per_step(self):
        if self.w.fp8:
            return self.launches_per_step_fp8()
        return 3 + (1 if self.parts > 1 else 0)

    def e2e_plan(self):
        m, w = self.m, self.w
        pairs = [(t, pinned(t)) for t in (m.chunk_query, w.queries[0], m.append_keys, m.append_values, self.aslots,
                                          self.cbt, self.csl, self.qsl, self.bt, self.cl)]
        outs = [(self.pout, pinned(self.pout)), (self.outs[0], pinned(self.outs[0]))]
        return E2EPlan(self, pairs, outs)

    def launches_per_step_fp8(self):
        return 4 + (1 if self.parts > 1 else 0)  # append, widen, query to f16, prefill, decode (+ merge)

    def run(self, timer=None, step=0):
        m, w = self.m, self.w
        if w.fp8:
            ks, vs = w.extra["k_scale"], w.extra["v_scale"]
            self.pkv.reshape_and_cache_fp8(m.append_keys, m.append_values, w.key_caches[0], w.value_caches[0],
                                           self.aslots, ks, vs)
            self.pkv.paged_attention_prefill_chunk_fp8(self.pout, m.chunk_query, w.key_caches[0], w.value_caches[0],
                                                       self.cbt, self.csl, self.qsl, int(m.chunk_lens.max()), w.scale,
                                                       ks, vs, workspace=self.pws)
        else:
            self.pkv.reshape_and_cache(m.append_keys, m.append_values, w.key_caches[0], w.value_caches[0],
                                       self.aslots)
            self.pkv.paged_attention_prefill_chunk(self.pout, m.chunk_query, w.key_caches[0], w.value_caches[0],
                                                   self.cbt, self.csl, self.qsl, int(m.chunk_lens.max()), w.scale)
        if timer:
            timer.begin()
        self.attend(0)
        if timer:
            timer.end()

    def run_units(self, step=0):
        self.attend(0)


class MultiTokenStep:
    """Multi-token decode (speculative verification): append each sequence's
    draft tokens, then the causal attention of all of them over the cache
    (``paged_attention_decode_multi``; ``via_prefill`` times the chunked-prefill
    call on the same step instead)."""

    def __init__(self, m, via_prefill=False, library=True):
        self.m, self.w = m, m.decode
        self.via_prefill = via_prefill
        self.units_per_step = 1
        dev = m.chunk_query.device
        self.aslots = torch.from_numpy(m.append_slots).to(dev)
        self.cbt = torch.from_numpy(m.chunk_tables).to(dev)
        self.csl = torch.from_numpy(m.seq_lens).to(dev)
        self.qsl = torch.from_numpy(m.query_start_loc).to(dev)
        self.out = torch.empty_like(m.chunk_query)
        self.max_q = int(m.chunk_lens.max())
        self.max_len = int(m.seq_lens.max())
        w = m.decode
        R, Hkv, B = len(m.seq_lens), w.num_kv_heads, w.block_size
        self.layers = 1
        self.part, self.parts = 0, 1
        if library:
            import paged_kv_cache_409_b200 as pkv
            self.pkv = pkv
            self.part = 0 if via_prefill else pkv.decode_multi_partition_size(R, Hkv, B, self.max_len)
            Tq, Hq, D = m.chunk_query.shape
            need = pkv.decode_workspace_size(Tq, Hq, D, self.max_len, self.part) if self.part else 0
            self.ws = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
            self.parts = -(-self.max_len // self.part) if self.part else 1
        t = m.chunk_query.element_size()
        self.kv_bytes = 2 * int(m.seq_lens.astype(np.int64).sum()) * w.num_kv_heads * w.head_dim * t
        nblocks = int(((m.seq_lens.astype(np.int64) + w.block_size - 1) // w.block_size).sum())
        self.decode_bytes = self.kv_bytes + 2 * m.chunk_query.numel() * t + 4 * nblocks + 8 * len(m.seq_lens)
        self.tokens = int(m.chunk_lens.sum())
        self.kernel = ("paged_attention_prefill_chunk (tcgen05)" if via_prefill else
                       "paged_attention_decode_multi_step (append, then the multi-token decode as its "
                       "programmatic dependent, + merge kernel)")

    def config(self):
        m = self.m
        return {"num_seqs": len(m.chunk_lens), "draft_tokens": self.tokens,
                "draft_len_range": [int(m.chunk_lens.min()), int(m.chunk_lens.max())],
                "context_range": [int(m.chunk_c0.min()), int(m.chunk_c0.max())],
                "partition_size": self.part, "call": "prefill_chunk" if self.via_prefill else "decode_multi"}

    def oracle_sample(self, budget_s, max_seqs=64):
        """Oracle append + causal attention of the first sequences' drafts."""
        sys.path.insert(0, os.path.join(ROOT, "tests"))
        from parity_helpers import oracle_prefill_chunks
        m, w = self.m, self.w
        chunks = np.arange(min(max_seqs, len(m.chunk_lens)))
        pre_k, pre_v = w.key_caches[0].cpu(), w.value_caches[0].cpu()
        done, t0 = 0, time.perf_counter()
        while True:
            oracle_prefill_chunks(m, pre_k, pre_v, chunks)
            done += 1
            el = time.perf_counter() - t0
            if el >= budget_s:
                break
        ntok = int(m.chunk_lens[chunks].sum())
        return ntok * done / el, done, f"{len(chunks)} sequences ({ntok} draft tokens)", el

    def launches_per_step(self):
        return 2 + (1 if self.parts > 1 else 0)

    def e2e_plan(self):
        m = self.m
        pairs = [(t, pinned(t)) for t in (m.chunk_query, m.append_keys, m.append_values, self.aslots, self.cbt,
                                          self.csl, self.qsl)]
        return E2EPlan(self, pairs, [(self.out, pinned(self.out))])

    def run(self, timer=None, step=0):
        m, w = self.m, self.w
        if timer is None and not self.via_prefill:  # append + attention as one library call
            self.pkv.paged_attention_decode_multi_step(
                m.append_keys, m.append_values, self.aslots, self.out, m.chunk_query, w.key_caches[0],
                w.value_caches[0], self.cbt, self.csl, self.qsl, self.max_q, self.max_len, w.scale,
                partition_size=self.part, workspace=self.ws)
            return
        self.pkv.reshape_and_cache(m.append_keys, m.append_values, w.key_caches[0], w.value_caches[0], self.aslots)
        if timer:  # separate calls, so that events can bracket the attention
            timer.begin()
        self.run_units(step)
        if timer:
            timer.end()

    def run_units(self, step=0):
        m, w = self.m, self.w
        if self.via_prefill:
            self.pkv.paged_attention_prefill_chunk(self.out, m.chunk_query, w.key_caches[0], w.value_caches[0],
                                                   self.cbt, self.csl, self.qsl, self.max_q, w.scale)
        else:
            self.pkv.paged_attention_decode_multi(self.out, m.chunk_query, w.key_caches[0], w.value_caches[0],
                                                  self.cbt, self.csl, self.qsl, self.max_q, self.max_len, w.scale,
                                                  partition_size=self.part, workspace=self.ws)


# DRAM traffic of the decode call per algorithmic byte, from one ncu capture
# (dram__bytes_read.sum + dram__bytes_write.sum, --clock-control none) of the
# same kernels on a smaller case of the workload: traffic grows with the blocks
# read, so it scales to the full launch by the algorithmic bytes.  A workload
# is listed only while its kernels are unchanged since the capture.  Figures in
# MB (1e6 bytes): DRAM read, DRAM written, algorithmic bytes of the captured
# launch(es).
TRAFFIC_CAPTURES = {
    "llama7b_decode_f16": {"case": "paged_decode_mma_kernel, the llama7b batch cut to 16 sequences",
                           "read_mb": 287.47136, "write_mb": 3.24992, "algorithmic_mb": 285.38096},
    "mixed_step_bf16": {"case": "paged_decode_mma_kernel, the mixed step's decode cut to 8 sequences",
                        "read_mb": 575.264768, "write_mb": 3.259648, "algorithmic_mb": 574.8748},
    "multi_token_decode_bf16": {"case": "paged_decode_multi_kernel (tcgen05, persistent), the 64-sequence batch",
                                "read_mb": 588.89472, "write_mb": 4.645376, "algorithmic_mb": 586.926064},
    "llama7b_decode_fp8": {"case": "paged_decode_fp8_kernel, the llama7b batch on E4M3 pools cut to 32 sequences",
                           "read_mb": 305.044736, "write_mb": 3.660288, "algorithmic_mb": 303.293652},
    "gqa70b_decode_fp8": {"case": "paged_decode_fp8_kernel (32-token units), one gqa70b layer on E4M3 pools cut to "
                                  "64 sequences",
                          "read_mb": 171.1424, "write_mb": 3.097856, "algorithmic_mb": 171.248148},
    "gqa70b_decode_bf16": {"case": "paged_decode_mma_kernel, one gqa70b layer cut to 64 sequences",
                           "read_mb": 341.175808, "write_mb": 3.977472, "algorithmic_mb": 340.378132},
    "mixed_step_fp8": {"case": "paged_decode_fp8_kernel, the E4M3 mixed step's decode cut to 8 sequences",
                       "read_mb": 287.688448, "write_mb": 3.3216, "algorithmic_mb": 287.511728},
    # the whole workload was captured (its distinct blocks fit the capture size rule): not scaled
    "shared_prefix_decode_f16": {"case": "paged_decode_mma_kernel, the whole shared-prefix workload",
                                 "read_mb": 155.9552, "write_mb": 4.007168, "algorithmic_mb": 3227.190064,
                                 "whole": True},
}


def traffic_ratio(name):
    c = TRAFFIC_CAPTURES[name]
    return (c["read_mb"] + c["write_mb"]) / c["algorithmic_mb"]


def make_step(name, device, rank, seqs=None, layers=None, library=True):
    """The named workload as a timed step.  ``library=False`` (the oracle's arm) builds the same inputs
    without loading the CUDA library; the shared-prefix setup (copy-on-write of the partial prefix block,
    the private tokens' append) is then done with plain torch indexing."""
    from paged_kv_cache_409_b200 import workloads
    if name == "llama7b_decode_f16":
        w = workloads.llama7b_decode_f16(device=device, seed=1002 + rank, num_seqs=seqs or 64)
        return DecodeStep(w, library=library), "llama7b_decode_f16" + (f" ({seqs} sequences)" if seqs else "")
    if name == "llama7b_decode_fp8":
        w = workloads.llama7b_decode_fp8(device=device, seed=1002 + rank, num_seqs=seqs or 64)
        return DecodeStep(w, library=library), "llama7b_decode_fp8" + (f" ({seqs} sequences)" if seqs else "")
    if name in ("gqa70b_decode_fp8", "gqa70b_decode_bf16"):
        fp8 = name.endswith("fp8")
        per_layer = (0.9e9 if fp8 else 1.75e9) * (seqs or 256) / 256  # pools of one layer plus headroom
        free = torch.cuda.mem_get_info()[0] if torch.cuda.is_available() else 16e9
        fit = int(max(1, min(80, (free - 8e9) // per_layer)))
        layers = min(fit, layers) if layers else fit
        if not library:
            layers = 1  # the oracle reads one layer; its pools are the first layer's of the full workload
        make = workloads.gqa70b_decode_fp8 if fp8 else workloads.gqa70b_decode_bf16
        w = make(device=device, num_layers=layers, seed=1003 + rank, num_seqs=seqs or 256)
        note = "" if layers == 80 else f", {layers} distinct layer pools cycled"
        return DecodeStep(w, layers_per_step=80, library=library), f"{name} (80 layers per step{note})"
    if name == "tiny_decode_f32":
        return DecodeStep(workloads.tiny_decode_f32(device=device), library=library), name
    if name == "shared_prefix_decode_f16":
        sp = workloads.shared_prefix_decode_f16(device=device, seed=1004 + rank)
        st = DecodeStep(sp.step, library=library)
        kc, vc = sp.step.key_caches[0], sp.step.value_caches[0]
        pairs = torch.from_numpy(sp.cow_pairs).to(device)
        slots = torch.from_numpy(sp.private_slots).to(device)
        if library:
            st.pkv.copy_blocks([kc], [vc], pairs)
            st.pkv.reshape_and_cache(sp.private_keys, sp.private_values, kc, vc, slots)
        else:
            for c, new in ((kc, sp.private_keys), (vc, sp.private_values)):
                c[pairs[:, 1]] = c[pairs[:, 0]]
                c.view(-1, *c.shape[2:])[slots] = new
        return st, name
    if name in ("mixed_step_bf16", "mixed_step_fp8"):
        make = workloads.mixed_step_bf16 if name == "mixed_step_bf16" else workloads.mixed_step_fp8
        m = make(device=device, seed=1005 + rank, num_decode=seqs or 192)
        return MixedStep(m, library=library), name + (f" ({seqs} decode sequences)" if seqs else "")
    if name in ("multi_token_decode_bf16", "multi_token_decode_bf16_via_prefill"):
        m = workloads.multi_token_decode_bf16(device=device, seed=1006 + rank, num_seqs=seqs or 64)
        return MultiTokenStep(m, via_prefill=name.endswith("via_prefill"), library=library), name + (
            f" ({seqs} sequences)" if seqs else "")
    raise SystemExit(f"unknown config {name}")


# ----------------------------------------------------------------------------- timing helpers

class EventTimer:
    """CUDA events around one unit per step, on the launching stream."""

    def __init__(self):
        self.pairs = []

    def begin(self):
        e = torch.cuda.Event(enable_timing=True)
        e.record()
        self.pairs.append([e, None])

    def end(self):
        e = torch.cuda.Event(enable_timing=True)
        e.record()
        self.pairs[-1][1] = e

    def mean_ms(self):
        return statistics.fmean(a.elapsed_time(b) for a, b in self.pairs)


class ClockSampler:
    """SM clock and throttle reasons sampled through NVML (read-only queries)
    from a background thread every ~2 ms; ``window`` keeps the samples taken
    inside the timed region."""

    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4}

    def __init__(self, device_index):
        import threading
        self.samples, self.t_lo, self.t_hi = [], None, None
        self.stop_evt = threading.Event()
        self.thread = None
        self.nvml = None
        try:
            import pynvml
            pynvml.nvmlInit()
            props = torch.cuda.get_device_properties(device_index)
            want = (int(props.pci_domain_id), int(props.pci_bus_id), int(props.pci_device_id))
            for i in range(pynvml.nvmlDeviceGetCount()):
                h = pynvml.nvmlDeviceGetHandleByIndex(i)
                pci = pynvml.nvmlDeviceGetPciInfo(h)
                if (int(pci.domain), int(pci.bus), int(pci.device)) == want:
                    self.nvml, self.h = pynvml, h
                    self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
                    break
        except Exception:
            self.nvml = None

    def _loop(self):
        n = self.nvml
        while not self.stop_evt.is_set():
            try:
                sm = n.nvmlDeviceGetClockInfo(self.h, n.NVML_CLOCK_SM)
                rs = n.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((time.perf_counter(), sm, rs))
            except Exception:
                pass
            time.sleep(0.002)

    def start(self):
        import threading
        if self.nvml:
            self.thread = threading.Thread(target=self._loop, daemon=True)
            self.thread.start()

    def mark(self, lo, hi):
        self.t_lo, self.t_hi = lo, hi

    def stop(self):
        if not self.thread:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        self.stop_evt.set()
        self.thread.join(timeout=2)
        win = [x for x in self.samples if self.t_lo is not None and self.t_lo <= x[0] <= self.t_hi]
        use = win if win else self.samples
        if not use:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["no samples"]}
        reasons = sorted({k for _, _, r in use for k, bit in self.REASONS.items() if r & bit})
        return {"sm_mhz": statistics.median(x[1] for x in use), "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(use), "in_timed_region": bool(win)}


def dist_setup(n_gpus, backend=None):
    """Rank / world size from the torchrun environment; one process per GPU."""
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        import torch.distributed as dist
        backend = backend or ("nccl" if torch.cuda.is_available() else "gloo")
        if backend == "nccl":
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return ws, rank, local


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, ws, device=None):
    """Max of a per-rank float over all ranks (the slowest rank sets the time)."""
    if ws == 1:
        return x
    import torch.distributed as dist
    dev = device or ("cuda" if dist.get_backend() == "nccl" else "cpu")
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(ws, units_per_rank, max_ms_per_step):
    """Whole-job throughput: units all ranks processed / the slowest rank's time."""
    return ws * units_per_rank / (max_ms_per_step / 1e3)


# ----------------------------------------------------------------------------- CPU baseline (oracle)

def disjoint_block_pairs(num_blocks, block_bytes, target_bytes=512 << 20, seed=7):
    """(src, dst) pairs over distinct blocks, no dst among the srcs: about target_bytes of each pool's
    blocks are copied per launch (capped at half the pool)."""
    n = int(min(num_blocks // 2, max(1, target_bytes // block_bytes)))
    perm = np.random.default_rng(seed).permutation(num_blocks)
    return np.stack([perm[:n], perm[n:2 * n]], 1).astype(np.int64)


def index_kernel_figures(step, hbm_gbs, launches=20):
    """copy_blocks and reshape_and_cache timed alone with CUDA events, after every other measurement
    (copy_blocks overwrites pool blocks).  copy_blocks moves ~0.5 GB of each of the K and V pools per
    launch (inputs larger than L2); the append writes one step's new tokens (L2-sized, launch-bound)."""
    pkv, w = step.pkv, step.w
    kc, vc = w.key_caches[0], w.value_caches[0]
    block_bytes = kc[0].numel() * kc.element_size()
    pairs = torch.from_numpy(disjoint_block_pairs(kc.shape[0], block_bytes)).to(kc.device)
    ev = lambda: torch.cuda.Event(enable_timing=True)

    def timed(fn):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        a, b = ev(), ev()
        a.record()
        for _ in range(launches):
            fn()
        b.record()
        torch.cuda.synchronize()
        return a.elapsed_time(b) / launches

    ms = timed(lambda: pkv.copy_blocks([kc], [vc], pairs))
    moved = 2 * 2 * pairs.shape[0] * block_bytes  # K and V, read and written
    app_ms = timed(lambda: step.append(0))
    nk = w.new_keys[0]
    app_bytes = 2 * nk.numel() * (nk.element_size() + kc.element_size())  # K and V rows read, pool rows written
    return {"copy_blocks": {"pairs": int(pairs.shape[0]), "bytes_per_launch": moved, "ms": ms,
                            "achieved_gbs": moved / ms / 1e6, "frac": moved / ms / 1e6 / hbm_gbs},
            "append": {"kernel": "reshape_and_cache_fp8" if w.fp8 else "reshape_and_cache",
                       "tokens": int(nk.shape[0]), "bytes_per_launch": app_bytes, "us": app_ms * 1e3,
                       "achieved_gbs": app_bytes / app_ms / 1e6,
                       "note": "one step's append: launch-bound, its bytes fit in L2"}}


def host_cores():
    """Host cores this process may run on."""
    try:
        return len(os.sched_getaffinity(0))
    except (AttributeError, OSError):
        return os.cpu_count() or 1


def oracle_threads(n):
    """Set the oracle's host threads; returns the number in force."""
    import oracle
    return oracle.get().num_threads(n)


def oracle_sample(step, budget_s, max_seqs=None):
    """Time the oracle (append + decode) on whole steps or a sequence sample, host cores."""
    import oracle
    w = step.w
    orc = oracle.get()
    S = w.num_seqs
    seqs = np.arange(S if max_seqs is None else min(S, max_seqs))
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from parity_helpers import compact_tables, snapshot_blocks
    used, bt = compact_tables(w.block_tables[seqs], w.context_lens[seqs], w.block_size)
    kn, code = oracle.storage(snapshot_blocks(w.key_caches[0], used))
    vn, _ = oracle.storage(snapshot_blocks(w.value_caches[0], used))
    kn, vn = kn.copy(), vn.copy()
    B = w.block_size
    remap = {int(b): i for i, b in enumerate(used)}
    slots = np.array([remap[int(s) // B] * B + int(s) % B for s in w.slot_mapping[seqs]], dtype=np.int64)
    idx = torch.from_numpy(seqs).to(w.queries[0].device)
    q, qcode = oracle.storage(w.queries[0][idx])
    nk = oracle.storage(w.new_keys[0][idx])[0]
    nv = oracle.storage(w.new_values[0][idx])[0]
    lens = w.context_lens[seqs]
    done, t0 = 0, time.perf_counter()
    while True:
        if w.fp8:
            ks, vs = w.extra["k_scale"], w.extra["v_scale"]
            orc.reshape_and_cache_fp8(nk, nv, kn, vn, slots, qcode, ks, vs)
            orc.paged_attention_decode_kv(q, qcode, kn, vn, oracle.E4M3, ks, vs, bt, lens, w.scale)
        else:
            orc.reshape_and_cache(nk, nv, kn, vn, slots, code)
            orc.paged_attention_decode(q, kn, vn, bt, lens, w.scale, code)
        done += 1
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    return len(seqs) * done / el, done, len(seqs), el


def cpu_baselines(step, args):
    """The oracle timed on all host cores (the reported cpu_baseline) and on one thread, each on about half
    of --cpu-budget seconds of the same workload (whole steps, or a sequence sample of large ones)."""
    w = step.w
    out = []
    for n in (host_cores(), 1):
        cores = oracle_threads(n)
        if hasattr(step, "oracle_sample"):
            v, done, what, el = step.oracle_sample(args.cpu_budget / 2)
            out.append({"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                        "sample": f"{done} x (append + causal attention of {what}), {el:.1f} s, {cores} threads"})
        elif step.layers == 1:
            v, done, k, el = oracle_sample(step, args.cpu_budget / 2, max_seqs=None if w.num_seqs <= 64 else 16)
            out.append({"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                        "sample": f"{done} x (append + decode of {k} sequences), {el:.1f} s, {cores} threads"})
        else:
            v, done, k, el = oracle_sample(step, args.cpu_budget / 2, max_seqs=16)
            out.append({"value": v / step.layers, "unit": f"tokens/s ({step.layers}-layer steps)", "cores": cores,
                        "kind": "oracle", "sample": f"{done} x one layer of {k} sequences, {el:.1f} s, {cores} "
                                                    f"threads; /{step.layers} layers"})
    oracle_threads(host_cores())
    return out[0], out[1]


# ----------------------------------------------------------------------------- main

def run_reference(args, ws, rank):
    """The oracle as it stands, on all host cores, on a bounded sample of the workload.  Only the oracle
    is loaded: the inputs are the same seeded workload, built with torch alone."""
    if rank != 0:
        return
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    step, cname = make_step(args.config, dev, 0, library=False)
    w = step.w
    cores = oracle_threads(host_cores())
    times = []
    if hasattr(step, "oracle_sample"):
        for i in range(args.warmup + args.steps):
            v, done, what, el = step.oracle_sample(0.0)
            if i >= args.warmup:
                times.append(el)
        per = statistics.fmean(times)
        value = v * el / per
        sample_text = f"append + causal attention of {what} per step"
        sample = what
    else:
        sample = w.num_seqs if w.num_seqs <= 64 else 16
        for i in range(args.warmup + args.steps):
            v, done, n, el = oracle_sample(step, 0.0, max_seqs=sample)
            if i >= args.warmup:
                times.append(el)
        per = statistics.fmean(times)
        value = sample / per
        sample_text = (f"append + decode of {'all' if sample == w.num_seqs else 'the first'} {sample} of "
                       f"{w.num_seqs} sequences per step")
        if step.layers > 1:
            value /= step.layers
            sample_text += f" (one layer; tokens/s of {step.layers}-layer steps)"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": per * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": cname, "sample": sample},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": f"{sample_text}, {cores} threads"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_swap(args, ws, rank):
    """Pre-emption swap: every block of the llama7b-shaped batch to page-locked
    host memory and back (swap_blocks), GB/s per direction."""
    import paged_kv_cache_409_b200 as pkv
    from paged_kv_cache_409_b200 import workloads
    w = workloads.llama7b_decode_f16(device="cuda", seed=1002 + rank)
    B = w.block_size
    nblk = ((w.context_lens.astype(np.int64) + B - 1) // B)
    used = np.concatenate([w.block_tables[s, :nblk[s]] for s in range(w.num_seqs)]).astype(np.int64)
    n = len(used)
    kc, vc = w.key_caches[0], w.value_caches[0]
    hk = torch.empty((n,) + tuple(kc.shape[1:]), dtype=kc.dtype).pin_memory()
    hv = torch.empty_like(hk).pin_memory()
    out_pairs = torch.from_numpy(np.stack([used, np.arange(n)], 1)).cuda()
    in_pairs = torch.from_numpy(np.stack([np.arange(n), used], 1)).cuda()
    nbytes = 2 * n * kc[0].numel() * kc.element_size()
    for _ in range(args.warmup):
        pkv.swap_blocks(kc, vc, hk, hv, out_pairs)
        pkv.swap_blocks(hk, hv, kc, vc, in_pairs)
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    t_out = t_in = 0.0
    for _ in range(args.steps):
        ev[0].record()
        pkv.swap_blocks(kc, vc, hk, hv, out_pairs)
        ev[1].record()
        pkv.swap_blocks(hk, hv, kc, vc, in_pairs)
        ev[2].record()
        torch.cuda.synchronize()
        t_out += ev[0].elapsed_time(ev[1])
        t_in += ev[1].elapsed_time(ev[2])
    assert pkv.get_device_error() == 0
    line = {"metric": "swap_blocks GB/s (device pool <-> page-locked host pool)", "value":
            nbytes / (t_out / args.steps / 1e3) / 1e9, "unit": "GB/s", "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": (t_out + t_in) / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f16", "data": "synthetic",
            "config": {"workload": "llama7b_decode_f16: all blocks in use", "blocks": int(n), "bytes": int(nbytes)},
            "swap_out_gbs": nbytes / (t_out / args.steps / 1e3) / 1e9,
            "swap_in_gbs": nbytes / (t_in / args.steps / 1e3) / 1e9, "gpu_launches": 2 * args.steps}
    if rank == 0:
        print(json.dumps(line), flush=True)


def capture(fn):
    """fn's launches captured once in a CUDA graph (after one run on a side stream), replayed once."""
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        fn()
    torch.cuda.current_stream().wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    g.replay()
    torch.cuda.synchronize()
    return g


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default="llama7b_decode_f16")
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle time for cpu_baseline")
    ap.add_argument("--seqs", type=int, default=None,
                    help="fewer sequences of the named workload (small profiling cases)")
    ap.add_argument("--layers", type=int, default=None, help="cap on distinct layer pools (gqa70b_decode_bf16)")
    ap.add_argument("--no-graph", dest="graph", action="store_false",
                    help="launch every kernel of every step instead of replaying one captured CUDA graph")
    ap.add_argument("--min-timed-ms", type=float, default=1000.0,
                    help="repeat the timed region of --steps steps until at least this much has been timed")
    ap.add_argument("--max-regions", type=int, default=1000, help="cap on the number of timed regions")
    ap.add_argument("--flush-l2", action="store_true",
                    help="write a 512 MB buffer before every timed step (outside its events) so that no step "
                         "finds the previous one's K/V in L2; the steps' own durations are summed")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    ws, rank, local = dist_setup(args.gpus)
    if args.impl == "reference":
        run_reference(args, ws, rank)
        if ws > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return

    import paged_kv_cache_409_b200 as pkv
    pkv.load_library()
    if args.config == "swap_llama7b_f16":
        run_swap(args, ws, rank)
        return
    dev = torch.device("cuda", torch.cuda.current_device())
    step, cname = make_step(args.config, dev, rank, args.seqs, args.layers)
    torch.cuda.synchronize()

    # warm-up, then timed regions of exactly K steps between barriers, repeated until enough time is timed
    clocks = ClockSampler(torch.cuda.current_device())
    clocks.start()
    for i in range(args.warmup):
        step.run(step=i)
    torch.cuda.synchronize()
    barrier(ws)
    timer = EventTimer()
    graph = unit_graph = None
    if args.graph:
        graph = capture(lambda: step.run(step=0))
        unit_graph = capture(lambda: step.run_units(step=0))
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev) if args.flush_l2 else None

    def region(fn):
        """K steps of fn between a barrier and a synchronize on both sides; the max over ranks."""
        barrier(ws)
        torch.cuda.synchronize()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        per = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)] if flush is not None else None
        t0.record()
        for i in range(args.steps):
            if flush is not None:
                flush.fill_(i & 0xFF)
                per[i][0].record()
            fn(i)
            if flush is not None:
                per[i][1].record()
        t1.record()
        torch.cuda.synchronize()
        ms = sum(a.elapsed_time(b) for a, b in per) if flush is not None else t0.elapsed_time(t1)
        return max_over_ranks(ms, ws)  # every rank gets the same value, so every rank decides alike

    def repeat(fn, min_ms):
        out = []
        while not out or (sum(out) < min_ms and len(out) < args.max_regions):
            out.append(region(fn))
        return out

    h0 = time.perf_counter()
    torch.cuda.nvtx.range_push("timed")
    regions = repeat((lambda i: graph.replay()) if graph is not None else (lambda i: step.run(timer=timer, step=i)),
                     args.min_timed_ms)
    torch.cuda.nvtx.range_pop()
    clocks.mark(h0, time.perf_counter())
    clk = clocks.stop()
    ms_step = statistics.median(regions) / args.steps
    if unit_graph is not None:
        # the decode calls of the step alone, replayed as captured: the roofline's unit
        unit_regions = repeat(lambda i: unit_graph.replay(), args.min_timed_ms / 4)
        unit_ms = statistics.median(unit_regions) / (args.steps * step.units_per_step)
        unit_how = "CUDA graph of the step's decode calls alone, replayed (median region)"
    else:
        unit_ms = max_over_ranks(timer.mean_ms(), ws)
        unit_how = "CUDA events around each decode call of the timed steps (mean)"
    del graph, unit_graph, flush
    assert pkv.get_device_error() == 0, "device error word set during the run"

    # end to end through the public API: pinned host inputs in, result out, every step
    w = step.w
    e2e = step.e2e_plan()
    e2e_steps = max(3, min(args.steps, 50))
    e2e.start()
    for i in range(3):
        e2e.run(i)
    e2e.finish()
    torch.cuda.synchronize()
    barrier(ws)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    e2e.start()
    for i in range(e2e_steps):
        e2e.run(i)
    e2e.finish()
    e1.record()
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, ws)
    barrier(ws)

    pk, pk_kind = peaks()
    hbm = float(pk["hbm_gbs"])
    tokens_per_step = step.tokens
    value = weak_scaling_value(ws, tokens_per_step, ms_step)
    achieved = step.decode_bytes / (unit_ms / 1e3) / 1e9
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None,
        "dtype": {torch.float16: "f16", torch.bfloat16: "bf16", torch.float32: "f32"}[w.dtype] + (
            " (e4m3 KV pools)" if getattr(w, "fp8", False) else ""),
        "data": "synthetic",
        "config": {"workload": cname, "num_seqs": w.num_seqs, "num_q_heads": w.num_q_heads,
                   "num_kv_heads": w.num_kv_heads, "head_dim": w.head_dim, "block_size": w.block_size,
                   "layers_per_step": step.layers, "partition_size": step.part, "cuda_graph": bool(args.graph),
                   "l2": ("L2 flushed (512 MB written) before every step, outside the step's events; "
                          if args.flush_l2 else "") + (step.l2_note() if hasattr(step, "l2_note") else
                                                       "inputs larger than L2 (K/V pools %.2f GB per layer)" % (
                       2 * w.key_caches[0].numel() * w.key_caches[0].element_size() / 1e9)),
                   "parallelism": f"replicas x{ws}"},
        "kv_gbs": step.kv_bytes * step.layers / (ms_step / 1e3) / 1e9,
        "roofline": {"bound": "hbm", "kernel": getattr(step, "kernel", "paged_attention_decode (decode + merge kernels)"),
                     "achieved": achieved, "peak": hbm, "peak_kind": pk_kind, "unit": "GB/s",
                     "frac": achieved / hbm, "frac_of_8000_nominal": achieved / 8000.0, "traffic": None},
        "e2e": {"value": weak_scaling_value(ws, tokens_per_step, e2e_ms), "unit": "tokens/s",
                "h2d_bytes_per_step": e2e.h2d, "d2h_bytes_per_step": e2e.d2h, "ms_per_step": e2e_ms,
                "copies": "inputs packed into one pinned buffer (one host-to-device copy per step), results "
                          "copied back per tensor; on two side streams, overlapping the neighbouring steps' "
                          "kernels (two device sets)",
                "result_matches_device_run": e2e.matches()},
        "gpu_launches": step.launches_per_step() * args.steps,
        "timed_regions": len(regions), "timed_ms": sum(regions),
        "clocks": clk,
    }
    line["roofline"]["unit_ms"] = unit_ms
    line["roofline"]["unit_timing"] = unit_how
    if hasattr(step, "config"):
        line["config"].update(step.config())
    if args.config in TRAFFIC_CAPTURES and not args.seqs:
        cap = TRAFFIC_CAPTURES[args.config]
        # DRAM bytes per decode call
        line["roofline"]["traffic"] = ((cap["read_mb"] + cap["write_mb"]) * 1e6 if cap.get("whole") else
                                       traffic_ratio(args.config) * step.decode_bytes)
        line["roofline"]["traffic_unit"] = "bytes per launch"
        line["roofline"]["traffic_source"] = "ncu DRAM bytes of " + cap["case"] + (
            "" if cap.get("whole") else ", scaled by algorithmic bytes")
    if getattr(step, "unique_kv_bytes", None) and 2 * step.unique_kv_bytes < step.kv_bytes * step.layers:
        # shared blocks: most logical bytes come from L2, so the HBM fraction above exceeds 1 by design
        uniq = step.unique_kv_bytes / step.layers
        line["roofline"]["distinct_kv_bytes_per_launch"] = uniq
        line["roofline"]["achieved_distinct_gbs"] = uniq / (unit_ms / 1e3) / 1e9
        line["roofline"]["note"] = ("achieved counts logical K/V bytes (each sequence's blocks); %.0f%% of them are "
                                    "shared blocks served from L2, so frac > 1 measures the reuse, not HBM"
                                    % (100 * (1 - uniq / step.kv_bytes)))
    if isinstance(step, MixedStep):
        line["prefill_tokens_per_s"] = ws * step.prefill_tokens / (ms_step / 1e3)
        line["prefill_flops_per_step"] = step.prefill_flops
    if rank == 0 and ws == 1 and args.cpu_budget > 0:
        line["cpu_baseline"], line["cpu_baseline_1_thread"] = cpu_baselines(step, args)
    if ws == 1 and type(step) is DecodeStep:
        try:
            line["index_kernels"] = index_kernel_figures(step, hbm)
        except Exception as exc:  # an extra figure never costs the main line
            line["index_kernels"] = {"error": f"{type(exc).__name__}: {exc}"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
