"""FP8 (E4M3) pools on the GPU against the CPU oracle: the quantising append is
bit-exact over whole pools, decode over E4M3 pools is within the 16-bit
tolerance of the oracle's double-precision attention over the same codes."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_409_b200 as pkv
from paged_kv_cache_409_b200 import workloads
from parity_helpers import assert_close, gpu_decode_step, gpu_tables, oracle_decode_step, oracle_prefill_chunks, \
    to_device

pytestmark = pytest.mark.gpu

DT = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


def special_values(dtype, scale):
    """Values that probe the rounding: exact code midpoints times a power-of-two
    scale, saturation, zeros of both signs, subnormal codes, non-finite input."""
    codes = np.arange(0x7F, dtype=np.uint8)
    vals = oracle.get().to_double(codes, oracle.E4M3)
    mids = (vals[:-1] + vals[1:]) / 2
    xs = np.concatenate([mids, -mids, vals, [448.0, 449.0, 464.0, 465.0, 1e4, -1e4, 0.0, -0.0, 2.0 ** -10,
                                             -2.0 ** -10, 2.0 ** -10 * 1.01, 2.0 ** -12]])
    x = torch.from_numpy(xs * scale).to(dtype)
    if dtype == torch.float32:
        x = torch.cat([x, torch.tensor([float("nan"), float("inf"), -float("inf")])])
    return x


@pytest.mark.parametrize("src", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("Hkv,D,B", [(4, 64, 16), (8, 128, 32), (2, 128, 8), (1, 16, 16)])
def test_fp8_append_bit_exact(src, Hkv, D, B):
    dtype = DT[src]
    g = torch.Generator().manual_seed(Hkv * 100 + D + B)
    NB, T = 29, 120
    row = Hkv * D
    kc = torch.randint(0, 256, (NB, B, Hkv, D), generator=g, dtype=torch.uint8)
    vc = torch.randint(0, 256, (NB, B, Hkv, D), generator=g, dtype=torch.uint8)
    k = (torch.randn(T, Hkv, D, generator=g) * 3).to(dtype)
    v = (torch.randn(T, Hkv, D, generator=g) * torch.exp2(torch.randint(-12, 12, (T, Hkv, D), generator=g)
                                                           .float())).to(dtype)
    sp = special_values(dtype, 0.25)
    n = min(sp.numel(), T * row // 2)
    v.view(-1)[:n] = sp[:n]
    k.view(-1)[-n:] = special_values(dtype, 0.0371)[:n]
    slots = torch.randperm(NB * B, generator=g)[:T].to(torch.int64)
    slots[::5] = -1
    for k_scale, v_scale in ((0.0371, 0.25), (1.0, 3.3e-3)):
        # the library takes fp32 scales: give the oracle the same values
        k_scale, v_scale = float(np.float32(k_scale)), float(np.float32(v_scale))
        kn, vn = kc.numpy().copy(), vc.numpy().copy()
        oracle.get().reshape_and_cache_fp8(oracle.storage(k)[0], oracle.storage(v)[0], kn, vn, slots.numpy(),
                                          oracle.storage(k)[1], k_scale, v_scale)
        kd, vd = kc.cuda(), vc.cuda()
        pkv.reshape_and_cache_fp8(k.cuda(), v.cuda(), kd, vd, slots.cuda(), k_scale, v_scale)
        torch.cuda.synchronize()
        assert pkv.get_device_error() == 0
        kg, vg = kd.cpu().numpy(), vd.cpu().numpy()
        bad = np.argwhere(kg != kn)
        assert bad.size == 0, f"K codes differ at {bad[:5].tolist()}: gpu {kg[tuple(bad[0])]:#x} oracle " \
                              f"{kn[tuple(bad[0])]:#x}"
        bad = np.argwhere(vg != vn)
        assert bad.size == 0, f"V codes differ at {bad[:5].tolist()}: gpu {vg[tuple(bad[0])]:#x} oracle " \
                              f"{vn[tuple(bad[0])]:#x}"


def ragged_lens(B):
    # single token, block edges, a ragged tail, several partitions
    return [1, B - 1, B, B + 1, 3 * B + 5, 37, 300]


CASES = [(q, B, G) for q in ("f16", "bf16") for B in (8, 16, 32) for G in (1, 2, 4, 8)]


@pytest.mark.parametrize("q,B,G", CASES)
def test_fp8_decode_matches_oracle(q, B, G):
    w = workloads.decode_workload("fp8", ragged_lens(B), 2 * G, 2, 128, B, DT[q], seed=B * 13 + G,
                                  poison=True, fp8_scales=(0.0123, 0.0171))
    pre_k, pre_v = w.key_caches[0].clone(), w.value_caches[0].clone()
    ref, k_after, v_after, used = oracle_decode_step(w, pre_k=pre_k, pre_v=pre_v)
    to_device(w)
    # partitions of 1 and 3 blocks end inside a 32-token unit of grouped blocks
    for part in (0, B, 3 * B, 4 * B):
        w.key_caches[0], w.value_caches[0] = pre_k.cuda(), pre_v.cuda()
        out = gpu_decode_step(w, partition_size=part)
        torch.cuda.synchronize()
        assert pkv.get_device_error() == 0
        assert_close(out, ref, DT[q], f"fp8 q {q} B{B} G{G} partition {part}")
    got_k = w.key_caches[0][torch.from_numpy(used).cuda()].cpu().numpy()
    got_v = w.value_caches[0][torch.from_numpy(used).cuda()].cpu().numpy()
    assert np.array_equal(got_k, k_after) and np.array_equal(got_v, v_after)


def test_fp8_one_token_context_returns_scaled_v():
    """c = 1: the output is v_scale times the appended V row, read back from the GPU pool."""
    w = workloads.decode_workload("fp8one", [1, 1, 1], 8, 2, 128, 16, torch.float16, seed=5,
                                  fp8_scales=(0.05, 0.0625))
    ref, _, _, _ = oracle_decode_step(w, pre_k=w.key_caches[0].clone(), pre_v=w.value_caches[0].clone())
    to_device(w)
    out = gpu_decode_step(w, partition_size=0)
    assert_close(out, ref, torch.float16, "fp8 c=1")
    rows = w.value_caches[0].view(-1, 2, 128)[torch.from_numpy(w.slot_mapping).cuda()]   # [3, Hkv, D] codes
    v = rows.view(torch.float8_e4m3fn).double() * 0.0625
    direct = v[:, [h // 4 for h in range(8)]]
    assert torch.allclose(out.double(), direct, rtol=1e-3, atol=0)


def test_fp8_rejects_unsupported():
    q = torch.zeros(2, 4, 64, device="cuda", dtype=torch.float16)
    kc = torch.zeros(4, 16, 2, 64, device="cuda", dtype=torch.uint8)
    bt = torch.zeros(2, 1, dtype=torch.int32, device="cuda")
    cl = torch.ones(2, dtype=torch.int32, device="cuda")
    with pytest.raises(pkv.PagedKVError) as e:  # head_dim 64 is not built for FP8
        pkv.paged_attention_decode_fp8(torch.empty_like(q), q, kc, kc, bt, cl, 0.1, 1.0, 1.0, 1)
    assert e.value.status == -2
    q32 = torch.zeros(2, 4, 128, device="cuda")
    kc = torch.zeros(4, 16, 2, 128, device="cuda", dtype=torch.uint8)
    with pytest.raises(pkv.PagedKVError) as e:  # fp32 query
        pkv.paged_attention_decode_fp8(torch.empty_like(q32), q32, kc, kc, bt, cl, 0.1, 1.0, 1.0, 1)
    assert e.value.status == -2
    q16 = q32.half()
    with pytest.raises(pkv.PagedKVError) as e:  # scale <= 0
        pkv.paged_attention_decode_fp8(torch.empty_like(q16), q16, kc, kc, bt, cl, 0.1, 0.0, 1.0, 1)
    assert e.value.status == -1


def test_llama7b_decode_fp8_full_sampled():
    """The 64-sequence llama7b batch on FP8 pools in the launch configuration the benchmark times;
    eight sampled sequences against the oracle."""
    w = workloads.llama7b_decode_fp8(device="cuda", poison=True)
    pre_k, pre_v = w.key_caches[0].clone(), w.value_caches[0].clone()
    part = pkv.decode_partition_size(w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim, w.block_size,
                                     w.max_context_len, 3,
                                     int(w.context_lens.sum()))
    out = gpu_decode_step(w, partition_size=part)
    torch.cuda.synchronize()
    assert pkv.get_device_error() == 0
    seqs = np.array([0, 7, 19, 31, 40, 52, 60, 63])
    ref, _, _, _ = oracle_decode_step(w, seqs=seqs, pre_k=pre_k.cpu(), pre_v=pre_v.cpu())
    assert_close(out[torch.from_numpy(seqs).cuda()], ref, torch.float16, "llama7b fp8")


def test_gqa70b_decode_fp8_one_layer_sampled():
    """256 sequences, 64 q heads over 8 KV heads, lognormal contexts, bf16 query, FP8 pools (one layer)."""
    w = workloads.gqa70b_decode_fp8(device="cuda", num_layers=1, poison=True)
    pre_k, pre_v = w.key_caches[0].clone(), w.value_caches[0].clone()
    part = pkv.decode_partition_size(w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim, w.block_size,
                                     w.max_context_len, 3,
                                     int(w.context_lens.sum()))
    out = gpu_decode_step(w, partition_size=part)
    torch.cuda.synchronize()
    assert pkv.get_device_error() == 0
    order = np.argsort(w.context_lens)
    seqs = np.concatenate([order[:3], order[-3:], [100, 200]])
    ref, _, _, _ = oracle_decode_step(w, seqs=seqs, pre_k=pre_k.cpu(), pre_v=pre_v.cpu())
    assert_close(out[torch.from_numpy(seqs).cuda()], ref, torch.bfloat16, "gqa70b fp8")


PREFILL_CASES = [
    # dtype, D, B, Hq, Hkv, c0s, ns
    (torch.bfloat16, 128, 32, 32, 8, [0, 300], [512, 77]),
    (torch.float16, 128, 16, 8, 8, [5, 0, 129], [1, 130, 128]),
    (torch.bfloat16, 64, 8, 16, 2, [1000, 0], [33, 257]),
    (torch.float16, 64, 16, 4, 2, [17], [300]),
    (torch.bfloat16, 128, 16, 16, 2, [255, 64], [200, 16]),
]


@pytest.mark.parametrize("case", PREFILL_CASES, ids=[f"case{i}" for i in range(len(PREFILL_CASES))])
def test_fp8_prefill_matches_oracle(case):
    """Quantising append of every chunk token, then chunked prefill over the E4M3 pools."""
    dtype, D, B, Hq, Hkv, c0s, ns = case
    m = workloads.mixed_workload("p8", [], c0s, ns, Hq, Hkv, D, B, dtype, seed=sum(c0s) + sum(ns) + D + B,
                                 poison=True, fp8_scales=(0.0119, 0.0143))
    w = m.decode
    pre_k, pre_v = w.key_caches[0].clone(), w.value_caches[0].clone()
    ref = oracle_prefill_chunks(m, pre_k, pre_v)
    dev = "cuda"
    kc, vc = pre_k.to(dev), pre_v.to(dev)
    ks, vs = w.extra["k_scale"], w.extra["v_scale"]
    pkv.reshape_and_cache_fp8(m.append_keys.to(dev), m.append_values.to(dev), kc, vc,
                              torch.from_numpy(m.append_slots).to(dev), ks, vs)
    out = torch.empty_like(m.chunk_query, device=dev)
    pkv.paged_attention_prefill_chunk_fp8(out, m.chunk_query.to(dev), kc, vc, torch.from_numpy(m.chunk_tables).to(dev),
                                          torch.from_numpy(m.seq_lens).to(dev),
                                          torch.from_numpy(m.query_start_loc).to(dev), int(m.chunk_lens.max()),
                                          w.scale, ks, vs)
    torch.cuda.synchronize()
    assert pkv.get_device_error() == 0
    assert_close(out, ref, dtype, f"fp8 prefill {case}")


def test_fp8_prefill_rejects_small_workspace():
    q = torch.zeros(4, 2, 64, device="cuda", dtype=torch.float16)
    kc = torch.zeros(2, 16, 2, 64, device="cuda", dtype=torch.uint8)
    i32 = torch.zeros(2, dtype=torch.int32, device="cuda")
    ws = torch.empty(1024, dtype=torch.uint8, device="cuda")
    lib = pkv.load_library()
    rc = lib.pkv_paged_attention_prefill_chunk_fp8(
        q.data_ptr(), q.data_ptr(), kc.data_ptr(), kc.data_ptr(), i32.data_ptr(), (i32[:1] + 4).data_ptr(),
        torch.tensor([0, 4], dtype=torch.int32, device="cuda").data_ptr(), 1, 4, 4, 0.1, 1.0, 1.0, 2, 2, 64, 16, 2,
        2, 1, ws.data_ptr(), 16, torch.cuda.current_stream().cuda_stream)
    assert rc == -5


def test_mixed_step_fp8_sampled():
    """The mixed step on E4M3 pools in the benchmark's launch configuration (quantising append of
    every token, FP8 chunked prefill, FP8 decode with the recommended split): sampled decode
    sequences and prefill rows against the oracle."""
    m = workloads.mixed_step_fp8(device="cuda")
    w = m.decode
    kc, vc = w.key_caches[0], w.value_caches[0]
    pre_k, pre_v = kc.clone(), vc.clone()
    ks, vs = w.extra["k_scale"], w.extra["v_scale"]
    pkv.reshape_and_cache_fp8(m.append_keys, m.append_values, kc, vc, torch.from_numpy(m.append_slots).cuda(), ks, vs)
    pout = torch.empty_like(m.chunk_query)
    pkv.paged_attention_prefill_chunk_fp8(pout, m.chunk_query, kc, vc, torch.from_numpy(m.chunk_tables).cuda(),
                                          torch.from_numpy(m.seq_lens).cuda(),
                                          torch.from_numpy(m.query_start_loc).cuda(), int(m.chunk_lens.max()),
                                          w.scale, ks, vs)
    bt, cl, _ = gpu_tables(w)
    part = pkv.decode_partition_size(w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim, w.block_size,
                                     w.max_context_len, 3,
                                     int(w.context_lens.sum()))
    dout = torch.empty_like(w.queries[0])
    pkv.paged_attention_decode_fp8(dout, w.queries[0], kc, vc, bt, cl, w.scale, ks, vs, w.max_context_len,
                                   partition_size=part)
    torch.cuda.synchronize()
    assert pkv.get_device_error() == 0
    order = np.argsort(w.context_lens)
    dsample = np.unique(np.concatenate([order[:2], order[-3:], np.arange(7, w.num_seqs, 47)]))
    ref, _, _, _ = oracle_decode_step(w, seqs=dsample, pre_k=pre_k, pre_v=pre_v)
    assert_close(dout[torch.from_numpy(dsample).cuda()], ref, torch.bfloat16, "fp8 mixed decode sample")
    sel = np.zeros(int(m.query_start_loc[-1]), dtype=np.uint8)
    for r in range(len(m.chunk_lens)):
        q0, n = int(m.query_start_loc[r]), int(m.chunk_lens[r])
        for i in (0, 1, 31, 32, 127, 128, 255, 256, n - 1):
            if 0 <= i < n:
                sel[q0 + i] = 1
    ref = oracle_prefill_chunks(m, pre_k, pre_v, row_select=sel)
    rows = np.nonzero(sel)[0]
    assert_close(pout[torch.from_numpy(rows).cuda()], ref[rows], torch.bfloat16, "fp8 mixed prefill sample")
