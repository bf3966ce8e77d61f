"""swap_blocks between the device pool and a page-locked host pool: bit-exact round trip."""
import ctypes

import numpy as np
import pytest
import torch

import paged_kv_cache_409_b200 as pkv

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16, torch.float32])
def test_swap_out_and_back_bit_exact(dtype):
    g = torch.Generator(device="cuda").manual_seed(2)
    NB, NH, B, Hkv, D = 64, 32, 16, 4, 128
    kc = torch.randn(NB, B, Hkv, D, generator=g, device="cuda").to(dtype)
    vc = torch.randn(NB, B, Hkv, D, generator=g, device="cuda").to(dtype)
    hk = torch.zeros(NH, B, Hkv, D, dtype=dtype).pin_memory()
    hv = torch.zeros(NH, B, Hkv, D, dtype=dtype).pin_memory()
    k0, v0 = kc.cpu(), vc.cpu()
    out_pairs = torch.tensor([[3, 0], [10, 5], [11, 6], [40, 7], [63, 31]], dtype=torch.int64)
    pkv.swap_blocks(kc, vc, hk, hv, out_pairs.cuda())             # pairs in device memory
    torch.cuda.synchronize()
    iv = lambda t: t.view(torch.int16) if t.element_size() == 2 else t.view(torch.int32)
    assert torch.equal(iv(hk[out_pairs[:, 1]]), iv(k0[out_pairs[:, 0]]))
    assert torch.equal(iv(hv[out_pairs[:, 1]]), iv(v0[out_pairs[:, 0]]))
    untouched = torch.ones(NH, dtype=torch.bool)
    untouched[out_pairs[:, 1]] = False
    assert torch.count_nonzero(hk[untouched]) == 0
    kc[out_pairs[:, 0].cuda()] = 0                                  # the device copies are gone
    in_pairs = torch.stack([out_pairs[:, 1], torch.tensor([20, 21, 22, 23, 24])], 1).pin_memory()
    pkv.swap_blocks(hk, hv, kc, vc, in_pairs)                       # pairs in pinned host memory
    torch.cuda.synchronize()
    assert torch.equal(iv(kc[in_pairs[:, 1].cuda()].cpu()), iv(k0[out_pairs[:, 0]]))
    assert torch.equal(iv(vc[in_pairs[:, 1].cuda()].cpu()), iv(v0[out_pairs[:, 0]]))
    assert pkv.get_device_error() == 0


def test_swap_rejects_pageable_host_memory_and_bad_ids():
    lib = pkv.load_library()
    kc = torch.zeros(4, 16, 1, 64, dtype=torch.float16, device="cuda")
    pageable = np.zeros((4, 16, 1, 64), dtype=np.float16)
    pairs = torch.tensor([[0, 1]], dtype=torch.int64, device="cuda")
    rc = lib.pkv_swap_blocks(kc.data_ptr(), kc.data_ptr(), pageable.ctypes.data, pageable.ctypes.data,
                             pairs.data_ptr(), 1, 16 * 64 * 2, 4, 4, torch.cuda.current_stream().cuda_stream)
    assert rc == -1
    bad = torch.tensor([[0, 9]], dtype=torch.int64, device="cuda")
    hk = torch.zeros(4, 16, 1, 64, dtype=torch.float16).pin_memory()
    pkv.swap_blocks(kc, kc, hk, hk, bad)
    assert pkv.get_device_error() & pkv._binding.DEVERR_PAIR
