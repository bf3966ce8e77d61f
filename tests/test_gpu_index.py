"""reshape_and_cache and copy_blocks on the GPU: bit-exact against the oracle over whole pools."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_409_b200 as pkv
from parity_helpers import bits

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype", [torch.float32, torch.float16, torch.bfloat16])
@pytest.mark.parametrize("Hkv,D,B", [(4, 64, 16), (8, 128, 32), (1, 64, 8), (3, 128, 16)])
def test_reshape_and_cache_bit_exact(dtype, Hkv, D, B):
    g = torch.Generator().manual_seed(Hkv * 1000 + D + B)
    NB, T = 37, 150
    kc = torch.randn(NB, B, Hkv, D, generator=g).to(dtype)
    vc = torch.randn(NB, B, Hkv, D, generator=g).to(dtype)
    kc[0, 0, 0, 0] = float("nan")  # NaN bits must travel untouched
    k = torch.randn(T, Hkv, D, generator=g).to(dtype)
    v = torch.randn(T, Hkv, D, generator=g).to(dtype)
    slots = torch.randperm(NB * B, generator=g)[:T].to(torch.int64)
    slots[::7] = -1  # padding tokens
    kn, code = oracle.storage(kc)
    vn, _ = oracle.storage(vc)
    kn, vn = kn.copy(), vn.copy()
    oracle.get().reshape_and_cache(oracle.storage(k)[0], oracle.storage(v)[0], kn, vn, slots.numpy(), code)
    kd, vd = kc.cuda(), vc.cuda()
    pkv.reshape_and_cache(k.cuda(), v.cuda(), kd, vd, slots.cuda())
    assert np.array_equal(bits(kd), kn.view(bits(kd).dtype))
    assert np.array_equal(bits(vd), vn.view(bits(vd).dtype))
    assert pkv.get_device_error() == 0


def test_reshape_and_cache_empty():
    kc = torch.zeros(2, 16, 1, 64, dtype=torch.float16, device="cuda")
    e = torch.zeros(0, 1, 64, dtype=torch.float16, device="cuda")
    pkv.reshape_and_cache(e, e, kc, kc, torch.zeros(0, dtype=torch.int64, device="cuda"))
    assert torch.count_nonzero(kc) == 0


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16, torch.float32])
def test_copy_blocks_bit_exact_many_layers(dtype):
    g = torch.Generator().manual_seed(3)
    L, NB, B, Hkv, D = 40, 24, 16, 2, 64  # more layers than one launch takes
    kcs = [torch.randn(NB, B, Hkv, D, generator=g).to(dtype) for _ in range(L)]
    vcs = [torch.randn(NB, B, Hkv, D, generator=g).to(dtype) for _ in range(L)]
    pairs = torch.tensor([[0, 10], [0, 11], [3, 12], [5, 20], [7, 23]], dtype=torch.int64)
    kn = [oracle.storage(c)[0].copy() for c in kcs]
    vn = [oracle.storage(c)[0].copy() for c in vcs]
    oracle.get().copy_blocks(kn, vn, pairs.numpy())
    kd = [c.cuda() for c in kcs]
    vd = [c.cuda() for c in vcs]
    pkv.copy_blocks(kd, vd, pairs.cuda())
    for a, b in zip(kd + vd, kn + vn):
        assert np.array_equal(bits(a), b.view(bits(a).dtype))


def test_copy_blocks_large_block():
    """A 128 KB block (16 x 32 heads x 128 x fp16): several CTAs per block."""
    g = torch.Generator(device="cuda").manual_seed(4)
    kc = torch.randn(300, 16, 32, 128, generator=g, device="cuda").half()
    vc = torch.randn(300, 16, 32, 128, generator=g, device="cuda").half()
    src = torch.arange(0, 100, dtype=torch.int64)
    dst = torch.arange(150, 250, dtype=torch.int64)
    pairs = torch.stack([src, dst], 1).cuda()
    ek, ev = kc.clone(), vc.clone()
    ek[dst.cuda()] = kc[src.cuda()]
    ev[dst.cuda()] = vc[src.cuda()]
    pkv.copy_blocks([kc], [vc], pairs)
    assert torch.equal(bits_t(kc), bits_t(ek)) and torch.equal(bits_t(vc), bits_t(ev))


def bits_t(t):
    return t.view(torch.int16)
