"""GPU: swap of whole sequences between the device pools and pinned host pools (evicting
sequences to CPU memory when the device pool runs short), against the oracle's byte copies;
a sequence swapped out and back in decodes to bit-identical output."""
import math

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_392_b200 import binding as B
from paged_kv_cache_392_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clean_faults():
    B.device_faults(clear=True)
    yield
    assert B.device_faults(clear=True) == []


@pytest.mark.parametrize("dtype,Hkv,D", [("f16", 8, 128), ("bf16", 4, 64), ("f32", 2, 64)])
def test_swap_kernels_bit_exact(dtype, Hkv, D):
    NB, NH = 64, 40
    rng = np.random.default_rng(7)
    kp = W.randn(torch, (NB, Hkv, 16, D), dtype, 1.0, 20, "cpu")
    vp = W.randn(torch, (NB, Hkv, 16, D), dtype, 1.0, 21, "cpu")
    hk = W.randn(torch, (NH, Hkv, 16, D), dtype, 1.0, 22, "cpu").pin_memory()
    hv = W.randn(torch, (NH, Hkv, 16, D), dtype, 1.0, 23, "cpu").pin_memory()
    out_pairs = np.stack([rng.permutation(NB)[:30], rng.permutation(NH)[:30]], 1).astype(np.int32)
    in_pairs = np.stack([rng.permutation(NH)[:25], rng.permutation(NB)[:25]], 1).astype(np.int32)
    dk, dv = kp.cuda(), vp.cuda()
    ek, ev = W.to_numpy_bits(hk).copy(), W.to_numpy_bits(hv).copy()
    B.kv_swap_out(torch.from_numpy(out_pairs).cuda(), dk, dv, hk, hv)
    torch.cuda.synchronize()
    oracle.kv_swap(out_pairs, W.to_numpy_bits(kp), W.to_numpy_bits(vp), ek, ev)
    assert np.array_equal(W.to_numpy_bits(hk), ek) and np.array_equal(W.to_numpy_bits(hv), ev)
    gk, gv = W.to_numpy_bits(dk).copy(), W.to_numpy_bits(dv).copy()
    B.kv_swap_in(torch.from_numpy(in_pairs).cuda(), hk, hv, dk, dv)
    torch.cuda.synchronize()
    oracle.kv_swap(in_pairs, ek, ev, gk, gv)
    assert np.array_equal(W.to_numpy_bits(dk), gk) and np.array_equal(W.to_numpy_bits(dv), gv)


def test_sequence_swapped_out_and_back_decodes_identically():
    """Eviction round trip through the block manager: 6 sequences (two of them forked
    siblings), swap two out, let new traffic reuse their device blocks, swap them back in
    to fresh blocks; their decode output is bit-identical."""
    Hq, Hkv, D = 8, 2, 128
    NB, NH = 96, 64
    bm = B.BlockManager(NB, free_order=np.random.default_rng(1).permutation(NB))
    bm.set_host_pool(NH)
    lens = {0: 100, 1: 250, 2: 33, 3: 400}
    for s, n in lens.items():
        bm.add_seq(s, n)
    bm.fork(1, 4)                  # 4 shares 1's blocks
    bm.fork(3, 5)
    seqs = [0, 1, 2, 3, 4, 5]
    kp = W.randn(torch, (NB, Hkv, 16, D), "bf16", 0.5, 30, "cpu").cuda()
    vp = W.randn(torch, (NB, Hkv, 16, D), "bf16", 0.5, 31, "cpu").cuda()
    hk = torch.zeros((NH, Hkv, 16, D), dtype=torch.bfloat16).pin_memory()
    hv = torch.zeros_like(hk).pin_memory()
    q = W.randn(torch, (6, Hq, D), "bf16", 1.0, 32, "cpu").cuda()
    scale = 1 / math.sqrt(D)

    def decode(ids):
        bt, ln = bm.block_tables(ids, 32)
        return B.paged_attn_decode(q[:len(ids)].contiguous(), kp, vp,
                                   torch.from_numpy(bt).cuda(), torch.from_numpy(ln).cuda(),
                                   scale, partition_tokens=64)

    before = decode([1, 4])
    p1 = bm.swap_out(1)
    p4 = bm.swap_out(4)
    B.kv_swap_out(torch.from_numpy(np.concatenate([p1, p4])).cuda(), kp, vp, hk, hv)
    # new traffic reuses the freed device blocks and scribbles over them
    bm.add_seq(10, 16 * 12)
    bt10, _ = bm.block_tables([10], 32)
    kp[torch.from_numpy(bt10[0][bt10[0] >= 0]).long().cuda()] = 7.0
    bm.free_seq(10)
    i1 = bm.swap_in(1)
    i4 = bm.swap_in(4)
    B.kv_swap_in(torch.from_numpy(np.concatenate([i1, i4])).cuda(), hk, hv, kp, vp)
    after = decode([1, 4])
    assert torch.equal(before, after)
    assert bm.num_host_free() == NH


def test_swap_rejects_bad_ids_and_unpinned_host_memory():
    kp = torch.zeros((8, 2, 16, 64), dtype=torch.float16, device="cuda")
    vp = torch.zeros_like(kp)
    hk = torch.zeros((4, 2, 16, 64), dtype=torch.float16).pin_memory()
    hv = torch.zeros_like(hk).pin_memory()
    B.kv_swap_out(torch.tensor([[0, 4]], dtype=torch.int32, device="cuda"), kp, vp, hk, hv)
    assert B.device_faults() == ["bad copy pair"]
    with pytest.raises(ValueError):
        B.kv_swap_out(torch.tensor([[0, 1]], dtype=torch.int32, device="cuda"), kp, vp,
                      torch.zeros_like(hk), hv)          # not pinned: refused before any launch
