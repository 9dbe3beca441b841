"""GPU parity with 32-token physical blocks (the pages allow blocks of 16 or 32 tokens).  The
kernels work in 16-token sub-blocks, so a 32-token block is two of them, read through one
table entry.  Everything is checked against the fp64 oracle on the same pools, and the writes
and copies bit for bit; partitions of 48 tokens split 32-token blocks in the middle."""
import math

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_392_b200 import binding as B
from paged_kv_cache_392_b200 import workloads as W

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-5, "f16": 2e-3, "bf16": 1e-2}
RAGGED = [1, 2, 15, 16, 17, 31, 32, 33, 63, 64, 65, 100, 511, 512, 513, 1500]


@pytest.fixture(autouse=True)
def _clean_faults():
    B.device_faults(clear=True)
    yield
    assert B.device_faults(clear=True) == []


def bits(t):
    return W.to_numpy_bits(t)


def u8(t):
    return t.detach().cpu().contiguous().numpy()


def wl32(lens, Hq, Hkv, D, dtype, seed, pt=0):
    wl = W.make_workload("b32", lens, Hq, Hkv, D, dtype, seed, pool_factor=1.3,
                         partition_tokens=pt, block_size=32)
    if dtype == "f32":
        wl.kv_std = 1.0
    return wl


@pytest.mark.parametrize("dtype,D", [("f32", 64), ("f16", 128), ("bf16", 128), ("bf16", 64)])
@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (8, 2), (8, 1)])
@pytest.mark.parametrize("pt", [0, 48])
def test_fused_step_with_32_token_blocks(dtype, D, Hq, Hkv, pt):
    if dtype == "f32" and Hq // Hkv == 8 and D == 128:
        pytest.skip("not built")
    wl = wl32(RAGGED, Hq, Hkv, D, dtype, 3 * Hq + Hkv + D + pt, pt)
    vals = W.make_values(wl, "cpu")
    d = {k: v.cuda() for k, v in vals.items()}
    kp2, vp2 = d["k_pool"].clone(), d["v_pool"].clone()
    bt = torch.from_numpy(wl.block_tables).cuda()
    lens = torch.from_numpy(wl.context_lens).cuda()
    sl = torch.from_numpy(wl.slot_mapping).cuda()
    out = B.kv_write_and_decode(d["q"], d["k_new"], d["v_new"], sl, d["k_pool"], d["v_pool"],
                                bt, lens, wl.scale, partition_tokens=pt)
    B.kv_write(d["k_new"], d["v_new"], sl, kp2, vp2)
    out2 = B.paged_attn_decode(d["q"], kp2, vp2, bt, lens, wl.scale, partition_tokens=pt)
    torch.cuda.synchronize()
    assert torch.equal(d["k_pool"], kp2) and torch.equal(d["v_pool"], vp2)
    assert np.array_equal(bits(out), bits(out2))
    kp, vp = bits(vals["k_pool"]).copy(), bits(vals["v_pool"]).copy()
    oracle.kv_write(bits(vals["k_new"]), bits(vals["v_new"]), wl.slot_mapping, kp, vp)
    assert np.array_equal(bits(d["k_pool"]), kp) and np.array_equal(bits(d["v_pool"]), vp)
    ref = oracle.paged_attn_decode(bits(vals["q"]), kp, vp, wl.block_tables, wl.context_lens,
                                   wl.scale, dtype)
    err = float(np.max(np.abs(out.double().cpu().numpy() - ref)))
    assert err <= TOL[dtype], err


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (8, 2), (16, 2)])
@pytest.mark.parametrize("pt", [0, 48])
def test_fp8_step_with_32_token_blocks(dtype, Hq, Hkv, pt):
    wl = wl32(RAGGED, Hq, Hkv, 128, dtype, 5 * Hq + Hkv + pt, pt)
    vals = {k: v.cuda() for k, v in W.make_values_fp8(wl, "cpu").items()}
    assert vals["v_pool"].shape == (wl.num_blocks, Hkv, 2, 128, 16)
    kp0, vp0 = u8(vals["k_pool"]).copy(), u8(vals["v_pool"]).copy()
    kp2, vp2 = vals["k_pool"].clone(), vals["v_pool"].clone()
    bt = torch.from_numpy(wl.block_tables).cuda()
    lens = torch.from_numpy(wl.context_lens).cuda()
    sl = torch.from_numpy(wl.slot_mapping).cuda()
    out = B.kv_write_fp8_and_decode(vals["q"], vals["k_new"], vals["v_new"], sl,
                                    vals["k_scale"], vals["v_scale"], vals["k_pool"],
                                    vals["v_pool"], bt, lens, wl.scale, partition_tokens=pt)
    B.kv_write_fp8(vals["k_new"], vals["v_new"], sl, vals["k_scale"], vals["v_scale"], kp2, vp2)
    out2 = B.paged_attn_decode_fp8(vals["q"], kp2, vp2, vals["k_scale"], vals["v_scale"], bt,
                                   lens, wl.scale, partition_tokens=pt)
    torch.cuda.synchronize()
    assert torch.equal(vals["k_pool"], kp2) and torch.equal(vals["v_pool"], vp2)
    assert np.array_equal(bits(out), bits(out2))
    ks, vs = u8(vals["k_scale"]), u8(vals["v_scale"])
    oracle.kv_write_fp8(bits(vals["k_new"]), bits(vals["v_new"]), wl.slot_mapping, ks, vs, kp0,
                        vp0, dtype)
    assert np.array_equal(u8(vals["k_pool"]), kp0) and np.array_equal(u8(vals["v_pool"]), vp0)
    ref = oracle.paged_attn_decode_fp8(bits(vals["q"]), kp0, vp0, ks, vs, wl.block_tables,
                                       wl.context_lens, wl.scale, dtype)
    err = float(np.max(np.abs(out.double().cpu().numpy() - ref)))
    assert err <= TOL[dtype], err


@pytest.mark.parametrize("dtype", ["f16", "f32"])
def test_kv_write_and_copy_blocks_with_32_token_blocks(dtype):
    NB, Hkv, D, T = 40, 4, 64, 50
    kp = W.randn(torch, (NB, Hkv, 32, D), dtype, 1.0, 1, "cpu")
    vp = W.randn(torch, (NB, Hkv, 32, D), dtype, 1.0, 2, "cpu")
    kn = W.randn(torch, (T, Hkv, D), dtype, 1.0, 3, "cpu")
    vn = W.randn(torch, (T, Hkv, D), dtype, 1.0, 4, "cpu")
    slots = np.random.default_rng(5).choice(NB * 32, size=T, replace=False).astype(np.int64)
    slots[7] = -1
    dk, dv = kp.cuda(), vp.cuda()
    B.kv_write(kn.cuda(), vn.cuda(), torch.from_numpy(slots).cuda(), dk, dv)
    ek, ev = bits(kp).copy(), bits(vp).copy()
    oracle.kv_write(bits(kn), bits(vn), slots, ek, ev)
    assert np.array_equal(bits(dk), ek) and np.array_equal(bits(dv), ev)
    pairs = np.array([[1, 30], [5, 31], [9, 32]], np.int32)
    B.kv_copy_blocks(torch.from_numpy(pairs).cuda(), dk, dv)
    oracle.kv_copy_blocks(pairs, ek, ev)
    assert np.array_equal(bits(dk), ek) and np.array_equal(bits(dv), ev)
    bad = torch.tensor([NB * 32, 3], dtype=torch.int64, device="cuda")    # one past the pool
    B.kv_write(kn[:2].cuda(), vn[:2].cuda(), bad, dk, dv)
    assert B.device_faults() == ["bad slot"]


def test_fork_step_with_32_token_blocks_through_the_block_manager():
    """2 prompts x 4 samples sharing a 70-token prefix in 32-token blocks: the first appended
    token copies the shared partial block for 3 samples of each prompt (6 pairs), then the
    fused step; against the oracle and against private copies of every block."""
    NB, Hkv, D = 60, 4, 128
    bm = B.BlockManager(NB, block_size=32, free_order=np.random.default_rng(0).permutation(NB))
    seqs = []
    for p in range(2):
        bm.add_seq(p * 4, 70)
        for k in range(1, 4):
            bm.fork(p * 4, p * 4 + k)
        seqs += [p * 4 + k for k in range(4)]
    slots, pairs = bm.append_slots(seqs)
    assert len(pairs) == 6
    kp = W.randn(torch, (NB, Hkv, 32, D), "bf16", 0.5, 1, "cpu").cuda()
    vp = W.randn(torch, (NB, Hkv, 32, D), "bf16", 0.5, 2, "cpu").cuda()
    kp0, vp0 = bits(kp).copy(), bits(vp).copy()
    B.kv_copy_blocks(torch.from_numpy(pairs).cuda(), kp, vp)
    bt, lens = bm.block_tables(seqs, 4)
    kn = W.randn(torch, (8, Hkv, D), "bf16", 0.5, 3, "cpu").cuda()
    vn = W.randn(torch, (8, Hkv, D), "bf16", 0.5, 4, "cpu").cuda()
    q = W.randn(torch, (8, 8, D), "bf16", 1.0, 5, "cpu").cuda()
    out = B.kv_write_and_decode(q, kn, vn, torch.from_numpy(slots).cuda(), kp, vp,
                                torch.from_numpy(bt).cuda(), torch.from_numpy(lens).cuda(),
                                1 / math.sqrt(D))
    torch.cuda.synchronize()
    oracle.kv_copy_blocks(pairs, kp0, vp0)
    oracle.kv_write(bits(kn), bits(vn), slots, kp0, vp0)
    assert np.array_equal(bits(kp), kp0) and np.array_equal(bits(vp), vp0)
    ref = oracle.paged_attn_decode(bits(q), kp0, vp0, bt, lens, 1 / math.sqrt(D), "bf16")
    assert np.max(np.abs(out.double().cpu().numpy() - ref)) <= TOL["bf16"]
    # private layout: each sequence's blocks copied to blocks of its own
    kp2 = torch.empty((8 * 4, Hkv, 32, D), dtype=torch.bfloat16, device="cuda")
    vp2 = torch.empty_like(kp2)
    bt2 = np.full_like(bt, -1)
    for i in range(8):
        for j in range(int((bt[i] >= 0).sum())):
            kp2[i * 4 + j] = kp[int(bt[i, j])]
            vp2[i * 4 + j] = vp[int(bt[i, j])]
            bt2[i, j] = i * 4 + j
    out2 = B.paged_attn_decode(q, kp2, vp2, torch.from_numpy(bt2).cuda(),
                               torch.from_numpy(lens).cuda(), 1 / math.sqrt(D))
    assert torch.equal(out, out2)
