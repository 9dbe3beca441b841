"""GPU parity: the CUDA path through the C ABI against the fp64 oracle on the same seeded
inputs.  kv_write and kv_copy_blocks must match bit for bit; decode attention within
1e-5 (fp32), 2e-3 (fp16), 1e-2 (bf16) max absolute error, accumulated in fp32."""
import math

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_392_b200 import binding as B
from paged_kv_cache_392_b200 import workloads as W

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-5, "f16": 2e-3, "bf16": 1e-2}
TDT = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


@pytest.fixture(autouse=True)
def _clean_faults():
    B.device_faults(clear=True)
    yield
    faults = B.device_faults(clear=True)
    assert faults == [], faults


def bits(t):
    return W.to_numpy_bits(t)


def as_f64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def run_step(wl, vals, partition_tokens=None, rows=None, write=True):
    """kv_write of each sequence's newest token, then decode; same on the oracle.
    Returns (gpu_out float64 [S,Hq,D] or rows, oracle_out)."""
    dev = torch.device("cuda")
    d = {k: v.to(dev) for k, v in vals.items()}
    bt = torch.from_numpy(wl.block_tables).to(dev)
    lens = torch.from_numpy(wl.context_lens).to(dev)
    slots = torch.from_numpy(wl.slot_mapping).to(dev)
    pt = wl.partition_tokens if partition_tokens is None else partition_tokens
    if write:
        B.kv_write(d["k_new"], d["v_new"], slots, d["k_pool"], d["v_pool"])
    out = B.paged_attn_decode(d["q"], d["k_pool"], d["v_pool"], bt, lens, wl.scale,
                              partition_tokens=pt)
    torch.cuda.synchronize()
    kp, vp = bits(vals["k_pool"]).copy(), bits(vals["v_pool"]).copy()
    if write:
        oracle.kv_write(bits(vals["k_new"]), bits(vals["v_new"]), wl.slot_mapping, kp, vp)
        # the GPU pools after the write must equal the oracle's byte for byte
        assert np.array_equal(bits(d["k_pool"]), kp)
        assert np.array_equal(bits(d["v_pool"]), vp)
    ref = oracle.paged_attn_decode(bits(vals["q"]), kp, vp, wl.block_tables, wl.context_lens,
                                   wl.scale, wl.dtype, rows=rows)
    got = as_f64(out)
    if rows is not None:
        got = got[rows[:, 0], rows[:, 1]]
    return got, ref


def small_wl(lens, Hq, Hkv, D, dtype, seed, partition_tokens=0, spare_factor=1.3):
    wl = W.make_workload("case", lens, Hq, Hkv, D, dtype, seed, pool_factor=spare_factor,
                         partition_tokens=partition_tokens)
    if dtype == "f32":
        wl.kv_std = 1.0
    return wl


def test_tiny_config_fp32():
    wl = W.tiny()
    vals = W.make_values(wl, "cpu")
    got, ref = run_step(wl, vals)
    assert np.max(np.abs(got - ref)) <= TOL["f32"]


RAGGED = [1, 2, 15, 16, 17, 31, 33, 100, 255, 256, 257, 511, 512, 513, 700, 1024, 1500]


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (8, 4), (8, 2), (8, 1)])
def test_decode_parity_shapes(dtype, D, Hq, Hkv):
    if dtype == "f32" and D == 128 and Hq // Hkv == 8:
        pytest.skip("fp32, D 128, group 8 is not built")
    wl = small_wl(RAGGED, Hq, Hkv, D, dtype, seed=Hq * 100 + Hkv * 10 + D)
    vals = W.make_values(wl, "cpu")
    got, ref = run_step(wl, vals)
    err = np.max(np.abs(got - ref))
    assert err <= TOL[dtype], err


@pytest.mark.parametrize("pt", [16, 32, 64, 128, 512, 2048])
@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_split_partitions_and_lse_reduce(pt, dtype):
    wl = small_wl(RAGGED + [2047, 2048, 2049], 8, 2, 128, dtype, seed=pt, partition_tokens=pt)
    vals = W.make_values(wl, "cpu")
    got, ref = run_step(wl, vals)
    err = np.max(np.abs(got - ref))
    assert err <= TOL[dtype], (pt, err)


@pytest.mark.parametrize("longest", [2048, 2049, 16384, 16400])
def test_lse_reduce_one_warp_and_eight_warp_rows(longest):
    """The reduce takes one warp per row while no row has more than 8 partitions and 8 warps
    per row beyond that (each warp loading batches of 8 partitions, rescaling its sums when a
    later batch holds a larger max).  256-token partitions: the longest sequence gives 8
    partitions (one warp), 9 (eight warps, one partition for most), 64 (eight warps, one full
    batch each) or 65 (a second batch for warp 0).  Every row count from 1 up is present;
    fp32 holds the merge to 1e-5."""
    lens = [1, 16, 255, 256, 257, 511, 513, 1023, 1025, 1500, 2047, longest]
    wl = small_wl(lens, 4, 2, 64, "f32", seed=longest, partition_tokens=256)
    vals = W.make_values(wl, "cpu")
    got, ref = run_step(wl, vals)
    err = np.max(np.abs(got - ref))
    assert err <= TOL["f32"], (longest, err)


def test_split_and_unsplit_agree_closely():
    wl = small_wl([3000, 1800, 4096], 4, 4, 128, "f32", seed=5)
    vals = W.make_values(wl, "cpu")
    a, ref = run_step(wl, vals, partition_tokens=64)
    # unsplit: 256 blocks per work unit, 64 per warp (more than one table chunk of 32)
    b, ref_b = run_step(wl, vals, partition_tokens=4096)
    assert np.array_equal(ref, ref_b)
    assert np.max(np.abs(a - ref)) <= 1e-5 and np.max(np.abs(b - ref)) <= 1e-5


def test_permutation_of_physical_blocks_is_bit_exact():
    wl = small_wl(RAGGED, 8, 2, 128, "bf16", seed=77)
    vals = {k: v.cuda() for k, v in W.make_values(wl, "cpu").items()}
    bt = torch.from_numpy(wl.block_tables).cuda()
    lens = torch.from_numpy(wl.context_lens).cuda()
    out1 = B.paged_attn_decode(vals["q"], vals["k_pool"], vals["v_pool"], bt, lens, wl.scale)
    perm = torch.from_numpy(np.random.default_rng(1).permutation(wl.num_blocks)).cuda()
    kp = torch.empty_like(vals["k_pool"])
    vp = torch.empty_like(vals["v_pool"])
    kp[perm] = vals["k_pool"]
    vp[perm] = vals["v_pool"]
    bt2 = torch.where(bt >= 0, perm[bt.clamp(min=0).long()].int(), bt)
    out2 = B.paged_attn_decode(vals["q"], kp, vp, bt2.contiguous(), lens, wl.scale)
    assert torch.equal(out1, out2)


def test_unused_slots_and_free_blocks_are_never_read():
    wl = small_wl([5, 17, 40], 4, 2, 64, "f16", seed=8, spare_factor=2.0)
    vals = W.make_values(wl, "cpu")
    kp, vp = vals["k_pool"], vals["v_pool"]
    used = np.zeros((wl.num_blocks, 16), bool)
    for s, L in enumerate(wl.context_lens):
        for t in range(L):
            used[wl.block_tables[s, t // 16], t % 16] = True
    mask = torch.from_numpy(~used)[:, None, :].expand(-1, kp.shape[1], -1)
    kp[mask] = float("inf")
    vp[mask] = float("nan")
    got, ref = run_step(wl, vals, write=False)
    assert np.all(np.isfinite(got)) and np.max(np.abs(got - ref)) <= TOL["f16"]


def test_kv_write_bit_exact_and_skip():
    wl = W.gqa(num_seqs=32)
    vals = W.make_values(wl, "cpu")
    slots = wl.slot_mapping.copy()
    slots[::5] = -1
    d = {k: v.cuda() for k, v in vals.items()}
    B.kv_write(d["k_new"], d["v_new"], torch.from_numpy(slots).cuda(), d["k_pool"], d["v_pool"])
    kp, vp = bits(vals["k_pool"]).copy(), bits(vals["v_pool"]).copy()
    oracle.kv_write(bits(vals["k_new"]), bits(vals["v_new"]), slots, kp, vp)
    assert np.array_equal(bits(d["k_pool"]), kp) and np.array_equal(bits(d["v_pool"]), vp)


@pytest.mark.parametrize("dtype,Hkv,D", [("f16", 32, 128), ("bf16", 8, 64), ("f32", 2, 64)])
def test_kv_copy_blocks_bit_exact(dtype, Hkv, D):
    NB = 300
    rng = np.random.default_rng(4)
    blocks = rng.permutation(NB)
    pairs = np.stack([blocks[:112], blocks[112:224]], 1).astype(np.int32)
    kp = W.randn(torch, (NB, Hkv, 16, D), dtype, 1.0, 10, "cpu")
    vp = W.randn(torch, (NB, Hkv, 16, D), dtype, 1.0, 11, "cpu")
    dk, dv = kp.cuda(), vp.cuda()
    B.kv_copy_blocks(torch.from_numpy(pairs).cuda(), dk, dv)
    ek, ev = bits(kp).copy(), bits(vp).copy()
    oracle.kv_copy_blocks(pairs, ek, ev)
    assert np.array_equal(bits(dk), ek) and np.array_equal(bits(dv), ev)


def test_fork_workload_shared_equals_private_and_cow_keeps_parent():
    """Parallel sampling: 2 prompts x 4 samples sharing a 100-token prefix; one decode step
    with copy-on-write; the result equals the same batch laid out with private copies."""
    NB = 80
    bm = B.BlockManager(NB, free_order=np.random.default_rng(0).permutation(NB))
    seqs = []
    for p in range(2):
        bm.add_seq(p * 4, 100)
        for k in range(1, 4):
            bm.fork(p * 4, p * 4 + k)
        seqs += [p * 4 + k for k in range(4)]
    Hq = Hkv = 4
    D = 128
    kp = W.randn(torch, (NB, Hkv, 16, D), "f16", 0.5, 1, "cpu").cuda()
    vp = W.randn(torch, (NB, Hkv, 16, D), "f16", 0.5, 2, "cpu").cuda()
    parent_blocks = {p: bm.block_table(p * 4) for p in range(2)}
    before = {p: (kp[parent_blocks[p]].clone(), vp[parent_blocks[p]].clone()) for p in range(2)}
    slots, pairs = bm.append_slots(seqs)
    assert len(pairs) == 6
    B.kv_copy_blocks(torch.from_numpy(pairs).cuda(), kp, vp)
    kn = W.randn(torch, (8, Hkv, D), "f16", 0.5, 3, "cpu").cuda()
    vn = W.randn(torch, (8, Hkv, D), "f16", 0.5, 4, "cpu").cuda()
    B.kv_write(kn, vn, torch.from_numpy(slots).cuda(), kp, vp)
    bt, lens = bm.block_tables(seqs, 8)
    q = W.randn(torch, (8, Hq, D), "f16", 1.0, 5, "cpu").cuda()
    out = B.paged_attn_decode(q, kp, vp, torch.from_numpy(bt).cuda(),
                              torch.from_numpy(lens).cuda(), 1 / math.sqrt(D))
    # parent's prompt blocks other than the copied one are untouched; the copied source
    # block differs from its copy only in the slot the writer filled
    for p in range(2):
        ok, ov = before[p]
        assert torch.equal(kp[parent_blocks[p][:-1]], ok[:-1])
        assert torch.equal(vp[parent_blocks[p][:-1]], ov[:-1])
    # private layout: every sequence gets its own copy of every block
    kp2 = torch.empty((8 * 8, Hkv, 16, D), dtype=torch.float16, device="cuda")
    vp2 = torch.empty_like(kp2)
    bt2 = np.full((8, 8), -1, np.int32)
    for i in range(8):
        n = int(np.sum(bt[i] >= 0))
        for j in range(n):
            kp2[i * 8 + j] = kp[int(bt[i, j])]
            vp2[i * 8 + j] = vp[int(bt[i, j])]
            bt2[i, j] = i * 8 + j
    out2 = B.paged_attn_decode(q, kp2, vp2, torch.from_numpy(bt2).cuda(),
                               torch.from_numpy(lens).cuda(), 1 / math.sqrt(D))
    assert torch.equal(out, out2)
    ref = oracle.paged_attn_decode(bits(q), bits(kp), bits(vp), bt, lens, 1 / math.sqrt(D), "f16")
    assert np.max(np.abs(as_f64(out) - ref)) <= TOL["f16"]


# ---- full-size workloads, every row -------------------------------------------------------
@pytest.mark.parametrize("name", ["opt13b", "gqa", "long"])
def test_full_size_workloads_every_row(name):
    """The full batches of the bench (seeded values drawn on the GPU): kv_write, then decode;
    every (sequence, query head) row against the fp64 oracle."""
    wl = W.CONFIGS[name]()
    vals = W.make_values(wl, "cuda")
    got, ref = run_step(wl, vals)
    assert got.shape == ref.shape == (wl.num_seqs, wl.num_q_heads, wl.head_dim)
    err = float(np.max(np.abs(got - ref)))
    print("%s: max abs error over all %d rows: %.3e (tolerance %g)"
          % (name, wl.num_seqs * wl.num_q_heads, err, TOL[wl.dtype]))
    assert err <= TOL[wl.dtype], err


# ---- device-side range checks -------------------------------------------------------------
def test_bad_device_values_set_fault_bits_and_touch_nothing_else():
    wl = small_wl([20, 40], 4, 4, 64, "f16", seed=9)
    vals = {k: v.cuda() for k, v in W.make_values(wl, "cpu").items()}
    kp0 = vals["k_pool"].clone()
    # slot out of range
    bad = torch.tensor([wl.num_blocks * 16, 3], dtype=torch.int64, device="cuda")
    B.kv_write(vals["k_new"], vals["v_new"], bad, vals["k_pool"], vals["v_pool"])
    assert B.device_faults() == ["bad slot"]
    kp_ref = kp0.clone()
    kp_ref[0, :, 3] = vals["k_new"][1]          # the valid slot was still written
    assert torch.equal(vals["k_pool"], kp_ref)
    # block id out of range in a table
    bt = torch.from_numpy(wl.block_tables).cuda()
    bt[1, 1] = wl.num_blocks + 5
    lens = torch.from_numpy(wl.context_lens).cuda()
    B.paged_attn_decode(vals["q"], vals["k_pool"], vals["v_pool"], bt, lens, wl.scale)
    assert B.device_faults() == ["bad block id"]
    # context length out of range
    lens2 = torch.tensor([0, 10_000], dtype=torch.int32, device="cuda")
    B.paged_attn_decode(vals["q"], vals["k_pool"], vals["v_pool"],
                        torch.from_numpy(wl.block_tables).cuda(), lens2, wl.scale)
    assert B.device_faults() == ["bad context length"]
    # copy pair out of range
    B.kv_copy_blocks(torch.tensor([[0, wl.num_blocks]], dtype=torch.int32, device="cuda"),
                     vals["k_pool"], vals["v_pool"])
    assert B.device_faults() == ["bad copy pair"]


@pytest.mark.parametrize("name", ["beam", "prefix"])
def test_sharing_workloads_decode_step(name):
    """One decode step of the beam-search / shared-prefix workloads (tables from the product
    block manager): copy-on-write copies, kv_write, decode, against the oracle; and the same
    step over private copies of every block is bit-identical."""
    import bench
    wl, pairs = bench.build_workload(name)
    d = W.make_values(wl, "cuda")
    kp, vp = bits(d["k_pool"]).copy(), bits(d["v_pool"]).copy()    # before the step
    bt = torch.from_numpy(wl.block_tables).cuda()
    lens = torch.from_numpy(wl.context_lens).cuda()
    B.kv_copy_blocks(torch.from_numpy(pairs).cuda(), d["k_pool"], d["v_pool"])
    B.kv_write(d["k_new"], d["v_new"], torch.from_numpy(wl.slot_mapping).cuda(), d["k_pool"],
               d["v_pool"])
    out = B.paged_attn_decode(d["q"], d["k_pool"], d["v_pool"], bt, lens, wl.scale)
    torch.cuda.synchronize()
    oracle.kv_copy_blocks(pairs, kp, vp)
    oracle.kv_write(bits(d["k_new"]), bits(d["v_new"]), wl.slot_mapping, kp, vp)
    assert np.array_equal(bits(d["k_pool"]), kp) and np.array_equal(bits(d["v_pool"]), vp)
    ref = oracle.paged_attn_decode(bits(d["q"]), kp, vp, wl.block_tables, wl.context_lens,
                                   wl.scale, wl.dtype)
    err = float(np.max(np.abs(as_f64(out) - ref)))
    print("%s: max abs error over all %d rows: %.3e" % (name, wl.num_seqs * wl.num_q_heads, err))
    assert err <= TOL[wl.dtype], err
    # private layout: gather every sequence's blocks into its own fresh blocks
    nb = (wl.context_lens + 15) // 16
    total = int(nb.sum())
    src = np.concatenate([wl.block_tables[i, :nb[i]] for i in range(wl.num_seqs)])
    kp2 = d["k_pool"][torch.from_numpy(src).long().cuda()].contiguous()
    vp2 = d["v_pool"][torch.from_numpy(src).long().cuda()].contiguous()
    bt2 = np.full_like(wl.block_tables, -1)
    off = 0
    for i in range(wl.num_seqs):
        bt2[i, :nb[i]] = np.arange(off, off + nb[i])
        off += nb[i]
    assert off == total
    out2 = B.paged_attn_decode(d["q"], kp2, vp2, torch.from_numpy(bt2).cuda(), lens, wl.scale)
    assert torch.equal(out, out2)
