"""GPU: kv_write_and_decode, the newest token's kv_write done inside the decode kernel,
against the oracle's kv_write followed by its decode, and bit for bit against the two
separate calls on the same inputs."""
import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_392_b200 import binding as B
from paged_kv_cache_392_b200 import workloads as W

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-5, "f16": 2e-3, "bf16": 1e-2}
RAGGED = [1, 2, 15, 16, 17, 31, 33, 100, 255, 256, 257, 511, 512, 513, 700, 1024, 1500]


@pytest.fixture(autouse=True)
def _clean_faults():
    B.device_faults(clear=True)
    yield
    assert B.device_faults(clear=True) == []


def bits(t):
    return W.to_numpy_bits(t)


def u8(t):
    return t.detach().cpu().contiguous().numpy()


def fused_and_separate(wl, vals, slots, pt):
    """Run the fused call on one copy of the pools and kv_write + paged_attn_decode on
    another; return (out_fused, out_separate, pools_fused, pools_separate)."""
    d = {k: v.cuda() for k, v in vals.items()}
    kp2, vp2 = d["k_pool"].clone(), d["v_pool"].clone()
    bt = torch.from_numpy(wl.block_tables).cuda()
    lens = torch.from_numpy(wl.context_lens).cuda()
    sl = torch.from_numpy(slots).cuda()
    out1 = B.kv_write_and_decode(d["q"], d["k_new"], d["v_new"], sl, d["k_pool"], d["v_pool"],
                                 bt, lens, wl.scale, partition_tokens=pt)
    B.kv_write(d["k_new"], d["v_new"], sl, kp2, vp2)
    out2 = B.paged_attn_decode(d["q"], kp2, vp2, bt, lens, wl.scale, partition_tokens=pt)
    torch.cuda.synchronize()
    return out1, out2, (d["k_pool"], d["v_pool"]), (kp2, vp2)


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (8, 2), (16, 2)])
@pytest.mark.parametrize("pt", [0, 64])
def test_fused_step_matches_oracle_and_separate_calls(dtype, Hq, Hkv, pt):
    D = 64 if dtype == "f32" else 128
    wl = W.make_workload("fused", RAGGED, Hq, Hkv, D, dtype, 31 * Hq + Hkv + pt,
                         pool_factor=1.3, partition_tokens=pt)
    if dtype == "f32":
        wl.kv_std = 1.0
    vals = W.make_values(wl, "cpu")
    out1, out2, (kp1, vp1), (kp2, vp2) = fused_and_separate(wl, vals, wl.slot_mapping, pt)
    assert np.array_equal(bits(kp1), bits(kp2)) and np.array_equal(bits(vp1), bits(vp2))
    assert np.array_equal(bits(out1), bits(out2))
    kp, vp = bits(vals["k_pool"]).copy(), bits(vals["v_pool"]).copy()
    oracle.kv_write(bits(vals["k_new"]), bits(vals["v_new"]), wl.slot_mapping, kp, vp)
    assert np.array_equal(bits(kp1), kp) and np.array_equal(bits(vp1), vp)
    ref = oracle.paged_attn_decode(bits(vals["q"]), kp, vp, wl.block_tables, wl.context_lens,
                                   wl.scale, dtype)
    err = np.max(np.abs(out1.double().cpu().numpy() - ref))
    assert err <= TOL[dtype], err


def test_fused_skips_minus_one_slots():
    wl = W.make_workload("skip", RAGGED, 8, 2, 128, "bf16", 5, pool_factor=1.3)
    vals = W.make_values(wl, "cpu")
    slots = wl.slot_mapping.copy()
    slots[::3] = -1
    out1, out2, (kp1, vp1), (kp2, vp2) = fused_and_separate(wl, vals, slots, 0)
    assert np.array_equal(bits(kp1), bits(kp2)) and np.array_equal(bits(vp1), bits(vp2))
    assert np.array_equal(bits(out1), bits(out2))
    kp, vp = bits(vals["k_pool"]).copy(), bits(vals["v_pool"]).copy()
    oracle.kv_write(bits(vals["k_new"]), bits(vals["v_new"]), slots, kp, vp)
    assert np.array_equal(bits(kp1), kp) and np.array_equal(bits(vp1), vp)


def test_fused_refuses_a_slot_that_is_not_the_newest_position():
    wl = W.make_workload("bad", [20, 40, 33], 4, 4, 64, "f16", 6, pool_factor=1.5)
    vals = {k: v.cuda() for k, v in W.make_values(wl, "cpu").items()}
    kp0, vp0 = vals["k_pool"].clone(), vals["v_pool"].clone()
    slots = wl.slot_mapping.copy()
    slots[1] -= 1                       # position L-2 of sequence 1: not the newest token
    out = B.kv_write_and_decode(vals["q"], vals["k_new"], vals["v_new"],
                                torch.from_numpy(slots).cuda(), vals["k_pool"],
                                vals["v_pool"], torch.from_numpy(wl.block_tables).cuda(),
                                torch.from_numpy(wl.context_lens).cuda(), wl.scale)
    assert B.device_faults() == ["bad slot"]
    # sequences 0 and 2 were written, sequence 1 was not
    kp_ref, vp_ref = kp0.clone(), vp0.clone()
    for s in (0, 2):
        sl = int(wl.slot_mapping[s])
        kp_ref[sl // 16, :, sl % 16] = vals["k_new"][s]
        vp_ref[sl // 16, :, sl % 16] = vals["v_new"][s]
    assert torch.equal(vals["k_pool"], kp_ref) and torch.equal(vals["v_pool"], vp_ref)
    assert torch.isfinite(out).all()


@pytest.mark.parametrize("name", ["opt13b", "gqa", "long"])
def test_fused_full_size_matches_separate_calls(name):
    """The bench's default launch configuration at full size: bit-identical to the two
    separate calls, and every row within tolerance of the fp64 oracle."""
    wl = W.CONFIGS[name]()
    vals = W.make_values(wl, "cuda")
    kp0, vp0 = bits(vals["k_pool"]).copy(), bits(vals["v_pool"]).copy()   # before the write
    out1, out2, (kp1, vp1), (kp2, vp2) = fused_and_separate(wl, vals, wl.slot_mapping, 0)
    assert torch.equal(kp1, kp2) and torch.equal(vp1, vp2)
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))
    oracle.kv_write(bits(vals["k_new"]), bits(vals["v_new"]), wl.slot_mapping, kp0, vp0)
    assert np.array_equal(bits(kp1), kp0) and np.array_equal(bits(vp1), vp0)
    ref = oracle.paged_attn_decode(bits(vals["q"]), kp0, vp0, wl.block_tables,
                                   wl.context_lens, wl.scale, wl.dtype)
    err = float(np.max(np.abs(out1.double().cpu().numpy() - ref)))
    print("%s fused: max abs error over all %d rows: %.3e"
          % (name, wl.num_seqs * wl.num_q_heads, err))
    assert err <= TOL[wl.dtype], err


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (8, 2), (16, 2)])
@pytest.mark.parametrize("pt", [0, 64])
def test_fused_fp8_step_matches_oracle_and_separate_calls(dtype, Hq, Hkv, pt):
    wl = W.make_workload("f8", RAGGED, Hq, Hkv, 128, dtype, 17 * Hq + Hkv + pt,
                         pool_factor=1.3, partition_tokens=pt)
    vals = {k: v.cuda() for k, v in W.make_values_fp8(wl, "cpu").items()}
    kp2, vp2 = vals["k_pool"].clone(), vals["v_pool"].clone()
    kp0, vp0 = u8(vals["k_pool"]).copy(), u8(vals["v_pool"]).copy()
    bt = torch.from_numpy(wl.block_tables).cuda()
    lens = torch.from_numpy(wl.context_lens).cuda()
    sl = torch.from_numpy(wl.slot_mapping).cuda()
    slots = wl.slot_mapping.copy()
    sl[::4] = -1
    slots[::4] = -1
    out1 = B.kv_write_fp8_and_decode(vals["q"], vals["k_new"], vals["v_new"], sl,
                                     vals["k_scale"], vals["v_scale"], vals["k_pool"],
                                     vals["v_pool"], bt, lens, wl.scale, partition_tokens=pt)
    B.kv_write_fp8(vals["k_new"], vals["v_new"], sl, vals["k_scale"], vals["v_scale"], kp2, vp2)
    out2 = B.paged_attn_decode_fp8(vals["q"], kp2, vp2, vals["k_scale"], vals["v_scale"], bt,
                                   lens, wl.scale, partition_tokens=pt)
    torch.cuda.synchronize()
    assert torch.equal(vals["k_pool"], kp2) and torch.equal(vals["v_pool"], vp2)
    assert np.array_equal(bits(out1), bits(out2))
    ks, vs = vals["k_scale"].cpu().numpy(), vals["v_scale"].cpu().numpy()
    oracle.kv_write_fp8(bits(vals["k_new"]), bits(vals["v_new"]), slots, ks, vs, kp0, vp0, dtype)
    assert np.array_equal(u8(vals["k_pool"]), kp0) and np.array_equal(u8(vals["v_pool"]), vp0)
    ref = oracle.paged_attn_decode_fp8(bits(vals["q"]), kp0, vp0, ks, vs, wl.block_tables,
                                       wl.context_lens, wl.scale, dtype)
    err = np.max(np.abs(out1.double().cpu().numpy() - ref))
    assert err <= TOL[dtype], err


def test_fused_fp8_refuses_a_slot_that_is_not_the_newest_position():
    wl = W.make_workload("f8bad", [20, 40, 33], 8, 2, 128, "bf16", 7, pool_factor=1.5)
    vals = {k: v.cuda() for k, v in W.make_values_fp8(wl, "cpu").items()}
    kp0, vp0 = vals["k_pool"].clone(), vals["v_pool"].clone()
    slots = wl.slot_mapping.copy()
    slots[2] -= 1
    sl = torch.from_numpy(slots).cuda()
    B.kv_write_fp8_and_decode(vals["q"], vals["k_new"], vals["v_new"], sl, vals["k_scale"],
                              vals["v_scale"], vals["k_pool"], vals["v_pool"],
                              torch.from_numpy(wl.block_tables).cuda(),
                              torch.from_numpy(wl.context_lens).cuda(), wl.scale)
    assert B.device_faults() == ["bad slot"]
    sl_ok = torch.from_numpy(wl.slot_mapping).cuda()
    sl_ok[2] = -1                     # what should have been written: sequences 0 and 1
    B.kv_write_fp8(vals["k_new"], vals["v_new"], sl_ok, vals["k_scale"], vals["v_scale"], kp0,
                   vp0)
    torch.cuda.synchronize()
    assert torch.equal(vals["k_pool"], kp0) and torch.equal(vals["v_pool"], vp0)


def test_fused_fp8_full_size_gqa_every_row():
    wl = W.gqa()
    vals = W.make_values_fp8(wl, "cuda")
    kp0, vp0 = u8(vals["k_pool"]).copy(), u8(vals["v_pool"]).copy()
    out = B.kv_write_fp8_and_decode(vals["q"], vals["k_new"], vals["v_new"],
                                    torch.from_numpy(wl.slot_mapping).cuda(), vals["k_scale"],
                                    vals["v_scale"], vals["k_pool"], vals["v_pool"],
                                    torch.from_numpy(wl.block_tables).cuda(),
                                    torch.from_numpy(wl.context_lens).cuda(), wl.scale)
    torch.cuda.synchronize()
    ks, vs = u8(vals["k_scale"]), u8(vals["v_scale"])
    oracle.kv_write_fp8(bits(vals["k_new"]), bits(vals["v_new"]), wl.slot_mapping, ks, vs, kp0,
                        vp0, "bf16")
    assert np.array_equal(u8(vals["k_pool"]), kp0) and np.array_equal(u8(vals["v_pool"]), vp0)
    ref = oracle.paged_attn_decode_fp8(bits(vals["q"]), kp0, vp0, ks, vs, wl.block_tables,
                                       wl.context_lens, wl.scale, "bf16")
    err = float(np.max(np.abs(out.double().cpu().numpy() - ref)))
    print("gqa fused fp8: max abs error over all %d rows: %.3e" % (wl.num_seqs * 32, err))
    assert err <= TOL["bf16"], err


@pytest.mark.parametrize("name", ["fork", "beam", "prefix"])
def test_fused_step_on_sharing_workloads(name):
    """The bench's step on the block-manager workloads: copy-on-write copies, then the fused
    write-and-decode; the new tokens land in blocks the copies made private.  Pools bit-exact
    with the oracle's copy + write, output bit-identical to the separate calls and every
    row within tolerance of the oracle."""
    import bench
    wl, pairs = bench.build_workload(name)
    d = W.make_values(wl, "cuda")
    kp0, vp0 = bits(d["k_pool"]).copy(), bits(d["v_pool"]).copy()
    bt = torch.from_numpy(wl.block_tables).cuda()
    lens = torch.from_numpy(wl.context_lens).cuda()
    sl = torch.from_numpy(wl.slot_mapping).cuda()
    pr = torch.from_numpy(np.ascontiguousarray(pairs, np.int32)).cuda()
    kp2, vp2 = d["k_pool"].clone(), d["v_pool"].clone()
    if len(pairs):
        B.kv_copy_blocks(pr, d["k_pool"], d["v_pool"])
        B.kv_copy_blocks(pr, kp2, vp2)
    out = B.kv_write_and_decode(d["q"], d["k_new"], d["v_new"], sl, d["k_pool"], d["v_pool"],
                                bt, lens, wl.scale)
    B.kv_write(d["k_new"], d["v_new"], sl, kp2, vp2)
    out2 = B.paged_attn_decode(d["q"], kp2, vp2, bt, lens, wl.scale)
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), out2.view(torch.int16))
    oracle.kv_copy_blocks(np.ascontiguousarray(pairs, np.int32), kp0, vp0)
    oracle.kv_write(bits(d["k_new"]), bits(d["v_new"]), wl.slot_mapping, kp0, vp0)
    assert np.array_equal(bits(d["k_pool"]), kp0) and np.array_equal(bits(d["v_pool"]), vp0)
    ref = oracle.paged_attn_decode(bits(d["q"]), kp0, vp0, wl.block_tables, wl.context_lens,
                                   wl.scale, wl.dtype)
    err = float(np.max(np.abs(out.double().cpu().numpy() - ref)))
    print("%s fused: max abs error over all %d rows: %.3e"
          % (name, wl.num_seqs * wl.num_q_heads, err))
    assert err <= TOL[wl.dtype], err
