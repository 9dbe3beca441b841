"""GPU parity of the FP8 (E4M3) KV cache: the quantising write bit for bit, decode attention
within the q/out dtype's tolerance, against the oracle on the same seeded inputs."""
import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_392_b200 import binding as B
from paged_kv_cache_392_b200 import workloads as W

pytestmark = pytest.mark.gpu

TOL = {"f16": 2e-3, "bf16": 1e-2}


@pytest.fixture(autouse=True)
def _clean_faults():
    B.device_faults(clear=True)
    yield
    assert B.device_faults(clear=True) == []


def bits(t):
    return W.to_numpy_bits(t)


def u8(t):
    return t.detach().cpu().contiguous().numpy()


@pytest.mark.parametrize("dtype", ["f16", "bf16", "f32"])
def test_kv_write_fp8_bit_exact(dtype):
    wl = W.make_workload("w", [3, 17, 40, 100, 16], 4, 4, 128, dtype, 9)
    v = {k: t.cuda() for k, t in W.make_values_fp8(wl, "cpu").items()}
    slots = wl.slot_mapping.copy()
    slots[1] = -1
    # push some values past the largest code: they must saturate to +-448
    kn = v["k_new"].clone()
    kn[0, 0, :4] = torch.tensor([1e4, -1e4, 500.0, -0.0], dtype=kn.dtype)
    kp0, vp0 = u8(v["k_pool"]).copy(), u8(v["v_pool"]).copy()
    B.kv_write_fp8(kn, v["v_new"], torch.from_numpy(slots).cuda(), v["k_scale"], v["v_scale"],
                   v["k_pool"], v["v_pool"])
    torch.cuda.synchronize()
    oracle.kv_write_fp8(bits(kn), bits(v["v_new"]), slots, u8(v["k_scale"]), u8(v["v_scale"]),
                        kp0, vp0, dtype)
    assert np.array_equal(u8(v["k_pool"]), kp0) and np.array_equal(u8(v["v_pool"]), vp0)


RAGGED = [1, 2, 15, 16, 17, 33, 100, 255, 511, 512, 513, 1024, 1500]


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (8, 4), (8, 2), (16, 2)])
@pytest.mark.parametrize("pt", [0, 64])
def test_decode_fp8_parity(dtype, Hq, Hkv, pt):
    wl = W.make_workload("c", RAGGED, Hq, Hkv, 128, dtype, Hq * 10 + Hkv + pt,
                         partition_tokens=pt, pool_factor=1.3)
    v = {k: t.cuda() for k, t in W.make_values_fp8(wl, "cpu").items()}
    slots = torch.from_numpy(wl.slot_mapping).cuda()
    B.kv_write_fp8(v["k_new"], v["v_new"], slots, v["k_scale"], v["v_scale"], v["k_pool"],
                   v["v_pool"])
    out = B.paged_attn_decode_fp8(v["q"], v["k_pool"], v["v_pool"], v["k_scale"], v["v_scale"],
                                  torch.from_numpy(wl.block_tables).cuda(),
                                  torch.from_numpy(wl.context_lens).cuda(), wl.scale,
                                  partition_tokens=pt)
    torch.cuda.synchronize()
    ref = oracle.paged_attn_decode_fp8(bits(v["q"]), u8(v["k_pool"]), u8(v["v_pool"]),
                                       u8(v["k_scale"]), u8(v["v_scale"]), wl.block_tables,
                                       wl.context_lens, wl.scale, dtype)
    err = np.max(np.abs(out.double().cpu().numpy() - ref))
    assert err <= TOL[dtype], err


def test_decode_fp8_ignores_nan_codes_past_the_context():
    wl = W.make_workload("n", [5, 17, 40], 8, 2, 128, "bf16", 4, pool_factor=2.0)
    v = {k: t.cuda() for k, t in W.make_values_fp8(wl, "cpu").items()}
    used = np.zeros((wl.num_blocks, 16), bool)
    for s, L in enumerate(wl.context_lens):
        for t in range(L):
            used[wl.block_tables[s, t // 16], t % 16] = True
    kp, vp = v["k_pool"].cpu(), v["v_pool"].cpu()
    slot_of = np.array([4 * ((t & 7) >> 1) + 2 * (t >> 3) + (t & 1) for t in range(16)])
    for b in range(wl.num_blocks):
        for t in range(16):
            if not used[b, t]:
                kp[b, :, t, :] = 0x7F            # NaN codes
                vp[b, :, :, slot_of[t]] = 0xFF
    v["k_pool"], v["v_pool"] = kp.cuda(), vp.cuda()
    out = B.paged_attn_decode_fp8(v["q"], v["k_pool"], v["v_pool"], v["k_scale"], v["v_scale"],
                                  torch.from_numpy(wl.block_tables).cuda(),
                                  torch.from_numpy(wl.context_lens).cuda(), wl.scale)
    ref = oracle.paged_attn_decode_fp8(bits(v["q"]), u8(v["k_pool"]), u8(v["v_pool"]),
                                       u8(v["k_scale"]), u8(v["v_scale"]), wl.block_tables,
                                       wl.context_lens, wl.scale, "bf16")
    got = out.double().cpu().numpy()
    assert np.all(np.isfinite(got)) and np.max(np.abs(got - ref)) <= TOL["bf16"]


def test_decode_fp8_full_size_gqa_every_row():
    wl = W.gqa()
    v = W.make_values_fp8(wl, "cuda")
    out = B.paged_attn_decode_fp8(v["q"], v["k_pool"], v["v_pool"], v["k_scale"], v["v_scale"],
                                  torch.from_numpy(wl.block_tables).cuda(),
                                  torch.from_numpy(wl.context_lens).cuda(), wl.scale)
    ref = oracle.paged_attn_decode_fp8(bits(v["q"]), u8(v["k_pool"]), u8(v["v_pool"]),
                                       u8(v["k_scale"]), u8(v["v_scale"]), wl.block_tables,
                                       wl.context_lens, wl.scale, "bf16")
    err = float(np.max(np.abs(out.double().cpu().numpy() - ref)))
    print("gqa fp8: max abs error over all %d rows: %.3e" % (wl.num_seqs * 32, err))
    assert err <= TOL["bf16"], err


def test_fp8_blocks_copy_and_swap_bit_exact():
    NB, Hkv, D = 40, 4, 128
    g = torch.Generator().manual_seed(5)
    kp = torch.randint(0, 255, (NB, Hkv, 16, D), dtype=torch.uint8, generator=g)
    vp = torch.randint(0, 255, (NB, Hkv, D, 16), dtype=torch.uint8, generator=g)
    dk, dv = kp.cuda(), vp.cuda()
    desc = B.make_desc(0, Hkv, Hkv, D, NB, 1, B.PKV_FP8_E4M3)
    pairs = torch.tensor([[1, 30], [5, 31]], dtype=torch.int32, device="cuda")
    import ctypes
    rc = B.lib().kv_copy_blocks(ctypes.byref(desc), ctypes.c_void_p(pairs.data_ptr()), 2,
                                ctypes.c_void_p(dk.data_ptr()), ctypes.c_void_p(dv.data_ptr()),
                                ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0, B.last_error()
    torch.cuda.synchronize()
    ek, ev = kp.clone(), vp.clone()
    ek[[30, 31]] = kp[[1, 5]]
    ev[[30, 31]] = vp[[1, 5]]
    assert torch.equal(dk.cpu(), ek) and torch.equal(dv.cpu(), ev)


def test_decode_fp8_full_size_opt13b_every_row():
    """The OPT-13B-shaped batch in the bench's launch configuration: one query head per kv
    head (4 warps per CTA) and the library's wide FP8 partition, through the fused call."""
    wl = W.opt13b()
    vals = W.make_values_fp8(wl, "cuda")
    desc = B.make_desc(wl.num_seqs, wl.num_q_heads, wl.num_kv_heads, wl.head_dim,
                       wl.num_blocks, wl.max_blocks_per_seq, vals["q"].dtype)
    assert B.fp8_partition_tokens(desc) == 2048       # one unit per (sequence, kv head)
    kp0, vp0 = u8(vals["k_pool"]).copy(), u8(vals["v_pool"]).copy()
    out = B.kv_write_fp8_and_decode(vals["q"], vals["k_new"], vals["v_new"],
                                    torch.from_numpy(wl.slot_mapping).cuda(), vals["k_scale"],
                                    vals["v_scale"], vals["k_pool"], vals["v_pool"],
                                    torch.from_numpy(wl.block_tables).cuda(),
                                    torch.from_numpy(wl.context_lens).cuda(), wl.scale)
    torch.cuda.synchronize()
    ks, vs = u8(vals["k_scale"]), u8(vals["v_scale"])
    oracle.kv_write_fp8(bits(vals["k_new"]), bits(vals["v_new"]), wl.slot_mapping, ks, vs, kp0,
                        vp0, "f16")
    assert np.array_equal(u8(vals["k_pool"]), kp0) and np.array_equal(u8(vals["v_pool"]), vp0)
    ref = oracle.paged_attn_decode_fp8(bits(vals["q"]), kp0, vp0, ks, vs, wl.block_tables,
                                       wl.context_lens, wl.scale, "f16")
    err = float(np.max(np.abs(out.double().cpu().numpy() - ref)))
    print("opt13b fp8 (f16 q): max abs error over all %d rows: %.3e (tolerance %g)"
          % (wl.num_seqs * 40, err, TOL["f16"]))
    assert err <= TOL["f16"], err


@pytest.mark.parametrize("gain", [8.0, 32.0])
def test_decode_fp8_f16_q_enters_exactly(gain):
    """An f16 q reaches the score tiles unrounded (every E4M3 code and every f16 q value are
    f16 values, and the products accumulate in fp32).  A sharp softmax, q scaled by 8 or 32,
    makes the output sensitive to any rounding of q: a q carried with about 8 significant
    bits moves the scores by ~2^-9 * gain and misses the f16 tolerance, while only the f16
    weights and the f16 output round here."""
    wl = W.make_workload("x", [16, 100, 257, 700, 1500], 8, 2, 128, "f16", 77, pool_factor=1.3)
    v = {k: t.cuda() for k, t in W.make_values_fp8(wl, "cpu").items()}
    v["q"] = v["q"] * gain                        # a power of two: exact in f16
    out = B.paged_attn_decode_fp8(v["q"], v["k_pool"], v["v_pool"], v["k_scale"], v["v_scale"],
                                  torch.from_numpy(wl.block_tables).cuda(),
                                  torch.from_numpy(wl.context_lens).cuda(), wl.scale)
    torch.cuda.synchronize()
    ref = oracle.paged_attn_decode_fp8(bits(v["q"]), u8(v["k_pool"]), u8(v["v_pool"]),
                                       u8(v["k_scale"]), u8(v["v_scale"]), wl.block_tables,
                                       wl.context_lens, wl.scale, "f16")
    err = float(np.max(np.abs(out.double().cpu().numpy() - ref)))
    print("fp8, f16 q x %g: max abs error %.3e (tolerance %g)" % (gain, err, TOL["f16"]))
    assert err <= TOL["f16"], err
