"""GPU: the distinctness rules the boundary checks on the device.  kv_write / kv_write_fp8
skip every token whose slot another token of the call also names; kv_copy_blocks skips a
pair whose destination another pair also names or some pair reads as its source; kv_swap_*
skips pairs that share a destination; FP8 writes skip heads whose scale is not finite and
> 0.  Each sets its fault bit, and everything else is carried out bit for bit as the oracle
does it on the entries that remain."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_392_b200 import binding as B
from paged_kv_cache_392_b200 import workloads as W

pytestmark = pytest.mark.gpu

DUP = "duplicate slot or copy destination"


@pytest.fixture(autouse=True)
def _clean_faults():
    B.device_faults(clear=True)
    yield
    assert B.device_faults(clear=True) == []


def bits(t):
    return W.to_numpy_bits(t)


def u8(t):
    return t.detach().cpu().contiguous().numpy()


def drop_repeated(slots):
    """The slots the library writes: -1 for every slot named more than once (all of them)."""
    out = slots.copy()
    vals, counts = np.unique(slots[slots != -1], return_counts=True)
    out[np.isin(slots, vals[counts > 1])] = -1
    return out


def slots_with_repeats(T, NB, seed):
    rng = np.random.default_rng(seed)
    s = rng.choice(NB * 16, size=T, replace=False).astype(np.int64)
    s[35 % T] = s[3]                 # two tokens in different 32-token tiles
    s[11] = s[12] = s[10]            # three tokens in one tile
    s[20] = -1
    s[21] = -1                       # two skips are not a repeat
    return s


@pytest.mark.parametrize("T", [40, 5000])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_kv_write_skips_repeated_slots(T, dtype):
    Hkv, D = 4, 64 if dtype == "f32" else 128
    NB = T // 8 + 64
    kp = W.randn(torch, (NB, Hkv, 16, D), dtype, 1.0, 1, "cpu")
    vp = W.randn(torch, (NB, Hkv, 16, D), dtype, 1.0, 2, "cpu")
    kn = W.randn(torch, (T, Hkv, D), dtype, 1.0, 3, "cpu")
    vn = W.randn(torch, (T, Hkv, D), dtype, 1.0, 4, "cpu")
    slots = slots_with_repeats(T, NB, T)
    dk, dv = kp.cuda(), vp.cuda()
    B.kv_write(kn.cuda(), vn.cuda(), torch.from_numpy(slots).cuda(), dk, dv)
    assert B.device_faults() == [DUP]
    ek, ev = bits(kp).copy(), bits(vp).copy()
    oracle.kv_write(bits(kn), bits(vn), drop_repeated(slots), ek, ev)
    assert np.array_equal(bits(dk), ek) and np.array_equal(bits(dv), ev)


def test_kv_write_without_repeats_over_many_chunks_is_bit_exact():
    """5000 distinct slots: the check streams slot_mapping in several chunks and flags
    nothing; every token lands."""
    T, Hkv, D, NB = 5000, 2, 128, 700
    kp = W.randn(torch, (NB, Hkv, 16, D), "f16", 1.0, 5, "cpu")
    vp = W.randn(torch, (NB, Hkv, 16, D), "f16", 1.0, 6, "cpu")
    kn = W.randn(torch, (T, Hkv, D), "f16", 1.0, 7, "cpu")
    vn = W.randn(torch, (T, Hkv, D), "f16", 1.0, 8, "cpu")
    slots = np.random.default_rng(9).choice(NB * 16, size=T, replace=False).astype(np.int64)
    dk, dv = kp.cuda(), vp.cuda()
    B.kv_write(kn.cuda(), vn.cuda(), torch.from_numpy(slots).cuda(), dk, dv)
    ek, ev = bits(kp).copy(), bits(vp).copy()
    oracle.kv_write(bits(kn), bits(vn), slots, ek, ev)
    assert np.array_equal(bits(dk), ek) and np.array_equal(bits(dv), ev)


def test_kv_write_fp8_skips_repeated_slots_and_bad_scales():
    T, Hkv, D = 40, 4, 128
    wl = W.make_workload("w", [1] * T, Hkv, Hkv, D, "bf16", 3)
    NB = wl.num_blocks
    v = {k: t.cuda() for k, t in W.make_values_fp8(wl, "cpu").items()}
    slots = slots_with_repeats(T, NB, 1)
    kp0, vp0 = u8(v["k_pool"]).copy(), u8(v["v_pool"]).copy()
    B.kv_write_fp8(v["k_new"], v["v_new"], torch.from_numpy(slots).cuda(), v["k_scale"],
                   v["v_scale"], v["k_pool"], v["v_pool"])
    assert B.device_faults() == [DUP]
    ks, vs = u8(v["k_scale"]), u8(v["v_scale"])
    oracle.kv_write_fp8(bits(v["k_new"]), bits(v["v_new"]), drop_repeated(slots), ks, vs,
                        kp0, vp0, "bf16")
    assert np.array_equal(u8(v["k_pool"]), kp0) and np.array_equal(u8(v["v_pool"]), vp0)

    # a zero K scale on head 1 and a NaN V scale on head 2: those heads are not written
    bad_k, bad_v = v["k_scale"].clone(), v["v_scale"].clone()
    bad_k[1] = 0.0
    bad_v[2] = float("nan")
    fresh = np.random.default_rng(2).choice(NB * 16, size=T, replace=False).astype(np.int64)
    kp1, vp1 = u8(v["k_pool"]).copy(), u8(v["v_pool"]).copy()
    B.kv_write_fp8(v["k_new"], v["v_new"], torch.from_numpy(fresh).cuda(), bad_k, bad_v,
                   v["k_pool"], v["v_pool"])
    assert B.device_faults() == ["bad fp8 scale"]
    good = [0, 3]                      # the heads with usable scales, written by the oracle
    kn = np.ascontiguousarray(bits(v["k_new"])[:, good])
    vn = np.ascontiguousarray(bits(v["v_new"])[:, good])
    sub_k = np.ascontiguousarray(kp1[:, good])
    sub_v = np.ascontiguousarray(vp1[:, good])
    oracle.kv_write_fp8(kn, vn, fresh, ks[good].copy(), vs[good].copy(), sub_k, sub_v, "bf16")
    kp1[:, good], vp1[:, good] = sub_k, sub_v
    assert np.array_equal(u8(v["k_pool"]), kp1) and np.array_equal(u8(v["v_pool"]), vp1)


def test_kv_copy_blocks_skips_conflicting_pairs():
    NB, Hkv, D = 64, 4, 128
    kp = W.randn(torch, (NB, Hkv, 16, D), "f16", 1.0, 11, "cpu")
    vp = W.randn(torch, (NB, Hkv, 16, D), "f16", 1.0, 12, "cpu")
    pairs = np.array([[1, 40],     # fine
                      [2, 41],     # destination 41 named twice: skipped
                      [3, 41],     # skipped
                      [4, 5],      # destination 5 is the source of the next pair: skipped
                      [5, 42],     # fine (reads 5, which is then not written)
                      [6, 6],      # destination is its own source: skipped
                      [7, 43]],    # fine
                     np.int32)
    dk, dv = kp.cuda(), vp.cuda()
    B.kv_copy_blocks(torch.from_numpy(pairs).cuda(), dk, dv)
    assert B.device_faults() == [DUP]
    ek, ev = bits(kp).copy(), bits(vp).copy()
    oracle.kv_copy_blocks(pairs[[0, 4, 6]].copy(), ek, ev)
    assert np.array_equal(bits(dk), ek) and np.array_equal(bits(dv), ev)


def test_kv_swap_out_skips_pairs_sharing_a_destination():
    NB, NH, Hkv, D = 16, 8, 2, 64
    kp = W.randn(torch, (NB, Hkv, 16, D), "bf16", 1.0, 21, "cpu").cuda()
    vp = W.randn(torch, (NB, Hkv, 16, D), "bf16", 1.0, 22, "cpu").cuda()
    hk = torch.zeros((NH, Hkv, 16, D), dtype=torch.bfloat16).pin_memory()
    hv = torch.zeros_like(hk).pin_memory()
    pairs = torch.tensor([[3, 0], [4, 1], [5, 1], [3, 2]], dtype=torch.int32, device="cuda")
    B.kv_swap_out(pairs, kp, vp, hk, hv)
    assert B.device_faults() == [DUP]
    assert torch.equal(hk[0], kp[3].cpu()) and torch.equal(hv[2], vp[3].cpu())
    assert torch.count_nonzero(hk[1]) == 0 and torch.count_nonzero(hv[1]) == 0


def test_read_probe_streams_a_power_of_two_of_chunks_and_faults_nothing():
    """The bandwidth probe reads the largest power-of-two number of chunks that fits and
    leaves the device fault word clean; the buffer is only read."""
    buf = torch.arange(5 << 20, dtype=torch.int32, device="cuda")      # 20 MiB
    ref = buf.clone()
    for chunk in (2048, 4096, 8192, 16384):
        n = B.read_probe(buf, chunk)
        assert n == (16 << 20)                    # 2^k chunks: 16 MiB of the 20 MiB
    torch.cuda.synchronize()
    assert B.device_faults(clear=True) == []
    assert torch.equal(buf, ref)
