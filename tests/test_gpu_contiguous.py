"""GPU: attn_decode_contiguous, the decode over a contiguous cache [S][H_kv][Lmax][D] with no
block table (the baseline the pages compare the paged kernel with), against the fp64 oracle
run on the same bytes viewed as a paged pool with identity block tables, and bit for bit
against paged_attn_decode over the paged pool the cache was gathered from."""
import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_392_b200 import binding as B
from paged_kv_cache_392_b200 import workloads as W

pytestmark = pytest.mark.gpu

TOL = {"f16": 2e-3, "bf16": 1e-2}
RAGGED = [1, 2, 15, 16, 17, 31, 33, 100, 255, 256, 257, 511, 512, 513, 700, 1024, 1500]


@pytest.fixture(autouse=True)
def _clean_faults():
    B.device_faults(clear=True)
    yield
    assert B.device_faults(clear=True) == []


def bits(t):
    return W.to_numpy_bits(t)


def gather_contiguous(pool, block_tables, lens, lmax):
    """[S, H_kv, Lmax, D] cache holding each sequence's tokens in order; rows past its
    context are NaN (they must never be read)."""
    S = block_tables.shape[0]
    _, Hkv, _, D = pool.shape
    out = torch.full((S, Hkv, lmax, D), float("nan"), dtype=pool.dtype, device=pool.device)
    for s in range(S):
        L = int(lens[s])
        t = torch.arange(L, device=pool.device)
        blk = torch.from_numpy(block_tables[s]).to(pool.device).long()[t // 16]
        out[s, :, :L] = pool[blk, :, t % 16].permute(1, 0, 2)
    return out


def as_identity_pool(cache):
    """The same bytes viewed as a paged pool: block j of sequence s is pool block
    s * (Lmax / 16) + j, so the identity table s -> [s*nb, s*nb + nb) reads them."""
    S, Hkv, lmax, D = cache.shape
    nb = lmax // 16
    pool = cache.reshape(S, Hkv, nb, 16, D).permute(0, 2, 1, 3, 4).reshape(S * nb, Hkv, 16, D)
    bt = (np.arange(S, dtype=np.int32)[:, None] * nb + np.arange(nb, dtype=np.int32)[None])
    return pool.contiguous(), bt


def check(wl, vals, pt, full_oracle=True):
    d = {k: v.cuda() for k, v in vals.items()}
    bt = torch.from_numpy(wl.block_tables).cuda()
    lens = torch.from_numpy(wl.context_lens).cuda()
    lmax = wl.max_blocks_per_seq * 16
    kc = gather_contiguous(d["k_pool"], wl.block_tables, wl.context_lens, lmax)
    vc = gather_contiguous(d["v_pool"], wl.block_tables, wl.context_lens, lmax)
    out_c = B.attn_decode_contiguous(d["q"], kc, vc, lens, wl.scale, partition_tokens=pt)
    out_p = B.paged_attn_decode(d["q"], d["k_pool"], d["v_pool"], bt, lens, wl.scale,
                                partition_tokens=pt)
    torch.cuda.synchronize()
    assert torch.equal(out_c.view(torch.int16), out_p.view(torch.int16))
    kp_id, bt_id = as_identity_pool(kc)
    vp_id, _ = as_identity_pool(vc)
    ref = oracle.paged_attn_decode(bits(d["q"]), bits(kp_id), bits(vp_id), bt_id,
                                   wl.context_lens, wl.scale, wl.dtype)
    err = float(np.max(np.abs(out_c.double().cpu().numpy() - ref)))
    assert err <= TOL[wl.dtype], err
    return err


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (8, 2), (8, 1)])
@pytest.mark.parametrize("pt", [0, 64])
def test_contiguous_decode_matches_oracle_and_paged(dtype, D, Hq, Hkv, pt):
    wl = W.make_workload("contig", RAGGED, Hq, Hkv, D, dtype, 7 * Hq + Hkv + D + pt,
                         pool_factor=1.3, partition_tokens=pt)
    check(wl, W.make_values(wl, "cpu"), pt)


@pytest.mark.parametrize("name", ["opt13b", "gqa"])
def test_contiguous_full_size(name):
    wl = W.CONFIGS[name]()
    err = check(wl, W.make_values(wl, "cuda"), 0)
    print("%s contiguous: max abs error over all %d rows: %.3e"
          % (name, wl.num_seqs * wl.num_q_heads, err))


def test_contiguous_rejects_fp32_and_bad_lengths():
    wl = W.make_workload("c32", [20, 40], 2, 2, 64, "f32", 1)
    d = {k: v.cuda() for k, v in W.make_values(wl, "cpu").items()}
    kc = torch.zeros((2, 2, 48, 64), dtype=torch.float32, device="cuda")
    with pytest.raises(B.PkvError):
        B.attn_decode_contiguous(d["q"], kc, kc, torch.tensor([20, 40], dtype=torch.int32,
                                                              device="cuda"), wl.scale)
    q = d["q"].half()
    kc = torch.zeros((2, 2, 48, 64), dtype=torch.float16, device="cuda")
    B.attn_decode_contiguous(q, kc, kc, torch.tensor([20, 49], dtype=torch.int32,
                                                     device="cuda"), wl.scale)
    assert B.device_faults() == ["bad context length"]
