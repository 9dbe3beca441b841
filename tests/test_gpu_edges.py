"""GPU edge cases of the decode step against the oracle: block tables filled to the last
slot, one-token sequences, a thousand partitions per sequence, and a batch whose sequences
all share one physical block list (every CTA reads the same blocks)."""
import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_392_b200 import binding as B
from paged_kv_cache_392_b200 import workloads as W

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-5, "f16": 2e-3, "bf16": 1e-2}


@pytest.fixture(autouse=True)
def _clean_faults():
    B.device_faults(clear=True)
    yield
    assert B.device_faults(clear=True) == []


def bits(t):
    return W.to_numpy_bits(t)


def fused_step_vs_oracle(wl, pt=0, fused=True):
    vals = W.make_values(wl, "cpu")
    d = {k: v.cuda() for k, v in vals.items()}
    bt = torch.from_numpy(wl.block_tables).cuda()
    lens = torch.from_numpy(wl.context_lens).cuda()
    sl = torch.from_numpy(wl.slot_mapping).cuda()
    if fused:
        out = B.kv_write_and_decode(d["q"], d["k_new"], d["v_new"], sl, d["k_pool"],
                                    d["v_pool"], bt, lens, wl.scale, partition_tokens=pt)
    else:
        B.kv_write(d["k_new"], d["v_new"], sl, d["k_pool"], d["v_pool"])
        out = B.paged_attn_decode(d["q"], d["k_pool"], d["v_pool"], bt, lens, wl.scale,
                                  partition_tokens=pt)
    torch.cuda.synchronize()
    kp, vp = bits(vals["k_pool"]).copy(), bits(vals["v_pool"]).copy()
    oracle.kv_write(bits(vals["k_new"]), bits(vals["v_new"]), wl.slot_mapping, kp, vp)
    assert np.array_equal(bits(d["k_pool"]), kp) and np.array_equal(bits(d["v_pool"]), vp)
    ref = oracle.paged_attn_decode(bits(vals["q"]), kp, vp, wl.block_tables, wl.context_lens,
                                   wl.scale, wl.dtype)
    return np.max(np.abs(out.double().cpu().numpy() - ref))


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("fused", [True, False])
def test_tables_filled_to_the_last_slot(dtype, fused):
    # the longest sequence ends exactly at max_blocks_per_seq * 16, the new token in the very
    # last slot of its table
    lens = [16, 32, 160, 1024, 2048]
    wl = W.make_workload("full", lens, 8, 2, 64 if dtype == "f32" else 128, dtype, 41,
                         pool_factor=1.0)
    assert wl.context_lens.max() == wl.max_blocks_per_seq * 16
    assert wl.num_blocks == int(sum(L // 16 for L in lens))       # every pool block in use
    err = fused_step_vs_oracle(wl, fused=fused)
    assert err <= TOL[dtype], err


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_one_token_sequences(dtype):
    wl = W.make_workload("one", [1] * 37, 16, 4, 128, dtype, 42, pool_factor=1.0)
    err = fused_step_vs_oracle(wl)
    assert err <= TOL[dtype], err


def test_a_thousand_partitions_per_sequence():
    # 16-token partitions over 16384 tokens: 1024 partial states per (sequence, head) row
    wl = W.make_workload("parts", [16384, 16000], 8, 2, 128, "bf16", 43)
    err = fused_step_vs_oracle(wl, pt=16)
    assert err <= TOL["bf16"], err


def test_every_sequence_reading_the_same_blocks():
    # 24 sequences over one shared 43-block list (a common 688-token prefix) plus a private
    # last block each, where the new token lands: all CTAs read the same prefix blocks
    S, L = 24, 700
    wl = W.make_workload("shared", [L] * S, 8, 2, 128, "f16", 44)
    nshared = (L - 1) // 16
    bt = wl.block_tables.copy()
    prefix = bt[0, :nshared].copy()
    bt[:, :nshared] = prefix
    free = sorted(set(range(wl.num_blocks)) - set(prefix.tolist()))
    bt[:, nshared] = free[:S]
    wl.block_tables = bt
    wl.slot_mapping = bt[:, nshared].astype(np.int64) * 16 + (L - 1) % 16
    err = fused_step_vs_oracle(wl)
    assert err <= TOL["f16"], err
