"""The synthetic workloads match their stated recipe (shapes, dtypes, seeds, length
distributions, placement) and their tables are well formed: every sequence's blocks are
distinct pool blocks, shared by no other sequence, and each slot is the sequence's position
L-1 (CPU only)."""
import math

import numpy as np
import pytest

from paged_kv_cache_392_b200 import workloads as W


def _well_formed(wl):
    S, maxB = wl.block_tables.shape
    assert S == wl.num_seqs and maxB == wl.max_blocks_per_seq
    used = []
    for s, L in enumerate(wl.context_lens):
        n = -(-int(L) // 16)
        row = wl.block_tables[s]
        assert np.all(row[:n] >= 0) and np.all(row[:n] < wl.num_blocks)
        assert np.all(row[n:] == -1)
        used.extend(row[:n].tolist())
        pos = int(L) - 1
        assert wl.slot_mapping[s] == int(row[pos // 16]) * 16 + pos % 16
    assert len(used) == len(set(used))            # private blocks, none shared
    assert sorted(wl.free_order.tolist()) == list(range(wl.num_blocks))
    return len(used)


def test_tiny():
    wl = W.tiny()
    assert (wl.num_seqs, wl.num_q_heads, wl.num_kv_heads, wl.head_dim) == (4, 2, 2, 64)
    assert wl.dtype == "f32" and wl.seed == 0 and wl.num_blocks == 16
    assert wl.context_lens.tolist() == [5, 17, 33, 48]
    assert wl.scale == pytest.approx(1 / 8)
    assert _well_formed(wl) == 1 + 2 + 3 + 3


def test_opt13b_shape():
    wl = W.opt13b()
    assert (wl.num_seqs, wl.num_q_heads, wl.num_kv_heads, wl.head_dim) == (64, 40, 40, 128)
    assert wl.dtype == "f16" and wl.seed == 1
    L = wl.context_lens
    assert L.min() >= 16 and L.max() <= 2048 and int(L.sum()) == 39531
    need = _well_formed(wl)
    assert wl.num_blocks == math.ceil(1.1 * need)
    # lognormal around 512: the median sits near it, some lengths hit the 2048 clip
    assert 300 < np.median(L) < 800 and (L == 2048).sum() >= 1


def test_gqa_shape():
    wl = W.gqa()
    assert (wl.num_seqs, wl.num_q_heads, wl.num_kv_heads, wl.head_dim) == (128, 32, 8, 128)
    assert wl.dtype == "bf16" and wl.seed == 2
    L = wl.context_lens
    assert L.min() >= 256 and L.max() <= 4096 and int(L.sum()) == 287041
    assert wl.num_blocks == math.ceil(1.1 * _well_formed(wl))


def test_long_context_shape():
    wl = W.long_context()
    assert (wl.num_seqs, wl.num_q_heads, wl.num_kv_heads, wl.head_dim) == (8, 32, 8, 128)
    assert wl.dtype == "bf16" and wl.seed == 4 and wl.partition_tokens == 512
    assert wl.context_lens.tolist() == [32768] * 8
    assert wl.num_blocks == math.ceil(1.1 * _well_formed(wl))


def test_fork_pool_size():
    # 16 prompts x (65 shared blocks + 7 copies + 8 x 2 private tail blocks), 1.1x
    assert W.fork_pool_blocks() == math.ceil(1.1 * 16 * 88)


def test_values_are_seeded_and_shaped():
    wl = W.tiny()
    a, b = W.make_values(wl, "cpu"), W.make_values(wl, "cpu")
    for k in ("q", "k_pool", "v_pool", "k_new", "v_new"):
        assert np.array_equal(W.to_numpy_bits(a[k]), W.to_numpy_bits(b[k]))
    assert tuple(a["k_pool"].shape) == (16, 2, 16, 64)
    assert tuple(a["q"].shape) == (4, 2, 64)


def test_fp8_values():
    wl = W.make_workload("f8", [20, 40], 8, 2, 128, "bf16", 3)
    v = W.make_values_fp8(wl, "cpu")
    assert tuple(v["k_pool"].shape) == (wl.num_blocks, 2, 16, 128)
    assert tuple(v["v_pool"].shape) == (wl.num_blocks, 2, 128, 16)      # V transposed
    codes = np.concatenate([v["k_pool"].numpy().ravel(), v["v_pool"].numpy().ravel()])
    assert not np.any((codes & 0x7F) == 0x7F)        # no NaN codes: values saturate at 448
    ks = v["k_scale"].numpy()
    assert ks[1] > ks[0] and np.allclose(v["v_scale"].numpy(), 1.1 * ks, rtol=1e-6)
