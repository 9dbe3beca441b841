"""Pins for the fp64 oracle: checks against things other than the oracle itself.

Each test ties the oracle to what the pages or the mathematics fix: brute-force contiguous
attention, a library routine (torch's fp64 scaled-dot-product attention) on the contiguous
layout, closed forms, invariants of the paged layout (placement permutation, shared vs private
blocks), the split/merge identity, the binary16 / bfloat16 definitions, and the pages' worked
examples under tests/golden/.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_392_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- number formats
def test_f16_decoder_matches_ieee_binary16_for_all_patterns():
    bits = np.arange(65536, dtype=np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([oracle.f16_to_f64(b) for b in bits])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


def test_bf16_decoder_matches_upper_half_of_binary32_for_all_patterns():
    bits = np.arange(65536, dtype=np.uint32)
    with np.errstate(invalid="ignore"):
        ref = (bits << 16).astype(np.uint32).view(np.float32).astype(np.float64)
    got = np.array([oracle.bf16_to_f64(b) for b in bits])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


# ---------------------------------------------------------------- helpers
def _rand_case(rng, lens, Hq, Hkv, D, B=16, spare=3, dtype="f32"):
    """Contiguous per-sequence K/V plus a random paged placement of the same data.

    Returns (q, kc, vc, k_pool, v_pool, bt) where kc[s] is [L_s, Hkv, D] (contiguous) and the
    pools hold the same rows scattered through bt; every other slot is noise."""
    S = len(lens)
    nblk = [-(-L // B) for L in lens]
    NB = sum(nblk) + spare
    q = rng.standard_normal((S, Hq, D)).astype(np.float32)
    k_pool = rng.standard_normal((NB, Hkv, B, D)).astype(np.float32) * 7.0
    v_pool = rng.standard_normal((NB, Hkv, B, D)).astype(np.float32) * 7.0
    perm = rng.permutation(NB)
    bt = np.full((S, max(nblk) + 2), -1, np.int32)
    kc, vc, off = [], [], 0
    for s, L in enumerate(lens):
        bt[s, :nblk[s]] = perm[off:off + nblk[s]]
        off += nblk[s]
        k = rng.standard_normal((L, Hkv, D)).astype(np.float32)
        v = rng.standard_normal((L, Hkv, D)).astype(np.float32)
        for t in range(L):  # scatter by hand: pool[block, head, offset, :]
            k_pool[bt[s, t // B], :, t % B, :] = k[t]
            v_pool[bt[s, t // B], :, t % B, :] = v[t]
        kc.append(k)
        vc.append(v)
    return q, kc, vc, k_pool, v_pool, bt


def _brute(q, kc, vc, scale, Hq, Hkv):
    """Contiguous, unpaged attention in fp64 with numpy (no table)."""
    g = Hq // Hkv
    out = np.zeros(q.shape, np.float64)
    for s in range(q.shape[0]):
        for h in range(Hq):
            K = kc[s][:, h // g, :].astype(np.float64)
            V = vc[s][:, h // g, :].astype(np.float64)
            x = K @ q[s, h].astype(np.float64) * scale
            w = np.exp(x - x.max())
            out[s, h] = w @ V / w.sum()
    return out


# ---------------------------------------------------------------- brute force / library
@pytest.mark.parametrize("Hq,Hkv,D,B", [(2, 2, 64, 16), (4, 2, 32, 16), (8, 1, 16, 16),
                                        (4, 2, 32, 32)])
def test_oracle_matches_bruteforce_contiguous_attention(Hq, Hkv, D, B):
    rng = np.random.default_rng(11)
    lens = [1, 5, 15, 16, 17, 31, 32, 33, 48, 70]
    q, kc, vc, kp, vp, bt = _rand_case(rng, lens, Hq, Hkv, D, B=B)
    scale = 1.0 / math.sqrt(D)
    got = oracle.paged_attn_decode(q, kp, vp, bt, np.array(lens, np.int32), scale, "f32")
    ref = _brute(q, kc, vc, scale, Hq, Hkv)
    assert np.max(np.abs(got - ref)) <= 1e-12


def test_oracle_matches_torch_sdpa_fp64_on_contiguous_layout():
    rng = np.random.default_rng(12)
    lens = [3, 16, 31, 64]
    Hq, Hkv, D = 4, 4, 64
    q, kc, vc, kp, vp, bt = _rand_case(rng, lens, Hq, Hkv, D)
    scale = 0.37
    got = oracle.paged_attn_decode(q, kp, vp, bt, np.array(lens, np.int32), scale, "f32")
    for s, L in enumerate(lens):
        Q = torch.from_numpy(q[s].astype(np.float64))[:, None, :]          # [H, 1, D]
        K = torch.from_numpy(kc[s].astype(np.float64)).permute(1, 0, 2)    # [H, L, D]
        V = torch.from_numpy(vc[s].astype(np.float64)).permute(1, 0, 2)
        ref = torch.nn.functional.scaled_dot_product_attention(Q, K, V, scale=scale)
        assert np.max(np.abs(got[s] - ref[:, 0, :].numpy())) <= 1e-12


def test_oracle_16bit_inputs_match_bruteforce_on_upcast_values():
    rng = np.random.default_rng(13)
    lens = [7, 16, 40]
    Hq, Hkv, D = 4, 2, 64
    q, kc, vc, kp, vp, bt = _rand_case(rng, lens, Hq, Hkv, D)
    for name in ("f16", "bf16"):
        td = torch.float16 if name == "f16" else torch.bfloat16

        def cast(a):
            return torch.from_numpy(a).to(td)

        bits = lambda t: t.view(torch.int16).numpy().view(np.uint16)  # noqa: E731
        back = lambda t: t.to(torch.float32).numpy()  # noqa: E731
        qt, kt, vt = cast(q), cast(kp), cast(vp)
        got = oracle.paged_attn_decode(bits(qt), bits(kt), bits(vt), bt,
                                       np.array(lens, np.int32), 0.125, name)
        kc2 = [back(cast(k)) for k in kc]
        vc2 = [back(cast(v)) for v in vc]
        ref = _brute(back(qt), kc2, vc2, 0.125, Hq, Hkv)
        assert np.max(np.abs(got - ref)) <= 1e-12


def test_golden_closed_form_example():
    with open(os.path.join(GOLDEN, "attention_closed_form.json")) as f:
        g = json.load(f)
    D, NB, B = g["head_dim"], g["num_blocks"], 16
    rng = np.random.default_rng(5)
    kp = rng.standard_normal((NB, 1, B, D)).astype(np.float32) * 50
    vp = rng.standard_normal((NB, 1, B, D)).astype(np.float32) * 50
    blk = g["physical_block"]
    kp[blk, 0, :2] = np.array(g["keys"], np.float32)
    vp[blk, 0, :2] = np.array(g["values"], np.float32)
    q = np.array(g["q"], np.float32).reshape(1, 1, D)
    out = oracle.paged_attn_decode(q, kp, vp, np.array([[blk]], np.int32),
                                   np.array([2], np.int32), g["scale"], "f32")
    assert np.max(np.abs(out[0, 0] - np.array(g["expected"]))) <= g["abs_tol"]


# ---------------------------------------------------------------- closed forms
def _tiny_arrays(seed=0, dtype="f32"):
    wl = W.tiny()
    vals = W.make_values(wl, "cpu")
    a = {k: W.to_numpy_bits(v) for k, v in vals.items()}
    return wl, a


def test_len1_returns_v0_exactly():
    wl, a = _tiny_arrays()
    lens = np.ones(wl.num_seqs, np.int32)
    out = oracle.paged_attn_decode(a["q"], a["k_pool"], a["v_pool"], wl.block_tables, lens,
                                   wl.scale, "f32")
    for s in range(wl.num_seqs):
        blk = wl.block_tables[s, 0]
        for h in range(wl.num_q_heads):
            assert np.array_equal(out[s, h], a["v_pool"][blk, h, 0].astype(np.float64))


def test_zero_query_or_zero_scale_gives_mean_of_values():
    wl, a = _tiny_arrays()
    for q, scale in ((np.zeros_like(a["q"]), wl.scale), (a["q"], 0.0)):
        out = oracle.paged_attn_decode(q, a["k_pool"], a["v_pool"], wl.block_tables,
                                       wl.context_lens, scale, "f32")
        for s, L in enumerate(wl.context_lens):
            for h in range(wl.num_q_heads):
                rows = [a["v_pool"][wl.block_tables[s, t // 16], h, t % 16].astype(np.float64)
                        for t in range(L)]
                assert np.max(np.abs(out[s, h] - np.mean(rows, axis=0))) <= 1e-12


def test_equal_keys_give_mean_and_dominant_key_gives_its_value():
    wl, a = _tiny_arrays()
    kp = a["k_pool"].copy()
    kp[:] = kp[0, 0, 0]
    out = oracle.paged_attn_decode(a["q"], kp, a["v_pool"], wl.block_tables, wl.context_lens,
                                   wl.scale, "f32")
    s, L = 3, int(wl.context_lens[3])
    rows = [a["v_pool"][wl.block_tables[s, t // 16], 1, t % 16].astype(np.float64)
            for t in range(L)]
    assert np.max(np.abs(out[s, 1] - np.mean(rows, axis=0))) <= 1e-12
    # one key aligned with q and 60+ logits above the rest: out = that token's V to e^-60
    kp = np.zeros_like(a["k_pool"])
    j = 21
    blk, off = wl.block_tables[s, j // 16], j % 16
    q = a["q"].copy()
    q[s, 1] = 0.0
    q[s, 1, 0] = 1.0
    kp[blk, 1, off, 0] = 80.0 / wl.scale
    out = oracle.paged_attn_decode(q, kp, a["v_pool"], wl.block_tables, wl.context_lens,
                                   wl.scale, "f32")
    assert np.max(np.abs(out[s, 1] - a["v_pool"][blk, 1, off].astype(np.float64))) <= 1e-20


# ---------------------------------------------------------------- paged-layout invariants
def test_output_unchanged_under_any_permutation_of_physical_blocks():
    wl, a = _tiny_arrays()
    ref = oracle.paged_attn_decode(a["q"], a["k_pool"], a["v_pool"], wl.block_tables,
                                   wl.context_lens, wl.scale, "f32")
    rng = np.random.default_rng(9)
    for _ in range(3):
        perm = rng.permutation(wl.num_blocks)        # new home of each old block
        kp = np.empty_like(a["k_pool"])
        vp = np.empty_like(a["v_pool"])
        kp[perm] = a["k_pool"]
        vp[perm] = a["v_pool"]
        bt = np.where(wl.block_tables >= 0, perm[np.maximum(wl.block_tables, 0)], -1)
        got = oracle.paged_attn_decode(a["q"], kp, vp, bt.astype(np.int32), wl.context_lens,
                                       wl.scale, "f32")
        assert np.array_equal(got, ref)


def test_shared_blocks_equal_private_copies():
    rng = np.random.default_rng(21)
    Hq = Hkv = 2
    D, B, L = 32, 16, 37
    NB = 12
    kp = rng.standard_normal((NB, Hkv, B, D)).astype(np.float32)
    vp = rng.standard_normal((NB, Hkv, B, D)).astype(np.float32)
    q = rng.standard_normal((2, Hq, D)).astype(np.float32)
    q[1] = q[0]
    shared = np.array([[4, 7, 1], [4, 7, 1]], np.int32)    # two sequences, same blocks
    kp[[9, 10, 11]] = kp[[4, 7, 1]]                         # private copies
    vp[[9, 10, 11]] = vp[[4, 7, 1]]
    private = np.array([[4, 7, 1], [9, 10, 11]], np.int32)
    lens = np.array([L, L], np.int32)
    o1 = oracle.paged_attn_decode(q, kp, vp, shared, lens, 0.2, "f32")
    o2 = oracle.paged_attn_decode(q, kp, vp, private, lens, 0.2, "f32")
    assert np.array_equal(o1, o2) and np.array_equal(o1[0], o1[1])


def test_gqa_consecutive_grouping_equals_mha_with_replicated_kv_heads():
    rng = np.random.default_rng(22)
    lens = [9, 33]
    Hq, Hkv, D = 6, 2, 16
    q, kc, vc, kp, vp, bt = _rand_case(rng, lens, Hq, Hkv, D)
    g = Hq // Hkv
    gqa = oracle.paged_attn_decode(q, kp, vp, bt, np.array(lens, np.int32), 0.3, "f32")
    kr = np.repeat(kp, g, axis=1)     # head h of the MHA pool = kv head h // g
    vr = np.repeat(vp, g, axis=1)
    mha = oracle.paged_attn_decode(q, kr, vr, bt, np.array(lens, np.int32), 0.3, "f32")
    assert np.array_equal(gqa, mha)


def test_tokens_past_context_len_are_not_read():
    wl, a = _tiny_arrays()
    ref = oracle.paged_attn_decode(a["q"], a["k_pool"], a["v_pool"], wl.block_tables,
                                   wl.context_lens, wl.scale, "f32")
    kp, vp = a["k_pool"].copy(), a["v_pool"].copy()
    used = np.zeros((wl.num_blocks, 16), bool)
    for s, L in enumerate(wl.context_lens):
        for t in range(L):
            used[wl.block_tables[s, t // 16], t % 16] = True
    unused = ~used                            # [block, offset], all heads
    kp.transpose(0, 2, 1, 3)[unused] = np.float32(1e30)
    vp.transpose(0, 2, 1, 3)[unused] = np.float32(np.nan)
    got = oracle.paged_attn_decode(a["q"], kp, vp, wl.block_tables, wl.context_lens,
                                   wl.scale, "f32")
    assert np.array_equal(got, ref)


# ---------------------------------------------------------------- split / merge identity
@pytest.mark.parametrize("P", [16, 32, 48, 512])
def test_split_lse_merge_equals_one_pass(P):
    rng = np.random.default_rng(31)
    lens = [5, 100, 257]
    Hq, Hkv, D = 4, 2, 32
    q, kc, vc, kp, vp, bt = _rand_case(rng, lens, Hq, Hkv, D)
    one = oracle.paged_attn_decode(q, kp, vp, bt, np.array(lens, np.int32), 0.4, "f32")
    for s, L in enumerate(lens):
        for h in range(Hq):
            out, part = oracle.split_lse_row(s, h, q, kp, vp, bt, np.array(lens, np.int32),
                                             0.4, "f32", P)
            assert part.shape[0] == -(-L // P)
            assert np.max(np.abs(out - one[s, h])) <= 1e-12
            # each partial: l_p >= 1 (its max term is exp(0)) and o_p / l_p is the partition's
            # own softmax average, checked by brute force on the contiguous copy
            K = kc[s][:, h // 2].astype(np.float64)
            V = vc[s][:, h // 2].astype(np.float64)
            x = K @ q[s, h].astype(np.float64) * 0.4
            for p in range(part.shape[0]):
                xs = x[p * P:(p + 1) * P]
                assert part[p, D] == pytest.approx(xs.max(), abs=1e-12)
                assert part[p, D + 1] >= 1.0
                w = np.exp(xs - xs.max())
                assert np.max(np.abs(part[p, :D] - w @ V[p * P:(p + 1) * P])) <= 1e-9


# ---------------------------------------------------------------- kv_write / kv_copy_blocks
def test_kv_write_places_rows_at_their_slots_and_nothing_else():
    rng = np.random.default_rng(41)
    NB, Hkv, B, D, T = 6, 3, 16, 8, 5
    kp = rng.standard_normal((NB, Hkv, B, D)).astype(np.float32)
    vp = rng.standard_normal((NB, Hkv, B, D)).astype(np.float32)
    kn = rng.standard_normal((T, Hkv, D)).astype(np.float32)
    vn = rng.standard_normal((T, Hkv, D)).astype(np.float32)
    slots = np.array([0, 95, -1, 17, 40], np.int64)
    k2, v2 = kp.copy(), vp.copy()
    oracle.kv_write(kn, vn, slots, k2, v2)
    kf, vf = kp.reshape(NB, Hkv, B, D).copy(), vp.copy()
    for t, sl in enumerate(slots):       # slot -> (block, offset) written out by hand
        if sl < 0:
            continue
        kf[sl // B, :, sl % B] = kn[t]
        vf[sl // B, :, sl % B] = vn[t]
    assert np.array_equal(k2, kf) and np.array_equal(v2, vf)
    with pytest.raises(oracle.OracleError):
        oracle.kv_write(kn, vn, np.array([0, 96, -1, 1, 2], np.int64), k2, v2)


def test_kv_write_16bit_is_a_byte_copy():
    rng = np.random.default_rng(42)
    kp = rng.integers(0, 65535, (4, 2, 16, 8), dtype=np.uint16)
    vp = rng.integers(0, 65535, (4, 2, 16, 8), dtype=np.uint16)
    kn = np.array(rng.integers(0, 65535, (2, 2, 8)), np.uint16)
    kn[0, 0, 0] = 0x7E01                       # a NaN pattern must survive unchanged
    vn = np.array(rng.integers(0, 65535, (2, 2, 8)), np.uint16)
    oracle.kv_write(kn, vn, np.array([63, 5], np.int64), kp, vp)
    assert np.array_equal(kp[3, :, 15], kn[0]) and np.array_equal(vp[0, :, 5], vn[1])


def test_kv_copy_blocks_copies_whole_blocks():
    rng = np.random.default_rng(43)
    kp = rng.standard_normal((8, 2, 16, 4)).astype(np.float32)
    vp = rng.standard_normal((8, 2, 16, 4)).astype(np.float32)
    k0, v0 = kp.copy(), vp.copy()
    oracle.kv_copy_blocks(np.array([[1, 5], [2, 7]], np.int32), kp, vp)
    exp_k, exp_v = k0.copy(), v0.copy()
    exp_k[5], exp_v[5], exp_k[7], exp_v[7] = k0[1], v0[1], k0[2], v0[2]
    assert np.array_equal(kp, exp_k) and np.array_equal(vp, exp_v)
    with pytest.raises(oracle.OracleError):
        oracle.kv_copy_blocks(np.array([[1, 8]], np.int32), kp, vp)


def test_kv_swap_copies_blocks_between_pools():
    rng = np.random.default_rng(44)
    dk = rng.standard_normal((6, 2, 16, 8)).astype(np.float32)
    dv = rng.standard_normal((6, 2, 16, 8)).astype(np.float32)
    hk = np.zeros((4, 2, 16, 8), np.float32)
    hv = np.zeros((4, 2, 16, 8), np.float32)
    pairs = np.array([[5, 0], [1, 3]], np.int32)
    oracle.kv_swap(pairs, dk, dv, hk, hv)
    ek, ev = np.zeros_like(hk), np.zeros_like(hv)
    ek[[0, 3]] = dk[[5, 1]]
    ev[[0, 3]] = dv[[5, 1]]
    assert np.array_equal(hk, ek) and np.array_equal(hv, ev)
    with pytest.raises(oracle.OracleError):
        oracle.kv_swap(np.array([[0, 4]], np.int32), dk, dv, hk, hv)
