"""Pins for the oracle's FP8 (E4M3) KV-cache functions, against torch's float8_e4m3fn
conversions (a library routine) and the format definition."""
import numpy as np
import pytest
import torch

import oracle


def test_e4m3_decoder_matches_torch_for_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().double().numpy()
    got = np.array([oracle.e4m3_to_f64(c) for c in codes])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan) and np.array_equal(got[~nan], ref[~nan])
    assert nan.sum() == 2                       # S.1111.111 only; no infinities


def _grid():
    vals = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).float().numpy()
    vals = np.sort(vals[np.isfinite(vals)])
    mids = (vals[1:] + vals[:-1]) / 2           # exact ties: round to even
    eps = np.float32(1e-7)
    rng = np.random.default_rng(0)
    rnd = (rng.standard_normal(20000) * rng.choice([1e-3, 0.05, 1, 30, 200], 20000))
    x = np.concatenate([vals, mids, mids * (1 + eps), mids * (1 - eps), rnd]).astype(np.float32)
    return x[np.abs(x) < 464]


def test_e4m3_encoder_matches_torch_rounding_in_range():
    x = _grid()
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.f32_to_e4m3(v) for v in x], np.uint8)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, (x[bad[:5]], got[bad[:5]], ref[bad[:5]])


def test_e4m3_encoder_saturates_and_keeps_nan():
    for v, code in ((448.0, 0x7E), (463.9, 0x7E), (464.0, 0x7E), (1e30, 0x7E),
                    (float("inf"), 0x7E), (-1e30, 0xFE), (-float("inf"), 0xFE)):
        assert oracle.f32_to_e4m3(v) == code
    assert oracle.f32_to_e4m3(float("nan")) == 0x7F
    assert oracle.f32_to_e4m3(-0.0) == 0x80 and oracle.f32_to_e4m3(0.0) == 0x00


@pytest.mark.parametrize("B", [16, 32])
def test_kv_write_fp8_quantises_into_the_two_layouts(B):
    rng = np.random.default_rng(1)
    NB, Hkv, D, T = 5, 2, 8, 3
    kn = torch.from_numpy(rng.standard_normal((T, Hkv, D)).astype(np.float32)).half()
    vn = torch.from_numpy(rng.standard_normal((T, Hkv, D)).astype(np.float32)).half()
    ks = np.array([0.01, 0.02], np.float32)
    vs = np.array([0.03, 0.005], np.float32)
    kp = np.zeros((NB, Hkv, B, D), np.uint8)
    vp = np.zeros((NB, Hkv, B // 16, D, 16), np.uint8)     # each 16-token half transposed
    slots = np.array([17, -1, 79], np.int64)
    bits = lambda t: t.view(torch.int16).numpy().view(np.uint16)  # noqa: E731
    oracle.kv_write_fp8(bits(kn), bits(vn), slots, ks, vs, kp, vp, "f16")
    ek = np.zeros_like(kp)
    ev = np.zeros_like(vp)
    # the V format: slot p of a transposed row holds token 2*(p//4) + p%2 + 8*((p//2)%2)
    token_of_slot = [2 * (p // 4) + p % 2 + 8 * ((p // 2) % 2) for p in range(16)]
    assert sorted(token_of_slot) == list(range(16))
    for t, sl in enumerate(slots):
        if sl < 0:
            continue
        blk, off = sl // B, sl % B
        vslot = token_of_slot.index(off % 16)
        for h in range(Hkv):
            qk = torch.from_numpy(kn[t, h].float().numpy() / ks[h]).to(torch.float8_e4m3fn)
            qv = torch.from_numpy(vn[t, h].float().numpy() / vs[h]).to(torch.float8_e4m3fn)
            ek[blk, h, off, :] = qk.view(torch.uint8).numpy()
            ev[blk, h, off // 16, :, vslot] = qv.view(torch.uint8).numpy()
    assert np.array_equal(kp, ek) and np.array_equal(vp, ev)


@pytest.mark.parametrize("B", [16, 32])
def test_fp8_decode_matches_bruteforce_on_dequantised_values(B):
    rng = np.random.default_rng(2)
    Hq, Hkv, D = 8, 2, 32
    lens = [1, 15, 16, 17, 31, 32, 33, 40, 70]
    nblk = [-(-L // B) for L in lens]
    NB = sum(nblk) + 2
    kp = rng.integers(0, 256, (NB, Hkv, B, D), dtype=np.uint8)
    vp = rng.integers(0, 256, (NB, Hkv, B // 16, D, 16), dtype=np.uint8)
    kp[(kp & 0x7F) == 0x7F] = 0x10              # no NaN codes
    vp[(vp & 0x7F) == 0x7F] = 0x10
    ks = rng.uniform(0.001, 0.01, Hkv).astype(np.float32)
    vs = rng.uniform(0.001, 0.01, Hkv).astype(np.float32)
    perm = rng.permutation(NB)
    bt = np.full((len(lens), max(nblk)), -1, np.int32)
    off = 0
    for s, n in enumerate(nblk):
        bt[s, :n] = perm[off:off + n]
        off += n
    q = rng.standard_normal((len(lens), Hq, D)).astype(np.float32)
    got = oracle.paged_attn_decode_fp8(q, kp, vp, ks, vs, bt, np.array(lens, np.int32), 0.2,
                                       "f32")
    table = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    token_of_slot = [2 * (p // 4) + p % 2 + 8 * ((p // 2) % 2) for p in range(16)]
    g = Hq // Hkv
    for s, L in enumerate(lens):
        for h in range(Hq):
            hk = h // g
            K = np.array([table[kp[bt[s, t // B], hk, t % B, :]] for t in range(L)]) * ks[hk]
            V = np.array([table[vp[bt[s, t // B], hk, (t % B) // 16, :,
                                   token_of_slot.index(t % 16)]]
                          for t in range(L)]) * vs[hk]
            x = K @ q[s, h].astype(np.float64) * 0.2
            w = np.exp(x - x.max())
            assert np.max(np.abs(got[s, h] - w @ V / w.sum())) <= 1e-12
