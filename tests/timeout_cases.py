"""Decode calls shared by tests/test_gpu_timeout.py and its child process: the same seeded
inputs through whichever library build the process loaded.  In each "withhold" case the
first work unit (sequence 0, kv head 0, partition 0) gives its warp 0 at least two blocks,
so a build that withholds that warp's block 1 times out there; the "normal" case gives
sequence 0 a single block, so no build ever reaches the withheld stage."""
import torch

from paged_kv_cache_392_b200 import binding as B
from paged_kv_cache_392_b200 import workloads as W

# name: (context lengths, H_q, H_kv, D, dtype, fp8 cache, seed)
CASES = {
    "tc_bf16": ([100, 40, 700, 17], 8, 2, 128, "bf16", False, 101),     # tensor cores, 2 warps
    "simt_f32": ([200, 33, 70], 2, 2, 64, "f32", False, 102),           # CUDA cores, 4 warps
    "fp8_bf16": ([100, 40, 300], 8, 2, 128, "bf16", True, 103),          # E4M3 cache, 2 warps
    "normal_f16": ([10, 300, 33], 4, 4, 128, "f16", False, 104),         # seq 0: one block
}
WITHHOLD = [n for n in CASES if not n.startswith("normal")]


def workload(name):
    lens, hq, hkv, d, dt, fp8, seed = CASES[name]
    wl = W.make_workload(name, lens, hq, hkv, d, dt, seed, pool_factor=1.3)
    if dt == "f32":
        wl.kv_std = 1.0
    vals = (W.make_values_fp8 if fp8 else W.make_values)(wl, "cpu")
    return wl, vals, fp8


def run(name, device):
    wl, vals, fp8 = workload(name)
    d = {k: v.to(device) for k, v in vals.items()}
    bt = torch.from_numpy(wl.block_tables).to(device)
    lens = torch.from_numpy(wl.context_lens).to(device)
    if fp8:
        return B.paged_attn_decode_fp8(d["q"], d["k_pool"], d["v_pool"], d["k_scale"],
                                       d["v_scale"], bt, lens, wl.scale)
    return B.paged_attn_decode(d["q"], d["k_pool"], d["v_pool"], bt, lens, wl.scale)


def out_bits(out):
    return W.to_numpy_bits(out).copy()
