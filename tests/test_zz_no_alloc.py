"""The allocation-free decode entry point against the workspace entry point and the fp64
oracle (GPU).

paged_attn_decode_no_alloc serves callers that cannot allocate device memory (an engine
that gives all free HBM to its KV pool, a plugin interface that forbids allocation inside
the op, a loop where cudaMalloc would synchronise the device): it keeps the split-context
scratch in the library's own static device array.  This file is collected last so that a
run stopping at the first failure has already run every other test; it also passes alone
in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_392_b200 import binding as B
from paged_kv_cache_392_b200 import workloads as W

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-5, "f16": 2e-3, "bf16": 1e-2}


def _case(dtype, seed):
    # lengths span several 256-token partitions and a ragged tail, so the split path and
    # its scratch are used; 48 query heads over 12 kv heads (groups of 4)
    lens = [1, 17, 255, 256, 700, 1500, 2049, 3333]
    wl = W.make_workload("no_alloc", lens, 48, 12, 128, dtype, seed, partition_tokens=256)
    vals = {k: v.cuda() for k, v in W.make_values(wl, "cpu").items()}
    bt = torch.from_numpy(wl.block_tables).cuda()
    lens_d = torch.from_numpy(wl.context_lens).cuda()
    return wl, vals, bt, lens_d


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
def test_no_alloc_matches_workspace_entry_on_two_calls(dtype):
    """Same kernels, same partitions: the output must be bit-identical to paged_attn_decode's
    with a caller workspace, on each of two calls in a row (the second one finds the first
    one's partials in the static scratch), and within tolerance of the fp64 oracle."""
    wl, v, bt, lens = _case(dtype, 11)
    desc = B.decode_desc(v["q"], v["k_pool"], v["v_pool"], bt, wl.partition_tokens)
    assert 0 < B.attn_workspace_bytes(desc) <= B.STATIC_WORKSPACE_BYTES
    ref = B.paged_attn_decode(v["q"], v["k_pool"], v["v_pool"], bt, lens, wl.scale,
                              partition_tokens=wl.partition_tokens)
    exact = oracle.paged_attn_decode(W.to_numpy_bits(v["q"]), W.to_numpy_bits(v["k_pool"]),
                                     W.to_numpy_bits(v["v_pool"]), wl.block_tables,
                                     wl.context_lens, wl.scale, dtype)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for _ in range(2):
        out = torch.full_like(v["q"], float("nan"))
        rc = B.lib().paged_attn_decode_no_alloc(
            ctypes.byref(desc), ctypes.c_void_p(v["q"].data_ptr()),
            ctypes.c_void_p(v["k_pool"].data_ptr()), ctypes.c_void_p(v["v_pool"].data_ptr()),
            ctypes.c_void_p(bt.data_ptr()), ctypes.c_void_p(lens.data_ptr()),
            ctypes.c_float(wl.scale), ctypes.c_void_p(out.data_ptr()), stream)
        assert rc == 0, B.last_error()
        torch.cuda.synchronize()
        assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
        err = float(np.max(np.abs(out.double().cpu().numpy() - exact)))
        assert np.isfinite(err) and err <= TOL[dtype], err
    assert B.device_faults(clear=True) == []


def test_no_alloc_rejects_batches_beyond_its_scratch():
    wl, v, bt, lens = _case("bf16", 12)
    # 1024 sequences x 48 heads x 16-token partitions of up to 3333 tokens: far beyond 32 MiB
    desc = B.make_desc(1024, 48, 12, 128, wl.num_blocks, wl.max_blocks_per_seq,
                       torch.bfloat16, partition_tokens=16)
    assert B.attn_workspace_bytes(desc) > B.STATIC_WORKSPACE_BYTES
    rc = B.lib().paged_attn_decode_no_alloc(
        ctypes.byref(desc), ctypes.c_void_p(v["q"].data_ptr()),
        ctypes.c_void_p(v["k_pool"].data_ptr()), ctypes.c_void_p(v["v_pool"].data_ptr()),
        ctypes.c_void_p(bt.data_ptr()), ctypes.c_void_p(lens.data_ptr()),
        ctypes.c_float(wl.scale), ctypes.c_void_p(v["q"].data_ptr()), None)
    assert rc == 1 and "static workspace" in B.last_error()
