"""GPU: the bounded shared-memory barrier wait running out, without any fault.

A test build of the library (short wait limit, and warp 0 of the first CTA withholds the
copy and the arrival of its second block) runs decode calls in a child process, one per
decode kernel (tensor-core 16-bit, CUDA-core fp32, E4M3 cache).  Each call must return
PKV_OK with PKV_FAULT_TIMEOUT set, leave every other work unit's output bit-identical to
the normal library's, and leave the context usable: a later call in the same process that
never reaches the withheld stage matches the normal library bit for bit with no fault."""
import json
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_392_b200 import binding as B
from paged_kv_cache_392_b200 import build as pbuild
from paged_kv_cache_392_b200 import workloads as W
from tests import timeout_cases as C

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
DEFINES = ["-DPKV_WAIT_TIMEOUT_NS=2000000ull", "-DPKV_TEST_WITHHOLD_BLOCK=1"]
TOL = {"f32": 1e-5, "f16": 2e-3, "bf16": 1e-2}


@pytest.fixture(scope="module")
def child_results(tmp_path_factory):
    lib = pbuild.build(out=pbuild.variant_path(DEFINES), defines=DEFINES)
    out = tmp_path_factory.mktemp("timeout")
    env = dict(os.environ, PKV_LIB=lib)
    subprocess.run([sys.executable, os.path.join(ROOT, "tests", "_timeout_child.py"),
                    str(out)], env=env, check=True, timeout=600, cwd=ROOT)
    with open(os.path.join(out, "faults.json")) as f:
        faults = json.load(f)
    return {n: (np.load(os.path.join(out, n + ".npy")), faults[n]) for n in C.CASES}


@pytest.mark.parametrize("name", C.WITHHOLD)
def test_wait_runs_out_sets_the_fault_and_spares_other_units(child_results, name):
    got, rec = child_results[name]
    assert rec["faults"] == ["barrier wait timed out"], rec
    assert rec["seconds"] < 30, rec
    B.device_faults(clear=True)
    ref = C.out_bits(C.run(name, "cuda"))          # the normal library, same inputs
    assert B.device_faults(clear=True) == []
    wl, _, _ = C.workload(name)
    g = wl.num_q_heads // wl.num_kv_heads
    spared = np.ones((wl.num_seqs, wl.num_q_heads), bool)
    spared[0, :g] = False                          # the query heads of (sequence 0, kv head 0)
    assert np.array_equal(got[spared], ref[spared])
    assert got.shape == ref.shape


def test_context_stays_usable_after_a_timeout(child_results):
    got, rec = child_results["normal_f16"]
    assert rec["faults"] == [], rec
    B.device_faults(clear=True)
    ref = C.out_bits(C.run("normal_f16", "cuda"))
    assert np.array_equal(got, ref)
    wl, vals, _ = C.workload("normal_f16")
    exact = oracle.paged_attn_decode(W.to_numpy_bits(vals["q"]), W.to_numpy_bits(vals["k_pool"]),
                                     W.to_numpy_bits(vals["v_pool"]), wl.block_tables,
                                     wl.context_lens, wl.scale, wl.dtype)
    val = torch.from_numpy(got).view(torch.float16).double().numpy()
    assert np.max(np.abs(val - exact)) <= TOL["f16"]
