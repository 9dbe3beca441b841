"""CPU checks of the C ABI: the library loads, exports every symbol include/pkv.h declares,
and rejects bad arguments on the host before any launch (no GPU needed)."""
import ctypes
import os
import re
import subprocess

import pytest

from paged_kv_cache_392_b200 import binding as B
from paged_kv_cache_392_b200 import build as pbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pkv.h")


def header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"\b([a-z_][a-z0-9_]*)\s*\(", text)
    return sorted({n for n in names
                   if n.startswith(("pkv_", "paged_attn_decode", "attn_decode", "kv_"))})


@pytest.fixture(scope="module")
def lib():
    pbuild.build()
    return B.lib()


def test_header_declares_the_binding_exports():
    assert header_functions() == sorted(B.EXPORTS)


def test_library_exports_every_header_symbol(lib):
    out = subprocess.check_output(["nm", "-D", "--defined-only", B.LIB_PATH], text=True)
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for name in header_functions():
        assert name in exported, name
        assert getattr(lib, name) is not None


def test_version_and_error_strings(lib):
    assert "sm_100a" in B.version()
    assert isinstance(B.last_error(), str)


def _desc(**kw):
    d = dict(num_seqs=4, num_q_heads=8, num_kv_heads=2, head_dim=128, num_blocks=64,
             max_blocks_per_seq=8, dtype=1, partition_tokens=0, block_size=16)
    d.update(kw)
    return B.AttnDesc(d["num_seqs"], d["num_q_heads"], d["num_kv_heads"], d["head_dim"],
                      d["block_size"], d["num_blocks"], d["max_blocks_per_seq"],
                      d["dtype"], d["partition_tokens"])


def test_workspace_bytes(lib):
    # 8 blocks * 16 = 128 tokens <= 512: one partition, no scratch
    assert B.attn_workspace_bytes(_desc()) == 0
    d = _desc(max_blocks_per_seq=100, partition_tokens=512)      # 1600 tokens: 4 parts
    rows = 4 * 8 * 4
    o = (rows * 128 * 4 + 255) // 256 * 256
    assert B.attn_workspace_bytes(d) == o + rows * 2 * 4
    with pytest.raises(B.PkvError):
        B.attn_workspace_bytes(_desc(head_dim=80))


@pytest.mark.parametrize("kw,code", [
    (dict(head_dim=96), 3), (dict(block_size=24), 3), (dict(num_q_heads=6), 3),
    (dict(num_q_heads=7), 1), (dict(dtype=9), 1), (dict(num_blocks=0), 1),
    (dict(partition_tokens=100), 1), (dict(max_blocks_per_seq=0), 1),
    (dict(num_seqs=-1), 1), (dict(dtype=0, head_dim=128, num_q_heads=16), 3),
])
def test_decode_rejects_bad_descriptors_before_launch(lib, kw, code):
    d = _desc(**kw)
    fake = ctypes.c_void_p(1 << 20)
    rc = lib.paged_attn_decode(ctypes.byref(d), fake, fake, fake, fake, fake, 0.1, fake,
                               None, 0, None)
    assert rc == code, B.last_error()
    assert B.last_error()


def test_decode_rejects_bad_pointers_and_workspace(lib):
    d = _desc()
    a = ctypes.c_void_p(1 << 20)
    rc = lib.paged_attn_decode(ctypes.byref(d), None, a, a, a, a, 0.1, a, None, 0, None)
    assert rc == 1 and "NULL" in B.last_error()
    rc = lib.paged_attn_decode(ctypes.byref(d), ctypes.c_void_p((1 << 20) + 8), a, a, a, a,
                               0.1, a, None, 0, None)
    assert rc == 1 and "aligned" in B.last_error()
    rc = lib.paged_attn_decode(ctypes.byref(d), a, a, a, a, a, float("nan"), a, None, 0, None)
    assert rc == 1
    d2 = _desc(max_blocks_per_seq=100, partition_tokens=512)
    rc = lib.paged_attn_decode(ctypes.byref(d2), a, a, a, a, a, 0.1, a, None, 0, None)
    assert rc == 1 and "workspace" in B.last_error()
    rc = lib.paged_attn_decode(ctypes.byref(d2), a, a, a, a, a, 0.1, a,
                               ctypes.c_void_p((1 << 20) + 16), 1 << 24, None)
    assert rc == 1 and "256" in B.last_error()


def test_empty_batches_launch_nothing(lib):
    d = _desc(num_seqs=0)
    assert lib.paged_attn_decode(ctypes.byref(d), None, None, None, None, None, 0.1, None,
                                 None, 0, None) == 0
    assert lib.kv_write(ctypes.byref(d), None, None, None, 0, None, None, None) == 0
    assert lib.kv_copy_blocks(ctypes.byref(d), None, 0, None, None, None) == 0


def test_kv_ops_reject_bad_arguments(lib):
    d = _desc()
    a = ctypes.c_void_p(1 << 20)
    assert lib.kv_write(ctypes.byref(d), a, a, a, -1, a, a, None) == 1
    assert lib.kv_write(ctypes.byref(d), a, None, a, 3, a, a, None) == 1
    assert lib.kv_write(ctypes.byref(d), a, a, ctypes.c_void_p((1 << 20) + 4), 3, a, a,
                        None) == 1
    assert lib.kv_copy_blocks(ctypes.byref(d), None, 2, a, a, None) == 1
    assert lib.kv_copy_blocks(ctypes.byref(_desc(head_dim=80)), a, 2, a, a, None) == 3
    assert lib.pkv_device_faults(None, 0, None) == 1


def test_swap_rejects_host_memory_the_device_cannot_reach(lib):
    import numpy as np
    d = _desc()
    a = ctypes.c_void_p(1 << 20)
    plain = np.zeros(64, np.uint8)          # pageable host memory: never handed to a kernel
    rc = lib.kv_swap_out(ctypes.byref(d), a, 1, a, a, ctypes.c_void_p(plain.ctypes.data),
                         ctypes.c_void_p(plain.ctypes.data), 4, None)
    assert rc in (1, 4) and B.last_error()
    assert lib.kv_swap_in(ctypes.byref(d), a, -1, a, a, 4, a, a, None) == 1
    assert lib.kv_swap_out(ctypes.byref(d), None, 0, None, None, None, None, 0, None) == 0


def test_fp8_partition_choice_reports_the_callers_or_a_library_size(lib):
    # a partition the caller sets is kept as is
    assert lib.pkv_fp8_partition_tokens(ctypes.byref(_desc(partition_tokens=256))) == 256
    # left to the library: 512, or 2048 for batches that fill the GPU on their own (the
    # wide choice needs a device to count its SMs, so on a host without one it is 512)
    n = lib.pkv_fp8_partition_tokens(ctypes.byref(_desc()))
    assert n in (512, 2048)
    # an invalid descriptor returns 0 and says why
    assert lib.pkv_fp8_partition_tokens(ctypes.byref(_desc(partition_tokens=24))) == 0
    assert "multiple of 16" in B.last_error()
    # the wide choice never needs more scratch than the default split
    big = _desc(num_seqs=64, num_q_heads=40, num_kv_heads=40, max_blocks_per_seq=128)
    assert lib.pkv_fp8_partition_tokens(ctypes.byref(big)) in (512, 2048)


def test_fault_bits_agree_across_header_binding_and_kernels():
    """pkv.h's PKV_FAULT_* values, the binding's decoder and the kernels' constants name the
    same bits."""
    text = open(HEADER).read()
    header = {int(v, 16) for v in re.findall(r"#define PKV_FAULT_\w+\s+(0x[0-9a-fA-F]+)u", text)}
    cuh = open(os.path.join(ROOT, "paged_kv_cache_392_b200", "csrc", "faults.cuh")).read()
    kernels = {int(v, 16) for v in re.findall(r"constexpr unsigned kFault\w+ = (0x[0-9a-f]+)u",
                                                cuh)}
    assert header == kernels == set(B.FAULT_BITS)
    assert len(header) == 7


def test_contiguous_decode_rejects_bad_arguments_before_launch(lib):
    a = ctypes.c_void_p(1 << 20)
    f = lib.attn_decode_contiguous
    assert f(ctypes.byref(_desc(dtype=0, num_q_heads=2)), a, a, a, a, 0.1, a, None, 0,
             None) == 3                                    # fp32: not built
    assert f(ctypes.byref(_desc(num_seqs=0)), None, None, None, None, 0.1, None, None, 0,
             None) == 0                                    # empty batch: nothing to do
    assert f(ctypes.byref(_desc()), a, None, a, a, 0.1, a, None, 0, None) == 1
    assert "NULL" in B.last_error()
    big = _desc(num_seqs=4096, num_kv_heads=8, num_q_heads=8, max_blocks_per_seq=4096)
    assert f(ctypes.byref(big), a, a, a, a, 0.1, a, None, 0, None) == 3
    assert "32-bit" in B.last_error()
    d2 = _desc(max_blocks_per_seq=100, partition_tokens=512)
    assert f(ctypes.byref(d2), a, a, a, a, 0.1, a, None, 0, None) == 1
    assert "workspace" in B.last_error()


def test_read_probe_rejects_bad_arguments_before_launch(lib):
    f = lib.pkv_read_probe
    n = ctypes.c_size_t(7)
    a = ctypes.c_void_p(1 << 20)
    assert f(None, 1 << 20, 8192, 0, ctypes.byref(n), None) == 1
    assert "aligned" in B.last_error()
    assert f(ctypes.c_void_p((1 << 20) + 8), 1 << 20, 8192, 0, ctypes.byref(n), None) == 1
    assert f(a, 1 << 20, 1000, 0, ctypes.byref(n), None) == 1    # unsupported chunk
    assert "chunk_bytes" in B.last_error()
    assert f(a, 4096, 8192, 0, ctypes.byref(n), None) == 1       # less than one chunk
    assert n.value == 7                                           # untouched on failure
