"""fp64 CPU oracle for the paged KV-cache decode path -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's ``cpu_baseline`` leg may import
this package.  It shares no code with the CUDA library: the numerics live in
``pkv_oracle.c`` (plain C, double precision), the block-manager rules in
``block_manager.py`` (plain Python).  Arrays are numpy; 16-bit inputs are passed as their raw
bit patterns (``uint16``) or as ``float16``, together with a dtype name.

Sources followed: "Memory Optimization in LLM Serving with PagedAttention" (sections "How
PagedAttention Works" and "Advanced Capabilities: Memory Sharing with Copy-on-Write") and
"vLLM and PagedAttention: How Ideas from Operating Systems Accelerated LLM Inference".
"""
import ctypes
import os

import numpy as np

from . import build as _build

DTYPES = {"f32": 0, "f16": 1, "bf16": 2}
ELEM_SIZE = {"f32": 4, "f16": 2, "bf16": 2}
ERRORS = {0: "ok", 1: "bad argument", 2: "bad context length", 3: "bad block id",
          4: "bad slot", 5: "out of memory"}

_lib = None


class OracleError(RuntimeError):
    pass


def lib():
    """Load (building first if needed) the compiled oracle."""
    global _lib
    if _lib is None:
        # PKV_ORACLE_LIB lets the mutation tests load a deliberately broken build of this
        # same source in a child process; normal use builds and loads liboracle.so.
        path = os.environ.get("PKV_ORACLE_LIB") or _build.build()
        L = ctypes.CDLL(path)
        vp, i32, f64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_double
        L.orc_f16_to_f64.argtypes = [ctypes.c_uint16]
        L.orc_f16_to_f64.restype = f64
        L.orc_bf16_to_f64.argtypes = [ctypes.c_uint16]
        L.orc_bf16_to_f64.restype = f64
        L.orc_num_threads.restype = i32
        L.orc_paged_attn_decode.argtypes = [i32] * 7 + [vp, i32, vp, vp, i32, vp, vp, f64,
                                                        vp, i32, vp, i32]
        L.orc_paged_attn_decode.restype = i32
        L.orc_split_lse_row.argtypes = [i32] * 9 + [vp, i32, vp, vp, i32, vp, vp, f64, i32,
                                                    vp, vp]
        L.orc_split_lse_row.restype = i32
        L.orc_kv_write.argtypes = [i32] * 6 + [vp, vp, vp, vp, vp]
        L.orc_kv_write.restype = i32
        L.orc_kv_copy_blocks.argtypes = [i32, vp] + [i32] * 5 + [vp, vp]
        L.orc_kv_copy_blocks.restype = i32
        L.orc_kv_swap.argtypes = [i32, vp, vp, vp, i32, vp, vp, i32, ctypes.c_size_t]
        L.orc_kv_swap.restype = i32
        L.orc_e4m3_to_f64.argtypes = [ctypes.c_uint8]
        L.orc_e4m3_to_f64.restype = f64
        L.orc_f32_to_e4m3.argtypes = [ctypes.c_float]
        L.orc_f32_to_e4m3.restype = ctypes.c_uint8
        L.orc_kv_write_fp8.argtypes = [i32] * 5 + [vp, vp, i32, vp, vp, vp, vp, vp]
        L.orc_kv_write_fp8.restype = i32
        L.orc_paged_attn_decode_fp8.argtypes = [i32] * 7 + [vp, i32, vp, vp, vp, vp, vp, vp,
                                                            f64, vp, i32, vp, i32]
        L.orc_paged_attn_decode_fp8.restype = i32
        _lib = L
    return _lib


def num_threads() -> int:
    return lib().orc_num_threads()


def _ptr(a):
    return ctypes.c_void_p(a.ctypes.data) if a is not None else None


def _as_bits(a, dtype):
    """Return a C-contiguous array whose bytes are the values of ``dtype``."""
    a = np.ascontiguousarray(a)
    if dtype == "f32":
        if a.dtype != np.float32:
            raise TypeError("f32 data must be float32")
    elif a.dtype not in (np.uint16, np.int16, np.float16):
        raise TypeError("%s data must be float16 or raw 16-bit patterns" % dtype)
    return a


def _check(rc, what):
    if rc != 0:
        raise OracleError("%s: %s" % (what, ERRORS.get(rc, rc)))


def f16_to_f64(bits: int) -> float:
    return lib().orc_f16_to_f64(int(bits) & 0xFFFF)


def bf16_to_f64(bits: int) -> float:
    return lib().orc_bf16_to_f64(int(bits) & 0xFFFF)


def paged_attn_decode(q, k_pool, v_pool, block_tables, context_lens, scale, dtype,
                      rows=None, q_dtype=None, nthreads=None):
    """Decode attention through the block tables, exact softmax in fp64.

    q: [S, Hq, D]; k_pool, v_pool: [NB, Hkv, B, D]; block_tables: int32 [S, maxB];
    context_lens: int32 [S]; dtype: KV dtype name ("f32", "f16", "bf16"); q_dtype defaults
    to dtype.  rows: optional int array [n, 2] of (sequence, query head) to compute.
    Returns float64 [S, Hq, D] (rows=None) or [n, D].
    """
    q_dtype = q_dtype or dtype
    q = _as_bits(q, q_dtype)
    k_pool = _as_bits(k_pool, dtype)
    v_pool = _as_bits(v_pool, dtype)
    S, Hq, D = q.shape
    NB, Hkv, B, D2 = k_pool.shape
    if D2 != D or v_pool.shape != k_pool.shape:
        raise ValueError("shape mismatch")
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    if bt.ndim != 2 or bt.shape[0] != S:
        raise ValueError("block_tables must be [S, maxB]")
    lens = np.ascontiguousarray(context_lens, dtype=np.int32)
    if rows is None:
        out = np.empty((S, Hq, D), np.float64)
        rr, n = None, 0
    else:
        rr = np.ascontiguousarray(rows, dtype=np.int32).reshape(-1, 2)
        n = rr.shape[0]
        out = np.empty((n, D), np.float64)
    nt = nthreads or num_threads()
    rc = lib().orc_paged_attn_decode(S, Hq, Hkv, D, B, NB, bt.shape[1], _ptr(q),
                                     DTYPES[q_dtype], _ptr(k_pool), _ptr(v_pool),
                                     DTYPES[dtype], _ptr(bt), _ptr(lens), float(scale),
                                     _ptr(rr), n, _ptr(out), nt)
    _check(rc, "paged_attn_decode")
    return out


def split_lse_row(s, h, q, k_pool, v_pool, block_tables, context_lens, scale, dtype,
                  partition_tokens, q_dtype=None):
    """Split-context attention for one (s, h) row merged by log-sum-exp, in fp64.

    Returns (out [D], partials [num_partitions, D + 2] holding (o_p, m_p, l_p)).
    """
    q_dtype = q_dtype or dtype
    q = _as_bits(q, q_dtype)
    k_pool = _as_bits(k_pool, dtype)
    v_pool = _as_bits(v_pool, dtype)
    S, Hq, D = q.shape
    NB, Hkv, B, _ = k_pool.shape
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    lens = np.ascontiguousarray(context_lens, dtype=np.int32)
    L = int(lens[s])
    P = int(partition_tokens)
    npart = max(1, (L + P - 1) // P)
    out = np.empty(D, np.float64)
    partials = np.empty((npart, D + 2), np.float64)
    rc = lib().orc_split_lse_row(s, h, S, Hq, Hkv, D, B, NB, bt.shape[1], _ptr(q),
                                 DTYPES[q_dtype], _ptr(k_pool), _ptr(v_pool), DTYPES[dtype],
                                 _ptr(bt), _ptr(lens), float(scale), P, _ptr(out),
                                 _ptr(partials))
    _check(rc, "split_lse_row")
    return out, partials


def kv_write(k_new, v_new, slot_mapping, k_pool, v_pool):
    """Scatter new K/V rows [T, Hkv, D] into the pools [NB, Hkv, B, D], in place."""
    for a in (k_new, v_new, k_pool, v_pool):
        if not a.flags.c_contiguous:
            raise ValueError("arrays must be C-contiguous")
    T, Hkv, D = k_new.shape
    NB, Hkv2, B, D2 = k_pool.shape
    if (Hkv2, D2) != (Hkv, D) or v_new.shape != k_new.shape or v_pool.shape != k_pool.shape:
        raise ValueError("shape mismatch")
    if k_new.dtype.itemsize != k_pool.dtype.itemsize:
        raise TypeError("element size mismatch")
    sm = np.ascontiguousarray(slot_mapping, dtype=np.int64)
    rc = lib().orc_kv_write(T, Hkv, D, B, NB, k_pool.dtype.itemsize, _ptr(k_new), _ptr(v_new),
                            _ptr(sm), _ptr(k_pool), _ptr(v_pool))
    _check(rc, "kv_write")


def kv_copy_blocks(pairs, k_pool, v_pool):
    """Copy whole blocks src -> dst for each (src, dst) pair in both pools, in place."""
    for a in (k_pool, v_pool):
        if not a.flags.c_contiguous:
            raise ValueError("arrays must be C-contiguous")
    NB, Hkv, B, D = k_pool.shape
    pr = np.ascontiguousarray(pairs, dtype=np.int32).reshape(-1, 2)
    rc = lib().orc_kv_copy_blocks(pr.shape[0], _ptr(pr), Hkv, D, B, NB,
                                  k_pool.dtype.itemsize, _ptr(k_pool), _ptr(v_pool))
    _check(rc, "kv_copy_blocks")


def kv_swap(pairs, src_k, src_v, dst_k, dst_v):
    """Block dst of (dst_k, dst_v) := block src of (src_k, src_v) for each (src, dst) pair.
    Pools are [blocks, Hkv, B, D] arrays of one element size (device <-> host swap)."""
    for a in (src_k, src_v, dst_k, dst_v):
        if not a.flags.c_contiguous:
            raise ValueError("arrays must be C-contiguous")
    if src_k.shape[1:] != dst_k.shape[1:] or src_k.dtype.itemsize != dst_k.dtype.itemsize:
        raise ValueError("block shapes differ")
    bb = int(np.prod(src_k.shape[1:])) * src_k.dtype.itemsize
    pr = np.ascontiguousarray(pairs, dtype=np.int32).reshape(-1, 2)
    rc = lib().orc_kv_swap(pr.shape[0], _ptr(pr), _ptr(src_k), _ptr(src_v), src_k.shape[0],
                           _ptr(dst_k), _ptr(dst_v), dst_k.shape[0], bb)
    _check(rc, "kv_swap")


# ---- FP8 (E4M3) KV cache: per-head fp32 scales, K [NB,Hkv,B,D], V [NB,Hkv,D,B] codes ------
def e4m3_to_f64(code: int) -> float:
    return lib().orc_e4m3_to_f64(int(code) & 0xFF)


def f32_to_e4m3(x: float) -> int:
    return int(lib().orc_f32_to_e4m3(float(x)))


def _fp8_v_shape_ok(v_pool, NB, Hkv, B, D):
    """FP8 V pools: [NB, Hkv, B/16, D, 16] (each 16-token half of a block transposed), which
    for B = 16 may also be given as [NB, Hkv, D, 16]."""
    return v_pool.shape == (NB, Hkv, B // 16, D, 16) or (B == 16 and v_pool.shape ==
                                                          (NB, Hkv, D, 16))


def kv_write_fp8(k_new, v_new, slot_mapping, k_scale, v_scale, k_pool, v_pool, dtype):
    """Quantise new K/V rows [T, Hkv, D] of ``dtype`` into uint8 E4M3 pools, in place:
    K pool [NB, Hkv, B, D]; V pool [NB, Hkv, B/16, D, 16]: each 16-token half of a block
    transposed, slot p of a row holding token 2*(p//4) + p%2 + 8*((p//2)%2) of the half
    ([NB, Hkv, D, 16] when B = 16)."""
    k_new = _as_bits(k_new, dtype)
    v_new = _as_bits(v_new, dtype)
    T, Hkv, D = k_new.shape
    NB, Hkv2, B, D2 = k_pool.shape
    if (Hkv2, D2) != (Hkv, D) or not _fp8_v_shape_ok(v_pool, NB, Hkv, B, D):
        raise ValueError("shape mismatch")
    for a in (k_pool, v_pool):
        if a.dtype != np.uint8 or not a.flags.c_contiguous:
            raise TypeError("pools must be C-contiguous uint8")
    ks = np.ascontiguousarray(k_scale, np.float32)
    vs = np.ascontiguousarray(v_scale, np.float32)
    sm = np.ascontiguousarray(slot_mapping, np.int64)
    rc = lib().orc_kv_write_fp8(T, Hkv, D, B, NB, _ptr(k_new), _ptr(v_new), DTYPES[dtype],
                                _ptr(sm), _ptr(ks), _ptr(vs), _ptr(k_pool), _ptr(v_pool))
    _check(rc, "kv_write_fp8")


def paged_attn_decode_fp8(q, k_pool, v_pool, k_scale, v_scale, block_tables, context_lens,
                          scale, q_dtype, rows=None, nthreads=None):
    """Decode attention over E4M3 pools (values code * per-head scale), exact in fp64."""
    q = _as_bits(q, q_dtype)
    S, Hq, D = q.shape
    NB, Hkv, B, D2 = k_pool.shape
    if D2 != D or not _fp8_v_shape_ok(v_pool, NB, Hkv, B, D):
        raise ValueError("shape mismatch")
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    lens = np.ascontiguousarray(context_lens, dtype=np.int32)
    ks = np.ascontiguousarray(k_scale, np.float32)
    vs = np.ascontiguousarray(v_scale, np.float32)
    if rows is None:
        out = np.empty((S, Hq, D), np.float64)
        rr, n = None, 0
    else:
        rr = np.ascontiguousarray(rows, dtype=np.int32).reshape(-1, 2)
        n = rr.shape[0]
        out = np.empty((n, D), np.float64)
    rc = lib().orc_paged_attn_decode_fp8(S, Hq, Hkv, D, B, NB, bt.shape[1], _ptr(q),
                                         DTYPES[q_dtype], _ptr(np.ascontiguousarray(k_pool)),
                                         _ptr(np.ascontiguousarray(v_pool)), _ptr(ks), _ptr(vs),
                                         _ptr(bt), _ptr(lens), float(scale), _ptr(rr), n,
                                         _ptr(out), nthreads or num_threads())
    _check(rc, "paged_attn_decode_fp8")
    return out
