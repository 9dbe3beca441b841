"""ctypes binding for libpkv.so: argument marshalling only.

Every step of the decode path runs in the library's CUDA kernels; this module checks torch
tensors' devices, dtypes, shapes and contiguity, turns them into the C ABI's pointers and
sizes (``include/pkv.h``), and raises ``PkvError`` on a non-zero status.  There is no
fallback: if ``libpkv.so`` is missing, the first call raises.
"""
import ctypes
import os

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
# PKV_LIB names another build of the same sources to load instead (a variant compiled with
# build(out=..., defines=...), such as the CUDA-core-only decode used for A/B measurements).
LIB_PATH = os.environ.get("PKV_LIB") or os.path.join(HERE, "libpkv.so")

PKV_OK = 0
STATUS = {0: "PKV_OK", 1: "PKV_ERR_INVALID", 2: "PKV_ERR_OOM", 3: "PKV_ERR_UNSUPPORTED",
          4: "PKV_ERR_CUDA", 5: "PKV_ERR_NOT_FOUND"}
FAULT_BITS = {0x1: "bad context length", 0x2: "bad block id", 0x4: "bad slot",
              0x8: "bad copy pair", 0x10: "barrier wait timed out",
              0x20: "duplicate slot or copy destination", 0x40: "bad fp8 scale"}
DTYPE_CODE = {torch.float32: 0, torch.float16: 1, torch.bfloat16: 2, torch.uint8: 3}
PKV_FP8_E4M3 = 3
BLOCK_SIZE = 16

# Every symbol include/pkv.h declares.
EXPORTS = [
    "pkv_last_error", "pkv_version", "pkv_attn_workspace_bytes", "paged_attn_decode",
    "kv_write", "kv_copy_blocks", "pkv_device_faults", "paged_attn_decode_no_alloc",
    "pkv_bm_create", "pkv_bm_destroy",
    "pkv_bm_add_seq", "pkv_bm_append_slot", "pkv_bm_append_slots", "pkv_bm_fork",
    "pkv_bm_free_seq", "pkv_bm_block_table", "pkv_bm_block_tables", "pkv_bm_seq_len",
    "pkv_bm_refcount", "pkv_bm_num_free", "pkv_bm_num_seqs", "pkv_bm_free_list",
    "kv_swap_out", "kv_swap_in", "pkv_bm_set_host_pool", "pkv_bm_swap_out", "pkv_bm_swap_in",
    "pkv_bm_is_swapped", "pkv_bm_num_host_free", "kv_write_fp8", "paged_attn_decode_fp8",
    "kv_write_and_decode", "kv_write_fp8_and_decode", "pkv_fp8_partition_tokens",
    "attn_decode_contiguous", "pkv_read_probe",
]


class PkvError(RuntimeError):
    def __init__(self, status, message):
        super().__init__("%s: %s" % (STATUS.get(status, status), message))
        self.status = status


class OutOfBlocks(PkvError):
    pass


class AttnDesc(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "num_seqs", "num_q_heads", "num_kv_heads", "head_dim", "block_size", "num_blocks",
        "max_blocks_per_seq", "dtype", "partition_tokens")]


_lib = None


def lib():
    """Load libpkv.so (built in-tree by ``python -m paged_kv_cache_392_b200.build``), or the
    build that ``PKV_LIB`` names."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError("libpkv.so is not built (%s); run "
                           "`python -m paged_kv_cache_392_b200.build`" % LIB_PATH)
    L = ctypes.CDLL(LIB_PATH)
    vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    P = ctypes.POINTER
    dp = P(AttnDesc)
    sig = {
        "pkv_last_error": ([], ctypes.c_char_p),
        "pkv_version": ([], ctypes.c_char_p),
        "pkv_attn_workspace_bytes": ([dp], sz),
        "pkv_fp8_partition_tokens": ([dp], i32),
        "paged_attn_decode": ([dp, vp, vp, vp, vp, vp, ctypes.c_float, vp, vp, sz, vp], i32),
        "paged_attn_decode_no_alloc": ([dp, vp, vp, vp, vp, vp, ctypes.c_float, vp, vp], i32),
        "kv_write": ([dp, vp, vp, vp, i32, vp, vp, vp], i32),
        "kv_write_and_decode": ([dp, vp, vp, vp, vp, vp, vp, vp, vp, ctypes.c_float, vp, vp,
                                 sz, vp], i32),
        "kv_copy_blocks": ([dp, vp, i32, vp, vp, vp], i32),
        "attn_decode_contiguous": ([dp, vp, vp, vp, vp, ctypes.c_float, vp, vp, sz, vp], i32),
        "pkv_device_faults": ([P(ctypes.c_uint32), ctypes.c_int, vp], i32),
        "pkv_bm_create": ([i32, i32, vp, P(vp)], i32),
        "pkv_bm_destroy": ([vp], None),
        "pkv_bm_add_seq": ([vp, i64, i32], i32),
        "pkv_bm_append_slot": ([vp, i64, P(i64), P(i32), P(i32)], i32),
        "pkv_bm_append_slots": ([vp, vp, i32, vp, vp, P(i32)], i32),
        "pkv_bm_fork": ([vp, i64, i64], i32),
        "pkv_bm_free_seq": ([vp, i64], i32),
        "pkv_bm_block_table": ([vp, i64, vp, i32, P(i32)], i32),
        "pkv_bm_block_tables": ([vp, vp, i32, i32, vp, vp], i32),
        "pkv_bm_seq_len": ([vp, i64, P(i32)], i32),
        "pkv_bm_refcount": ([vp, i32, P(i32)], i32),
        "pkv_bm_num_free": ([vp], i32),
        "pkv_bm_num_seqs": ([vp], i32),
        "pkv_bm_free_list": ([vp, vp, i32], i32),
        "kv_swap_out": ([dp, vp, i32, vp, vp, vp, vp, i32, vp], i32),
        "kv_swap_in": ([dp, vp, i32, vp, vp, i32, vp, vp, vp], i32),
        "pkv_bm_set_host_pool": ([vp, i32, vp], i32),
        "pkv_bm_swap_out": ([vp, i64, vp, i32, P(i32)], i32),
        "pkv_bm_swap_in": ([vp, i64, vp, i32, P(i32)], i32),
        "pkv_bm_is_swapped": ([vp, i64, P(i32)], i32),
        "pkv_bm_num_host_free": ([vp], i32),
        "kv_write_fp8": ([dp, vp, vp, vp, i32, vp, vp, vp, vp, vp], i32),
        "paged_attn_decode_fp8": ([dp, vp, vp, vp, vp, vp, vp, vp, ctypes.c_float, vp, vp, sz,
                                   vp], i32),
        "kv_write_fp8_and_decode": ([dp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, ctypes.c_float,
                                     vp, vp, sz, vp], i32),
        "pkv_read_probe": ([vp, sz, i32, i32, P(sz), vp], i32),
    }
    for name, (args, res) in sig.items():
        f = getattr(L, name)
        f.argtypes = args
        f.restype = res
    _lib = L
    return L


def last_error():
    return lib().pkv_last_error().decode()


def version():
    return lib().pkv_version().decode()


def _check(rc):
    if rc != PKV_OK:
        msg = last_error()
        if rc == 2:
            raise OutOfBlocks(rc, msg)
        raise PkvError(rc, msg)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _stream(stream, device):
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream)


def _dev(t, name, dtype=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % name)
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if dtype is not None and t.dtype != dtype:
        raise TypeError("%s must be %s, got %s" % (name, dtype, t.dtype))


def make_desc(num_seqs, num_q_heads, num_kv_heads, head_dim, num_blocks, max_blocks_per_seq,
              dtype, partition_tokens=0, block_size=BLOCK_SIZE):
    code = DTYPE_CODE[dtype] if isinstance(dtype, torch.dtype) else int(dtype)
    return AttnDesc(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, num_blocks,
                    max_blocks_per_seq, code, partition_tokens)


def _pool_desc(k_pool, v_pool, num_seqs=0, num_q_heads=1, max_blocks_per_seq=1,
               partition_tokens=0):
    _dev(k_pool, "k_pool")
    _dev(v_pool, "v_pool", k_pool.dtype)
    if k_pool.dim() != 4 or v_pool.shape != k_pool.shape:
        raise ValueError("pools must both be [num_blocks, num_kv_heads, block_size, head_dim]")
    NB, Hkv, B, D = k_pool.shape
    if k_pool.dtype not in DTYPE_CODE:
        raise TypeError("unsupported pool dtype %s" % k_pool.dtype)
    return make_desc(num_seqs, num_q_heads, Hkv, D, NB, max_blocks_per_seq, k_pool.dtype,
                     partition_tokens, B)


def attn_workspace_bytes(desc):
    n = lib().pkv_attn_workspace_bytes(ctypes.byref(desc))
    err = last_error()
    if n == 0 and err:
        raise PkvError(1, err)
    return n


def fp8_partition_tokens(desc):
    """Partition size (tokens) the FP8 decode uses for ``desc`` on the current device."""
    n = lib().pkv_fp8_partition_tokens(ctypes.byref(desc))
    if n == 0:
        raise PkvError(1, last_error())
    return n


def decode_desc(q, k_pool, v_pool, block_tables, partition_tokens=0):
    S, Hq, D = q.shape
    return _pool_desc(k_pool, v_pool, S, Hq, block_tables.shape[1], partition_tokens)


def paged_attn_decode(q, k_pool, v_pool, block_tables, context_lens, scale, out=None,
                      workspace=None, partition_tokens=0, stream=None):
    """out[s, h] = softmax(q[s, h] . K^T * scale) . V over the sequence's paged tokens.

    q [S, H_q, D]; pools [NB, H_kv, 16, D] (same dtype as q); block_tables int32 [S, maxB];
    context_lens int32 [S]; out [S, H_q, D] (allocated if None); workspace: uint8 CUDA
    tensor of at least attn_workspace_bytes(desc) bytes (allocated if None and needed)."""
    _dev(q, "q", k_pool.dtype)
    _dev(block_tables, "block_tables", torch.int32)
    _dev(context_lens, "context_lens", torch.int32)
    if q.dim() != 3 or block_tables.dim() != 2 or block_tables.shape[0] != q.shape[0] or \
            context_lens.shape != (q.shape[0],):
        raise ValueError("q [S,Hq,D], block_tables [S,maxB], context_lens [S] expected")
    desc = decode_desc(q, k_pool, v_pool, block_tables, partition_tokens)
    if q.shape[2] != k_pool.shape[3]:
        raise ValueError("head_dim mismatch")
    if out is None:
        out = torch.empty_like(q)
    else:
        _dev(out, "out", q.dtype)
        if out.shape != q.shape:
            raise ValueError("out must have q's shape")
    need = attn_workspace_bytes(desc)
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    nbytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(lib().paged_attn_decode(ctypes.byref(desc), _ptr(q), _ptr(k_pool), _ptr(v_pool),
                                   _ptr(block_tables), _ptr(context_lens), float(scale),
                                   _ptr(out), _ptr(workspace), nbytes,
                                   _stream(stream, q.device)))
    return out


def attn_decode_contiguous(q, k_cache, v_cache, context_lens, scale, out=None, workspace=None,
                           partition_tokens=0, stream=None):
    """The same decode over a contiguous cache with no block table: k_cache / v_cache
    [S, H_kv, Lmax, D] (Lmax a multiple of 16), token t of sequence s at row t."""
    _dev(q, "q")
    _dev(k_cache, "k_cache", q.dtype)
    _dev(v_cache, "v_cache", q.dtype)
    _dev(context_lens, "context_lens", torch.int32)
    if q.dim() != 3 or k_cache.dim() != 4 or v_cache.shape != k_cache.shape or \
            k_cache.shape[0] != q.shape[0] or k_cache.shape[3] != q.shape[2] or \
            context_lens.shape != (q.shape[0],):
        raise ValueError("q [S,Hq,D], caches [S,H_kv,Lmax,D], context_lens [S] expected")
    S, Hq, D = q.shape
    Hkv, lmax = k_cache.shape[1], k_cache.shape[2]
    if lmax % BLOCK_SIZE:
        raise ValueError("Lmax must be a multiple of %d" % BLOCK_SIZE)
    desc = make_desc(S, Hq, Hkv, D, 1, lmax // BLOCK_SIZE, q.dtype, partition_tokens)
    if out is None:
        out = torch.empty_like(q)
    else:
        _dev(out, "out", q.dtype)
    need = attn_workspace_bytes(desc)
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    nbytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(lib().attn_decode_contiguous(ctypes.byref(desc), _ptr(q), _ptr(k_cache),
                                        _ptr(v_cache), _ptr(context_lens), float(scale),
                                        _ptr(out), _ptr(workspace), nbytes,
                                        _stream(stream, q.device)))
    return out


def kv_write_and_decode(q, k_new, v_new, slot_mapping, k_pool, v_pool, block_tables,
                        context_lens, scale, out=None, workspace=None, partition_tokens=0,
                        stream=None):
    """kv_write of each sequence's newest token (k_new / v_new [S, H_kv, D], slot_mapping
    int64 [S]: -1 or the slot of position context_lens[s]-1) and paged_attn_decode, in one
    launch.  Same result as the two calls when the slots' blocks are private to their
    sequences."""
    _dev(q, "q", k_pool.dtype)
    _dev(k_new, "k_new", k_pool.dtype)
    _dev(v_new, "v_new", k_pool.dtype)
    _dev(slot_mapping, "slot_mapping", torch.int64)
    _dev(block_tables, "block_tables", torch.int32)
    _dev(context_lens, "context_lens", torch.int32)
    if q.dim() != 3 or block_tables.dim() != 2 or block_tables.shape[0] != q.shape[0] or \
            context_lens.shape != (q.shape[0],):
        raise ValueError("q [S,Hq,D], block_tables [S,maxB], context_lens [S] expected")
    desc = decode_desc(q, k_pool, v_pool, block_tables, partition_tokens)
    if q.shape[2] != k_pool.shape[3]:
        raise ValueError("head_dim mismatch")
    if k_new.shape != (q.shape[0], k_pool.shape[1], q.shape[2]) or v_new.shape != k_new.shape \
            or slot_mapping.shape != (q.shape[0],):
        raise ValueError("k_new / v_new [S, H_kv, D] and slot_mapping [S] expected")
    if out is None:
        out = torch.empty_like(q)
    else:
        _dev(out, "out", q.dtype)
        if out.shape != q.shape:
            raise ValueError("out must have q's shape")
    need = attn_workspace_bytes(desc)
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    nbytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(lib().kv_write_and_decode(ctypes.byref(desc), _ptr(q), _ptr(k_new), _ptr(v_new),
                                     _ptr(slot_mapping), _ptr(k_pool), _ptr(v_pool),
                                     _ptr(block_tables), _ptr(context_lens), float(scale),
                                     _ptr(out), _ptr(workspace), nbytes,
                                     _stream(stream, q.device)))
    return out


STATIC_WORKSPACE_BYTES = 32 << 20   # PKV_STATIC_WORKSPACE_BYTES in include/pkv.h


def paged_attn_decode_no_alloc(q, k_pool, v_pool, block_tables, context_lens, scale,
                               out, partition_tokens=0, stream=None):
    """paged_attn_decode for callers that cannot allocate device memory: the split scratch
    lives in the library's own static device array (STATIC_WORKSPACE_BYTES per GPU) and
    ``out`` must be given.  Calls that overlap on the GPU share that array and race."""
    _dev(q, "q", k_pool.dtype)
    _dev(block_tables, "block_tables", torch.int32)
    _dev(context_lens, "context_lens", torch.int32)
    _dev(out, "out", q.dtype)
    if q.dim() != 3 or out.shape != q.shape or block_tables.dim() != 2 or \
            block_tables.shape[0] != q.shape[0] or context_lens.shape != (q.shape[0],):
        raise ValueError("q/out [S,Hq,D], block_tables [S,maxB], context_lens [S] expected")
    desc = decode_desc(q, k_pool, v_pool, block_tables, partition_tokens)
    _check(lib().paged_attn_decode_no_alloc(
        ctypes.byref(desc), _ptr(q), _ptr(k_pool), _ptr(v_pool), _ptr(block_tables),
        _ptr(context_lens), float(scale), _ptr(out), _stream(stream, q.device)))
    return out


def read_probe(buf, chunk_bytes=8192, ctas_per_sm=0, stream=None):
    """Stream the device buffer ``buf`` (any dtype, contiguous) through shared memory in
    permuted ``chunk_bytes`` copies and discard it; returns the bytes read (the largest
    power-of-two number of chunks that fits).  A read-bandwidth denominator for the roofline.
    ``ctas_per_sm`` sets the concurrency (0: as many CTAs as fit)."""
    if not (isinstance(buf, torch.Tensor) and buf.is_cuda and buf.is_contiguous()):
        raise ValueError("buf must be a contiguous CUDA tensor")
    n = ctypes.c_size_t()
    _check(lib().pkv_read_probe(_ptr(buf), buf.numel() * buf.element_size(), int(chunk_bytes),
                                int(ctas_per_sm), ctypes.byref(n), _stream(stream, buf.device)))
    return n.value


def kv_write(k_new, v_new, slot_mapping, k_pool, v_pool, stream=None):
    """k_pool[slot // 16, :, slot % 16] = k_new[t] (and V) for every t with slot != -1."""
    desc = _pool_desc(k_pool, v_pool)
    _dev(k_new, "k_new", k_pool.dtype)
    _dev(v_new, "v_new", k_pool.dtype)
    _dev(slot_mapping, "slot_mapping", torch.int64)
    T = k_new.shape[0]
    if k_new.shape != (T, k_pool.shape[1], k_pool.shape[3]) or v_new.shape != k_new.shape or \
            slot_mapping.shape != (T,):
        raise ValueError("k_new/v_new [T, H_kv, D] and slot_mapping [T] expected")
    _check(lib().kv_write(ctypes.byref(desc), _ptr(k_new), _ptr(v_new), _ptr(slot_mapping), T,
                          _ptr(k_pool), _ptr(v_pool), _stream(stream, k_pool.device)))


def _block_pools_desc(k_pool, v_pool):
    """Descriptor for whole-block moves: 16-bit / fp32 pools, or FP8 pools (uint8, V stored
    [NB, H_kv, D, 16]; a block's bytes are moved the same way)."""
    if k_pool.dtype == torch.uint8:
        NB, Hkv, Bs, D = _fp8_pools(k_pool, v_pool)
        return make_desc(0, Hkv, Hkv, D, NB, 1, PKV_FP8_E4M3, 0, Bs)
    return _pool_desc(k_pool, v_pool)


def kv_copy_blocks(src_dst_pairs, k_pool, v_pool, stream=None):
    """Block dst of both pools becomes a copy of block src, for each (src, dst) row."""
    desc = _block_pools_desc(k_pool, v_pool)
    _dev(src_dst_pairs, "src_dst_pairs", torch.int32)
    if src_dst_pairs.dim() != 2 or src_dst_pairs.shape[1] != 2:
        raise ValueError("src_dst_pairs must be [P, 2]")
    _check(lib().kv_copy_blocks(ctypes.byref(desc), _ptr(src_dst_pairs),
                                src_dst_pairs.shape[0], _ptr(k_pool), _ptr(v_pool),
                                _stream(stream, k_pool.device)))


def _host_pool(t, name, like):
    if not isinstance(t, torch.Tensor) or t.is_cuda or not t.is_pinned():
        raise ValueError("%s must be a pinned host tensor" % name)
    if not t.is_contiguous() or t.dtype != like.dtype or t.shape[1:] != like.shape[1:]:
        raise ValueError("%s must be [blocks, H_kv, 16, D] like the pools" % name)


def kv_swap_out(pairs, k_pool, v_pool, host_k, host_v, stream=None):
    """host block h := device block g for each (g, h) row of ``pairs`` (device int32)."""
    desc = _pool_desc(k_pool, v_pool)
    _dev(pairs, "pairs", torch.int32)
    _host_pool(host_k, "host_k", k_pool)
    _host_pool(host_v, "host_v", k_pool)
    if host_v.shape != host_k.shape:
        raise ValueError("host_k and host_v differ")
    _check(lib().kv_swap_out(ctypes.byref(desc), _ptr(pairs), pairs.shape[0], _ptr(k_pool),
                             _ptr(v_pool), _ptr(host_k), _ptr(host_v), host_k.shape[0],
                             _stream(stream, k_pool.device)))


def kv_swap_in(pairs, host_k, host_v, k_pool, v_pool, stream=None):
    """device block g := host block h for each (h, g) row of ``pairs`` (device int32)."""
    desc = _pool_desc(k_pool, v_pool)
    _dev(pairs, "pairs", torch.int32)
    _host_pool(host_k, "host_k", k_pool)
    _host_pool(host_v, "host_v", k_pool)
    if host_v.shape != host_k.shape:
        raise ValueError("host_k and host_v differ")
    _check(lib().kv_swap_in(ctypes.byref(desc), _ptr(pairs), pairs.shape[0], _ptr(host_k),
                            _ptr(host_v), host_k.shape[0], _ptr(k_pool), _ptr(v_pool),
                            _stream(stream, k_pool.device)))


def _fp8_pools(k_pool, v_pool):
    """FP8 pools, uint8 E4M3 codes: K [NB, H_kv, B, D] and V [NB, H_kv, B/16, D, 16] (each
    16-token half of a block transposed), which for B = 16 may also be [NB, H_kv, D, 16]."""
    _dev(k_pool, "k_pool", torch.uint8)
    _dev(v_pool, "v_pool", torch.uint8)
    if k_pool.dim() != 4:
        raise ValueError("FP8 K pool: [NB, H_kv, B, D]")
    NB, Hkv, Bs, D = k_pool.shape
    if v_pool.shape != (NB, Hkv, Bs // 16, D, 16) and not (
            Bs == 16 and v_pool.shape == (NB, Hkv, D, 16)):
        raise ValueError("FP8 V pool: [NB, H_kv, B/16, D, 16] (or [NB, H_kv, D, 16] for B 16)")
    return k_pool.shape


def kv_write_fp8(k_new, v_new, slot_mapping, k_scale, v_scale, k_pool, v_pool, stream=None):
    """Quantise new K/V rows [T, H_kv, D] (f16/bf16/f32) into the FP8 pools' slots."""
    NB, Hkv, Bs, D = _fp8_pools(k_pool, v_pool)
    _dev(k_new, "k_new")
    _dev(v_new, "v_new", k_new.dtype)
    _dev(slot_mapping, "slot_mapping", torch.int64)
    _dev(k_scale, "k_scale", torch.float32)
    _dev(v_scale, "v_scale", torch.float32)
    T = k_new.shape[0]
    if k_new.shape != (T, Hkv, D) or v_new.shape != k_new.shape or \
            slot_mapping.shape != (T,) or k_scale.shape != (Hkv,) or v_scale.shape != (Hkv,):
        raise ValueError("k_new/v_new [T, H_kv, D], slot_mapping [T], scales [H_kv] expected")
    desc = make_desc(0, Hkv, Hkv, D, NB, 1, k_new.dtype, 0, Bs)
    _check(lib().kv_write_fp8(ctypes.byref(desc), _ptr(k_new), _ptr(v_new), _ptr(slot_mapping),
                              T, _ptr(k_scale), _ptr(v_scale), _ptr(k_pool), _ptr(v_pool),
                              _stream(stream, k_pool.device)))


def paged_attn_decode_fp8(q, k_pool, v_pool, k_scale, v_scale, block_tables, context_lens,
                          scale, out=None, workspace=None, partition_tokens=0, stream=None):
    """Decode attention over FP8 pools; q/out f16 or bf16 [S, H_q, D]."""
    NB, Hkv, Bs, D = _fp8_pools(k_pool, v_pool)
    _dev(q, "q")
    _dev(k_scale, "k_scale", torch.float32)
    _dev(v_scale, "v_scale", torch.float32)
    _dev(block_tables, "block_tables", torch.int32)
    _dev(context_lens, "context_lens", torch.int32)
    S, Hq, Dq = q.shape
    if Dq != D or block_tables.shape[0] != S or context_lens.shape != (S,):
        raise ValueError("q [S,Hq,D], block_tables [S,maxB], context_lens [S] expected")
    desc = make_desc(S, Hq, Hkv, D, NB, block_tables.shape[1], q.dtype, partition_tokens, Bs)
    if out is None:
        out = torch.empty_like(q)
    need = attn_workspace_bytes(desc)
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    nbytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(lib().paged_attn_decode_fp8(ctypes.byref(desc), _ptr(q), _ptr(k_pool), _ptr(v_pool),
                                       _ptr(k_scale), _ptr(v_scale), _ptr(block_tables),
                                       _ptr(context_lens), float(scale), _ptr(out),
                                       _ptr(workspace), nbytes, _stream(stream, q.device)))
    return out


def kv_write_fp8_and_decode(q, k_new, v_new, slot_mapping, k_scale, v_scale, k_pool, v_pool,
                            block_tables, context_lens, scale, out=None, workspace=None,
                            partition_tokens=0, stream=None):
    """kv_write_fp8 of each sequence's newest token (k_new / v_new [S, H_kv, D] in q's dtype,
    slot_mapping int64 [S]: -1 or the slot of position context_lens[s]-1) fused into
    paged_attn_decode_fp8: one launch, same pools and output as the two calls."""
    NB, Hkv, Bs, D = _fp8_pools(k_pool, v_pool)
    _dev(q, "q")
    _dev(k_new, "k_new", q.dtype)
    _dev(v_new, "v_new", q.dtype)
    _dev(slot_mapping, "slot_mapping", torch.int64)
    _dev(k_scale, "k_scale", torch.float32)
    _dev(v_scale, "v_scale", torch.float32)
    _dev(block_tables, "block_tables", torch.int32)
    _dev(context_lens, "context_lens", torch.int32)
    S, Hq, Dq = q.shape
    if Dq != D or block_tables.shape[0] != S or context_lens.shape != (S,):
        raise ValueError("q [S,Hq,D], block_tables [S,maxB], context_lens [S] expected")
    if k_new.shape != (S, Hkv, D) or v_new.shape != k_new.shape or slot_mapping.shape != (S,):
        raise ValueError("k_new / v_new [S, H_kv, D] and slot_mapping [S] expected")
    desc = make_desc(S, Hq, Hkv, D, NB, block_tables.shape[1], q.dtype, partition_tokens, Bs)
    if out is None:
        out = torch.empty_like(q)
    need = attn_workspace_bytes(desc)
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    nbytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(lib().kv_write_fp8_and_decode(
        ctypes.byref(desc), _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(slot_mapping),
        _ptr(k_scale), _ptr(v_scale), _ptr(k_pool), _ptr(v_pool), _ptr(block_tables),
        _ptr(context_lens), float(scale), _ptr(out), _ptr(workspace), nbytes,
        _stream(stream, q.device)))
    return out


def device_faults(clear=True, stream=None, device=None):
    """Synchronise and return the device fault word's set bits as names."""
    word = ctypes.c_uint32(0)
    dev = device if device is not None else torch.device("cuda", torch.cuda.current_device())
    _check(lib().pkv_device_faults(ctypes.byref(word), 1 if clear else 0,
                                   _stream(stream, dev)))
    return [name for bit, name in FAULT_BITS.items() if word.value & bit]


class BlockManager:
    """Host block manager (C++ in libpkv): free list, reference counts, copy-on-write fork.

    Sequence ids are Python ints (int64).  Methods raise OutOfBlocks when the pool is
    exhausted (the manager is then unchanged) and PkvError for other failures."""

    def __init__(self, num_blocks, block_size=BLOCK_SIZE, free_order=None):
        import numpy as np
        self._np = np
        h = ctypes.c_void_p()
        order = None
        if free_order is not None:
            order = np.ascontiguousarray(free_order, dtype=np.int32)
            if order.shape != (num_blocks,):
                raise ValueError("free_order must have num_blocks entries")
        _check(lib().pkv_bm_create(num_blocks, block_size,
                                   order.ctypes.data if order is not None else None,
                                   ctypes.byref(h)))
        self._h = h
        self.num_blocks = num_blocks
        self.block_size = block_size

    def close(self):
        if getattr(self, "_h", None):
            lib().pkv_bm_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def add_seq(self, seq, num_tokens):
        _check(lib().pkv_bm_add_seq(self._h, seq, num_tokens))

    def append_slot(self, seq):
        slot = ctypes.c_int64()
        src, dst = ctypes.c_int32(), ctypes.c_int32()
        _check(lib().pkv_bm_append_slot(self._h, seq, ctypes.byref(slot), ctypes.byref(src),
                                        ctypes.byref(dst)))
        return slot.value, ((src.value, dst.value) if src.value >= 0 else None)

    def append_slots(self, seqs):
        """One slot for each sequence, in order, all or nothing.
        Returns (slots int64 [n], cow_pairs int32 [k, 2]) as numpy arrays."""
        np = self._np
        s = np.ascontiguousarray(seqs, dtype=np.int64)
        n = s.shape[0]
        slots = np.empty(n, np.int64)
        pairs = np.empty((max(n, 1), 2), np.int32)
        k = ctypes.c_int32()
        _check(lib().pkv_bm_append_slots(self._h, s.ctypes.data, n, slots.ctypes.data,
                                         pairs.ctypes.data, ctypes.byref(k)))
        return slots, pairs[:k.value].copy()

    def fork(self, parent, child):
        _check(lib().pkv_bm_fork(self._h, parent, child))

    def free_seq(self, seq):
        _check(lib().pkv_bm_free_seq(self._h, seq))

    def block_table(self, seq):
        np = self._np
        n = ctypes.c_int32()
        rc = lib().pkv_bm_block_table(self._h, seq, None, 0, ctypes.byref(n))
        if rc not in (0, 1):       # 1 = capacity too small: *n still holds the length
            _check(rc)
        out = np.empty(max(n.value, 1), np.int32)
        _check(lib().pkv_bm_block_table(self._h, seq, out.ctypes.data, n.value,
                                        ctypes.byref(n)))
        return out[:n.value].tolist()

    def block_tables(self, seqs, max_blocks):
        """Pack tables [n, max_blocks] (-1 padded) and lengths [n] for a batch."""
        np = self._np
        s = np.ascontiguousarray(seqs, dtype=np.int64)
        out = np.empty((s.shape[0], max_blocks), np.int32)
        lens = np.empty(s.shape[0], np.int32)
        _check(lib().pkv_bm_block_tables(self._h, s.ctypes.data, s.shape[0], max_blocks,
                                         out.ctypes.data, lens.ctypes.data))
        return out, lens

    def seq_len(self, seq):
        n = ctypes.c_int32()
        _check(lib().pkv_bm_seq_len(self._h, seq, ctypes.byref(n)))
        return n.value

    def refcount(self, block):
        n = ctypes.c_int32()
        _check(lib().pkv_bm_refcount(self._h, block, ctypes.byref(n)))
        return n.value

    def num_free(self):
        return lib().pkv_bm_num_free(self._h)

    def num_seqs(self):
        return lib().pkv_bm_num_seqs(self._h)

    def free_order(self):
        np = self._np
        n = lib().pkv_bm_free_list(self._h, None, 0)
        out = np.empty(max(n, 1), np.int32)
        lib().pkv_bm_free_list(self._h, out.ctypes.data, n)
        return out[:n].tolist()

    # -- host (swap) pool ------------------------------------------------------------------
    def set_host_pool(self, num_host_blocks, free_order=None):
        np = self._np
        order = None
        if free_order is not None:
            order = np.ascontiguousarray(free_order, dtype=np.int32)
        _check(lib().pkv_bm_set_host_pool(self._h, num_host_blocks,
                                          order.ctypes.data if order is not None else None))

    def _swap(self, fn, seq):
        np = self._np
        n = ctypes.c_int32()
        cap = max(1, len(self.block_table(seq)))
        out = np.empty((cap, 2), np.int32)
        _check(fn(self._h, seq, out.ctypes.data, cap, ctypes.byref(n)))
        return out[:n.value].copy()

    def swap_out(self, seq):
        """Evict ``seq`` to host blocks; returns int32 [n, 2] (device block, host block)."""
        return self._swap(lib().pkv_bm_swap_out, seq)

    def swap_in(self, seq):
        """Bring ``seq`` back; returns int32 [n, 2] (host block, device block)."""
        return self._swap(lib().pkv_bm_swap_in, seq)

    def is_swapped(self, seq):
        v = ctypes.c_int32()
        _check(lib().pkv_bm_is_swapped(self._h, seq, ctypes.byref(v)))
        return bool(v.value)

    def num_host_free(self):
        return lib().pkv_bm_num_host_free(self._h)
