"""Seeded synthetic inputs for the paged decode path.

This module only draws random numbers and lays out block tables; it holds none of the
method's arithmetic.  The same arrays feed the CUDA library and the fp64 oracle.

Shapes follow the workloads the source pages and their experiment platform suggest (OPT-13B
fp16 decode with 16-token blocks, "vLLM and PagedAttention: How Ideas from Operating Systems
Accelerated LLM Inference"), plus a grouped-query and a long-context case:

  tiny      4 seqs, lens {5,17,33,48}, 2 heads MHA, D 64, fp32, 16-block pool, seed 0
  opt13b    64 seqs, 40 heads MHA, D 128, fp16, lens lognormal(ln 512, 1) clipped 16..2048,
            pool 1.1x the need, shuffled placement, seed 1
  gqa       128 seqs, 32 q / 8 kv heads, D 128, bf16, lens uniform 256..4096, seed 2
  fork      16 prompts x 8 samples sharing 1025 prefilled tokens, 32 decode steps, fp16,
            32 heads MHA, D 128, seed 3 (block tables come from the block manager)
  long      8 seqs x 32768 tokens, 32 q / 8 kv heads, D 128, bf16, 512-token partitions, seed 4

Context lengths are post-write: the decode step writes the new token at position len-1 and
attention covers all len tokens.  Block tables are padded with -1 past each sequence's last
block; the free order is a seeded permutation of the pool.
"""
from dataclasses import dataclass, field
import math

import numpy as np

BLOCK_SIZE = 16


@dataclass
class Workload:
    name: str
    num_seqs: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    dtype: str                      # "f32" | "f16" | "bf16"
    context_lens: np.ndarray        # int32 [S]
    block_tables: np.ndarray        # int32 [S, maxB], -1 padded
    num_blocks: int
    free_order: np.ndarray          # int32 [NB] placement permutation
    slot_mapping: np.ndarray        # int64 [S]: slot of position len-1
    scale: float
    seed: int
    partition_tokens: int = 0       # 0 = library's choice
    q_std: float = 1.0
    kv_std: float = 0.5
    block_size: int = BLOCK_SIZE
    extra: dict = field(default_factory=dict)

    @property
    def max_blocks_per_seq(self):
        return self.block_tables.shape[1]

    @property
    def elem_size(self):
        return 4 if self.dtype == "f32" else 2

    def kv_bytes(self):
        """K and V bytes the decode reads: every cached token once per KV head."""
        return int(self.context_lens.astype(np.int64).sum()) * self.num_kv_heads * \
            self.head_dim * self.elem_size * 2


def _tables(lens, num_blocks, rng, block_size=BLOCK_SIZE, max_blocks=None):
    """Place each sequence's blocks in the order of a seeded permutation of the pool."""
    lens = np.asarray(lens, np.int64)
    nblk = (lens + block_size - 1) // block_size
    need = int(nblk.sum())
    if need > num_blocks:
        raise ValueError("pool too small")
    order = rng.permutation(num_blocks).astype(np.int32)
    maxB = int(max_blocks if max_blocks is not None else max(1, int(nblk.max(initial=1))))
    bt = np.full((len(lens), maxB), -1, np.int32)
    off = 0
    for s, n in enumerate(nblk):
        bt[s, :n] = order[off:off + n]
        off += n
    return bt, order


def _slots(lens, bt, block_size=BLOCK_SIZE):
    pos = np.asarray(lens, np.int64) - 1
    blk = bt[np.arange(len(lens)), pos // block_size].astype(np.int64)
    return blk * block_size + pos % block_size


def make_workload(name, lens, num_q_heads, num_kv_heads, head_dim, dtype, seed,
                  pool_factor=1.1, num_blocks=None, partition_tokens=0, q_std=1.0,
                  kv_std=0.5, rng=None, max_blocks=None, block_size=BLOCK_SIZE):
    rng = rng if rng is not None else np.random.Generator(np.random.PCG64(seed))
    lens = np.asarray(lens, np.int32)
    need = int(((lens.astype(np.int64) + block_size - 1) // block_size).sum())
    if num_blocks is None:
        num_blocks = max(1, int(math.ceil(pool_factor * need)))
    bt, order = _tables(lens, num_blocks, rng, block_size=block_size, max_blocks=max_blocks)
    return Workload(name=name, num_seqs=len(lens), num_q_heads=num_q_heads,
                    num_kv_heads=num_kv_heads, head_dim=head_dim, dtype=dtype,
                    context_lens=lens, block_tables=bt, num_blocks=num_blocks,
                    free_order=order, slot_mapping=_slots(lens, bt, block_size),
                    scale=1.0 / math.sqrt(head_dim), seed=seed,
                    partition_tokens=partition_tokens, q_std=q_std, kv_std=kv_std,
                    block_size=block_size)


def tiny():
    return make_workload("tiny", [5, 17, 33, 48], 2, 2, 64, "f32", seed=0, num_blocks=16,
                         kv_std=1.0)


def opt13b(num_seqs=64, seed=1, block_size=BLOCK_SIZE):
    rng = np.random.Generator(np.random.PCG64(seed))
    lens = np.clip(np.rint(rng.lognormal(math.log(512.0), 1.0, num_seqs)), 16, 2048)
    return make_workload("opt13b", lens.astype(np.int32), 40, 40, 128, "f16", seed, rng=rng,
                         block_size=block_size)


def gqa(num_seqs=128, seed=2, block_size=BLOCK_SIZE):
    rng = np.random.Generator(np.random.PCG64(seed))
    lens = rng.integers(256, 4096, size=num_seqs, endpoint=True)
    return make_workload("gqa", lens.astype(np.int32), 32, 8, 128, "bf16", seed, rng=rng,
                         block_size=block_size)


def long_context(num_seqs=8, seq_len=32768, seed=4, block_size=BLOCK_SIZE):
    return make_workload("long", [seq_len] * num_seqs, 32, 8, 128, "bf16", seed,
                         partition_tokens=512, block_size=block_size)


# fork / parallel-sampling workload parameters (block tables come from a block manager)
FORK = dict(num_prompts=16, samples=8, prompt_tokens=1024, shared_generated=1, steps=32,
            num_heads=32, head_dim=128, dtype="f16", seed=3)


def fork_pool_blocks(num_prompts=16, samples=8, prompt_tokens=1024, shared_generated=1,
                     steps=32, factor=1.1):
    """Pool size for the fork workload: the blocks all samples hold at the end, x factor."""
    shared = -(-(prompt_tokens + shared_generated) // BLOCK_SIZE)
    final = prompt_tokens + shared_generated + steps
    per_sample = -(-final // BLOCK_SIZE)
    # the last shared block is partly full: each sample but one copies it once
    private = per_sample - shared + 1
    need = num_prompts * (shared + (samples - 1) * private + (private - 1))
    return int(math.ceil(factor * need))


CONFIGS = {"tiny": tiny, "opt13b": opt13b, "gqa": gqa, "long": long_context}


# ---- values -----------------------------------------------------------------------------
def _torch_dtype(torch, name):
    return {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}[name]


def randn(torch, shape, dtype, std, seed, device):
    """N(0, std^2) values of ``dtype`` (rounded to nearest even from fp32), from a seeded
    generator: numpy PCG64 on the host, torch's Philox generator on a GPU."""
    td = _torch_dtype(torch, dtype)
    if str(device) == "cpu":
        g = np.random.Generator(np.random.PCG64(seed))
        a = g.standard_normal(size=shape, dtype=np.float32)
        if std != 1.0:
            a *= np.float32(std)
        return torch.from_numpy(a).to(td)
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    t = torch.empty(shape, dtype=torch.float32, device=device)
    t.normal_(0.0, 1.0, generator=gen)
    if std != 1.0:
        t.mul_(std)
    return t.to(td)


def make_values(wl, device="cpu", torch=None):
    """q [S,Hq,D], k_pool/v_pool [NB,Hkv,B,D], k_new/v_new [S,Hkv,D] as torch tensors."""
    if torch is None:
        import torch  # noqa: F811
    S, Hq, Hkv, D, NB = wl.num_seqs, wl.num_q_heads, wl.num_kv_heads, wl.head_dim, \
        wl.num_blocks
    base = wl.seed * 1000003
    return {
        "q": randn(torch, (S, Hq, D), wl.dtype, wl.q_std, base + 1, device),
        "k_pool": randn(torch, (NB, Hkv, wl.block_size, D), wl.dtype, wl.kv_std, base + 2,
                        device),
        "v_pool": randn(torch, (NB, Hkv, wl.block_size, D), wl.dtype, wl.kv_std, base + 3,
                        device),
        "k_new": randn(torch, (S, Hkv, D), wl.dtype, wl.kv_std, base + 4, device),
        "v_new": randn(torch, (S, Hkv, D), wl.dtype, wl.kv_std, base + 5, device),
    }


def to_numpy_bits(t):
    """Host numpy view of a torch tensor: float32 stays float32, 16-bit types become their
    raw uint16 bit patterns."""
    import torch
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.float32:
        return t.numpy()
    return t.view(torch.int16).numpy().view(np.uint16)


def fp8_scales(wl, which):
    """Per-kv-head scales for the FP8 cache: about 4.5 standard deviations map to the
    largest E4M3 code (448), slightly different per head."""
    h = np.arange(wl.num_kv_heads, dtype=np.float32)
    base = np.float32(wl.kv_std * 4.5 / 448.0) * (np.float32(1.0) + np.float32(0.05) * h)
    return base * (np.float32(1.0) if which == "k" else np.float32(1.1))


def make_values_fp8(wl, device="cpu", torch=None):
    """Inputs for an FP8 KV cache: q and new K/V as for ``make_values`` (in wl.dtype); the
    pools as random E4M3 codes of N(0, kv_std^2) values at the per-head scales,
    K [NB, Hkv, B, D] and V [NB, Hkv, D, 16] (16-token blocks) or [NB, Hkv, B/16, D, 16];
    scales as fp32 tensors."""
    if torch is None:
        import torch  # noqa: F811
    vals = make_values(wl, device, torch)
    NB, Hkv, D = wl.num_blocks, wl.num_kv_heads, wl.head_dim
    base = wl.seed * 1000003
    ks = torch.from_numpy(fp8_scales(wl, "k")).to(device)
    vs = torch.from_numpy(fp8_scales(wl, "v")).to(device)

    def codes(shape, scale, seed, head_axis):
        x = randn(torch, shape, "f32", wl.kv_std, seed, device)
        view = [1] * len(shape)
        view[head_axis] = -1
        x = (x / scale.view(view)).clamp(-448.0, 448.0)
        return x.to(torch.float8_e4m3fn).view(torch.uint8).contiguous()

    vals["k_pool"] = codes((NB, Hkv, wl.block_size, D), ks, base + 6, 1)
    # V: each 16-token half of a block transposed ([NB, Hkv, D, 16] for 16-token blocks)
    vshape = (NB, Hkv, D, 16) if wl.block_size == 16 else (NB, Hkv, wl.block_size // 16, D, 16)
    vals["v_pool"] = codes(vshape, vs, base + 7, 1)
    vals["k_scale"] = ks
    vals["v_scale"] = vs
    return vals
