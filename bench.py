"""Benchmark of the paged decode path: KV GB/s, sequences/s and fraction of HBM roofline.

One step = one pass of the whole hot path over one batch: copy-on-write block copies (when the
workload forks or shares blocks), kv_write of each sequence's new token, and paged decode
attention (with the split / log-sum-exp reduce for sequences longer than one partition).  By
default the write runs inside the decode kernel (kv_write_and_decode); --separate-write times
the two calls.

    python bench.py [--gpus N] [--steps K] [--warmup W]
                    [--workload opt13b|gqa|long|fork|beam|prefix|tiny] [--kv-fp8]
                    [--impl pkv|reference] [--no-cpu-baseline] [--separate-write]
                    [--l2-flush] [--swap-probe] [--no-read-probe] [--contiguous]
                    [--layout paged|contiguous] [--decode-only] [--lib-defines '-D...']

N > 1 runs under torchrun, one process per GPU; every rank decodes its own replica of the
batch (weak scaling, no data-path collective); time is the max over ranks.  Rank 0 prints
one JSON line.  ``--impl reference`` times the fp64 CPU oracle on a bounded sample of the
same workload on the host cores.
"""
import argparse
import datetime
import gc
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "paged decode attention KV GB/s & seqs/s, % of B200 HBM roofline"
# Buffer sets of the pipelined end-to-end run (the host runs up to E2E_BUFS - 1 steps ahead)
E2E_BUFS = 3
FALLBACK_HBM_GBS = 6650.0
L2_BYTES = 126 * 1000 * 1000     # B200 L2 (126 MB)

WORKLOAD_TEXT = {
    "tiny": "tiny decode step: 4 seqs, context {5,17,33,48}, 2 heads MHA, head_dim 64, fp32, "
            "block 16, 16-block pool, kv_write of one token per sequence",
    "opt13b": "OPT-13B-shaped decode: 64 seqs, 40 heads MHA, head_dim 128, fp16 KV, block 16, "
              "context lognormal(median 512, sigma 1) clipped 16..2048, shuffled placement, "
              "pool 1.1x need, kv_write of one token per sequence",
    "gqa": "GQA decode (Llama-3-8B-like): 128 seqs, 32 q / 8 kv heads, head_dim 128, bf16 KV, "
           "block 16, context uniform 256..4096, shuffled placement, kv_write of one token per "
           "sequence",
    "long": "long-context split decode: 8 seqs x 32768 tokens, 32 q / 8 kv heads, head_dim 128, "
            "bf16 KV, block 16, fully shuffled blocks, 512-token partitions + LSE reduce",
    "beam": "beam search: 16 requests x width 4, 500-token prompts, 64 generated tokens with "
            "seeded parent selection each step (forks, frees, copy-on-write), then one decode "
            "step over the 64 beams; fp16, 40 heads MHA, head_dim 128, block 16",
    "prefix": "shared system prompt: 64 requests forked from one 1000-token prefix, each "
              "appending its own 64..512-token prompt, then one decode step; bf16, 32 q / 8 "
              "kv heads, head_dim 128, block 16",
    "fork": "parallel-sampling fork: 16 prompts x 8 samples sharing 1025 prefilled tokens, first "
            "decode step (112 copy-on-write block copies, 128 kv_writes, decode over 1026 "
            "tokens), fp16, 32 heads MHA, head_dim 128, block 16",
}


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="opt13b", choices=sorted(WORKLOAD_TEXT))
    ap.add_argument("--impl", default="pkv", choices=["pkv", "reference"])
    ap.add_argument("--partition-tokens", type=int, default=None)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-read-probe", action="store_true",
                    help="skip the read-bandwidth probe (the library's streaming copy of a "
                         "4 GiB buffer in the decode's chunk size) reported beside the peak")
    ap.add_argument("--kv-fp8", action="store_true",
                    help="FP8 (E4M3) KV cache: kv_write_fp8 + paged_attn_decode_fp8 "
                         "(opt13b, gqa, long)")
    ap.add_argument("--swap-probe", action="store_true",
                    help="also time swapping the batch's blocks to pinned host memory and "
                         "back (kv_swap_out / kv_swap_in over PCIe)")
    ap.add_argument("--contiguous", action="store_true",
                    help="place each sequence's blocks contiguously and in order (paged "
                         "kernel over a contiguous layout) instead of shuffled")
    ap.add_argument("--layout", default="paged", choices=["paged", "contiguous"],
                    help="contiguous: time attn_decode_contiguous over a [S][H_kv][Lmax][D] "
                         "cache with no block table (the same tokens, gathered from the "
                         "pools), decode only; compare with --decode-only on the paged pools")
    ap.add_argument("--block-size", type=int, default=16, choices=[16, 32],
                    help="tokens per physical KV block (opt13b, gqa, long); the configs "
                         "use 16")
    ap.add_argument("--decode-only", action="store_true",
                    help="the step is the decode call alone (no kv_write)")
    ap.add_argument("--separate-write", action="store_true",
                    help="the newest token's write as its own kernel (kv_write / "
                         "kv_write_fp8) before the decode, instead of the fused call")
    ap.add_argument("--decode-events-every", type=int, default=10,
                    help="bracket every E-th decode call of the timed graph with CUDA events "
                         "(the roofline's decode duration); the others run without them, "
                         "since each event node costs about 1 %% of a step")
    ap.add_argument("--l2-flush", action="store_true",
                    help="write a 256 MiB buffer before every step, outside the timed work "
                         "(step and decode calls are then event-bracketed); on by default "
                         "for workloads whose unique KV bytes fit twice in L2")
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="target CPU time of the oracle baseline sample")
    ap.add_argument("--lib-defines", default="",
                    help="time a variant build of the library compiled with these macros "
                         "(space-separated, e.g. '-DPKV_DECODE_FORCE_SIMT' for the "
                         "CUDA-core decode at every dtype); the line names the variant")
    return ap.parse_args(argv)


# ---- workload construction ---------------------------------------------------------------
def _new_bm(model_block_manager, NB, rng):
    if model_block_manager:
        from oracle.block_manager import BlockManagerModel
        return _ModelAdapter(BlockManagerModel(NB, free_order=rng.permutation(NB)))
    from paged_kv_cache_392_b200 import binding as B
    return B.BlockManager(NB, free_order=rng.permutation(NB))


def _beam_search(bm, rng, n_req=16, width=4, prompt=500, steps=64):
    """Each step every beam appends one token, then each request keeps `width` survivors
    drawn (with replacement) from its beams; survivors are forks, the old beams are freed."""
    beams, nxt = [], 0
    for r in range(n_req):
        bm.add_seq(nxt, prompt)
        group = [nxt]
        nxt += 1
        for _ in range(1, width):
            bm.fork(group[0], nxt)
            group.append(nxt)
            nxt += 1
        beams.append(group)
    copies = 0
    for _ in range(steps):
        _, pairs = bm.append_slots([b for g in beams for b in g])
        copies += len(pairs)
        for r in range(n_req):
            parents = rng.integers(0, width, size=width)
            new = []
            for pi in parents:
                bm.fork(beams[r][int(pi)], nxt)
                new.append(nxt)
                nxt += 1
            for b in beams[r]:
                bm.free_seq(b)
            beams[r] = new
    return [b for g in beams for b in g], copies


def _shared_prefix(bm, rng, n_req=64, prefix=1000, lo=64, hi=512):
    """Requests forked from one cached prefix sequence, each appending its own prompt."""
    tmpl = 1 << 40
    bm.add_seq(tmpl, prefix)
    reqs = list(range(n_req))
    for r in reqs:
        bm.fork(tmpl, r)
    user = rng.integers(lo, hi, size=n_req, endpoint=True)
    copies = 0
    for t in range(int(user.max())):
        active = [r for r in reqs if user[r] > t]
        _, pairs = bm.append_slots(active)
        copies += len(pairs)
    return reqs, copies


def _sharing_workload(name, model_block_manager):
    from paged_kv_cache_392_b200 import workloads as W
    if name == "beam":
        Hq = Hkv = 40
        dtype, seed = "f16", 5
        NB = 2600
    else:
        Hq, Hkv = 32, 8
        dtype, seed = "bf16", 6
        NB = 6400
    rng = np.random.default_rng(seed)
    bm = _new_bm(model_block_manager, NB, rng)
    if name == "beam":
        seqs, copies = _beam_search(bm, rng)
    else:
        seqs, copies = _shared_prefix(bm, rng)
    slots, pairs = bm.append_slots(seqs)          # the decode step's own new token
    bt, lens = bm.block_tables(seqs, 256)
    maxB = int((bt >= 0).sum(axis=1).max())
    bt = np.ascontiguousarray(bt[:, :maxB])
    in_use = NB - bm.num_free()
    private = int(((lens.astype(np.int64) + 15) // 16).sum())
    wl = W.Workload(name=name, num_seqs=len(seqs), num_q_heads=Hq, num_kv_heads=Hkv,
                    head_dim=128, dtype=dtype, context_lens=lens, block_tables=bt,
                    num_blocks=NB, free_order=np.asarray(bm.free_order(), np.int32),
                    slot_mapping=np.asarray(slots, np.int64), scale=1.0 / math.sqrt(128),
                    seed=seed)
    wl.extra["unique_blocks"] = in_use
    wl.extra["sharing"] = {"blocks_in_use": in_use, "blocks_without_sharing": private,
                           "saving": round(1.0 - in_use / private, 4),
                           "copy_on_write_copies_before_step": copies}
    bm.close()
    return wl, np.asarray(pairs, np.int32).reshape(-1, 2)


def build_workload(name, model_block_manager=False, block_size=16):
    """Return (Workload, cow_pairs int32 [P, 2]).  The fork workload's tables come from a
    block manager: the product's C++ one, or the oracle's Python model for the CPU arm."""
    from paged_kv_cache_392_b200 import workloads as W
    if block_size != 16 and name not in ("opt13b", "gqa", "long"):
        raise SystemExit("--block-size 32 applies to the opt13b, gqa and long workloads")
    if name in ("beam", "prefix"):
        return _sharing_workload(name, model_block_manager)
    if name != "fork":
        if block_size != 16:
            return W.CONFIGS[name](block_size=block_size), np.zeros((0, 2), np.int32)
        return W.CONFIGS[name](), np.zeros((0, 2), np.int32)
    f = W.FORK
    NB = W.fork_pool_blocks()
    rng = np.random.default_rng(f["seed"])
    if model_block_manager:
        from oracle.block_manager import BlockManagerModel
        bm = _ModelAdapter(BlockManagerModel(NB, free_order=rng.permutation(NB)))
    else:
        from paged_kv_cache_392_b200 import binding as B
        bm = B.BlockManager(NB, free_order=rng.permutation(NB))
    seqs = []
    prompt = f["prompt_tokens"] + f["shared_generated"]
    for p in range(f["num_prompts"]):
        bm.add_seq(p * f["samples"], prompt)
        for k in range(1, f["samples"]):
            bm.fork(p * f["samples"], p * f["samples"] + k)
        seqs += [p * f["samples"] + k for k in range(f["samples"])]
    slots, pairs = bm.append_slots(seqs)
    maxB = -(-(prompt + f["steps"]) // 16)
    bt, lens = bm.block_tables(seqs, maxB)
    wl = W.Workload(name="fork", num_seqs=len(seqs), num_q_heads=f["num_heads"],
                    num_kv_heads=f["num_heads"], head_dim=f["head_dim"], dtype=f["dtype"],
                    context_lens=lens, block_tables=bt, num_blocks=NB,
                    free_order=np.asarray(bm.free_order(), np.int32), slot_mapping=slots,
                    scale=1.0 / math.sqrt(f["head_dim"]), seed=f["seed"])
    wl.extra["unique_blocks"] = NB - bm.num_free()
    bm.close()
    return wl, pairs


class _ModelAdapter:
    """The oracle block-manager model behind the product manager's batch interface."""

    def __init__(self, model):
        self.m = model

    def add_seq(self, s, n):
        self.m.add_seq(s, n)

    def fork(self, p, c):
        self.m.fork(p, c)

    def free_seq(self, s):
        self.m.free_seq(s)

    def append_slots(self, seqs):
        slots, pairs = self.m.append_slots(seqs)
        return np.asarray(slots, np.int64), np.asarray(pairs, np.int32).reshape(-1, 2)

    def block_tables(self, seqs, maxB):
        bt = np.full((len(seqs), maxB), -1, np.int32)
        for i, s in enumerate(seqs):
            t = self.m.block_table(s)
            bt[i, :len(t)] = t
        return bt, np.array([self.m.seq_len(s) for s in seqs], np.int32)

    def num_free(self):
        return self.m.num_free()

    def free_order(self):
        return self.m.free_order()

    def close(self):
        pass


def contiguous_placement(wl):
    """Re-place every sequence's blocks back to back in pool order (block j of sequence s at
    pool block off_s + j): the layout a contiguous cache would have, read through the same
    block tables by the same kernel."""
    Bs = wl.block_size
    nblk = (wl.context_lens.astype(np.int64) + Bs - 1) // Bs
    bt = np.full_like(wl.block_tables, -1)
    off = 0
    for s_, n in enumerate(nblk):
        bt[s_, :n] = np.arange(off, off + n, dtype=np.int32)
        off += n
    wl.block_tables = bt
    pos = wl.context_lens.astype(np.int64) - 1
    wl.slot_mapping = bt[np.arange(wl.num_seqs), pos // Bs].astype(np.int64) * Bs + pos % Bs
    wl.extra["placement"] = "contiguous"


def algorithmic_bytes(wl, pairs, split_rows=0, kv_es=None):
    """Bytes one step must move, counted from the definition of each kernel's work.
    kv_es: bytes per cached K/V element (default the workload dtype's; 1 for FP8)."""
    es = wl.elem_size
    kv_es = kv_es or es
    S, Hq, Hkv, D = wl.num_seqs, wl.num_q_heads, wl.num_kv_heads, wl.head_dim
    kv = int(wl.context_lens.astype(np.int64).sum()) * Hkv * D * kv_es * 2  # K and V once
    qo = S * Hq * D * es * 2                              # q read + out written
    Bs = wl.block_size
    tables = int(((wl.context_lens + Bs - 1) // Bs).sum()) * 4 + S * 4
    ws = 0
    if split_rows:                                        # partials written + read
        ws = split_rows * (D + 2) * 4 * 2
    write = S * Hkv * D * (es + kv_es) * 2 + S * 8        # kv_write: read new + write pool
    copy = len(pairs) * Hkv * Bs * D * kv_es * 2 * 2      # each pair: read + write K and V
    return {"kv": kv, "decode": kv + qo + tables + ws, "kv_write": write, "kv_copy": copy,
            "step": kv + qo + tables + ws + write + copy}


def split_rows(wl, partition_tokens):
    """(query-head rows, partitions) of sequences that span more than one partition."""
    pt = partition_tokens or 512
    nparts = -(-wl.context_lens.astype(np.int64) // pt)
    multi = nparts[nparts > 1]
    return int(multi.sum()) * wl.num_q_heads, int(nparts.max())


def kv_utilisation(wl):
    """Fraction of the allocated KV slots that hold a token, from the block tables: every
    distinct physical block counts 16 slots once, filled as far as the furthest sequence that
    maps it has written.  Without sharing this is sum(L) / (B * sum(ceil(L / B))); the
    only waste is each sequence's partly filled last block."""
    Bs = getattr(wl, "block_size", 16)
    fill = {}
    for s_, L in enumerate(wl.context_lens.astype(np.int64)):
        nb = -(-int(L) // Bs)
        for j in range(nb):
            b = int(wl.block_tables[s_, j])
            fill[b] = max(fill.get(b, 0), min(Bs, int(L) - Bs * j))
    slots = Bs * len(fill)
    return {"tokens_in_blocks": int(sum(fill.values())), "slots_allocated": slots,
            "frac": round(sum(fill.values()) / slots, 4) if slots else None,
            "pages_figure": "about 96 % with 16-token blocks (vs 20-38 % for contiguous "
                            "reservation), OPT-13B on a 40 GB A100"}


def uses_l2_flush(args, wl, nbytes, fp8):
    """Flush L2 between steps when the bytes a step really reads (shared blocks once) would
    fit in it twice over; otherwise the working set itself keeps L2 from carrying over."""
    uniq_kv = (wl.extra["unique_blocks"] * wl.num_kv_heads * wl.block_size * wl.head_dim *
               (1 if fp8 else wl.elem_size) * 2 if "unique_blocks" in wl.extra
               else nbytes["kv"])
    return bool(args.l2_flush or uniq_kv < 2 * L2_BYTES)


def step_config(args, wl, npairs, pt_run, nbytes, flush, fp8):
    """The line's ``config``: the workload and how a step runs (both arms print the same)."""
    decode_only = args.decode_only or args.layout == "contiguous"
    fused = not args.separate_write and not decode_only
    cfg = {
        "workload": WORKLOAD_TEXT[args.workload],
        "name": args.workload,
        "num_seqs": wl.num_seqs, "num_q_heads": wl.num_q_heads,
        "num_kv_heads": wl.num_kv_heads, "head_dim": wl.head_dim,
        "block_size": wl.block_size, "kv_dtype": "fp8-e4m3" if fp8 else wl.dtype,
        "context_tokens": int(wl.context_lens.sum()),
        "partition_tokens": pt_run, "cow_pairs_per_step": npairs,
        "kv_bytes_per_step": nbytes["kv"], "step_bytes": nbytes["step"],
        "l2": ("flushed: 256 MiB written before every step, outside the timed "
               "work (step and decode calls event-bracketed)" if flush
               else "no flush: KV working set %.2f GB per step > 126 MB L2" %
               (nbytes["kv"] / 1e9)),
        "parallelism": "replicas x%d" % int(os.environ.get("WORLD_SIZE", "1")),
        "placement": wl.extra.get("placement", "shuffled"),
        "kv_write": ("none: the step is the decode call alone" if decode_only else
                     "fused into the decode kernel" if fused else
                     "separate %s kernel" % ("kv_write_fp8" if fp8 else "kv_write")),
    }
    if args.layout == "contiguous":
        cfg["layout"] = ("contiguous [S][H_kv][Lmax][D] cache, Lmax = %d, no block table"
                         % (wl.max_blocks_per_seq * wl.block_size))
    return cfg


# ---- environment: peaks, clocks, profile traffic ----------------------------------------
def hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            v = float(json.load(f)["hbm_gbs"])
        return v, "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


DECODE_SOURCES = ("attn_decode.cuh", "attn_decode_tc.cuh", "ptx.cuh", "faults.cuh")
DECODE_FP8_SOURCES = DECODE_SOURCES + ("attn_decode_fp8.cuh", "pkv_cuda.cu")


def _code_only(text):
    """Source text without comments, trailing spaces and blank lines: what the compiler sees
    of it (the kernel sources hold no comment markers inside string literals)."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return "\n".join(ln.rstrip() for ln in text.splitlines() if ln.strip())


def _launcher_fp8_section(text):
    """The FP8 part of the launcher file: from its section banner to the next banner."""
    a = text.index("// ---- FP8 (E4M3) KV cache")
    j = text.find("\n// ---- ", a + 1)
    return text[a:j + 1] if j >= 0 else text[a:]


def kernel_source_sha(fp8=False):
    """Hash of the decode kernels' code (kernels and their launch shape; comments left out);
    the FP8 kernel's launch constants live in the launcher's FP8 section, so its hash covers
    that section too."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "paged_kv_cache_392_b200", "csrc")
    for name in (DECODE_FP8_SOURCES if fp8 else DECODE_SOURCES):
        with open(os.path.join(csrc, name)) as f:
            text = f.read()
        if name == "pkv_cuda.cu":
            text = _launcher_fp8_section(text)
        h.update(name.encode() + b"\0" + _code_only(text).encode())
    return h.hexdigest()[:16]


def profile_traffic(workload, fp8=False):
    """DRAM bytes per decode launch from the committed ncu summary for this workload, or
    None when there is none or it was taken on different kernel sources."""
    path = os.path.join(ROOT, "profiles", "paged_attn_decode_%s%s.md"
                        % ("fp8_" if fp8 else "", workload))
    try:
        text = open(path).read()
    except OSError:
        return None
    m = re.search(r"dram_bytes_per_launch:\s*([0-9.eE+]+)", text)
    sha = re.search(r"kernel_source_sha:\s*([0-9a-f]+)", text)
    if not m or not sha or sha.group(1) != kernel_source_sha(fp8):
        return None
    return float(m.group(1))


class ClockSampler:
    """nvidia-smi clock / throttle sampling in the background (every 100 ms)."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index      # nvidia-smi -i argument (GPU UUID or index)
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        self.t0 = time.time()

    def stop(self):
        if not self.proc:
            return
        time.sleep(0.25)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---- distributed plumbing -----------------------------------------------------------------
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(world, backend="nccl"):
    if world <= 1:
        return None
    import torch.distributed as dist
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return dist


def max_over_ranks(dist, value, device):
    """Max of a float over all ranks (identity with one rank)."""
    if dist is None:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(dist, device):
    if dist is not None:
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def swap_probe(torch, B, wl, kp, vp, device, reps=5):
    """Swap every block of the batch out to pinned host memory and back in, timed with CUDA
    events; returns GB/s each way (block bytes of K and V / time)."""
    used = np.unique(wl.block_tables[wl.block_tables >= 0]).astype(np.int32)
    n = len(used)
    hk = torch.empty((n,) + tuple(kp.shape[1:]), dtype=kp.dtype).pin_memory()
    hv = torch.empty_like(hk).pin_memory()
    out_pairs = torch.from_numpy(np.stack([used, np.arange(n, dtype=np.int32)], 1)).to(device)
    in_pairs = torch.from_numpy(np.stack([np.arange(n, dtype=np.int32), used], 1)).to(device)
    nbytes = 2 * n * kp[0].numel() * kp.element_size()
    res = {}
    for name, call in (("out", lambda: B.kv_swap_out(out_pairs, kp, vp, hk, hv)),
                       ("in", lambda: B.kv_swap_in(in_pairs, hk, hv, kp, vp))):
        call()
        torch.cuda.synchronize()
        best = 0.0
        for _ in range(reps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            call()
            b.record()
            torch.cuda.synchronize()
            best = max(best, nbytes / (a.elapsed_time(b) * 1e-3) / 1e9)
        res[name + "_gbs"] = round(best, 2)
    res["bytes"] = nbytes
    res["blocks"] = n
    return res


def time_block_manager(B, wl, steps=200):
    """Host cost of one decode step's block-manager work for this batch: append one slot to
    every sequence (on-demand block allocation, copy-on-write decisions) and export the
    padded block tables, through the C ABI from Python (the binding's marshalling included).
    The sequences start one token short of the workload's lengths and grow by one a step."""
    import time
    S = wl.num_seqs
    lens = [int(x) for x in wl.context_lens]
    grow = (steps + wl.block_size - 1) // wl.block_size + 1
    nb = int(sum((L + wl.block_size - 1) // wl.block_size + grow for L in lens))
    bm = B.BlockManager(nb, block_size=wl.block_size)
    try:
        for i, L in enumerate(lens):
            bm.add_seq(i, L - 1)
        seqs = list(range(S))
        maxb = max((L + steps + wl.block_size - 1) // wl.block_size for L in lens)
        t_app = t_tab = 0.0
        for _ in range(steps):
            t0 = time.perf_counter()
            bm.append_slots(seqs)
            t1 = time.perf_counter()
            bm.block_tables(seqs, maxb)
            t2 = time.perf_counter()
            t_app += t1 - t0
            t_tab += t2 - t1
    finally:
        bm.close()
    return {"append_slots_us": round(t_app / steps * 1e6, 2),
            "block_tables_us": round(t_tab / steps * 1e6, 2), "seqs": S, "steps": steps,
            "what": "host C++ block manager per decode step through the Python binding: "
                    "one slot for every sequence, then the padded [S, max_blocks] tables"}


def time_aux_kernels(torch, B, wl, pairs, kp, vp, kn, vn, slots, device, fp8, ksc, vsc,
                     nbytes, calls=20, reps=10):
    """kv_write (or kv_write_fp8) of the step's new tokens and kv_copy_blocks, each timed
    alone: a CUDA graph of `calls` back-to-back calls replayed `reps` times between CUDA
    events.  Workloads without copy-on-write pairs copy one block per sequence (its last
    block into a block no table maps), the most a decode step can need.  Both are small and
    L2-warm when back to back, so they measure launch-bound kernels as a step runs them."""
    kv_es = 1 if fp8 else wl.elem_size
    if len(pairs):
        cp, source = np.ascontiguousarray(pairs, np.int32), "the step's copy-on-write pairs"
    else:
        used = np.zeros(wl.num_blocks, bool)
        used[wl.block_tables[wl.block_tables >= 0]] = True
        free = np.flatnonzero(~used)
        n = min(wl.num_seqs, len(free))
        last = (wl.context_lens.astype(np.int64) - 1) // wl.block_size
        src = wl.block_tables[np.arange(n), last[:n]]
        cp = np.stack([src, free[:n]], 1).astype(np.int32)
        source = "one per sequence: its last block into a block no table maps"
    cp_d = torch.from_numpy(cp).to(device)
    copy_bytes = len(cp) * wl.num_kv_heads * wl.block_size * wl.head_dim * kv_es * 2 * 2

    def write():
        if fp8:
            B.kv_write_fp8(kn, vn, slots, ksc, vsc, kp, vp)
        else:
            B.kv_write(kn, vn, slots, kp, vp)

    res = {}
    gs = torch.cuda.Stream(device)
    for name, call, nb in (("kv_write_fp8" if fp8 else "kv_write", write, nbytes["kv_write"]),
                           ("kv_copy_blocks", lambda: B.kv_copy_blocks(cp_d, kp, vp),
                            copy_bytes)):
        with torch.cuda.stream(gs):
            call()
        gs.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=gs):
            for _ in range(calls):
                call()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(gs):
            g.replay()
            a.record(gs)
            for _ in range(reps):
                g.replay()
            b.record(gs)
        gs.synchronize()
        us = a.elapsed_time(b) * 1e3 / (calls * reps)
        res[name] = {"us": round(us, 3), "bytes": int(nb), "gbs": round(nb / (us * 1e-6) / 1e9, 1)}
        del g
    res["kv_copy_blocks"]["pairs"] = int(len(cp))
    res["kv_copy_blocks"]["pairs_source"] = source
    res["timing"] = ("CUDA graph of %d back-to-back calls replayed %d times, CUDA events; "
                     "L2-warm" % (calls, reps))
    return res


def read_probe_gbs(torch, B, device, chunk, gib=4, reps=3, per_sm=(2, 4, 6, 8, 0)):
    """The library's streaming probe (pkv_read_probe: pseudo-randomly permuted chunk-sized
    bulk copies of a gib-GiB buffer into shared memory, nothing else), best over reps and over
    a few concurrencies (CTAs per SM; 0 = as many as fit): the read ceiling for copies of the
    decode's size, set beside the copy-based peak.  Returns (GB/s, CTAs per SM of the best)."""
    x = torch.empty(gib << 30, dtype=torch.uint8, device=device)
    x.fill_(1)
    best, best_per = 0.0, None
    for per in per_sm:
        for _ in range(reps + 1):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            n = B.read_probe(x, chunk, per)
            b.record()
            torch.cuda.synchronize()
            gbs = n / (a.elapsed_time(b) * 1e-3) / 1e9
            if gbs > best:
                best, best_per = gbs, per
    faults = B.device_faults(clear=True)
    del x
    torch.cuda.empty_cache()
    if faults:
        raise RuntimeError("device faults in the read probe: %s" % faults)
    return round(best, 1), best_per


# ---- the CUDA path --------------------------------------------------------------------------
def gpu_uuid(torch, device):
    try:
        u = str(torch.cuda.get_device_properties(device).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        return str(device.index)


def run_pkv(args):
    import torch
    from paged_kv_cache_392_b200 import build as pbuild
    defines = args.lib_defines.split()
    if defines:             # before the binding is imported: it loads the library PKV_LIB names
        os.environ["PKV_LIB"] = pbuild.build(out=pbuild.variant_path(defines), defines=defines)
    else:
        pbuild.build()
    from paged_kv_cache_392_b200 import binding as B
    from paged_kv_cache_392_b200 import workloads as W

    world, rank, local = dist_env()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    dist = init_dist(world)

    wl, pairs = build_workload(args.workload, block_size=args.block_size)
    if args.contiguous:
        if args.workload in ("fork", "beam", "prefix"):
            raise SystemExit("--contiguous does not apply to the sharing workloads")
        contiguous_placement(wl)
    pt = args.partition_tokens if args.partition_tokens is not None else wl.partition_tokens
    fp8 = args.kv_fp8
    if fp8 and (args.workload not in ("opt13b", "gqa", "long") or wl.head_dim != 128):
        raise SystemExit("--kv-fp8 applies to the opt13b, gqa and long workloads")
    vals = W.make_values_fp8(wl, device) if fp8 else W.make_values(wl, device)
    q, kp, vp, kn, vn = (vals[k] for k in ("q", "k_pool", "v_pool", "k_new", "v_new"))
    ksc, vsc = vals.get("k_scale"), vals.get("v_scale")
    bt = torch.from_numpy(wl.block_tables).to(device)
    lens = torch.from_numpy(wl.context_lens).to(device)
    slots = torch.from_numpy(np.ascontiguousarray(wl.slot_mapping, np.int64)).to(device)
    pairs_d = torch.from_numpy(np.ascontiguousarray(pairs, np.int32)).to(device)
    out = torch.empty_like(q)
    desc = B.make_desc(wl.num_seqs, wl.num_q_heads, wl.num_kv_heads, wl.head_dim,
                       wl.num_blocks, bt.shape[1], q.dtype, pt or 0, wl.block_size)
    ws_bytes = B.attn_workspace_bytes(desc)
    ws = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=device)
    npairs = len(pairs)
    # the partition the library will use (the FP8 decode may pick a wider one)
    pt_run = B.fp8_partition_tokens(desc) if fp8 else (pt or 512)
    rows_split, pmax = split_rows(wl, pt_run)
    nbytes = algorithmic_bytes(wl, pairs, rows_split, kv_es=1 if fp8 else None)

    # The newest token's write runs inside the decode kernel (kv_write_and_decode,
    # kv_write_fp8_and_decode) unless --separate-write asks for the two calls, or the step is
    # the decode alone (--decode-only, --layout contiguous).
    contig = args.layout == "contiguous"
    decode_only = args.decode_only or contig
    if contig and (fp8 or npairs or args.workload in ("fork", "beam", "prefix", "tiny")):
        raise SystemExit("--layout contiguous applies to the opt13b, gqa and long workloads")
    fused = not args.separate_write and not decode_only
    kc = vc = None
    if contig:      # the same tokens in a [S][H_kv][Lmax][D] reservation per sequence
        Bs = wl.block_size
        lmax = wl.max_blocks_per_seq * Bs
        kc = torch.zeros((wl.num_seqs, wl.num_kv_heads, lmax, wl.head_dim), dtype=kp.dtype,
                         device=device)
        vc = torch.zeros_like(kc)
        for s_ in range(wl.num_seqs):
            L = int(wl.context_lens[s_])
            t = torch.arange(L, device=device)
            blk = bt[s_].long()[t // Bs]
            kc[s_, :, :L] = kp[blk, :, t % Bs].permute(1, 0, 2)
            vc[s_, :, :L] = vp[blk, :, t % Bs].permute(1, 0, 2)
        nbytes["decode"] -= int(((wl.context_lens + Bs - 1) // Bs).sum()) * 4 + wl.num_seqs * 4
        nbytes["step"] = nbytes["decode"]

    def write(kn_, vn_, slots_):
        if fused or decode_only:
            return
        if fp8:
            B.kv_write_fp8(kn_, vn_, slots_, ksc, vsc, kp, vp)
        else:
            B.kv_write(kn_, vn_, slots_, kp, vp)

    def decode(q_, kn_, vn_, slots_, bt_, lens_, out_):
        if contig:
            B.attn_decode_contiguous(q_, kc, vc, lens_, wl.scale, out=out_, workspace=ws,
                                     partition_tokens=pt)
        elif fp8 and fused:
            B.kv_write_fp8_and_decode(q_, kn_, vn_, slots_, ksc, vsc, kp, vp, bt_, lens_,
                                      wl.scale, out=out_, workspace=ws, partition_tokens=pt)
        elif fp8:
            B.paged_attn_decode_fp8(q_, kp, vp, ksc, vsc, bt_, lens_, wl.scale, out=out_,
                                    workspace=ws, partition_tokens=pt)
        elif fused:
            B.kv_write_and_decode(q_, kn_, vn_, slots_, kp, vp, bt_, lens_, wl.scale,
                                  out=out_, workspace=ws, partition_tokens=pt)
        else:
            B.paged_attn_decode(q_, kp, vp, bt_, lens_, wl.scale, out=out_, workspace=ws,
                                partition_tokens=pt)

    def step():
        if npairs:
            B.kv_copy_blocks(pairs_d, kp, vp)
        write(kn, vn, slots)
        decode(q, kn, vn, slots, bt, lens, out)

    launches_per_step = ((1 if npairs else 0) + (0 if fused or decode_only else 1) + 1 +
                         (1 if pmax > 1 else 0))
    decode_call_bytes = nbytes["decode"] + (nbytes["kv_write"] if fused else 0)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    faults = B.device_faults(clear=True)
    if faults:
        raise RuntimeError("device faults during warm-up: %s" % faults)

    # Runs of N consecutive steps are captured as one CUDA graph on a side stream, with an
    # event-record node on each side of every E-th decode call; the timed loop replays the
    # graph, so neither host launch overhead nor gaps between launches leak into device
    # time.  The decode-call durations come from those events (the last replay's N / E
    # calls).  An event node serialises the stream around it, so bracketing every call
    # would slow the step it measures by about 5 %.
    flush = uses_l2_flush(args, wl, nbytes, fp8)
    scrub = torch.empty(256 << 20, dtype=torch.uint8, device=device) if flush else None
    K = args.steps
    N = max(1, min(50, K // 4))   # at least 4 replays, so the line carries a spread
    E = 1 if flush else max(1, args.decode_events_every)
    gs = torch.cuda.Stream(device)
    ev = [(torch.cuda.Event(enable_timing=True, external=True),
           torch.cuda.Event(enable_timing=True, external=True)) for _ in range(N)]
    timed = [j for j in range(N) if j % E == 0]
    # flush mode: an event after the flush of every step marks where the step's own work
    # starts, so the step time leaves the flush out
    evs = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(N)]

    def capture(nsteps):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=gs):
            for j in range(nsteps):
                if scrub is not None:
                    scrub.fill_(j & 0xFF)       # evict the previous step's lines from L2
                    evs[j].record(gs)
                if npairs:
                    B.kv_copy_blocks(pairs_d, kp, vp)
                write(kn, vn, slots)
                if j % E == 0:
                    ev[j][0].record(gs)
                decode(q, kn, vn, slots, bt, lens, out)
                if j % E == 0:
                    ev[j][1].record(gs)
        return g

    g_run = capture(N)
    g_rem = capture(K % N) if K % N else None
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(gpu_uuid(torch, device))
    with torch.cuda.stream(gs):
        for _ in range(max(1, -(-args.warmup // N))):
            g_run.replay()
        barrier(dist, device)
        torch.cuda.synchronize()
        sampler.start()
        torch.cuda.nvtx.range_push("timed steps")
        t0.record(gs)
        if g_rem is not None:
            g_rem.replay()
        # an event after each replay of N steps: the spread of the per-step time
        rep_ev = [torch.cuda.Event(enable_timing=True) for _ in range(K // N)]
        for r in range(K // N):
            g_run.replay()
            rep_ev[r].record(gs)
        t1.record(gs)
        torch.cuda.synchronize()
        torch.cuda.nvtx.range_pop()
        barrier(dist, device)
    sampler.stop()
    ms_local = t0.elapsed_time(t1)
    if scrub is not None:   # step time without the flush: flush end -> decode call end
        ms_local = statistics.fmean(evs[j].elapsed_time(ev[j][1]) for j in range(N)) * K
    if scrub is not None:   # the last replay's steps, each without its flush
        per_step = [evs[j].elapsed_time(ev[j][1]) for j in range(N)]
    else:                   # one replay of N steps at a time
        per_step = [rep_ev[r - 1].elapsed_time(rep_ev[r]) / N for r in range(1, len(rep_ev))]
    step_pcts = (np.percentile(per_step, [10, 50, 90]).tolist() if len(per_step) >= 2 else None)
    ms = max_over_ranks(dist, ms_local, device)
    decode_ms = statistics.fmean(ev[j][0].elapsed_time(ev[j][1]) for j in timed)
    decode_ms = max_over_ranks(dist, decode_ms, device)
    faults = B.device_faults(clear=True)
    if faults:
        raise RuntimeError("device faults during timing: %s" % faults)
    del g_run, g_rem

    # ---- end to end through the public API with host buffers -------------------------
    # Every step copies its inputs (q, new K/V, slots, tables, lengths, copy pairs) from pinned
    # host memory and reads its output back.  "serial": one step at a time, synchronised.
    # "pipelined": E2E_BUFS input/output buffer sets; the copies of step i+1 run on a copy
    # stream while step i computes and step i-1's output copies on a third stream (all three
    # in one graph a step), and the host stays at most E2E_BUFS - 1 steps ahead.
    host_in = {"q": q, "kn": kn, "vn": vn, "slots": slots, "bt": bt, "lens": lens,
               "pairs": pairs_d}
    pin = {k: v.cpu().pin_memory() for k, v in host_in.items()}
    h2d = sum(t.numel() * t.element_size() for k, t in pin.items()
              if k != "pairs" or npairs)
    d2h = out.numel() * out.element_size()
    torch.cuda.synchronize()
    main = torch.cuda.Stream(device)          # graphs are captured on non-default streams
    copy_stream = torch.cuda.Stream(device)
    nbuf = E2E_BUFS
    bufs = [host_in] + [{k: v.clone() for k, v in host_in.items()} for _ in range(nbuf - 1)]
    outs = [out] + [torch.empty_like(out) for _ in range(nbuf - 1)]
    outs_h = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(nbuf)]

    def run_kernels(b):
        d = bufs[b]
        if npairs:
            B.kv_copy_blocks(d["pairs"], kp, vp)
        write(d["kn"], d["vn"], d["slots"])
        decode(d["q"], d["kn"], d["vn"], d["slots"], d["bt"], d["lens"], outs[b])

    def h2d_copy(b, stream):
        with torch.cuda.stream(stream):
            for k, t in bufs[b].items():
                if k != "pairs" or npairs:
                    t.copy_(pin[k], non_blocking=True)

    def e2e_serial_step():
        with torch.cuda.stream(main):
            h2d_copy(0, main)
            run_kernels(0)
            outs_h[0].copy_(outs[0], non_blocking=True)
        main.synchronize()

    # One CUDA graph per buffer phase holds a whole pipelined step on three streams: the
    # kernels of step i (buffer set i mod n) on the compute stream, the input copies of step
    # i+1 into the next set on a copy stream, and the output copy of step i-1 on a third.
    # Graph launches on one stream run in order, so buffer reuse needs no other sync, and a
    # step costs the host one graph launch.
    d2h_stream = torch.cuda.Stream(device)
    for b in range(nbuf):
        with torch.cuda.stream(main):
            run_kernels(b)                 # warm the library paths outside capture
        main.synchronize()
    g_step = []
    for b in range(nbuf):
        nxt, prv = (b + 1) % nbuf, (b - 1) % nbuf
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=main):
            fork = torch.cuda.Event()
            fork.record(main)
            copy_stream.wait_event(fork)
            d2h_stream.wait_event(fork)
            with torch.cuda.stream(copy_stream):
                for k, t in bufs[nxt].items():
                    if k != "pairs" or npairs:
                        t.copy_(pin[k], non_blocking=True)
            with torch.cuda.stream(d2h_stream):
                outs_h[prv].copy_(outs[prv], non_blocking=True)
            run_kernels(b)
            j1, j2 = torch.cuda.Event(), torch.cuda.Event()
            j1.record(copy_stream)
            j2.record(d2h_stream)
            main.wait_event(j1)
            main.wait_event(j2)
        g_step.append(g)
    torch.cuda.synchronize()
    step_done = [torch.cuda.Event() for _ in range(nbuf)]

    def e2e_pipelined(n):
        h2d_copy(0, main)                  # fill: the first step's inputs
        for i in range(n):
            b = i % nbuf
            with torch.cuda.stream(main):
                g_step[b].replay()
            step_done[b].record(main)
            if i >= nbuf - 1:              # the host is at most nbuf - 1 steps ahead
                step_done[(i - nbuf + 1) % nbuf].synchronize()
        last = (n - 1) % nbuf              # drain: the last step's output
        with torch.cuda.stream(main):
            outs_h[last].copy_(outs[last], non_blocking=True)
        main.synchronize()

    # pipelined e2e: at least 1000 steps (about 0.13 s on the headline batch), so that the
    # pipeline's fill and drain and the first replays of the freshly captured graphs
    # do not dominate a short run
    Ke = max(1000, K)
    Ks = max(1, min(K, 1000))     # serial mode: at most 1000 synchronised steps
    for _ in range(max(3, args.warmup // 4)):
        e2e_serial_step()
    e2e_pipelined(4 * nbuf)
    gc.disable()                  # no collector pauses inside the host-driven loops
    barrier(dist, device)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.nvtx.range_push("e2e serial")
    e0.record(main)
    for _ in range(Ks):
        e2e_serial_step()
    e1.record(main)
    torch.cuda.synchronize()
    torch.cuda.nvtx.range_pop()
    e2e_serial_ms = max_over_ranks(dist, e0.elapsed_time(e1) / Ks, device)
    barrier(dist, device)
    torch.cuda.synchronize()
    torch.cuda.nvtx.range_push("e2e pipelined")
    e0.record(main)
    e2e_pipelined(Ke)
    e1.record(main)                # e2e_pipelined returned after the last output landed
    torch.cuda.synchronize()
    torch.cuda.nvtx.range_pop()
    gc.enable()
    e2e_ms = max_over_ranks(dist, e0.elapsed_time(e1) / Ke, device)
    barrier(dist, device)
    faults = B.device_faults(clear=True)
    if faults:
        raise RuntimeError("device faults during the end-to-end runs: %s" % faults)
    torch.cuda.nvtx.range_push("kv_write / kv_copy_blocks alone")
    aux = time_aux_kernels(torch, B, wl, pairs, kp, vp, kn, vn, slots, device, fp8, ksc, vsc,
                           nbytes)
    torch.cuda.nvtx.range_pop()
    faults = B.device_faults(clear=True)
    if faults:
        raise RuntimeError("device faults in the kv_write / kv_copy_blocks timing: %s" % faults)

    result = None
    if rank == 0:
        bm_host = time_block_manager(B, wl)
        peak, peak_kind = hbm_peak()
        step_ms = ms / K
        kv_gbs = world * nbytes["kv"] / (step_ms * 1e-3) / 1e9
        # When a step is the decode call alone (fused write, no copy-on-write copies), the
        # step time is that call's duration, taken with no event node inside the loop; the
        # roofline uses it.  Otherwise it uses the event-bracketed calls.
        only_call = (fused or decode_only) and not npairs and scrub is None
        bracketed = decode_call_bytes / (decode_ms * 1e-3) / 1e9
        call_ms = step_ms if only_call else decode_ms
        achieved = decode_call_bytes / (call_ms * 1e-3) / 1e9
        # the committed summaries were taken on 16-token blocks in the paged layout
        traffic = (None if args.separate_write or decode_only or contig
                   or wl.block_size != 16 else profile_traffic(args.workload, fp8))
        # one 16-token K (or V) copy of the decode
        probe_chunk = 16 * wl.head_dim * (1 if fp8 else 4 if wl.dtype == "f32" else 2)
        probe, probe_per = ((None, None) if args.no_read_probe
                            else read_probe_gbs(torch, B, device,
                                                max(2048, min(16384, probe_chunk))))
        swap = swap_probe(torch, B, wl, kp, vp, device) if args.swap_probe and not fp8 else None
        result = {
            "metric": METRIC,
            "value": round(kv_gbs, 2),
            "unit": "GB/s",
            "n_gpus": world,
            "steps": K,
            "warmup": args.warmup,
            "ms_per_step": round(step_ms, 5),
            "ms_per_step_p10_p50_p90": ([round(x, 5) for x in step_pcts] if step_pcts else None),
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": ("f32 accumulate over fp8-e4m3 KV (codes widened exactly to f16 for "
                      "f16 tensor-core tiles), %s q/out" % wl.dtype) if fp8 else
                     "f32 accumulate over %s KV" % wl.dtype,
            "data": "synthetic (seeded), no weights",
            "seqs_per_s": round(world * wl.num_seqs / (step_ms * 1e-3), 1),
            "hbm_frac_step": round(kv_gbs / world / peak, 4),
            "hbm_frac_step_of_8TBs_spec": round(kv_gbs / world / 8000.0, 4),
            "config": step_config(args, wl, npairs, pt_run, nbytes, scrub is not None, fp8),
            "roofline": {
                "bound": "hbm",
                "kernel": ("attn_decode_contiguous (contiguous decode + lse_reduce)" if contig
                           else "%s (%sdecode + lse_reduce)" % (
                               {(True, True): "kv_write_fp8_and_decode", (True, False):
                                "paged_attn_decode_fp8", (False, True): "kv_write_and_decode",
                                (False, False): "paged_attn_decode"}[(fp8, fused)],
                               "newest-token write + " if fused else "")),
                "achieved": round(achieved, 1),
                "peak": peak,
                "peak_kind": peak_kind,
                "peak_basis": ("copy-based: read + write bytes of a device-to-device copy, so "
                               "a read-dominated stream can exceed it; frac_of_8TBs_spec "
                               "is the fraction of the HBM3e specification"),
                "unit": "GB/s",
                "frac": round(achieved / peak, 4),
                "frac_of_8TBs_spec": round(achieved / 8000.0, 4),
                "read_probe_gbs": probe,
                "read_probe_chunk_bytes": (None if probe is None
                                           else max(2048, min(16384, probe_chunk))),
                "read_probe_ctas_per_sm": probe_per,
                "frac_of_read_probe": round(achieved / probe, 4) if probe else None,
                "traffic": traffic,
                "algorithmic_bytes": decode_call_bytes,
                "avg_launch_ms": round(call_ms, 5),
                "launch_timing": ("step: one decode call per step, events around the whole "
                                  "timed loop" if only_call else
                                  "event-bracketed calls, every %d-th of the timed graph" % E),
                "achieved_bracketed": round(bracketed, 1),
                "avg_launch_ms_bracketed": round(decode_ms, 5),
                "timed_launches_per_graph": len(timed),
            },
            "e2e": {"value": round(world * nbytes["kv"] / (e2e_ms * 1e-3) / 1e9, 2),
                    "unit": "GB/s", "ms_per_step": round(e2e_ms, 5),
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "steps": Ke, "mode": "pipelined: input copies of step i+1 and the output "
                                          "copy of step i-1 overlap step i's kernels "
                                          "(three streams in one CUDA graph a step; %d "
                                          "buffer sets, the host at most %d steps ahead)"
                                          % (E2E_BUFS, E2E_BUFS - 1),
                    "serial_value": round(world * nbytes["kv"] / (e2e_serial_ms * 1e-3) / 1e9,
                                          2),
                    "serial_ms_per_step": round(e2e_serial_ms, 5),
                    "l2": "not flushed between steps" if scrub is not None else
                          "working set larger than L2"},
            "gpu_launches": K * launches_per_step,
            "write_and_copy_kernels": aux,
            "block_manager_host": bm_host,
            "kv_utilisation": kv_utilisation(wl),
            "swap": swap,
            "clocks": sampler.summary(),
        }
        if "unique_blocks" in wl.extra:
            uniq = wl.extra["unique_blocks"] * wl.num_kv_heads * wl.block_size * wl.head_dim * \
                wl.elem_size * 2
            result["config"]["unique_kv_bytes"] = uniq
            result["unique_kv_gbs"] = round(world * uniq / (step_ms * 1e-3) / 1e9, 2)
        if "sharing" in wl.extra:
            result["sharing"] = wl.extra["sharing"]
        result["cache_bytes"] = {"paged_pools": 2 * kp.numel() * kp.element_size(),
                                 "contiguous_reservation": (2 * kc.numel() * kc.element_size()
                                                            if contig else None)}
        if defines:
            result["library"] = {"variant_defines": defines,
                                 "path": os.path.basename(os.environ["PKV_LIB"])}
        if world == 1 and not args.no_cpu_baseline and not fp8:
            result["cpu_baseline"] = cpu_baseline(wl, vals, args.cpu_seconds)
    if dist is not None:
        barrier(dist, device)
        dist.destroy_process_group()
    return result


# ---- the fp64 oracle on the host cores ------------------------------------------------------
def _seq_kv_bytes(wl, s):
    return int(wl.context_lens[s]) * wl.num_kv_heads * wl.head_dim * wl.elem_size * 2


def _pick_sequences(wl, bytes_budget):
    """Sequences, in a seeded shuffled order, until their KV bytes reach the budget."""
    order = np.random.default_rng(12345).permutation(wl.num_seqs)
    chosen, total = [], 0
    for s in order:
        chosen.append(int(s))
        total += _seq_kv_bytes(wl, s)
        if total >= bytes_budget:
            break
    return sorted(chosen), total


def _oracle_rows(wl, seqs):
    return np.array([(s, h) for s in seqs for h in range(wl.num_q_heads)], np.int32)


def _calibrate(oracle, wl, host, nthreads=None):
    """Oracle KV bytes per second on this host, from one mid-sized sequence."""
    s = int(np.argsort(wl.context_lens)[wl.num_seqs // 2])
    rows = _oracle_rows(wl, [s])
    t = time.perf_counter()
    oracle.paged_attn_decode(host["q"], host["k_pool"], host["v_pool"], wl.block_tables,
                             wl.context_lens, wl.scale, wl.dtype, rows=rows, nthreads=nthreads)
    dt = max(time.perf_counter() - t, 1e-4)
    return _seq_kv_bytes(wl, s) / dt


def _time_oracle(oracle, wl, host, seconds, nthreads=None):
    """The oracle on a sample of the batch, repeated to about `seconds` of host time."""
    rate = _calibrate(oracle, wl, host, nthreads)
    seqs, nbytes = _pick_sequences(wl, rate * seconds)
    rows = _oracle_rows(wl, seqs)
    reps, t = 0, time.perf_counter()
    while True:     # repeat the sample (whole batch when it is small) until ~seconds
        oracle.paged_attn_decode(host["q"], host["k_pool"], host["v_pool"], wl.block_tables,
                                 wl.context_lens, wl.scale, wl.dtype, rows=rows,
                                 nthreads=nthreads)
        reps += 1
        dt = time.perf_counter() - t
        if dt >= 0.8 * seconds or reps >= 1000:
            break
    return {"value": round(reps * nbytes / dt / 1e9, 4), "unit": "GB/s",
            "seqs_per_s": round(reps * len(seqs) / dt, 3), "seconds": round(dt, 2),
            "sample": "decode attention of %d of %d sequences (all %d query heads, %d context "
                      "tokens) of the same batch, repeated %d times, fp64, exact two-pass "
                      "softmax" % (len(seqs), wl.num_seqs, wl.num_q_heads,
                                   int(wl.context_lens[seqs].sum()), reps)}


def cpu_baseline(wl, vals, seconds):
    """The oracle on every usable host core (OpenMP over rows), then on one core."""
    import oracle
    from paged_kv_cache_392_b200 import workloads as W
    host = {k: W.to_numpy_bits(vals[k]) for k in ("q", "k_pool", "v_pool")}
    res = _time_oracle(oracle, wl, host, seconds)
    res.update({"cores": oracle.num_threads(), "kind": "oracle"})
    one = _time_oracle(oracle, wl, host, seconds / 3, nthreads=1)
    one["cores"] = 1
    res["single_core"] = one
    return res


def run_reference(args):
    world, rank, _ = dist_env()
    if rank != 0:
        return None
    import oracle
    import torch
    from paged_kv_cache_392_b200 import workloads as W
    wl, pairs = build_workload(args.workload, model_block_manager=True,
                               block_size=args.block_size)
    if args.contiguous:
        contiguous_placement(wl)
    pt = args.partition_tokens if args.partition_tokens is not None else wl.partition_tokens
    pt_run = pt or 512
    step_bytes = algorithmic_bytes(wl, pairs, split_rows(wl, pt_run)[0])
    flush = uses_l2_flush(args, wl, step_bytes, False)
    vals = W.make_values(wl, "cpu", torch=torch)
    host = {k: W.to_numpy_bits(v).copy() for k, v in vals.items()}
    rate = _calibrate(oracle, wl, host)
    budget_s = max(0.02, min(1.0, 90.0 / max(1, args.steps + args.warmup)))
    seqs, nbytes = _pick_sequences(wl, rate * budget_s)
    rows = _oracle_rows(wl, seqs)
    sel = np.array(seqs)
    chosen = set(seqs)
    # the sample's copy-on-write pairs: those whose destination one of its sequences maps
    dst_of = {int(b) for s in seqs for b in wl.block_tables[s] if b >= 0}
    sp = np.array([p for p in pairs if int(p[1]) in dst_of], np.int32).reshape(-1, 2)
    kn, vn = host["k_new"][sel].copy(), host["v_new"][sel].copy()
    slots = wl.slot_mapping[sel].copy()

    def step():
        if len(sp):
            oracle.kv_copy_blocks(sp, host["k_pool"], host["v_pool"])
        oracle.kv_write(kn, vn, slots, host["k_pool"], host["v_pool"])
        oracle.paged_attn_decode(host["q"], host["k_pool"], host["v_pool"], wl.block_tables,
                                 wl.context_lens, wl.scale, wl.dtype, rows=rows)

    for _ in range(args.warmup):
        step()
    t = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = (time.perf_counter() - t) / max(1, args.steps)
    gbs = nbytes / dt / 1e9
    sample = ("per step: kv_write + decode attention of %d of %d sequences (%d context "
              "tokens, all %d query heads)%s, fp64 oracle" %
              (len(seqs), wl.num_seqs, int(wl.context_lens[sel].sum()), wl.num_q_heads,
               (", %d copy-on-write pairs" % len(sp)) if len(sp) else ""))
    assert len(chosen) == len(seqs)
    return {
        "metric": METRIC, "value": round(gbs, 4), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt * 1e3, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded), no weights", "impl": "reference",
        "seqs_per_s": round(len(seqs) / dt, 3),
        "config": step_config(args, wl, len(pairs), pt_run, step_bytes, flush, False),
        "cpu_baseline": {"value": round(gbs, 4), "unit": "GB/s", "kind": "oracle",
                         "cores": oracle.num_threads(), "sample": sample},
        "e2e": {"value": round(gbs, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main(argv=None):
    args = parse_args(argv)
    world, rank, _ = dist_env()
    if args.gpus != world and world > 1:
        print("warning: --gpus %d but WORLD_SIZE %d" % (args.gpus, world), file=sys.stderr)
    res = run_reference(args) if args.impl == "reference" else run_pkv(args)
    if rank == 0 and res is not None:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
