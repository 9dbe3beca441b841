"""CPU checks of bench.py's host logic: the reference (oracle) arm's JSON line, the
multi-process launch where rank 0 alone reports, and the max-over-ranks timing reduction
over a world-size-2 gloo group."""
import json
import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402

KEYS = {"metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
        "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "impl",
        "cpu_baseline", "e2e"}


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_reference_arm_prints_one_json_line():
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload",
                          "tiny", "--steps", "2", "--warmup", "1"], cwd=ROOT,
                         capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr
    lines = [ln for ln in out.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert KEYS <= set(d)
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"
    assert d["cpu_baseline"]["cores"] >= 1


def test_reference_arm_under_two_ranks_reports_once():
    env = dict(os.environ, OMP_NUM_THREADS="1")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), "bench.py",
           "--impl", "reference", "--workload", "tiny", "--gpus", "2", "--steps", "1",
           "--warmup", "0"]
    out = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300, env=env)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1 and json.loads(lines[0])["n_gpus"] == 2


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    w, r, lr = bench.dist_env()
    dist = bench.init_dist(w, backend="gloo")
    dev = torch.device("cpu")
    bench.barrier(dist, dev)
    m = bench.max_over_ranks(dist, 1.5 + rank, dev)
    bench.barrier(dist, dev)
    dist.destroy_process_group()
    q.put((r, w, m))


def test_max_over_ranks_with_gloo_world_size_2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res == [(0, 2, 2.5), (1, 2, 2.5)]


def test_algorithmic_bytes_and_split_rows():
    from paged_kv_cache_392_b200 import workloads as W
    wl = W.tiny()
    import numpy as np
    nb = bench.algorithmic_bytes(wl, np.zeros((0, 2), np.int32))
    assert nb["kv"] == (5 + 17 + 33 + 48) * 2 * 64 * 4 * 2
    assert nb["decode"] > nb["kv"] and nb["kv_copy"] == 0
    rows, pmax = bench.split_rows(wl, 16)
    # lengths 5, 17, 33, 48 over 16-token partitions: 1, 2, 3, 3 partitions
    assert pmax == 3 and rows == (2 + 3 + 3) * 2


def test_algorithmic_bytes_of_the_tiny_step_by_hand():
    """The byte count the roofline divides by, for the tiny workload (4 sequences, lengths
    5, 17, 33, 48; 2 heads; D 64; fp32), written out term by term."""
    wl, pairs = bench.build_workload("tiny")
    nb = bench.algorithmic_bytes(wl, pairs)
    tokens = 5 + 17 + 33 + 48
    assert nb["kv"] == tokens * 2 * 64 * 4 * 2                       # K and V, read once
    qo = 4 * 2 * 64 * 4 * 2                                          # q read, out written
    tables = (1 + 2 + 3 + 3) * 4 + 4 * 4                             # table entries + lengths
    assert nb["decode"] == nb["kv"] + qo + tables
    assert nb["kv_write"] == 4 * 2 * 64 * (4 + 4) * 2 + 4 * 8        # new K/V in, slots out
    assert nb["kv_copy"] == 0
    # split: 2 rows x 130 floats written and read per partial state
    nb2 = bench.algorithmic_bytes(wl, pairs, split_rows=2)
    assert nb2["decode"] - nb["decode"] == 2 * (64 + 2) * 4 * 2
    # FP8 pools: one byte per cached K/V element
    assert bench.algorithmic_bytes(wl, pairs, kv_es=1)["kv"] == tokens * 2 * 64 * 1 * 2


def test_split_rows_counts_only_sequences_that_span_partitions():
    wl, _ = bench.build_workload("tiny")
    # 16-token partitions: lengths 5 | 17 | 33 | 48 span 1 | 2 | 3 | 3 partitions
    rows, pmax = bench.split_rows(wl, 16)
    assert pmax == 3 and rows == (2 + 3 + 3) * wl.num_q_heads
    assert bench.split_rows(wl, 0) == (0, 1)


def _fake_workload(lens, tables):
    class _W:
        pass
    w = _W()
    w.context_lens = np.asarray(lens, np.int32)
    w.block_tables = np.asarray(tables, np.int32)
    return w


def test_kv_utilisation_follows_the_pages_waste_examples():
    """The pages' worked examples (300 and 50 tokens in 16-token blocks): slots allocated and
    filled as the fixture states; a block that two sequences map counts once."""
    golden = json.load(open(os.path.join(ROOT, "tests", "golden", "waste_examples.json")))
    for c in golden["cases"]:
        nb = c["paged_blocks"]
        u = bench.kv_utilisation(_fake_workload([c["tokens"]], [list(range(nb))]))
        assert u["slots_allocated"] == c["paged_slots"]
        assert u["slots_allocated"] - u["tokens_in_blocks"] == c["paged_wasted"]
    # two sequences sharing a full first block: 16 + 5 + 9 tokens in 3 distinct blocks
    u = bench.kv_utilisation(_fake_workload([21, 25], [[7, 3], [7, 4]]))
    assert u["slots_allocated"] == 48 and u["tokens_in_blocks"] == 16 + 5 + 9


def test_both_arms_describe_the_step_with_one_config():
    args = bench.parse_args(["--workload", "fork"])
    wl, pairs = bench.build_workload("fork")
    wl2, pairs2 = bench.build_workload("fork", model_block_manager=True)
    assert np.array_equal(wl.block_tables, wl2.block_tables)
    assert np.array_equal(pairs, pairs2)
    rows, _ = bench.split_rows(wl, 512)
    nb = bench.algorithmic_bytes(wl, pairs, rows)
    c1 = bench.step_config(args, wl, len(pairs), 512, nb, bench.uses_l2_flush(args, wl, nb, False),
                           False)
    c2 = bench.step_config(args, wl2, len(pairs2), 512, nb,
                           bench.uses_l2_flush(args, wl2, nb, False), False)
    assert c1 == c2 and c1["cow_pairs_per_step"] == 112


def test_block_manager_host_timing_leaves_no_sequence_behind():
    """The bench's host timing of one step's block-manager work: it must run on the host
    alone (no GPU), append exactly one slot per sequence per step, and report both parts."""
    from paged_kv_cache_392_b200 import binding as B
    from paged_kv_cache_392_b200 import workloads as W
    wl = W.make_workload("bm", [5, 17, 33, 48, 1], 2, 2, 64, "f32", 3)
    r = bench.time_block_manager(B, wl, steps=40)
    assert r["seqs"] == 5 and r["steps"] == 40
    assert r["append_slots_us"] > 0 and r["block_tables_us"] > 0
