"""The product's C++ block manager against the plain-Python model, bit for bit: block tables,
slots, copy-on-write pairs, reference counts and free-list order (CPU only)."""
import numpy as np
import pytest

from oracle.block_manager import BlockManagerModel, OutOfBlocks as ModelOOM
from paged_kv_cache_392_b200 import binding as B
from paged_kv_cache_392_b200 import build as pbuild
from paged_kv_cache_392_b200 import workloads as W


@pytest.fixture(scope="module", autouse=True)
def _built():
    pbuild.build()


def same_state(bm, model, seqs):
    assert bm.num_free() == model.num_free()
    assert bm.free_order() == model.free_order()
    assert [bm.refcount(b) for b in range(model.num_blocks)] == model.ref
    assert bm.num_seqs() == len(model.tables)
    for s in seqs:
        assert bm.block_table(s) == model.block_table(s)
        assert bm.seq_len(s) == model.seq_len(s)


@pytest.mark.parametrize("seed,block_size", [(0, 16), (1, 16), (2, 16), (3, 32), (4, 32)])
def test_random_traffic_matches_model(seed, block_size):
    rng = np.random.default_rng(seed)
    NB = 48 if block_size == 16 else 30
    order = rng.permutation(NB)
    bm = B.BlockManager(NB, block_size=block_size, free_order=order)
    model = BlockManagerModel(NB, block_size=block_size, free_order=order)
    live, nxt = [], 100
    for _ in range(1500):
        op = int(rng.integers(0, 12))
        if op == 0 or not live:
            n = int(rng.integers(0, 70))
            try:
                model.add_seq(nxt, n)
            except ModelOOM:
                with pytest.raises(B.OutOfBlocks):
                    bm.add_seq(nxt, n)
                continue
            bm.add_seq(nxt, n)
            live.append(nxt)
            nxt += 1
        elif op == 1:
            p = live[int(rng.integers(len(live)))]
            model.fork(p, nxt)
            bm.fork(p, nxt)
            live.append(nxt)
            nxt += 1
        elif op == 2:
            s = live.pop(int(rng.integers(len(live))))
            model.free_seq(s)
            bm.free_seq(s)
        elif op == 3:
            batch = [live[int(i)] for i in rng.integers(0, len(live), size=min(6, len(live)))]
            batch = list(dict.fromkeys(batch))
            try:
                ms, mp = model.append_slots(batch)
            except ModelOOM:
                with pytest.raises(B.OutOfBlocks):
                    bm.append_slots(batch)
                continue
            slots, pairs = bm.append_slots(batch)
            assert slots.tolist() == ms
            assert [tuple(x) for x in pairs.tolist()] == mp
        else:
            s = live[int(rng.integers(len(live)))]
            try:
                m = model.append_slot(s)
            except ModelOOM:
                with pytest.raises(B.OutOfBlocks):
                    bm.append_slot(s)
                continue
            assert bm.append_slot(s) == m
        same_state(bm, model, live)


def test_fork_workload_copy_pattern():
    """16 prompts of 1024 tokens + 1 shared generated token, forked into 8 samples, then 32
    decode steps: the shared partial block is copied by 7 of 8 samples at step 1, never
    again; the parent's blocks are left to the last sample."""
    P, S8 = 16, 8
    NB = W.fork_pool_blocks()
    rng = np.random.default_rng(3)
    order = rng.permutation(NB)
    bm = B.BlockManager(NB, free_order=order)
    model = BlockManagerModel(NB, free_order=order)
    seqs = []
    for p in range(P):
        parent = p * S8
        bm.add_seq(parent, 1025)
        model.add_seq(parent, 1025)
        for k in range(1, S8):
            bm.fork(parent, parent + k)
            model.fork(parent, parent + k)
        seqs += [parent + k for k in range(S8)]
    shared = {p: model.block_table(p * S8) for p in range(P)}
    assert all(model.refcount(b) == 8 for t in shared.values() for b in t)
    total_pairs = []
    for step in range(32):
        slots, pairs = bm.append_slots(seqs)
        ms, mp = model.append_slots(seqs)
        assert slots.tolist() == ms and [tuple(x) for x in pairs.tolist()] == mp
        if step == 0:
            assert len(mp) == 7 * P
            assert all(src == shared[i // 7][-1] for i, (src, dst) in enumerate(mp))
        else:
            assert mp == []
        total_pairs += mp
    same_state(bm, model, seqs)
    for p in range(P):
        for b in shared[p][:-1]:
            assert model.refcount(b) == 8           # prompt blocks still shared by all
        assert model.refcount(shared[p][-1]) == 1   # the last sample kept the original
        assert model.block_table(p * S8 + 7)[64] == shared[p][-1]
    for s in seqs:
        assert model.seq_len(s) == 1057 and len(model.block_table(s)) == 67
    # pool: 1.1 x (65 shared + 7 copies + 8 x 2 private) per prompt
    assert NB == int(np.ceil(1.1 * 16 * 88))
    assert NB - bm.num_free() == 16 * 88


def test_errors_leave_state_unchanged():
    bm = B.BlockManager(4)
    with pytest.raises(B.OutOfBlocks):
        bm.add_seq(1, 100)
    assert bm.num_free() == 4 and bm.num_seqs() == 0
    bm.add_seq(1, 16 * 3)
    bm.add_seq(2, 16)
    before = (bm.free_order(), bm.block_table(1), bm.block_table(2))
    with pytest.raises(B.OutOfBlocks):
        bm.append_slots([1, 2])
    assert (bm.free_order(), bm.block_table(1), bm.block_table(2)) == before
    assert bm.seq_len(1) == 48 and bm.seq_len(2) == 16
    with pytest.raises(B.PkvError):
        bm.append_slot(99)
    with pytest.raises(B.PkvError):
        bm.fork(1, 2)
    with pytest.raises(B.PkvError):
        bm.refcount(4)
    with pytest.raises(B.PkvError):
        B.BlockManager(4, free_order=[0, 1, 1, 2])
    with pytest.raises(B.PkvError):
        B.BlockManager(4, block_size=24)


def test_packed_tables():
    bm = B.BlockManager(20)
    bm.add_seq(5, 20)
    bm.add_seq(6, 40)
    t, lens = bm.block_tables([6, 5], 4)
    assert t.tolist() == [[2, 3, 4, -1], [0, 1, -1, -1]] and lens.tolist() == [40, 20]
    with pytest.raises(B.PkvError):
        bm.block_tables([6], 2)


@pytest.mark.parametrize("seed", [0, 1])
def test_swap_traffic_matches_model(seed):
    """Swap-out / swap-in mixed with appends, forks and frees: bit-exact with the model."""
    rng = np.random.default_rng(100 + seed)
    NB, NH = 40, 30
    order, horder = rng.permutation(NB), rng.permutation(NH)
    bm = B.BlockManager(NB, free_order=order)
    bm.set_host_pool(NH, horder)
    model = BlockManagerModel(NB, free_order=order)
    model.set_host_pool(NH, horder)
    live, nxt = [], 0
    for _ in range(1500):
        op = int(rng.integers(0, 10))
        on_gpu = [s for s in live if not model.is_swapped(s)]
        swapped = [s for s in live if model.is_swapped(s)]
        if op == 0 or not live:
            act = "add"
        elif op == 1 and on_gpu:
            act = "fork"
        elif op == 2:
            act = "free"
        elif op == 3 and on_gpu:
            act = "out"
        elif op == 4 and swapped:
            act = "in"
        elif on_gpu:
            act = "append"
        else:
            act = "none"
        try:
            if act == "add":
                n = int(rng.integers(0, 60))
                model.add_seq(nxt, n)
                bm.add_seq(nxt, n)
                live.append(nxt)
                nxt += 1
            elif act == "fork":
                p = on_gpu[int(rng.integers(len(on_gpu)))]
                model.fork(p, nxt)
                bm.fork(p, nxt)
                live.append(nxt)
                nxt += 1
            elif act == "free":
                s = live.pop(int(rng.integers(len(live))))
                model.free_seq(s)
                bm.free_seq(s)
            elif act == "out":
                s = on_gpu[int(rng.integers(len(on_gpu)))]
                pairs = model.swap_out(s)
                assert [tuple(x) for x in bm.swap_out(s).tolist()] == pairs
            elif act == "in":
                s = swapped[int(rng.integers(len(swapped)))]
                pairs = model.swap_in(s)
                assert [tuple(x) for x in bm.swap_in(s).tolist()] == pairs
            elif act == "append":
                s = on_gpu[int(rng.integers(len(on_gpu)))]
                m = model.append_slot(s)
                assert bm.append_slot(s) == m
        except ModelOOM:
            # the product must refuse the same operation and stay unchanged
            call = {"add": lambda: bm.add_seq(nxt, n), "out": lambda: bm.swap_out(s),
                    "in": lambda: bm.swap_in(s), "append": lambda: bm.append_slot(s)}[act]
            with pytest.raises(B.OutOfBlocks):
                call()
            if live:
                s = live.pop(0)
                model.free_seq(s)
                bm.free_seq(s)
        assert bm.num_host_free() == len(model.host_free)
        same_state(bm, model, [s for s in live if not model.is_swapped(s)])
        for s in live:
            assert bm.is_swapped(s) == model.is_swapped(s)


def test_swapped_sequences_refuse_use():
    bm = B.BlockManager(8)
    bm.set_host_pool(8)
    bm.add_seq(1, 20)
    bm.swap_out(1)
    for call in (lambda: bm.append_slot(1), lambda: bm.fork(1, 2),
                 lambda: bm.block_tables([1], 4), lambda: bm.swap_out(1)):
        with pytest.raises(B.PkvError):
            call()
    assert bm.swap_in(1).shape == (2, 2)
    with pytest.raises(B.PkvError):
        bm.swap_in(1)
    bm.free_seq(1)
    assert bm.num_free() == 8 and bm.num_host_free() == 8


@pytest.mark.parametrize("name", ["beam", "prefix"])
def test_sharing_workloads_match_model(name):
    """Beam search and shared-prefix traffic: the product manager and the model build the
    same tables, slots and copy-on-write pairs; sharing saves blocks."""
    import bench
    wl, pairs = bench.build_workload(name)
    wl2, pairs2 = bench.build_workload(name, model_block_manager=True)
    assert np.array_equal(wl.block_tables, wl2.block_tables)
    assert np.array_equal(wl.slot_mapping, wl2.slot_mapping)
    assert np.array_equal(wl.context_lens, wl2.context_lens)
    assert np.array_equal(pairs, pairs2)
    sh = wl.extra["sharing"]
    assert sh == wl2.extra["sharing"]
    assert 0.3 < sh["saving"] < 0.95
    if name == "beam":
        assert len(pairs) > 0        # the decode step's token lands in shared partial blocks
