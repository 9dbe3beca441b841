"""Pins for the block-manager model (oracle/block_manager.py) against the pages' rules and
worked examples."""
import json
import os

import numpy as np
import pytest

from oracle.block_manager import BlockManagerModel, OutOfBlocks

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_pages_waste_examples():
    with open(os.path.join(GOLDEN, "waste_examples.json")) as f:
        g = json.load(f)
    for c in g["cases"]:
        assert c["contiguous_reserved"] - c["tokens"] == c["contiguous_wasted"]
        bm = BlockManagerModel(200, g["block_size"])
        bm.add_seq("a", 0)
        for _ in range(c["tokens"]):          # on-demand: one slot per generated token
            bm.append_slot("a")
        assert len(bm.block_table("a")) == c["paged_blocks"]
        assert len(bm.block_table("a")) * g["block_size"] == c["paged_slots"]
        assert bm.waste("a") == c["paged_wasted"]
        assert bm.num_free() == 200 - c["paged_blocks"]


def test_on_demand_allocation_only_at_block_boundaries():
    bm = BlockManagerModel(10, 16, free_order=[3, 1, 4, 0, 5, 9, 2, 6, 8, 7])
    bm.add_seq(0, 0)
    slots = [bm.append_slot(0)[0] for _ in range(40)]
    assert bm.block_table(0) == [3, 1, 4]
    assert slots == [3 * 16 + i for i in range(16)] + [1 * 16 + i for i in range(16)] + \
        [4 * 16 + i for i in range(8)]
    assert bm.waste(0) == 8


def test_fork_shares_blocks_and_copy_on_write_follows_refcount():
    bm = BlockManagerModel(40, 16)
    bm.add_seq("p", 20)                       # blocks 0, 1 (block 1 holds 4 tokens)
    for c in range(1, 4):
        bm.fork("p", c)
    assert [bm.refcount(b) for b in (0, 1)] == [4, 4]
    pairs = []
    for s in ("p", 1, 2, 3):
        slot, cow = bm.append_slot(s)
        pairs.append(cow)
    # the first three holders see refcount > 1 and copy; the last sees 1 and writes in place
    assert pairs == [(1, 2), (1, 3), (1, 4), None]
    assert bm.block_table("p") == [0, 2] and bm.block_table(3) == [0, 1]
    assert [bm.refcount(b) for b in range(5)] == [4, 1, 1, 1, 1]
    # appends that stay in a now-private block never copy again
    for s in ("p", 1, 2, 3):
        assert bm.append_slot(s)[1] is None


def test_fork_at_block_boundary_needs_no_copy():
    bm = BlockManagerModel(20, 16)
    bm.add_seq(0, 32)
    bm.fork(0, 1)
    _, c0 = bm.append_slot(0)
    _, c1 = bm.append_slot(1)
    assert c0 is None and c1 is None and bm.block_table(0)[:2] == bm.block_table(1)[:2]


def test_free_returns_blocks_fifo_when_refcount_reaches_zero():
    bm = BlockManagerModel(6, 16)
    bm.add_seq("a", 33)                       # 0, 1, 2
    bm.fork("a", "b")
    bm.free_seq("a")
    assert bm.free_order() == [3, 4, 5]
    bm.free_seq("b")
    assert bm.free_order() == [3, 4, 5, 0, 1, 2]
    assert all(bm.refcount(b) == 0 for b in range(6))


def test_out_of_blocks_changes_nothing():
    bm = BlockManagerModel(3, 16)
    with pytest.raises(OutOfBlocks):
        bm.add_seq(0, 64)
    assert bm.num_free() == 3 and 0 not in bm.tables
    bm.add_seq(0, 32)
    bm.add_seq(1, 16)
    state = (list(bm.free), list(bm.ref), {k: list(v) for k, v in bm.tables.items()},
             dict(bm.lens))
    with pytest.raises(OutOfBlocks):
        bm.append_slots([0, 1])
    assert state == (list(bm.free), list(bm.ref), {k: list(v) for k, v in bm.tables.items()},
                     dict(bm.lens))


@pytest.mark.parametrize("B", [16, 32])
def test_random_traffic_invariants(B):
    rng = np.random.default_rng(7)
    NB = 64
    bm = BlockManagerModel(NB, B, free_order=rng.permutation(NB))
    live, nxt = [], 0
    for step in range(3000):
        op = rng.integers(0, 10)
        try:
            if op == 0 or not live:
                bm.add_seq(nxt, int(rng.integers(0, 40)))
                live.append(nxt)
                nxt += 1
            elif op == 1:
                bm.fork(live[int(rng.integers(len(live)))], nxt)
                live.append(nxt)
                nxt += 1
            elif op == 2:
                s = live.pop(int(rng.integers(len(live))))
                bm.free_seq(s)
            else:
                bm.append_slot(live[int(rng.integers(len(live)))])
        except OutOfBlocks:
            s = live.pop(0)
            bm.free_seq(s)
        # reference counts equal the number of table entries naming each block
        count = [0] * NB
        for s in live:
            for b in bm.block_table(s):
                count[b] += 1
        assert count == bm.ref
        # free blocks are exactly the unreferenced ones; nothing is lost or duplicated
        assert sorted(bm.free_order()) == [b for b in range(NB) if count[b] == 0]
        # only the last block of a sequence is partly empty
        for s in live:
            assert 0 <= bm.waste(s) < B or bm.seq_len(s) == 0


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_swap_fork_cow_traffic_keeps_every_sequence_readable(seed):
    """Data-level pin of fork, copy-on-write and swap: device and host memory are simulated
    cell by cell, the model's copy pairs and slots are applied as a caller would, and every
    live sequence must read back exactly the tokens it holds, through its own table, from
    the pool it lives in."""
    rng = np.random.default_rng(300 + seed)
    NB, NH, B = 40, 30, 16
    bm = BlockManagerModel(NB, B, free_order=rng.permutation(NB))
    bm.set_host_pool(NH, rng.permutation(NH))
    dev = [[None] * B for _ in range(NB)]
    host = [[None] * B for _ in range(NH)]
    want, nxt = {}, 0          # seq -> list of token labels it holds

    def write(seq, slot):
        dev[slot // B][slot % B] = (seq, len(want[seq]))
        want[seq].append((seq, len(want[seq])))

    for _ in range(2500):
        live = list(want)
        on_gpu = [s for s in live if not bm.is_swapped(s)]
        off = [s for s in live if bm.is_swapped(s)]
        op = int(rng.integers(0, 10))
        try:
            if op == 0 or not live:
                n = int(rng.integers(0, 50))
                bm.add_seq(nxt, n)
                want[nxt] = []
                tbl = bm.block_table(nxt)
                for t in range(n):
                    write(nxt, tbl[t // B] * B + t % B)
                nxt += 1
            elif op == 1 and on_gpu:
                p = on_gpu[int(rng.integers(len(on_gpu)))]
                bm.fork(p, nxt)
                want[nxt] = list(want[p])
                nxt += 1
            elif op == 2:
                s = live[int(rng.integers(len(live)))]
                bm.free_seq(s)
                del want[s]
            elif op == 3 and on_gpu:
                s = on_gpu[int(rng.integers(len(on_gpu)))]
                for g, h in bm.swap_out(s):
                    host[h] = list(dev[g])
            elif op == 4 and off:
                s = off[int(rng.integers(len(off)))]
                for h, g in bm.swap_in(s):
                    dev[g] = list(host[h])
            elif on_gpu:
                s = on_gpu[int(rng.integers(len(on_gpu)))]
                slot, cow = bm.append_slot(s)
                if cow is not None:
                    dev[cow[1]] = list(dev[cow[0]])
                write(s, slot)
        except OutOfBlocks:
            s = live[0]
            bm.free_seq(s)
            del want[s]
        for s, toks in want.items():
            mem = host if bm.is_swapped(s) else dev
            tbl = bm.block_table(s)
            assert bm.seq_len(s) == len(toks)
            assert [mem[tbl[t // B]][t % B] for t in range(len(toks))] == toks
        # host blocks are never shared: each belongs to one swapped sequence or is free
        held = [h for s in want if bm.is_swapped(s) for h in bm.block_table(s)]
        assert sorted(held + list(bm.host_free_order())) == list(range(NH))


def _planted(name):
    """A copy of the model class with one plausible mistake in its swap or fork logic."""
    class Mutant(BlockManagerModel):
        pass

    if name == "swap_out frees shared blocks":
        def swap_out(self, seq):
            table = self.tables[seq]
            if len(table) > len(self.host_free):
                raise OutOfBlocks("host pool exhausted")
            pairs = []
            for j, blk in enumerate(table):
                h = self.host_free.popleft()
                pairs.append((blk, h))
                if self.ref[blk] > 0:             # drops every holder, not just this one
                    self.ref[blk] = 0
                    self.free.append(blk)
                table[j] = h
            self.swapped.add(seq)
            return pairs
        Mutant.swap_out = swap_out
    elif name == "swap_in pairs rotated":
        orig = BlockManagerModel.swap_in

        def swap_in(self, seq):
            p = orig(self, seq)
            return [(p[(i + 1) % len(p)][0], g) for i, (_, g) in enumerate(p)]
        Mutant.swap_in = swap_in
    elif name == "fork shares without a reference":
        def fork(self, parent, child):
            if parent in self.swapped:
                raise ValueError("parent is swapped out")
            self.tables[child] = list(self.tables[parent])
            self.lens[child] = self.lens[parent]     # refcounts not raised
        Mutant.fork = fork
    return Mutant


@pytest.mark.parametrize("name", ["swap_out frees shared blocks", "swap_in pairs rotated",
                                  "fork shares without a reference"])
def test_planted_mistakes_fail_the_data_level_pin(name, monkeypatch):
    import sys
    mod = sys.modules[__name__]
    monkeypatch.setattr(mod, "BlockManagerModel", _planted(name))
    failed = 0
    for seed in (0, 1, 2):
        try:
            test_swap_fork_cow_traffic_keeps_every_sequence_readable(seed)
        except (AssertionError, KeyError, ValueError, IndexError, TypeError):
            failed += 1
    assert failed > 0, name
