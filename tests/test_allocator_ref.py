"""Pins of the reference block manager against the pages' behavioural statements.

Glossary entry "PagedAttention" (ultralytics.com): a new block only when the
previous one is full, from any free location; sharing with reference counts;
copy-on-write before writing a block others use; finished sequences return
their blocks at once.  iplexlaw.co.kr blog ("two answers to one request"): full
shared blocks stay shared, only the block that must split is copied; blocks
without references are freed.  The waste bound (less than one block per
sequence) is the glossary's "only the unfilled part of the last block".
"""
import numpy as np
import pytest

from oracle import RefBlockManager


def _check_invariants(bm):
    refs = [0] * bm.num_blocks
    for t in bm.tables.values():
        for b in t:
            refs[b] += 1
    assert refs == bm.ref                          # counts equal table references
    free = set(bm.free)
    assert len(free) == len(bm.free)
    assert all(bm.ref[b] == 0 for b in free)       # a free block has no reference
    for s, t in bm.tables.items():                 # waste < one block per sequence
        assert len(t) == -(-bm.lens[s] // bm.block_size)


def test_fifo_and_lazy_growth():
    bm = RefBlockManager(10, 4, free_order=[5, 3, 9, 0, 1, 2, 4, 6, 7, 8])
    s = bm.alloc_seq(5)
    assert bm.tables[s] == [5, 3]
    slots = []
    for _ in range(3):                             # fills positions 5, 6, 7 of block 3
        slot, cow = bm.append_token(s)
        assert cow is None
        slots.append(slot)
    assert slots == [3 * 4 + 1, 3 * 4 + 2, 3 * 4 + 3] and bm.tables[s] == [5, 3]
    slot, cow = bm.append_token(s)                 # block full -> next free block, slot 0
    assert bm.tables[s] == [5, 3, 9] and slot == 9 * 4 and cow is None
    _check_invariants(bm)


def test_parallel_sampling_cow_trace():
    """n=3 samples of one prompt whose last block is partly filled: the first two
    writers copy it, the last holder writes in place; full blocks stay shared."""
    bs = 16
    bm = RefBlockManager(20, bs)
    p = bm.alloc_seq(40)                           # blocks 0, 1 full; block 2 holds 8 tokens
    kids = [bm.fork(p), bm.fork(p)]
    assert bm.ref[0] == bm.ref[1] == bm.ref[2] == 3
    events = [bm.append_token(s) for s in [p] + kids]
    cows = [c for _, c in events]
    assert cows[0] == (2, 3) and cows[1] == (2, 4) and cows[2] is None
    assert [s for s, _ in events] == [3 * bs + 8, 4 * bs + 8, 2 * bs + 8]
    assert bm.ref[0] == bm.ref[1] == 3             # full shared blocks never copied
    assert bm.ref[2] == 1 and bm.ref[3] == 1 and bm.ref[4] == 1
    _check_invariants(bm)
    # full shared prefix: appending allocates a fresh block, no copy
    q = bm.alloc_seq(32)
    k = bm.fork(q)
    slot, cow = bm.append_token(k)
    assert cow is None and bm.tables[k][:2] == bm.tables[q][:2] and len(bm.tables[k]) == 3
    _check_invariants(bm)


def test_free_on_zero_and_immediate_return():
    bm = RefBlockManager(8, 16)
    p = bm.alloc_seq(20)
    c = bm.fork(p)
    before = bm.num_free()
    bm.free_seq(p)                                 # still referenced by the child
    assert bm.num_free() == before
    bm.free_seq(c)                                 # now both blocks return, in table order
    assert bm.num_free() == 8 and list(bm.free)[-2:] == [0, 1]
    _check_invariants(bm)


def test_out_of_blocks_leaves_state_unchanged():
    bm = RefBlockManager(3, 16)
    s = bm.alloc_seq(30)
    with pytest.raises(MemoryError):
        bm.alloc_seq(40)
    assert bm.num_free() == 1 and list(bm.tables) == [s]
    t = bm.fork(s)
    u = bm.fork(s)
    bm.append_token(s)                             # copy-on-write takes the last free block
    with pytest.raises(MemoryError):
        bm.append_token(t)                         # block still shared by t and u: needs a copy
    assert bm.lens[t] == 30 and bm.ref[bm.tables[t][-1]] == 2
    bm.free_seq(u)
    slot, cow = bm.append_token(t)                 # now the last holder: writes in place
    assert cow is None
    _check_invariants(bm)


def test_random_trace_invariants():
    rng = np.random.default_rng(0)
    bm = RefBlockManager(400, 16)
    live = []
    for step in range(3000):
        op = rng.integers(0, 10)
        try:
            if op == 0 or not live:
                live.append(bm.alloc_seq(int(rng.integers(0, 60))))
            elif op == 1:
                live.append(bm.fork(live[rng.integers(len(live))]))
            elif op == 2 and len(live) > 1:
                bm.free_seq(live.pop(rng.integers(len(live))))
            else:
                bm.append_token(live[rng.integers(len(live))])
        except MemoryError:
            pass
        if step % 100 == 0:
            _check_invariants(bm)
            used = sum(1 for r in bm.ref if r > 0)
            assert used + bm.num_free() == bm.num_blocks
    _check_invariants(bm)
