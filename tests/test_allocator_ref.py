"""Pins of the reference block manager against the pages' behavioural statements.

Glossary entry "PagedAttention" (ultralytics.com): a new block only when the
previous one is full, from any free location; sharing with reference counts;
copy-on-write before writing a block others use; finished sequences return
their blocks at once.  iplexlaw.co.kr blog ("two answers to one request"): full
shared blocks stay shared, only the block that must split is copied; blocks
without references are freed.  "Le cache KV et PagedAttention" (gyaansetu.com):
pages, not whole sequences, move to the CPU when memory is short and come back
later.  The waste bound (less than one block per
sequence) is the glossary's "only the unfilled part of the last block".
"""
import numpy as np
import pytest

from oracle import RefBlockManager


def _check_invariants(bm):
    refs = [0] * bm.num_blocks
    for s, t in bm.tables.items():
        if s in bm.swapped:
            continue
        for b in t:
            refs[b] += 1
    assert refs == bm.ref                          # counts equal table references
    host_used = [h for s in bm.swapped for h in bm.tables[s]]
    assert len(set(host_used)) == len(host_used)   # a host block holds one page
    assert not set(host_used) & set(bm.host_free)
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


# -- swap to a host pool ---------------------------------------------------------

def _fill(pool_k, pool_v, bm, seq, rng):
    """Give every slot of a sequence distinct contents (written through its slots)."""
    for pos in range(bm.lens[seq]):
        slot = bm.slot(seq, pos)
        b, o = divmod(slot, bm.block_size)
        pool_k[b, o] = rng.standard_normal(pool_k.shape[2:])
        pool_v[b, o] = rng.standard_normal(pool_v.shape[2:])


def _logical(pool, bm, seq):
    return np.stack([pool[divmod(bm.slot(seq, p), bm.block_size)] for p in range(bm.lens[seq])])


def test_swap_round_trip_restores_every_token():
    """Pages go to the host and back; the logical sequence is unchanged although
    its device blocks are new and the old ones were reused in between."""
    import oracle
    rng = np.random.default_rng(7)
    NB, NH, shape = 24, 12, (16, 2, 8)
    dk, dv = np.zeros((NB,) + shape), np.zeros((NB,) + shape)
    hk, hv = np.zeros((NH,) + shape), np.zeros((NH,) + shape)
    bm = RefBlockManager(NB, 16)
    bm.set_host_pool(NH)
    a, b = bm.alloc_seq(70), bm.alloc_seq(40)          # 5 + 3 blocks
    _fill(dk, dv, bm, a, rng)
    _fill(dk, dv, bm, b, rng)
    want_k, want_v = _logical(dk, bm, a), _logical(dv, bm, a)
    old_table = list(bm.tables[a])
    free_before = bm.num_free()
    out = bm.swap_out(a)
    assert [d for d, _ in out] == old_table and [h for _, h in out] == [0, 1, 2, 3, 4]
    assert bm.num_free() == free_before + 5 and list(bm.host_free) == list(range(5, NH))
    assert oracle.swap_blocks(hk, hv, dk, dv, out) == 0
    c = bm.alloc_seq(bm.num_free() * 16)                # takes every free block, a's old ones too
    assert set(bm.tables[c]) & set(old_table)
    _fill(dk, dv, bm, c, rng)                           # overwrite them
    bm.free_seq(c)
    back = bm.swap_in(a)
    assert [h for h, _ in back] == [0, 1, 2, 3, 4]
    assert oracle.swap_blocks(dk, dv, hk, hv, back) == 0
    assert bm.tables[a] == [d for _, d in back]
    assert np.array_equal(_logical(dk, bm, a), want_k) and np.array_equal(_logical(dv, bm, a), want_v)
    assert list(bm.host_free) == list(range(5, NH)) + [0, 1, 2, 3, 4]
    _check_invariants(bm)


def test_swap_out_of_a_shared_prefix_keeps_the_other_copy():
    bm = RefBlockManager(16, 16)
    bm.set_host_pool(8)
    p = bm.alloc_seq(40)                                # blocks 0, 1, 2
    c = bm.fork(p)
    pairs = bm.swap_out(c)
    assert pairs == [(0, 0), (1, 1), (2, 2)]
    assert bm.ref[:3] == [1, 1, 1] and bm.num_free() == 13   # parent still holds them
    back = bm.swap_in(c)
    assert [d for _, d in back] == [3, 4, 5]            # private copies, sharing not restored
    assert bm.ref[:6] == [1] * 6
    _check_invariants(bm)


def test_swap_without_room_changes_nothing():
    bm = RefBlockManager(8, 16)
    bm.set_host_pool(2)
    a = bm.alloc_seq(48)                                # 3 blocks > 2 host blocks
    state = (list(bm.free), list(bm.ref), list(bm.tables[a]), list(bm.host_free))
    with pytest.raises(MemoryError):
        bm.swap_out(a)
    assert state == (list(bm.free), list(bm.ref), list(bm.tables[a]), list(bm.host_free))
    bm.set_host_pool(4)
    bm.swap_out(a)
    b = bm.alloc_seq(8 * 16 - 16)                       # leaves 1 device block free
    with pytest.raises(MemoryError):
        bm.swap_in(a)
    assert a in bm.swapped and bm.num_free() == 1
    bm.free_seq(a)                                      # a swapped sequence frees host blocks
    assert sorted(bm.host_free) == [0, 1, 2, 3] and not bm.swapped
    bm.free_seq(b)
    _check_invariants(bm)


def test_random_trace_with_swaps_invariants():
    rng = np.random.default_rng(3)
    bm = RefBlockManager(200, 16)
    bm.set_host_pool(150)
    live = []
    for step in range(3000):
        op = rng.integers(0, 12)
        try:
            if op == 0 or not live:
                live.append(bm.alloc_seq(int(rng.integers(0, 60))))
            elif op == 1:
                s = live[rng.integers(len(live))]
                if s not in bm.swapped:
                    live.append(bm.fork(s))
            elif op == 2 and len(live) > 1:
                bm.free_seq(live.pop(rng.integers(len(live))))
            elif op == 3:
                s = live[rng.integers(len(live))]
                (bm.swap_in if s in bm.swapped else bm.swap_out)(s)
            else:
                s = live[rng.integers(len(live))]
                if s not in bm.swapped:
                    bm.append_token(s)
        except MemoryError:
            pass
        if step % 100 == 0:
            _check_invariants(bm)
            used = sum(1 for r in bm.ref if r > 0)
            assert used + bm.num_free() == bm.num_blocks
            host_used = sum(len(bm.tables[s]) for s in bm.swapped)
            assert host_used + len(bm.host_free) == 150
    _check_invariants(bm)


# -- shared-prefix groups -----------------------------------------------------------

def test_prefix_groups_of_parallel_samples():
    """Parallel sampling shares the prompt's blocks (glossary entry, sharing
    section): the three samples form one group over the prompt's full blocks;
    the partly filled block does not count, and neither does a lone sequence."""
    bm = RefBlockManager(32, 16)
    lone = bm.alloc_seq(50)                       # blocks 0..3
    p = bm.alloc_seq(40)                          # blocks 4, 5, 6 (6 holds 8 tokens)
    kids = [bm.fork(p), bm.fork(p)]
    short = bm.alloc_seq(9)                       # block 7: no full block
    assert bm.prefix_groups([lone, p] + kids + [short]) == ([0, 3], [1, 2, 3], [2])
    bm.append_token(kids[0])                      # copy-on-write of block 6
    for _ in range(30):
        bm.append_token(p)                        # p fills block 6 and takes another
    assert bm.prefix_groups([kids[1], lone, p, kids[0]]) == ([0, 3], [0, 2, 3], [2])
    # a second family after the first, members in batch order
    q = bm.alloc_seq(33)
    qk = bm.fork(q)
    assert bm.prefix_groups([q, p, qk, kids[0]]) == ([0, 2, 4], [0, 2, 1, 3], [2, 2])


def test_prefix_groups_stop_at_first_different_block():
    bm = RefBlockManager(64, 16)
    a = bm.alloc_seq(64)                          # 4 full blocks
    b = bm.fork(a)
    c = bm.fork(a)
    # give b a different third block by hand (as a later copy-on-write would)
    bm.ref[bm.tables[b][2]] -= 1
    bm.tables[b][2] = bm._pop()
    assert bm.prefix_groups([a, b, c]) == ([0, 3], [0, 1, 2], [2])
    assert bm.prefix_groups([a, c]) == ([0, 2], [0, 1], [4])
