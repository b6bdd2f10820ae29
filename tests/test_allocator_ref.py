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


# -- prefix caching across requests (full-block keys) --------------------------------

def _cached_bm(nb=32):
    bm = RefBlockManager(nb, 16)
    bm.set_prefix_cache(True)
    return bm


SYS = list(range(1000, 1040))        # a 40-token system prompt: 2 full blocks + 8 tokens


def test_same_system_prompt_reuses_full_blocks():
    """Glossary entry: requests that start with the same system prompt share one
    copy of it; hashing whole blocks extends sharing across requests."""
    bm = _cached_bm()
    a, ca = bm.alloc_seq_tokens(SYS + [1, 2, 3])
    b, cb = bm.alloc_seq_tokens(SYS + [7, 8])
    assert (ca, cb) == (0, 32)
    assert bm.tables[a] == [0, 1, 2] and bm.tables[b] == [0, 1, 3]   # the 8-token tail is not shared
    assert bm.ref[:4] == [2, 2, 1, 1]
    c, cc = bm.alloc_seq_tokens(SYS[:16] + [5] * 30)                   # differs inside block 1
    assert cc == 16 and bm.tables[c] == [0, 4, 5] and bm.ref[0] == 3
    _check_invariants(bm)


def test_two_requests_share_their_common_system_prompt_block():
    """Worked by hand from the glossary entry's sharing section: requests that
    start with the same system prompt reuse one copy of it, each block counted
    by a reference counter, and hashing whole blocks is what carries the sharing
    from one request to the next.  Free list as in the worked example:
    [41, 7, 19, 2, 33], then 11 and 5 (no other block of the 64 is free).
      A = S + U1 + 5 tokens   -> no hit, blocks [41, 7, 19]
      B = S + U2 + 3 tokens   -> S hits 41 (16 tokens), U2 misses: [41, 2, 33]
      D = U1 + S              -> no hit: U1 at the start is not A's second block
                                 (its keys and values follow S there): [11, 5]
      A freed                 -> 41 keeps B's reference; 7 (full, keyed) and 19
                                 go to the back of the free list: [7, 19]
      E = S + U1 + 1 token    -> hits 41 and 7 (taken back out of the free
                                 list), 32 tokens; its tail gets 19: [41, 7, 19]"""
    S, U1, U2 = list(range(100, 116)), list(range(200, 216)), list(range(300, 316))
    bm = RefBlockManager(64, 16, free_order=[41, 7, 19, 2, 33, 11, 5])
    bm.set_prefix_cache(True)
    a, ca = bm.alloc_seq_tokens(S + U1 + [1] * 5)
    assert (bm.tables[a], ca) == ([41, 7, 19], 0)
    b, cb = bm.alloc_seq_tokens(S + U2 + [2] * 3)
    assert (bm.tables[b], cb) == ([41, 2, 33], 16)
    assert [bm.ref[x] for x in (41, 7, 19, 2, 33)] == [2, 1, 1, 1, 1]
    d, cd = bm.alloc_seq_tokens(U1 + S)
    assert (bm.tables[d], cd) == ([11, 5], 0)
    assert bm.ref[7] == 1 and list(bm.free) == []
    bm.free_seq(a)
    assert list(bm.free) == [7, 19] and [bm.ref[x] for x in (41, 7, 19)] == [1, 0, 0]
    e, ce = bm.alloc_seq_tokens(S + U1 + [3])
    assert (bm.tables[e], ce) == ([41, 7, 19], 32)
    assert [bm.ref[x] for x in (41, 7, 19, 2, 33, 11, 5)] == [2, 1, 1, 1, 1, 1, 1]
    assert list(bm.free) == []
    _check_invariants(bm)


def test_a_block_is_keyed_by_its_whole_prefix():
    """The same 16 tokens after a different first block are a different block."""
    bm = _cached_bm()
    x, y, z = [1] * 16, [2] * 16, [3] * 16
    a, _ = bm.alloc_seq_tokens(x + y)
    b, cb = bm.alloc_seq_tokens(z + y)
    assert cb == 0 and set(bm.tables[a]).isdisjoint(bm.tables[b])
    c, cc = bm.alloc_seq_tokens(x + y + z)
    assert cc == 32 and bm.tables[c][:2] == bm.tables[a]


def test_released_blocks_stay_cached_until_reused():
    bm = _cached_bm(8)
    a, _ = bm.alloc_seq_tokens(SYS)                      # blocks 0, 1, 2
    bm.free_seq(a)
    assert list(bm.free) == [3, 4, 5, 6, 7, 0, 1, 2]
    b, cb = bm.alloc_seq_tokens(SYS[:32] + [9] * 4)      # hits 0, 1 out of the free list
    assert cb == 32 and bm.tables[b] == [0, 1, 3]
    assert list(bm.free) == [4, 5, 6, 7, 2]
    bm.free_seq(b)
    # a large request takes every free block, in order: the cached ones lose their keys
    c = bm.alloc_seq(8 * 16)
    assert bm.tables[c] == [4, 5, 6, 7, 2, 0, 1, 3] and not bm.cache
    bm.free_seq(c)
    d, cd = bm.alloc_seq_tokens(SYS)
    assert cd == 0
    _check_invariants(bm)


def test_reused_parent_does_not_revive_stale_children():
    """Block P held prompt A's first block, then was reused for prompt B's; a
    prompt made of B's first block and A's second must not hit A's second block."""
    bm = _cached_bm(4)
    a0, a1, b0 = [1] * 16, [2] * 16, [3] * 16
    a, _ = bm.alloc_seq_tokens(a0 + a1)                  # blocks 0 (a0), 1 (a1)
    bm.free_seq(a)                                       # free list [2, 3, 0, 1], both cached
    filler = bm.alloc_seq(32)                            # takes 2, 3
    b, _ = bm.alloc_seq_tokens(b0)                       # takes 0: a0's key dropped, b0 registered
    assert bm.tables[b] == [0]
    c, cc = bm.alloc_seq_tokens(b0 + a1)
    assert cc == 16 and bm.tables[c] == [0, 1]           # block 1 is not a hit ...
    assert bm.ref[1] == 1                                # ... it was taken from the free list as new
    bm.free_seq(filler)
    _check_invariants(bm)


def test_out_of_blocks_with_cache_changes_nothing():
    bm = _cached_bm(4)
    a, _ = bm.alloc_seq_tokens(SYS)                      # 0, 1, 2
    bm.free_seq(a)
    b = bm.alloc_seq(16)                                 # takes 3
    state = (list(bm.free), list(bm.ref), dict(bm.cache))
    with pytest.raises(MemoryError):
        bm.alloc_seq_tokens(SYS + [0] * 9)               # 2 hits to wake + 2 new > 3 free
    assert state == (list(bm.free), list(bm.ref), dict(bm.cache))
    bm.free_seq(b)


def test_prefix_cache_hits_hold_the_right_tokens():
    """Requests over a few system prompts, released and reallocated at random;
    each request writes only its uncached tokens, yet reading any live request
    back through its table gives its whole logical token stream (content is a
    function of (prefix, position), as a transformer's K/V is)."""
    import oracle
    rng = np.random.default_rng(8)
    NB = 40
    bm = _cached_bm(NB)
    pool = np.full((NB, 16, 1, 4), -1.0, dtype=np.float32)
    systems = [rng.integers(0, 9, size=n).tolist() for n in (37, 64, 20)]

    def content(tokens):
        # row of position i: (hash of the tokens up to i, i, token, 0)
        h, rows = 0, []
        for i, t in enumerate(tokens):
            h = (h * 131 + t + 1) % 1000003
            rows.append([h, i, t, 0])
        return np.asarray(rows, dtype=np.float32).reshape(-1, 1, 4)

    live = {}
    for step in range(300):
        if live and (rng.random() < 0.4 or bm.num_free() < 8):
            s = list(live)[int(rng.integers(len(live)))]
            bm.free_seq(s)
            del live[s]
            continue
        toks = systems[int(rng.integers(3))] + rng.integers(0, 9, size=int(rng.integers(0, 30))).tolist()
        try:
            s, cached = bm.alloc_seq_tokens(toks)
        except MemoryError:
            continue
        assert cached % 16 == 0 and cached <= len(toks)
        rows = content(toks)
        slots = bm.slots(s, cached, len(toks) - cached)
        oracle.kv_write(rows[cached:], rows[cached:], oracle.F32, np.asarray(slots, np.int64), pool, pool.copy(),
                        oracle.F32, 16)
        live[s] = toks
        for q, qt in live.items():
            got = oracle.gather(pool, bm.tables[q], len(qt), 16)
            assert np.array_equal(got, content(qt)), "request %d reads wrong tokens" % q
    _check_invariants(bm)


def test_evicted_prefix_is_not_served_from_overwritten_blocks():
    """A cached prompt whose blocks were handed out for other data must miss:
    reading it back gives its own tokens, written again."""
    import oracle
    bm = _cached_bm(6)
    pool = np.zeros((6, 16, 1, 1), dtype=np.float32)

    def put(tokens):
        s, cached = bm.alloc_seq_tokens(tokens)
        rows = np.asarray(tokens, dtype=np.float32).reshape(-1, 1, 1)
        slots = np.asarray(bm.slots(s, cached, len(tokens) - cached), np.int64)
        oracle.kv_write(rows[cached:], rows[cached:], oracle.F32, slots, pool, pool.copy(), oracle.F32, 16)
        return s, cached

    x = list(range(1, 49))                              # 3 full blocks
    a, _ = put(x)
    bm.free_seq(a)
    other, _ = put([7] * 96)                            # takes all 6 blocks, x's included
    bm.free_seq(other)
    b, cached = put(x)
    assert cached == 0
    assert oracle.gather(pool, bm.tables[b], 48, 16).ravel().tolist() == x
