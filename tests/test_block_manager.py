"""Parity of the native C++ block manager with the oracle's reference manager
(CPU only; integer work, compared exactly)."""
import json
import os

import numpy as np
import pytest

from oracle import RefBlockManager


@pytest.fixture(scope="module")
def BM():
    from paged_kv_cache_404_b200 import build
    build.build()
    from paged_kv_cache_404_b200 import BlockManager
    return BlockManager


def test_worked_example(BM, golden_dir):
    g = json.load(open(os.path.join(golden_dir, "worked_example.json")))
    bm = BM(g["pool_blocks"], g["block_size"], free_order=g["free_blocks"])
    s = bm.alloc_seq(g["num_tokens"])
    assert bm.block_table(s).tolist() == g["expected_block_table"]
    assert bm.free_list().tolist() == g["expected_free_after"]
    slots = bm.slots(s, 0, g["num_tokens"])
    assert slots[0] == 41 * 16 and slots[16] == 7 * 16 and slots[39] == 19 * 16 + 7
    assert len(bm.block_table(s)) * g["block_size"] - g["num_tokens"] == g["unused_slots_paged"]


def _same_state(bm, ref, live):
    assert bm.free_list().tolist() == list(ref.free)
    for s in live:
        assert bm.block_table(s).tolist() == ref.tables[s]
        assert bm.seq_len(s) == ref.lens[s]
        assert bm.is_swapped(s) == (s in ref.swapped)
    for b in range(ref.num_blocks):
        assert bm.refcount(b) == ref.ref[b]
    assert bm.num_free_host() == len(ref.host_free)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_random_traces_match_reference(BM, seed):
    rng = np.random.default_rng(seed)
    NB = 300
    order = rng.permutation(NB)
    bm, ref = BM(NB, 16, free_order=order), RefBlockManager(NB, 16, free_order=order)
    live = []
    for step in range(2500):
        op = int(rng.integers(0, 10))
        if op == 0 or not live:
            n = int(rng.integers(0, 70))
            try:
                r = ref.alloc_seq(n)
            except MemoryError:
                with pytest.raises(Exception):
                    bm.alloc_seq(n)
                continue
            assert bm.alloc_seq(n) == r
            live.append(r)
        elif op == 1:
            p = live[int(rng.integers(len(live)))]
            r = ref.fork(p)
            assert bm.fork(p) == r
            live.append(r)
        elif op == 2 and len(live) > 1:
            s = live.pop(int(rng.integers(len(live))))
            ref.free_seq(s)
            bm.free_seq(s)
        else:
            k = int(rng.integers(1, 6))
            seqs = [live[int(rng.integers(len(live)))] for _ in range(k)]
            seqs = list(dict.fromkeys(seqs))
            exp_slots, exp_pairs = [], []
            ok = True
            for s in seqs:
                try:
                    slot, cow = ref.append_token(s)
                except MemoryError:
                    ok = False
                    break
                exp_slots.append(slot)
                if cow:
                    exp_pairs.append(cow)
            if not ok:
                # the reference raised part-way; replay the successful prefix on the native side
                done = len(exp_slots)
                if done:
                    slots, pairs = bm.append_tokens(seqs[:done])
                    assert slots.tolist() == exp_slots
                with pytest.raises(Exception):
                    bm.append_tokens(seqs[done:done + 1])
                continue
            slots, pairs = bm.append_tokens(seqs)
            assert slots.tolist() == exp_slots
            assert [tuple(p) for p in pairs.tolist()] == exp_pairs
        if step % 250 == 0:
            _same_state(bm, ref, live)
    _same_state(bm, ref, live)


def test_parallel_sampling_trace(BM):
    bm = BM(64, 16)
    p = bm.alloc_seq(1000 % 64 + 40)          # 40 + 40 = 80 tokens: 5 blocks, last one full
    q = bm.alloc_seq(40)                      # 3 blocks, last holds 8
    kids = [bm.fork(q), bm.fork(q)]
    slots, pairs = bm.append_tokens([q] + kids + [p])
    assert [tuple(x) for x in pairs.tolist()] == [(7, 8), (7, 9)]
    assert bm.refcount(7) == 1 and bm.refcount(5) == 3 and bm.refcount(6) == 3
    assert slots[2] == 7 * 16 + 8             # the last holder writes in place
    assert slots[3] == 10 * 16                # full last block: next free block


def test_errors(BM):
    from paged_kv_cache_404_b200 import PagedKVError
    bm = BM(2, 16)
    with pytest.raises(PagedKVError):
        bm.alloc_seq(40)
    with pytest.raises(PagedKVError):
        bm.fork(7)
    with pytest.raises(PagedKVError):
        bm.free_seq(3)
    with pytest.raises(PagedKVError):
        BM(4, 16, free_order=[0, 0])


@pytest.mark.parametrize("seed", [0, 1])
def test_random_traces_with_swaps_match_reference(BM, seed):
    """Allocation, fork, copy-on-write, release and swap to a host pool: the
    native manager emits the same pairs and reaches the same state."""
    from paged_kv_cache_404_b200 import PagedKVError
    rng = np.random.default_rng(100 + seed)
    NB, NH = 160, 120
    order = rng.permutation(NB)
    bm, ref = BM(NB, 16, free_order=order), RefBlockManager(NB, 16, free_order=order)
    bm.set_host_pool(NH)
    ref.set_host_pool(NH)
    live = []
    for step in range(2500):
        op = int(rng.integers(0, 12))
        if op == 0 or not live:
            n = int(rng.integers(0, 70))
            try:
                r = ref.alloc_seq(n)
            except MemoryError:
                with pytest.raises(PagedKVError):
                    bm.alloc_seq(n)
                continue
            assert bm.alloc_seq(n) == r
            live.append(r)
            continue
        s = live[int(rng.integers(len(live)))]
        if op == 1 and len(live) > 1:
            live.remove(s)
            ref.free_seq(s)
            bm.free_seq(s)
        elif op == 2:
            swap = ref.swap_in if s in ref.swapped else ref.swap_out
            native = bm.swap_in if s in ref.swapped else bm.swap_out
            try:
                exp = swap(s)
            except MemoryError:
                with pytest.raises(PagedKVError) as e:
                    native(s)
                assert e.value.status == 4                    # PKV_ENOMEM, state unchanged
                continue
            assert [tuple(p) for p in native(s).tolist()] == exp
        elif s in ref.swapped:
            # a swapped sequence cannot be forked or grown
            with pytest.raises(PagedKVError) as e:
                (bm.fork if op == 3 else bm.append_token)(s)
            assert e.value.status == 6                        # PKV_ESWAPPED
        elif op == 3:
            r = ref.fork(s)
            assert bm.fork(s) == r
            live.append(r)
        else:
            try:
                exp = ref.append_token(s)
            except MemoryError:
                with pytest.raises(PagedKVError):
                    bm.append_token(s)
                continue
            assert bm.append_token(s) == exp
        if step % 200 == 0:
            _same_state(bm, ref, live)
    _same_state(bm, ref, live)


def test_swap_errors(BM):
    from paged_kv_cache_404_b200 import PagedKVError
    bm = BM(8, 16)
    a = bm.alloc_seq(40)
    with pytest.raises(PagedKVError):
        bm.swap_out(a)                 # no host pool yet: ENOMEM
    bm.set_host_pool(4)
    with pytest.raises(PagedKVError):
        bm.swap_in(a)                  # not swapped
    pairs = bm.swap_out(a)
    assert pairs.tolist() == [[0, 0], [1, 1], [2, 2]]
    assert bm.block_table(a).tolist() == [0, 1, 2] and bm.seq_len(a) == 40
    for call in (lambda: bm.slots(a, 0, 1), lambda: bm.tables([a], 4), lambda: bm.append_token(a)):
        with pytest.raises(PagedKVError):
            call()
    with pytest.raises(PagedKVError):
        bm.set_host_pool(8)            # host blocks in use
    with pytest.raises(PagedKVError):
        bm.swap_out(a)                 # already swapped
    bm.free_seq(a)
    assert bm.num_free_host() == 4 and bm.num_free() == 8
    bm.set_host_pool(8)
    assert bm.num_free_host() == 8


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_prefix_groups_match_reference(BM, seed):
    """Random families of forks with divergent continuations: the native hints
    equal the reference manager's for random batches."""
    rng = np.random.default_rng(300 + seed)
    NB = 600
    order = rng.permutation(NB)
    bm, ref = BM(NB, 16, free_order=order), RefBlockManager(NB, 16, free_order=order)
    live = []
    for fam in range(12):
        n = int(rng.integers(0, 120))
        a, r = bm.alloc_seq(n), ref.alloc_seq(n)
        assert a == r
        live.append(a)
        for _ in range(int(rng.integers(0, 4))):
            src = live[int(rng.integers(len(live)))]
            assert bm.fork(src) == ref.fork(src)
            live.append(len(live))
    for _ in range(400):
        s = live[int(rng.integers(len(live)))]
        assert bm.append_token(s) == ref.append_token(s)
    for _ in range(20):
        batch = [live[int(i)] for i in rng.choice(len(live), size=int(rng.integers(1, len(live))), replace=False)]
        offs, mem, sh = bm.prefix_groups(batch)
        r_offs, r_mem, r_sh = ref.prefix_groups(batch)
        assert (offs.tolist(), mem.tolist(), sh.tolist()) == (r_offs, r_mem, r_sh)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_prefix_cache_traces_match_reference(BM, seed):
    """Prompts drawn from a few system prompts plus random user tokens, with
    releases, forks and appends in between: same hits, tables, free list order
    and cache size as the reference manager."""
    from paged_kv_cache_404_b200 import PagedKVError
    rng = np.random.default_rng(500 + seed)
    NB = 220
    order = rng.permutation(NB)
    bm, ref = BM(NB, 16, free_order=order), RefBlockManager(NB, 16, free_order=order)
    bm.set_prefix_cache(True)
    ref.set_prefix_cache(True)
    systems = [rng.integers(0, 50, size=int(rng.integers(10, 90))).tolist() for _ in range(4)]
    live = []
    for step in range(1500):
        op = int(rng.integers(0, 10))
        if op <= 3 or not live:
            toks = systems[int(rng.integers(len(systems)))] + rng.integers(0, 3, size=int(rng.integers(0, 40))).tolist()
            try:
                exp = ref.alloc_seq_tokens(toks)
            except MemoryError:
                with pytest.raises(PagedKVError):
                    bm.alloc_seq_tokens(toks)
                continue
            assert bm.alloc_seq_tokens(toks) == exp
            live.append(exp[0])
        elif op <= 5 and len(live) > 1:
            s = live.pop(int(rng.integers(len(live))))
            ref.free_seq(s)
            bm.free_seq(s)
        elif op == 6:
            s = live[int(rng.integers(len(live)))]
            r = ref.fork(s)
            assert bm.fork(s) == r
            live.append(r)
        else:
            s = live[int(rng.integers(len(live)))]
            try:
                exp = ref.append_token(s)
            except MemoryError:
                with pytest.raises(PagedKVError):
                    bm.append_token(s)
                continue
            assert bm.append_token(s) == exp
        if step % 100 == 0:
            _same_state(bm, ref, live)
            assert bm.num_cached_blocks() == len(ref.cache)
    _same_state(bm, ref, live)


def test_beam_search_trace_matches_reference(BM):
    """The full beam workload's allocator trace (16 requests x 4 beams, 48 steps
    of fork / free / append with copy-on-write) on both managers."""
    import workloads as W
    w = W.WORKLOADS["beam"]
    R, B = w.num_prompts, w.samples
    NB = R * (-(-w.prefix_len // 16)) + R * B * (w.len_hi // 16 + 3)
    order = W.free_order(w, NB)
    bm, ref = BM(NB, 16, free_order=order), RefBlockManager(NB, 16, free_order=order)
    beams = []
    for r in range(R):
        p = bm.alloc_seq(w.prefix_len)
        assert ref.alloc_seq(w.prefix_len) == p
        kids = [bm.fork(p) for _ in range(B - 1)]
        assert [ref.fork(p) for _ in range(B - 1)] == kids
        beams.append([p] + kids)
    pairs_total = 0
    for t in range(w.len_hi):
        parents = W.beam_parents(w, t)
        new = []
        for r, old in enumerate(beams):
            kids = [bm.fork(old[int(q)]) for q in parents[r]]
            assert [ref.fork(old[int(q)]) for q in parents[r]] == kids
            for s in old:
                bm.free_seq(s)
                ref.free_seq(s)
            new.append(kids)
        beams = new
        flat = [s for kids in beams for s in kids]
        slots, pairs = bm.append_tokens(flat)
        res = [ref.append_token(s) for s in flat]
        assert slots.tolist() == [x[0] for x in res]
        assert [tuple(x) for x in pairs.tolist()] == [x[1] for x in res if x[1] is not None]
        pairs_total += len(pairs)
        if t % 8 == 0:
            _same_state(bm, ref, flat)
    _same_state(bm, ref, [s for kids in beams for s in kids])
    assert pairs_total > 0


def test_fork_many_and_free_many_equal_single_calls(BM):
    from paged_kv_cache_404_b200 import PagedKVError
    a, b = BM(64, 16), BM(64, 16)
    for m in (a, b):
        m.alloc_seq(40)
        m.alloc_seq(17)
    kids_a = a.fork_many([0, 1, 0, 0])
    kids_b = [b.fork(p) for p in [0, 1, 0, 0]]
    assert kids_a.tolist() == kids_b
    a.free_many([0, 3])
    b.free_seq(0)
    b.free_seq(3)
    assert a.free_list().tolist() == b.free_list().tolist()
    for blk in range(64):
        assert a.refcount(blk) == b.refcount(blk)
    with pytest.raises(PagedKVError):
        a.free_many([2, 2])            # listed twice: nothing freed
    assert a.seq_len(2) == 40
    with pytest.raises(PagedKVError):
        a.fork_many([1, 99])           # unknown parent: nothing forked
    assert a.fork_many([1]).tolist() == [6]


@pytest.mark.parametrize("seed", [0, 1, 2, 3])
def test_mixed_feature_traces_match_reference(BM, seed):
    """Every feature at once: prefix caching (hits on live and on free cached
    blocks), plain allocation, fork, release, single and batched appends with
    copy-on-write, swap out / in (whose fresh blocks may evict cached keys) and
    prefix groups of resident batches.  Same results and state as the reference."""
    from paged_kv_cache_404_b200 import PagedKVError
    rng = np.random.default_rng(700 + seed)
    NB, NH = 200, 120
    order = rng.permutation(NB)
    bm, ref = BM(NB, 16, free_order=order), RefBlockManager(NB, 16, free_order=order)
    for m in (bm, ref):
        m.set_prefix_cache(True)
        m.set_host_pool(NH)
    systems = [rng.integers(0, 40, size=int(rng.integers(16, 80))).tolist() for _ in range(3)]
    live = []

    def resident():
        return [s for s in live if s not in ref.swapped]

    for step in range(3000):
        op = int(rng.integers(0, 14))
        if op <= 2 or not live:
            toks = systems[int(rng.integers(len(systems)))] + rng.integers(0, 3, size=int(rng.integers(0, 30))).tolist()
            try:
                exp = ref.alloc_seq_tokens(toks)
            except MemoryError:
                with pytest.raises(PagedKVError):
                    bm.alloc_seq_tokens(toks)
                continue
            assert bm.alloc_seq_tokens(toks) == exp
            live.append(exp[0])
        elif op == 3:
            n = int(rng.integers(0, 50))
            try:
                r = ref.alloc_seq(n)
            except MemoryError:
                with pytest.raises(PagedKVError):
                    bm.alloc_seq(n)
                continue
            assert bm.alloc_seq(n) == r
            live.append(r)
        elif op == 4 and len(live) > 1:
            s = live.pop(int(rng.integers(len(live))))
            ref.free_seq(s)
            bm.free_seq(s)
        elif op == 5:
            res = resident()
            if not res:
                continue
            s = res[int(rng.integers(len(res)))]
            r = ref.fork(s)
            assert bm.fork(s) == r
            live.append(r)
        elif op == 6:
            s = live[int(rng.integers(len(live)))]
            swap = ref.swap_in if s in ref.swapped else ref.swap_out
            native = bm.swap_in if s in ref.swapped else bm.swap_out
            try:
                exp = swap(s)
            except MemoryError:
                with pytest.raises(PagedKVError):
                    native(s)
                continue
            assert [tuple(p) for p in native(s).tolist()] == exp
        elif op == 7:
            res = resident()
            if len(res) < 2:
                continue
            batch = [res[int(i)] for i in rng.choice(len(res), size=int(rng.integers(2, len(res) + 1)), replace=False)]
            offs, mem, sh = bm.prefix_groups(batch)
            assert (offs.tolist(), mem.tolist(), sh.tolist()) == tuple(ref.prefix_groups(batch))
        elif op <= 10:
            res = resident()
            if not res:
                continue
            batch = [res[int(i)] for i in rng.choice(len(res), size=min(len(res), int(rng.integers(1, 6))),
                                                       replace=False)]
            if len(batch) > ref.num_free():
                continue                       # a batch that cannot fail part-way
            exp = [ref.append_token(s) for s in batch]
            slots, pairs = bm.append_tokens(batch)
            assert slots.tolist() == [e[0] for e in exp]
            assert [tuple(p) for p in pairs.tolist()] == [e[1] for e in exp if e[1] is not None]
        else:
            res = resident()
            if not res:
                continue
            s = res[int(rng.integers(len(res)))]
            try:
                exp = ref.append_token(s)
            except MemoryError:
                with pytest.raises(PagedKVError):
                    bm.append_token(s)
                continue
            assert bm.append_token(s) == exp
        if step % 150 == 0:
            _same_state(bm, ref, live)
            assert bm.num_cached_blocks() == len(ref.cache)
    _same_state(bm, ref, live)
    assert bm.num_cached_blocks() == len(ref.cache)


def test_batched_append_stops_at_the_first_sequence_out_of_blocks(BM):
    """One pkv_bm_append_tokens call that runs out of blocks part-way: it returns
    PKV_ENOMEM, reports how many sequences got their slot, those keep it (with
    their copy-on-write pairs), the failing sequence and the rest are unchanged."""
    import ctypes as C
    from paged_kv_cache_404_b200 import _lib as L
    order = list(range(12))
    bm, ref = BM(12, 16, free_order=order), RefBlockManager(12, 16, free_order=order)
    # a: 3 full blocks (its next token needs a block); b: a fork of c (copy-on-write);
    # c: 2 blocks with room; d: 1 full block
    seqs = []
    for m in (bm, ref):
        a = m.alloc_seq(48)
        c = m.alloc_seq(20)
        b = m.fork(c)
        d = m.alloc_seq(16)
        seqs = [a, b, c, d]
    assert ref.num_free() == 12 - 3 - 2 - 1
    # use up all but 2 free blocks
    for m in (bm, ref):
        m.alloc_seq(16 * 4)
    batch = seqs                      # a takes 1 block, b 1 (copy-on-write), c writes in place, d finds none
    exp = []
    for s in batch:
        try:
            exp.append(ref.append_token(s))
        except MemoryError:
            break
    assert len(exp) == 3 and ref.num_free() == 0
    arr = np.asarray(batch, dtype=np.int32)
    slots = np.empty(4, dtype=np.int64)
    pairs = np.empty((4, 2), dtype=np.int64)
    npairs, ndone = C.c_int(), C.c_int()
    st = bm._lib.pkv_bm_append_tokens(bm._h, arr.ctypes.data, 4, slots.ctypes.data, pairs.ctypes.data,
                                      C.byref(npairs), C.byref(ndone))
    assert st == L.PKV_ENOMEM and ndone.value == 3
    assert slots[:3].tolist() == [e[0] for e in exp]
    assert [tuple(p) for p in pairs[:npairs.value].tolist()] == [e[1] for e in exp if e[1] is not None]
    _same_state(bm, ref, seqs)        # d unchanged on both sides
    assert bm.seq_len(seqs[3]) == 16


def test_native_manager_on_the_hand_worked_system_prompt_case(BM):
    """The hand-worked system-prompt sharing case of the reference manager's pins
    (worked example's free list; two requests share their first block, a request
    that starts with another's second block gets no hit, a freed keyed block is
    taken back out of the free list), on the native manager."""
    S, U1, U2 = list(range(100, 116)), list(range(200, 216)), list(range(300, 316))
    bm = BM(64, 16, free_order=[41, 7, 19, 2, 33, 11, 5])
    bm.set_prefix_cache(True)
    a, ca = bm.alloc_seq_tokens(S + U1 + [1] * 5)
    assert (bm.block_table(a).tolist(), ca) == ([41, 7, 19], 0)
    b, cb = bm.alloc_seq_tokens(S + U2 + [2] * 3)
    assert (bm.block_table(b).tolist(), cb) == ([41, 2, 33], 16)
    assert [bm.refcount(x) for x in (41, 7, 19, 2, 33)] == [2, 1, 1, 1, 1]
    d, cd = bm.alloc_seq_tokens(U1 + S)
    assert (bm.block_table(d).tolist(), cd) == ([11, 5], 0)
    bm.free_seq(a)
    assert bm.free_list().tolist() == [7, 19]
    e, ce = bm.alloc_seq_tokens(S + U1 + [3])
    assert (bm.block_table(e).tolist(), ce) == ([41, 7, 19], 32)
    assert [bm.refcount(x) for x in (41, 7, 19, 2, 33, 11, 5)] == [2, 1, 1, 1, 1, 1, 1]
    assert bm.num_free() == 0
