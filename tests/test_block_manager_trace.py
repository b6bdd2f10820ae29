"""The block manager's optional event trace (JSON lines): the record the pages
recommend keeping (when blocks are allocated, tables, sharing, copies, frees,
sequence lengths, concurrent requests).  The trace of a random history is
complete enough to replay that history on the reference manager, which must
reproduce every result the trace recorded (CPU only)."""
import io
import json

import numpy as np
import pytest

from oracle import RefBlockManager


@pytest.fixture(scope="module")
def BM():
    from paged_kv_cache_404_b200 import build
    build.build()
    from paged_kv_cache_404_b200 import BlockManager
    return BlockManager


def _history(bm, rng, steps):
    from paged_kv_cache_404_b200 import PagedKVError
    bm.set_host_pool(40)
    live = []
    for _ in range(steps):
        op = int(rng.integers(0, 10))
        try:
            if op == 0 or not live:
                live.append(bm.alloc_seq(int(rng.integers(0, 60))))
            elif op == 1:
                live.extend(bm.fork_many([live[int(rng.integers(len(live)))] for _ in range(2)]).tolist())
            elif op == 2 and len(live) > 2:
                bm.free_seq(live.pop(int(rng.integers(len(live)))))
            elif op == 3 and len(live) > 3:
                gone = [live.pop(int(rng.integers(len(live)))) for _ in range(2)]
                bm.free_many(gone)
            elif op == 4:
                s = live[int(rng.integers(len(live)))]
                (bm.swap_in if bm.is_swapped(s) else bm.swap_out)(s)
            else:
                res = [s for s in live if not bm.is_swapped(s)]
                if res:
                    bm.append_tokens([res[int(i)] for i in rng.choice(len(res), min(3, len(res)), replace=False)])
        except PagedKVError:
            pass                     # out of blocks: the call changed nothing (or, for appends, is traced)


@pytest.mark.parametrize("seed", [0, 1])
def test_trace_replays_on_the_reference_manager(BM, seed):
    rng = np.random.default_rng(900 + seed)
    NB = 120
    order = rng.permutation(NB).tolist()
    buf = io.StringIO()
    bm = BM(NB, 16, free_order=order, trace=buf)
    _history(bm, rng, 600)
    events = [json.loads(l) for l in buf.getvalue().splitlines()]
    assert events[0]["op"] == "create" and events[-1]["free"] == bm.num_free()
    assert all(e["t_ns"] <= f["t_ns"] for e, f in zip(events, events[1:]))
    ops = {e["op"] for e in events}
    assert {"alloc", "fork", "append", "free", "swap_out", "host_pool"} <= ops

    ref = None
    live = set()
    for e in events:
        op = e["op"]
        if op == "create":
            ref = RefBlockManager(e["num_blocks"], e["block_size"], free_order=e["free_order"])
        elif op == "host_pool":
            ref.set_host_pool(e["blocks"])
        elif op == "alloc":
            assert ref.alloc_seq(e["tokens"]) == e["seq"] and ref.tables[e["seq"]] == e["table"]
            live.add(e["seq"])
        elif op == "fork":
            assert [ref.fork(p) for p in e["parents"]] == e["children"]
            live.update(e["children"])
        elif op == "append":
            got = [ref.append_token(s) for s in e["seqs"]]
            assert [g[0] for g in got] == e["slots"]
            assert [list(g[1]) for g in got if g[1] is not None] == e["cow"]
            assert [ref.lens[s] for s in e["seqs"]] == e["lens"]
        elif op == "free":
            dev, host_blocks = [], []
            for s, table, host in zip(e["seqs"], e["tables"], e["host"]):
                assert ref.tables[s] == table and (s in ref.swapped) == host
                (host_blocks if host else dev).extend(table)
                ref.free_seq(s)
                live.discard(s)
            assert e["freed"] == [b for b in dict.fromkeys(dev) if ref.ref[b] == 0]
            assert e["freed_host"] == host_blocks
        elif op in ("swap_out", "swap_in"):
            assert [list(p) for p in getattr(ref, op)(e["seq"])] == e["pairs"]
        assert e["live"] == len(live) and e["free"] == ref.num_free()


def test_trace_records_prefix_cache_reuse(BM):
    buf = io.StringIO()
    bm = BM(64, 16, trace=buf)
    bm.set_prefix_cache(True)
    toks = list(range(40))
    a, _ = bm.alloc_seq_tokens(toks)
    b, cached = bm.alloc_seq_tokens(toks)
    ev = [json.loads(l) for l in buf.getvalue().splitlines()]
    allocs = [e for e in ev if e["op"] == "alloc"]
    assert [e["cached_tokens"] for e in allocs] == [0, 32] and cached == 32
    assert allocs[1]["table"][:2] == allocs[0]["table"][:2]       # the two full blocks are shared
    assert allocs[1]["live"] == 2


def test_no_trace_by_default(BM):
    bm = BM(16, 16)
    assert bm._trace is None
    s = bm.alloc_seq(20)
    bm.free_seq(s)
    assert bm._live == set()      # nothing tracked when no trace is open


def test_trace_of_an_append_that_runs_out_part_way(BM):
    from paged_kv_cache_404_b200 import PagedKVError
    buf = io.StringIO()
    bm = BM(5, 16, trace=buf)     # 1 + 2 + 1 blocks below leave one free
    a = bm.alloc_seq(16)          # full: its next token needs a block
    b = bm.alloc_seq(32)          # full too
    c = bm.alloc_seq(16)
    with pytest.raises(PagedKVError):
        bm.append_tokens([a, b, c])   # one free block: a gets it, b finds none
    last = json.loads(buf.getvalue().splitlines()[-1])
    assert last["op"] == "append" and last["seqs"] == [a] and last["lens"] == [17]
    assert last["error"] and last["free"] == 0 and last["live"] == 3
