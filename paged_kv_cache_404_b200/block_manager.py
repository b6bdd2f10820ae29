"""Python face of the native host block manager (pkv_bm_* in pagedkv.h).

The manager itself is C++ (csrc/block_manager.cpp); this class only marshals
numpy arrays.  It runs on the CPU and needs no GPU.

Optional event trace (JSON lines).  The iplexlaw.co.kr blog post on
PagedAttention and the vLLM KV cache, section "Memory management and the
technical differences", advises recording when blocks are allocated, the block
tables, the conditions of sharing, copies and releases, sequence lengths and
the number of concurrent requests; this trace keeps that record: every
allocation, fork, append, release and swap writes
one line with a monotonic timestamp (t_ns), the operation's inputs and results
(tables, slots, copy-on-write pairs, blocks actually freed, swap pairs, tokens
reused from the prefix cache), and the live-sequence and free-block counts after
it.  Off by default; when off the cost is one comparison per call.
"""
import ctypes as C
import json
import time

import numpy as np

from . import _lib as L


class BlockManager:
    def __init__(self, num_blocks, block_size=16, free_order=None, trace=None):
        """trace: None, a path (opened for writing) or a text stream that receives
        one JSON line per state-changing call."""
        self._trace, self._own_trace, self._live = None, False, set()
        self._lib = L.lib()
        h = C.c_void_p()
        if free_order is None:
            st = self._lib.pkv_bm_create(num_blocks, block_size, None, 0, C.byref(h))
        else:
            fo = np.ascontiguousarray(free_order, dtype=np.int32)
            st = self._lib.pkv_bm_create(num_blocks, block_size, fo.ctypes.data, fo.size, C.byref(h))
        L.check("pkv_bm_create", st)
        self._h = h
        self.num_blocks = num_blocks
        self.block_size = block_size
        if trace is not None:
            self._own_trace = isinstance(trace, str)
            self._trace = open(trace, "w") if self._own_trace else trace
            self._emit("create", num_blocks=num_blocks, block_size=block_size,
                       free_order=None if free_order is None else np.asarray(free_order).tolist())

    def _emit(self, op, **fields):
        rec = {"t_ns": time.monotonic_ns(), "op": op}
        rec.update(fields)
        rec["live"] = len(self._live)
        rec["free"] = self.num_free()
        self._trace.write(json.dumps(rec) + "\n")

    def close(self):
        if self._trace is not None and self._own_trace:
            self._trace.close()
        self._trace = None
        if self._h:
            self._lib.pkv_bm_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:  # noqa: BLE001 - interpreter shutdown
            pass

    def alloc_seq(self, num_tokens):
        out = C.c_int32()
        L.check("pkv_bm_alloc_seq", self._lib.pkv_bm_alloc_seq(self._h, int(num_tokens), C.byref(out)))
        if self._trace is not None:
            self._live.add(out.value)
            self._emit("alloc", seq=out.value, tokens=int(num_tokens), table=self.block_table(out.value).tolist())
        return out.value

    def fork(self, parent):
        out = C.c_int32()
        L.check("pkv_bm_fork", self._lib.pkv_bm_fork(self._h, int(parent), C.byref(out)))
        if self._trace is not None:
            self._live.add(out.value)
            self._emit("fork", parents=[int(parent)], children=[out.value])
        return out.value

    def fork_many(self, parents):
        """Fork every parent, in order; returns the children (int32 array)."""
        par = np.ascontiguousarray(parents, dtype=np.int32)
        out = np.empty(max(par.size, 1), dtype=np.int32)
        L.check("pkv_bm_fork_many", self._lib.pkv_bm_fork_many(self._h, par.ctypes.data, par.size, out.ctypes.data))
        kids = out[:par.size].copy()
        if self._trace is not None:
            self._live.update(kids.tolist())
            self._emit("fork", parents=par.tolist(), children=kids.tolist())
        return kids

    def _freed_record(self, seqs):
        """Per sequence to be freed: its table, and whether it sits in the host pool."""
        return [(int(s), self.block_table(s).tolist(), self.is_swapped(s)) for s in seqs]

    def _emit_free(self, before):
        """One event per call: the device blocks whose count reached 0 (back in the
        free list, first-appearance order) and the host blocks returned."""
        dev, host = [], []
        for s, table, swapped in before:
            self._live.discard(s)
            (host if swapped else dev).extend(table)
        self._emit("free", seqs=[b[0] for b in before], tables=[b[1] for b in before],
                   host=[b[2] for b in before],
                   freed=[b for b in dict.fromkeys(dev) if self.refcount(b) == 0], freed_host=host)

    def free_many(self, seqs):
        s = np.ascontiguousarray(seqs, dtype=np.int32)
        before = self._freed_record(s.tolist()) if self._trace is not None else None
        L.check("pkv_bm_free_many", self._lib.pkv_bm_free_many(self._h, s.ctypes.data, s.size))
        if before is not None:
            self._emit_free(before)

    def append_tokens(self, seqs):
        """One new slot per sequence, in order. Returns (slots int64 [n], cow pairs int64 [k, 2])."""
        seqs = np.ascontiguousarray(seqs, dtype=np.int32)
        n = seqs.size
        slots = np.empty(n, dtype=np.int64)
        pairs = np.empty((max(n, 1), 2), dtype=np.int64)
        npairs, ndone = C.c_int(), C.c_int()
        st = self._lib.pkv_bm_append_tokens(self._h, seqs.ctypes.data, n, slots.ctypes.data, pairs.ctypes.data,
                                            C.byref(npairs), C.byref(ndone))
        if self._trace is not None:
            done = n if st == L.PKV_OK else ndone.value
            self._emit("append", seqs=seqs[:done].tolist(), slots=slots[:done].tolist(),
                       cow=pairs[:npairs.value].tolist(), lens=[self.seq_len(x) for x in seqs[:done].tolist()],
                       **({} if st == L.PKV_OK else {"error": L.status_string(st)}))
        if st != L.PKV_OK:
            raise L.PagedKVError("pkv_bm_append_tokens", st)
        return slots, pairs[:npairs.value].copy()

    def append_token(self, seq):
        slots, pairs = self.append_tokens([seq])
        return int(slots[0]), (tuple(int(x) for x in pairs[0]) if len(pairs) else None)

    def free_seq(self, seq):
        before = self._freed_record([int(seq)]) if self._trace is not None else None
        L.check("pkv_bm_free_seq", self._lib.pkv_bm_free_seq(self._h, int(seq)))
        if before is not None:
            self._emit_free(before)

    def num_free(self):
        return self._lib.pkv_bm_num_free(self._h)

    def seq_len(self, seq):
        out = C.c_int32()
        L.check("pkv_bm_seq_len", self._lib.pkv_bm_seq_len(self._h, int(seq), C.byref(out)))
        return out.value

    def refcount(self, block):
        out = C.c_int32()
        L.check("pkv_bm_refcount", self._lib.pkv_bm_refcount(self._h, int(block), C.byref(out)))
        return out.value

    def block_table(self, seq):
        n = C.c_int()
        self._lib.pkv_bm_block_table(self._h, int(seq), None, 0, C.byref(n))
        out = np.empty(max(n.value, 1), dtype=np.int32)
        L.check("pkv_bm_block_table",
                self._lib.pkv_bm_block_table(self._h, int(seq), out.ctypes.data, out.size, C.byref(n)))
        return out[:n.value].copy()

    def slots(self, seq, start, count):
        out = np.empty(max(count, 1), dtype=np.int64)
        L.check("pkv_bm_slots", self._lib.pkv_bm_slots(self._h, int(seq), int(start), int(count), out.ctypes.data))
        return out[:count].copy()

    def tables(self, seqs, max_blocks, pad=-1):
        """Padded block tables int32 [n, max_blocks] and lengths int32 [n]."""
        seqs = np.ascontiguousarray(seqs, dtype=np.int32)
        tab = np.empty((seqs.size, max_blocks), dtype=np.int32)
        lens = np.empty(seqs.size, dtype=np.int32)
        L.check("pkv_bm_tables", self._lib.pkv_bm_tables(self._h, seqs.ctypes.data, seqs.size, tab.ctypes.data,
                                                         int(max_blocks), int(pad), lens.ctypes.data))
        return tab, lens

    def free_list(self):
        n = C.c_int()
        self._lib.pkv_bm_free_list(self._h, None, 0, C.byref(n))
        out = np.empty(max(n.value, 1), dtype=np.int32)
        L.check("pkv_bm_free_list", self._lib.pkv_bm_free_list(self._h, out.ctypes.data, out.size, C.byref(n)))
        return out[:n.value].copy()

    # --- prefix caching across requests (full-block keys) ----------------------

    def set_prefix_cache(self, enable=True):
        L.check("pkv_bm_set_prefix_cache", self._lib.pkv_bm_set_prefix_cache(self._h, int(bool(enable))))
        if self._trace is not None:
            self._emit("prefix_cache", enable=bool(enable))

    def alloc_seq_tokens(self, tokens):
        """New sequence for a prompt given by token ids; returns (seq, tokens already cached)."""
        t = np.ascontiguousarray(tokens, dtype=np.int32)
        seq, cached = C.c_int32(), C.c_int()
        L.check("pkv_bm_alloc_seq_tokens", self._lib.pkv_bm_alloc_seq_tokens(
            self._h, t.ctypes.data if t.size else None, t.size, C.byref(seq), C.byref(cached)))
        if self._trace is not None:
            self._live.add(seq.value)
            self._emit("alloc", seq=seq.value, tokens=int(t.size), table=self.block_table(seq.value).tolist(),
                       cached_tokens=cached.value)
        return seq.value, cached.value

    def num_cached_blocks(self):
        return self._lib.pkv_bm_num_cached_blocks(self._h)

    def prefix_groups(self, seqs):
        """Shared-prefix hints of a batch: (offsets int32 [g+1], members int32 [m], shared int32 [g])."""
        seqs = np.ascontiguousarray(seqs, dtype=np.int32)
        n = seqs.size
        offs = np.zeros(n + 1, dtype=np.int32)
        mem = np.zeros(max(n, 1), dtype=np.int32)
        sh = np.zeros(max(n, 1), dtype=np.int32)
        ng = C.c_int()
        L.check("pkv_bm_prefix_groups", self._lib.pkv_bm_prefix_groups(
            self._h, seqs.ctypes.data, n, offs.ctypes.data, mem.ctypes.data, sh.ctypes.data, C.byref(ng)))
        g = ng.value
        return offs[:g + 1].copy(), mem[:offs[g]].copy(), sh[:g].copy()

    # --- host pool and swap (fine-grained eviction) -------------------------

    def set_host_pool(self, num_host_blocks):
        L.check("pkv_bm_set_host_pool", self._lib.pkv_bm_set_host_pool(self._h, int(num_host_blocks)))
        if self._trace is not None:
            self._emit("host_pool", blocks=int(num_host_blocks))

    def _swap(self, fn, name, seq):
        n = C.c_int()
        cap = max(len(self.block_table(seq)), 1)
        pairs = np.empty((cap, 2), dtype=np.int64)
        L.check(name, fn(self._h, int(seq), pairs.ctypes.data, cap, C.byref(n)))
        return pairs[:n.value].copy()

    def swap_out(self, seq):
        """Move a sequence to host blocks; returns (device block, host block) pairs int64 [k, 2]."""
        pairs = self._swap(self._lib.pkv_bm_swap_out, "pkv_bm_swap_out", seq)
        if self._trace is not None:
            self._emit("swap_out", seq=int(seq), pairs=pairs.tolist())
        return pairs

    def swap_in(self, seq):
        """Bring a swapped sequence back; returns (host block, device block) pairs int64 [k, 2]."""
        pairs = self._swap(self._lib.pkv_bm_swap_in, "pkv_bm_swap_in", seq)
        if self._trace is not None:
            self._emit("swap_in", seq=int(seq), pairs=pairs.tolist())
        return pairs

    def is_swapped(self, seq):
        out = C.c_int()
        L.check("pkv_bm_is_swapped", self._lib.pkv_bm_is_swapped(self._h, int(seq), C.byref(out)))
        return bool(out.value)

    def num_free_host(self):
        return self._lib.pkv_bm_num_free_host(self._h)
