"""Reference block manager for the paged KV cache (test infrastructure only).

Written from the pages' description of the host side of PagedAttention:

- "PagedAttention" glossary entry (ultralytics.com), section "Como funciona la
  paginacion": a request receives a new block only when its previous one is
  full, from any free location, and its block table records the order.  The
  worked example pops blocks from the front of a free list ([41, 7, 19, 2, 33])
  and stores token `pos` at (block_table[pos // block_size], pos % block_size).
- same page, "Compartir bloques entre secuencias": sequences may point at the
  same physical blocks, counted by a per-block reference count; a sequence that
  must write into a block others still use first copies it (copy-on-write).
- iplexlaw.co.kr blog, sections on logical vs physical order and "two answers
  to one request": the prompt is allocated first, then the last block is filled,
  and a new block is added only when needed; full shared blocks stay shared,
  only the block that must split is copied; blocks with no references are freed.
- same glossary page, "Tecnicas relacionadas" (continuous batching): a finished
  sequence's blocks return to the free pool at once.
- same glossary page, end of the sharing section: hashing whole blocks extends
  sharing across requests (prompt caching).
- "Le cache KV et PagedAttention" (gyaansetu.com), fine-grained eviction: when
  memory runs out, a sequence's small pages can go to the CPU instead of the
  whole sequence being dropped, and come back later.

Readings where the pages are silent: the free list is first-in first-out (pop
from the front, freed blocks appended to the back in table order); a
copy-on-write copies the whole block and moves the writer to the copy, leaving
the last holder (reference count 1) to write in place; running out of free
blocks raises MemoryError and leaves the state unchanged.  Swap moves all of a
sequence's pages at once to a host pool with its own first-in first-out free
list (ids 0..n-1); a page shared with another sequence is copied out and comes
back as a private block; a swapped sequence can only be swapped in or freed.
Prefix caching keys a full prompt block by its exact token ids and its parent
block's registration (a number never reused), registers only prompt blocks,
reuses the longest run of matching leading full blocks, keeps an unused
registered block's key while it waits in the free list (a hit takes it back
out of the list), and drops the key when the block is handed out for new data.
"""
from collections import deque


class RefBlockManager:
    def __init__(self, num_blocks, block_size, free_order=None):
        if free_order is None:
            free_order = range(num_blocks)
        free_order = [int(b) for b in free_order]
        # A free list may name only some blocks (the rest are owned elsewhere,
        # as in the worked example's five free blocks of a 64-block pool).
        assert len(set(free_order)) == len(free_order), "a block may be free only once"
        assert all(0 <= b < num_blocks for b in free_order), "block id out of range"
        self.num_blocks = num_blocks
        self.block_size = block_size
        self.free = deque(free_order)
        self.ref = [0] * num_blocks
        self.tables = {}
        self.lens = {}
        self._next = 0
        self.host_free = deque()
        self.swapped = set()
        self.prefix_cache = False
        self.cache = {}            # (parent serial, token tuple) -> (block, serial)
        self.key_of = {}           # block -> its key
        self._serial = 0

    # -- allocation ---------------------------------------------------------
    def _pop(self):
        if not self.free:
            raise MemoryError("no free block")
        b = self.free.popleft()
        assert self.ref[b] == 0
        self.ref[b] = 1
        if b in self.key_of:              # new contents: forget the old key
            del self.cache[self.key_of.pop(b)]
        return b

    def alloc_seq(self, num_tokens):
        """New sequence holding `num_tokens` prompt tokens: ceil(n / bs) blocks."""
        need = -(-num_tokens // self.block_size)
        if need > len(self.free):
            raise MemoryError("not enough free blocks")
        seq = self._next
        self._next += 1
        self.tables[seq] = [self._pop() for _ in range(need)]
        self.lens[seq] = num_tokens
        return seq

    def set_prefix_cache(self, enable=True):
        self.prefix_cache = bool(enable)
        if not enable:
            self.cache.clear()
            self.key_of.clear()

    def alloc_seq_tokens(self, tokens):
        """New sequence for a prompt given by token ids.

        Returns (seq, number of leading tokens whose blocks came from the cache).
        """
        tokens = [int(t) for t in tokens]
        if not self.prefix_cache:
            return self.alloc_seq(len(tokens)), 0
        bs = self.block_size
        full = len(tokens) // bs
        need = -(-len(tokens) // bs)
        hits, parent = [], 0
        for j in range(full):
            key = (parent, tuple(tokens[j * bs:(j + 1) * bs]))
            if key not in self.cache:
                break
            block, parent = self.cache[key]
            hits.append(block)
        waking = [b for b in hits if self.ref[b] == 0]
        if need - len(hits) + len(waking) > len(self.free):
            raise MemoryError("not enough free blocks")
        for b in hits:
            if self.ref[b] == 0:
                self.free.remove(b)
            self.ref[b] += 1
        table = hits + [self._pop() for _ in range(need - len(hits))]
        for j in range(len(hits), full):
            self._serial += 1
            key = (parent, tuple(tokens[j * bs:(j + 1) * bs]))
            self.cache[key] = (table[j], self._serial)
            self.key_of[table[j]] = key
            parent = self._serial
        seq = self._next
        self._next += 1
        self.tables[seq] = table
        self.lens[seq] = len(tokens)
        return seq, len(hits) * bs

    def fork(self, parent):
        """New sequence sharing every block of `parent` (reference counts + 1)."""
        seq = self._next
        self._next += 1
        self.tables[seq] = list(self.tables[parent])
        self.lens[seq] = self.lens[parent]
        for b in self.tables[seq]:
            self.ref[b] += 1
        return seq

    def append_token(self, seq):
        """Reserve the slot of the sequence's next token.

        Returns (slot, cow) where cow is None or the (src, dst) block pair that
        must be copied before the token is written.
        """
        n = self.lens[seq]
        table = self.tables[seq]
        cow = None
        if n % self.block_size == 0:
            # last block full (or no block yet): a fresh block, nothing to copy
            table.append(self._pop())
        else:
            last = table[-1]
            if self.ref[last] > 1:
                new = self._pop()
                self.ref[last] -= 1
                table[-1] = new
                cow = (last, new)
        slot = table[n // self.block_size] * self.block_size + n % self.block_size
        self.lens[seq] = n + 1
        return slot, cow

    def free_seq(self, seq):
        """Drop a finished sequence; blocks whose count reaches 0 return to the pool."""
        table = self.tables.pop(seq)
        del self.lens[seq]
        if seq in self.swapped:
            self.swapped.discard(seq)
            self.host_free.extend(table)
            return
        for b in table:
            self.ref[b] -= 1
            if self.ref[b] == 0:
                self.free.append(b)

    # -- swap to a host pool --------------------------------------------------
    def set_host_pool(self, num_host_blocks):
        assert not self.swapped, "host blocks still in use"
        self.host_free = deque(range(num_host_blocks))

    def swap_out(self, seq):
        """Move every page of a resident sequence to host blocks.

        Returns the (device block, host block) copies, in table order.
        """
        assert seq not in self.swapped
        table = self.tables[seq]
        if len(table) > len(self.host_free):
            raise MemoryError("not enough free host blocks")
        pairs = []
        for i, b in enumerate(table):
            h = self.host_free.popleft()
            pairs.append((b, h))
            self.ref[b] -= 1
            if self.ref[b] == 0:
                self.free.append(b)
            table[i] = h
        self.swapped.add(seq)
        return pairs

    def swap_in(self, seq):
        """Bring a swapped sequence back into fresh device blocks.

        Returns the (host block, device block) copies, in table order.
        """
        assert seq in self.swapped
        table = self.tables[seq]
        if len(table) > len(self.free):
            raise MemoryError("not enough free blocks")
        pairs = []
        for i, h in enumerate(table):
            b = self._pop()
            pairs.append((h, b))
            self.host_free.append(h)
            table[i] = b
        self.swapped.discard(seq)
        return pairs

    # -- shared prefixes ------------------------------------------------------
    def prefix_groups(self, seqs):
        """Sequences of a batch that start with the same physical block.

        Returns (offsets, members, shared): group g has batch indices
        members[offsets[g]:offsets[g+1]] (batch order) and shares its first
        shared[g] table entries, each a full block in every member.  Only
        groups of two or more are listed, in order of first appearance.
        """
        firsts = {}
        for i, s in enumerate(seqs):
            assert s not in self.swapped
            if self.lens[s] >= self.block_size:
                firsts.setdefault(self.tables[s][0], []).append(i)
        offsets, members, shared = [0], [], []
        for group in firsts.values():
            if len(group) < 2:
                continue
            tabs = [self.tables[seqs[i]] for i in group]
            full = min(self.lens[seqs[i]] // self.block_size for i in group)
            k = 0
            while k < full and all(t[k] == tabs[0][k] for t in tabs):
                k += 1
            members += group
            shared.append(k)
            offsets.append(len(members))
        return offsets, members, shared

    # -- queries ------------------------------------------------------------
    def slot(self, seq, pos):
        t = self.tables[seq]
        return t[pos // self.block_size] * self.block_size + pos % self.block_size

    def slots(self, seq, start, count):
        return [self.slot(seq, p) for p in range(start, start + count)]

    def num_free(self):
        return len(self.free)
