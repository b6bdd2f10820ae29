"""Shared set-up for the GPU parity tests.

Each case is built twice from the same seeded inputs (workloads/): the product
side uses the native block manager and the CUDA kernels through the C ABI; the
oracle side uses the reference block manager and the C oracle.  Integer
outputs (tables, slots, copy pairs, written bytes) are compared exactly;
attention outputs within the tolerances below.
"""
import math

import numpy as np
import torch

import oracle
import workloads as W

# Attention tolerances, |gpu - ref| <= ATOL + RTOL * |ref| element-wise:
#  - fp32 cache: fp32 accumulation over at most a few thousand terms;
#  - bf16 cache: 1e-2 absolute and relative, applied as allclose (a literal
#    "both <= 1e-2" fails on bf16 output rounding alone once |ref| >= 4);
#  - FP8 cache: 3e-2 against an oracle that dequantises the same bytes.
TOL = {"f32": (1e-5, 1e-5), "bf16": (1e-2, 1e-2), "fp8": (3e-2, 3e-2)}

ORC_DT = {"f32": oracle.F32, "bf16": oracle.BF16, "fp8": oracle.FP8_E4M3}


def to_np_bits(t: torch.Tensor) -> np.ndarray:
    """Raw bytes of a tensor as numpy (bf16 -> uint16 bits, fp8 -> uint8 codes)."""
    t = t.detach().contiguous().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype in (torch.uint8, torch.float8_e4m3fn):
        return t.view(torch.uint8).numpy()
    return t.numpy()


def out_to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def assert_close(gpu, ref, kind, what=""):
    atol, rtol = TOL[kind]
    err = np.abs(gpu - ref)
    bound = atol + rtol * np.abs(ref)
    bad = err > bound
    assert np.isfinite(gpu).all(), "%s: non-finite GPU output" % what
    assert not bad.any(), "%s: %d/%d elements out of tolerance; max abs err %.3g, worst at %s" % (
        what, int(bad.sum()), bad.size, float(err.max()), np.unravel_index(np.argmax(err - bound), err.shape))
    return float(err.max()), float((err / np.maximum(np.abs(ref), 1e-30)).max())


class DecodeCase:
    """One decode step of a workload: write the new token of every sequence,
    then attend over its whole context (which includes that token)."""

    def __init__(self, w, lens=None, device="cuda", sample=None, pool_blocks=None):
        from paged_kv_cache_404_b200 import BlockManager
        self.w = w
        self.device = device
        self.lens = np.asarray(W.context_lens(w) if lens is None else lens, dtype=np.int32)
        S = self.S = len(self.lens)
        need = int(sum(-(-int(L) // 16) for L in self.lens))
        self.NB = pool_blocks or W.pool_blocks(w, max(need, 1))
        order = W.free_order(w, self.NB)
        # product and oracle allocators from the same free-list order
        self.bm = BlockManager(self.NB, 16, free_order=order)
        self.ref = oracle.RefBlockManager(self.NB, 16, free_order=order)
        alloc = [s for s in W.allocation_order(w) if s < S] if w.lens == "tiny" else list(range(S))
        ids, rids = {}, {}
        for s in alloc:
            ids[s] = self.bm.alloc_seq(max(int(self.lens[s]) - 1, 0))
            rids[s] = self.ref.alloc_seq(max(int(self.lens[s]) - 1, 0))
        self.ids = [ids[s] for s in range(S)]
        self.rids = [rids[s] for s in range(S)]
        has_new = [int(L) > 0 for L in self.lens]
        step = [self.ids[s] for s in range(S) if has_new[s]]
        slots, pairs = self.bm.append_tokens(step)
        assert len(pairs) == 0
        rslots = [self.ref.append_token(self.rids[s])[0] for s in range(S) if has_new[s]]
        assert slots.tolist() == rslots, "block manager parity: new-token slots"
        full = np.full(S, -1, dtype=np.int64)
        full[np.array(has_new)] = slots
        self.slots = full
        self.max_blocks = max(1, max(-(-int(L) // 16) for L in self.lens))
        self.tables, lens_bm = self.bm.tables(self.ids, self.max_blocks, pad=-1)
        assert np.array_equal(lens_bm, self.lens)
        for s in range(S):
            assert self.tables[s][:len(self.ref.tables[self.rids[s]])].tolist() == self.ref.tables[self.rids[s]]
        self.max_len = int(self.lens.max()) if S else 0
        # seeded device data
        if w.cache_dtype == "f32":
            self.k_pool, self.v_pool = W.stale_fill(w, self.NB, device)
            self.k_scale = self.v_scale = 1.0
        else:
            self.k_pool, self.v_pool, self.k_scale, self.v_scale = W.random_pools(w, self.NB, device)
        self.q = W.queries(w, S, device)
        self.k_new, self.v_new = W.new_tokens(w, S, device)
        self.sample = np.arange(S) if sample is None else np.asarray(sample)

    # -------------------------------------------------------------- product side
    def run_gpu(self, partition_tokens=0, err=None):
        import paged_kv_cache_404_b200 as pkv
        dev = self.device
        self.g_slots = torch.from_numpy(self.slots).to(dev)
        self.g_tables = torch.from_numpy(self.tables).to(dev)
        self.g_lens = torch.from_numpy(self.lens).to(dev)
        self.g_err = torch.zeros(1, dtype=torch.int32, device=dev) if err is None else err
        self.ws = pkv.decode_workspace(self.S, self.w.num_heads, self.w.head_dim, self.max_len, partition_tokens,
                                       device=dev)
        self.out = torch.empty_like(self.q)
        pkv.paged_kv_write(self.k_new, self.v_new, self.g_slots, self.k_pool, self.v_pool, self.k_scale,
                           self.v_scale, err_count=self.g_err)
        pkv.paged_attention_decode(self.out, self.q, self.k_pool, self.v_pool, self.g_tables, self.g_lens,
                                   self.w.scale, self.max_len, self.ws, self.k_scale, self.v_scale,
                                   partition_tokens=partition_tokens, err_count=self.g_err)
        torch.cuda.synchronize()
        return self.out

    # -------------------------------------------------------------- oracle side
    def snapshot_pools(self):
        """Host copy of the pools' blocks referenced by the sampled sequences,
        taken before the product writes anything (the oracle's own input)."""
        used = sorted({int(b) for s in self.sample for b in self.ref.tables[self.rids[s]]})
        self.remap = np.full(self.NB, -1, dtype=np.int64)
        self.remap[used] = np.arange(len(used))
        idx = torch.tensor(used, dtype=torch.long, device=self.device)
        self.h_k = to_np_bits(self.k_pool.index_select(0, idx)).copy()
        self.h_v = to_np_bits(self.v_pool.index_select(0, idx)).copy()

    def run_oracle(self):
        w = self.w
        src = ORC_DT["f32" if w.cache_dtype == "f32" else "bf16"]
        # the oracle's own slots (reference manager), relabelled to the snapshot's block numbering
        rslots = np.array([self.ref.slot(self.rids[s], int(self.lens[s]) - 1) if self.lens[s] > 0 else -1
                           for s in range(self.S)], dtype=np.int64)
        blk = np.where(rslots >= 0, rslots // 16, 0)
        local = np.where((rslots >= 0) & (self.remap[blk] >= 0), self.remap[blk] * 16 + rslots % 16, -1)
        bad = oracle.kv_write(to_np_bits(self.k_new), to_np_bits(self.v_new), src, local, self.h_k, self.h_v,
                              ORC_DT[w.cache_dtype], 16, self.k_scale, self.v_scale)
        assert bad == 0
        tabs = np.full((len(self.sample), self.max_blocks), -1, dtype=np.int32)
        for i, s in enumerate(self.sample):
            t = self.ref.tables[self.rids[s]]
            tabs[i, :len(t)] = self.remap[t]
        q = to_np_bits(self.q)[self.sample]
        out, badref = oracle.paged_attention_decode(q, ORC_DT[w.q_dtype], self.h_k, self.h_v, ORC_DT[w.cache_dtype],
                                                    tabs, self.lens[self.sample], w.scale, self.k_scale,
                                                    self.v_scale)
        assert badref == 0
        self.ref_out = out
        self.ref_local_slots = local
        return out

    def check_written_rows(self):
        """Bytes the product wrote at each sampled sequence's new slot equal the oracle's."""
        gk = self.k_pool.view(self.NB * 16, -1)
        gv = self.v_pool.view(self.NB * 16, -1)
        hk = self.h_k.reshape(-1, gk.shape[1])
        hv = self.h_v.reshape(-1, gv.shape[1])
        for s in self.sample:
            if self.lens[s] == 0:
                continue
            gs = int(self.slots[s])
            ls = int(self.ref_local_slots[s])
            assert np.array_equal(to_np_bits(gk[gs]), hk[ls]), "K row of sequence %d" % s
            assert np.array_equal(to_np_bits(gv[gs]), hv[ls]), "V row of sequence %d" % s

    def compare(self):
        got = out_to_f64(self.out)[self.sample]
        return assert_close(got, self.ref_out, self.w.cache_dtype, self.w.name)


def scale_of(w):
    return 1.0 / math.sqrt(w.head_dim)


class SharedPrefixReplay:
    """Parallel sampling over shared prompts, replayed token by token on both sides.

    Each prompt's prefix is written once and shared by `samples` sequences
    through their tables (reference count = samples); every continuation token
    is appended in sequence order, with a copy-on-write of the shared partly
    filled block on a sequence's first divergent write.  Then one decode step:
    a new token for every sequence (copy, write), then attention.
    """

    def __init__(self, w, num_prompts=None, cont=None, device="cuda"):
        from paged_kv_cache_404_b200 import BlockManager
        self.w = w
        self.device = device
        self.P = num_prompts or w.num_prompts
        self.n = w.samples
        self.S = self.P * self.n
        self.cont = (W.continuation_lens(w)[:self.S] if cont is None else np.asarray(cont)).astype(np.int32)
        # pool size from a dry run of the reference manager (1.25x the peak use)
        dry = oracle.RefBlockManager(200000, 16)
        self._replay_alloc(dry, lambda *a: None, lambda m, seqs, c: [m.append_token(s) for s in seqs] and None)
        for s in list(dry.tables):
            dry.append_token(s)
        used = sum(1 for r in dry.ref if r > 0)
        self.NB = int(np.ceil(used * w.pool_factor)) + 1
        order = W.free_order(w, self.NB)
        self.bm = BlockManager(self.NB, 16, free_order=order)
        self.ref = oracle.RefBlockManager(self.NB, 16, free_order=order)
        self.kp, self.vp = W.stale_fill(w, self.NB, device)
        self.hk, self.hv = to_np_bits(self.kp).copy(), to_np_bits(self.vp).copy()
        total_prefix = self.P * w.prefix_len
        self.prefix_k, self.prefix_v = W.logical_kv(w, total_prefix, device, stream=50)
        self.cont_k, self.cont_v = W.logical_kv(w, int(self.cont.sum()) + 1, device, stream=60)
        self.q = W.queries(w, self.S, device)
        self.k_new, self.v_new = W.new_tokens(w, self.S, device)
        self.pairs_log = []

    def _replay_alloc(self, mgr, on_prefix, on_step):
        """Drive one manager (product or reference) through prompts, forks and
        continuations; returns the sequence ids in workload order."""
        w = self.w
        seqs = []
        for p in range(self.P):
            parent = mgr.alloc_seq(w.prefix_len)
            on_prefix(mgr, parent, p)
            seqs.append(parent)
            for _ in range(self.n - 1):
                seqs.append(mgr.fork(parent))
        cursor = 0
        for t in range(int(self.cont.max()) if self.S else 0):
            active = [i for i in range(self.S) if self.cont[i] > t]
            cursor = on_step(mgr, [seqs[i] for i in active], cursor) or cursor
        return seqs

    def run(self):
        import paged_kv_cache_404_b200 as pkv
        w, dev = self.w, self.device
        err = torch.zeros(1, dtype=torch.int32, device=dev)
        self.err = err

        # ---- product side (native manager + CUDA kernels)
        def prod_prefix(mgr, seq, p):
            slots = mgr.slots(seq, 0, w.prefix_len)
            sl = slice(p * w.prefix_len, (p + 1) * w.prefix_len)
            pkv.paged_kv_write(self.prefix_k[sl], self.prefix_v[sl], torch.from_numpy(slots).to(dev), self.kp,
                               self.vp, err_count=err)

        def prod_step(mgr, seqs, cursor):
            slots, pairs = mgr.append_tokens(seqs)
            if len(pairs):
                pkv.copy_blocks(self.kp, self.vp, torch.from_numpy(pairs).to(dev), err_count=err)
            n = len(seqs)
            pkv.paged_kv_write(self.cont_k[cursor:cursor + n], self.cont_v[cursor:cursor + n],
                               torch.from_numpy(slots).to(dev), self.kp, self.vp, err_count=err)
            self.pairs_log.append(("p", [tuple(x) for x in pairs.tolist()], slots.tolist()))
            return cursor + n

        self.ids = self._replay_alloc(self.bm, prod_prefix, prod_step)
        slots, pairs = self.bm.append_tokens(self.ids)
        self.step_pairs, self.step_slots = pairs, slots
        if len(pairs):
            pkv.copy_blocks(self.kp, self.vp, torch.from_numpy(pairs).to(dev), err_count=err)
        pkv.paged_kv_write(self.k_new, self.v_new, torch.from_numpy(slots).to(dev), self.kp, self.vp, err_count=err)
        self.lens = np.array([self.bm.seq_len(s) for s in self.ids], dtype=np.int32)
        self.max_blocks = int(max(-(-int(L) // 16) for L in self.lens))
        tabs, _ = self.bm.tables(self.ids, self.max_blocks, pad=-1)
        self.tables = tabs
        self.g_tables = torch.from_numpy(tabs).to(dev)
        self.g_lens = torch.from_numpy(self.lens).to(dev)
        self.max_len = int(self.lens.max())
        self.ws = pkv.decode_workspace(self.S, w.num_heads, w.head_dim, self.max_len, 0)
        self.out = torch.empty_like(self.q)
        pkv.paged_attention_decode(self.out, self.q, self.kp, self.vp, self.g_tables, self.g_lens, w.scale,
                                   self.max_len, self.ws, err_count=err)
        torch.cuda.synchronize()

        # ---- oracle side (reference manager + C oracle), same inputs
        ref_log = []
        pk, pv = to_np_bits(self.prefix_k), to_np_bits(self.prefix_v)
        ck, cv = to_np_bits(self.cont_k), to_np_bits(self.cont_v)

        def ref_prefix(mgr, seq, p):
            sl = slice(p * w.prefix_len, (p + 1) * w.prefix_len)
            oracle.kv_write(pk[sl], pv[sl], oracle.BF16, mgr.slots(seq, 0, w.prefix_len), self.hk, self.hv,
                            oracle.BF16, 16)

        def ref_step(mgr, seqs, cursor):
            res = [mgr.append_token(s) for s in seqs]
            slots = [r[0] for r in res]
            pairs = [r[1] for r in res if r[1] is not None]
            if pairs:
                oracle.copy_blocks(self.hk, self.hv, pairs)
            n = len(seqs)
            oracle.kv_write(ck[cursor:cursor + n], cv[cursor:cursor + n], oracle.BF16, slots, self.hk, self.hv,
                            oracle.BF16, 16)
            ref_log.append(("p", pairs, slots))
            return cursor + n

        self.rids = self._replay_alloc(self.ref, ref_prefix, ref_step)
        res = [self.ref.append_token(s) for s in self.rids]
        self.ref_step_slots = [r[0] for r in res]
        self.ref_step_pairs = [r[1] for r in res if r[1] is not None]
        if self.ref_step_pairs:
            oracle.copy_blocks(self.hk, self.hv, self.ref_step_pairs)
        oracle.kv_write(to_np_bits(self.k_new), to_np_bits(self.v_new), oracle.BF16, self.ref_step_slots, self.hk,
                        self.hv, oracle.BF16, 16)
        self.ref_log = ref_log
        return self

    def oracle_decode(self, sample):
        tabs = np.full((len(sample), self.max_blocks), -1, dtype=np.int32)
        for i, s in enumerate(sample):
            t = self.ref.tables[self.rids[s]]
            tabs[i, :len(t)] = t
        lens = np.array([self.ref.lens[self.rids[s]] for s in sample], dtype=np.int32)
        out, bad = oracle.paged_attention_decode(to_np_bits(self.q)[sample], oracle.BF16, self.hk, self.hv,
                                                 oracle.BF16, tabs, lens, self.w.scale)
        assert bad == 0
        return out
