"""GPU parity of paged_attention_prefill (causal multi-token attention through
block tables) against the oracle.

Prompts are allocated through the block manager (allocate first, then fill the
last block), their K/V written with paged_kv_write at the prompt's slots, into
pools whose every other byte is NaN (bf16 NaN, or the E4M3 NaN code for an FP8
cache), so a read of a slot past a context or of a wrong block shows.  Small cases are compared on every element, the full-size
workload on sampled rows, in the launch configuration the benchmark uses.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests.helpers import assert_close, out_to_f64, to_np_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from paged_kv_cache_404_b200 import build
    build.build()
    assert torch.cuda.is_available()


class PrefillCase:
    """Sequences with context lengths `ctx` whose last `nq` tokens are queries."""

    def __init__(self, Hq, Hkv, ctx, nq, seed, nan_pool=True, cache="bf16", k_growth=None):
        import paged_kv_cache_404_b200 as pkv
        self.w = W.Workload("pf", Hq, Hkv, 128, cache, "bf16", len(ctx), "uniform", 1, 1, seed=seed)
        self.cache = cache
        self.ctx = np.asarray(ctx, np.int32)
        self.nq = np.asarray(nq, np.int32)
        need = int(sum(-(-int(c) // 16) for c in ctx))
        self.NB = need + 9
        rng = np.random.default_rng(seed)
        self.bm = pkv.BlockManager(self.NB, 16, free_order=rng.permutation(self.NB))
        self.ids = [self.bm.alloc_seq(int(c)) for c in ctx]
        self.maxb = max(1, max(-(-int(c) // 16) for c in ctx))
        self.tables, _ = self.bm.tables(self.ids, self.maxb, pad=-1)
        shape = (self.NB, 16, Hkv, 128)
        if nan_pool and cache == "fp8":
            self.kp = torch.full(shape, 0x7F, dtype=torch.uint8, device="cuda")
            self.vp = torch.full(shape, 0xFF, dtype=torch.uint8, device="cuda")
        elif nan_pool:
            self.kp = torch.full(shape, float("nan"), dtype=torch.bfloat16, device="cuda")
            self.vp = torch.full(shape, float("nan"), dtype=torch.bfloat16, device="cuda")
        else:
            self.kp, self.vp, _, _ = W.random_pools(self.w, self.NB, "cuda")
        total = int(self.ctx.sum())
        k, v = W.logical_kv(self.w, total, "cuda", stream=80)
        if k_growth and total:
            # keys that grow along the sequence: token p of a prompt scaled by 1 + p / k_growth
            pos = torch.from_numpy(np.concatenate([np.arange(int(c)) for c in ctx]).astype(np.float32)).cuda()
            k = (k.float() * (1.0 + pos / k_growth).view(-1, *([1] * (k.dim() - 1)))).to(k.dtype)
        # per-tensor FP8 scales amax / 448 of the written tokens (1 for bf16)
        self.k_scale = float(k.abs().max().float().item()) / 448.0 if cache == "fp8" and total else 1.0
        self.v_scale = float(v.abs().max().float().item()) / 448.0 if cache == "fp8" and total else 1.0
        slots = np.concatenate([self.bm.slots(s, 0, int(c)) for s, c in zip(self.ids, ctx)]) if total else []
        if total:
            pkv.paged_kv_write(k, v, torch.from_numpy(np.asarray(slots, np.int64)).cuda(), self.kp, self.vp,
                               self.k_scale, self.v_scale)
        self.qs = np.concatenate([[0], np.cumsum(self.nq)]).astype(np.int32)
        self.q = W.queries(W.scaled(self.w, num_seqs=int(self.qs[-1])), int(self.qs[-1]), "cuda")

    def run(self, max_query_len=None, tables=None):
        import paged_kv_cache_404_b200 as pkv
        self.out = torch.full_like(self.q, 7.0)
        self.err = torch.zeros(1, dtype=torch.int32, device="cuda")
        tabs = self.tables if tables is None else tables
        mq = int(self.nq.max()) if max_query_len is None else max_query_len
        pkv.paged_attention_prefill(self.out, self.q, self.kp, self.vp, torch.from_numpy(tabs).cuda(),
                                    torch.from_numpy(self.ctx).cuda(), torch.from_numpy(self.qs).cuda(),
                                    self.w.scale, mq, err_count=self.err, k_scale=self.k_scale,
                                    v_scale=self.v_scale)
        torch.cuda.synchronize()
        return self.out

    def oracle(self, rows=None, tables=None):
        tabs = self.tables if tables is None else tables
        cdt = oracle.FP8_E4M3 if self.cache == "fp8" else oracle.BF16
        return oracle.paged_attention_prefill(to_np_bits(self.q), oracle.BF16, to_np_bits(self.kp),
                                              to_np_bits(self.vp), cdt, tabs, self.ctx, self.qs,
                                              self.w.scale, self.k_scale, self.v_scale, rows=rows)


RAGGED = ([1, 15, 16, 17, 64, 65, 200, 300, 100, 129, 33],
          [1, 15, 16, 17, 64, 65, 200, 37, 1, 128, 20])


@pytest.mark.parametrize("cache", ["bf16", "fp8"])
def test_growing_keys_move_the_reference_max(cache):
    """Keys whose magnitude grows along the prompt (1 + p / 40): every KV tile's largest
    score exceeds the previous tiles' by more than 2^8 in the exponent, so each row's
    reference maximum moves tile after tile and O is rescaled in TMEM mid-row (the bf16
    kernel computes a tile's probabilities before its maximum is known and redoes them
    there).  Every element against the oracle."""
    c = PrefillCase(16, 4, [700, 520, 300, 129], [700, 400, 300, 1], seed=77, cache=cache, k_growth=40.0)
    got = out_to_f64(c.run())
    ref, bad = c.oracle()
    assert bad == 0 and int(c.err.item()) == 0
    assert np.isfinite(got).all()
    assert_close(got, ref, cache, "prefill growing keys")


@pytest.mark.parametrize("Hq,Hkv", [(8, 8), (16, 4), (64, 8)])
def test_ragged_prompts_every_element(Hq, Hkv):
    """Whole prompts of 1..200 tokens (ragged tails, block and tile edges), a
    prompt after a cached prefix (300 / 37), a one-token step (100 / 1)."""
    c = PrefillCase(Hq, Hkv, *RAGGED, seed=40 + Hq)
    got = out_to_f64(c.run())
    ref, bad = c.oracle()
    assert bad == 0 and int(c.err.item()) == 0
    assert_close(got, ref, "bf16", "prefill G=%d" % (Hq // Hkv))


@pytest.mark.parametrize("Hq,Hkv", [(8, 8), (64, 8)])
def test_fp8_cache_ragged_prompts_every_element(Hq, Hkv):
    """The same ragged prompts over an FP8 E4M3 cache (codes turned into f16 in
    shared memory, per-tensor scales); unowned bytes hold the E4M3 NaN code."""
    c = PrefillCase(Hq, Hkv, *RAGGED, seed=50 + Hq, cache="fp8")
    got = out_to_f64(c.run())
    ref, bad = c.oracle()
    assert bad == 0 and int(c.err.item()) == 0
    assert_close(got, ref, "fp8", "fp8 prefill G=%d" % (Hq // Hkv))


@pytest.mark.parametrize("mode", ["big", "tiny", "mixed"])
@pytest.mark.parametrize("Hq,Hkv", [(8, 8), (64, 8)])
def test_fp8_cache_q_beyond_f16_range(mode, Hq, Hkv):
    """The FP8-cache prompt pass multiplies in f16; every finite bf16 q must
    still give the oracle's result (entries past 65,504, entries below f16's
    normal range, heads of very different magnitudes)."""
    from tests.test_gpu_decode import scale_q_magnitudes
    c = PrefillCase(Hq, Hkv, *RAGGED, seed=60 + Hq, cache="fp8")
    q, kf = scale_q_magnitudes(c.q, mode)
    c.q = q
    c.k_scale *= kf
    got = out_to_f64(c.run())
    ref, bad = c.oracle()
    assert bad == 0 and int(c.err.item()) == 0
    assert_close(got, ref, "fp8", "fp8 prefill q %s G=%d" % (mode, Hq // Hkv))


def test_fp8_cache_long_prompts_sampled_rows():
    """FP8 cache, prompts of 1,000..3,000 tokens (many KV tiles, both staging
    slots reused), 32/8 heads; rows sampled, first and last of every prompt."""
    lens = [3000, 1000, 2047, 1537]
    c = PrefillCase(32, 8, lens, lens, seed=51, nan_pool=False, cache="fp8")
    got = out_to_f64(c.run())
    assert int(c.err.item()) == 0
    rng = np.random.default_rng(52)
    rows = np.sort(rng.choice(int(c.qs[-1]), 40, replace=False))
    rows = np.unique(np.concatenate([rows, c.qs[1:] - 1, c.qs[:-1]]))
    ref, _ = c.oracle(rows=rows)
    assert_close(got[rows], ref[rows], "fp8", "fp8 long prompts")


def test_fp8_cache_bad_ids_are_counted():
    c = PrefillCase(16, 4, [90, 40], [90, 10], seed=53, nan_pool=False, cache="fp8")
    tabs = c.tables.copy()
    tabs[0, 2] = c.NB + 5
    tabs[1, 0] = -3
    got = out_to_f64(c.run(tables=tabs))
    ref, bad = c.oracle(tables=tabs)
    assert bad == 2 and int(c.err.item()) == bad
    assert_close(got, ref, "fp8", "fp8 bad ids")


def test_one_token_rows_equal_decode():
    """nq = 1 is a decode step: the prefill result matches the decode kernel's."""
    import paged_kv_cache_404_b200 as pkv
    c = PrefillCase(32, 8, [700, 33, 1, 4096], [1, 1, 1, 1], seed=41, nan_pool=False)
    got = c.run()
    dec = torch.empty_like(c.q)
    ws = pkv.decode_workspace(4, 32, 128, 4096)
    pkv.paged_attention_decode(dec, c.q, c.kp, c.vp, torch.from_numpy(c.tables).cuda(),
                               torch.from_numpy(c.ctx).cuda(), c.w.scale, 4096, ws)
    torch.cuda.synchronize()
    assert_close(out_to_f64(got), out_to_f64(dec), "bf16", "prefill vs decode")


def test_bad_block_ids_and_lengths_are_counted():
    c = PrefillCase(16, 4, [90, 40, 50], [90, 10, 60], seed=42, nan_pool=False)   # third: nq > ctx
    tabs = c.tables.copy()
    tabs[0, 2] = c.NB + 5          # a bad id inside the first prompt
    tabs[1, 0] = -3                # and in the cached prefix of the second
    got = out_to_f64(c.run(tables=tabs))
    rows = list(range(0, 100))     # the first two sequences' rows
    tabs_ok = tabs[:2]
    ref, bad = oracle.paged_attention_prefill(to_np_bits(c.q)[:100], oracle.BF16, to_np_bits(c.kp),
                                              to_np_bits(c.vp), oracle.BF16, tabs_ok, c.ctx[:2], c.qs[:3],
                                              c.w.scale)
    assert bad == 2
    assert int(c.err.item()) == bad + 1           # + the inconsistent third sequence
    assert_close(got[rows], ref, "bf16", "bad ids")
    assert not got[100:].any()                    # its rows are zeroed


def test_full_size_prefill_sampled_rows():
    """The benchmark's prompt pass (16 prompts of 512..4,096 tokens, 64/8 heads),
    launched exactly as bench.py launches it; rows sampled across the batch."""
    w = W.WORKLOADS["prefill70b"]
    lens = W.context_lens(w)
    c = PrefillCase(w.num_heads, w.num_kv_heads, lens, lens, seed=w.seed, nan_pool=False)
    got = out_to_f64(c.run())
    assert int(c.err.item()) == 0
    rng = np.random.default_rng(43)
    rows = np.sort(rng.choice(int(c.qs[-1]), 48, replace=False))
    rows = np.unique(np.concatenate([rows, c.qs[1:] - 1, c.qs[:-1]]))   # first and last row of every prompt
    ref, _ = c.oracle(rows=rows)
    assert_close(got[rows], ref[rows], "bf16", "prefill70b")


def test_full_size_fp8_prefill_sampled_rows():
    """The FP8-cache prompt pass as bench.py times it (16 prompts of 512..4,096
    tokens, 64/8 heads, scales amax/448 of the prompts' K and V); rows sampled."""
    w = W.WORKLOADS["prefill70b_fp8"]
    lens = W.context_lens(w)
    c = PrefillCase(w.num_heads, w.num_kv_heads, lens, lens, seed=w.seed, nan_pool=False, cache="fp8")
    got = out_to_f64(c.run())
    assert int(c.err.item()) == 0
    rng = np.random.default_rng(47)
    rows = np.sort(rng.choice(int(c.qs[-1]), 48, replace=False))
    rows = np.unique(np.concatenate([rows, c.qs[1:] - 1, c.qs[:-1]]))
    ref, _ = c.oracle(rows=rows)
    assert_close(got[rows], ref[rows], "fp8", "prefill70b_fp8")


@pytest.mark.parametrize("cache", ["bf16", "fp8"])
def test_context_past_the_shared_memory_validity_bits(cache):
    """A 33,000-token context (2,063 blocks): past the 2,048 blocks whose validity
    the kernel keeps in shared memory, block ids are checked per tile from the
    table; a bad id there is skipped and counted once."""
    c = PrefillCase(8, 8, [33000], [200], seed=48, nan_pool=False, cache=cache)
    tabs = c.tables.copy()
    tabs[0, 2055] = -1
    got = out_to_f64(c.run(tables=tabs))
    ref, bad = c.oracle(tables=tabs)
    assert bad == 1 and int(c.err.item()) == 1
    assert_close(got, ref, cache, "33k context %s" % cache)


def test_sequences_without_queries_and_oversized_launch():
    """A sequence with no new tokens between others, and max_query_len above the
    longest: nothing is written for the empty one, the others match the oracle."""
    c = PrefillCase(16, 4, [50, 40, 90], [20, 0, 90], seed=45)
    got = out_to_f64(c.run(max_query_len=300))
    ref, bad = c.oracle()
    assert bad == 0 and int(c.err.item()) == 0
    assert c.qs.tolist() == [0, 20, 20, 110]
    assert_close(got, ref, "bf16", "empty query list")
