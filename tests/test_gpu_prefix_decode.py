"""Shared-prefix decode: sequences that begin with the same physical blocks
read those blocks once for the whole group.

Glossary entry "PagedAttention", section "Compartir bloques entre secuencias":
parallel samples, beams and requests with the same system prompt point at one
copy of the shared prefix.  The grouped decode must give the oracle's result
(the plain definition, within the bf16 tolerance) whatever the hints say.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests.helpers import SharedPrefixReplay, assert_close, out_to_f64, to_np_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from paged_kv_cache_404_b200 import build
    build.build()
    assert torch.cuda.is_available()


def _hdr(ws):
    """(num_items, num_subs, num_members) from the workspace header."""
    h = ws[:32].cpu().view(torch.int32).tolist()
    return h[1], h[5], h[6]


def _grouped(q, kp, vp, tables, lens, scale, max_len, offs, mem, sh, P=0, k_scale=1.0, v_scale=1.0):
    import paged_kv_cache_404_b200 as pkv
    S, Hq, D = q.shape
    ws = pkv.decode_workspace(S, Hq, D, max_len, P, shared=True)
    out = torch.empty_like(q)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    dev = lambda a: torch.as_tensor(np.asarray(a, dtype=np.int32)).cuda()  # noqa: E731
    pkv.paged_attention_decode_shared(out, q, kp, vp, tables, lens, scale, max_len, ws, dev(offs), dev(mem),
                                      dev(sh), k_scale=k_scale, v_scale=v_scale, partition_tokens=P, err_count=err)
    torch.cuda.synchronize()
    return out, int(err.item()), ws


@pytest.fixture(scope="module")
def replay():
    return SharedPrefixReplay(W.WORKLOADS["shared_prefix"]).run()


def test_hints_match_reference_manager(replay):
    rp = replay
    offs, mem, sh = rp.bm.prefix_groups(rp.ids)
    r_offs, r_mem, r_sh = rp.ref.prefix_groups(rp.rids)
    assert offs.tolist() == r_offs and mem.tolist() == r_mem and sh.tolist() == r_sh
    # 64 prompts x 3 samples: one group per prompt, 62 full prefix blocks shared
    assert len(sh) == rp.P and set(sh.tolist()) == {rp.w.prefix_len // 16}
    assert mem.tolist() == list(range(rp.S))


def test_shared_prefix_full_size_matches_oracle(replay):
    rp = replay
    offs, mem, sh = rp.bm.prefix_groups(rp.ids)
    out, err, ws = _grouped(rp.q, rp.kp, rp.vp, rp.g_tables, rp.g_lens, rp.w.scale, rp.max_len, offs, mem, sh)
    assert err == 0
    _, nsubs, nmem = _hdr(ws)
    assert (nsubs, nmem) == (rp.P, rp.S)          # G = 4: three members fit one subgroup
    sample = np.sort(np.random.default_rng(21).choice(rp.S, 30, replace=False))
    assert_close(out_to_f64(out)[sample], rp.oracle_decode(sample), "bf16", "grouped decode")
    # and close to the plain decode everywhere (both are within the tolerance of the exact result)
    assert_close(out_to_f64(out), out_to_f64(rp.out), "bf16", "grouped vs plain")


@pytest.mark.parametrize("P", [16, 64, 256, 1024])
def test_shared_prefix_partition_sizes(P):
    w = W.scaled(W.WORKLOADS["shared_prefix"], num_prompts=6)
    rp = SharedPrefixReplay(w).run()
    offs, mem, sh = rp.bm.prefix_groups(rp.ids)
    out, err, _ = _grouped(rp.q, rp.kp, rp.vp, rp.g_tables, rp.g_lens, w.scale, rp.max_len, offs, mem, sh, P=P)
    assert err == 0
    assert_close(out_to_f64(out), rp.oracle_decode(np.arange(rp.S)), "bf16", "P=%d" % P)


def test_wrong_hints_cost_nothing_but_time():
    """Overlapping groups, members out of range, shared counts far too large,
    members of different prompts in one group: still the oracle's result."""
    w = W.scaled(W.WORKLOADS["shared_prefix"], num_prompts=8)
    rp = SharedPrefixReplay(w).run()
    S = rp.S
    rng = np.random.default_rng(5)
    offs, mem, sh = [0], [], []
    for g in range(12):
        n = int(rng.integers(1, 7))
        members = rng.integers(-3, S + 3, size=n).tolist()
        mem += members
        offs.append(len(mem))
        sh.append(int(rng.choice([0, 1, 30, 62, 63, 10 ** 6])))
    # one honest group too, listed after a group that already claimed one of its members
    mem += [0, 1, 2]
    offs.append(len(mem))
    sh.append(62)
    out, err, _ = _grouped(rp.q, rp.kp, rp.vp, rp.g_tables, rp.g_lens, w.scale, rp.max_len, offs, mem, sh)
    assert err == 0
    assert_close(out_to_f64(out), rp.oracle_decode(np.arange(S)), "bf16", "wrong hints")


def _fork_family(w, n_kids, prefix_tokens, extra, seed):
    """A parent of `prefix_tokens` tokens, n_kids forks, then extra[i] tokens
    appended to member i (copy-on-write as needed); pools of random data."""
    import paged_kv_cache_404_b200 as pkv
    NB = 256
    bm = pkv.BlockManager(NB, 16, free_order=np.random.default_rng(seed).permutation(NB))
    ids = [bm.alloc_seq(prefix_tokens)]
    ids += [bm.fork(ids[0]) for _ in range(n_kids)]
    kp, vp, _, _ = W.random_pools(w, NB, "cuda")
    for i, s in enumerate(ids):
        for _ in range(extra[i]):
            _, pair = bm.append_token(s)
            if pair:
                pkv.copy_blocks(kp, vp, torch.tensor([pair], dtype=torch.int64, device="cuda"))
    lens = np.array([bm.seq_len(s) for s in ids], dtype=np.int32)
    maxb = int(max(-(-int(L) // 16) for L in lens))
    tabs, _ = bm.tables(ids, maxb, pad=-1)
    return bm, ids, kp, vp, tabs, lens


@pytest.mark.parametrize("extra", [[0, 0, 0], [0, 5, 40], [17, 0, 300]])
def test_gqa8_group_of_three_splits_into_subgroups(extra):
    """G = 8 query heads per KV head: two members fill the 16 score columns, so a
    group of three becomes subgroups of 1 and 2.  With no appended tokens the
    whole context is shared and the subgroup items write the outputs directly."""
    w = W.scaled(W.WORKLOADS["gqa70b"], num_seqs=3)
    bm, ids, kp, vp, tabs, lens = _fork_family(w, 2, 128, extra, seed=11)
    offs, mem, sh = bm.prefix_groups(ids)
    assert offs.tolist() == [0, 3] and sh.tolist() == [8]
    q = W.queries(w, 3, "cuda")
    g_t, g_l = torch.from_numpy(tabs).cuda(), torch.from_numpy(lens).cuda()
    max_len = int(lens.max())
    out, err, ws = _grouped(q, kp, vp, g_t, g_l, w.scale, max_len, offs, mem, sh)
    assert err == 0
    _, nsubs, nmem = _hdr(ws)
    assert (nsubs, nmem) == (2, 3)
    ref, bad = oracle.paged_attention_decode(to_np_bits(q), oracle.BF16, to_np_bits(kp), to_np_bits(vp),
                                             oracle.BF16, tabs, lens, w.scale)
    assert bad == 0
    assert_close(out_to_f64(out), ref, "bf16", "gqa8 subgroups %s" % extra)


def test_more_subgroups_than_the_plans_shared_memory_copies():
    """4,200 prompts of 17-40 tokens, each forked once: 4,200 two-member groups
    sharing their full blocks (one or two; G = 8: two members per subgroup), more
    subgroups than the plan keeps in shared memory (4,096); every element against
    the oracle."""
    import paged_kv_cache_404_b200 as pkv
    R = 4200
    w = W.scaled(W.WORKLOADS["gqa70b"], num_seqs=2 * R, num_heads=16, num_kv_heads=2)
    NB = 3 * R + 16
    rng = np.random.default_rng(4200)
    bm = pkv.BlockManager(NB, 16, free_order=rng.permutation(NB))
    ids = []
    for r in range(R):
        parent = bm.alloc_seq(int(rng.integers(17, 41)))
        ids += [parent, bm.fork(parent)]
    lens = np.array([bm.seq_len(s) for s in ids], dtype=np.int32)
    tabs, _ = bm.tables(ids, 3, pad=-1)
    offs, mem, sh = bm.prefix_groups(ids)
    assert len(offs) == R + 1 and all(int(x) in (1, 2) for x in sh)
    kp, vp, _, _ = W.random_pools(w, NB, "cuda")
    q = W.queries(w, 2 * R, "cuda")
    g_t, g_l = torch.from_numpy(tabs).cuda(), torch.from_numpy(lens).cuda()
    out, err, ws = _grouped(q, kp, vp, g_t, g_l, w.scale, int(lens.max()), offs, mem, sh)
    assert err == 0
    _, nsubs, nmem = _hdr(ws)
    assert (nsubs, nmem) == (R, 2 * R)
    ref, bad = oracle.paged_attention_decode(to_np_bits(q), oracle.BF16, to_np_bits(kp), to_np_bits(vp),
                                             oracle.BF16, tabs, lens, w.scale)
    assert bad == 0
    assert_close(out_to_f64(out), ref, "bf16", "4,200 subgroups")


def test_fp8_cache_ignores_hints_and_equals_plain_decode():
    import paged_kv_cache_404_b200 as pkv
    w = W.scaled(W.WORKLOADS["fp8_long"], num_seqs=3)
    bm, ids, kp, vp, tabs, lens = _fork_family(w, 2, 600, [0, 3, 70], seed=12)
    _, _, ks, vs = W.random_pools(w, 4, "cuda")
    offs, mem, sh = bm.prefix_groups(ids)
    q = W.queries(w, 3, "cuda")
    g_t, g_l = torch.from_numpy(tabs).cuda(), torch.from_numpy(lens).cuda()
    max_len = int(lens.max())
    out, err, ws = _grouped(q, kp, vp, g_t, g_l, w.scale, max_len, offs, mem, sh, k_scale=ks, v_scale=vs)
    assert err == 0 and _hdr(ws)[1] == 0
    plain = torch.empty_like(q)
    ws2 = pkv.decode_workspace(3, w.num_heads, w.head_dim, max_len)
    pkv.paged_attention_decode(plain, q, kp, vp, g_t, g_l, w.scale, max_len, ws2, ks, vs)
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), plain.view(torch.int16))


def test_prefix_cache_end_to_end():
    """Requests over three system prompts: each request's prompt is allocated
    through the prefix cache, only its uncached tokens are written, and the
    grouped decode reads the shared blocks once.  Pools equal the oracle's
    byte for byte (same managers' decisions on both sides), and the outputs
    equal the oracle's attention over each request's whole logical stream."""
    import paged_kv_cache_404_b200 as pkv
    w = W.scaled(W.WORKLOADS["shared_prefix"], num_prompts=3)
    rng = np.random.default_rng(77)
    sys_lens = [300, 517, 64]
    systems = [rng.integers(0, 30000, size=n).tolist() for n in sys_lens]
    reqs = [(p, rng.integers(0, 30000, size=int(rng.integers(0, 200))).tolist()) for p in range(3) for _ in range(4)]
    rng.shuffle(reqs)
    NB = 400
    order = W.free_order(w, NB)
    bm, ref = pkv.BlockManager(NB, 16, free_order=order), oracle.RefBlockManager(NB, 16, free_order=order)
    bm.set_prefix_cache(True)
    ref.set_prefix_cache(True)
    kp, vp = W.stale_fill(w, NB, "cuda")
    hk, hv = to_np_bits(kp).copy(), to_np_bits(vp).copy()
    # K/V of a system prompt's tokens are the same in every request that starts with it
    sys_kv = [W.logical_kv(w, n, "cuda", stream=70 + p) for p, n in enumerate(sys_lens)]
    ids, rids, logical = [], [], []
    for r, (p, user) in enumerate(reqs):
        toks = systems[p] + user
        s, cached = bm.alloc_seq_tokens(toks)
        rs, rcached = ref.alloc_seq_tokens(toks)
        assert cached == rcached and bm.block_table(s).tolist() == ref.tables[rs]
        uk, uv = W.logical_kv(w, len(user), "cuda", stream=100 + r)
        k = torch.cat([sys_kv[p][0], uk]) if len(user) else sys_kv[p][0]
        v = torch.cat([sys_kv[p][1], uv]) if len(user) else sys_kv[p][1]
        n = len(toks)
        if n > cached:
            slots = bm.slots(s, cached, n - cached)
            pkv.paged_kv_write(k[cached:].contiguous(), v[cached:].contiguous(), torch.from_numpy(slots).cuda(),
                               kp, vp)
            oracle.kv_write(to_np_bits(k[cached:]), to_np_bits(v[cached:]), oracle.BF16,
                            np.asarray(ref.slots(rs, cached, n - cached), np.int64), hk, hv, oracle.BF16, 16)
        ids.append(s)
        rids.append(rs)
        logical.append((to_np_bits(k), to_np_bits(v)))
    torch.cuda.synchronize()
    assert bm.num_cached_blocks() == len(ref.cache) > 0
    assert np.array_equal(to_np_bits(kp), hk) and np.array_equal(to_np_bits(vp), hv)

    lens = np.array([bm.seq_len(s) for s in ids], dtype=np.int32)
    maxb = int(max(-(-int(L) // 16) for L in lens))
    tabs, _ = bm.tables(ids, maxb, pad=-1)
    offs, mem, sh = bm.prefix_groups(ids)
    assert len(sh) == 3 and sorted(sh.tolist()) == sorted(n // 16 for n in sys_lens)
    q = W.queries(w, len(ids), "cuda")
    out, err, _ = _grouped(q, kp, vp, torch.from_numpy(tabs).cuda(), torch.from_numpy(lens).cuda(), w.scale,
                           int(lens.max()), offs, mem, sh)
    assert err == 0
    # oracle: each request's whole logical K/V laid out contiguously in a pool of its own
    for i, (k, v) in enumerate(logical):
        n = k.shape[0]
        nb = -(-n // 16)
        ck = np.zeros((nb * 16,) + k.shape[1:], dtype=k.dtype)
        cv = np.zeros_like(ck)
        ck[:n], cv[:n] = k, v
        ck, cv = ck.reshape((nb, 16) + k.shape[1:]), cv.reshape((nb, 16) + k.shape[1:])
        ref_out, bad = oracle.paged_attention_decode(to_np_bits(q)[i:i + 1], oracle.BF16, ck, cv, oracle.BF16,
                                                     np.arange(nb, dtype=np.int32)[None], lens[i:i + 1], w.scale)
        assert bad == 0
        assert_close(out_to_f64(out)[i:i + 1], ref_out, "bf16", "request %d" % i)


@pytest.mark.parametrize("Hq,Hkv,D,dtype", [(2, 2, 64, "f32"), (16, 4, 64, "bf16"), (32, 2, 128, "bf16")])
def test_hints_ignored_where_no_grouped_kernel_exists(Hq, Hkv, D, dtype):
    """fp32, head_dim 64 and 16 query heads per KV head have no grouped kernel:
    the shared entry point runs the plain decode (in its own workspace layout)
    and gives the plain decode's bits."""
    import paged_kv_cache_404_b200 as pkv
    w = W.Workload("hint", Hq, Hkv, D, dtype, dtype, 3, "uniform", 1, 1, seed=13)
    bm, ids, kp, vp, tabs, lens = _fork_family(w, 2, 150, [0, 7, 60], seed=13)
    offs, mem, sh = bm.prefix_groups(ids)
    assert len(sh) == 1
    q = W.queries(w, 3, "cuda")
    g_t, g_l = torch.from_numpy(tabs).cuda(), torch.from_numpy(lens).cuda()
    max_len = int(lens.max())
    out, err, ws = _grouped(q, kp, vp, g_t, g_l, w.scale, max_len, offs, mem, sh)
    assert err == 0 and _hdr(ws)[1] == 0
    plain = torch.empty_like(q)
    ws2 = pkv.decode_workspace(3, Hq, D, max_len)
    pkv.paged_attention_decode(plain, q, kp, vp, g_t, g_l, w.scale, max_len, ws2)
    torch.cuda.synchronize()
    bits = torch.int32 if dtype == "f32" else torch.int16
    assert torch.equal(out.view(bits), plain.view(bits))
