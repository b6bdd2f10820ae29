"""GPU parity of paged_attention_decode (+ the step's KV write) against the oracle.

Small cases and the full-size workloads are compared on every output element,
the full-size ones in the launch configuration the benchmark uses (automatic
partitioning).
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests.helpers import DecodeCase, ORC_DT, assert_close, out_to_f64, to_np_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from paged_kv_cache_404_b200 import build
    build.build()
    assert torch.cuda.is_available()


def _run(case, P=0):
    case.snapshot_pools()
    case.run_gpu(partition_tokens=P)
    case.run_oracle()
    case.check_written_rows()
    return case.compare()


# ------------------------------------------------------------------ tiny workload (fp32)

def test_tiny_workload_fills_by_writes_and_matches():
    """Tiny workload: every token written through the KV write (as the worked
    example stores its keys), then one decode; whole pools compared byte for byte."""
    import paged_kv_cache_404_b200 as pkv
    w = W.WORKLOADS["tiny"]
    lens = W.context_lens(w)
    NB = W.pool_blocks(w, 0)
    order = W.free_order(w, NB)
    bm, ref = pkv.BlockManager(NB, 16, free_order=order), oracle.RefBlockManager(NB, 16, free_order=order)
    ids, rids = {}, {}
    for s in W.allocation_order(w):
        ids[s], rids[s] = bm.alloc_seq(int(lens[s])), ref.alloc_seq(int(lens[s]))
    assert bm.block_table(ids[3]).tolist() == [41, 7, 19] == ref.tables[rids[3]]
    total = int(lens.sum())
    k, v = W.logical_kv(w, total, "cuda", stream=50)
    slots = np.concatenate([bm.slots(ids[s], 0, int(lens[s])) for s in range(4)])
    rslots = np.concatenate([ref.slots(rids[s], 0, int(lens[s])) for s in range(4)])
    assert np.array_equal(slots, rslots)
    kp, vp = W.stale_fill(w, NB, "cuda")
    hk, hv = to_np_bits(kp).copy(), to_np_bits(vp).copy()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pkv.paged_kv_write(k, v, torch.from_numpy(slots).cuda(), kp, vp, err_count=err)
    oracle.kv_write(to_np_bits(k), to_np_bits(v), oracle.F32, rslots, hk, hv, oracle.F32, 16)
    assert np.array_equal(to_np_bits(kp), hk) and np.array_equal(to_np_bits(vp), hv)
    # the 40-token request reads back intact through its table
    off = int(lens[:3].sum())
    assert np.array_equal(oracle.gather(hk, ref.tables[rids[3]], 40, 16), to_np_bits(k)[off:off + 40])
    tabs, tl = bm.tables([ids[s] for s in range(4)], 3, pad=-1)
    assert np.array_equal(tl, lens)
    q = W.queries(w, 4, "cuda")
    for P in (0, 16, 32):
        ws = pkv.decode_workspace(4, 2, 64, 40, P)
        out = torch.empty_like(q)
        pkv.paged_attention_decode(out, q, kp, vp, torch.from_numpy(tabs).cuda(), torch.from_numpy(lens).cuda(),
                                   w.scale, 40, ws, partition_tokens=P, err_count=err)
        rtab = np.full((4, 3), -1, np.int32)
        for s in range(4):
            rtab[s, :len(ref.tables[rids[s]])] = ref.tables[rids[s]]
        ref_out, bad = oracle.paged_attention_decode(to_np_bits(q), oracle.F32, hk, hv, oracle.F32, rtab, lens,
                                                     w.scale)
        assert bad == 0
        assert_close(out_to_f64(out), ref_out, "f32", "tiny P=%d" % P)
    assert int(err.item()) == 0


# ------------------------------------------------------------------ small cases, every element

SMALL = {
    "mha13b": dict(num_seqs=6),
    "gqa70b": dict(num_seqs=5),
    "shared_prefix_shape": dict(),
    "fp8_long": dict(num_seqs=6),
}


def _small_workload(name):
    if name == "shared_prefix_shape":
        base = W.WORKLOADS["shared_prefix"]
        return W.scaled(base, lens="uniform", len_lo=1, len_hi=700, num_seqs=7)
    return W.scaled(W.WORKLOADS[name], **SMALL[name])


RAGGED = [1, 2, 15, 16, 17, 31, 33, 100, 255, 257, 511, 700]


@pytest.mark.parametrize("name", sorted(SMALL))
@pytest.mark.parametrize("P", [0, 16, 48, 256, 4096])
def test_small_cases_every_element(name, P):
    w = _small_workload(name)
    rng = np.random.default_rng(hash((name, P)) % 2**32)
    lens = rng.choice(RAGGED, size=w.num_seqs if w.lens != "shared" else 7).astype(np.int32)
    _run(DecodeCase(w, lens=lens), P)


@pytest.mark.parametrize("P", [16, 48])
def test_merge_of_few_and_many_rows_past_its_first_round(P):
    """The merge loads 16 partitions per warp in its first round when it has at most
    32 (sequence, query head) rows per SM, 8 when it has more; both forms here, with
    more partitions than that first round (16- and 48-token pieces of ragged contexts
    up to 700 tokens), every element against the oracle."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    for rows in (sms * 8, sms * 40):
        S = -(-rows // 64)
        w = W.scaled(W.WORKLOADS["gqa70b"], num_seqs=S)
        rng = np.random.default_rng(S * 1000 + P)
        lens = rng.choice(RAGGED, size=S).astype(np.int32)
        lens[0] = 700
        _run(DecodeCase(w, lens=lens), P)


@pytest.mark.parametrize("P", [0, 16])
def test_batch_past_the_plans_shared_memory_copies(P):
    """4,500 sequences: the plan keeps the block counts of the first 4,096 in shared
    memory and reads the others' from global memory; every element against the
    oracle (contexts of 1-200 tokens, one KV head for eight query heads)."""
    w = W.scaled(W.WORKLOADS["gqa70b"], num_seqs=4500, num_heads=8, num_kv_heads=1)
    rng = np.random.default_rng(4500 + P)
    lens = rng.integers(1, 201, size=4500).astype(np.int32)
    lens[-1] = 200
    _run(DecodeCase(w, lens=lens), P)


@pytest.mark.parametrize("G,D", [(1, 64), (2, 128), (4, 128), (8, 64), (8, 128), (16, 128), (12, 128), (3, 64)])
def test_group_sizes_and_head_dims(G, D):
    w = W.scaled(W.WORKLOADS["gqa70b"], num_heads=2 * G, num_kv_heads=2, head_dim=D, num_seqs=4)
    _run(DecodeCase(w, lens=np.array([5, 16, 129, 300], np.int32)), 0)
    _run(DecodeCase(w, lens=np.array([5, 16, 129, 300], np.int32)), 64)


@pytest.mark.parametrize("G", [1, 4, 8, 16])
def test_fp8_group_sizes(G):
    w = W.scaled(W.WORKLOADS["fp8_long"], num_heads=2 * G, num_kv_heads=2, num_seqs=4)
    _run(DecodeCase(w, lens=np.array([1, 17, 250, 1000], np.int32)), 0)


# ------------------------------------------------------------------ full-size workloads (every element)

def test_full_mha13b_every_element():
    w = W.WORKLOADS["mha13b"]
    case = DecodeCase(w)
    _run(case, 0)


def test_full_gqa70b_every_element():
    """The benchmark's headline batch (256 x 4,096 tokens, 64/8 heads, 4 GiB of
    K/V) in its launch configuration, every output element against the oracle."""
    _run(DecodeCase(W.WORKLOADS["gqa70b"]), 0)


def test_full_fp8_long_every_element():
    """All 128 sequences of the FP8 workload (contexts 256..32,768, split
    partitions and their merge), every output element against the oracle."""
    _run(DecodeCase(W.WORKLOADS["fp8_long"]), 0)


# ------------------------------------------------------------------ FP8 cache: q of any finite bf16 magnitude

# Powers of two per query head (exact in bf16): far above and far below 1.
HEAD_EXP = (17, -20, 8, 0, -8, 12, 3, -14)


def scale_q_magnitudes(q, mode):
    """q (bf16, [..., heads, head_dim]) rescaled by powers of two; returns the new
    tensor and the factor for k_scale that keeps scores in a useful range.
      big:   every entry x 2^12, and one entry of head 1 set to 70,000 (past f16's 65,504)
      tiny:  every entry x 2^-20, the K cache x 2^20 (scores unchanged, q below f16's normal range)
      mixed: head h x 2^HEAD_EXP[h % 8], one entry of head 0 set to -70,000"""
    x = q.float()
    H = x.shape[-2]
    if mode == "big":
        x = x * 2.0 ** 12
        x[..., 1 % H, 5] = 70000.0
        return x.to(torch.bfloat16), 1.0
    if mode == "tiny":
        return (x * 2.0 ** -20).to(torch.bfloat16), 2.0 ** 20
    f = torch.tensor([2.0 ** HEAD_EXP[h % 8] for h in range(H)], device=x.device)
    x = x * f[:, None]
    x[..., 0, 7] = -70000.0
    return x.to(torch.bfloat16), 1.0


@pytest.mark.parametrize("mode", ["big", "tiny", "mixed"])
@pytest.mark.parametrize("G", [4, 8, 16])
def test_fp8_q_beyond_f16_range(mode, G):
    """The FP8 decode multiplies in f16; q is bf16, whose range f16 does not
    span.  Every finite bf16 q must still give the oracle's result: entries past
    65,504, entries below f16's normal range, and heads of very different
    magnitudes in one group (each head's scaling lands on its own score column)."""
    w = W.scaled(W.WORKLOADS["fp8_long"], num_heads=2 * G, num_kv_heads=2, num_seqs=4)
    for P in (0, 64):
        case = DecodeCase(w, lens=np.array([1, 17, 250, 1000], np.int32))
        case.q, kf = scale_q_magnitudes(case.q, mode)
        case.k_scale *= kf
        _run(case, P)


# ------------------------------------------------------------------ edge cases

def test_empty_and_single_token_and_maximum():
    w = W.scaled(W.WORKLOADS["gqa70b"], num_seqs=5)
    lens = np.array([0, 1, 16, 0, 2048], dtype=np.int32)
    case = DecodeCase(w, lens=lens)
    _run(case, 0)
    out = out_to_f64(case.out)
    assert np.all(out[0] == 0) and np.all(out[3] == 0)
    # len 1: exactly the value row of the single token (bf16 in, bf16 out)
    v_row = to_np_bits(case.v_new)[1]
    got = to_np_bits(case.out)[1].reshape(8, 8, 128)
    assert np.array_equal(got, np.broadcast_to(v_row[:, None, :], got.shape))


def test_million_token_context_every_element():
    """A context of 2^20 tokens (65,536 blocks, 4 GiB of K/V in the pool) beside a
    5-token and a 70,001-token one: automatic partitions, then 64-token partitions
    (16,384 partials merged per row of the long context); every element against
    the oracle."""
    w = W.scaled(W.WORKLOADS["gqa70b"], num_seqs=3)
    case = DecodeCase(w, lens=np.array([1 << 20, 5, 70001], np.int32))
    _run(case, 0)
    _run(case, 64)
    assert int(case.g_err.item()) == 0


def test_maximum_table_width_is_respected():
    """A context that uses every table entry (len == max_blocks * 16)."""
    w = W.scaled(W.WORKLOADS["mha13b"], num_seqs=3, num_heads=4, num_kv_heads=4)
    case = DecodeCase(w, lens=np.array([64, 64, 64], np.int32))
    assert case.max_blocks == 4
    _run(case, 32)


def test_stale_nan_tail_is_ignored():
    """Slots past the context in a sequence's last block hold NaN: no effect."""
    w = W.scaled(W.WORKLOADS["gqa70b"], num_seqs=4)
    lens = np.array([5, 21, 40, 77], np.int32)
    case = DecodeCase(w, lens=lens)
    case.snapshot_pools()
    case.run_gpu()
    before = case.out.clone()
    nan = torch.tensor(0x7FC0, dtype=torch.int16).view(torch.bfloat16)
    for s, L in enumerate(lens):
        last = int(case.tables[s][(L - 1) // 16])
        case.k_pool[last, L % 16:] = nan
        case.v_pool[last, L % 16:] = nan
    import paged_kv_cache_404_b200 as pkv
    out = torch.empty_like(case.q)
    pkv.paged_attention_decode(out, case.q, case.k_pool, case.v_pool, case.g_tables, case.g_lens, w.scale,
                               case.max_len, case.ws)
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), before.view(torch.int16))


def test_fp8_nan_codes_in_tail_are_ignored():
    w = W.scaled(W.WORKLOADS["fp8_long"], num_seqs=3)
    lens = np.array([3, 30, 260], np.int32)
    case = DecodeCase(w, lens=lens)
    case.snapshot_pools()
    case.run_gpu()
    before = case.out.clone()
    for s, L in enumerate(lens):
        last = int(case.tables[s][(L - 1) // 16])
        case.k_pool[last, L % 16:] = 0x7F
        case.v_pool[last, L % 16:] = 0xFF
    import paged_kv_cache_404_b200 as pkv
    out = torch.empty_like(case.q)
    pkv.paged_attention_decode(out, case.q, case.k_pool, case.v_pool, case.g_tables, case.g_lens, w.scale,
                               case.max_len, case.ws, case.k_scale, case.v_scale)
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), before.view(torch.int16))


def test_placement_permutation_is_bitwise_invariant_on_gpu():
    import paged_kv_cache_404_b200 as pkv
    w = W.scaled(W.WORKLOADS["gqa70b"], num_seqs=6)
    case = DecodeCase(w, lens=np.array([7, 100, 333, 1024, 1500, 2049], np.int32))
    case.run_gpu()
    perm = torch.randperm(case.NB, generator=torch.Generator().manual_seed(3)).cuda()
    kp2 = torch.empty_like(case.k_pool)
    vp2 = torch.empty_like(case.v_pool)
    kp2[perm] = case.k_pool
    vp2[perm] = case.v_pool
    t = case.g_tables.long()
    t2 = torch.where(t >= 0, perm[t.clamp(min=0)], t).int()
    for P in (0, 64):
        ws = pkv.decode_workspace(case.S, w.num_heads, w.head_dim, case.max_len, P)
        a, b = torch.empty_like(case.q), torch.empty_like(case.q)
        pkv.paged_attention_decode(a, case.q, case.k_pool, case.v_pool, case.g_tables, case.g_lens, w.scale,
                                   case.max_len, ws, partition_tokens=P)
        pkv.paged_attention_decode(b, case.q, kp2, vp2, t2, case.g_lens, w.scale, case.max_len, ws,
                                   partition_tokens=P)
        torch.cuda.synchronize()
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_repeated_calls_are_bitwise_deterministic():
    import paged_kv_cache_404_b200 as pkv
    w = W.scaled(W.WORKLOADS["fp8_long"], num_seqs=16)
    case = DecodeCase(w)
    case.run_gpu()
    first = case.out.clone()
    for _ in range(3):
        pkv.paged_attention_decode(case.out, case.q, case.k_pool, case.v_pool, case.g_tables, case.g_lens,
                                   w.scale, case.max_len, case.ws, case.k_scale, case.v_scale)
    torch.cuda.synchronize()
    assert torch.equal(case.out.view(torch.int16), first.view(torch.int16))


def test_invalid_block_ids_are_skipped_and_counted():
    import paged_kv_cache_404_b200 as pkv
    w = W.scaled(W.WORKLOADS["gqa70b"], num_seqs=3)
    case = DecodeCase(w, lens=np.array([40, 40, 40], np.int32))
    case.snapshot_pools()
    case.run_gpu()
    tabs = case.tables.copy()
    tabs[1, 1] = case.NB + 5
    tabs[2, 0] = -3
    g_t = torch.from_numpy(tabs).cuda()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.empty_like(case.q)
    for P in (0, 16):
        err.zero_()
        ws = pkv.decode_workspace(case.S, w.num_heads, w.head_dim, case.max_len, P)
        pkv.paged_attention_decode(out, case.q, case.k_pool, case.v_pool, g_t, case.g_lens, w.scale,
                                   case.max_len, ws, partition_tokens=P, err_count=err)
        torch.cuda.synchronize()
        assert int(err.item()) == 2
        # oracle semantics for the same bad ids: the tokens of those blocks are left out
        case.run_oracle()
        rt = np.full((3, case.max_blocks), -1, np.int32)
        for s in range(3):
            rt[s, :len(case.ref.tables[case.rids[s]])] = case.remap[case.ref.tables[case.rids[s]]]
        rt[1, 1] = case.h_k.shape[0] + 5
        rt[2, 0] = -3
        ref, bad = oracle.paged_attention_decode(to_np_bits(case.q), ORC_DT["bf16"], case.h_k, case.h_v,
                                                 ORC_DT["bf16"], rt, case.lens, w.scale)
        assert bad == 2
        assert_close(out_to_f64(out), ref, "bf16", "bad ids P=%d" % P)


def test_bad_context_lengths_are_clamped_and_counted():
    import paged_kv_cache_404_b200 as pkv
    w = W.scaled(W.WORKLOADS["gqa70b"], num_seqs=3)
    case = DecodeCase(w, lens=np.array([40, 40, 40], np.int32))
    case.run_gpu()
    lens = torch.tensor([40, -5, 10**6], dtype=torch.int32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.empty_like(case.q)
    pkv.paged_attention_decode(out, case.q, case.k_pool, case.v_pool, case.g_tables, lens, w.scale, 40, case.ws,
                               err_count=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 2
    assert torch.equal(out[0].view(torch.int16), case.out[0].view(torch.int16))
    assert torch.all(out[1] == 0)
    assert torch.equal(out[2].view(torch.int16), case.out[2].view(torch.int16))   # clamped to 40
