"""Pins of the CPU oracle against what the pages and the mathematics fix.

CPU only.  None of these re-types the oracle's formula: they use the pages'
worked example and printed numbers, closed forms of softmax attention, a
brute-force route through a different representation (contiguous numpy arrays
and a library softmax), invariants (placement, partitioning, sharing) and the
E4M3 format as decoded by a library.
"""
import json
import math
import os

import numpy as np
import pytest
import torch
from scipy.special import softmax as sp_softmax

import oracle
from oracle import RefBlockManager

F32, BF16, FP8 = oracle.F32, oracle.BF16, oracle.FP8_E4M3


# ---------------------------------------------------------------- worked example

def test_worked_example(golden_dir):
    """Glossary entry 'PagedAttention', worked PyTorch example and its printed output."""
    g = json.load(open(os.path.join(golden_dir, "worked_example.json")))
    bs, D, NB = g["block_size"], g["head_dim"], g["pool_blocks"]
    bm = RefBlockManager(NB, bs, free_order=g["free_blocks"])
    seq = bm.alloc_seq(g["num_tokens"])
    table = bm.tables[seq]
    assert len(table) == g["blocks_needed"]
    assert table == g["expected_block_table"]
    assert list(bm.free) == g["expected_free_after"]
    # store the keys through the table, read them back through it
    keys = torch.randn(g["num_tokens"], 1, D, generator=torch.Generator().manual_seed(0)).numpy()
    pool = np.zeros((NB, bs, 1, D), dtype=np.float32)
    other = np.zeros_like(pool)
    slots = np.array(bm.slots(seq, 0, g["num_tokens"]), dtype=np.int64)
    assert oracle.kv_write(keys, keys, F32, slots, pool, other, F32, bs) == 0
    gathered = oracle.gather(pool, table, g["num_tokens"], bs)
    assert np.array_equal(gathered, keys) == g["keys_intact"]
    assert len(table) * bs - g["num_tokens"] == g["unused_slots_paged"]
    assert g["reservation_tokens"] - g["num_tokens"] == g["unused_slots_reserved"]
    # derived slot values: token 0 -> block 41, token 16 -> block 7, token 39 -> block 19 slot 7
    assert slots[0] == 41 * 16 and slots[16] == 7 * 16 and slots[39] == 19 * 16 + 7
    # the last block holds 8 tokens; only blocks 41, 7, 19 were touched
    touched = sorted(set(int(s) // bs for s in slots))
    assert touched == [7, 19, 41]
    assert np.count_nonzero(pool.reshape(NB, -1).any(axis=1)) == 3


def test_tiny_workload_tables():
    """The tiny workload starts its free list like the worked example."""
    import workloads as W
    w = W.WORKLOADS["tiny"]
    lens = W.context_lens(w)
    fo = W.free_order(w, W.pool_blocks(w, 0))
    assert list(fo[:5]) == [41, 7, 19, 2, 33] and sorted(fo) == list(range(64))
    bm = RefBlockManager(64, 16, free_order=fo)
    ids = {}
    for s in W.allocation_order(w):
        ids[s] = bm.alloc_seq(int(lens[s]))
    assert bm.tables[ids[3]] == [41, 7, 19]
    assert bm.tables[ids[0]] == [2] and bm.tables[ids[1]] == [33]
    assert len(bm.tables[ids[2]]) == 1 and bm.tables[ids[2]][0] == fo[5]
    assert bm.num_free() == 64 - 6


# ---------------------------------------------------------------- memory arithmetic

def test_memory_arithmetic(golden_dir):
    m = json.load(open(os.path.join(golden_dir, "memory_arithmetic.json")))
    for key in ("llama13b_sequence", "llama31_70b_sequence"):
        c = m[key]
        b = oracle.kv_cache_bytes(c["layers"], c["kv_heads"], c["head_dim"], c["elem_bytes"], c["tokens"])
        assert abs(b / 1e9 - c["page_value_gb"]) <= c["page_rounding_gb"], (key, b)
    c = m["llama31_70b_256_users"]
    b = oracle.kv_cache_bytes(c["layers"], c["kv_heads"], c["head_dim"], c["elem_bytes"], c["tokens"])
    assert b == 320 * 2**30  # exact: 343.6 GB
    assert abs(b / 1e9 - c["page_value_gb"]) / c["page_value_gb"] <= c["page_relative_slack"]
    c = m["internal_fragmentation"]
    assert round(100 * (1 - c["used"] / c["reserved"])) == c["page_percent"]
    fp8 = oracle.kv_cache_bytes(80, 8, 128, 1, 4096)
    bf16 = oracle.kv_cache_bytes(80, 8, 128, 2, 4096)
    assert fp8 / bf16 == m["fp8_half"]["ratio"]


# ---------------------------------------------------------------- attention helpers

def _build(lens, Hq, Hkv, D, seed, NB=None, bs=16, dtype=np.float64):
    """Random fp32 q and pools with a random placement; returns pieces + logical K/V."""
    rng = np.random.default_rng(seed)
    S = len(lens)
    nblk = [-(-L // bs) for L in lens]
    NB = NB or (sum(nblk) + 5)
    perm = rng.permutation(NB)
    maxb = max(1, max(nblk))
    tables = np.full((S, maxb), -1, dtype=np.int32)
    o = 0
    for s in range(S):
        tables[s, :nblk[s]] = perm[o:o + nblk[s]]
        o += nblk[s]
    kp = rng.standard_normal((NB, bs, Hkv, D)).astype(np.float32)
    vp = rng.standard_normal((NB, bs, Hkv, D)).astype(np.float32)
    q = rng.standard_normal((S, Hq, D)).astype(np.float32)
    return q, kp, vp, tables, np.array(lens, dtype=np.int32)


def _contiguous_reference(q, kp, vp, tables, lens, scale, bs=16):
    """Brute force through another route: rebuild each sequence's contiguous
    K and V with numpy fancy indexing (pool[table].reshape(...)[:len], as the
    worked example reads a request back) and take a library softmax."""
    S, Hq, D = q.shape
    Hkv = kp.shape[2]
    G = Hq // Hkv
    out = np.zeros((S, Hq, D))
    for s in range(S):
        L = int(lens[s])
        if L == 0:
            continue
        nb = -(-L // bs)
        K = kp[tables[s, :nb]].reshape(-1, Hkv, D)[:L].astype(np.float64)
        V = vp[tables[s, :nb]].reshape(-1, Hkv, D)[:L].astype(np.float64)
        for h in range(Hq):
            kv = h // G
            w = sp_softmax(scale * (K[:, kv, :] @ q[s, h].astype(np.float64)))
            out[s, h] = w @ V[:, kv, :]
    return out


def _decode(q, kp, vp, tables, lens, scale, **kw):
    out, bad = oracle.paged_attention_decode(q, F32, kp, vp, F32, tables, lens, scale, **kw)
    assert bad == 0
    return out


# ---------------------------------------------------------------- closed forms

def test_len_one_returns_v0_exactly():
    q, kp, vp, tables, lens = _build([1, 1, 1], 4, 2, 64, seed=1)
    out = _decode(q, kp, vp, tables, lens, 0.125)
    for s in range(3):
        b = tables[s, 0]
        for h in range(4):
            assert np.array_equal(out[s, h], vp[b, 0, h // 2].astype(np.float64))


def test_zero_query_gives_mean_of_v():
    q, kp, vp, tables, lens = _build([37, 16, 5], 2, 2, 64, seed=2)
    q[:] = 0
    out = _decode(q, kp, vp, tables, lens, 0.125)
    for s, L in enumerate(lens):
        V = vp[tables[s]].reshape(-1, 2, 64)[:L].astype(np.float64)
        assert np.allclose(out[s], V.mean(axis=0), rtol=0, atol=1e-13)


def test_equal_keys_give_mean_of_v():
    q, kp, vp, tables, lens = _build([40], 2, 1, 64, seed=3)
    kp[:] = kp[0, 0]  # every key row identical
    out = _decode(q, kp, vp, tables, lens, 0.125)
    V = vp[tables[0]].reshape(-1, 1, 64)[:40].astype(np.float64)
    for h in range(2):
        assert np.allclose(out[0, h], V[:, 0].mean(axis=0), rtol=0, atol=1e-13)


def test_constant_values_give_that_row():
    q, kp, vp, tables, lens = _build([33, 64], 4, 4, 128, seed=4)
    row = np.linspace(-3, 3, 128).astype(np.float32)
    vp[:] = row
    out = _decode(q, kp, vp, tables, lens, 1 / math.sqrt(128))
    assert np.allclose(out, np.broadcast_to(row.astype(np.float64), out.shape), rtol=0, atol=1e-13)


def test_two_tokens_logistic():
    q, kp, vp, tables, lens = _build([2], 1, 1, 64, seed=5)
    scale = 0.125
    b = tables[0, 0]
    k0, k1 = kp[b, 0, 0].astype(np.float64), kp[b, 1, 0].astype(np.float64)
    v0, v1 = vp[b, 0, 0].astype(np.float64), vp[b, 1, 0].astype(np.float64)
    delta = scale * float(q[0, 0].astype(np.float64) @ (k0 - k1))
    sig = 1.0 / (1.0 + math.exp(-delta))
    expect = sig * v0 + (1 - sig) * v1
    out = _decode(q, kp, vp, tables, lens, scale)
    assert np.allclose(out[0, 0], expect, rtol=0, atol=1e-13)


def test_empty_context_is_zero():
    q, kp, vp, tables, lens = _build([0, 5], 2, 2, 64, seed=6)
    out = _decode(q, kp, vp, tables, lens, 0.125)
    assert np.all(out[0] == 0) and np.any(out[1] != 0)


# ---------------------------------------------------------------- brute force / invariants

@pytest.mark.parametrize("Hq,Hkv,D", [(2, 2, 64), (8, 2, 64), (8, 1, 128), (16, 2, 128)])
def test_paged_equals_contiguous(Hq, Hkv, D):
    lens = [1, 15, 16, 17, 40, 100, 257]
    q, kp, vp, tables, lens = _build(lens, Hq, Hkv, D, seed=7 + Hq)
    scale = 1 / math.sqrt(D)
    out = _decode(q, kp, vp, tables, lens, scale)
    ref = _contiguous_reference(q, kp, vp, tables, lens, scale)
    assert np.allclose(out, ref, rtol=1e-12, atol=1e-12)


def _library_values(codes_or_bits, kind):
    """Values of raw bf16 bit patterns / E4M3 codes, decoded by torch (a library)."""
    t = torch.from_numpy(np.ascontiguousarray(codes_or_bits))
    if kind == "bf16":
        return t.view(torch.bfloat16).to(torch.float64).numpy()
    return t.view(torch.float8_e4m3fn).to(torch.float64).numpy()


def test_bf16_paged_equals_contiguous():
    q, kp, vp, tables, lens = _build([1, 9, 16, 33, 130], 8, 2, 128, seed=21)
    bits = lambda a: torch.from_numpy(a).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    qb, kb, vb = bits(q), bits(kp), bits(vp)
    out, bad = oracle.paged_attention_decode(qb, BF16, kb, vb, BF16, tables, lens, 0.09)
    ref = _contiguous_reference(_library_values(qb, "bf16"), _library_values(kb, "bf16"),
                                _library_values(vb, "bf16"), tables, lens, 0.09)
    assert bad == 0 and np.allclose(out, ref, rtol=1e-12, atol=1e-12)


def test_fp8_paged_equals_dequantised_contiguous():
    """FP8 cache: attention over the stored codes times the per-tensor scales."""
    q, kp, vp, tables, lens = _build([3, 16, 45, 200], 4, 1, 128, seed=22)
    rng = np.random.default_rng(23)
    kc = rng.integers(0, 256, kp.shape).astype(np.uint8)
    vc = rng.integers(0, 256, vp.shape).astype(np.uint8)
    kc[(kc & 0x7F) == 0x7F] = 0x33      # no NaN codes
    vc[(vc & 0x7F) == 0x7F] = 0x21
    bits = torch.from_numpy(q).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    ks, vs = 0.0213, 1.75
    out, bad = oracle.paged_attention_decode(bits, BF16, kc, vc, FP8, tables, lens, 0.088, ks, vs)
    ref = _contiguous_reference(_library_values(bits, "bf16"), _library_values(kc, "fp8") * ks,
                                _library_values(vc, "fp8") * vs, tables, lens, 0.088)
    assert bad == 0 and np.allclose(out, ref, rtol=1e-11, atol=1e-11)


def test_gqa_equals_mha_with_repeated_kv_heads():
    """GQA with Hkv heads equals MHA whose KV heads repeat each GQA head G times."""
    q, kp, vp, tables, lens = _build([20, 50], 8, 2, 64, seed=8)
    out = _decode(q, kp, vp, tables, lens, 0.125)
    kp4 = np.ascontiguousarray(np.repeat(kp, 4, axis=2))
    vp4 = np.ascontiguousarray(np.repeat(vp, 4, axis=2))
    out4 = _decode(q, kp4, vp4, tables, lens, 0.125)
    assert np.array_equal(out, out4)


def test_placement_permutation_is_bitwise_invariant():
    q, kp, vp, tables, lens = _build([3, 31, 47, 64, 200], 8, 2, 128, seed=9)
    out = _decode(q, kp, vp, tables, lens, 0.1)
    rng = np.random.default_rng(99)
    NB = kp.shape[0]
    perm = rng.permutation(NB)        # old block b moves to perm[b]
    kp2 = np.empty_like(kp)
    vp2 = np.empty_like(vp)
    kp2[perm] = kp
    vp2[perm] = vp
    tables2 = np.where(tables >= 0, perm[np.maximum(tables, 0)], -1).astype(np.int32)
    out2 = _decode(q, kp2, vp2, tables2, lens, 0.1)
    assert np.array_equal(out, out2)


@pytest.mark.parametrize("P", [16, 32, 48, 64, 112, 4096])
def test_partitioned_merge_equals_single_pass(P):
    q, kp, vp, tables, lens = _build([1, 16, 17, 95, 96, 97, 500], 4, 2, 64, seed=10)
    single = _decode(q, kp, vp, tables, lens, 0.125)
    split = _decode(q, kp, vp, tables, lens, 0.125, partition_tokens=P)
    assert np.allclose(single, split, rtol=1e-13, atol=1e-14)


def test_stale_slots_are_not_read():
    """Bytes beyond a sequence's length (tail of its last block) never matter."""
    q, kp, vp, tables, lens = _build([5, 21], 2, 2, 64, seed=11)
    out = _decode(q, kp, vp, tables, lens, 0.125)
    kp2, vp2 = kp.copy(), vp.copy()
    for s, L in enumerate(lens):
        last = tables[s, (L - 1) // 16]
        kp2[last, L % 16:] = np.nan
        vp2[last, L % 16:] = np.inf
    out2 = _decode(q, kp2, vp2, tables, lens, 0.125)
    assert np.array_equal(out, out2)


def test_invalid_block_ids_are_skipped_and_counted():
    q, kp, vp, tables, lens = _build([40], 2, 2, 64, seed=12)
    t2 = tables.copy()
    t2[0, 1] = kp.shape[0] + 7  # second block out of range
    out, bad = oracle.paged_attention_decode(q, F32, kp, vp, F32, t2, lens, 0.125)
    assert bad == 1
    # equals attention over the 24 remaining tokens (first and third block)
    K = np.concatenate([kp[tables[0, 0]], kp[tables[0, 2], :8]]).astype(np.float64)
    V = np.concatenate([vp[tables[0, 0]], vp[tables[0, 2], :8]]).astype(np.float64)
    for h in range(2):
        w = sp_softmax(0.125 * (K[:, h] @ q[0, h].astype(np.float64)))
        assert np.allclose(out[0, h], w @ V[:, h], atol=1e-12)


def test_shared_prefix_reads_identical_kv_until_cow():
    """Sequences sharing prefix blocks see the same logical K/V; after the
    copy-on-write the copy equals the source except the newly written slot."""
    bs, Hkv, D = 16, 2, 64
    bm = RefBlockManager(32, bs)
    parent = bm.alloc_seq(40)
    kids = [bm.fork(parent) for _ in range(2)]
    rng = np.random.default_rng(13)
    kp = rng.standard_normal((32, bs, Hkv, D)).astype(np.float32)
    vp = rng.standard_normal((32, bs, Hkv, D)).astype(np.float32)
    g = [oracle.gather(kp, bm.tables[s], 40, bs) for s in [parent] + kids]
    assert all(np.array_equal(g[0], x) for x in g[1:])
    src = bm.tables[kids[0]][-1]
    slot, cow = bm.append_token(kids[0])
    assert cow is not None and cow[0] == src
    oracle.copy_blocks(kp, vp, [cow])
    newk = rng.standard_normal((1, Hkv, D)).astype(np.float32)
    oracle.kv_write(newk, newk, F32, [slot], kp, vp, F32, bs)
    dst = cow[1]
    assert np.array_equal(kp[dst, :8], kp[src, :8])          # prefix part copied
    assert np.array_equal(kp[dst, 8], newk[0])                # new token in the copy
    assert np.array_equal(kp[dst, 9:], kp[src, 9:])           # rest of the block copied too
    # the other sequences still read the original prefix
    assert np.array_equal(oracle.gather(kp, bm.tables[parent], 40, bs), g[0])


# ---------------------------------------------------------------- FP8 E4M3

def _torch_e4m3_values():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    return codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()


def test_e4m3_decode_all_codes_match_library():
    ref = _torch_e4m3_values()
    for c in range(256):
        v = oracle.e4m3_decode(c)
        if np.isnan(ref[c]):
            assert math.isnan(v), c
        else:
            assert v == ref[c], (c, v, ref[c])


def test_e4m3_format_landmarks():
    assert oracle.e4m3_decode(0x7E) == 448.0 and oracle.e4m3_decode(0xFE) == -448.0
    assert math.isnan(oracle.e4m3_decode(0x7F)) and math.isnan(oracle.e4m3_decode(0xFF))
    assert oracle.e4m3_decode(0x01) == 2.0**-9          # smallest subnormal
    assert oracle.e4m3_decode(0x07) == 7 * 2.0**-9      # largest subnormal
    assert oracle.e4m3_decode(0x08) == 2.0**-6          # smallest normal
    assert oracle.e4m3_decode(0x38) == 1.0
    assert oracle.e4m3_decode(0x80) == 0.0 and math.copysign(1, oracle.e4m3_decode(0x80)) < 0


def _brute_encode(x, finite_vals):
    """Nearest finite E4M3 code by exhaustive search; ties go to the even code;
    saturating above 448."""
    a = abs(float(x))
    sign = 0x80 if math.copysign(1.0, float(x)) < 0 else 0
    if a >= 448.0:
        return sign | 0x7E
    best, bestd = None, None
    for c in range(0x7F):  # 0x00..0x7E: non-negative finite codes
        d = abs(finite_vals[c] - a)
        if bestd is None or d < bestd or (d == bestd and c % 2 == 0):
            best, bestd = c, d
    return sign | best


def test_e4m3_encode_matches_brute_force_sweep():
    vals = _torch_e4m3_values()
    rng = np.random.default_rng(14)
    xs = np.concatenate([
        rng.uniform(-500, 500, 3000), rng.uniform(-1, 1, 3000), rng.uniform(-0.02, 0.02, 2000),
        np.array([0.0, -0.0, 448.0, 449.0, 464.0, 480.0, 1e9, -1e9, np.inf, -np.inf,
                  2.0**-10, 2.0**-10 * 1.0000001, 3 * 2.0**-10, 5 * 2.0**-10]),
    ]).astype(np.float32)
    # every exact midpoint between neighbouring finite values (ties to even)
    pos = vals[:0x7F]
    mids = ((pos[:-1] + pos[1:]) / 2).astype(np.float32)
    xs = np.concatenate([xs, mids, -mids])
    for x in xs:
        assert oracle.e4m3_encode(x) == _brute_encode(x, vals), x


def test_e4m3_encode_matches_library_cast_in_range():
    rng = np.random.default_rng(15)
    xs = rng.uniform(-448, 448, 20000).astype(np.float32)
    lib = torch.from_numpy(xs).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ours = oracle.e4m3_encode_array(xs)
    assert np.array_equal(ours, lib)


# ---------------------------------------------------------------- KV write / copy

def test_kv_write_bf16_is_raw_copy_and_touches_nothing_else():
    rng = np.random.default_rng(16)
    NB, bs, Hkv, D = 8, 16, 2, 64
    kp = rng.integers(0, 65535, (NB, bs, Hkv, D)).astype(np.uint16)
    vp = rng.integers(0, 65535, (NB, bs, Hkv, D)).astype(np.uint16)
    k = rng.integers(0, 65535, (5, Hkv, D)).astype(np.uint16)
    v = rng.integers(0, 65535, (5, Hkv, D)).astype(np.uint16)
    slots = np.array([3, -1, 127, NB * bs, 64], dtype=np.int64)
    kp0, vp0 = kp.copy(), vp.copy()
    bad = oracle.kv_write(k, v, BF16, slots, kp, vp, BF16, bs)
    assert bad == 1
    flat_k, flat_v = kp.reshape(-1, Hkv, D), vp.reshape(-1, Hkv, D)
    exp_k, exp_v = kp0.reshape(-1, Hkv, D).copy(), vp0.reshape(-1, Hkv, D).copy()
    for i, s in enumerate(slots):
        if 0 <= s < NB * bs:
            exp_k[s], exp_v[s] = k[i], v[i]
    assert np.array_equal(flat_k, exp_k) and np.array_equal(flat_v, exp_v)


def test_kv_write_fp8_matches_library_cast():
    rng = np.random.default_rng(17)
    NB, bs, Hkv, D = 4, 16, 2, 128
    x = torch.randn(3, Hkv, D, generator=torch.Generator().manual_seed(3)) * 3
    xb = x.to(torch.bfloat16)
    kbits = xb.view(torch.int16).numpy().view(np.uint16)
    vbits = (xb * 0.5).view(torch.int16).numpy().view(np.uint16)
    ks, vs = np.float32(0.0123), np.float32(0.5)
    kp = np.zeros((NB, bs, Hkv, D), np.uint8)
    vp = np.zeros((NB, bs, Hkv, D), np.uint8)
    slots = np.array([0, 17, 63], dtype=np.int64)
    assert oracle.kv_write(kbits, vbits, BF16, slots, kp, vp, FP8, bs, ks, vs) == 0
    for src, pool, sc in ((xb, kp, ks), (xb * 0.5, vp, vs)):
        q = (src.float() / torch.tensor(sc)).clamp(-448, 448)   # fp32 division, saturate
        lib = q.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        flat = pool.reshape(-1, Hkv, D)
        for i, s in enumerate(slots):
            assert np.array_equal(flat[s], lib[i])


def test_copy_blocks_semantics():
    rng = np.random.default_rng(18)
    kp = rng.standard_normal((10, 16, 2, 64)).astype(np.float32)
    vp = rng.standard_normal((10, 16, 2, 64)).astype(np.float32)
    k0, v0 = kp.copy(), vp.copy()
    bad = oracle.copy_blocks(kp, vp, [[1, 5], [2, 7], [3, 99]])
    assert bad == 1
    exp_k, exp_v = k0.copy(), v0.copy()
    exp_k[5], exp_v[5], exp_k[7], exp_v[7] = k0[1], v0[1], k0[2], v0[2]
    assert np.array_equal(kp, exp_k) and np.array_equal(vp, exp_v)
    with pytest.raises(ValueError):
        oracle.copy_blocks(kp, vp, [[1, 5], [2, 5]])
    with pytest.raises(ValueError):
        oracle.copy_blocks(kp, vp, [[1, 5], [5, 6]])


def test_swap_blocks_between_pools_of_different_sizes():
    """Cross-pool page copy: block src of the source pool lands in block dst of the
    destination pool, nothing else changes (fancy indexing is the brute force)."""
    rng = np.random.default_rng(19)
    dk = rng.standard_normal((6, 16, 2, 8)).astype(np.float32)
    dv = rng.standard_normal((6, 16, 2, 8)).astype(np.float32)
    hk = np.zeros((9, 16, 2, 8), np.float32)
    hv = np.zeros((9, 16, 2, 8), np.float32)
    pairs = np.array([[5, 8], [0, 2], [3, 0], [6, 1], [1, 9], [-2, 3]])
    assert oracle.swap_blocks(hk, hv, dk, dv, pairs) == 3
    ek, ev = np.zeros_like(hk), np.zeros_like(hv)
    ek[[8, 2, 0]], ev[[8, 2, 0]] = dk[[5, 0, 3]], dv[[5, 0, 3]]
    assert np.array_equal(hk, ek) and np.array_equal(hv, ev)
    d0 = dk.copy()
    assert oracle.swap_blocks(dk, dv, hk, hv, [[8, 1]]) == 0      # and back, into another block
    assert np.array_equal(dk[1], d0[5]) and np.array_equal(np.delete(dk, 1, 0), np.delete(d0, 1, 0))
    with pytest.raises(ValueError):
        oracle.swap_blocks(hk, hv, dk, dv, [[0, 4], [1, 4]])
    # the same src twice is fine (two copies of one page)
    assert oracle.swap_blocks(hk, hv, dk, dv, [[2, 4], [2, 5]]) == 0
    assert np.array_equal(hk[4], dk[2]) and np.array_equal(hk[5], dk[2])


# ------------------------------------------------------------------ causal prefill

def _prefill_case(seed, lens, nqs, Hq, Hkv, D, dtype=np.float32):
    """Scattered pools and tables from the reference manager; q rows per sequence."""
    rng = np.random.default_rng(seed)
    NB = sum(-(-L // 16) for L in lens) + 7
    bm = RefBlockManager(NB, 16, free_order=rng.permutation(NB))
    ids = [bm.alloc_seq(L) for L in lens]
    maxb = max(-(-L // 16) for L in lens)
    tabs = np.full((len(lens), maxb), -1, np.int32)
    for i, s in enumerate(ids):
        tabs[i, :len(bm.tables[s])] = bm.tables[s]
    kp = rng.standard_normal((NB, 16, Hkv, D)).astype(dtype)
    vp = rng.standard_normal((NB, 16, Hkv, D)).astype(dtype)
    qs = np.concatenate([[0], np.cumsum(nqs)]).astype(np.int32)
    q = rng.standard_normal((int(qs[-1]), Hq, D)).astype(dtype)
    return q, kp, vp, tabs, np.asarray(lens, np.int32), qs


def _numpy_causal(q, kp, vp, tabs, lens, qs, scale):
    """Brute force: gather each sequence's logical K/V with numpy indexing, mask
    keys after the query's position, library softmax."""
    T, Hq, D = q.shape
    Hkv = kp.shape[2]
    G = Hq // Hkv
    out = np.zeros((T, Hq, D))
    for s in range(len(lens)):
        L = int(lens[s])
        t = np.arange(L)
        K = kp[tabs[s][t // 16], t % 16].astype(np.float64)       # [L, Hkv, D]
        V = vp[tabs[s][t // 16], t % 16].astype(np.float64)
        nq = int(qs[s + 1] - qs[s])
        for i in range(nq):
            r = int(qs[s]) + i
            pos = L - nq + i
            for h in range(Hq):
                sc = scale * (K[:pos + 1, h // G] @ q[r, h].astype(np.float64))
                out[r, h] = sp_softmax(sc) @ V[:pos + 1, h // G]
    return out


@pytest.mark.parametrize("Hq,Hkv", [(2, 2), (8, 2)])
def test_prefill_equals_numpy_causal_attention(Hq, Hkv):
    # a whole prompt (37 tokens), a prompt after a 15-token cached prefix, a 1-token step
    q, kp, vp, tabs, lens, qs = _prefill_case(31, [37, 20, 16], [37, 5, 1], Hq, Hkv, 32)
    got, bad = oracle.paged_attention_prefill(q, oracle.F32, kp, vp, oracle.F32, tabs, lens, qs, 0.3)
    assert bad == 0
    np.testing.assert_allclose(got, _numpy_causal(q, kp, vp, tabs, lens, qs, 0.3), rtol=1e-12, atol=1e-12)


def test_prefill_first_position_returns_v0():
    q, kp, vp, tabs, lens, qs = _prefill_case(32, [40], [40], 4, 2, 16)
    got, _ = oracle.paged_attention_prefill(q, oracle.F32, kp, vp, oracle.F32, tabs, lens, qs, 0.5)
    b0 = tabs[0][0]
    for h in range(4):
        assert np.array_equal(got[0, h], kp.dtype.type(1) * vp[b0, 0, h // 2].astype(np.float64))


def test_prefill_row_equals_decode_of_its_prefix():
    """Row i of a prompt is the decode of the first pos + 1 tokens."""
    q, kp, vp, tabs, lens, qs = _prefill_case(33, [50], [12], 4, 4, 16)
    got, _ = oracle.paged_attention_prefill(q, oracle.F32, kp, vp, oracle.F32, tabs, lens, qs, 0.25)
    for i in range(12):
        pos = 50 - 12 + i
        dec, _ = oracle.paged_attention_decode(q[i:i + 1], oracle.F32, kp, vp, oracle.F32, tabs,
                                               np.array([pos + 1], np.int32), 0.25)
        np.testing.assert_allclose(got[i], dec[0], rtol=1e-13, atol=1e-13)


def test_prefill_fp8_equals_numpy_causal_of_library_decoded_codes():
    """FP8 cache in the prefill: E4M3 codes times per-tensor scales (distinct for K
    and V), against the causal brute force on torch's decoding of the same codes."""
    q, kp, vp, tabs, lens, qs = _prefill_case(35, [45, 70], [45, 23], 8, 2, 32)
    ks, vs = 0.0123, 0.0371
    kc = torch.from_numpy(kp / ks).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    vc = torch.from_numpy(vp / vs).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    bits = lambda a: torch.from_numpy(a).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)  # noqa: E731
    qb = bits(q)
    got, bad = oracle.paged_attention_prefill(qb, oracle.BF16, kc, vc, FP8, tabs, lens, qs, 0.2, ks, vs)
    assert bad == 0
    ref = _numpy_causal(_library_values(qb, "bf16"), _library_values(kc, "fp8") * ks,
                        _library_values(vc, "fp8") * vs, tabs, lens, qs, 0.2)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_prefill_bf16_and_row_subset():
    q, kp, vp, tabs, lens, qs = _prefill_case(34, [33, 70], [33, 40], 4, 2, 32)
    bits = lambda a: torch.from_numpy(a).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)  # noqa: E731
    qb, kb, vb = bits(q), bits(kp), bits(vp)
    full, _ = oracle.paged_attention_prefill(qb, oracle.BF16, kb, vb, oracle.BF16, tabs, lens, qs, 0.2)
    ref = _numpy_causal(oracle.bf16_to_f64(qb), oracle.bf16_to_f64(kb), oracle.bf16_to_f64(vb), tabs, lens, qs, 0.2)
    np.testing.assert_allclose(full, ref, rtol=1e-12, atol=1e-12)
    part, _ = oracle.paged_attention_prefill(qb, oracle.BF16, kb, vb, oracle.BF16, tabs, lens, qs, 0.2,
                                             rows=[0, 32, 50])
    assert np.array_equal(part[[0, 32, 50]], full[[0, 32, 50]]) and not part[1].any()
