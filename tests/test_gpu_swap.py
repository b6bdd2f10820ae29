"""Block swap between the device pool and a page-locked host pool (GPU).

"Le cache KV et PagedAttention" (gyaansetu.com), fine-grained eviction: when
device memory runs out, a sequence's pages move to the CPU, not the whole
sequence, and come back when it runs again.  The copies are byte copies, so
they are compared bit for bit with the oracle; a decode after a round trip
must give the same bits as before it.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests.helpers import DecodeCase, to_np_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from paged_kv_cache_404_b200 import build
    build.build()
    assert torch.cuda.is_available()


def _pool(nb, dtype, seed, where):
    """Pool [nb, 16, 8, 64] of random bytes (any bit pattern: the copy is blind to values)."""
    es = torch.empty((), dtype=dtype).element_size()
    g = torch.Generator().manual_seed(seed)
    t = torch.randint(0, 256, (nb, 16, 8, 64 * es), dtype=torch.uint8, generator=g).view(dtype)
    if where == "host":
        return t.pin_memory()
    return t.cuda()


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.uint8, torch.float32])
@pytest.mark.parametrize("src_where,dst_where", [("cuda", "host"), ("host", "cuda"), ("cuda", "cuda")])
def test_swap_blocks_bit_exact(dtype, src_where, dst_where):
    import paged_kv_cache_404_b200 as pkv
    sk, sv = _pool(40, dtype, 1, src_where), _pool(40, dtype, 2, src_where)
    dk, dv = _pool(23, dtype, 3, dst_where), _pool(23, dtype, 4, dst_where)
    hsk, hsv = to_np_bits(sk).copy(), to_np_bits(sv).copy()
    hdk, hdv = to_np_bits(dk).copy(), to_np_bits(dv).copy()
    pairs = np.array([[39, 0], [0, 22], [17, 5], [17, 6], [40, 1], [3, 23], [-1, 2], [8, 9]], dtype=np.int64)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pkv.swap_blocks(dk, dv, sk, sv, torch.from_numpy(pairs).cuda(), err_count=err)
    torch.cuda.synchronize()
    bad = oracle.swap_blocks(hdk, hdv, hsk, hsv, pairs)
    assert int(err.item()) == bad == 3
    u8 = lambda a: a.view(np.uint8)  # noqa: E731 - random bits include NaNs: compare bytes
    assert np.array_equal(u8(to_np_bits(dk)), u8(hdk)) and np.array_equal(u8(to_np_bits(dv)), u8(hdv))
    assert np.array_equal(u8(to_np_bits(sk)), u8(hsk)) and np.array_equal(u8(to_np_bits(sv)), u8(hsv))


def test_swap_pairs_in_pinned_host_memory():
    import paged_kv_cache_404_b200 as pkv
    sk, sv = _pool(12, torch.bfloat16, 5, "cuda"), _pool(12, torch.bfloat16, 6, "cuda")
    dk, dv = _pool(12, torch.bfloat16, 7, "host"), _pool(12, torch.bfloat16, 8, "host")
    pairs = torch.tensor([[3, 11], [4, 0]], dtype=torch.int64).pin_memory()
    pkv.swap_blocks(dk, dv, sk, sv, pairs)
    torch.cuda.synchronize()
    assert torch.equal(dk[11].cuda().view(torch.int16), sk[3].view(torch.int16))
    assert torch.equal(dv[0].cuda().view(torch.int16), sv[4].view(torch.int16))


def test_swap_refuses_pageable_host_memory():
    import ctypes as C

    import paged_kv_cache_404_b200 as pkv
    from paged_kv_cache_404_b200 import _lib as L
    sk, sv = _pool(4, torch.uint8, 9, "cuda"), _pool(4, torch.uint8, 10, "cuda")
    hk = torch.zeros((4, 16, 8, 64), dtype=torch.uint8)          # pageable
    hv = torch.zeros_like(hk)
    pairs = torch.tensor([[0, 1]], dtype=torch.int64, device="cuda")
    with pytest.raises(ValueError):
        pkv.swap_blocks(hk, hv, sk, sv, pairs)
    st = L.lib().pkv_swap_blocks(C.c_void_p(hk.data_ptr()), C.c_void_p(hv.data_ptr()), 4,
                                 C.c_void_p(sk.data_ptr()), C.c_void_p(sv.data_ptr()), 4, sk[0].numel(),
                                 C.c_void_p(pairs.data_ptr()), 1, None, None)
    assert st == L.PKV_EINVAL
    assert int(hk.sum()) == 0


def test_swap_many_pairs_to_host():
    """More pairs than one launch's grid.y allows (65535): split into slices."""
    import paged_kv_cache_404_b200 as pkv
    n = 70000
    kp = torch.arange(n * 16 * 4, dtype=torch.int32, device="cuda").reshape(n, 16, 1, 4).float()
    vp = -kp
    hk = torch.empty_like(kp, device="cpu").pin_memory()
    hv = torch.empty_like(vp, device="cpu").pin_memory()
    perm = np.random.default_rng(4).permutation(n)
    pairs = np.stack([np.arange(n), perm], axis=1).astype(np.int64)
    pkv.swap_blocks(hk, hv, kp, vp, torch.from_numpy(pairs).cuda())
    torch.cuda.synchronize()
    idx = torch.from_numpy(perm)
    assert torch.equal(hk[idx], kp.cpu()) and torch.equal(hv[idx], vp.cpu())


SWAP_CASES = {
    "gqa70b_mixed": lambda: W.scaled(W.WORKLOADS["gqa70b"], num_seqs=24, lens="uniform", len_lo=1, len_hi=2100),
    "fp8_long_small": lambda: W.scaled(W.WORKLOADS["fp8_long"], num_seqs=16, len_hi=5000),
}


@pytest.mark.parametrize("name", sorted(SWAP_CASES))
def test_decode_after_swap_round_trip_is_bitwise_unchanged(name):
    """Decode; swap every other sequence out to a pinned host pool; let another
    sequence take (and overwrite) every free device block; swap back in to fresh
    blocks; decode again through the new tables: same bits."""
    import paged_kv_cache_404_b200 as pkv
    w = SWAP_CASES[name]()
    case = DecodeCase(w, sample=np.arange(0, w.num_seqs, 5))
    case.snapshot_pools()
    first = case.run_gpu().clone()
    case.run_oracle()
    case.compare()

    bm = case.bm
    shape = tuple(case.k_pool.shape[1:])
    NH = case.NB
    hk = torch.empty((NH,) + shape, dtype=case.k_pool.dtype).pin_memory()
    hv = torch.empty_like(hk).pin_memory()
    bm.set_host_pool(NH)
    victims = [case.ids[s] for s in range(case.S) if s % 2 == 1 and case.lens[s] > 0]
    before = {s: bm.block_table(s).tolist() for s in victims}
    out_pairs = np.concatenate([bm.swap_out(s) for s in victims])
    pkv.swap_blocks(hk, hv, case.k_pool, case.v_pool, torch.from_numpy(out_pairs).cuda())

    filler = bm.alloc_seq(bm.num_free() * 16)
    fb = torch.from_numpy(bm.block_table(filler).astype(np.int64)).cuda()
    case.k_pool.view(torch.uint8)[fb] = 0x7F          # 3.4e38 in bf16, NaN in E4M3
    case.v_pool.view(torch.uint8)[fb] = 0x7F
    bm.free_seq(filler)

    in_pairs = np.concatenate([bm.swap_in(s) for s in victims])
    pkv.swap_blocks(case.k_pool, case.v_pool, hk, hv, torch.from_numpy(in_pairs).cuda())
    assert any(bm.block_table(s).tolist() != before[s] for s in victims)

    tables, lens = bm.tables(case.ids, case.max_blocks, pad=-1)
    assert np.array_equal(lens, case.lens)
    out = torch.empty_like(case.q)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pkv.paged_attention_decode(out, case.q, case.k_pool, case.v_pool, torch.from_numpy(tables).cuda(),
                               torch.from_numpy(case.lens).cuda(), w.scale, case.max_len, case.ws,
                               case.k_scale, case.v_scale, err_count=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert torch.equal(out.view(torch.int16), first.view(torch.int16))
