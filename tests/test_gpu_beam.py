"""Beam search over paged blocks: at every step each request keeps its beams
drawn (seeded) from its current ones -- forks, frees and copy-on-write of the
shared partly filled block every step -- then the step's tokens are written
and decoded (glossary entry "PagedAttention", sharing section: parallel
sampling and beam search share blocks, copy-on-write before writing a block
others still use).  Product (native manager + CUDA kernels) and oracle
(reference manager + C oracle) replay the same trace; every copy pair and slot
is compared exactly, the pools byte for byte, the decode within tolerance."""
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


def _beam_step(mgr, beams, parents, native):
    """Fork the chosen parents, free the old beams, reserve one slot per new beam."""
    new = []
    for r, old in enumerate(beams):
        kids = [mgr.fork(old[int(p)]) for p in parents[r]]
        for s in old:
            mgr.free_seq(s)
        new.append(kids)
    flat = [s for kids in new for s in kids]
    if native:
        slots, pairs = mgr.append_tokens(flat)
        return new, slots.tolist(), [tuple(x) for x in pairs.tolist()]
    res = [mgr.append_token(s) for s in flat]
    return new, [x[0] for x in res], [x[1] for x in res if x[1] is not None]


@pytest.mark.parametrize("prompt,steps", [(70, 12), (64, 20)])
def test_beam_trace_matches_oracle(prompt, steps):
    import paged_kv_cache_404_b200 as pkv
    w = W.scaled(W.WORKLOADS["beam"], num_prompts=4, samples=4, num_seqs=16, prefix_len=prompt, len_hi=steps)
    R, B = w.num_prompts, w.samples
    NB = R * (-(-prompt // 16)) + R * B * (steps // 16 + 3) + 8
    order = W.free_order(w, NB)
    bm, ref = pkv.BlockManager(NB, 16, free_order=order), oracle.RefBlockManager(NB, 16, free_order=order)
    kp, vp = W.stale_fill(w, NB, "cuda")
    hk, hv = to_np_bits(kp).copy(), to_np_bits(vp).copy()
    pk, pv = W.logical_kv(w, R * prompt, "cuda", stream=50)
    beams, rbeams = [], []
    for r in range(R):
        p, rp = bm.alloc_seq(prompt), ref.alloc_seq(prompt)
        sl = slice(r * prompt, (r + 1) * prompt)
        pkv.paged_kv_write(pk[sl], pv[sl], torch.from_numpy(bm.slots(p, 0, prompt)).cuda(), kp, vp)
        oracle.kv_write(to_np_bits(pk[sl]), to_np_bits(pv[sl]), oracle.BF16, ref.slots(rp, 0, prompt), hk, hv,
                        oracle.BF16, 16)
        beams.append([p] + [bm.fork(p) for _ in range(B - 1)])
        rbeams.append([rp] + [ref.fork(rp) for _ in range(B - 1)])
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    total_pairs = 0
    for t in range(steps):
        parents = W.beam_parents(w, t)
        beams, slots, pairs = _beam_step(bm, beams, parents, True)
        rbeams, rslots, rpairs = _beam_step(ref, rbeams, parents, False)
        assert slots == rslots and pairs == rpairs, "step %d" % t
        assert bm.free_list().tolist() == list(ref.free)
        total_pairs += len(pairs)
        kn, vn = W.new_tokens(w, R * B, "cuda", stream=100 + t)
        if pairs:
            pkv.copy_blocks(kp, vp, torch.tensor(pairs, dtype=torch.int64, device="cuda"), err_count=err)
            oracle.copy_blocks(hk, hv, rpairs)
        pkv.paged_kv_write(kn, vn, torch.tensor(slots, dtype=torch.int64, device="cuda"), kp, vp, err_count=err)
        oracle.kv_write(to_np_bits(kn), to_np_bits(vn), oracle.BF16, np.asarray(rslots, np.int64), hk, hv,
                        oracle.BF16, 16)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert total_pairs > 0                                   # copy-on-write happened
    assert np.array_equal(to_np_bits(kp), hk) and np.array_equal(to_np_bits(vp), hv)

    flat = [s for kids in beams for s in kids]
    rflat = [s for kids in rbeams for s in kids]
    L = prompt + steps
    maxb = -(-L // 16)
    tabs, lens = bm.tables(flat, maxb, pad=-1)
    assert (lens == L).all()
    for i, s in enumerate(rflat):
        assert tabs[i][:len(ref.tables[s])].tolist() == ref.tables[s]
    offs, mem, sh = bm.prefix_groups(flat)
    assert len(sh) == R                                      # one group per request: the shared prompt
    q = W.queries(w, R * B, "cuda")
    ws = pkv.decode_workspace(R * B, w.num_heads, w.head_dim, L, 0, shared=True)
    out = torch.empty_like(q)
    g = lambda a: torch.from_numpy(np.asarray(a, np.int32)).cuda()  # noqa: E731
    pkv.paged_attention_decode_shared(out, q, kp, vp, g(tabs), g(lens), w.scale, L, ws, g(offs), g(mem), g(sh),
                                      err_count=err)
    torch.cuda.synchronize()
    ref_out, bad = oracle.paged_attention_decode(to_np_bits(q), oracle.BF16, hk, hv, oracle.BF16, tabs, lens, w.scale)
    assert bad == 0 and int(err.item()) == 0
    assert_close(out_to_f64(out), ref_out, "bf16", "beam decode")
