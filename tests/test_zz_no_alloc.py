"""The decode entry point for callers that cannot allocate device memory.

pkv_paged_attention_decode_noalloc takes no workspace: it runs on a fixed
device array the library declares, so a caller with no allocator (or one that
must not call cudaMalloc/cudaFree on its hot path) can still decode.  These
checks call it through the C ABI, twice in a row on different problems (the
second call finds the first one's leftovers in the shared scratch), and compare
each result with the workspace entry point's, within the bf16 / FP8 attention
tolerances the other decode tests use.  This file is collected last on purpose.
"""
import ctypes as C

import numpy as np
import pytest
import torch

import workloads as W

pytestmark = pytest.mark.gpu

TOL = {"bf16": 1e-2, "fp8": 3e-2}   # |a - b| <= tol + tol * |b|, as in the other decode tests


@pytest.fixture(scope="module")
def lib():
    from paged_kv_cache_404_b200 import build
    build.build()
    from paged_kv_cache_404_b200 import _lib
    assert torch.cuda.is_available()
    return _lib


def _problem(w, lens):
    import paged_kv_cache_404_b200 as pkv
    need = int(sum(-(-int(L) // 16) for L in lens))
    NB = W.pool_blocks(w, need)
    bm = pkv.BlockManager(NB, 16, free_order=W.free_order(w, NB))
    ids = [bm.alloc_seq(int(L)) for L in lens]
    tabs, tl = bm.tables(ids, max(-(-int(L) // 16) for L in lens), pad=-1)
    kp, vp, ks, vs = W.random_pools(w, NB, "cuda")
    q = W.queries(w, len(lens), "cuda")
    return dict(w=w, kp=kp, vp=vp, ks=ks, vs=vs, q=q, tabs=torch.from_numpy(tabs).cuda(),
                lens=torch.from_numpy(tl).cuda(), max_len=int(max(lens)), NB=NB)


def _with_workspace(pr, P):
    import paged_kv_cache_404_b200 as pkv
    w = pr["w"]
    ws = pkv.decode_workspace(len(pr["q"]), w.num_heads, w.head_dim, pr["max_len"], P)
    out = torch.empty_like(pr["q"])
    pkv.paged_attention_decode(out, pr["q"], pr["kp"], pr["vp"], pr["tabs"], pr["lens"], w.scale, pr["max_len"],
                               ws, pr["ks"], pr["vs"], partition_tokens=P)
    return out


def _noalloc_abi(lib, pr, P, err):
    w = pr["w"]
    q, kp = pr["q"], pr["kp"]
    out = torch.empty_like(q)
    S, Hq, D = q.shape
    NB, bs, Hkv, _ = kp.shape
    cache = lib.PKV_FP8_E4M3 if kp.dtype == torch.uint8 else lib.PKV_BF16
    p = lambda t: C.c_void_p(t.data_ptr())
    st = lib.lib().pkv_paged_attention_decode_noalloc(
        p(out), p(q), lib.PKV_BF16, p(kp), p(pr["vp"]), cache, p(pr["tabs"]), pr["tabs"].shape[1], p(pr["lens"]),
        S, pr["max_len"], NB, bs, Hq, Hkv, D, w.scale, pr["ks"], pr["vs"], P, p(err),
        C.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st, out


def _close(a, b, kind):
    a = a.float().cpu().numpy().astype(np.float64)
    b = b.float().cpu().numpy().astype(np.float64)
    tol = TOL[kind]
    assert np.isfinite(a).all()
    assert np.all(np.abs(a - b) <= tol + tol * np.abs(b)), float(np.abs(a - b).max())


def test_noalloc_matches_workspace_entry_two_calls_in_a_row(lib):
    rng = np.random.default_rng(11)
    first = _problem(W.scaled(W.WORKLOADS["gqa70b"], num_seqs=64),
                     rng.integers(1, 2049, size=64).astype(np.int32))
    second = _problem(W.scaled(W.WORKLOADS["fp8_long"], num_seqs=32),
                      np.minimum(np.floor(np.exp(rng.uniform(np.log(16), np.log(8192), 32))), 8192).astype(np.int32))
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    for pr, P, kind in ((first, 0, "bf16"), (second, 512, "fp8")):
        st, got = _noalloc_abi(lib, pr, P, err)
        assert st == lib.PKV_OK, lib.status_string(st)
        ref = _with_workspace(pr, P)
        torch.cuda.synchronize()
        _close(got, ref, kind)
    assert int(err.item()) == 0


def test_noalloc_refuses_problems_beyond_its_scratch(lib):
    """Bounds whose scratch would exceed the fixed array are refused before any launch."""
    need = lib.lib().pkv_decode_workspace_bytes(256, 64, 128, 4096, 0)
    assert need > (32 << 20)
    pr = _problem(W.scaled(W.WORKLOADS["gqa70b"], num_seqs=2), np.array([16, 16], np.int32))
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    q, kp = pr["q"], pr["kp"]
    out = torch.full_like(q, 7.0)
    p = lambda t: C.c_void_p(t.data_ptr())
    st = lib.lib().pkv_paged_attention_decode_noalloc(
        p(out), p(q), lib.PKV_BF16, p(kp), p(pr["vp"]), lib.PKV_BF16, p(pr["tabs"]), pr["tabs"].shape[1],
        p(pr["lens"]), 256, 4096, pr["NB"], 16, 64, 8, 128, pr["w"].scale, 1.0, 1.0, 0, p(err), None)
    assert st == lib.PKV_EINVAL
    torch.cuda.synchronize()
    assert torch.all(out == 7.0)    # nothing was launched
