"""Guard rows around every pool and output, standing in for a memory checker
(compute-sanitizer is not available here): each buffer the kernels touch is the
middle slice of a larger allocation whose first and last rows hold a canary
pattern.  Writes and copies are given the out-of-range indices nearest the pool
(the first slot past the end, a negative slot, a copy whose destination is one
block past the end), decode and prefill run over the pools, and afterwards every
guard byte must still hold the canary and the out-of-range indices must have been
counted."""
import pytest
import torch

pytestmark = pytest.mark.gpu

G = 3            # guard rows (blocks, or output rows) on each side


@pytest.fixture(scope="module", autouse=True)
def _built():
    from paged_kv_cache_404_b200 import build
    build.build()
    assert torch.cuda.is_available()


def _guarded(shape, dtype, canary):
    """(whole buffer, middle view of `shape`) with G canary rows before and after."""
    whole = torch.empty((shape[0] + 2 * G,) + tuple(shape[1:]), dtype=dtype, device="cuda")
    whole.view(torch.uint8).fill_(canary)
    return whole, whole[G:G + shape[0]]


def _guards_intact(whole, canary):
    b = whole.view(torch.uint8)
    n = b.shape[0]
    return bool((b[:G] == canary).all()) and bool((b[n - G:] == canary).all())


@pytest.mark.parametrize("cache", ["bf16", "fp8"])
def test_kernels_stay_inside_their_buffers(cache):
    import paged_kv_cache_404_b200 as pkv
    NB, Hkv, Hq, D = 40, 2, 8, 128
    cdt = torch.uint8 if cache == "fp8" else torch.bfloat16
    kw, kp = _guarded((NB, 16, Hkv, D), cdt, 0x5A)
    vw, vp = _guarded((NB, 16, Hkv, D), cdt, 0xA5)
    kp.zero_()
    vp.zero_()
    ks, vs = (0.01, 0.02) if cache == "fp8" else (1.0, 1.0)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")

    # writes: 5 valid slots, then the first slot past the pool and a negative one (skipped: padding)
    T = 7
    k = torch.randn(T, Hkv, D, device="cuda").to(torch.bfloat16)
    v = torch.randn(T, Hkv, D, device="cuda").to(torch.bfloat16)
    slots = torch.tensor([0, 17, 33, 16 * NB - 1, 100, 16 * NB, -1], dtype=torch.int64, device="cuda")
    pkv.paged_kv_write(k, v, slots, kp, vp, ks, vs, err_count=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 1                            # 16 * NB counted; -1 is padding
    assert _guards_intact(kw, 0x5A) and _guards_intact(vw, 0xA5)

    # copies: valid pairs, then one whose destination is one block past the end
    pairs = torch.tensor([[0, 5], [2, NB - 1], [1, NB]], dtype=torch.int64, device="cuda")
    pkv.copy_blocks(kp, vp, pairs, err_count=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 2
    assert _guards_intact(kw, 0x5A) and _guards_intact(vw, 0xA5)

    # decode over three sequences (one with a table entry past the pool): output rows guarded
    S = 3
    tabs = torch.tensor([[0, 1, 2, 3], [5, 6, NB, 7], [NB - 1, -1, -1, -1]], dtype=torch.int32, device="cuda")
    lens = torch.tensor([60, 64, 9], dtype=torch.int32, device="cuda")
    q = torch.randn(S, Hq, D, device="cuda").to(torch.bfloat16)
    ow, out = _guarded((S, Hq, D), torch.bfloat16, 0x3C)
    ws = pkv.decode_workspace(S, Hq, D, 64, 16, device="cuda")
    pkv.paged_attention_decode(out, q, kp, vp, tabs, lens, D ** -0.5, 64, ws, ks, vs, partition_tokens=16,
                               err_count=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 3                            # the bad table entry, once
    assert _guards_intact(ow, 0x3C) and torch.isfinite(out.float()).all()

    # prefill: 2 sequences, output rows of the queries only (the scales are ignored for bf16)
    qs = torch.tensor([0, 20, 30], dtype=torch.int32, device="cuda")
    qq = torch.randn(30, Hq, D, device="cuda").to(torch.bfloat16)
    pw, pout = _guarded((30, Hq, D), torch.bfloat16, 0xC3)
    pkv.paged_attention_prefill(pout, qq, kp, vp, tabs[:2], lens[:2], qs, D ** -0.5, 20, err_count=err,
                                k_scale=ks, v_scale=vs)
    torch.cuda.synchronize()
    assert int(err.item()) >= 3
    assert _guards_intact(pw, 0xC3) and torch.isfinite(pout.float()).all()
    assert _guards_intact(kw, 0x5A) and _guards_intact(vw, 0xA5)
