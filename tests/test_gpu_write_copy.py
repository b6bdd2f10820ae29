"""GPU parity of paged_kv_write and copy_blocks: bit-exact against the oracle,
whole pools compared (every untouched byte too)."""
import numpy as np
import pytest
import torch

import oracle
from tests.helpers import to_np_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from paged_kv_cache_404_b200 import build
    build.build()
    assert torch.cuda.is_available()


def _pool(shape, dtype, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    if dtype == torch.uint8:
        x = torch.randint(0, 256, shape, generator=g, device="cuda", dtype=torch.int32).to(torch.uint8)
        x[(x & 0x7F) == 0x7F] = 0x11
        return x
    return torch.randn(shape, generator=g, device="cuda").to(dtype)


CASES = [
    ("f32", torch.float32, torch.float32, oracle.F32, oracle.F32, 2, 64),
    ("bf16", torch.bfloat16, torch.bfloat16, oracle.BF16, oracle.BF16, 8, 128),
    ("bf16->fp8", torch.bfloat16, torch.uint8, oracle.BF16, oracle.FP8_E4M3, 8, 128),
    ("f32->fp8", torch.float32, torch.uint8, oracle.F32, oracle.FP8_E4M3, 4, 64),
    ("bf16 D64", torch.bfloat16, torch.bfloat16, oracle.BF16, oracle.BF16, 1, 64),
]


@pytest.mark.parametrize("name,src_t,cache_t,src_o,cache_o,Hkv,D", CASES, ids=[c[0] for c in CASES])
def test_write_bit_exact(name, src_t, cache_t, src_o, cache_o, Hkv, D):
    import paged_kv_cache_404_b200 as pkv
    NB, T = 37, 300
    kp = _pool((NB, 16, Hkv, D), cache_t, 1)
    vp = _pool((NB, 16, Hkv, D), cache_t, 2)
    hk, hv = to_np_bits(kp).copy(), to_np_bits(vp).copy()
    g = torch.Generator(device="cuda").manual_seed(3)
    k = (torch.randn((T, Hkv, D), generator=g, device="cuda") * 4).to(src_t)
    v = (torch.randn((T, Hkv, D), generator=g, device="cuda") * 0.01).to(src_t)
    rng = np.random.default_rng(4)
    slots = rng.choice(NB * 16, size=T, replace=False).astype(np.int64)
    slots[::17] = -1                      # padding
    slots[5] = NB * 16                    # out of range
    slots[6] = NB * 16 + 1000
    ks, vs = (0.0371, 0.00019) if cache_t == torch.uint8 else (1.0, 1.0)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pkv.paged_kv_write(k, v, torch.from_numpy(slots).cuda(), kp, vp, ks, vs, err_count=err)
    bad = oracle.kv_write(to_np_bits(k), to_np_bits(v), src_o, slots, hk, hv, cache_o, 16, ks, vs)
    torch.cuda.synchronize()
    assert int(err.item()) == bad == 2
    assert np.array_equal(to_np_bits(kp), hk)
    assert np.array_equal(to_np_bits(vp), hv)


def test_fp8_write_sweep_edges():
    """Quantisation edges: saturation, exact midpoints (ties to even), subnormals, signed zero."""
    import paged_kv_cache_404_b200 as pkv
    vals = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).float()
    fin = vals[torch.isfinite(vals)]
    pos = torch.sort(fin[fin >= 0]).values.unique()
    mids = (pos[:-1] + pos[1:]) / 2
    extra = torch.tensor([0.0, -0.0, 448.0, 449.0, 464.0, 465.0, 1e30, -1e30, 1e-30, -1e-30, 2.0**-10,
                          3 * 2.0**-10, float("inf"), float("-inf")])
    x = torch.cat([fin, mids, -mids, extra, torch.linspace(-500, 500, 4001)])
    n = (x.numel() + 1023) // 1024 * 1024
    x = torch.cat([x, torch.zeros(n - x.numel())]).reshape(-1, 8, 128)
    T = x.shape[0]
    kp = torch.zeros((T // 16 + 1, 16, 8, 128), dtype=torch.uint8, device="cuda")
    vp = torch.zeros_like(kp)
    slots = torch.arange(T, dtype=torch.int64)
    for scale in (1.0, 0.5, 3.0):
        pkv.paged_kv_write(x.cuda(), x.cuda(), slots.cuda(), kp, vp, scale, scale)
        hk = np.zeros(tuple(kp.shape), np.uint8)
        hv = np.zeros_like(hk)
        oracle.kv_write(x.numpy(), x.numpy(), oracle.F32, slots.numpy(), hk, hv, oracle.FP8_E4M3, 16, scale, scale)
        torch.cuda.synchronize()
        assert np.array_equal(to_np_bits(kp), hk)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.uint8, torch.float32])
def test_copy_blocks_bit_exact(dtype):
    import paged_kv_cache_404_b200 as pkv
    NB = 64
    kp = _pool((NB, 16, 8, 128), dtype, 5)
    vp = _pool((NB, 16, 8, 128), dtype, 6)
    hk, hv = to_np_bits(kp).copy(), to_np_bits(vp).copy()
    pairs = np.array([[1, 40], [2, 41], [3, 42], [63, 0], [5, 99], [-1, 7], [10, 11]], dtype=np.int64)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pkv.copy_blocks(kp, vp, torch.from_numpy(pairs).cuda(), err_count=err)
    bad = oracle.copy_blocks(hk, hv, pairs)
    torch.cuda.synchronize()
    assert int(err.item()) == bad == 2
    assert np.array_equal(to_np_bits(kp), hk) and np.array_equal(to_np_bits(vp), hv)


def test_copy_blocks_many_pairs():
    """More pairs than one launch's grid.y allows (65535): split into slices."""
    import paged_kv_cache_404_b200 as pkv
    NB = 2 * 70000
    kp = torch.arange(NB * 16, dtype=torch.int32, device="cuda").reshape(NB, 16, 1, 1).float()
    vp = -kp
    src = np.arange(70000, dtype=np.int64)
    pairs = np.stack([src, src + 70000], axis=1)
    pkv.copy_blocks(kp, vp, torch.from_numpy(pairs).cuda())
    torch.cuda.synchronize()
    assert torch.equal(kp[70000:], kp[:70000]) and torch.equal(vp[70000:], vp[:70000])


def test_fp8_pool_is_half_of_bf16():
    """Glossary entry, 'Tecnicas relacionadas': an FP8 cache takes half the bytes of a 16-bit one."""
    a = torch.empty((100, 16, 8, 128), dtype=torch.bfloat16, device="cuda")
    b = torch.empty((100, 16, 8, 128), dtype=torch.uint8, device="cuda")
    assert b.numel() * b.element_size() * 2 == a.numel() * a.element_size()
