"""The C ABI library loads, exports every symbol include/pagedkv.h declares, and
rejects bad arguments on the host before any CUDA call (CPU only)."""
import ctypes as C
import os
import re

import pytest

from tests.conftest import ROOT


@pytest.fixture(scope="module")
def L():
    from paged_kv_cache_404_b200 import build
    build.build()
    from paged_kv_cache_404_b200 import _lib
    return _lib


def _declared():
    src = open(os.path.join(ROOT, "include", "pagedkv.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(pkv_\w+)\s*\(", src)))


def test_every_declared_symbol_is_exported(L):
    names = _declared()
    assert len(names) >= 19
    lib = L.lib()
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(L.SIGNATURES), "binding and header disagree"


def test_version_and_status_strings(L):
    assert L.lib().pkv_version() == 1
    assert L.status_string(L.PKV_OK) == "ok"
    assert L.status_string(L.PKV_EINVAL) == "invalid argument"
    assert L.status_string(99) == "unknown status"


FAKE = C.c_void_p(0x10000)      # 16-byte aligned, never dereferenced (validation fails first)
ODD = C.c_void_p(0x10008)       # 8-byte aligned only


def _write(L, **kw):
    a = dict(k=FAKE, v=FAKE, src=L.PKV_BF16, slots=FAKE, n=4, kp=FAKE, vp=FAKE, cache=L.PKV_BF16, nb=8, bs=16,
             hkv=8, d=128, ks=1.0, vs=1.0, err=None)
    a.update(kw)
    return L.lib().pkv_paged_kv_write(a["k"], a["v"], a["src"], a["slots"], a["n"], a["kp"], a["vp"], a["cache"],
                                      a["nb"], a["bs"], a["hkv"], a["d"], a["ks"], a["vs"], a["err"], None)


def test_write_validation(L):
    assert _write(L, n=0) == L.PKV_OK                     # nothing to do, no CUDA call
    assert _write(L, n=-1) == L.PKV_EINVAL
    assert _write(L, bs=32) == L.PKV_EUNSUPPORTED
    assert _write(L, src=L.PKV_FP8_E4M3, cache=L.PKV_BF16) == L.PKV_EUNSUPPORTED
    assert _write(L, src=L.PKV_F32, cache=L.PKV_BF16) == L.PKV_EUNSUPPORTED
    assert _write(L, cache=L.PKV_FP8_E4M3, ks=0.0) == L.PKV_EINVAL
    assert _write(L, k=None) == L.PKV_EINVAL
    assert _write(L, kp=ODD) == L.PKV_EINVAL
    assert _write(L, hkv=1, d=4) == L.PKV_EUNSUPPORTED     # 8-byte rows cannot be moved in 16-byte chunks
    assert _write(L, nb=0) == L.PKV_EINVAL


def _decode(L, **kw):
    a = dict(out=FAKE, q=FAKE, qdt=L.PKV_BF16, kp=FAKE, vp=FAKE, cdt=L.PKV_BF16, bt=FAKE, mb=256, cl=FAKE, S=4,
             maxlen=4096, nb=1024, bs=16, hq=64, hkv=8, d=128, P=0, ws=FAKE, wsb=1 << 30, err=None)
    a.update(kw)
    return L.lib().pkv_paged_attention_decode(
        a["out"], a["q"], a["qdt"], a["kp"], a["vp"], a["cdt"], a["bt"], a["mb"], a["cl"], a["S"], a["maxlen"],
        a["nb"], a["bs"], a["hq"], a["hkv"], a["d"], 0.088, 1.0, 1.0, a["P"], a["ws"], a["wsb"], a["err"], None)


def test_decode_validation(L):
    assert _decode(L, S=0) == L.PKV_OK
    assert _decode(L, hq=60) == L.PKV_EINVAL               # 60 % 8 != 0
    assert _decode(L, d=96) == L.PKV_EUNSUPPORTED
    assert _decode(L, bs=8) == L.PKV_EUNSUPPORTED
    assert _decode(L, qdt=L.PKV_F32) == L.PKV_EUNSUPPORTED  # fp32 q with a bf16 cache
    assert _decode(L, cdt=L.PKV_FP8_E4M3, d=64) == L.PKV_EUNSUPPORTED
    assert _decode(L, hq=256, hkv=8) == L.PKV_EUNSUPPORTED  # group 32 > 16 on tensor cores
    assert _decode(L, P=24) == L.PKV_EINVAL                 # not a multiple of the block size
    assert _decode(L, out=None) == L.PKV_EINVAL
    assert _decode(L, q=ODD) == L.PKV_EINVAL
    assert _decode(L, ws=C.c_void_p(0x10010)) == L.PKV_EINVAL  # workspace must be 256-byte aligned
    assert _decode(L, wsb=1024) == L.PKV_EINVAL             # too small
    assert _decode(L, mb=0) == L.PKV_EINVAL


def _noalloc(L, **kw):
    a = dict(out=FAKE, q=FAKE, qdt=L.PKV_BF16, kp=FAKE, vp=FAKE, cdt=L.PKV_BF16, bt=FAKE, mb=256, cl=FAKE, S=256,
             maxlen=4096, nb=1024, bs=16, hq=64, hkv=8, d=128, P=0, err=None)
    a.update(kw)
    return L.lib().pkv_paged_attention_decode_noalloc(
        a["out"], a["q"], a["qdt"], a["kp"], a["vp"], a["cdt"], a["bt"], a["mb"], a["cl"], a["S"], a["maxlen"],
        a["nb"], a["bs"], a["hq"], a["hkv"], a["d"], 0.088, 1.0, 1.0, a["P"], a["err"], None)


def test_noalloc_validation_order(L):
    """The no-alloc decode runs the decode's own checks before its scratch limit,
    so an unsupported configuration reports PKV_EUNSUPPORTED whatever its size;
    only a supported one that needs more than the fixed scratch gets PKV_EINVAL.
    Every case here returns before any CUDA call."""
    f = L.lib().pkv_decode_workspace_bytes
    assert f(256, 64, 128, 4096, 0) > (32 << 20)           # the default case is over the limit
    assert _noalloc(L) == L.PKV_EINVAL
    assert _noalloc(L, S=0) == L.PKV_OK                     # nothing to do
    assert _noalloc(L, d=256) == L.PKV_EUNSUPPORTED         # big and unsupported: the configuration decides
    assert _noalloc(L, hq=256, hkv=8) == L.PKV_EUNSUPPORTED  # group 32 > 16 with a bf16 cache
    assert _noalloc(L, cdt=L.PKV_FP8_E4M3, d=64) == L.PKV_EUNSUPPORTED
    assert _noalloc(L, bs=8) == L.PKV_EUNSUPPORTED
    assert _noalloc(L, hq=60) == L.PKV_EINVAL
    assert _noalloc(L, P=24) == L.PKV_EINVAL
    assert _noalloc(L, out=None) == L.PKV_EINVAL
    assert _noalloc(L, q=ODD) == L.PKV_EINVAL


def test_workspace_bytes(L):
    f = L.lib().pkv_decode_workspace_bytes
    a = f(256, 64, 128, 4096, 0)
    b = f(256, 64, 128, 4096, 1024)
    c = f(256, 64, 128, 4096, 4096)
    assert a > b > c > 0
    # partials dominate: S * Hq * parts * D floats
    assert a >= 256 * 64 * 16 * 128 * 4
    assert f(256, 64, 128, 4096, 24) == 0                   # not a multiple of 16
    assert f(4, 2, 64, 0, 0) > 0


def test_automatic_partitions_of_small_batches(L):
    """Automatic partitioning cuts 128-token pieces instead of 256 only while the
    workspace of the smaller pieces stays within the no-alloc scratch (32 MiB):
    small batches get enough pieces to occupy the warps, large batches keep
    their workspace, and anything the no-alloc decode accepted with 256-token
    pieces it still accepts."""
    f, g = L.lib().pkv_decode_workspace_bytes, L.lib().pkv_decode_workspace_bytes_shared
    lim = 32 << 20
    assert f(4, 2, 64, 1024, 0) == f(4, 2, 64, 1024, 128)          # tiny
    assert g(64, 32, 128, 1048, 0) == g(64, 32, 128, 1048, 128)    # 16 x 4 beams, 32 heads
    assert f(64, 40, 128, 2048, 0) == f(64, 40, 128, 2048, 128)    # 64 sequences x 40 heads
    assert f(64, 64, 128, 2048, 128) > lim                          # 64 x 64 heads: 128 does not fit
    assert f(64, 64, 128, 2048, 0) == f(64, 64, 128, 2048, 256)
    assert f(256, 64, 128, 4096, 0) == f(256, 64, 128, 4096, 256)  # large batches unchanged
    assert f(128, 32, 128, 32768, 0) == f(128, 32, 128, 32768, 256)
    for S, H, M in ((64, 64, 2048), (8, 1, 125200), (2, 64, 16384), (192, 32, 1513), (1, 8, 1 << 20)):
        if f(S, H, 128, M, 256) <= lim:
            assert f(S, H, 128, M, 0) <= lim, (S, H, M)


def test_copy_validation(L):
    f = L.lib().pkv_copy_blocks
    assert f(FAKE, FAKE, 32768, FAKE, 0, 10, None, None) == L.PKV_OK
    assert f(FAKE, FAKE, 32760, FAKE, 2, 10, None, None) == L.PKV_EINVAL
    assert f(FAKE, FAKE, 32768, None, 2, 10, None, None) == L.PKV_EINVAL
    assert f(ODD, FAKE, 32768, FAKE, 2, 10, None, None) == L.PKV_EINVAL
    assert f(FAKE, FAKE, 32768, FAKE, -1, 10, None, None) == L.PKV_EINVAL


def test_python_binding_refuses_cpu_tensors():
    import torch
    import paged_kv_cache_404_b200 as pkv
    k = torch.zeros(1, 8, 128, dtype=torch.bfloat16)
    pool = torch.zeros(4, 16, 8, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        pkv.paged_kv_write(k, k, torch.zeros(1, dtype=torch.int64), pool, pool)


def _prefill(L, **kw):
    a = dict(out=FAKE, q=FAKE, qdt=L.PKV_BF16, kp=FAKE, vp=FAKE, cdt=L.PKV_BF16, bt=FAKE, mb=256, cl=FAKE, qs=FAKE,
             S=4, T=4096, mq=1024, nb=1024, bs=16, hq=64, hkv=8, d=128, ks=1.0, vs=1.0, err=None)
    a.update(kw)
    return L.lib().pkv_paged_attention_prefill(
        a["out"], a["q"], a["qdt"], a["kp"], a["vp"], a["cdt"], a["bt"], a["mb"], a["cl"], a["qs"], a["S"], a["T"],
        a["mq"], a["nb"], a["bs"], a["hq"], a["hkv"], a["d"], 0.088, a["ks"], a["vs"], a["err"], None)


def test_prefill_validation(L):
    assert _prefill(L, S=0) == L.PKV_OK                     # nothing to do, no CUDA call
    assert _prefill(L, mq=0) == L.PKV_OK
    assert _prefill(L, S=-1) == L.PKV_EINVAL
    assert _prefill(L, mb=0) == L.PKV_EINVAL
    assert _prefill(L, hq=60) == L.PKV_EINVAL               # 60 % 8 != 0
    assert _prefill(L, bs=32) == L.PKV_EUNSUPPORTED
    assert _prefill(L, qdt=L.PKV_F32) == L.PKV_EUNSUPPORTED
    assert _prefill(L, cdt=L.PKV_F32) == L.PKV_EUNSUPPORTED
    assert _prefill(L, d=64) == L.PKV_EUNSUPPORTED
    assert _prefill(L, cdt=L.PKV_FP8_E4M3, ks=float("nan")) == L.PKV_EINVAL
    assert _prefill(L, cdt=L.PKV_FP8_E4M3, vs=float("inf")) == L.PKV_EINVAL
    assert _prefill(L, S=70000) == L.PKV_EUNSUPPORTED       # grid z limit
    assert _prefill(L, mq=65535 * 256 + 1, T=65535 * 256 + 1) == L.PKV_EUNSUPPORTED   # grid y: 256-row tiles
    assert _prefill(L, hq=70000, hkv=70000) == L.PKV_EUNSUPPORTED
    assert _prefill(L, out=None) == L.PKV_EINVAL
    assert _prefill(L, qs=None) == L.PKV_EINVAL
    assert _prefill(L, q=ODD) == L.PKV_EINVAL
    assert _prefill(L, cl=C.c_void_p(0x10002)) == L.PKV_EINVAL   # int32 arrays must be 4-byte aligned
