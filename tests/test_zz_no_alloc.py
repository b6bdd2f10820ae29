"""The decode entry point for callers that cannot allocate device memory.

pkv_paged_attention_decode_noalloc takes no workspace: it runs on a fixed
device array the library declares, so a caller with no allocator (a plug-in
inside a host program that owns all device memory, or a loop that must not call
cudaMalloc/cudaFree because they synchronise the device) can still decode.
These checks call it through the C ABI, two calls in a row on different
problems (the second finds the first one's leftovers in the shared scratch).
It runs the same kernels with the same partitioning as the workspace entry
point, so its output must equal that entry point's bit for bit; each output is
also compared with the oracle within the decode tolerances.  This file is
collected last on purpose.
"""
import ctypes as C

import numpy as np
import pytest
import torch

import workloads as W
from tests.helpers import DecodeCase

pytestmark = pytest.mark.gpu

LIMIT = 32 << 20    # PKV_NOALLOC_SCRATCH_BYTES


@pytest.fixture(scope="module")
def lib():
    from paged_kv_cache_404_b200 import build
    build.build()
    from paged_kv_cache_404_b200 import _lib
    assert torch.cuda.is_available()
    return _lib


def _noalloc_abi(lib, case, P, err, max_len=None, out=None):
    """The no-alloc call on a DecodeCase's device inputs (after its run_gpu)."""
    q, kp = case.q, case.k_pool
    out = torch.empty_like(q) if out is None else out
    S, Hq, D = q.shape
    NB, bs, Hkv, _ = kp.shape
    cache = lib.PKV_FP8_E4M3 if kp.dtype == torch.uint8 else lib.PKV_BF16
    p = lambda t: C.c_void_p(t.data_ptr())  # noqa: E731
    st = lib.lib().pkv_paged_attention_decode_noalloc(
        p(out), p(q), lib.PKV_BF16, p(kp), p(case.v_pool), cache, p(case.g_tables), case.g_tables.shape[1],
        p(case.g_lens), S, case.max_len if max_len is None else max_len, NB, bs, Hq, Hkv, D, case.w.scale,
        case.k_scale, case.v_scale, P, p(err), C.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st, out


def _workspace_decode(case, P, max_len):
    import paged_kv_cache_404_b200 as pkv
    ws = pkv.decode_workspace(case.S, case.w.num_heads, case.w.head_dim, max_len, P)
    out = torch.empty_like(case.q)
    pkv.paged_attention_decode(out, case.q, case.k_pool, case.v_pool, case.g_tables, case.g_lens, case.w.scale,
                               max_len, ws, case.k_scale, case.v_scale, partition_tokens=P)
    return out


def _bits_equal(a, b):
    return torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_noalloc_matches_workspace_entry_two_calls_in_a_row(lib):
    """A bf16 GQA batch (automatic partitions), then an FP8 batch of long mixed
    contexts (512-token partitions): each no-alloc result equals the workspace
    entry point's bit for bit and the oracle's within tolerance."""
    rng = np.random.default_rng(11)
    cases = [
        (DecodeCase(W.scaled(W.WORKLOADS["gqa70b"], num_seqs=64),
                    lens=rng.integers(1, 2049, size=64).astype(np.int32)), 0),
        (DecodeCase(W.scaled(W.WORKLOADS["fp8_long"], num_seqs=32),
                    lens=np.minimum(np.floor(np.exp(rng.uniform(np.log(16), np.log(8192), 32))), 8192)
                    .astype(np.int32)), 512),
    ]
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    for case, P in cases:
        case.snapshot_pools()
        case.run_gpu(partition_tokens=P)          # writes the step's token, then the workspace decode
        st, got = _noalloc_abi(lib, case, P, err)
        assert st == lib.PKV_OK, lib.status_string(st)
        torch.cuda.synchronize()
        assert _bits_equal(got, case.out), "no-alloc and workspace decodes differ (%s)" % case.w.name
        case.run_oracle()
        case.out = got
        case.compare()
    assert int(err.item()) == 0


def test_noalloc_accepts_a_need_of_exactly_its_limit(lib):
    """8 sequences, one head, head_dim 128, 16-token partitions and
    max_context_len 125,200 need exactly the fixed scratch (7,825 partitions per
    sequence); 125,201 needs one more partition and is refused untouched."""
    f = lib.lib().pkv_decode_workspace_bytes
    assert f(8, 1, 128, 125200, 16) == LIMIT
    assert f(8, 1, 128, 125201, 16) > LIMIT
    w = W.scaled(W.WORKLOADS["gqa70b"], num_heads=1, num_kv_heads=1, num_seqs=8)
    case = DecodeCase(w, lens=np.array([1, 16, 17, 100, 300, 40, 2, 64], np.int32))
    case.snapshot_pools()
    case.run_gpu(partition_tokens=16)
    ref = _workspace_decode(case, 16, 125200)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    st, got = _noalloc_abi(lib, case, 16, err, max_len=125200)
    assert st == lib.PKV_OK, lib.status_string(st)
    torch.cuda.synchronize()
    assert _bits_equal(got, ref)
    case.run_oracle()
    case.out = got
    case.compare()
    sentinel = torch.full_like(case.q, 7.0)
    st, _ = _noalloc_abi(lib, case, 16, err, max_len=125201, out=sentinel)
    assert st == lib.PKV_EINVAL
    torch.cuda.synchronize()
    assert torch.all(sentinel == 7.0)
    assert int(err.item()) == 0


def test_noalloc_refuses_problems_beyond_its_scratch(lib):
    """Two real 16-token sequences, but bounds (max_context_len 16,384 with
    16-token partitions, 64 query heads) whose scratch is about 65 MiB: refused
    before any launch, the output untouched.  The buffers match the arguments,
    so the call would stay in bounds even if it ran."""
    f = lib.lib().pkv_decode_workspace_bytes
    assert f(2, 64, 128, 16384, 16) > 2 * LIMIT
    case = DecodeCase(W.scaled(W.WORKLOADS["gqa70b"], num_seqs=2), lens=np.array([16, 16], np.int32))
    case.run_gpu(partition_tokens=16)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    sentinel = torch.full_like(case.q, 7.0)
    st, _ = _noalloc_abi(lib, case, 16, err, max_len=16384, out=sentinel)
    assert st == lib.PKV_EINVAL
    torch.cuda.synchronize()
    assert torch.all(sentinel == 7.0)    # nothing was launched
    assert int(err.item()) == 0
