"""Shared-prefix parallel sampling (64 prompts x 3 samples, 1,000-token prefix):
copy-on-write pairs, slots, tables and pool bytes equal the oracle's exactly,
and the decode step matches the oracle."""
import numpy as np
import pytest
import torch

import workloads as W
from tests.helpers import SharedPrefixReplay, assert_close, out_to_f64, to_np_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from paged_kv_cache_404_b200 import build
    build.build()
    assert torch.cuda.is_available()


def _check(rp, sample):
    assert rp.pairs_log == rp.ref_log, "copy-on-write pairs / slots differ from the reference manager"
    assert rp.step_slots.tolist() == rp.ref_step_slots
    assert [tuple(p) for p in rp.step_pairs.tolist()] == rp.ref_step_pairs
    for i in range(rp.S):
        assert rp.tables[i][:len(rp.ref.tables[rp.rids[i]])].tolist() == rp.ref.tables[rp.rids[i]]
    assert int(rp.err.item()) == 0
    assert np.array_equal(to_np_bits(rp.kp), rp.hk) and np.array_equal(to_np_bits(rp.vp), rp.hv)
    ref = rp.oracle_decode(sample)
    assert_close(out_to_f64(rp.out)[sample], ref, "bf16", "shared prefix")


def test_shared_prefix_full_size():
    w = W.WORKLOADS["shared_prefix"]
    rp = SharedPrefixReplay(w).run()
    # divergence: every prompt's partly filled last prefix block is copied at most n-1 times
    first_pairs = [p for _, pairs, _ in rp.pairs_log for p in pairs]
    assert len(first_pairs) + len(rp.step_pairs) <= w.num_prompts * (w.samples - 1)
    rng = np.random.default_rng(9)
    _check(rp, np.sort(rng.choice(rp.S, 24, replace=False)))
    # memory saved by sharing, next to the glossary's "up to 55%" (context, not a target)
    shared = len({int(b) for t in rp.tables for b in t if b >= 0})
    unshared = int(sum(-(-int(L) // 16) for L in rp.lens))
    saving = 1 - shared / unshared
    print("shared-prefix memory saving: %.1f%% (%d vs %d blocks)" % (100 * saving, shared, unshared))
    assert 0.3 < saving < 0.7


def test_divergence_step_all_continuations_empty():
    """All continuations 0: the decode step's first write diverges every prompt:
    2 copies per prompt (the last holder writes in place)."""
    w = W.scaled(W.WORKLOADS["shared_prefix"], num_prompts=16)
    rp = SharedPrefixReplay(w, cont=np.zeros(48, np.int32)).run()
    assert len(rp.step_pairs) == 16 * 2
    _check(rp, np.arange(48))
