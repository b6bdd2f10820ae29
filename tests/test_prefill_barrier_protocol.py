"""Model check of the tcgen05 prefill kernel's mbarrier protocol (host only).

The kernel's roles (TMA producer, FP8 converter warps, the MMA issuer, the tensor
core executing one thread's products in issue order, two softmax warpgroups)
synchronise through mbarriers that are waited on by phase parity.  A parity wait
is only correct while the barrier is at the awaited phase or one past it: two
phases on, it reads as "not yet" (a deadlock until the bounded wait gives up), two
phases behind as "done" (a read of data not written yet).

This test replays the protocol of paged_kv_cache_404_b200/csrc/prefill_tc.cu as
generators under a seeded random scheduler and checks, at every wait, that the
barrier is exactly there, and that every schedule runs to completion.  It covers
one and two score buffers per Q tile (the kernel runs two) with 2- and 4-stage
K/V rings, bf16 (producer zeroes V tails, may wait for the landing) and FP8
(staging ring, four converters).  A planted mistake (one P barrier per Q tile
instead of one per buffer, as an earlier form of the kernel had) must be caught.
"""
import random

import pytest


class _Bar:
    def __init__(self, name, count):
        self.name, self.count, self.pending, self.done = name, count, count, 0

    def arrive(self):
        self.pending -= 1
        if self.pending == 0:
            self.done += 1
            self.pending = self.count


def _run(nt, fp8, seed, stages, nbuf, per_buffer_p=True, rescale_p=0.3):
    """One schedule; returns the list of protocol violations (empty if none)."""
    rng = random.Random(seed)
    ntiles = max(nt)
    bars = {}
    issues = []
    tensor_q = []      # the tensor core: products and commits, in issue order
    tma = []           # copies in flight: the barrier each completes on

    def bar(name, count=1):
        bars.setdefault(name, _Bar(name, count))
        return bars[name]

    nconv = 4 if fp8 else 1
    for i in range(stages):
        bar("kv_full%d" % i, nconv), bar("kv_empty%d" % i), bar("v_ready%d" % i, nconv)
    for t in range(2):
        for b in range(nbuf):
            bar("s_full%d%d" % (t, b)), bar("p_full%d%d" % (t, b)), bar("pv_done%d%d" % (t, b))
    for b in range(2):
        bar("stg_full%d" % b), bar("stg_empty%d" % b, nconv)

    def pbar(t, j):
        return ("p_full%d%d" % (t, j % nbuf), j // nbuf) if per_buffer_p else ("p_full%d0" % t, j)

    def wait(name, phase):
        return ("wait", name, phase)

    def producer():
        for j in range(ntiles):
            if fp8:
                if j >= 2:
                    yield wait("stg_empty%d" % (j & 1), (j >> 1) - 1)
                tma.append("stg_full%d" % (j & 1))
                yield ("step",)
            else:
                if j >= stages:
                    yield wait("kv_empty%d" % (j % stages), j // stages - 1)
                tma.append("kv_full%d" % (j % stages))
                yield ("step",)
                if rng.random() < 0.3:   # the sequence's last block: zero its tail once landed
                    yield wait("kv_full%d" % (j % stages), j // stages)
                bars["v_ready%d" % (j % stages)].arrive()
                yield ("step",)

    def converter():
        for j in range(ntiles):
            if j >= stages:
                yield wait("kv_empty%d" % (j % stages), j // stages - 1)
            yield wait("stg_full%d" % (j & 1), j >> 1)
            for n in ("stg_empty%d" % (j & 1), "kv_full%d" % (j % stages), "v_ready%d" % (j % stages)):
                bars[n].arrive()
            yield ("step",)

    def issuer():
        def issue_s(t, j):
            tensor_q.extend([("mma",), ("commit", "s_full%d%d" % (t, j % nbuf))])

        for j in range(min(nbuf, ntiles)):
            yield wait("kv_full%d" % (j % stages), j // stages)
            for t in range(2):
                if j < nt[t]:
                    issue_s(t, j)
                    yield ("step",)
        for j in range(ntiles):
            for t in range(2):
                if j < nt[t]:
                    yield wait(*pbar(t, j))
                    yield wait("v_ready%d" % (j % stages), j // stages)
                    tensor_q.extend([("mma",), ("commit", "pv_done%d%d" % (t, j % nbuf))])
                    yield ("step",)
                if j + nbuf < nt[t]:
                    yield wait("kv_full%d" % ((j + nbuf) % stages), (j + nbuf) // stages)
                    issue_s(t, j + nbuf)
                    yield ("step",)
            tensor_q.append(("commit", "kv_empty%d" % (j % stages)))
            yield ("step",)

    def softmax(t):
        for j in range(nt[t]):
            yield wait("s_full%d%d" % (t, j % nbuf), j // nbuf)
            if j > 0 and rng.random() < rescale_p:   # the reference max moved: O waits for PV(j-1)
                yield wait("pv_done%d%d" % (t, (j - 1) % nbuf), (j - 1) // nbuf)
            name, _ = pbar(t, j)
            bars[name].arrive()
            yield ("step",)
        if nt[t] > 0:
            yield wait("pv_done%d%d" % (t, (nt[t] - 1) % nbuf), (nt[t] - 1) // nbuf)

    roles = {"producer": producer(), "issuer": issuer(), "softmax0": softmax(0), "softmax1": softmax(1)}
    if fp8:
        for w in range(nconv):
            roles["converter%d" % w] = converter()
    cur = {k: next(g, None) for k, g in roles.items()}
    for _ in range(200000):
        ready = []
        for k, st in cur.items():
            if st is None:
                continue
            if st[0] == "wait":
                # the hardware's parity test: phase `phase` reads as complete when the
                # current phase's parity differs from its parity
                if (bars[st[1]].done & 1) != (st[2] & 1):
                    ready.append(k)
            else:
                ready.append(k)
        if tensor_q:
            ready.append("tensor")
        if tma:
            ready.append("tma")
        if not ready:
            if any(v is not None for v in cur.values()):
                issues.append("deadlock: " + ", ".join("%s waits %s" % (k, v[1:]) for k, v in cur.items() if v))
            return issues
        k = rng.choice(ready)
        if k == "tensor":
            op = tensor_q.pop(0)
            if op[0] == "commit":
                bars[op[1]].arrive()
        elif k == "tma":
            bars[tma.pop(rng.randrange(len(tma)))].arrive()
        else:
            st = cur[k]
            if st[0] == "wait":
                c = bars[st[1]].done
                if c not in (st[2], st[2] + 1):
                    issues.append("%s passed a wait for phase %d of %s with %d phases done" % (k, st[2], st[1], c))
            cur[k] = next(roles[k], None)
    issues.append("no progress bound reached")
    return issues


def _cases(n):
    rng = random.Random(1234)
    for i in range(n):
        n1 = rng.randint(1, 14)
        n0 = rng.randint(0, n1)   # Q tile 0 never reads more KV tiles than Q tile 1
        yield [n0, n1], i


@pytest.mark.parametrize("fp8,stages,nbuf", [(False, 4, 2), (True, 4, 2), (False, 2, 1), (False, 3, 1)])
def test_protocol_has_no_parity_aliasing_or_deadlock(fp8, stages, nbuf):
    for nt, seed in _cases(1500):
        issues = _run(nt, fp8, seed, stages, nbuf)
        assert not issues, (nt, seed, issues[:2])


def test_a_single_p_barrier_per_q_tile_is_caught():
    """With double-buffered scores the softmax may finish tile j+1 before the issuer
    takes P(j): one P barrier per Q tile then runs two phases ahead."""
    caught = sum(bool(_run(nt, False, seed, 4, 2, per_buffer_p=False)) for nt, seed in _cases(300))
    assert caught > 100
