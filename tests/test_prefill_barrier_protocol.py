"""Model checks of the tcgen05 prefill kernels' mbarrier protocols (host only).

Each kernel's roles (TMA producer, FP8 converter warps, the MMA issuer, the tensor
core executing one thread's products in issue order, two softmax warpgroups)
synchronise through mbarriers that are waited on by phase parity.  A parity wait
is only correct while the barrier is at the awaited phase or one past it: two
phases on, it reads as "not yet" (a deadlock until the bounded wait gives up), two
phases behind as "done" (a read of data not written yet).

The tests replay the protocols of paged_kv_cache_404_b200/csrc/prefill_tc.cu as
generators under a seeded random scheduler and check, at every wait, that the
barrier is exactly there, and that every schedule runs to completion.

- The FP8 kernel (64-key tiles): one and two score buffers per Q tile (the kernel
  runs two) with 2- and 4-stage K/V rings, FP8 (staging ring, four converters)
  and the same protocol without converters (one producer zeroing V tails, which
  may wait for the landing).  A planted mistake (one P barrier per Q tile instead
  of one per buffer, as an earlier form of the kernel had) must be caught.
- The bf16 kernel (128-key tiles, separate K and V rings, one score buffer per Q
  tile): besides the phase checks, data hazards on ring slots, score buffers and O,
  with three planted mistakes that must be caught.
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


# ---------------------------------------------------------------------------------
# The bf16 kernel: 128-key tiles, K and V in 2-stage rings apart, one score
# buffer per Q tile (P written over it), issue order PV_0(j), S_0(j+1), PV_1(j),
# S_1(j+1) per KV tile.  Besides the phase checks, this model tracks the data each
# tensor-core product reads and writes, and flags a hazard when
#  - a K or V ring slot is reloaded while a product that reads it is still queued,
#  - a score product writes a Q tile's buffer while its softmax is reading it, or
#    before the PV product that reads P from it has run,
#  - a softmax rescales O_t while a PV product into O_t is still queued.

def _run_bf16(nt, seed, kst=3, vst=2, plant=None):
    rng = random.Random(seed)
    ntiles = max(nt)
    bars, issues, tensor_q, tma = {}, [], [], []
    reading = {0: False, 1: False}   # softmax t between its score wait and its P arrival

    def bar(name, count=1):
        bars.setdefault(name, _Bar(name, count))
        return bars[name]

    for i in range(kst):
        bar("k_full%d" % i), bar("k_empty%d" % i)
    for i in range(vst):
        bar("v_full%d" % i), bar("v_ready%d" % i), bar("v_empty%d" % i)
    for t in range(2):
        bar("s_full%d" % t), bar("p_full%d" % t), bar("o_done%d" % t)

    def wait(name, phase):
        return ("wait", name, phase)

    def producer():
        for j in range(ntiles):
            if j >= kst:
                yield wait("k_empty%d" % (j % kst), j // kst - 1)
            tma.append(("k_full%d" % (j % kst), ("K", j % kst), j))
            yield ("step",)
            if j >= vst:
                yield wait("v_empty%d" % (j % vst), j // vst - 1)
            tma.append(("v_full%d" % (j % vst), ("V", j % vst), j))
            yield ("step",)
            if rng.random() < 0.3:   # the sequence's last block: zero its tail once landed
                yield wait("v_full%d" % (j % vst), j // vst)
            bars["v_ready%d" % (j % vst)].arrive()
            yield ("step",)

    def issuer():
        def s_mma(t, j):
            tensor_q.append(("S", {("K", j % kst)}, t, j))
            tensor_q.append(("commit", set(), "s_full%d" % t))

        def pv_mma(t, j):
            tensor_q.append(("PV", {("V", j % vst)}, t, j))

        if plant == "early_k_empty":   # a slot released before its products are issued
            tensor_q.append(("commit", set(), "k_empty0"))
        yield wait("k_full0", 0)
        for t in range(2):
            if nt[t] > 0:
                s_mma(t, 0)
        if plant != "early_k_empty":
            tensor_q.append(("commit", set(), "k_empty0"))
        yield ("step",)
        for j in range(ntiles):
            v_in = k_in = False
            if plant == "early_k_empty" and j + 1 < ntiles:
                tensor_q.append(("commit", set(), "k_empty%d" % ((j + 1) % kst)))
            order = [(t, kind) for t in range(2) for kind in ("pv", "s")]
            if plant == "s_before_pv":
                order = [(t, kind) for t in range(2) for kind in ("s", "pv")]
            for t, kind in order:
                if kind == "pv" and j < nt[t]:
                    yield wait("p_full%d" % t, j)
                    if not v_in:   # V landed (copy) and its empty rows zeroed (producer)
                        if plant != "no_v_landing":
                            yield wait("v_full%d" % (j % vst), j // vst)
                        yield wait("v_ready%d" % (j % vst), j // vst)
                        v_in = True
                    pv_mma(t, j)
                    if j == nt[t] - 1:
                        tensor_q.append(("commit", set(), "o_done%d" % t))
                    yield ("step",)
                if kind == "s" and j + 1 < nt[t]:
                    if not k_in:
                        yield wait("k_full%d" % ((j + 1) % kst), (j + 1) // kst)
                        k_in = True
                    s_mma(t, j + 1)
                    yield ("step",)
            if j + 1 < ntiles and plant != "early_k_empty":
                tensor_q.append(("commit", set(), "k_empty%d" % ((j + 1) % kst)))
            tensor_q.append(("commit", set(), "v_empty%d" % (j % vst)))
            yield ("step",)

    def softmax(t):
        for j in range(nt[t]):
            yield wait("s_full%d" % t, j)
            reading[t] = True
            if j > 0 and rng.random() < 0.3:   # a rescale of O_t: every PV into it has run
                if any(op[0] == "PV" and op[2] == t for op in tensor_q):
                    issues.append("softmax %d rescales O at tile %d with a PV product queued" % (t, j))
            yield ("step",)
            reading[t] = False
            bars["p_full%d" % t].arrive()
            yield ("step",)
        if nt[t] > 0:
            yield wait("o_done%d" % t, 0)

    roles = {"producer": producer(), "issuer": issuer(), "softmax0": softmax(0), "softmax1": softmax(1)}
    cur = {k: next(g, None) for k, g in roles.items()}
    pv_done = {0: -1, 1: -1}
    # how eagerly the tensor core and the copies progress, drawn per schedule, so that
    # some schedules let products or copies lag far behind the threads
    weight = {"tensor": rng.choice((0.05, 0.3, 1.0, 3.0)), "tma": rng.choice((0.05, 0.3, 1.0, 3.0))}
    for _ in range(400000):
        ready = [k for k, st in cur.items() if st is not None and
                 (st[0] != "wait" or (bars[st[1]].done & 1) != (st[2] & 1))]
        if tensor_q:
            ready.append("tensor")
        if tma:
            ready.append("tma")
        if not ready:
            if any(v is not None for v in cur.values()):
                issues.append("deadlock: " + ", ".join("%s waits %s" % (k, v[1:]) for k, v in cur.items() if v))
            return issues
        k = rng.choices(ready, weights=[weight.get(r, 1.0) for r in ready])[0]
        if k == "tensor":
            op = tensor_q.pop(0)
            if op[0] == "commit":
                bars[op[2]].arrive()
            elif op[0] == "S":
                t, j = op[2], op[3]
                if reading[t]:
                    issues.append("S_%d(%d) overwrote scores the softmax was reading" % (t, j))
                if j > 0 and pv_done[t] < j - 1:
                    issues.append("S_%d(%d) overwrote P_%d(%d) before its PV ran" % (t, j, t, j - 1))
            elif op[0] == "PV":
                pv_done[op[2]] = op[3]
                if any(x[1] == ("V", (op[3] % vst)) and x[2] == op[3] for x in tma):
                    issues.append("PV_%d(%d) read V before its copy landed" % (op[2], op[3]))
        elif k == "tma":
            name, slot, j = tma.pop(rng.randrange(len(tma)))
            # the copy lands: no queued product may still read the slot's previous tile
            if any(slot in op[1] for op in tensor_q):
                issues.append("%s slot %d overwritten by tile %d under a queued product" % (slot[0], slot[1], j))
            bars[name].arrive()
        else:
            st = cur[k]
            if st[0] == "wait":
                c = bars[st[1]].done
                if c not in (st[2], st[2] + 1):
                    issues.append("%s passed a wait for phase %d of %s with %d phases done" % (k, st[2], st[1], c))
            cur[k] = next(roles[k], None)
    issues.append("no progress bound reached")
    return issues


def _cases_bf16(n):
    rng = random.Random(4321)
    for i in range(n):
        if rng.random() < 0.15:   # Q tile 1 past the last query row: it reads no KV tile
            yield [rng.randint(1, 9), 0], i
            continue
        n1 = rng.randint(1, 9)
        n0 = rng.randint(0, n1)   # otherwise Q tile 0 never reads more KV tiles than Q tile 1
        yield [n0, n1], i


@pytest.mark.parametrize("kst,vst", [(2, 2), (3, 2), (2, 3), (4, 3)])
def test_bf16_protocol_is_free_of_hazards_and_deadlock(kst, vst):
    for nt, seed in _cases_bf16(1500):
        issues = _run_bf16(nt, seed, kst, vst)
        assert not issues, (nt, seed, issues[:2])


@pytest.mark.parametrize("plant,least", [("early_k_empty", 10), ("s_before_pv", 200), ("no_v_landing", 20)])
def test_bf16_protocol_mistakes_are_caught(plant, least):
    """Releasing a K slot before its products are issued lets the producer overwrite
    it under a queued product; issuing S_t(j+1) before PV_t(j) overwrites P_t(j); a PV
    issued on the producer's zeroing signal alone may read V before its copy lands
    (the V copy has its own barrier, apart from K's)."""
    caught = sum(bool(_run_bf16(nt, seed, 3, 2, plant=plant)) for nt, seed in _cases_bf16(300))
    assert caught >= least
