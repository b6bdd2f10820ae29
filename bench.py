"""Benchmark of the paged KV-cache decode step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload gqa70b]
                    [--impl ours|reference] [--partition P]

A step is one pass of the hot path over one batch: the KV write of every
sequence's new token (plus the copy-on-write block copies for the shared-prefix
workload), then paged decode attention over every context.  The default
workload is the Llama-3.1-70B-shaped GQA batch (256 sequences x 4,096 tokens,
64 query / 8 KV heads, head_dim 128, bf16).  The KV pools (5 GiB) exceed the
126 MB L2, so every step streams the cache from HBM.

Metric: effective KV bytes read per second (sum over sequences of
len * kv_heads * head_dim * 2 (K, V) * element size, divided by the step time);
also sequence-tokens per second and microseconds per step.

Multi-GPU (torchrun, one rank per GPU): every rank runs its own batch of the
same shape (independent sequences, no collective on the data path); the time is
the max over ranks and the value the sum over ranks (weak scaling).

--impl reference times the CPU oracle (the plain fp64 reference) on a bounded
sample of the same workload, on this host's cores.

--workload prefill70b measures the prompt pass instead (a separate line): 16
prompts of 512..4,096 tokens (Llama-3.1-70B shape) written into blocks with the
multi-token KV write, then causal paged attention over them; metric TFLOP/s of
the causal attention (4 * Hq * D * sum over query rows of keys attended),
roofline against the measured dense bf16 tensor peak.  --workload
prefill70b_fp8 is the same pass over an FP8 E4M3 cache (the products run in
f16, whose dense tensor rate equals bf16's).

--workload beam measures the beam-search step (a separate line): the host
block-manager work of every step (forks, frees, appends with copy-on-write,
tables, prefix groups) is done ahead and timed apart; the timed device step is
copy-on-write copies + KV write + shared-prefix decode with that step's inputs.

--swap measures block swap instead (a separate line, not the headline): a
quarter of the gqa70b batch (64 sequences x 4,096 tokens, 1 GiB of K+V) moves
from scattered device blocks to a page-locked host pool and back through
pkv_swap_blocks; the roofline is one contiguous copy-engine transfer of the
same bytes in the same direction, measured in the same run.
"""
import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "paged decode attention: effective KV HBM GB/s (% of B200 peak); seq-tokens/s"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0

DESCR = {
    "gqa70b": "Llama-3.1-70B-shaped GQA decode: 64 q / 8 kv heads, head_dim 128, bf16, 256 seqs x 4096 tokens, "
              "block 16, one new token per sequence",
    "mha13b": "LLaMA-13B-shaped MHA decode: 40 heads, head_dim 128, bf16, 64 seqs, lengths U[128, 2048], block 16",
    "shared_prefix": "shared-prefix parallel sampling: 64 prompts x n=3, 1000-token prefix + U{0..512}, GQA 32/8, "
                     "head_dim 128, bf16, copy-on-write + write + decode per step",
    "fp8_long": "FP8 E4M3 cache, GQA 32/8, head_dim 128, 128 seqs, lengths log-U[256, 32768], write + split decode",
    "prefill70b": "prompt pass, Llama-3.1-70B shape: 64 q / 8 kv heads, head_dim 128, bf16, 16 prompts of "
                  "U[512, 4096] tokens: multi-token KV write + causal paged attention",
    "prefill70b_fp8": "prompt pass, Llama-3.1-70B shape: 64 q / 8 kv heads, head_dim 128, bf16 q, FP8 E4M3 cache "
                      "(per-tensor scales), 16 prompts of U[512, 4096] tokens: multi-token KV write (quantising) + "
                      "causal paged attention",
    "beam": "beam search: 16 requests x 4 beams over a 1000-token prompt, GQA 32/8, head_dim 128, bf16; every "
            "step forks the kept beams, frees the old ones, copies shared partial blocks on write, writes one token "
            "per beam and decodes (shared-prefix decode)",
}


# ------------------------------------------------------------------ distributed helpers

def dist_env():
    """(rank, world, local_rank) from the torchrun environment (1 process by default)."""
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), int(os.environ.get("LOCAL_RANK", 0))


def reduce_max(value: float, world: int, device=None) -> float:
    """Max of a float over all ranks (the job's time is its slowest rank's)."""
    if world <= 1:
        return value
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def spread_us(ms_list):
    """p10 / median / p90 of per-step times (ms in, us out)."""
    ys = sorted(ms_list)
    at = lambda f: ys[min(len(ys) - 1, int(round(f * (len(ys) - 1))))]  # noqa: E731
    return {"p10": round(1e3 * at(0.1), 2), "median": round(1e3 * statistics.median(ys), 2),
            "p90": round(1e3 * at(0.9), 2)}


def rank_workload(w: W.Workload, rank: int) -> W.Workload:
    """Weak scaling: each rank gets an independent batch of the same shape (its own seed)."""
    return W.scaled(w, seed=w.seed + 1000 * rank) if rank else w


# ------------------------------------------------------------------ measurement helpers

def measured_peak_hbm():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:  # noqa: BLE001 - absent or unreadable: the pool's earlier figure
        return FALLBACK_HBM_GBS, "fallback"


DECODE_SOURCES = ("decode_tc.cu", "pkv_common.cuh", "decode_plan.cu", "api.cu")
PREFILL_SOURCES = ("prefill_tc.cu", "pkv_common.cuh", "api.cu")


def code_of(text: str) -> str:
    """C/C++/CUDA source without its comments, trailing spaces and blank lines: what a
    change of comments leaves the same (the kernels compile to the same code)."""
    out, i, n = [], 0, len(text)
    while i < n:
        if text.startswith("//", i):
            i = text.find("\n", i)
            i = n if i < 0 else i
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
        elif text[i] == '"':                                  # a string literal (inline PTX)
            j = i + 1
            while j < n and text[j] != '"':
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        else:
            out.append(text[i])
            i += 1
    lines = (line.rstrip() for line in "".join(out).splitlines())
    return "\n".join(line for line in lines if line)


def kernel_source_hash(files=DECODE_SOURCES, read=None):
    """Hash of the kernel sources' code (comments left out), keying the committed ncu
    traffic of a workload to the code it was captured from."""
    h = hashlib.sha256()
    for f in files:
        if read is None:
            with open(os.path.join(ROOT, "paged_kv_cache_404_b200", "csrc", f), encoding="utf-8") as fh:
                text = fh.read()
        else:
            text = read(f)
        h.update(code_of(text).encode("utf-8"))
    return h.hexdigest()[:16]


def ncu_traffic(workload):
    """DRAM bytes per decode launch from a committed ncu capture, if it was taken
    on the current kernel source (else None)."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f).get(workload)
    except Exception:  # noqa: BLE001
        return None
    files = PREFILL_SOURCES if workload.startswith("prefill") else DECODE_SOURCES
    if not rec or rec.get("source_hash") != kernel_source_hash(files):
        return None
    return rec.get("dram_bytes_per_launch")


class ClockSampler:
    """SM clock and clock-event (throttle) reasons sampled through NVML (read
    only) every ~2 ms on a background thread during the timed region."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"),
               ("hw_power_brake", "nvmlClocksEventReasonHwPowerBrakeSlowdown"))

    def __init__(self, device, period_s=0.002):
        self.device = device
        self.period = period_s
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._stop = None

    def __enter__(self):
        import threading
        try:
            import pynvml
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(self.device).uuid)
            h = pynvml.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            masks = [(n, getattr(pynvml, c)) for n, c in self.REASONS if hasattr(pynvml, c)]
        except Exception:  # noqa: BLE001 - no NVML: no clock record
            return self
        self._stop = threading.Event()

        def run():
            while not self._stop.is_set():
                try:
                    self.samples.append(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM))
                    r = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                    self.reasons.update(n for n, m in masks if r & m)
                except Exception:  # noqa: BLE001
                    return
                self._stop.wait(self.period)

        self._thread = threading.Thread(target=run, daemon=True)
        self._thread.start()
        return self

    def __exit__(self, *exc):
        if self._stop is not None:
            self._stop.set()
            self._thread.join(timeout=2)

    def summary(self):
        if not self.samples:
            return None
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples), "source": "nvml"}


# ------------------------------------------------------------------ workload set-up (product side)

class Step:
    """Device-resident inputs of one decode step and the calls that run it."""

    def __init__(self, w: W.Workload, device, partition=0, prefix_groups=True, cont=None):
        import paged_kv_cache_404_b200 as pkv
        self.pkv = pkv
        self.w = w
        self.device = device
        self.partition = partition
        self.groups = None
        if w.lens == "shared":
            self._setup_shared(cont)
        else:
            self._setup_flat()
        self.max_len = int(self.lens.max())
        self.g_slots = torch.from_numpy(self.slots).to(device)
        self.g_tables = torch.from_numpy(self.tables).to(device)
        self.g_lens = torch.from_numpy(self.lens).to(device)
        self.g_pairs = torch.from_numpy(self.pairs).to(device) if len(self.pairs) else None
        if self.groups is not None and prefix_groups:
            # shared-prefix decode: each prompt's blocks are read once for its samples
            offs, mem, sh = self.groups
            self.g_offs = torch.from_numpy(offs).to(device)
            self.g_mem = torch.from_numpy(mem).to(device)
            self.g_sh = torch.from_numpy(sh).to(device)
        else:
            self.groups = None
        self.ws = pkv.decode_workspace(self.S, w.num_heads, w.head_dim, self.max_len, partition, device=device,
                                       shared=self.groups is not None)
        self.out = torch.empty_like(self.q)
        self.err = torch.zeros(1, dtype=torch.int32, device=device)
        elem = 1 if w.cache_dtype == "fp8" else 2
        self.kv_bytes = int(self.lens.astype(np.int64).sum()) * w.num_kv_heads * w.head_dim * 2 * elem
        self.seq_tokens = int(self.lens.astype(np.int64).sum())
        # write + plan + decode (+ merge when a split is possible) (+ copy-on-write copy)
        merge = (partition or 256) < self.max_len or self.groups is not None
        self.launches = 3 + int(merge) + int(self.g_pairs is not None)

    def _setup_flat(self):
        pkv, w, dev = self.pkv, self.w, self.device
        lens = W.context_lens(w)
        self.S = len(lens)
        need = int(sum(-(-int(L) // 16) for L in lens))
        NB = W.pool_blocks(w, need)
        bm = pkv.BlockManager(NB, 16, free_order=W.free_order(w, NB))
        ids = [bm.alloc_seq(int(L) - 1) for L in lens]
        slots, pairs = bm.append_tokens(ids)
        self.slots, self.pairs = slots, pairs
        self.tables, self.lens = bm.tables(ids, max(-(-int(L) // 16) for L in lens), pad=-1)
        self.k_pool, self.v_pool, self.k_scale, self.v_scale = W.random_pools(w, NB, dev)
        self.q = W.queries(w, self.S, dev)
        self.k_new, self.v_new = W.new_tokens(w, self.S, dev)
        self.NB = NB

    def _setup_shared(self, cont=None):
        """Prompts written once and forked; continuations replayed token by token
        (copy-on-write on first divergence); the step is the next token of all.
        cont: continuation lengths (default: the workload's; all zero makes the
        step the divergence step, where every prompt's partly filled block splits)."""
        pkv, w, dev = self.pkv, self.w, self.device
        cont = W.continuation_lens(w) if cont is None else np.asarray(cont, np.int32)
        S = self.S = w.num_prompts * w.samples
        est = w.num_prompts * (-(-w.prefix_len // 16)) + int(sum(-(-(int(c) + 17) // 16) for c in cont)) + S
        NB = int(math.ceil(est * w.pool_factor))
        bm = pkv.BlockManager(NB, 16, free_order=W.free_order(w, NB))
        kp, vp = W.stale_fill(w, NB, dev)
        pk, pv = W.logical_kv(w, w.num_prompts * w.prefix_len, dev, stream=50)
        ck, cv = W.logical_kv(w, int(cont.sum()) + 1, dev, stream=60)
        ids = []
        for p in range(w.num_prompts):
            parent = bm.alloc_seq(w.prefix_len)
            sl = slice(p * w.prefix_len, (p + 1) * w.prefix_len)
            pkv.paged_kv_write(pk[sl], pv[sl], torch.from_numpy(bm.slots(parent, 0, w.prefix_len)).to(dev), kp, vp)
            ids += [parent] + [bm.fork(parent) for _ in range(w.samples - 1)]
        cur = 0
        for t in range(int(cont.max())):
            act = [ids[i] for i in range(S) if cont[i] > t]
            slots, pairs = bm.append_tokens(act)
            if len(pairs):
                pkv.copy_blocks(kp, vp, torch.from_numpy(pairs).to(dev))
            pkv.paged_kv_write(ck[cur:cur + len(act)], cv[cur:cur + len(act)], torch.from_numpy(slots).to(dev), kp, vp)
            cur += len(act)
        self.slots, self.pairs = bm.append_tokens(ids)
        self.tables, self.lens = bm.tables(ids, max(-(-int(bm.seq_len(s)) // 16) for s in ids), pad=-1)
        self.groups = bm.prefix_groups(ids)
        # memory saved by sharing: physical blocks in use vs one private copy per sequence
        used = len({int(b) for row in self.tables for b in row if b >= 0})
        private = int(sum(-(-int(L) // 16) for L in self.lens))
        self.mem_saving = 1.0 - used / private
        self.k_pool, self.v_pool, self.k_scale, self.v_scale = kp, vp, 1.0, 1.0
        self.q = W.queries(w, S, dev)
        self.k_new, self.v_new = W.new_tokens(w, S, dev)
        self.NB = NB
        torch.cuda.synchronize()

    def copy_and_write(self):
        if self.g_pairs is not None:
            self.pkv.copy_blocks(self.k_pool, self.v_pool, self.g_pairs, err_count=self.err)
        self.pkv.paged_kv_write(self.k_new, self.v_new, self.g_slots, self.k_pool, self.v_pool, self.k_scale,
                                self.v_scale, err_count=self.err)

    def decode(self):
        if self.groups is not None:
            self.pkv.paged_attention_decode_shared(self.out, self.q, self.k_pool, self.v_pool, self.g_tables,
                                                   self.g_lens, self.w.scale, self.max_len, self.ws, self.g_offs,
                                                   self.g_mem, self.g_sh, self.k_scale, self.v_scale,
                                                   partition_tokens=self.partition, err_count=self.err)
            return
        self.pkv.paged_attention_decode(self.out, self.q, self.k_pool, self.v_pool, self.g_tables, self.g_lens,
                                        self.w.scale, self.max_len, self.ws, self.k_scale, self.v_scale,
                                        partition_tokens=self.partition, err_count=self.err)

    def run(self):
        self.copy_and_write()
        self.decode()


def time_steps(step: Step, steps: int, warmup: int, world: int, device):
    """K timed steps between a barrier + synchronize on both sides, timed with CUDA
    events on the launching stream at the start and the end only (an event between
    two kernels keeps the second from starting before the first has finished, so
    per-step events would hide the overlap of a step's kernels).  A second pass
    over the same steps records events around the write and the decode call of
    each step, for their split and spread."""
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        step.run()
    torch.cuda.synchronize()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for _ in range(steps):
        step.run()
    end.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    total_ms = start.elapsed_time(end)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for a, b, c in ev:
        a.record(stream)
        step.copy_and_write()
        b.record(stream)
        step.decode()
        c.record(stream)
    torch.cuda.synchronize()
    decode_ms = [b.elapsed_time(c) for _, b, c in ev]
    write_ms = [a.elapsed_time(b) for a, b, _ in ev]
    return total_ms, decode_ms, write_ms


def divergence_step(w, device, args):
    """The shared-prefix step right after the prompts: all continuations empty, so
    every prompt's partly filled last block is copied for all but its last holder."""
    step = Step(w, device, prefix_groups=not args.no_prefix_groups, cont=np.zeros(w.num_prompts * w.samples))
    reps = 20
    for _ in range(3):
        step.run()
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(reps)]
    for a, b, c in ev:
        a.record()
        step.copy_and_write()
        b.record()
        step.decode()
        c.record()
    torch.cuda.synchronize()
    cw = statistics.median(a.elapsed_time(b) for a, b, _ in ev)
    dec = statistics.median(b.elapsed_time(c) for _, b, c in ev)
    npairs = len(step.pairs)
    block_bytes = step.k_pool[0].numel() * step.k_pool.element_size()
    return {"copy_pairs": npairs, "copy_bytes": 2 * npairs * block_bytes, "us_copy_and_write": round(1e3 * cw, 2),
            "us_decode": round(1e3 * dec, 2), "device_errors": int(step.err.item())}


def pack_inputs(tensors, device, copies=1):
    """One pinned host buffer holding the bytes of `tensors` (name -> tensor), and
    `copies` device buffers of the same layout with a view per name in each, so that
    a step's inputs go up in one copy.  Offsets are 256-byte aligned.  Returns
    (host buffer, [device buffers], [views per device buffer], input bytes)."""
    offs, total = {}, 0
    for n, v in tensors.items():
        offs[n] = total
        total += -(-v.numel() * v.element_size() // 256) * 256
    host = torch.empty(max(total, 256), dtype=torch.uint8).pin_memory()
    for n, v in tensors.items():
        nb = v.numel() * v.element_size()
        host[offs[n]:offs[n] + nb].copy_(v.detach().cpu().contiguous().view(-1).view(torch.uint8))
    devs, views = [], []
    for _ in range(copies):
        d = torch.empty(max(total, 256), dtype=torch.uint8, device=device)
        devs.append(d)
        views.append({n: d[offs[n]:offs[n] + v.numel() * v.element_size()].view(v.dtype).view(v.shape)
                      for n, v in tensors.items()})
    return host, devs, views, sum(v.numel() * v.element_size() for v in tensors.values())


def time_e2e(step, steps: int, warmup: int, world: int, names=None):
    """The same step through the public API from pinned HOST buffers.  Every
    step copies its inputs (q, new K/V, slots, tables, lengths, copy pairs)
    host->device and reads its output back device->host inside the timed
    region.  The inputs are packed into one pinned buffer and go up in one copy
    (per-copy overhead, not bytes, dominates a step's uploads); the copies run
    on a second stream with two device input sets, so step i+1's uploads and
    step i-1's download overlap step i's kernels, as in a serving loop; the KV
    pools stay resident (they are the cache, not a per-step input).  Uploads
    and downloads use separate streams."""
    compute = torch.cuda.current_stream()
    up = torch.cuda.Stream(device=step.device)
    down = torch.cuda.Stream(device=step.device)
    if names is None:   # a decode Step
        names = ["q", "k_new", "v_new", "g_slots", "g_tables", "g_lens"] + (
            ["g_pairs"] if step.g_pairs is not None else [])
        if step.groups is not None:
            names += ["g_offs", "g_mem", "g_sh"]
    saved = {n: getattr(step, n) for n in names}
    host, dev_bufs, dev, h2d = pack_inputs(saved, step.device, copies=2)
    outs = [step.out, torch.empty_like(step.out)]
    out_host = [torch.empty(step.out.shape, dtype=step.out.dtype).pin_memory() for _ in range(2)]
    d2h = out_host[0].numel() * out_host[0].element_size()
    uploaded = [torch.cuda.Event() for _ in range(2)]
    computed = [torch.cuda.Event() for _ in range(2)]
    consumed = [torch.cuda.Event() for _ in range(2)]   # set b's inputs no longer needed
    downloaded = [torch.cuda.Event() for _ in range(2)]  # output b read back: free to overwrite

    def run(n_steps):
        for i in range(n_steps):
            b = i & 1
            with torch.cuda.stream(up):
                if i >= 2:
                    up.wait_event(consumed[b])
                dev_bufs[b].copy_(host, non_blocking=True)
                uploaded[b].record(up)
            compute.wait_event(uploaded[b])
            if i >= 2:
                compute.wait_event(downloaded[b])
            for n in names:
                setattr(step, n, dev[b][n])
            step.out = outs[b]
            step.run()
            computed[b].record(compute)
            consumed[b].record(compute)
            with torch.cuda.stream(down):
                down.wait_event(computed[b])
                out_host[b].copy_(outs[b], non_blocking=True)
                downloaded[b].record(down)
        compute.wait_stream(up)
        compute.wait_stream(down)

    run(warmup)
    torch.cuda.synchronize()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    a = torch.cuda.Event(enable_timing=True)
    z = torch.cuda.Event(enable_timing=True)
    a.record(compute)
    up.wait_event(a)
    down.wait_event(a)
    run(steps)
    z.record(compute)
    torch.cuda.synchronize()
    for n in names:
        setattr(step, n, saved[n])
    step.out = outs[0]
    return a.elapsed_time(z), h2d, d2h


# ------------------------------------------------------------------ CPU oracle timing

def oracle_sample_step(w: W.Workload, num_seqs: int, seed_offset=0):
    """Oracle inputs for `num_seqs` sequences of the workload (host, CPU
    generator): pool, tables, lengths, q and the step's new tokens."""
    import oracle
    if w.lens == "shared":
        lens = (w.prefix_len + W.continuation_lens(w) + 1).astype(np.int32)
    else:
        lens = W.context_lens(w)
    lens = lens[seed_offset:seed_offset + num_seqs]
    wn = W.scaled(w, num_seqs=len(lens))
    need = int(sum(-(-int(L) // 16) for L in lens))
    NB = need + 1
    ref = oracle.RefBlockManager(NB, 16, free_order=W.free_order(wn, NB))
    ids = [ref.alloc_seq(int(L) - 1) for L in lens]
    slots = [ref.append_token(s)[0] for s in ids]
    maxb = max(-(-int(L) // 16) for L in lens)
    tabs = np.full((len(lens), maxb), -1, np.int32)
    for i, s in enumerate(ids):
        tabs[i, :len(ref.tables[s])] = ref.tables[s]
    kp, vp, ks, vs = W.random_pools(wn, NB, "cpu")
    q = W.queries(wn, len(lens), "cpu")
    kn, vn = W.new_tokens(wn, len(lens), "cpu")
    bits = lambda t: t.view(torch.int16).numpy().view(np.uint16) if t.dtype == torch.bfloat16 else t.numpy()
    return dict(oracle=oracle, lens=lens, tabs=tabs, slots=np.array(slots, np.int64), kp=bits(kp).copy(),
                vp=bits(vp).copy(), ks=ks, vs=vs, q=bits(q), kn=bits(kn), vn=bits(vn), w=wn)


def oracle_run(d, threads=0):
    oracle = d["oracle"]
    w = d["w"]
    cdt = {"f32": oracle.F32, "bf16": oracle.BF16, "fp8": oracle.FP8_E4M3}[w.cache_dtype]
    sdt = oracle.F32 if w.cache_dtype == "f32" else oracle.BF16
    qdt = oracle.F32 if w.q_dtype == "f32" else oracle.BF16
    oracle.kv_write(d["kn"], d["vn"], sdt, d["slots"], d["kp"], d["vp"], cdt, 16, d["ks"], d["vs"])
    oracle.paged_attention_decode(d["q"], qdt, d["kp"], d["vp"], cdt, d["tabs"], d["lens"], w.scale, d["ks"],
                                  d["vs"], num_threads=threads)


def cpu_baseline(w: W.Workload, target_s=12.0):
    """The oracle as it stands (fp64, OpenMP over (sequence, head), all cores) on
    a bounded sample of the workload; returns the same metric (KV GB/s)."""
    import oracle
    elem = 1 if w.cache_dtype == "fp8" else 2
    per_tok = w.num_kv_heads * w.head_dim * 2 * elem
    n = 1
    d = oracle_sample_step(w, n)
    t0 = time.perf_counter()
    oracle_run(d)
    dt = time.perf_counter() - t0
    n = int(max(1, min(w.num_seqs, math.floor(target_s / max(dt, 1e-3)))))
    d = oracle_sample_step(w, n)
    t0 = time.perf_counter()
    oracle_run(d)
    dt = time.perf_counter() - t0
    toks = int(d["lens"].astype(np.int64).sum())
    return {"value": round(toks * per_tok / dt / 1e9, 4), "unit": "GB/s", "cores": oracle.max_threads(),
            "kind": "oracle",
            "sample": "%d of %d sequences (%d tokens), one write + decode step, fp64, %.2f s" % (
                n, w.num_seqs, toks, dt),
            "seq_tokens_per_s": round(toks / dt, 1)}


def run_reference(args, w, rank, world):
    """--impl reference: the CPU oracle, timed on this host, on bounded samples."""
    if rank != 0:
        return
    import oracle
    if w.name.startswith("prefill"):
        t0 = time.perf_counter()
        samples = [prefill_cpu_baseline(w, target_s=2.0) for _ in range(args.steps)]
        total = time.perf_counter() - t0
        value = statistics.mean(x["value"] for x in samples)
        line = {"metric": "causal paged prefill attention TFLOP/s (4*Hq*D*keys attended per query row)",
                "value": value, "unit": "TFLOP/s", "impl": "reference", "n_gpus": world, "steps": args.steps,
                "warmup": 0, "ms_per_step": round(1e3 * total / args.steps, 3), "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "config": {"workload": w.name + ": " + DESCR[w.name], "parallelism": "cpu (OpenMP)"},
                "cpu_baseline": dict(samples[-1], value=value),
                "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return
    elem = 1 if w.cache_dtype == "fp8" else 2
    per_tok = w.num_kv_heads * w.head_dim * 2 * elem
    # size one step's sample to about 3 s of CPU work
    probe = oracle_sample_step(w, 1)
    t0 = time.perf_counter()
    oracle_run(probe)
    dt = time.perf_counter() - t0
    n = int(max(1, min(w.num_seqs, math.floor(3.0 / max(dt, 1e-3)))))
    d = oracle_sample_step(w, n)
    for _ in range(args.warmup):
        oracle_run(d)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_run(d)
    total = time.perf_counter() - t0
    toks = int(d["lens"].astype(np.int64).sum())
    value = toks * per_tok * args.steps / total / 1e9
    sample = "%d of %d sequences (%d tokens) per step, fp64 oracle, write + decode" % (n, w.num_seqs, toks)
    line = {
        "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "impl": "reference",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * total / args.steps, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": args.workload + ": " + DESCR[args.workload], "global_batch": n,
                   "seq_len": int(d["lens"].max()), "parallelism": "cpu (OpenMP)"},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": oracle.max_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "seq_tokens_per_s": round(toks * args.steps / total, 1),
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ main

def measured_peak_tensor():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["bf16_tflops"]), "measured (cuBLAS bf16 burst)"
    except Exception:  # noqa: BLE001
        return 1590.0, "fallback"


class PrefillStep:
    """Device-resident inputs of one prompt pass: every prompt token's K/V written
    at its slot, then causal attention of every prompt token."""

    def __init__(self, w, device):
        import paged_kv_cache_404_b200 as pkv
        self.pkv, self.w, self.device = pkv, w, device
        lens = W.context_lens(w)
        self.S = len(lens)
        need = int(sum(-(-int(L) // 16) for L in lens))
        NB = W.pool_blocks(w, need)
        bm = pkv.BlockManager(NB, 16, free_order=W.free_order(w, NB))
        ids = [bm.alloc_seq(int(L)) for L in lens]
        self.total = int(lens.astype(np.int64).sum())
        slots = np.concatenate([bm.slots(s, 0, int(L)) for s, L in zip(ids, lens)])
        tables, self.lens = bm.tables(ids, max(-(-int(L) // 16) for L in lens), pad=-1)
        self.k_pool, self.v_pool = W.stale_fill(w, NB, device)
        self.k_new, self.v_new = W.logical_kv(w, self.total, device, stream=80)
        self.fp8 = w.cache_dtype == "fp8"
        # FP8: per-tensor scales amax / 448 of the prompt's K and V
        self.k_scale = float(self.k_new.abs().max().float().item()) / 448.0 if self.fp8 else 1.0
        self.v_scale = float(self.v_new.abs().max().float().item()) / 448.0 if self.fp8 else 1.0
        self.q = W.queries(W.scaled(w, num_seqs=self.total), self.total, device)
        self.out = torch.empty_like(self.q)
        self.g_slots = torch.from_numpy(slots.astype(np.int64)).to(device)
        self.g_tables = torch.from_numpy(tables).to(device)
        self.g_lens = torch.from_numpy(self.lens).to(device)
        self.g_qs = torch.from_numpy(np.concatenate([[0], np.cumsum(self.lens)]).astype(np.int32)).to(device)
        self.max_q = int(self.lens.max())
        self.err = torch.zeros(1, dtype=torch.int32, device=device)
        L64 = self.lens.astype(np.float64)
        self.flops = 4.0 * w.num_heads * w.head_dim * float((L64 * (L64 + 1) / 2).sum())
        self.kv_bytes = self.total * w.num_kv_heads * w.head_dim * 2 * (1 if self.fp8 else 2)

    def write(self):
        self.pkv.paged_kv_write(self.k_new, self.v_new, self.g_slots, self.k_pool, self.v_pool, self.k_scale,
                                self.v_scale, err_count=self.err)

    def run(self):
        self.write()
        self.attend()

    def attend(self):
        self.pkv.paged_attention_prefill(self.out, self.q, self.k_pool, self.v_pool, self.g_tables, self.g_lens,
                                         self.g_qs, self.w.scale, self.max_q, err_count=self.err,
                                         k_scale=self.k_scale, v_scale=self.v_scale)


def prefill_cpu_baseline(w, target_s=12.0):
    """The oracle's causal attention on a bounded sample of query rows."""
    import oracle
    rng = np.random.default_rng(7)
    lens = W.context_lens(w)
    L = int(lens.max())   # rows of the longest prompt: the costliest per row
    NB = -(-L // 16)
    tabs = np.arange(NB, dtype=np.int32)[None]
    g = torch.Generator().manual_seed(1234)
    kp = torch.randn((NB, 16, w.num_kv_heads, w.head_dim), generator=g).to(torch.bfloat16)
    vp = torch.randn((NB, 16, w.num_kv_heads, w.head_dim), generator=g).to(torch.bfloat16)
    q = torch.randn((L, w.num_heads, w.head_dim), generator=g).to(torch.bfloat16)
    bits = lambda t: t.view(torch.int16).numpy().view(np.uint16)  # noqa: E731
    qs = np.array([0, L], np.int32)
    fp8 = w.cache_dtype == "fp8"
    if fp8:   # E4M3 codes of the same values (scale 1: |x| < 448)
        kb = kp.float().to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        vb = vp.float().to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    else:
        kb, vb = bits(kp), bits(vp)
    cdt = oracle.FP8_E4M3 if fp8 else oracle.BF16

    def run(rows):
        t0 = time.perf_counter()
        oracle.paged_attention_prefill(bits(q), oracle.BF16, kb, vb, cdt, tabs,
                                       np.array([L], np.int32), qs, w.scale, rows=rows)
        return time.perf_counter() - t0

    rows = np.sort(rng.choice(L, 4, replace=False))
    dt = run(rows)
    n = int(max(4, min(L, 4 * target_s / max(dt, 1e-3))))
    rows = np.sort(rng.choice(L, n, replace=False))
    dt = run(rows)
    flops = 4.0 * w.num_heads * w.head_dim * float((rows + 1).sum())
    return {"value": round(flops / dt / 1e12, 6), "unit": "TFLOP/s", "cores": oracle.max_threads(), "kind": "oracle",
            "sample": "%d query rows of a %d-token prompt (all 64 heads), fp64, %.2f s" % (n, L, dt)}


def run_prefill(args, w0, device, rank, world):
    w = rank_workload(w0, rank)
    step = PrefillStep(w, device)
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        step.write()
        step.attend()
    torch.cuda.synchronize()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    with ClockSampler(device) as clk:
        a0 = torch.cuda.Event(enable_timing=True)
        z0 = torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        for a, b, c in ev:
            a.record(stream)
            step.write()
            b.record(stream)
            step.attend()
            c.record(stream)
        z0.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    total_ms = reduce_max(a0.elapsed_time(z0), world, device)
    att_ms = statistics.mean(b.elapsed_time(c) for _, b, c in ev)
    wr_ms = statistics.mean(a.elapsed_time(b) for a, b, _ in ev)
    value = step.flops * world * args.steps / (total_ms / 1e3) / 1e12

    e2e = None
    if not args.no_e2e:
        # through the public API from pinned host buffers: inputs up, output down, every
        # step, pipelined as the decode lines are (time_e2e)
        n_e = max(3, args.steps // 4)
        e_ms, h2d, d2h = time_e2e(step, n_e, 2, world,
                                  names=["q", "k_new", "v_new", "g_slots", "g_tables", "g_lens", "g_qs"])
        e_ms = reduce_max(e_ms, world, device)
        e2e = {"value": round(step.flops * world * n_e / (e_ms / 1e3) / 1e12, 2), "unit": "TFLOP/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(e_ms / n_e, 4)}

    peak, peak_kind = measured_peak_tensor()
    achieved = step.flops / (att_ms / 1e3) / 1e12
    if rank == 0:
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            cpu = prefill_cpu_baseline(w, target_s=args.cpu_seconds)
        line = {
            "metric": "causal paged prefill attention TFLOP/s (4*Hq*D*keys attended per query row)",
            "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(total_ms / args.steps, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16 q, fp8 e4m3 cache (f16 products, fp32 accumulate)" if step.fp8 else "bf16 (fp32 accumulate)",
            "data": "synthetic (seeded N(0,1) q/K/V, seeded block placement)",
            "config": {"workload": w0.name + ": " + DESCR[w0.name], "global_batch": step.S * world,
                       "seq_len": step.max_q, "prompt_tokens": step.total,
                       "parallelism": "replicas: prompts sharded by rank, no collective",
                       "l2": "inputs larger than L2 (q %.0f MB + K/V %.0f MB per GPU vs 126 MB L2)" % (
                           step.q.numel() * 2 / 1e6, 2 * step.k_pool.numel() * step.k_pool.element_size() / 1e6)},
            "prompt_tokens_per_s": round(step.total * world * args.steps / (total_ms / 1e3), 1),
            "us_attention": round(1e3 * att_ms, 2), "us_write": round(1e3 * wr_ms, 2),
            "us_attention_spread": spread_us([b.elapsed_time(c) for _, b, c in ev]),
            "roofline": {"bound": "tensor", "achieved": round(achieved, 1), "peak": peak, "unit": "TFLOP/s",
                         "frac": round(achieved / peak, 4), "traffic": ncu_traffic(w0.name),
                         "kernel": ("prefill_fp8_kernel (64-key tiles" if step.fp8 else "prefill_bf16_kernel (128-key tiles")
                         + "; tcgen05.mma, TMEM accumulators)", "peak_source": peak_kind},
            "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": 2 * args.steps, "device_errors": int(step.err.item()),
            "clocks": clk.summary(),
        }
        return line
    return None


class BeamStep:
    """A beam-search trace: host decisions for every step prepared ahead (their
    host time measured), device inputs of every step resident before timing."""

    def __init__(self, w, device, total_steps):
        import paged_kv_cache_404_b200 as pkv
        self.pkv, self.w, self.device = pkv, w, device
        R, B, P = w.num_prompts, w.samples, w.prefix_len
        self.S = R * B
        NB = W.pool_blocks(w, R * (-(-P // 16)) + R * B * (total_steps // 16 + 3))
        bm = pkv.BlockManager(NB, 16, free_order=W.free_order(w, NB))
        self.k_pool, self.v_pool = W.stale_fill(w, NB, device)
        pk, pv = W.logical_kv(w, R * P, device, stream=50)
        beams = []
        for r in range(R):
            p = bm.alloc_seq(P)
            pkv.paged_kv_write(pk[r * P:(r + 1) * P], pv[r * P:(r + 1) * P],
                               torch.from_numpy(bm.slots(p, 0, P)).to(device), self.k_pool, self.v_pool)
            beams.append([p] + [bm.fork(p) for _ in range(B - 1)])
        beams = np.asarray(beams, dtype=np.int32)
        self.max_len = P + total_steps
        maxb = -(-self.max_len // 16)
        self.steps, host_s, self.pairs_total = [], 0.0, 0
        for t in range(total_steps):
            t0 = time.perf_counter()
            parents = W.beam_parents(w, t)
            # every request's kept beams fork from its current ones, then the old beams go
            par = np.take_along_axis(beams, parents, axis=1).ravel()
            kids = bm.fork_many(par)
            bm.free_many(beams.ravel())
            beams = kids.reshape(R, B)
            flat = kids
            slots, pairs = bm.append_tokens(flat)
            tabs, lens = bm.tables(flat, maxb, pad=-1)
            offs, mem, sh = bm.prefix_groups(flat)
            host_s += time.perf_counter() - t0
            g = lambda a, dt=torch.int32: torch.from_numpy(np.asarray(a)).to(device=device, dtype=dt)  # noqa: E731
            per_tok = w.num_kv_heads * w.head_dim * 2 * 2
            self.steps.append(dict(slots=g(slots, torch.int64), pairs=g(pairs, torch.int64) if len(pairs) else None,
                                   tables=g(tabs), lens=g(lens), offs=g(offs), mem=g(mem), sh=g(sh),
                                   kv_bytes=int(lens.astype(np.int64).sum()) * per_tok,
                                   unique_kv_bytes=unique_kv_bytes(tabs, lens, per_tok), npairs=len(pairs)))
            self.pairs_total += len(pairs)
        self.host_us_per_step = 1e6 * host_s / total_steps
        self.k_new, self.v_new = W.new_tokens(w, self.S, device)
        self.q = W.queries(w, self.S, device)
        self.out = torch.empty_like(self.q)
        self.ws = pkv.decode_workspace(self.S, w.num_heads, w.head_dim, self.max_len, 0, device=device, shared=True)
        self.err = torch.zeros(1, dtype=torch.int32, device=device)

    def copy_and_write(self, t):
        st = self.steps[t]
        if st["pairs"] is not None:
            self.pkv.copy_blocks(self.k_pool, self.v_pool, st["pairs"], err_count=self.err)
        self.pkv.paged_kv_write(self.k_new, self.v_new, st["slots"], self.k_pool, self.v_pool, err_count=self.err)

    def decode(self, t):
        st = self.steps[t]
        self.pkv.paged_attention_decode_shared(self.out, self.q, self.k_pool, self.v_pool, st["tables"], st["lens"],
                                               self.w.scale, self.max_len, self.ws, st["offs"], st["mem"], st["sh"],
                                               err_count=self.err)


def time_beam_e2e(step, idx, world):
    """Beam steps `idx` through the public API from pinned HOST buffers: every step
    uploads its inputs (slots, copy pairs, tables, lengths, prefix groups, new K/V,
    q) and reads its output back.  A step's inputs are packed into one pinned buffer
    and go up in one copy into a device buffer the step's tensors view; uploads run
    on one stream and downloads on another, overlapping the neighbouring steps'
    kernels; the output alternates between two buffers, with events ordering every
    reuse.  The host block-manager decisions are reported apart
    (host_block_manager_us_per_step).  Replaying a step is idempotent (same slots,
    same data, same copies).  Returns (ms, h2d bytes per step, d2h bytes per step)."""
    compute = torch.cuda.current_stream()
    up = torch.cuda.Stream(device=step.device)
    down = torch.cuda.Stream(device=step.device)
    common = ["q", "k_new", "v_new"]
    saved = {n: getattr(step, n) for n in common}
    packed = {}
    for t in set(idx):
        parts = {k: v for k, v in step.steps[t].items() if isinstance(v, torch.Tensor)}
        parts.update(saved)
        host, devs, views, nbytes = pack_inputs(parts, step.device)
        packed[t] = (host, devs[0], views[0], nbytes)
    originals = {t: dict(step.steps[t]) for t in packed}
    outs = [step.out, torch.empty_like(step.out)]
    out_host = [torch.empty(step.out.shape, dtype=step.out.dtype).pin_memory() for _ in range(2)]
    h2d = sum(packed[t][3] for t in idx) // len(idx)
    d2h = out_host[0].numel() * out_host[0].element_size()
    uploaded = [torch.cuda.Event() for _ in range(2)]
    computed = [torch.cuda.Event() for _ in range(2)]
    downloaded = [torch.cuda.Event() for _ in range(2)]
    consumed = {t: torch.cuda.Event() for t in packed}   # step t's device inputs read: free to refill
    used = set()                                          # steps whose `consumed` has been recorded

    def run(ts):
        for i, t in enumerate(ts):
            b = i & 1
            host, dev, views, _ = packed[t]
            with torch.cuda.stream(up):
                if t in used:                              # a repeated step index (fewer steps than uploads)
                    up.wait_event(consumed[t])
                dev.copy_(host, non_blocking=True)
                uploaded[b].record(up)
            compute.wait_event(uploaded[b])
            if i >= 2:
                compute.wait_event(downloaded[b])
            for k, v in views.items():
                if k in common:
                    setattr(step, k, v)
                else:
                    step.steps[t][k] = v
            step.out = outs[b]
            step.copy_and_write(t)
            step.decode(t)
            computed[b].record(compute)
            consumed[t].record(compute)
            used.add(t)
            with torch.cuda.stream(down):
                down.wait_event(computed[b])
                out_host[b].copy_(outs[b], non_blocking=True)
                downloaded[b].record(down)
        compute.wait_stream(up)
        compute.wait_stream(down)

    run(idx[:2])
    torch.cuda.synchronize()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    a = torch.cuda.Event(enable_timing=True)
    z = torch.cuda.Event(enable_timing=True)
    a.record(compute)
    up.wait_event(a)
    down.wait_event(a)
    run(idx)
    z.record(compute)
    torch.cuda.synchronize()
    for n in common:
        setattr(step, n, saved[n])
    for t, d in originals.items():
        step.steps[t] = d
    step.out = outs[0]
    return reduce_max(a.elapsed_time(z), world, step.device), h2d, d2h


def unique_kv_bytes(tables, lens, per_token):
    """KV bytes of the distinct (physical block, slot) pairs a decode step reads:
    a block shared by several sequences counts once, with the most tokens any of
    them reads from it."""
    tables = np.asarray(tables)
    lens = np.asarray(lens).astype(np.int64)
    nblk = -(-lens // 16)
    j = np.arange(tables.shape[1])[None, :]
    used = j < nblk[:, None]
    valid = np.minimum(16, lens[:, None] - 16 * j)
    blk = tables[used].astype(np.int64)
    cnt = valid[used]
    best = np.zeros(int(blk.max()) + 1 if blk.size else 1, dtype=np.int64)
    np.maximum.at(best, blk, cnt)
    return int(best.sum()) * per_token


class L2Flush:
    """A device buffer twice the 126 MB L2, written between timed steps so that no
    step finds the previous step's data in L2."""

    def __init__(self, device):
        self.buf = torch.empty(256 << 20, dtype=torch.uint8, device=device)

    def __call__(self):
        self.buf.fill_(1)


def run_beam(args, w0, device, rank, world):
    """Beam-search steps, each timed on its own with L2 flushed before it (the
    beams' KV, about 70 MB, would otherwise stay in the 126 MB L2 from one step
    to the next)."""
    w = rank_workload(w0, rank)
    step = BeamStep(w, device, args.warmup + args.steps)
    stream = torch.cuda.current_stream()
    flush = L2Flush(device)
    for t in range(args.warmup):
        flush()
        step.copy_and_write(t)
        step.decode(t)
    torch.cuda.synchronize()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    with ClockSampler(device) as clk:
        for i, (a, b, c) in enumerate(ev):
            t = args.warmup + i
            flush()
            a.record(stream)
            step.copy_and_write(t)
            b.record(stream)
            step.decode(t)
            c.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    total_ms = reduce_max(sum(a.elapsed_time(c) for a, _, c in ev), world, device)
    timed = step.steps[args.warmup:]
    kv = sum(st["kv_bytes"] for st in timed)
    ukv = sum(st["unique_kv_bytes"] for st in timed)
    value = kv * world / (total_ms / 1e3) / 1e9
    dec_ms = statistics.mean(b.elapsed_time(c) for _, b, c in ev)
    cw_ms = statistics.mean(a.elapsed_time(b) for a, b, _ in ev)
    e2e = None
    if not args.no_e2e:
        n_e = max(3, args.steps // 4)
        idx = [args.warmup + i % args.steps for i in range(n_e)]
        e_ms, h2d, d2h = time_beam_e2e(step, idx, world)
        e_kv = sum(step.steps[t]["kv_bytes"] for t in idx)
        e2e = {"value": round(e_kv * world / (e_ms / 1e3) / 1e9, 2), "unit": "GB/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": round(e_ms / n_e, 4)}
    peak, peak_kind = measured_peak_hbm()
    achieved = ukv / args.steps / (dec_ms / 1e3) / 1e9
    if rank == 0:
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            cpu = cpu_baseline(w0, target_s=args.cpu_seconds)
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(total_ms / args.steps, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded N(0,1) K/V/q, seeded beam choices and block placement)",
            "config": {"workload": "beam: " + DESCR["beam"], "global_batch": step.S * world,
                       "seq_len": step.max_len, "parallelism": "replicas: requests sharded by rank, no collective",
                       "l2": "flushed before every timed step (256 MB write, outside the timed region); value "
                             "counts logical KV bytes (the prompt once per beam)"},
            "us_decode": round(1e3 * dec_ms, 2), "us_copy_and_write": round(1e3 * cw_ms, 2),
            "us_decode_spread": spread_us([b.elapsed_time(c) for _, b, c in ev]),
            "logical_kv_bytes_per_step": kv // args.steps, "unique_kv_bytes_per_step": ukv // args.steps,
            "decode_call_logical_gbs": round(kv / args.steps / (dec_ms / 1e3) / 1e9, 1),
            "copy_pairs_per_step": round(sum(st["npairs"] for st in timed) / args.steps, 2),
            "host_block_manager_us_per_step": round(step.host_us_per_step, 1),
            "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                         "frac": round(achieved / peak, 4), "traffic": ncu_traffic("beam"),
                         "kernel": "paged_attention_decode_shared call (plan + grouped decode + merge); achieved "
                                   "counts unique KV bytes (a shared block once)", "peak_source": peak_kind},
            "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": sum(4 + (st["npairs"] > 0) for st in timed),
            "device_errors": int(step.err.item()), "clocks": clk.summary(),
        }
        return line
    return None


def run_swap(args, device):
    """Swap-out and swap-in throughput of pkv_swap_blocks over the host link."""
    import paged_kv_cache_404_b200 as pkv
    w = W.WORKLOADS["gqa70b"]
    nseq = args.num_seqs or 64
    per_seq = -(-w.len_lo // 16)
    blocks = nseq * per_seq
    NB = int(blocks * 2)
    bm = pkv.BlockManager(NB, 16, free_order=W.free_order(w, NB))
    others = bm.alloc_seq((NB - blocks) * 16 // 2)          # scatter: half the pool held elsewhere
    ids = [bm.alloc_seq(w.len_lo) for _ in range(nseq)]
    bm.set_host_pool(blocks)
    out_pairs = np.concatenate([bm.swap_out(s) for s in ids])
    in_pairs = np.concatenate([bm.swap_in(s) for s in ids])
    del others
    shape = (16, w.num_kv_heads, w.head_dim)
    dk = torch.randn((NB,) + shape, device=device).to(torch.bfloat16)
    dv = torch.randn((NB,) + shape, device=device).to(torch.bfloat16)
    hk = torch.empty((blocks,) + shape, dtype=torch.bfloat16).pin_memory()
    hv = torch.empty((blocks,) + shape, dtype=torch.bfloat16).pin_memory()
    g_out = torch.from_numpy(out_pairs).to(device)
    g_in = torch.from_numpy(in_pairs).to(device)
    nbytes = 2 * blocks * dk[0].numel() * 2
    err = torch.zeros(1, dtype=torch.int32, device=device)
    stream = torch.cuda.current_stream()

    def timed(fn, reps):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        ms = []
        for _ in range(reps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            torch.cuda.synchronize()
            ms.append(a.elapsed_time(b))
        return statistics.median(ms)

    reps = max(3, min(args.steps, 20))
    with ClockSampler(device) as clk:
        out_ms = timed(lambda: pkv.swap_blocks(hk, hv, dk, dv, g_out, err_count=err), reps)
        in_ms = timed(lambda: pkv.swap_blocks(dk, dv, hk, hv, g_in, err_count=err), reps)
        # copy-engine reference: the same bytes as two contiguous transfers per direction
        ck, cv = dk[:blocks], dv[:blocks]
        d2h_ms = timed(lambda: (hk.copy_(ck, non_blocking=True), hv.copy_(cv, non_blocking=True)), reps)
        h2d_ms = timed(lambda: (ck.copy_(hk, non_blocking=True), cv.copy_(hv, non_blocking=True)), reps)
    torch.cuda.synchronize()
    # bytes check: after a swap-out and a swap-in, sampled blocks hold what the host pool holds
    pkv.swap_blocks(hk, hv, dk, dv, g_out, err_count=err)
    pkv.swap_blocks(dk, dv, hk, hv, g_in, err_count=err)
    torch.cuda.synchronize()
    probe = in_pairs[:: max(1, blocks // 64)]
    ok = bool(torch.equal(dk[torch.from_numpy(probe[:, 1]).to(device)].cpu(), hk[torch.from_numpy(probe[:, 0])]))
    ok = ok and int(err.item()) == 0
    gbs = lambda ms: round(nbytes / (ms / 1e3) / 1e9, 2)  # noqa: E731
    # the oracle's block copy between host pools, on this host, for a bounded sample of the pairs
    cpu = None
    if not args.no_cpu_baseline:
        import oracle
        nsamp = min(len(out_pairs), 4096)
        hk_np = hk.view(torch.int16).numpy()
        hv_np = hv.view(torch.int16).numpy()
        dk_h = dk[:nsamp * 2].cpu().view(torch.int16).numpy()
        dv_h = dv[:nsamp * 2].cpu().view(torch.int16).numpy()
        samp = np.stack([np.arange(nsamp) * 2, np.arange(nsamp)], axis=1).astype(np.int64)
        t0 = time.perf_counter()
        oracle.swap_blocks(hk_np, hv_np, dk_h, dv_h, samp)
        dt = time.perf_counter() - t0
        cpu = {"value": round(2 * nsamp * dk[0].numel() * 2 / dt / 1e9, 3), "unit": "GB/s", "cores": 1,
               "kind": "oracle", "sample": "%d block pairs (K and V, %d KiB each) host pool to host pool, %.3f s" % (
                   nsamp, dk[0].numel() * 2 // 1024, dt)}
    line = {
        "metric": "block swap over the host link: GB/s (K+V bytes moved / time)",
        "value": round(2 * nbytes / ((out_ms + in_ms) / 1e3) / 1e9, 2),
        "unit": "GB/s", "n_gpus": 1, "steps": reps, "warmup": 3, "ms_per_step": round(out_ms + in_ms, 4),
        "higher_is_better": True, "dtype": "bf16 (byte copy)", "data": "synthetic",
        "config": {"workload": "swap: %d sequences x %d tokens of gqa70b (8 kv heads, head_dim 128, bf16), "
                               "%d scattered device blocks <-> page-locked host pool" % (nseq, w.len_lo, blocks),
                   "bytes_per_direction": nbytes},
        "swap_out": {"ms": round(out_ms, 4), "GB/s": gbs(out_ms), "copy_engine_GB/s": gbs(d2h_ms),
                     "frac": round(d2h_ms / out_ms, 4)},
        "swap_in": {"ms": round(in_ms, 4), "GB/s": gbs(in_ms), "copy_engine_GB/s": gbs(h2d_ms),
                    "frac": round(h2d_ms / in_ms, 4)},
        "roofline": {"bound": "host link", "achieved": round(2 * nbytes / ((out_ms + in_ms) / 1e3) / 1e9, 2),
                     "peak": round(2 * nbytes / ((d2h_ms + h2d_ms) / 1e3) / 1e9, 2), "unit": "GB/s",
                     "frac": round((d2h_ms + h2d_ms) / (out_ms + in_ms), 4),
                     "peak_source": "contiguous cudaMemcpyAsync of the same bytes, measured in this run"},
        "gpu_launches": 2 * reps, "bytes_restored": ok, "cpu_baseline": cpu, "clocks": clk.summary(),
    }
    print(json.dumps(line), flush=True)


def run_decode(args, w0, device, rank, world):
    """The decode step (write + copy-on-write copies + decode) of a flat or
    shared-prefix workload: K timed steps, e2e, roofline, CPU baseline."""
    w = rank_workload(w0, rank)
    step = Step(w, device, partition=args.partition, prefix_groups=not args.no_prefix_groups)
    torch.cuda.synchronize()

    with ClockSampler(device) as clk:
        total_ms, decode_ms, write_ms = time_steps(step, args.steps, args.warmup, world, device)
    err = int(step.err.item())
    max_ms = reduce_max(total_ms, world, device)
    ms_per_step = max_ms / args.steps
    bytes_all = step.kv_bytes * world
    value = bytes_all * args.steps / (max_ms / 1e3) / 1e9

    e2e = None
    if not args.no_e2e:
        e_steps = max(5, args.steps // 2)
        e_ms, h2d, d2h = time_e2e(step, e_steps, 3, world)
        e_ms = reduce_max(e_ms, world, device)
        e2e = {"value": round(bytes_all * e_steps / (e_ms / 1e3) / 1e9, 2), "unit": "GB/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "ms_per_step": round(e_ms / e_steps, 4)}

    peak, peak_kind = measured_peak_hbm()
    dec_ms = statistics.mean(decode_ms)
    elem = 1 if w.cache_dtype == "fp8" else 2
    ukv = unique_kv_bytes(step.tables, step.lens, w.num_kv_heads * w.head_dim * 2 * elem)
    shared = step.groups is not None
    # a shared-prefix decode reads a shared block once: its roofline counts unique bytes
    achieved = (ukv if shared else step.kv_bytes) / (dec_ms / 1e3) / 1e9
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                "frac": round(achieved / peak, 4), "traffic": ncu_traffic(w0.name),
                "kernel": ("paged_attention_decode_shared call (plan + grouped decode + merge); achieved counts "
                           "unique KV bytes (a shared block once)") if shared else
                          "paged_attention_decode call (plan + decode + merge launches)",
                "peak_source": peak_kind, "frac_of_nominal_8tbps": round(achieved / NOMINAL_HBM_GBS, 4)}
    if rank != 0:
        return None
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w0, target_s=args.cpu_seconds)
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": "fp8-e4m3 cache, bf16 q/out, fp32 accumulate" if w.cache_dtype == "fp8" else w.cache_dtype,
        "data": "synthetic (seeded N(0,1) K/V/q, seeded block placement)",
        "config": {"workload": w0.name + ": " + DESCR[w0.name], "global_batch": step.S * world,
                   "seq_len": step.max_len, "parallelism": "replicas: sequences sharded by rank, no collective",
                   "l2": "inputs larger than L2 (pools %.1f GiB per GPU vs 126 MB L2)" % (
                       2 * step.k_pool.numel() * step.k_pool.element_size() / 2**30),
                   "partition_tokens": args.partition or "auto",
                   "prefix_groups": shared},
        "seq_tokens_per_s": round(step.seq_tokens * world * args.steps / (max_ms / 1e3), 1),
        "us_per_step_per_layer": round(1e3 * ms_per_step, 2),
        "us_decode": round(1e3 * dec_ms, 2), "us_write": round(1e3 * statistics.mean(write_ms), 2),
        "us_decode_spread": spread_us(decode_ms),
        "pct_of_8tbps": round(100 * value / world / NOMINAL_HBM_GBS, 2),
        "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
        "gpu_launches": step.launches * args.steps, "device_errors": err,
        "clocks": clk.summary(),
    }
    if w.lens == "shared":
        line["logical_kv_bytes_per_step"] = step.kv_bytes
        line["unique_kv_bytes_per_step"] = ukv
        line["decode_call_logical_gbs"] = round(step.kv_bytes / (dec_ms / 1e3) / 1e9, 1)
        line["memory_saving_by_sharing"] = round(step.mem_saving, 4)
        line["divergence_step"] = divergence_step(w, device, args)
    return line


# The default run's other configurations (every workload the benchmark's
# configuration list names besides the headline), each reported with the
# fields of its own line; the tiny workload is a correctness case, not timed.
CONFIG_KEYS = ("value", "unit", "ms_per_step", "steps", "warmup", "dtype", "seq_tokens_per_s",
               "prompt_tokens_per_s", "us_decode", "us_write", "us_copy_and_write", "us_attention",
               "us_decode_spread", "us_attention_spread", "logical_kv_bytes_per_step", "unique_kv_bytes_per_step",
               "decode_call_logical_gbs", "memory_saving_by_sharing", "divergence_step", "copy_pairs_per_step",
               "roofline", "cpu_baseline", "gpu_launches", "device_errors", "clocks")


def run_configs(args, device, rank, world):
    import copy
    sub = copy.copy(args)
    sub.steps = max(5, min(args.steps, 30))
    sub.warmup = max(3, min(args.warmup, 5))
    sub.no_e2e = True
    sub.partition = 0
    sub.no_prefix_groups = False
    sub.cpu_seconds = min(args.cpu_seconds, 4.0)
    out = {}
    for name in ("mha13b", "shared_prefix", "fp8_long", "beam", "prefill70b"):
        w0 = W.WORKLOADS[name]
        if name == "beam":
            line = run_beam(sub, w0, device, rank, world)
        elif name.startswith("prefill"):
            line = run_prefill(sub, w0, device, rank, world)
        else:
            line = run_decode(sub, w0, device, rank, world)
        torch.cuda.empty_cache()
        if line is not None:
            entry = {"workload": line["config"]["workload"], "metric": line["metric"]}
            entry.update({k: line[k] for k in CONFIG_KEYS if k in line})
            out[name] = entry
    return out


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="gqa70b", choices=sorted(DESCR))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--partition", type=int, default=0, help="partition tokens (0 = automatic)")
    ap.add_argument("--num-seqs", type=int, default=0,
                    help="fewer sequences of the same shape (small cases for profiling; not a bench line)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="oracle work per CPU baseline (about)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="default run: skip the other configurations (the 'configs' object)")
    ap.add_argument("--swap", action="store_true", help="measure block swap to a host pool instead")
    ap.add_argument("--no-prefix-groups", action="store_true",
                    help="shared_prefix: plain decode (each sample reads the prompt's blocks itself)")
    args = ap.parse_args(argv)
    args.warmup = max(args.warmup, 3)

    rank, world, local = dist_env()
    w0 = W.WORKLOADS[args.workload]
    if args.num_seqs:
        w0 = W.scaled(w0, num_seqs=args.num_seqs, num_prompts=max(1, args.num_seqs // max(w0.samples, 1)))
    if args.impl == "reference":
        run_reference(args, w0, rank, world)
        return

    from paged_kv_cache_404_b200 import build as pkv_build
    if rank == 0:
        pkv_build.build()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if args.swap:
        run_swap(args, device)
        return
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)
        dist.barrier()
        pkv_build.build()

    if args.workload.startswith("prefill"):
        line = run_prefill(args, w0, device, rank, world)
    elif args.workload == "beam":
        line = run_beam(args, w0, device, rank, world)
    else:
        line = run_decode(args, w0, device, rank, world)
    if args.workload == "gqa70b" and not args.num_seqs and not args.no_configs:
        configs = run_configs(args, device, rank, world)
        if line is not None:
            line["configs"] = configs
    if rank == 0 and line is not None:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
