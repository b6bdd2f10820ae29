"""Seeded synthetic inputs for the paged KV-cache hot path.

This module is the one piece shared by the product tests/bench and the oracle
side.  It draws random numbers and fixes shapes; it contains none of the
method's arithmetic (no slot addressing, no attention, no quantisation rule of
the cache).  Both sides receive the same bytes from it.

Workloads are shaped like the PagedAttention pages' examples:
- "tiny": 4 sequences of lengths {1, 15, 16, 40} in a 64-block pool, fp32,
  head_dim 64; the 40-token request takes its blocks first from the free list
  [41, 7, 19, 2, 33] as in the glossary entry's worked example.
- "mha13b": LLaMA-13B-shaped multi-head attention (40 heads, head_dim 128).
- "gqa70b": Llama-3.1-70B-shaped grouped-query attention (64 query / 8 KV heads)
  at 4,096 tokens x 256 concurrent sequences.
- "shared_prefix": parallel sampling n=3 over 64 prompts sharing a 1,000-token
  prefix, continuations of 0..512 tokens.
- "fp8_long": FP8 E4M3 cache, log-uniform context lengths 256..32,768.
- "prefill70b": the prompt pass of the Llama-3.1-70B shape: 16 prompts of
  512..4,096 tokens written into blocks and attended causally.
- "prefill70b_fp8": the same prompt pass over an FP8 E4M3 cache (per-tensor
  scales amax/448 of the prompt's K and V).
- "beam": beam search, 16 requests x 4 beams over a 1,000-token prompt; at
  every step each request keeps 4 beams drawn (seeded) from its current ones:
  forks, frees and copy-on-write at every step.
"""
from dataclasses import dataclass, replace
import math

import numpy as np
import torch

BLOCK_SIZE = 16


@dataclass(frozen=True)
class Workload:
    name: str
    num_heads: int
    num_kv_heads: int
    head_dim: int
    cache_dtype: str          # "f32" | "bf16" | "fp8"
    q_dtype: str              # "f32" | "bf16"
    num_seqs: int
    lens: str                 # "tiny" | "uniform" | "const" | "shared" | "loguniform"
    len_lo: int
    len_hi: int
    seed: int
    block_size: int = BLOCK_SIZE
    pool_factor: float = 1.25
    # shared prefix (parallel sampling)
    num_prompts: int = 0
    samples: int = 0
    prefix_len: int = 0

    @property
    def group(self):
        return self.num_heads // self.num_kv_heads

    @property
    def scale(self):
        return 1.0 / math.sqrt(self.head_dim)


WORKLOADS = {
    "tiny": Workload("tiny", 2, 2, 64, "f32", "f32", 4, "tiny", 1, 40, seed=1),
    "mha13b": Workload("mha13b", 40, 40, 128, "bf16", "bf16", 64, "uniform", 128, 2048, seed=2),
    "gqa70b": Workload("gqa70b", 64, 8, 128, "bf16", "bf16", 256, "const", 4096, 4096, seed=3),
    "shared_prefix": Workload("shared_prefix", 32, 8, 128, "bf16", "bf16", 192, "shared", 0, 512, seed=4,
                              num_prompts=64, samples=3, prefix_len=1000),
    "fp8_long": Workload("fp8_long", 32, 8, 128, "fp8", "bf16", 128, "loguniform", 256, 32768, seed=5),
    "prefill70b": Workload("prefill70b", 64, 8, 128, "bf16", "bf16", 16, "uniform", 512, 4096, seed=6),
    "prefill70b_fp8": Workload("prefill70b_fp8", 64, 8, 128, "fp8", "bf16", 16, "uniform", 512, 4096, seed=6),
    "beam": Workload("beam", 32, 8, 128, "bf16", "bf16", 64, "beam", 0, 48, seed=7,
                     num_prompts=16, samples=4, prefix_len=1000),
}

TINY_LENS = (1, 15, 16, 40)
TINY_POOL_BLOCKS = 64
TINY_FREE_HEAD = (41, 7, 19, 2, 33)


def scaled(w: Workload, **kw) -> Workload:
    """A smaller (or otherwise changed) copy of a workload, same generator rules."""
    return replace(w, **kw)


def _np_rng(w: Workload, stream: int) -> np.random.Generator:
    return np.random.default_rng([w.seed, stream])


def context_lens(w: Workload) -> np.ndarray:
    """Context length of every sequence (int32), including the token of this step."""
    rng = _np_rng(w, 1)
    if w.lens == "tiny":
        return np.array(TINY_LENS, dtype=np.int32)
    if w.lens == "uniform":
        return rng.integers(w.len_lo, w.len_hi + 1, size=w.num_seqs).astype(np.int32)
    if w.lens == "const":
        return np.full(w.num_seqs, w.len_lo, dtype=np.int32)
    if w.lens == "beam":
        # every beam has the same length; this is the one half-way through the trace
        return np.full(w.num_seqs, w.prefix_len + w.len_hi // 2 + 1, dtype=np.int32)
    if w.lens == "loguniform":
        u = rng.uniform(math.log(w.len_lo), math.log(w.len_hi), size=w.num_seqs)
        return np.minimum(np.floor(np.exp(u)), w.len_hi).astype(np.int32)
    raise ValueError("workload %s has no flat length list" % w.name)


def continuation_lens(w: Workload) -> np.ndarray:
    """Shared-prefix workload: private continuation length of each sample, U{0..len_hi}."""
    rng = _np_rng(w, 2)
    return rng.integers(0, w.len_hi + 1, size=w.num_prompts * w.samples).astype(np.int32)


def beam_parents(w: Workload, step: int) -> np.ndarray:
    """Beam workload: for every request, which of its current beams each of the
    next step's beams continues (int32 [num_prompts, samples], seeded draws with
    replacement; a beam drawn by none is dropped)."""
    rng = np.random.default_rng([w.seed, 9, step])
    return rng.integers(0, w.samples, size=(w.num_prompts, w.samples)).astype(np.int32)


def allocation_order(w: Workload):
    """Order in which sequences take their blocks from the free list."""
    if w.lens == "tiny":
        # the 40-token request first (it receives [41, 7, 19] as in the worked example)
        return [3, 0, 1, 2]
    return list(range(w.num_seqs))


def pool_blocks(w: Workload, blocks_needed: int) -> int:
    """Pool size: 1.25x the blocks the workload needs (64 for the tiny one)."""
    if w.lens == "tiny":
        return TINY_POOL_BLOCKS
    return int(math.ceil(blocks_needed * w.pool_factor))


def free_order(w: Workload, num_blocks: int) -> np.ndarray:
    """Seeded order of the free list: a permutation of all physical block ids.

    For the tiny workload the list starts with the worked example's
    [41, 7, 19, 2, 33], followed by a seeded shuffle of the other ids.
    """
    rng = _np_rng(w, 3)
    if w.lens == "tiny":
        head = list(TINY_FREE_HEAD)
        rest = np.array([b for b in range(num_blocks) if b not in head], dtype=np.int64)
        rng.shuffle(rest)
        return np.array(head + rest.tolist(), dtype=np.int32)
    return rng.permutation(num_blocks).astype(np.int32)


# ---------------------------------------------------------------- tensors

_TORCH_DT = {"f32": torch.float32, "bf16": torch.bfloat16}


def torch_generator(w: Workload, stream: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(w.seed * 1000003 + stream)
    return g


def randn(shape, dtype: str, gen: torch.Generator, device, chunk: int = 1 << 26) -> torch.Tensor:
    """N(0,1) drawn in fp32 and rounded to `dtype` (bf16: round to nearest even).

    Large tensors are drawn in chunks of `chunk` elements from one generator.
    """
    out = torch.empty(shape, dtype=_TORCH_DT[dtype], device=device)
    flat = out.view(-1)
    n = flat.numel()
    for i in range(0, n, chunk):
        m = min(chunk, n - i)
        flat[i:i + m] = torch.randn(m, generator=gen, device=device, dtype=torch.float32).to(flat.dtype)
    return out


def pool_shape(w: Workload, num_blocks: int):
    return (num_blocks, w.block_size, w.num_kv_heads, w.head_dim)


def random_pools(w: Workload, num_blocks: int, device):
    """Filled K and V pools [NB, bs, Hkv, D]: every byte is seeded N(0,1) data.

    Bytes that no sequence owns stay as seeded, NaN-free values so that a stale
    read shows up as a wrong result.  For the fp8 workload the values are drawn
    in bf16 and stored as E4M3 with per-tensor scales amax(|x|)/448 (computed in
    fp32); returns (k_pool, v_pool, k_scale, v_scale), pools as uint8 codes.
    """
    shape = pool_shape(w, num_blocks)
    if w.cache_dtype in ("f32", "bf16"):
        k = randn(shape, w.cache_dtype, torch_generator(w, 10, device), device)
        v = randn(shape, w.cache_dtype, torch_generator(w, 11, device), device)
        return k, v, 1.0, 1.0
    pools = []
    scales = []
    for stream in (10, 11):
        x = randn(shape, "bf16", torch_generator(w, stream, device), device)
        amax = x.abs().max().float().item()
        s = float(np.float32(amax) / np.float32(448.0))
        pools.append(_to_e4m3_codes(x, s))
        scales.append(s)
        del x
    return pools[0], pools[1], scales[0], scales[1]


def _to_e4m3_codes(x: torch.Tensor, scale: float, chunk: int = 1 << 26) -> torch.Tensor:
    """Input preparation only: store a pre-existing cache as E4M3 codes (torch's cast)."""
    out = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    xf, of = x.view(-1), out.view(-1)
    for i in range(0, xf.numel(), chunk):
        y = (xf[i:i + chunk].float() / scale).clamp_(-448.0, 448.0)
        of[i:i + chunk] = y.to(torch.float8_e4m3fn).view(torch.uint8)
    return out


def queries(w: Workload, num_seqs: int, device) -> torch.Tensor:
    """Decode queries q [S, Hq, D]."""
    return randn((num_seqs, w.num_heads, w.head_dim), w.q_dtype, torch_generator(w, 20, device), device)


def new_tokens(w: Workload, num_tokens: int, device, stream: int = 30):
    """K and V of the tokens written this step, [T, Hkv, D] in the source dtype."""
    src = "f32" if w.cache_dtype == "f32" else "bf16"
    k = randn((num_tokens, w.num_kv_heads, w.head_dim), src, torch_generator(w, stream, device), device)
    v = randn((num_tokens, w.num_kv_heads, w.head_dim), src, torch_generator(w, stream + 1, device), device)
    return k, v


def logical_kv(w: Workload, num_tokens: int, device, stream: int):
    """K and V of `num_tokens` logical tokens (prompts, continuations), [T, Hkv, D]."""
    return new_tokens(w, num_tokens, device, stream=stream)


def stale_fill(w: Workload, num_blocks: int, device):
    """Seeded NaN-free initial pool contents for workloads filled by writes."""
    shape = pool_shape(w, num_blocks)
    dt = "f32" if w.cache_dtype == "f32" else "bf16"
    k = randn(shape, dt, torch_generator(w, 40, device), device)
    v = randn(shape, dt, torch_generator(w, 41, device), device)
    if w.cache_dtype == "fp8":
        return _to_e4m3_codes(k, 1.0), _to_e4m3_codes(v, 1.0)
    return k, v
