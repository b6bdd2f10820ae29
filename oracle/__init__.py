"""CPU oracle for the paged KV-cache hot path.

TEST INFRASTRUCTURE ONLY.  Only tests/, ``__graft_entry__.smoke()`` and
``bench.py``'s cpu_baseline / reference leg may import this package.  It shares
no code with the product library (``paged_kv_cache_404_b200``) and neither
imports the other.

The arithmetic lives in ``oracle.c`` (double precision, plain loops, OpenMP over
(sequence, query head)); ``allocator.py`` is the reference block manager.  Both
follow the PagedAttention pages (ultralytics.com glossary entry "PagedAttention",
sections "Como funciona la paginacion" and "Compartir bloques entre secuencias";
iplexlaw.co.kr blog, sections on logical vs physical order and the two-answer
example; gyaansetu.com "Le cache KV et PagedAttention").

Arrays are numpy, C-contiguous.  Element types: fp32 as float32, bf16 as the raw
uint16 bit pattern, FP8 E4M3 as the raw uint8 code.

Parity status: every function here is pinned by tests under tests/ that do not
re-type its formula (worked example, closed forms, brute force through a
different route, invariants, format tables); none is "parity unpinned".
"""
import ctypes as C
import os

import numpy as np

from . import build as _build
from .allocator import RefBlockManager  # noqa: F401

F32, BF16, FP8_E4M3 = 0, 1, 2
_NP_OF = {F32: np.float32, BF16: np.uint16, FP8_E4M3: np.uint8}

_lib = None


def lib():
    """Load liboracle.so, building it first when missing or stale."""
    global _lib
    if _lib is None:
        path = _build.build()
        L = C.CDLL(path)
        p = C.c_void_p
        L.orc_e4m3_decode.restype = C.c_double
        L.orc_e4m3_decode.argtypes = [C.c_uint8]
        L.orc_e4m3_encode.restype = C.c_uint8
        L.orc_e4m3_encode.argtypes = [C.c_float]
        L.orc_kv_write.restype = C.c_int
        L.orc_kv_write.argtypes = [p, p, C.c_int, p, C.c_int, p, p, C.c_int, C.c_int, C.c_int,
                                   C.c_int, C.c_int, C.c_float, C.c_float]
        L.orc_copy_blocks.restype = C.c_int
        L.orc_copy_blocks.argtypes = [p, p, C.c_size_t, p, C.c_int, C.c_int]
        L.orc_swap_blocks.restype = C.c_int
        L.orc_swap_blocks.argtypes = [p, p, C.c_int, p, p, C.c_int, C.c_size_t, p, C.c_int]
        L.orc_gather.restype = C.c_int
        L.orc_gather.argtypes = [p, C.c_size_t, p, C.c_int, C.c_int, C.c_int, p]
        L.orc_paged_attention_decode.restype = C.c_int
        L.orc_paged_attention_decode.argtypes = [p, p, C.c_int, p, p, C.c_int, p, C.c_int, p, C.c_int,
                                                 C.c_int, C.c_int, C.c_int, C.c_int, C.c_int,
                                                 C.c_double, C.c_double, C.c_double, C.c_int, C.c_int]
        L.orc_paged_attention_prefill.restype = C.c_int
        L.orc_paged_attention_prefill.argtypes = [p, p, C.c_int, p, p, C.c_int, p, C.c_int, p, p, C.c_int,
                                                  C.c_int, C.c_int, C.c_int, C.c_int, C.c_int, C.c_double,
                                                  C.c_double, C.c_double, p, C.c_int]
        L.orc_kv_cache_bytes.restype = C.c_double
        L.orc_kv_cache_bytes.argtypes = [C.c_int, C.c_int, C.c_int, C.c_int, C.c_double]
        L.orc_max_threads.restype = C.c_int
        L.orc_max_threads.argtypes = []
        _lib = L
    return _lib


def _ptr(a):
    return C.c_void_p(a.ctypes.data)


def _c(a, dtype=None):
    return np.ascontiguousarray(np.asarray(a) if dtype is None else np.asarray(a, dtype=dtype))


def e4m3_decode(code: int) -> float:
    """Value of one OFP8 E4M3 code (NaN for S.1111.111)."""
    return lib().orc_e4m3_decode(int(code) & 0xFF)


def e4m3_encode(x: float) -> int:
    """E4M3 code of a binary32 value: round to nearest even, saturate to +-448."""
    return int(lib().orc_e4m3_encode(float(np.float32(x))))


def e4m3_encode_array(x: np.ndarray) -> np.ndarray:
    """Element-wise :func:`e4m3_encode` of a float32 array."""
    x = np.asarray(x, dtype=np.float32).ravel()
    enc = lib().orc_e4m3_encode
    return np.array([enc(float(v)) for v in x], dtype=np.uint8)


def kv_write(k, v, src_dtype, slot_mapping, k_pool, v_pool, cache_dtype, block_size,
             k_scale=1.0, v_scale=1.0):
    """Byte-exact emulation of the KV append, in place on host pools.

    k, v: [T, Hkv, D] source arrays; slot_mapping: int64 [T]; pools:
    [NB, block_size, Hkv, D].  Returns the number of out-of-range slots skipped.
    """
    k = _c(k)
    v = _c(v)
    sm = _c(slot_mapping, np.int64)
    assert k_pool.flags.c_contiguous and v_pool.flags.c_contiguous
    T = sm.shape[0]
    NB, bs, Hkv, D = k_pool.shape
    assert bs == block_size
    r = lib().orc_kv_write(_ptr(k), _ptr(v), src_dtype, _ptr(sm), T, _ptr(k_pool), _ptr(v_pool),
                           cache_dtype, NB, bs, Hkv, D, float(k_scale), float(v_scale))
    if r < 0:
        raise ValueError("unsupported dtype combination")
    return r


def copy_blocks(k_pool, v_pool, pairs):
    """Copy whole physical blocks src -> dst in both pools, in place.

    pairs: int64 [n, 2].  Returns the number of out-of-range pairs skipped;
    raises on overlapping pair lists (repeated dst, or a dst that is a src).
    """
    pairs = _c(np.asarray(pairs, dtype=np.int64).reshape(-1, 2))
    NB = k_pool.shape[0]
    block_bytes = k_pool.nbytes // NB
    r = lib().orc_copy_blocks(_ptr(k_pool), _ptr(v_pool), block_bytes, _ptr(pairs), pairs.shape[0], NB)
    if r < 0:
        raise ValueError("overlapping copy pairs have no defined result")
    return r


def swap_blocks(dst_k, dst_v, src_k, src_v, pairs):
    """Copy whole blocks src (of the source pools) -> dst (of the destination pools).

    pairs: int64 [n, 2].  Returns the number of out-of-range pairs skipped;
    raises on a repeated dst.
    """
    pairs = _c(np.asarray(pairs, dtype=np.int64).reshape(-1, 2))
    assert dst_k.shape[1:] == src_k.shape[1:] and dst_k.dtype == src_k.dtype
    block_bytes = src_k.nbytes // src_k.shape[0]
    r = lib().orc_swap_blocks(_ptr(dst_k), _ptr(dst_v), dst_k.shape[0], _ptr(src_k), _ptr(src_v),
                              src_k.shape[0], block_bytes, _ptr(pairs), pairs.shape[0])
    if r < 0:
        raise ValueError("a repeated destination block has no defined result")
    return r


def gather(pool, table, length, block_size):
    """A request's first `length` token rows, read back through its block table.

    pool: [NB, block_size, ...]; returns an array [length, ...] of pool's dtype.
    """
    NB = pool.shape[0]
    row_shape = pool.shape[2:]
    row_bytes = pool.nbytes // (NB * block_size)
    tab = _c(np.asarray(table, dtype=np.int32))
    out = np.zeros((length,) + row_shape, dtype=pool.dtype)
    lib().orc_gather(_ptr(pool), row_bytes, _ptr(tab), int(length), block_size, NB, _ptr(out))
    return out


def paged_attention_decode(q, q_dtype, k_pool, v_pool, cache_dtype, block_tables, context_lens,
                           scale, k_scale=1.0, v_scale=1.0, partition_tokens=0, num_threads=0):
    """fp64 decode attention through block tables.

    q: [S, Hq, D]; pools [NB, bs, Hkv, D]; block_tables int32 [S, max_blocks];
    context_lens int32 [S].  Returns (out float64 [S, Hq, D], bad_entries).
    """
    q = _c(q)
    kp = _c(k_pool)
    vp = _c(v_pool)
    bt = _c(block_tables, np.int32)
    cl = _c(context_lens, np.int32)
    S, Hq, D = q.shape
    NB, bs, Hkv, D2 = kp.shape
    assert D2 == D and bt.shape[0] == S and cl.shape[0] == S
    out = np.zeros((S, Hq, D), dtype=np.float64)
    r = lib().orc_paged_attention_decode(_ptr(out), _ptr(q), q_dtype, _ptr(kp), _ptr(vp), cache_dtype,
                                         _ptr(bt), bt.shape[1], _ptr(cl), S, NB, bs, Hq, Hkv, D,
                                         float(scale), float(k_scale), float(v_scale),
                                         int(partition_tokens), int(num_threads))
    if r < 0:
        raise ValueError("bad arguments to the oracle decode")
    return out, r


def paged_attention_prefill(q, q_dtype, k_pool, v_pool, cache_dtype, block_tables, context_lens, query_start,
                            scale, k_scale=1.0, v_scale=1.0, rows=None, num_threads=0):
    """fp64 causal multi-token attention through block tables.

    q: [total_q, Hq, D]; query_start int32 [S + 1]; sequence s's queries are the
    last (query_start[s+1] - query_start[s]) of its context_lens[s] tokens.
    rows: optional iterable of query rows to compute (others stay 0).
    Returns (out float64 [total_q, Hq, D], bad_entries).
    """
    q = _c(q)
    kp = _c(k_pool)
    vp = _c(v_pool)
    bt = _c(block_tables, np.int32)
    cl = _c(context_lens, np.int32)
    qs = _c(query_start, np.int32)
    T, Hq, D = q.shape
    NB, bs, Hkv, D2 = kp.shape
    S = cl.shape[0]
    assert D2 == D and bt.shape[0] == S and qs.shape[0] == S + 1 and qs[-1] == T
    mask = None
    if rows is not None:
        mask = np.zeros(T, dtype=np.uint8)
        mask[np.asarray(list(rows), dtype=np.int64)] = 1
    out = np.zeros((T, Hq, D), dtype=np.float64)
    r = lib().orc_paged_attention_prefill(_ptr(out), _ptr(q), q_dtype, _ptr(kp), _ptr(vp), cache_dtype, _ptr(bt),
                                          bt.shape[1], _ptr(cl), _ptr(qs), S, NB, bs, Hq, Hkv, D, float(scale),
                                          float(k_scale), float(v_scale), _ptr(mask) if mask is not None else None,
                                          int(num_threads))
    if r < 0:
        raise ValueError("bad arguments to the oracle prefill")
    return out, r


def kv_cache_bytes(layers, num_kv_heads, head_dim, elem_bytes, tokens):
    """Bytes of a KV cache holding `tokens` tokens (K and V, all layers)."""
    return lib().orc_kv_cache_bytes(layers, num_kv_heads, head_dim, elem_bytes, float(tokens))


def max_threads():
    return lib().orc_max_threads()


def slot_of(table, pos, block_size):
    """Slot address of logical position `pos`: (table[pos // bs], pos % bs) as one int."""
    return int(table[pos // block_size]) * block_size + pos % block_size


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact value of bf16 bit patterns as float64."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
