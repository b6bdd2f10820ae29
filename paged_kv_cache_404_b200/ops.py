"""Python binding of the three hot-path calls (argument marshalling only).

Every step runs in the CUDA kernels of libpagedkv.so; this module turns torch
tensors into pointers, sizes and the current CUDA stream and raises on a
non-zero status.  Tensors must be CUDA, contiguous and 16-byte aligned.

dtypes: fp32 -> PKV_F32, bfloat16 -> PKV_BF16, uint8 or float8_e4m3fn (raw
E4M3 codes) -> PKV_FP8_E4M3.
"""
import ctypes as C

import torch

from . import _lib as L

BLOCK_SIZE = 16


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return L.PKV_F32
    if t.dtype == torch.bfloat16:
        return L.PKV_BF16
    if t.dtype in (torch.uint8, torch.float8_e4m3fn):
        return L.PKV_FP8_E4M3
    raise TypeError("unsupported dtype %s" % t.dtype)


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return C.c_void_p(t.data_ptr())


def _stream(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return C.c_void_p(s.cuda_stream)


def paged_kv_write(k, v, slot_mapping, k_pool, v_pool, k_scale=1.0, v_scale=1.0, err_count=None, stream=None):
    """Store new tokens' K and V ([T, Hkv, D]) at pool rows slot_mapping (int64 [T]).

    Pools are [num_blocks, 16, Hkv, D]; an FP8 pool stores E4M3(x / scale).
    """
    NB, bs, Hkv, D = k_pool.shape
    if slot_mapping.dtype != torch.int64:
        raise TypeError("slot_mapping must be int64")
    st = L.lib().pkv_paged_kv_write(_ptr(k), _ptr(v), _dtype_code(k), _ptr(slot_mapping), int(slot_mapping.numel()),
                                    _ptr(k_pool), _ptr(v_pool), _dtype_code(k_pool), NB, bs, Hkv, D,
                                    float(k_scale), float(v_scale), _ptr(err_count), _stream(stream))
    L.check("pkv_paged_kv_write", st)


def decode_workspace_bytes(num_seqs, num_heads, head_dim, max_context_len, partition_tokens=0):
    n = L.lib().pkv_decode_workspace_bytes(int(num_seqs), int(num_heads), int(head_dim), int(max_context_len),
                                           int(partition_tokens))
    if n == 0:
        raise ValueError("invalid workspace bounds")
    return int(n)


def decode_workspace_bytes_shared(num_seqs, num_heads, head_dim, max_context_len, partition_tokens=0):
    n = L.lib().pkv_decode_workspace_bytes_shared(int(num_seqs), int(num_heads), int(head_dim),
                                                  int(max_context_len), int(partition_tokens))
    if n == 0:
        raise ValueError("invalid workspace bounds")
    return int(n)


def decode_workspace(num_seqs, num_heads, head_dim, max_context_len, partition_tokens=0, device=None, shared=False):
    """Allocate (through torch) a decode workspace for these bounds (shared=True:
    for paged_attention_decode_shared)."""
    f = decode_workspace_bytes_shared if shared else decode_workspace_bytes
    n = f(num_seqs, num_heads, head_dim, max_context_len, partition_tokens)
    return torch.empty(n, dtype=torch.uint8, device=device or "cuda")


def paged_attention_decode(out, q, k_pool, v_pool, block_tables, context_lens, scale, max_context_len,
                           workspace, k_scale=1.0, v_scale=1.0, partition_tokens=0, err_count=None, stream=None):
    """out[s, h] = softmax(scale * q[s, h] . K) V over the sequence's context,
    K/V read through block_tables (int32 [S, max_blocks]); context_lens int32 [S]."""
    S, Hq, D = q.shape
    NB, bs, Hkv, D2 = k_pool.shape
    if D2 != D or out.shape != q.shape:
        raise ValueError("shape mismatch")
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32:
        raise TypeError("block_tables and context_lens must be int32")
    st = L.lib().pkv_paged_attention_decode(
        _ptr(out), _ptr(q), _dtype_code(q), _ptr(k_pool), _ptr(v_pool), _dtype_code(k_pool),
        _ptr(block_tables), int(block_tables.shape[1]), _ptr(context_lens), S, int(max_context_len), NB, bs,
        Hq, Hkv, D, float(scale), float(k_scale), float(v_scale), int(partition_tokens),
        _ptr(workspace), int(workspace.numel() * workspace.element_size()), _ptr(err_count), _stream(stream))
    L.check("pkv_paged_attention_decode", st)
    return out


def paged_attention_decode_shared(out, q, k_pool, v_pool, block_tables, context_lens, scale, max_context_len,
                                  workspace, group_offsets, group_seqs, group_shared_blocks, k_scale=1.0,
                                  v_scale=1.0, partition_tokens=0, err_count=None, stream=None):
    """paged_attention_decode that reads blocks shared by a group of sequences
    once for the group.  The groups (int32 device tensors, see
    BlockManager.prefix_groups) are hints; the kernels check them."""
    S, Hq, D = q.shape
    NB, bs, Hkv, D2 = k_pool.shape
    if D2 != D or out.shape != q.shape:
        raise ValueError("shape mismatch")
    for t in (block_tables, context_lens, group_offsets, group_seqs, group_shared_blocks):
        if t.dtype != torch.int32:
            raise TypeError("tables, lengths and groups must be int32")
    ng = int(group_shared_blocks.numel())
    if group_offsets.numel() != ng + 1:
        raise ValueError("group_offsets must have num_groups + 1 entries")
    st = L.lib().pkv_paged_attention_decode_shared(
        _ptr(out), _ptr(q), _dtype_code(q), _ptr(k_pool), _ptr(v_pool), _dtype_code(k_pool),
        _ptr(block_tables), int(block_tables.shape[1]), _ptr(context_lens), S, int(max_context_len), NB, bs,
        Hq, Hkv, D, float(scale), float(k_scale), float(v_scale), int(partition_tokens),
        _ptr(group_offsets) if ng else None, _ptr(group_seqs) if group_seqs.numel() else None,
        int(group_seqs.numel()), _ptr(group_shared_blocks) if ng else None, ng,
        _ptr(workspace), int(workspace.numel() * workspace.element_size()), _ptr(err_count), _stream(stream))
    L.check("pkv_paged_attention_decode_shared", st)
    return out


def paged_attention_prefill(out, q, k_pool, v_pool, block_tables, context_lens, query_start, scale, max_query_len,
                            err_count=None, stream=None, k_scale=1.0, v_scale=1.0):
    """Causal attention of each sequence's new tokens (the last nq of its context)
    over its whole context; q/out [total_q, Hq, D], query_start int32 [S + 1].
    k_scale / v_scale dequantise an FP8 E4M3 cache (ignored for bf16)."""
    T, Hq, D = q.shape
    NB, bs, Hkv, D2 = k_pool.shape
    S = int(context_lens.numel())
    if D2 != D or out.shape != q.shape:
        raise ValueError("shape mismatch")
    for t in (block_tables, context_lens, query_start):
        if t.dtype != torch.int32:
            raise TypeError("tables, lengths and query_start must be int32")
    if query_start.numel() != S + 1:
        raise ValueError("query_start must have num_seqs + 1 entries")
    st = L.lib().pkv_paged_attention_prefill(
        _ptr(out), _ptr(q), _dtype_code(q), _ptr(k_pool), _ptr(v_pool), _dtype_code(k_pool), _ptr(block_tables),
        int(block_tables.shape[1]), _ptr(context_lens), _ptr(query_start), S, T, int(max_query_len), NB, bs, Hq,
        Hkv, D, float(scale), float(k_scale), float(v_scale), _ptr(err_count), _stream(stream))
    L.check("pkv_paged_attention_prefill", st)
    return out


def paged_attention_decode_noalloc(out, q, k_pool, v_pool, block_tables, context_lens, scale, max_context_len,
                                   k_scale=1.0, v_scale=1.0, partition_tokens=0, err_count=None, stream=None):
    """paged_attention_decode for callers that cannot allocate: no workspace argument;
    the library's fixed device scratch (PKV_NOALLOC_SCRATCH_BYTES) is used instead."""
    S, Hq, D = q.shape
    NB, bs, Hkv, D2 = k_pool.shape
    if D2 != D or out.shape != q.shape:
        raise ValueError("shape mismatch")
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32:
        raise TypeError("block_tables and context_lens must be int32")
    st = L.lib().pkv_paged_attention_decode_noalloc(
        _ptr(out), _ptr(q), _dtype_code(q), _ptr(k_pool), _ptr(v_pool), _dtype_code(k_pool),
        _ptr(block_tables), int(block_tables.shape[1]), _ptr(context_lens), S, int(max_context_len), NB, bs,
        Hq, Hkv, D, float(scale), float(k_scale), float(v_scale), int(partition_tokens), _ptr(err_count),
        _stream(stream))
    L.check("pkv_paged_attention_decode_noalloc", st)
    return out


def copy_blocks(k_pool, v_pool, src_dst_pairs, err_count=None, stream=None):
    """Copy whole blocks src -> dst in both pools; src_dst_pairs int64 [n, 2] on the device."""
    if src_dst_pairs.dtype != torch.int64:
        raise TypeError("src_dst_pairs must be int64")
    NB = k_pool.shape[0]
    block_bytes = k_pool[0].numel() * k_pool.element_size()
    st = L.lib().pkv_copy_blocks(_ptr(k_pool), _ptr(v_pool), block_bytes, _ptr(src_dst_pairs),
                                 int(src_dst_pairs.numel() // 2), NB, _ptr(err_count), _stream(stream))
    L.check("pkv_copy_blocks", st)


def _pool_ptr(t):
    """Pointer of a pool that may live on the device or in page-locked host memory."""
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    if not t.is_cuda and not t.is_pinned():
        raise ValueError("a host pool must be page-locked (pin_memory)")
    return C.c_void_p(t.data_ptr())


def swap_blocks(dst_k, dst_v, src_k, src_v, src_dst_pairs, err_count=None, stream=None):
    """Copy whole blocks between pools (device <-> pinned host).

    src_dst_pairs: int64 [n, 2], on the device or in page-locked host memory.
    """
    if src_dst_pairs.dtype != torch.int64:
        raise TypeError("src_dst_pairs must be int64")
    if dst_k.shape[1:] != src_k.shape[1:] or dst_k.dtype != src_k.dtype:
        raise ValueError("pools differ in block shape or dtype")
    block_bytes = src_k[0].numel() * src_k.element_size()
    st = L.lib().pkv_swap_blocks(_pool_ptr(dst_k), _pool_ptr(dst_v), dst_k.shape[0], _pool_ptr(src_k),
                                 _pool_ptr(src_v), src_k.shape[0], block_bytes, _pool_ptr(src_dst_pairs),
                                 int(src_dst_pairs.numel() // 2), _ptr(err_count), _stream(stream))
    L.check("pkv_swap_blocks", st)
