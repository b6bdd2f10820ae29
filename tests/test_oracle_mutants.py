"""Planted mistakes: each mutant is a copy of the oracle with one plausible bug
(a dropped term, a wrong sign or index, a transposed operand), built on the CPU
in a temporary directory.  The pin suite must reject every one of them.

The mutants never touch the committed oracle; they are compiled from edited
copies of its source and loaded in place of it for the duration of one check.
"""
import os
import subprocess

import pytest

import oracle
import tests.test_allocator_ref as A
import tests.test_oracle_pins as P

SRC = os.path.join(os.path.dirname(oracle.__file__), "oracle.c")

MUTANTS = {
    "gqa_head_mapping": ("int g = h / group;", "int g = h % num_kv_heads;"),
    "dropped_scale": ("scores[t - t0] = scale * dot;", "scores[t - t0] = dot;"),
    "slot_offset": ("(size_t)(t % block_size)) * num_kv_heads + g)",
                    "(size_t)((t + 1) % block_size)) * num_kv_heads + g)"),
    "table_index": ("int32_t blk = table[t / block_size];\n    if (blk < 0 || blk >= num_blocks) return 0;",
                    "int32_t blk = table[t % block_size];\n    if (blk < 0 || blk >= num_blocks) return 0;"),
    "keys_from_value_pool": ("dot += qv[d] * (load_elem(k_pool,", "dot += qv[d] * (load_elem(v_pool,"),
    "exp_sign": ("w = exp(scores[t - t0] - m);", "w = exp(m - scores[t - t0]);"),
    "merge_drops_l": ("w = pl[p] * exp(pm[p] - M);", "w = exp(pm[p] - M);"),
    "v_scale_for_k": ("* k_scale)", "* v_scale)"),
    "e4m3_bias": ("ldexp(1.0 + (double)m / 8.0, e - 7)", "ldexp(1.0 + (double)m / 8.0, e - 8)"),
    "e4m3_subnormal": ("ldexp((double)m / 8.0, -6)", "ldexp((double)m / 8.0, -7)"),
    "e4m3_ties_odd": ("(a == mid && (c & 1))", "(a == mid && !(c & 1))"),
    "e4m3_no_saturation": ("if (a >= 448.0) return (uint8_t)(sign | 0x7E);",
                           "if (a >= 464.0) return (uint8_t)(sign | 0x7F);"),
    "write_v_with_k_scale": ("load_src_float(v, src_dtype, (size_t)i * row + e), v_scale)",
                             "load_src_float(v, src_dtype, (size_t)i * row + e), k_scale)"),
    "write_slot_row": ("(char*)k_pool + (size_t)slot * row * es", "(char*)k_pool + (size_t)(slot + 1) * row * es"),
    "copy_only_k": ("memcpy((char*)v_pool + (size_t)d * block_bytes", "if (0) memcpy((char*)v_pool + (size_t)d * block_bytes"),
    "swap_only_k": ("memcpy((char*)dst_v", "if (0) memcpy((char*)dst_v"),
    "swap_accepts_repeated_dst": ("for (j = i + 1; j < num_pairs; j++)", "for (j = num_pairs; j < num_pairs; j++)"),
    "swap_half_block": ("(const char*)src_k + (size_t)s * block_bytes, block_bytes);",
                        "(const char*)src_k + (size_t)s * block_bytes, block_bytes / 2);"),
    "prefill_excludes_itself": ("pos + 1, block_size, num_blocks, num_kv_heads, h / group,",
                                "pos, block_size, num_blocks, num_kv_heads, h / group,"),
    "prefill_position_ignores_prefix": ("pos = context_lens[s2] - (query_start[s2 + 1] - query_start[s2]) + (r - query_start[s2]);",
                                        "pos = (r - query_start[s2]);"),
    "prefill_attends_past_itself": [
        ("scores = (double*)malloc(sizeof(double) * (pos + 1));", "scores = (double*)malloc(sizeof(double) * (pos + 2));"),
        ("pos + 1, block_size, num_blocks, num_kv_heads, h / group,",
         "(pos + 2 <= context_lens[s2] ? pos + 2 : pos + 1), block_size, num_blocks, num_kv_heads, h / group,")],
    "prefill_head_mapping": ("pos + 1, block_size, num_blocks, num_kv_heads, h / group,",
                             "pos + 1, block_size, num_blocks, num_kv_heads, h % num_kv_heads,"),
    "prefill_k_with_v_scale": ("h / group, head_dim, scale, k_scale,\n                         v_scale, scores, &m, &l, o)",
                               "h / group, head_dim, scale, v_scale,\n                         v_scale, scores, &m, &l, o)"),
    "gather_wrong_slot": ("((size_t)blk * block_size + (size_t)(t % block_size)) * row_bytes, row_bytes);",
                          "((size_t)blk * block_size + (size_t)(t / block_size)) * row_bytes, row_bytes);"),
}

def _pins(golden):
    """Every pin, as callables that raise when the oracle is wrong."""
    fns = [
        lambda: P.test_worked_example(golden),
        P.test_len_one_returns_v0_exactly, P.test_zero_query_gives_mean_of_v,
        P.test_equal_keys_give_mean_of_v, P.test_constant_values_give_that_row,
        P.test_two_tokens_logistic, P.test_empty_context_is_zero,
        lambda: [P.test_paged_equals_contiguous(*a) for a in [(2, 2, 64), (8, 2, 64), (16, 2, 128)]],
        P.test_bf16_paged_equals_contiguous, P.test_fp8_paged_equals_dequantised_contiguous,
        P.test_gqa_equals_mha_with_repeated_kv_heads, P.test_placement_permutation_is_bitwise_invariant,
        lambda: [P.test_partitioned_merge_equals_single_pass(p) for p in (16, 48, 112)],
        P.test_stale_slots_are_not_read, P.test_invalid_block_ids_are_skipped_and_counted,
        P.test_shared_prefix_reads_identical_kv_until_cow,
        P.test_e4m3_decode_all_codes_match_library, P.test_e4m3_format_landmarks,
        P.test_e4m3_encode_matches_brute_force_sweep,
        P.test_kv_write_bf16_is_raw_copy_and_touches_nothing_else,
        P.test_kv_write_fp8_matches_library_cast, P.test_copy_blocks_semantics,
        P.test_swap_blocks_between_pools_of_different_sizes,
        lambda: [P.test_prefill_equals_numpy_causal_attention(*a) for a in [(2, 2), (8, 2)]],
        P.test_prefill_first_position_returns_v0, P.test_prefill_bf16_and_row_subset,
        P.test_prefill_fp8_equals_numpy_causal_of_library_decoded_codes,
    ]
    return fns


def _build_mutant(tmp, name, edits):
    """edits: one (old, new) pair or a list of them, applied to the oracle's source."""
    src = open(SRC).read()
    for old, new in ([edits] if isinstance(edits, tuple) else edits):
        assert src.count(old) >= 1, "mutation anchor not found: %s" % name
        src = src.replace(old, new)
    path_c = os.path.join(tmp, name + ".c")
    path_so = os.path.join(tmp, name + ".so")
    open(path_c, "w").write(src)
    subprocess.run(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
                    path_c, "-o", path_so, "-lm"], check=True)
    return path_so


def _load_like_oracle(path):
    saved = oracle._lib
    oracle._lib = None
    real_build = oracle._build.build
    oracle._build.build = lambda force=False: path
    try:
        L = oracle.lib()
    finally:
        oracle._build.build = real_build
        oracle._lib = saved
    return L


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_reject_planted_mistake(name, golden_dir, tmp_path):
    path = _build_mutant(str(tmp_path), name, MUTANTS[name])
    mutant = _load_like_oracle(path)
    saved = oracle._lib
    oracle._lib = mutant
    caught = []
    try:
        for fn in _pins(golden_dir):
            try:
                fn()
            except (Exception, pytest.fail.Exception) as e:  # noqa: BLE001 - any failure counts as a catch
                caught.append(repr(e)[:80])
                break
    finally:
        oracle._lib = saved
    assert caught, "no pin caught the planted mistake %s" % name


def test_pins_reject_allocator_copying_for_last_holder(monkeypatch):
    """Planted mistake in the reference block manager: copy-on-write even when
    the writer is the block's last holder."""
    from oracle import allocator

    def bad_append(self, seq):
        n = self.lens[seq]
        table = self.tables[seq]
        cow = None
        if n % self.block_size == 0:
            table.append(self._pop())
        else:
            last = table[-1]
            if self.ref[last] >= 1:      # the planted mistake
                new = self._pop()
                self.ref[last] -= 1
                if self.ref[last] == 0:
                    self.free.append(last)
                table[-1] = new
                cow = (last, new)
        slot = table[n // self.block_size] * self.block_size + n % self.block_size
        self.lens[seq] = n + 1
        return slot, cow

    monkeypatch.setattr(allocator.RefBlockManager, "append_token", bad_append)
    with pytest.raises(AssertionError):
        A.test_parallel_sampling_cow_trace()


def test_pins_reject_swap_out_that_keeps_device_blocks(monkeypatch):
    """Planted mistake in the reference block manager: swap-out copies the pages
    but never returns the device blocks to the free list."""
    from oracle import allocator

    def bad_swap_out(self, seq):
        table = self.tables[seq]
        if len(table) > len(self.host_free):
            raise MemoryError("not enough free host blocks")
        pairs = []
        for i, b in enumerate(table):
            h = self.host_free.popleft()
            pairs.append((b, h))
            self.ref[b] -= 1               # the planted mistake: no return to the free list
            table[i] = h
        self.swapped.add(seq)
        return pairs

    monkeypatch.setattr(allocator.RefBlockManager, "swap_out", bad_swap_out)
    with pytest.raises(AssertionError):
        A.test_swap_round_trip_restores_every_token()


def test_pins_reject_swap_in_that_restores_old_block_ids(monkeypatch):
    """Planted mistake: swap-in writes the pages back to the block ids they left,
    which other sequences may own by then."""
    from oracle import allocator

    def bad_swap_in(self, seq):
        table = self.tables[seq]
        pairs = []
        for i, h in enumerate(table):
            b = h                          # the planted mistake: host id reused as device id
            self.ref[b] += 1
            pairs.append((h, b))
            self.host_free.append(h)
            table[i] = b
        self.swapped.discard(seq)
        return pairs

    monkeypatch.setattr(allocator.RefBlockManager, "swap_in", bad_swap_in)
    with pytest.raises(AssertionError):
        A.test_swap_round_trip_restores_every_token()


@pytest.mark.parametrize("pin", ["test_a_block_is_keyed_by_its_whole_prefix",
                                 "test_two_requests_share_their_common_system_prompt_block"])
def test_pins_reject_prefix_cache_keyed_by_tokens_only(monkeypatch, pin):
    """Planted mistake: a full block is keyed by its own 16 tokens only, not by
    its prefix, so the same tokens after a different start alias one block.
    Both the synthetic pin and the hand-worked system-prompt case reject it."""
    from oracle import allocator
    real = allocator.RefBlockManager.alloc_seq_tokens

    def bad(self, tokens):
        saved = self._serial
        seq, cached = real(self, tokens)
        # re-key everything just registered without its parent
        for b, key in list(self.key_of.items()):
            if key[0] != 0:
                blk, serial = self.cache.pop(key)
                self.key_of[b] = (0, key[1])
                self.cache[(0, key[1])] = (blk, serial)
        return seq, cached

    monkeypatch.setattr(allocator.RefBlockManager, "alloc_seq_tokens", bad)
    with pytest.raises(AssertionError):
        getattr(A, pin)()


def test_pins_reject_prefix_cache_that_keeps_keys_of_reused_blocks(monkeypatch):
    """Planted mistake: a cached block handed out for new data keeps its key."""
    from oracle import allocator

    def bad_pop(self):
        if not self.free:
            raise MemoryError("no free block")
        b = self.free.popleft()
        self.ref[b] = 1
        return b

    monkeypatch.setattr(allocator.RefBlockManager, "_pop", bad_pop)
    with pytest.raises(AssertionError):
        A.test_evicted_prefix_is_not_served_from_overwritten_blocks()
