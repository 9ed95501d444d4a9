"""The pins catch plausible oracle mistakes.

Each case copies the oracle's C source to a temporary directory, plants one
mistake by text substitution (a dropped term, a wrong sign, a wrong index or
layout), builds it, swaps it in as the oracle's library and runs the pin
tests.  At least one pin must fail for every planted mistake.  The committed
oracle is never modified.
"""
import ctypes
import os
import subprocess

import pytest

import oracle
from tests import test_oracle_pins as pins
from tests import test_oracle_prefill as prefill_pins
from tests import test_oracle_block_manager as bm_pins
from tests import test_oracle_fp8 as fp8_pins
from tests import test_oracle_prefix as prefix_pins
from tests import test_oracle_swap as swap_pins

PIN_TESTS = [
    pins.test_block_count_golden,
    pins.test_write_roundtrip_and_untouched_rows,
    pins.test_copy_blocks_simultaneous_semantics,
    pins.test_copy_on_write_isolates_sharers,
    lambda: pins.test_attention_equals_dense_library_softmax([5, 16, 31, 48, 100], 8, 2, 64, 16),
    pins.test_attention_equals_torch_sdpa_gqa,
    pins.test_uniform_attention_gives_mean_of_v,
    pins.test_single_token_gives_its_value_row_exactly,
    pins.test_gqa_head_mapping_is_contiguous_groups,
    pins.test_two_token_closed_form_golden,
    pins.test_context_len_zero_gives_zero_output,
    lambda: pins.test_split_merge_equals_unsplit("ragged"),
    pins.test_lse_merge_closed_form,
    lambda: prefill_pins.test_prefill_equals_sdpa_with_bottom_right_causal_mask([31, 17, 0, 64], [1, 20, 48, 3],
                                                                                 6, 3, 64, 16),
    swap_pins.test_swap_out_then_in_equals_copy_blocks,
    swap_pins.test_swap_round_trip_restores_and_swap_out_reads_only,
    swap_pins.test_swap_of_a_permutation_is_a_gather,
    swap_pins.test_lru_worked_example_golden,
    bm_pins.test_block_manager_worked_example_golden,
    prefix_pins.test_fnv1a64_published_vectors,
    prefix_pins.test_keys_chain_over_the_prefix,
    prefix_pins.test_worked_example,
    prefix_pins.test_cached_blocks_worked_example,
    prefix_pins.test_release_keeps_the_key_and_share_revives,
    prefix_pins.test_allocation_evicts_least_recently_released_first,
    prefix_pins.test_first_sequence_in_order_becomes_holder,
    fp8_pins.test_decode_table_matches_library,
    fp8_pins.test_encode_golden,
    fp8_pins.test_write_quantizes_into_the_bf16_layout,
    lambda: fp8_pins.test_attention_equals_bf16_attention_on_exact_values(8, 2),
    lambda: bm_pins.test_conservation_invariants(0),
    lambda: bm_pins.test_append_block_counts_closed_form(0),
    bm_pins.test_slots_feed_the_table_walk,
    lambda: bm_pins.test_free_matches_python_restatement(0),
    lambda: swap_pins.test_lru_characterisation(0),
]

MUTANTS = {
    "in-block offset": ("int offset = (int)(slot % bs);", "int offset = (int)((slot / bs) % bs);"),
    "read offset": ("pool_row(block, hkv, i % bs, Hkv, bs, d);\n        double dot",
                    "pool_row(block, hkv, (i + 1) % bs, Hkv, bs, d);\n        double dot"),
    "gqa mapping": ("int hkv = hq / g;", "int hkv = hq % Hkv;"),
    "dropped scale": ("z[i - t_begin] = scale * dot;", "z[i - t_begin] = dot;"),
    "exp sign": ("double w = exp(z[i - t_begin] - m);", "double w = exp(m - z[i - t_begin]);"),
    "pool layout": ("(((size_t)block * (size_t)num_kv_heads + (size_t)head) * (size_t)bs + (size_t)offset)",
                    "(((size_t)block * (size_t)bs + (size_t)offset) * (size_t)num_kv_heads + (size_t)head)"),
    "transposed k": ("bf16_to_f64(krow[c])", "bf16_to_f64(krow[d - 1 - c])"),
    "sequential copy": ("memcpy(k_cache + dst, snap_k + (size_t)p * block_elems",
                        "memcpy(k_cache + dst, k_cache + (size_t)pairs[2 * p] * block_elems"),
    "missing normalisation": ("o[c] = (l > 0.0) ? acc[c] / l : 0.0;", "o[c] = (l > 0.0) ? acc[c] : 0.0;"),
    "merge drops rescale": ("L += l[p] * w;", "L += l[p];"),
    # prefill: a query also sees the next position, or misses its own
    "prefill causal bound +1": ("bs, hq, 0, pos + 1, scale", "bs, hq, 0, pos + 2 > context_lens[s] ? context_lens[s] : pos + 2, scale"),
    "prefill causal bound -1": ("bs, hq, 0, pos + 1, scale", "bs, hq, 0, pos, scale"),
    "prefill query position": ("int pos = context_lens[s] - q_len + (t - query_start[s]);",
                               "int pos = (t - query_start[s]);"),
    # swap: the key region copied into both host buffers; a block shifted by one;
    # the most recently used block chosen first; ties to the higher id
    "swap key into value": ("host_v[(size_t)i * block_elems + e] = v_cache[", "host_v[(size_t)i * block_elems + e] = k_cache["),
    "swap-in wrong block": ("k_cache[(size_t)ids[i] * block_elems + e] = host_k[",
                            "k_cache[(size_t)((ids[i] + 1) % num_blocks) * block_elems + e] = host_k["),
    "lru newest first": ("last_use[b] < last_use[best]", "last_use[b] > last_use[best]"),
    "lru ties to higher id": ("last_use[b] < last_use[best]", "last_use[b] <= last_use[best]"),
    # block manager: copy-on-write of unshared blocks; the old block keeps its
    # reference; a partly filled block allocated again; the slot offset from the
    # wrong position; freeing pushes before the count reaches zero; the free
    # list used first-in first-out
    "cow unshared": ("else if (refcount[cur] > 1) cow = 1;", "else if (refcount[cur] >= 1) cow = 1;"),
    "cow keeps reference": ("refcount[old] -= 1;", "refcount[old] -= 0;"),
    "partial block reallocated": ("int first_new = (pos0 + bs - 1) / bs;", "int first_new = pos0 / bs + (pos0 > 0);"),
    "slot offset": ("slot_mapping[off + t] = (int64_t)row[p / bs] * bs + p % bs;",
                    "slot_mapping[off + t] = (int64_t)row[p / bs] * bs + t % bs;"),
    "free pushes early": ("if (--refcount[b] == 0) {", "if (--refcount[b] >= 0) {"),
    "fifo free list": ("        b = free_stack[--*top];",
                       "        b = free_stack[0]; memmove(free_stack, free_stack + 1, sizeof(int32_t) * (size_t)(--*top));"),
    # prefix cache: keys without the chain; a holder's validity ignored; the
    # last inserter wins; the whole prompt looked up; FNV's multiply first
    "prefix key unchained": ("buf[i] = (uint8_t)(prev >> (8 * i));", "buf[i] = 0;"),
    "prefix holder unchecked": ("if (!valid_holder(b, key, block_hash, num_blocks)) break;",
                                "if (b < 0) break;"),
    "prefix last inserter wins": ("if (slot >= 0 && valid_holder(cvals[slot], key, block_hash, num_blocks)) continue;",
                                  "if (0) continue;"),
    # cached blocks: the key dropped on release (no cached state); the most
    # recently released block evicted first; eviction keeps the stale key; a
    # prefix hit leaves the block evictable; cached blocks not counted as
    # available
    "release drops key": ("if (block_hash[b] != 0) lru_stamp[b] = (*clock)++;",
                          "if (0) lru_stamp[b] = (*clock)++;"),
    "evict most recent": ("lru_stamp[c] < lru_stamp[b]", "lru_stamp[c] > lru_stamp[b]"),
    "eviction keeps key": ("block_hash[b] = 0; /* evicted", "/* evicted"),
    "hit not revived": ("if (refcount[b] == 0) lru_stamp[b] = -1;\n            refcount[b] += 1;",
                        "refcount[b] += 1;"),
    "cached not available": ("if (lru_stamp[b] >= 0) ++n;", "if (0) ++n;"),
    "prefix whole prompt": ("int look = n > 0 ? (n - 1) / bs : 0;", "int look = n / bs;"),
    "fnv multiply first": ("h ^= p[i];\n        h *= 1099511628211ull;", "h *= 1099511628211ull;\n        h ^= p[i];"),
    # fp8: subnormals one binade off; ties to the odd code; the scale multiplied
    # instead of divided on the way in; the key scale applied to the values
    "e4m3 subnormal exponent": ("if (e == 0) v = ldexp((double)m / 8.0, -6);", "if (e == 0) v = ldexp((double)m / 8.0, -7);"),
    "e4m3 ties to odd": ("(err == best_err && (c & 1) == 0)", "(err == best_err && (c & 1) == 1)"),
    "fp8 write scale inverted": ("float inv_k = 1.0f / k_scale[h], inv_v = 1.0f / v_scale[h];",
                                 "float inv_k = k_scale[h], inv_v = 1.0f / v_scale[h];"),
    "fp8 value scale": ("(oracle_e4m3_decode(vr[c]) * v_scale[hkv])", "(oracle_e4m3_decode(vr[c]) * k_scale[hkv])"),
    # the new token left out of the attended range (context_len - 1 tokens)
    "context off by one": ("hq, 0, context_lens[s], scale", "hq, 0, context_lens[s] - 1, scale"),
}


def _build_mutant(tmp_path, old, new):
    src = open(os.path.join(os.path.dirname(oracle.__file__), "pkv_oracle.c")).read()
    assert src.count(old) >= 1, f"mutation anchor not found: {old!r}"
    src = src.replace(old, new)
    path = tmp_path / "mutant.c"
    path.write_text(src)
    so = tmp_path / "libmutant.so"
    subprocess.check_call(["gcc", "-O1", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", str(so), str(path), "-lm"])
    return str(so)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name, tmp_path, monkeypatch):
    old, new = MUTANTS[name]
    so = _build_mutant(tmp_path, old, new)
    good = oracle._load()
    lib = ctypes.CDLL(so)
    # every function the oracle declared argument types for
    for fn, f in list(vars(good).items()):
        if fn.startswith("oracle_") and hasattr(f, "argtypes"):
            getattr(lib, fn).argtypes = f.argtypes
            getattr(lib, fn).restype = f.restype
    monkeypatch.setattr(oracle, "_lib", lib)
    caught = []
    for t in PIN_TESTS:
        try:
            t()
        except (AssertionError, IndexError, ValueError) as e:
            caught.append((getattr(t, "__name__", "lambda"), type(e).__name__))
    assert caught, f"no pin caught the planted mistake {name!r}"
