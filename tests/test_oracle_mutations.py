"""The oracle's pins are sensitive: plant a plausible mistake, the pins fail.

Each case edits a temporary copy of oracle/oracle.c (never the file itself),
compiles it with gcc, swaps it in for the oracle library, and runs the pin
tests that should notice.  At least one of them must fail for every planted
mistake; then the real library is restored.
"""
import os
import subprocess

import pytest

import oracle
import tests.test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "oracle.c")

# (name, text in oracle.c, planted replacement, pins expected to notice)
MUTATIONS = [
    ("causal_drops_own_key", "oracle_attend_dense(qv, *kbuf, *vbuf, p + 1,",
     "oracle_attend_dense(qv, *kbuf, *vbuf, p,", ["brute", "sdpa", "hyp"]),
    ("interleaved_gqa_heads", "int32_t h = g * G + gi;", "int32_t h = gi * c->Hkv + g;", ["brute", "sdpa", "hyp"]),
    ("dropped_scale", "        s *= scale;\n", "\n", ["brute", "sdpa", "two_key", "hyp"]),
    ("v_replaced_by_k", "out[d] += w * widen_bf16(V[j * ld + d]);", "out[d] += w * widen_bf16(K[j * ld + d]);",
     ["brute", "sdpa", "two_key", "hyp"]),
    ("gather_wrong_block", "int64_t blk = bt_row[b];", "int64_t blk = bt_row[b > 0 ? b - 1 : 0];",
     ["brute", "sdpa", "gather", "hyp"]),
    ("merge_ignores_weights", "        z += exp(lse[s] - mx);\n", "        z += 1.0;\n", ["split", "hyp_merge"]),
    ("slot_offset_shifted", "slot_mapping[query_start_loc[r] + i] = blk * block_size + p % block_size;",
     "slot_mapping[query_start_loc[r] + i] = blk * block_size + (p + 1) % block_size;", ["slots"]),
    ("kv_write_head_stride", "int64_t dst = ((blk * num_kv_heads + h) * block_size + off) * head_dim;",
     "int64_t dst = ((blk * num_kv_heads + (num_kv_heads - 1 - h)) * block_size + off) * head_dim;",
     ["kv_write", "slots", "hyp_move"]),
    ("lse_missing_max", "*lse = mx + log(z);", "*lse = log(z);", ["brute", "two_key", "hyp", "hyp_merge"]),
    ("pack_k_and_v_swapped", "memcpy(dk, k_cache + b * block_elems,", "memcpy(dk, v_cache + b * block_elems,",
     ["pack", "hyp_move"]),
    ("pack_block_off_by_one", "memcpy(dv, v_cache + b * block_elems,", "memcpy(dv, v_cache + (b + 1) % num_blocks * block_elems,",
     ["pack", "hyp_move"]),
    ("unpack_wrong_entry", "memcpy(k_cache + b * block_elems, staging + (2 * i) * block_elems,",
     "memcpy(k_cache + b * block_elems, staging + (2 * (n - 1 - i)) * block_elems,", ["unpack", "hyp_move"]),
]

CHECKS = {
    "brute": lambda: [pins.test_oracle_matches_pure_python_brute_force(w) for w in ("micro1", "micro4")],
    "hyp": lambda: pins.test_oracle_matches_brute_force_on_random_shapes(),
    "hyp_move": lambda: pins.test_data_movement_matches_brute_force_on_random_pools(),
    "hyp_merge": lambda: pins.test_split_merge_identity_on_random_cuts(),
    "sdpa": lambda: [pins.test_matches_torch_sdpa_on_unpaged_arrays(45, 20, 2)],
    "two_key": lambda: pins.test_hand_worked_two_key_example(),
    "split": lambda: pins.test_split_merge_reproduces_unsplit_attention(),
    "slots": lambda: pins.test_slot_mapping_matches_allocator_and_round_trips_through_gather(),
    "gather": lambda: pins.test_gather_walks_blocks_in_table_order(),
    "kv_write": lambda: pins.test_kv_write_byte_exact_and_preserves_untouched_slots(),
    "pack": lambda: pins.test_kv_pack_matches_brute_force_and_the_gather(),
    "unpack": lambda: pins.test_kv_unpack_inverts_pack_and_touches_nothing_else(),
}


@pytest.mark.parametrize("name,old,new,checks", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_planted_mistake_is_caught(name, old, new, checks, tmp_path, monkeypatch):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not found exactly once"
    mutated = tmp_path / "oracle_mut.c"
    mutated.write_text(src.replace(old, new))
    lib = tmp_path / "liboracle_mut.so"
    subprocess.check_call(["gcc", "-O1", "-std=c11", "-D_GNU_SOURCE", "-shared", "-fPIC", "-pthread",
                           "-o", str(lib), str(mutated), "-lm"])
    oracle._load()  # make sure the real one is built and cached first
    monkeypatch.setattr(oracle, "_lib", oracle._bind(str(lib)))
    caught = []
    for c in checks:
        try:
            CHECKS[c]()
        except (AssertionError, ValueError):
            caught.append(c)
    assert caught, f"planted mistake {name!r} passed every pin in {checks}"
