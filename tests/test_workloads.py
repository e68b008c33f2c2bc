"""The five synthetic workloads against their recipes: request counts, length ranges, head shapes,
pool sizes, the 8192-token budget of the mixed step, the shared 2048-token prefix, and the block
allocation every kernel relies on (distinct physical blocks per request except the shared prefix,
ids inside the pool, -1 past a request's last block, slots that never land in a shared block).
Host only."""
import numpy as np
import pytest

from paged_kv_cache_461_b200 import workloads as W

SPEC = {
    # name: (requests, (q heads, kv heads, head dim), pool blocks)
    "tiny_decode": (4, (4, 4, 64), 64),
    "llama3_8b_decode": (256, (32, 8, 128), 70_000),
    "mixed_step_8192": (None, (32, 8, 128), 70_000),
    "prefix_sharing": (128, (32, 8, 128), 32_768),
    "long_context_decode": (16, (64, 8, 128), 140_000),
}


def _check_allocation(lay):
    bt = lay.block_table
    need = (lay.seq_lens.astype(np.int64) + 15) // 16
    ns = lay.shared_prefix_blocks
    seen = {}
    for r in range(lay.num_seqs):
        row = bt[r]
        assert (row[:need[r]] >= 0).all() and (row[:need[r]] < lay.num_blocks).all()
        assert (row[need[r]:] == -1).all()
        for b in row[ns:need[r]].tolist():
            assert b not in seen, f"block {b} held by requests {seen[b]} and {r}"
            seen[b] = r
    if ns:
        shared = set(bt[0, :ns].tolist())
        assert all(set(bt[r, :ns].tolist()) == shared for r in range(lay.num_seqs))
        assert not shared & set(seen)
    # this step's slots: distinct, at each token's position, never inside a shared block
    slots = lay.slot_mapping
    assert len(np.unique(slots)) == len(slots)
    qsl = lay.query_start_loc
    for r in range(lay.num_seqs):
        pos = lay.ctx_lens[r] + np.arange(lay.q_lens[r])
        want = bt[r, pos // 16].astype(np.int64) * 16 + pos % 16
        assert np.array_equal(slots[qsl[r]:qsl[r + 1]], want)
        if ns:
            assert (pos >= ns * 16).all()


@pytest.mark.parametrize("name", list(SPEC))
def test_workload_matches_its_recipe(name):
    lay = W.workload_layout(name)
    R, (hq, hkv, d), nb = SPEC[name]
    assert (lay.num_q_heads, lay.num_kv_heads, lay.head_dim, lay.block_size) == (hq, hkv, d, 16)
    assert lay.num_blocks == nb
    if R is not None:
        assert lay.num_seqs == R
    c, q = lay.ctx_lens, lay.q_lens
    if name == "tiny_decode":
        assert c.tolist() == [17, 33, 64, 100] and (q == 1).all()
        assert lay.seq_lens.tolist() == [18, 34, 65, 101]
    elif name == "llama3_8b_decode":
        assert (q == 1).all() and c.min() >= 512 and c.max() <= 4096
    elif name == "mixed_step_8192":
        nd = lay.extra["num_decode"]
        assert nd == 192 and (q[:nd] == 1).all() and c[:nd].min() >= 256 and c[:nd].max() <= 4096
        chunks, cached = q[nd:], c[nd:]
        assert chunks.sum() == 8000 and lay.num_tokens == 8192
        assert chunks[:-1].min() >= 256 and chunks.max() <= 2048 and chunks[-1] >= 1
        assert cached.min() >= 0 and cached.max() <= 2048
    elif name == "prefix_sharing":
        assert (q == 1).all() and lay.shared_prefix_blocks == 128
        assert (c - 2048).min() >= 64 and (c - 2048).max() <= 1024
    elif name == "long_context_decode":
        assert (q == 1).all() and c.min() >= 32768 and c.max() <= 131072
    _check_allocation(lay)


@pytest.mark.parametrize("name", list(SPEC))
def test_workloads_are_deterministic_per_seed(name):
    a, b = W.workload_layout(name), W.workload_layout(name)
    assert np.array_equal(a.block_table, b.block_table) and np.array_equal(a.ctx_lens, b.ctx_lens)
    if name != "tiny_decode":
        other = W.workload_layout(name, seed=1234)
        assert not np.array_equal(other.block_table, a.block_table)


def test_neighbouring_logical_blocks_are_scattered():
    # ids come from a permutation of the pool: consecutive logical blocks are rarely adjacent
    lay = W.workload_layout("llama3_8b_decode")
    bt = lay.block_table
    need = (lay.seq_lens + 15) // 16
    adj = sum(int((np.diff(bt[r, :n]) == 1).sum()) for r, n in enumerate(need))
    total = int((need - 1).sum())
    assert adj < 0.01 * total


def test_values_follow_the_recipe():
    lay = W.workload_layout("tiny_decode")
    v = W.make_values_numpy(lay)
    q = W.bf16_bits_to_f32(v.q)
    assert q.shape == (4, 4, 64) and abs(float(q.mean())) < 0.2 and 0.8 < float(q.std()) < 1.2
    # unused pool slots hold the quiet-NaN sentinel; cached context slots hold finite values
    k = v.k_cache
    ctx_slots = lay.ctx_slots
    mask = np.zeros(lay.num_blocks * 16, dtype=bool)
    mask[ctx_slots] = True
    kk = k.transpose(0, 2, 1, 3).reshape(lay.num_blocks * 16, lay.num_kv_heads, lay.head_dim)
    assert (kk[~mask] == W.BF16_QNAN).all()
    assert np.isfinite(W.bf16_bits_to_f32(kk[mask])).all()
