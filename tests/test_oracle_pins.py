"""Pins for the fp64 oracle, checked against things other than itself.

Each test ties the oracle to a fact the pages or the mathematics fix:
a pure-Python brute force, closed forms, a hand-worked example, torch's fp64
scaled_dot_product_attention on unpaged data, and the invariances the pages
state (block ids are arbitrary, prefix blocks are reused as they are, chunked
prefill does not change results, one mixed step equals separate requests).
"""
import json
import math
import os

import numpy as np
import pytest

import oracle
from oracle import brute
from paged_kv_cache_461_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _written(layout, vals):
    """Pools after this step's KV write (oracle write)."""
    return oracle.kv_write(vals.k_new, vals.v_new, layout.slot_mapping, vals.k_cache, vals.v_cache)


def _micro_layouts():
    rng = np.random.default_rng(1234)
    cases = []
    for k in range(6):
        R = int(rng.integers(1, 4))
        ctx = rng.integers(0, 41, size=R)
        ql = rng.integers(1, 6, size=R)
        if k == 3:
            ql[0] = 0          # a request that contributes nothing this step
            ctx[0] = max(ctx[0], 1)
        Hkv = int(rng.choice([1, 2]))
        G = int(rng.choice([1, 2, 3]))
        lay = W.build_layout(f"micro{k}", ctx, ql, num_q_heads=Hkv * G, num_kv_heads=Hkv, head_dim=8,
                             num_blocks=40, rng=rng, seed=100 + k)
        cases.append(lay)
    return cases


def _nested(a):
    return a.tolist()


# ----------------------------------------------------------------------------
# brute force
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("which", ["tiny_decode"] + [f"micro{k}" for k in range(6)])
def test_oracle_matches_pure_python_brute_force(which):
    if which == "tiny_decode":
        lay = W.workload_layout("tiny_decode")
    else:
        lay = _micro_layouts()[int(which[5:])]
    vals = W.make_values_numpy(lay)
    kc, vc = _written(lay, vals)
    scale = 1.0 / math.sqrt(lay.head_dim)
    out, lse, err = oracle.attention_for(lay, kc, vc, vals.q, scale=scale)
    bt = [list(map(int, row)) for row in lay.block_table]
    bout, blse = brute.attention(_nested(vals.q), _nested(kc), _nested(vc), lay.query_start_loc.tolist(),
                                 lay.seq_lens.tolist(), bt, lay.num_q_heads, lay.num_kv_heads, lay.head_dim,
                                 scale)
    if lay.num_tokens:
        np.testing.assert_allclose(out, np.asarray(bout), rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse, np.asarray(blse), rtol=0, atol=1e-12)
    assert err < 1e-12
    assert not np.isnan(out).any(), "a sentinel (unused) slot was read"


try:
    from hypothesis import given, settings
    from hypothesis import strategies as st
except ImportError:  # pragma: no cover
    given = None


if given is not None:
    @settings(max_examples=150, deadline=None, derandomize=True)
    @given(data=st.data())
    def test_oracle_matches_brute_force_on_random_shapes(data):
        # random request mixes (empty requests included), GQA ratios, head dims, scales and pool slack
        R = data.draw(st.integers(1, 3))
        ctx = [data.draw(st.integers(0, 40)) for _ in range(R)]
        ql = [data.draw(st.integers(0, 5)) for _ in range(R)]
        Hkv = data.draw(st.sampled_from([1, 2]))
        G = data.draw(st.sampled_from([1, 2, 4]))
        D = data.draw(st.sampled_from([4, 8, 16]))
        scale = data.draw(st.floats(0.05, 1.0))
        seed = data.draw(st.integers(0, 2 ** 31 - 1))
        need = sum((c + q + 15) // 16 for c, q in zip(ctx, ql))
        lay = W.build_layout("hyp", ctx, ql, num_q_heads=Hkv * G, num_kv_heads=Hkv, head_dim=D,
                             num_blocks=need + data.draw(st.integers(0, 5)) + 1, seed=seed)
        vals = W.make_values_numpy(lay)
        kc, vc = _written(lay, vals)
        out, lse, _ = oracle.attention_for(lay, kc, vc, vals.q, scale=scale)
        bt = [list(map(int, row)) for row in lay.block_table]
        bout, blse = brute.attention(_nested(vals.q), _nested(kc), _nested(vc), lay.query_start_loc.tolist(),
                                     lay.seq_lens.tolist(), bt, lay.num_q_heads, lay.num_kv_heads, lay.head_dim,
                                     scale)
        if lay.num_tokens:
            np.testing.assert_allclose(out, np.asarray(bout), rtol=0, atol=1e-12)
            np.testing.assert_allclose(lse, np.asarray(blse), rtol=0, atol=1e-12)
            assert not np.isnan(out).any(), "a sentinel (unused) slot was read"


# ----------------------------------------------------------------------------
# closed forms
# ----------------------------------------------------------------------------

def _single_request(ctx, q_len, D=16, Hq=2, Hkv=1, seed=7, num_blocks=None):
    lay = W.build_layout("one", [ctx], [q_len], num_q_heads=Hq, num_kv_heads=Hkv, head_dim=D,
                         num_blocks=num_blocks, seed=seed)
    vals = W.make_values_numpy(lay)
    return lay, vals


def test_constant_v_returns_v():
    lay, vals = _single_request(37, 5)
    v = W.f32_to_bf16_bits(np.linspace(-3, 3, lay.head_dim).astype(np.float32))
    vals.v_new[:] = v
    vc = vals.v_cache.copy()
    slots = lay.ctx_slots
    vc[slots // 16, :, slots % 16, :] = v
    vals.v_cache[:] = vc
    kc, vcw = _written(lay, vals)
    out, _, _ = oracle.attention_for(lay, kc, vcw, vals.q)
    expect = W.bf16_bits_to_f32(v).astype(np.float64)
    np.testing.assert_allclose(out, np.broadcast_to(expect, out.shape), rtol=0, atol=1e-13)


def test_zero_query_gives_mean_of_visible_values():
    lay, vals = _single_request(21, 4, Hq=4, Hkv=2)
    vals.q[:] = 0
    kc, vc = _written(lay, vals)
    out, lse, _ = oracle.attention_for(lay, kc, vc, vals.q)
    for g in range(lay.num_kv_heads):
        Vg = W.bf16_bits_to_f32(oracle.gather_kv(vc, lay.block_table[0], int(lay.seq_lens[0]), g)).astype(np.float64)
        for i in range(4):
            p = 21 + i
            mean = Vg[:p + 1].mean(axis=0)
            for h in (2 * g, 2 * g + 1):
                np.testing.assert_allclose(out[i, h], mean, rtol=0, atol=1e-13)
                assert abs(lse[i, h] - math.log(p + 1)) < 1e-13


def test_single_key_returns_that_value():
    lay, vals = _single_request(0, 1)
    kc, vc = _written(lay, vals)
    out, lse, _ = oracle.attention_for(lay, kc, vc, vals.q)
    v0 = W.bf16_bits_to_f32(vals.v_new[0, 0]).astype(np.float64)
    np.testing.assert_array_equal(out[0, 0], v0)
    np.testing.assert_array_equal(out[0, 1], v0)


def test_peaked_softmax_selects_matching_key():
    D = 16
    lay, vals = _single_request(15, 1, D=D, Hq=1, Hkv=1)
    # orthogonal one-hot keys, query = lambda * key j*, so weight(j*) -> 1
    K = np.zeros((16, D), dtype=np.float32)
    for j in range(16):
        K[j, j] = 1.0
    kb = W.f32_to_bf16_bits(K)
    blk = lay.block_table[0, 0]
    vals.k_cache[blk, 0, :15] = kb[:15]
    vals.k_new[0, 0] = kb[15]
    jstar = 6
    vals.q[0, 0] = W.f32_to_bf16_bits(np.float32(512.0) * K[jstar])
    kc, vc = _written(lay, vals)
    out, _, _ = oracle.attention_for(lay, kc, vc, vals.q, scale=0.25)
    vj = W.bf16_bits_to_f32(vc[blk, 0, jstar]).astype(np.float64)
    np.testing.assert_allclose(out[0, 0], vj, rtol=0, atol=1e-12)


def test_hand_worked_two_key_example():
    with open(os.path.join(GOLDEN, "two_key_example.json")) as f:
        g = json.load(f)
    q = W.f32_to_bf16_bits(np.asarray(g["q"], np.float32))
    K = W.f32_to_bf16_bits(np.asarray(g["K"], np.float32))
    V = W.f32_to_bf16_bits(np.asarray(g["V"], np.float32))
    scale = eval(g["scale_expr"], {"log": math.log})
    out, lse, err = oracle.attend_dense(q, K, V, scale)
    np.testing.assert_allclose(out, g["expected_out"], rtol=0, atol=1e-14)
    assert abs(lse - eval(g["expected_lse_expr"], {"log": math.log})) < 1e-14
    assert err < 1e-15


def test_no_keys_gives_zero_and_minus_inf():
    out, lse, _ = oracle.attend_dense(np.zeros(4, np.uint16), np.zeros((0, 4), np.uint16),
                                      np.zeros((0, 4), np.uint16), 1.0)
    assert lse == -math.inf and not out.any()


# ----------------------------------------------------------------------------
# library routine on unpaged data
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("ctx,q_len,G", [(0, 33, 1), (45, 20, 2), (16, 1, 4), (100, 7, 3)])
def test_matches_torch_sdpa_on_unpaged_arrays(ctx, q_len, G):
    import torch
    import torch.nn.functional as F

    D, Hkv = 16, 2
    lay, vals = _single_request(ctx, q_len, D=D, Hq=Hkv * G, Hkv=Hkv, seed=ctx + q_len)
    kc, vc = _written(lay, vals)
    scale = 0.37
    out, lse, _ = oracle.attention_for(lay, kc, vc, vals.q, scale=scale)
    L = ctx + q_len
    K = W.bf16_bits_to_f32(oracle.gather_kv(kc, lay.block_table[0], L)).astype(np.float64)  # [L, Hkv, D]
    V = W.bf16_bits_to_f32(oracle.gather_kv(vc, lay.block_table[0], L)).astype(np.float64)
    Q = W.bf16_bits_to_f32(vals.q).astype(np.float64)  # [q, Hq, D]
    qt = torch.from_numpy(Q).permute(1, 0, 2)            # [Hq, q, D]
    kt = torch.from_numpy(K).permute(1, 0, 2).repeat_interleave(G, dim=0)
    vt = torch.from_numpy(V).permute(1, 0, 2).repeat_interleave(G, dim=0)
    pos_q = torch.arange(ctx, L).unsqueeze(1)
    pos_k = torch.arange(L).unsqueeze(0)
    mask = pos_k <= pos_q                                 # causal against the cached context
    ref = F.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask, scale=scale)
    np.testing.assert_allclose(out, ref.permute(1, 0, 2).numpy(), rtol=0, atol=1e-12)


# ----------------------------------------------------------------------------
# invariances stated by the pages
# ----------------------------------------------------------------------------

def test_block_id_permutation_invariance():
    lay = _micro_layouts()[1]
    vals = W.make_values_numpy(lay)
    kc, vc = _written(lay, vals)
    out, lse, _ = oracle.attention_for(lay, kc, vc, vals.q)
    perm = np.random.default_rng(5).permutation(lay.num_blocks)
    lay2 = W.permute_physical_blocks(lay, perm)
    vals2 = W.permute_pool_numpy(W.StepValues(vals.q, vals.k_new, vals.v_new, kc, vc), perm)
    out2, lse2, _ = oracle.attention_for(lay2, vals2.k_cache, vals2.v_cache, vals.q)
    assert np.array_equal(out, out2) and np.array_equal(lse, lse2)


def test_prefix_shared_blocks_equal_private_copies():
    rng = np.random.default_rng(9)
    suffix = rng.integers(3, 40, size=5)
    lay = W.build_layout("share", 64 + suffix, np.ones(5, np.int32), num_q_heads=4, num_kv_heads=2,
                         head_dim=8, num_blocks=120, rng=rng, seed=9, shared_prefix_tokens=64)
    vals = W.make_values_numpy(lay)
    kc, vc = _written(lay, vals)
    out, lse, _ = oracle.attention_for(lay, kc, vc, vals.q)
    lay2, copies = W.privatize_shared_prefix(lay)
    assert len(copies) == 4 * 4
    v2 = W.copy_blocks_numpy(W.StepValues(vals.q, vals.k_new, vals.v_new, kc, vc), copies)
    out2, lse2, _ = oracle.attention_for(lay2, v2.k_cache, v2.v_cache, vals.q)
    assert np.array_equal(out, out2) and np.array_equal(lse, lse2)
    # every request really did share the physical prefix blocks
    assert (lay.block_table[:, :4] == lay.block_table[0, :4]).all()


def test_chunked_prefill_equals_one_shot_prefill():
    D, Hq, Hkv = 16, 4, 2
    n = 70
    one, vals = _single_request(0, n, D=D, Hq=Hq, Hkv=Hkv, seed=11, num_blocks=12)
    kc, vc = _written(one, vals)
    full, lfull, _ = oracle.attention_for(one, kc, vc, vals.q)
    # the same prompt in three chunks, KV written before each chunk's attention
    kc2, vc2 = vals.k_cache.copy(), vals.v_cache.copy()
    pos = 0
    rows = []
    for chunk in (17, 40, 13):
        lay = W.StepLayout("chunk", Hq, Hkv, D, one.num_blocks, np.array([chunk], np.int32),
                           np.array([pos], np.int32), one.block_table)
        sl = slice(pos, pos + chunk)
        kc2, vc2 = oracle.kv_write(vals.k_new[sl], vals.v_new[sl], lay.slot_mapping, kc2, vc2)
        o, _, _ = oracle.attention_for(lay, kc2, vc2, vals.q[sl])
        rows.append(o)
        pos += chunk
    assert np.array_equal(np.concatenate(rows), full)


def test_last_prefill_row_equals_decode_at_that_position():
    one, vals = _single_request(20, 30, seed=12)
    kc, vc = _written(one, vals)
    full, _, _ = oracle.attention_for(one, kc, vc, vals.q)
    dec = W.StepLayout("dec", one.num_q_heads, one.num_kv_heads, one.head_dim, one.num_blocks,
                       np.array([1], np.int32), np.array([49], np.int32), one.block_table)
    o, _, _ = oracle.attention_for(dec, kc, vc, vals.q[-1:])
    assert np.array_equal(o[0], full[-1])


def test_mixed_step_equals_requests_run_separately():
    lay = _micro_layouts()[4]
    vals = W.make_values_numpy(lay)
    kc, vc = _written(lay, vals)
    out, _, _ = oracle.attention_for(lay, kc, vc, vals.q)
    qsl = lay.query_start_loc
    for r in range(lay.num_seqs):
        sub = W.StepLayout("one", lay.num_q_heads, lay.num_kv_heads, lay.head_dim, lay.num_blocks,
                           lay.q_lens[r:r + 1], lay.ctx_lens[r:r + 1], lay.block_table[r:r + 1])
        o, _, _ = oracle.attention_for(sub, kc, vc, vals.q[qsl[r]:qsl[r + 1]])
        assert np.array_equal(o, out[qsl[r]:qsl[r + 1]])


def test_shuffled_request_order_permutes_rows_only():
    lay = _micro_layouts()[5]
    vals = W.make_values_numpy(lay)
    kc, vc = _written(lay, vals)
    out, _, _ = oracle.attention_for(lay, kc, vc, vals.q)
    order = np.arange(lay.num_seqs)[::-1]
    qsl = lay.query_start_loc
    rows = np.concatenate([np.arange(qsl[r], qsl[r + 1]) for r in order]).astype(np.int64)
    lay2 = W.StepLayout("rev", lay.num_q_heads, lay.num_kv_heads, lay.head_dim, lay.num_blocks,
                        lay.q_lens[order], lay.ctx_lens[order], lay.block_table[order])
    out2, _, _ = oracle.attention_for(lay2, kc, vc, vals.q[rows])
    assert np.array_equal(out2, out[rows])


def test_split_merge_reproduces_unsplit_attention():
    rng = np.random.default_rng(3)
    D, n = 32, 300
    q = W.f32_to_bf16_bits(rng.standard_normal(D).astype(np.float32) * 3)
    K = W.f32_to_bf16_bits(rng.standard_normal((n, D)).astype(np.float32))
    V = W.f32_to_bf16_bits(rng.standard_normal((n, D)).astype(np.float32))
    full, lfull, _ = oracle.attend_dense(q, K, V, 0.2)
    for cuts in ([150], [1, 2, 299], [64, 128, 192, 256], [17, 18, 100]):
        edges = [0] + cuts + [n]
        parts = [oracle.attend_dense(q, K[a:b], V[a:b], 0.2) for a, b in zip(edges[:-1], edges[1:])]
        o = np.stack([p[0] for p in parts])
        lse = np.array([p[1] for p in parts])
        m, lm = oracle.merge_states(o, lse)
        np.testing.assert_allclose(m, full, rtol=0, atol=1e-13)
        assert abs(lm - lfull) < 1e-12
    # an empty part (no keys, lse = -inf) carries no weight
    e = oracle.attend_dense(q, K[:0], V[:0], 0.2)
    m, lm = oracle.merge_states(np.stack([e[0], full]), np.array([e[1], lfull]))
    np.testing.assert_allclose(m, full, rtol=0, atol=1e-15)


# ----------------------------------------------------------------------------
# KV write, gather, slot mapping
# ----------------------------------------------------------------------------

def _brute_kv_write(k_new, v_new, slots, kc, vc):
    kc, vc = kc.copy(), vc.copy()
    for t, s in enumerate(slots):
        if s < 0:
            continue
        for h in range(kc.shape[1]):
            for d in range(kc.shape[3]):
                kc[s // 16, h, s % 16, d] = k_new[t, h, d]
                vc[s // 16, h, s % 16, d] = v_new[t, h, d]
    return kc, vc


def test_kv_write_byte_exact_and_preserves_untouched_slots():
    lay = _micro_layouts()[2]
    vals = W.make_values_numpy(lay, sentinel="pattern")
    slots = lay.slot_mapping.copy()
    slots[::3] = -1                       # padding tokens are skipped
    kc, vc = oracle.kv_write(vals.k_new, vals.v_new, slots, vals.k_cache, vals.v_cache)
    bk, bv = _brute_kv_write(vals.k_new, vals.v_new, slots, vals.k_cache, vals.v_cache)
    assert np.array_equal(kc, bk) and np.array_equal(vc, bv)
    touched = np.zeros(lay.num_blocks * 16, bool)
    touched[slots[slots >= 0]] = True
    untouched = ~touched.reshape(lay.num_blocks, 16)
    k0 = vals.k_cache.transpose(0, 2, 1, 3)[untouched]
    assert np.array_equal(kc.transpose(0, 2, 1, 3)[untouched], k0)


def test_kv_write_row_stride_reads_strided_rows():
    lay = _micro_layouts()[0]
    vals = W.make_values_numpy(lay)
    T, Hkv, D = vals.k_new.shape
    wide = np.zeros((T, Hkv * D + 24), np.uint16)
    wide[:, 8:8 + Hkv * D] = vals.k_new.reshape(T, -1)
    wide_v = np.zeros_like(wide)
    wide_v[:, 8:8 + Hkv * D] = vals.v_new.reshape(T, -1)
    a = oracle.kv_write(vals.k_new, vals.v_new, lay.slot_mapping, vals.k_cache, vals.v_cache)
    b = oracle.kv_write(wide.reshape(-1)[8:], wide_v.reshape(-1)[8:], lay.slot_mapping, vals.k_cache,
                        vals.v_cache, row_stride=Hkv * D + 24)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_slot_mapping_matches_allocator_and_round_trips_through_gather():
    for lay in _micro_layouts() + [W.workload_layout("tiny_decode")]:
        s = oracle.slot_mapping(lay.query_start_loc, lay.seq_lens, lay.block_table)
        assert np.array_equal(s, lay.slot_mapping)
        vals = W.make_values_numpy(lay)
        kc, vc = _written(lay, vals)
        qsl = lay.query_start_loc
        for r in range(lay.num_seqs):
            L, c = int(lay.seq_lens[r]), int(lay.ctx_lens[r])
            Kr = oracle.gather_kv(kc, lay.block_table[r], L)
            Vr = oracle.gather_kv(vc, lay.block_table[r], L)
            assert np.array_equal(Kr[c:], vals.k_new[qsl[r]:qsl[r + 1]])
            assert np.array_equal(Vr[c:], vals.v_new[qsl[r]:qsl[r + 1]])
            # cached context is finite data, never a sentinel
            assert not np.any(Kr[:c] == W.BF16_QNAN)


def test_gather_walks_blocks_in_table_order():
    NB, Hkv, D = 6, 2, 4
    cache = np.arange(NB * Hkv * 16 * D, dtype=np.uint16).reshape(NB, Hkv, 16, D)
    bt = np.array([4, 1, 5], np.int32)
    L = 35
    out = oracle.gather_kv(cache, bt, L)
    for j in range(L):
        assert np.array_equal(out[j], cache[bt[j // 16], :, j % 16])


# ----------------------------------------------------------------------------
# block pack / unpack (KV transfer between a prefill and a decode instance)
# ----------------------------------------------------------------------------

def _brute_pack(k_cache, v_cache, ids):
    """Pure-Python pack: entry i = the block's values in memory order, K then V."""
    NB = k_cache.shape[0]
    flat_k = k_cache.reshape(NB, -1).tolist()
    flat_v = v_cache.reshape(NB, -1).tolist()
    elems = len(flat_k[0])
    out = []
    for b in ids.tolist():
        if 0 <= b < NB:
            out.append([flat_k[b], flat_v[b]])
        else:
            out.append([[0] * elems, [0] * elems])
    return np.array(out, dtype=np.uint16).reshape(len(ids), 2, elems)


def test_kv_pack_matches_brute_force_and_the_gather():
    rng = np.random.default_rng(77)
    NB, Hkv, D = 12, 3, 8
    k = rng.integers(0, 1 << 16, size=(NB, Hkv, 16, D), dtype=np.uint16)
    v = rng.integers(0, 1 << 16, size=(NB, Hkv, 16, D), dtype=np.uint16)
    ids = np.array([7, 2, 11, 0, 5], np.int32)
    st = oracle.kv_pack(k, v, ids)
    assert np.array_equal(st, _brute_pack(k, v, ids))
    # the packed K/V of a request whose table is `ids` are its gathered tokens, block by block
    L = 16 * len(ids)
    for c, cache in ((0, k), (1, v)):
        g = oracle.gather_kv(cache, ids, L)                              # [L, Hkv, D]
        packed = st[:, c].reshape(len(ids), Hkv, 16, D).transpose(0, 2, 1, 3).reshape(L, Hkv, D)
        assert np.array_equal(packed, g)
    # ids outside the pool pack zeros
    st2 = oracle.kv_pack(k, v, np.array([3, -1, NB], np.int32))
    assert np.array_equal(st2[0], st[0] * 0 + np.stack([k[3].reshape(-1), v[3].reshape(-1)]))
    assert not st2[1:].any()


def test_kv_unpack_inverts_pack_and_touches_nothing_else():
    rng = np.random.default_rng(78)
    NB, Hkv, D = 10, 2, 8
    k = rng.integers(0, 1 << 16, size=(NB, 16, Hkv, D), dtype=np.uint16)   # any layout: whole blocks move
    v = rng.integers(0, 1 << 16, size=(NB, 16, Hkv, D), dtype=np.uint16)
    src = np.array([1, 8, 4], np.int32)
    dst = np.array([9, 0, 3], np.int32)
    st = oracle.kv_pack(k, v, src)
    fill = np.full_like(k, W.BF16_QNAN)
    k2, v2 = oracle.kv_unpack(st, dst, fill, fill)
    for a, b in zip(src, dst):
        assert np.array_equal(k2[b], k[a]) and np.array_equal(v2[b], v[a])
    others = np.setdiff1d(np.arange(NB), dst)
    assert (k2[others] == W.BF16_QNAN).all() and (v2[others] == W.BF16_QNAN).all()
    # an id outside the pool is skipped
    k3, _ = oracle.kv_unpack(st, np.array([2, -5, NB + 1], np.int32), fill, fill)
    assert np.array_equal(k3[2], k[1]) and (k3[np.arange(NB) != 2] == W.BF16_QNAN).all()


def _brute_unpack(staging, ids, k_cache, v_cache):
    """Pure-Python unpack: entry i's K and V overwrite block ids[i] when it is inside the pool."""
    NB = k_cache.shape[0]
    k2 = k_cache.reshape(NB, -1).copy()
    v2 = v_cache.reshape(NB, -1).copy()
    for i, b in enumerate(ids.tolist()):
        if 0 <= b < NB:
            k2[b] = staging[i, 0]
            v2[b] = staging[i, 1]
    return k2.reshape(k_cache.shape), v2.reshape(v_cache.shape)


if given is not None:
    @settings(max_examples=100, deadline=None, derandomize=True)
    @given(data=st.data())
    def test_data_movement_matches_brute_force_on_random_pools(data):
        # random pools, random distinct slots with padding tokens, random block lists (ids outside the
        # pool included): KV write, pack and unpack against their pure-Python restatements, bit for bit
        seed = data.draw(st.integers(0, 2 ** 31 - 1))
        rng = np.random.default_rng(seed)
        NB = data.draw(st.integers(1, 9))
        Hkv = data.draw(st.integers(1, 3))
        D = data.draw(st.sampled_from([2, 4, 8]))
        T = data.draw(st.integers(0, min(20, NB * 16)))
        kc = rng.integers(0, 1 << 16, size=(NB, Hkv, 16, D), dtype=np.uint16)
        vc = rng.integers(0, 1 << 16, size=(NB, Hkv, 16, D), dtype=np.uint16)
        kn = rng.integers(0, 1 << 16, size=(T, Hkv, D), dtype=np.uint16)
        vn = rng.integers(0, 1 << 16, size=(T, Hkv, D), dtype=np.uint16)
        slots = rng.permutation(NB * 16)[:T].astype(np.int64)
        slots[rng.random(T) < 0.25] = -1
        a = oracle.kv_write(kn, vn, slots, kc, vc)
        b = _brute_kv_write(kn, vn, slots, kc, vc)
        assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
        n = data.draw(st.integers(0, 6))
        ids = rng.integers(-2, NB + 2, size=n).astype(np.int32)
        stg = oracle.kv_pack(kc, vc, ids)
        assert np.array_equal(stg, _brute_pack(kc, vc, ids))
        dst = rng.permutation(NB + 2)[:n].astype(np.int32) - 1          # distinct, some outside the pool
        u = oracle.kv_unpack(stg, dst, kc, vc)
        w = _brute_unpack(stg, dst, kc, vc)
        assert np.array_equal(u[0], w[0]) and np.array_equal(u[1], w[1])


if given is not None:
    @settings(max_examples=100, deadline=None, derandomize=True)
    @given(data=st.data())
    def test_split_merge_identity_on_random_cuts(data):
        # any cut of the keys into parts (empty parts included, in any order), attended part by part
        # and merged, equals one pass over all keys: the identity the split-KV path relies on
        seed = data.draw(st.integers(0, 2 ** 31 - 1))
        rng = np.random.default_rng(seed)
        D = data.draw(st.sampled_from([4, 16, 64]))
        n = data.draw(st.integers(1, 200))
        qs = data.draw(st.floats(0.1, 8.0))
        scale = data.draw(st.floats(0.01, 1.0))
        q = W.f32_to_bf16_bits(rng.standard_normal(D).astype(np.float32) * np.float32(qs))
        K = W.f32_to_bf16_bits(rng.standard_normal((n, D)).astype(np.float32))
        V = W.f32_to_bf16_bits(rng.standard_normal((n, D)).astype(np.float32))
        full, lfull, _ = oracle.attend_dense(q, K, V, scale)
        k = data.draw(st.integers(0, 6))
        edges = [0] + sorted(int(x) for x in rng.integers(0, n + 1, size=k)) + [n]
        spans = list(zip(edges[:-1], edges[1:]))
        order = rng.permutation(len(spans))
        parts = [oracle.attend_dense(q, K[a:b], V[a:b], scale) for a, b in (spans[i] for i in order)]
        m, lm = oracle.merge_states(np.stack([p[0] for p in parts]), np.array([p[1] for p in parts]))
        np.testing.assert_allclose(m, full, rtol=0, atol=1e-12)
        assert abs(lm - lfull) < 1e-10
