"""CUDA path against the oracle for the follow-on operations: the token-major (NHD)
cache layout, KV write fused into the decode kernel, and whole-block pack/unpack.

Bit-exact where the operation is data movement (NHD write and gather, the cache
bytes the fused kernel stores, pack/unpack).  Attention over an NHD cache, and
the fused write+decode, must give outputs bit-identical to the HND / unfused
path (the kernels see the same tiles) and within the parity gate of gpu_util
against the fp64 oracle.
"""
import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_461_b200 import api, build
from paged_kv_cache_461_b200 import workloads as W
from tests.gpu_util import (DevStep, assert_parity, oracle_for_step, to_dev_bf16, to_hnd, to_host_bits, to_nhd,
                            work_counts, write_and_attend_mixed)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    build.build()
    api.lib()


def _layout(name, ctx, q, Hq, Hkv, D, seed, extra_blocks=17):
    ctx, q = np.asarray(ctx), np.asarray(q)
    need = sum((int(c) + int(k) + 15) // 16 for c, k in zip(ctx, q))
    return W.build_layout(name, ctx, q, num_q_heads=Hq, num_kv_heads=Hkv, head_dim=D, num_blocks=need + extra_blocks,
                          seed=seed)


def _bits_equal(a: torch.Tensor, b: torch.Tensor) -> bool:
    return torch.equal(a.contiguous().view(torch.int16), b.contiguous().view(torch.int16))


# ----------------------------------------------------------------------------- NHD layout

@pytest.mark.parametrize("D,Hkv,T", [(64, 4, 7), (128, 8, 300), (128, 1, 33)])
def test_nhd_kv_write_bit_exact(D, Hkv, T):
    lay = _layout("w", [5] * T, [1] * T, Hkv, Hkv, D, seed=T + D)
    vals = W.make_values_numpy(lay, sentinel="pattern")
    slots = lay.slot_mapping.copy()
    slots[1::4] = -1
    kc, vc = oracle.kv_write(vals.k_new, vals.v_new, slots, vals.k_cache, vals.v_cache)
    st = DevStep(lay, vals, kv_layout="NHD")
    api.kv_write(st.k_new, st.v_new, torch.from_numpy(slots).cuda(), st.k_cache, st.v_cache, layout="NHD")
    torch.cuda.synchronize()
    assert np.array_equal(to_host_bits(to_hnd(st.k_cache)), kc)
    assert np.array_equal(to_host_bits(to_hnd(st.v_cache)), vc)


def test_nhd_gather_bit_exact():
    lay = _layout("g", [40, 0, 77], [3, 20, 1], 8, 4, 64, seed=5)
    vals = W.make_values_numpy(lay)
    st = DevStep(lay, vals, kv_layout="NHD")
    st.write()
    kc, _ = oracle.kv_write(vals.k_new, vals.v_new, lay.slot_mapping, vals.k_cache, vals.v_cache)
    for r in range(lay.num_seqs):
        L = int(lay.seq_lens[r])
        g = api.debug_gather_kv(st.k_cache, st.bt[r], L, layout="NHD")
        assert np.array_equal(to_host_bits(g), oracle.gather_kv(kc, lay.block_table[r], L))


NHD_CASES = [
    # (D, Hq, Hkv, ctx, q, split): decode, split decode, spec-verify shapes, prefill, mixed
    (128, 32, 8, [0, 15, 16, 17, 500, 1023], [1] * 6, 0),
    (128, 32, 8, [700, 2000, 33], [1, 1, 1], 64),
    (64, 16, 4, [100, 31], [2, 2], 0),
    (128, 32, 8, [0, 33, 200, 1000], [5, 130, 300, 129], 0),
    (64, 8, 8, [0, 140, 9, 300], [200, 77, 1, 1], 0),
    (128, 8, 1, [0, 1100, 5], [1, 400, 1], 0),
]


@pytest.mark.parametrize("D,Hq,Hkv,ctx,q,split", NHD_CASES)
def test_nhd_attention_matches_oracle_and_hnd_bitwise(D, Hq, Hkv, ctx, q, split):
    lay = _layout("nhd", ctx, q, Hq, Hkv, D, seed=sum(ctx) + len(q))
    vals = W.make_values_numpy(lay)
    hnd = DevStep(lay, vals)
    hnd.write()
    out_h, lse_h = hnd.attend(kv_split_tokens=split)
    nhd = DevStep(lay, vals, kv_layout="NHD")
    nhd.write()
    out_n, lse_n = nhd.attend(kv_split_tokens=split)
    torch.cuda.synchronize()
    assert api.read_device_status(nhd.workspace) == 0
    ref, ref_lse, _ = oracle_for_step(lay, vals)
    assert_parity(out_n, ref, lse_n, ref_lse, what=f"NHD D{D} Hq{Hq} Hkv{Hkv} split{split}")
    assert _bits_equal(out_n, out_h)
    assert torch.equal(lse_n, lse_h)


# ----------------------------------------------------------------------------- fused KV write + decode

FUSED_CASES = [
    # (D, Hq, Hkv, q_len, split, decode_max_query_len, layout)
    (128, 32, 8, 1, 0, 0, "HND"), (128, 32, 8, 1, 64, 0, "HND"), (128, 32, 8, 1, 0, 0, "NHD"),
    (128, 32, 8, 4, 0, 4, "HND"), (128, 32, 8, 4, 32, 4, "NHD"), (64, 16, 4, 2, 0, 0, "HND"),
    (128, 64, 8, 1, 128, 0, "NHD"), (64, 8, 8, 8, 16, 0, "HND"), (128, 8, 1, 1, 0, 0, "HND"),
]


@pytest.mark.parametrize("D,Hq,Hkv,q_len,split,dq,kv_layout", FUSED_CASES)
def test_fused_decode_equals_write_then_attend(D, Hq, Hkv, q_len, split, dq, kv_layout):
    rng = np.random.default_rng(D + Hq + q_len + split)
    ctx = np.concatenate([rng.integers(0, 900, size=10), [0, 15, 16, 31, 1200]])
    lay = _layout("fused", ctx, np.full(len(ctx), q_len, np.int32), Hq, Hkv, D, seed=int(ctx.sum()) % 991)
    vals = W.make_values_numpy(lay, sentinel="pattern")
    # unfused reference on the GPU: separate KV write, then attention
    ref_st = DevStep(lay, vals, kv_layout=kv_layout)
    ref_st.write()
    out_u, lse_u = ref_st.attend(kv_split_tokens=split, decode_max_query_len=dq)
    # fused: one call writes and attends
    st = DevStep(lay, vals, kv_layout=kv_layout)
    out_f, lse_f = st.write_and_attend_fused(kv_split_tokens=split, decode_max_query_len=dq)
    torch.cuda.synchronize()
    assert api.read_device_status(st.workspace) == 0
    n_dec, n_pf, _ = work_counts(st.workspace)
    assert n_dec > 0 and n_pf == 0
    assert _bits_equal(out_f, out_u), "fused output differs from write-then-attend"
    assert torch.equal(lse_f, lse_u)
    # the cache bytes the kernel stored equal the oracle's KV write, every other byte untouched
    kc, vc = oracle.kv_write(vals.k_new, vals.v_new, lay.slot_mapping, vals.k_cache, vals.v_cache)
    k_dev = to_hnd(st.k_cache) if kv_layout == "NHD" else st.k_cache
    v_dev = to_hnd(st.v_cache) if kv_layout == "NHD" else st.v_cache
    assert np.array_equal(to_host_bits(k_dev), kc)
    assert np.array_equal(to_host_bits(v_dev), vc)
    ref, ref_lse, _ = oracle_for_step(lay, vals)
    assert_parity(out_f, ref, lse_f, ref_lse, what=f"fused D{D} Hq{Hq} q{q_len} split{split} {kv_layout}")


def test_fused_decode_rejects_prefill_shaped_requests():
    lay = _layout("fx", [10, 20], [1, 40], 32, 8, 128, seed=3)
    st = DevStep(lay, W.make_values_numpy(lay))
    with pytest.raises(api.PaError) as e:
        st.write_and_attend_fused()
    assert e.value.status == 2


def test_fused_decode_full_size_llama3_8b_decode():
    lay = W.workload_layout("llama3_8b_decode")
    vals = W.make_values_torch(lay, "cuda")
    k0, v0 = vals.k_cache.clone(), vals.v_cache.clone()
    st = DevStep(lay, vals)
    st.write()
    out_u, lse_u = st.attend()
    k_written = st.k_cache.clone()
    st.k_cache.copy_(k0)
    st.v_cache.copy_(v0)
    out_f, lse_f = st.write_and_attend_fused()
    torch.cuda.synchronize()
    assert api.read_device_status(st.workspace) == 0
    assert _bits_equal(out_f, out_u) and torch.equal(lse_f, lse_u)
    assert _bits_equal(st.k_cache, k_written)


# ----------------------------------------------------------------------------- KV write + plan in one launch

MIXED_WRITE_CASES = [
    # (D, Hq, Hkv, q lens of the chunks, n decodes, layout, padding tokens)
    (128, 32, 8, (300, 129, 64, 1), 24, "HND", False),
    (128, 32, 8, (257, 40), 8, "NHD", True),
    (64, 16, 4, (200, 33), 12, "HND", True),
    (128, 32, 8, (), 40, "HND", False),          # decode only
    (128, 32, 8, (500, 300), 0, "HND", False),   # prefill only
]


@pytest.mark.parametrize("D,Hq,Hkv,chunks,n_dec,kv_layout,pad", MIXED_WRITE_CASES)
def test_mixed_write_equals_write_then_attend(D, Hq, Hkv, chunks, n_dec, kv_layout, pad):
    # pa_attention_mixed_write writes the step's rows in the launch that plans the step: the cache bytes
    # equal the oracle's KV write, the outputs pa_kv_write + pa_attention_mixed_ex bit for bit
    rng = np.random.default_rng(D + Hq + n_dec + len(chunks))
    ctx = list(rng.integers(0, 1500, size=n_dec)) + [int(c) for c in rng.integers(0, 900, size=len(chunks))]
    q = [1] * n_dec + list(chunks)
    lay = _layout("mixw", ctx, q, Hq, Hkv, D, seed=int(sum(ctx)) % 977)
    vals = W.make_values_numpy(lay, sentinel="pattern")
    slots = lay.slot_mapping.copy()
    if pad:
        slots[rng.random(len(slots)) < 0.1] = -1          # padding tokens: nothing written for them
    ref_st = DevStep(lay, vals, kv_layout=kv_layout)
    ref_st.slots = torch.from_numpy(slots).cuda()
    ref_st.write()
    out_u, lse_u = ref_st.attend()
    st = DevStep(lay, vals, kv_layout=kv_layout)
    st.slots = torch.from_numpy(slots).cuda()
    out_w, lse_w = write_and_attend_mixed(st)
    torch.cuda.synchronize()
    assert api.read_device_status(st.workspace) == 0
    assert _bits_equal(out_w, out_u), "output differs from write-then-attend"
    assert torch.equal(lse_w, lse_u)
    kc, vc = oracle.kv_write(vals.k_new, vals.v_new, slots, vals.k_cache, vals.v_cache)
    k_dev = to_hnd(st.k_cache) if kv_layout == "NHD" else st.k_cache
    v_dev = to_hnd(st.v_cache) if kv_layout == "NHD" else st.v_cache
    assert np.array_equal(to_host_bits(k_dev), kc)
    assert np.array_equal(to_host_bits(v_dev), vc)
    if not pad:
        ref, ref_lse, _ = oracle_for_step(lay, vals)
        assert_parity(out_w, ref, lse_w, ref_lse, what=f"mixed write D{D} {kv_layout} chunks{chunks}")


def test_mixed_write_reports_slots_outside_the_pool():
    lay = _layout("mixwb", [100, 200, 0], [1, 1, 90], 32, 8, 128, seed=5)
    vals = W.make_values_numpy(lay, sentinel="pattern")
    st = DevStep(lay, vals)
    slots = lay.slot_mapping.copy()
    slots[1] = lay.num_blocks * 16 + 5                    # outside the pool: not written, reported
    st.slots = torch.from_numpy(slots).cuda()
    for _ in range(3):                                    # the bit belongs to each call, set again each time
        write_and_attend_mixed(st)
        torch.cuda.synchronize()
        assert api.read_device_status(st.workspace) & api.DEVICE_BAD_SLOT
    ok = lay.slot_mapping.copy()
    st.slots = torch.from_numpy(ok).cuda()
    write_and_attend_mixed(st)                            # a clean call clears it
    torch.cuda.synchronize()
    assert api.read_device_status(st.workspace) == 0
    kc, _ = oracle.kv_write(vals.k_new, vals.v_new, ok, vals.k_cache, vals.v_cache)
    assert np.array_equal(to_host_bits(st.k_cache), kc)


def test_mixed_write_full_size_mixed_step_8192():
    lay = W.workload_layout("mixed_step_8192")
    vals = W.make_values_torch(lay, "cuda")
    k0, v0 = vals.k_cache.clone(), vals.v_cache.clone()
    st = DevStep(lay, vals)
    st.write()
    out_u, lse_u = st.attend()
    k_written, v_written = st.k_cache.clone(), st.v_cache.clone()
    st.k_cache.copy_(k0)
    st.v_cache.copy_(v0)
    out_w, lse_w = write_and_attend_mixed(st)
    torch.cuda.synchronize()
    assert api.read_device_status(st.workspace) == 0
    assert _bits_equal(out_w, out_u) and torch.equal(lse_w, lse_u)
    assert _bits_equal(st.k_cache, k_written) and _bits_equal(st.v_cache, v_written)


# ----------------------------------------------------------------------------- block pack / unpack

@pytest.mark.parametrize("D,Hkv,kv_layout", [(128, 8, "HND"), (64, 2, "NHD"), (128, 1, "HND")])
def test_pack_unpack_bit_exact(D, Hkv, kv_layout):
    rng = np.random.default_rng(D + Hkv)
    NB = 300
    k = rng.integers(0, 1 << 16, size=(NB, Hkv, 16, D), dtype=np.uint16)
    v = rng.integers(0, 1 << 16, size=(NB, Hkv, 16, D), dtype=np.uint16)
    if kv_layout == "NHD":
        k, v = k.transpose(0, 2, 1, 3).copy(), v.transpose(0, 2, 1, 3).copy()
    ids = rng.permutation(NB)[:120].astype(np.int32)
    ids[7] = -1
    ids[50] = NB + 3                                   # outside the pool: zeros
    kd, vd = to_dev_bf16(k), to_dev_bf16(v)
    ids_d = torch.from_numpy(ids).cuda()
    st = api.kv_pack(kd, vd, ids_d, layout=kv_layout)
    torch.cuda.synchronize()
    st_ref = oracle.kv_pack(k, v, ids)
    assert np.array_equal(to_host_bits(st), st_ref)
    # unpack into other blocks of a sentinel pool
    dst = rng.permutation(NB)[:120].astype(np.int32)
    dst[3] = -2
    fill_k = torch.full_like(kd, float("nan"))
    fill_v = torch.full_like(vd, float("nan"))
    sentinel = to_host_bits(fill_k)
    api.kv_unpack(st, torch.from_numpy(dst).cuda(), fill_k, fill_v, layout=kv_layout)
    torch.cuda.synchronize()
    rk, rv = oracle.kv_unpack(st_ref, dst, sentinel, sentinel)
    assert np.array_equal(to_host_bits(fill_k), rk)
    assert np.array_equal(to_host_bits(fill_v), rv)


def test_pack_full_size_request_blocks_sampled():
    lay = W.workload_layout("llama3_8b_decode")
    vals = W.make_values_torch(lay, "cuda")
    nblk = (lay.seq_lens + 15) // 16
    ids = np.concatenate([lay.block_table[r, :n] for r, n in enumerate(nblk)]).astype(np.int32)
    ids_d = torch.from_numpy(ids).cuda()
    st = api.kv_pack(vals.k_cache, vals.v_cache, ids_d)
    torch.cuda.synchronize()
    rng = np.random.default_rng(4)
    for i in list(rng.choice(len(ids), 64, replace=False)) + [0, len(ids) - 1]:
        b = int(ids[i])
        assert _bits_equal(st[i, 0], vals.k_cache[b].reshape(-1))
        assert _bits_equal(st[i, 1], vals.v_cache[b].reshape(-1))
    # round trip into a fresh pool restores the blocks
    k2 = torch.zeros_like(vals.k_cache)
    v2 = torch.zeros_like(vals.v_cache)
    api.kv_unpack(st, ids_d, k2, v2)
    torch.cuda.synchronize()
    assert _bits_equal(k2[ids_d.long()], vals.k_cache[ids_d.long()])
    assert _bits_equal(v2[ids_d.long()], vals.v_cache[ids_d.long()])


# ----------------------------------------------------------------------------- CUDA graph capture

@pytest.mark.parametrize("kind", ["mixed", "decode"])
def test_step_replays_from_a_cuda_graph_bit_identically(kind):
    # a mixed step forks prefill onto the library's side stream and joins it back: the whole call
    # must still capture into one graph and replay to the same bits as the eager call
    rng = np.random.default_rng(31)
    if kind == "mixed":
        ctx = list(rng.integers(0, 2000, size=20)) + [0, 700, 1500]
        q = [1] * 20 + [300, 129, 64]
    else:
        ctx, q = list(rng.integers(0, 3000, size=40)), [1] * 40
    lay = _layout("graph", ctx, q, 32, 8, 128, seed=17)
    st = DevStep(lay, W.make_values_numpy(lay))
    st.write()
    cap = torch.cuda.Stream()
    with torch.cuda.stream(cap):                     # eager call on the capture stream first: the binding
        out_e, lse_e = st.attend()                   # makes that stream's side stream and events here
    torch.cuda.synchronize()
    out_g = torch.full_like(out_e, float("nan"))
    lse_g = torch.full_like(lse_e, float("nan"))
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=cap):
        api.attention_mixed(st.q, st.k_cache, st.v_cache, st.qsl, st.seq_lens, st.bt, lay.max_query_len,
                            lay.max_seq_len, out=out_g, lse=lse_g, workspace=st.workspace)
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    assert _bits_equal(out_g, out_e) and torch.equal(lse_g, lse_e)
    assert api.read_device_status(st.workspace) == 0


@pytest.mark.parametrize("bad_slot", [False, True])
def test_mixed_write_replays_from_a_cuda_graph(bad_slot):
    # the write-and-plan launch keeps its call id in a graph: every replay must still clear the status word
    # before its writers report a slot outside the pool, and replay to the eager call's bits
    rng = np.random.default_rng(43)
    ctx = list(rng.integers(0, 2000, size=24)) + [0, 900]
    q = [1] * 24 + [260, 97]
    lay = _layout("graphw", ctx, q, 32, 8, 128, seed=23)
    vals = W.make_values_numpy(lay, sentinel="pattern")
    st = DevStep(lay, vals)
    slots = lay.slot_mapping.copy()
    if bad_slot:
        slots[3] = lay.num_blocks * 16 + 7                # a decode token's slot outside the pool
        slots[30] = lay.num_blocks * 16 + 100             # and a prefill token's
    st.slots = torch.from_numpy(slots).cuda()
    want = api.DEVICE_BAD_SLOT if bad_slot else 0
    cap = torch.cuda.Stream()
    with torch.cuda.stream(cap):                     # eager call on the capture stream first (side stream)
        out_e, lse_e = write_and_attend_mixed(st)
    torch.cuda.synchronize()
    assert api.read_device_status(st.workspace) == want
    out_g = torch.full_like(out_e, float("nan"))
    lse_g = torch.full_like(lse_e, float("nan"))
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=cap):
        api.attention_mixed_write(st.q, st.k_new, st.v_new, st.slots, st.k_cache, st.v_cache, st.qsl,
                                  st.seq_lens, st.bt, lay.max_query_len, lay.max_seq_len, out=out_g, lse=lse_g,
                                  workspace=st.workspace)
    for _ in range(4):
        st.workspace[:4].fill_(0xA5)                 # a stale status word: each replay clears it first
        g.replay()
        torch.cuda.synchronize()
        assert api.read_device_status(st.workspace) == want
        assert _bits_equal(out_g, out_e) and torch.equal(lse_g, lse_e)
    written = np.where(slots < lay.num_blocks * 16, slots, -1)  # a slot outside the pool writes nothing
    kc, vc = oracle.kv_write(vals.k_new, vals.v_new, written, vals.k_cache, vals.v_cache)
    assert np.array_equal(to_host_bits(st.k_cache), kc)
    assert np.array_equal(to_host_bits(st.v_cache), vc)


@pytest.mark.parametrize("mode", ["fused_decode", "prefill_only"])
def test_other_entry_points_replay_from_a_cuda_graph(mode):
    rng = np.random.default_rng(41)
    if mode == "fused_decode":
        ctx, q = list(rng.integers(0, 2500, size=30)), [1] * 30
    else:
        ctx, q = [0, 300, 1200], [400, 129, 77]
    lay = _layout("graph2", ctx, q, 32, 8, 128, seed=19)
    vals = W.make_values_numpy(lay, sentinel="pattern")
    st = DevStep(lay, vals)
    if mode == "fused_decode":
        out_e, lse_e = st.write_and_attend_fused()
        call = lambda o, l: api.attention_decode_fused(st.q, st.k_new, st.v_new, st.k_cache, st.v_cache, st.qsl,
                                                       st.seq_lens, st.bt, lay.max_query_len, lay.max_seq_len,
                                                       out=o, lse=l, workspace=st.workspace)
    else:
        st.write()
        out_e, lse_e = st.attend(decode_max_query_len=-1)
        call = lambda o, l: api.attention_mixed(st.q, st.k_cache, st.v_cache, st.qsl, st.seq_lens, st.bt,
                                                lay.max_query_len, lay.max_seq_len, out=o, lse=l,
                                                workspace=st.workspace, decode_max_query_len=-1)
    torch.cuda.synchronize()
    out_g = torch.full_like(out_e, float("nan"))
    lse_g = torch.full_like(lse_e, float("nan"))
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        call(out_g, lse_g)
    g.replay()
    torch.cuda.synchronize()
    assert _bits_equal(out_g, out_e) and torch.equal(lse_g, lse_e)
    assert api.read_device_status(st.workspace) == 0


# ----------------------------------------------------------------------------- binding argument checks

def test_binding_rejects_malformed_tensors_before_launching():
    # The C ABI sees pointers only; the binding checks dtype, device, contiguity and shapes first.
    lay = _layout("args", [17, 40, 3], [1, 1, 1], 8, 2, 128, seed=41)
    st = DevStep(lay, W.make_values_numpy(lay))
    st.write()
    T, Hq = lay.num_tokens, lay.num_q_heads

    def attend(**kw):
        a = dict(q=st.q, k_cache=st.k_cache, v_cache=st.v_cache, query_start_loc=st.qsl, seq_lens=st.seq_lens,
                 block_table=st.bt, max_query_len=lay.max_query_len, max_seq_len=lay.max_seq_len)
        a.update(kw)
        return api.attention_mixed(**a)

    with pytest.raises(TypeError, match="int32"):
        attend(seq_lens=st.seq_lens.long())
    with pytest.raises(TypeError, match="CUDA"):
        attend(query_start_loc=st.qsl.cpu())
    with pytest.raises(ValueError, match="contiguous"):
        attend(q=st.q.transpose(0, 1).contiguous().transpose(0, 1))
    with pytest.raises(ValueError, match="shape"):
        attend(lse=torch.empty(T, Hq + 1, device="cuda"))
    with pytest.raises(ValueError, match="block_table"):
        attend(block_table=st.bt[:-1])
    with pytest.raises(ValueError, match="v_cache"):
        attend(v_cache=st.v_cache[:-1])
    with pytest.raises(ValueError, match="slot_mapping"):
        api.kv_write(st.k_new, st.v_new, st.slots[:-1], st.k_cache, st.v_cache)
    with pytest.raises(TypeError, match="float32"):
        api.merge_attn_states(torch.zeros(2, 2, 3, 128, device="cuda"), torch.zeros(2, 2, 3, device="cuda"),
                              lse_out=torch.zeros(2, 2, device="cuda", dtype=torch.float64))
    # a block table wider than needed, as a column slice of a wider one, is still accepted
    wide = torch.full((lay.num_seqs, st.bt.shape[1] + 5), -1, dtype=torch.int32, device="cuda")
    wide[:, :st.bt.shape[1]] = st.bt
    got = attend(block_table=wide[:, :st.bt.shape[1]])
    ref = attend()
    torch.cuda.synchronize()
    assert _bits_equal(got, ref)
