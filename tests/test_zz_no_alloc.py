"""pa_attention_mixed_noalloc against pa_attention_mixed_ex.

The allocation-free entry point exists for callers that cannot allocate device
memory where attention runs (inside someone else's stream capture, or under a
host that owns every allocation): it takes no workspace and uses scratch
memory built into the library instead.  It must give the same results as the
entry point that takes a caller-allocated workspace -- here on two calls in a
row with different batches, so leftovers of the first call in the shared
scratch cannot leak into the second.  Both batches split long decode requests
(the split-KV partials live in the scratch) and mix in prefill chunks.

This file is collected last on purpose, and passes alone in a fresh process
as well as after the other tests.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

from paged_kv_cache_461_b200 import api, build
from paged_kv_cache_461_b200 import workloads as W
from tests.gpu_util import DevStep, assert_parity, bf16_to_f64, oracle_for_step

pytestmark = pytest.mark.gpu


def _batch(seed):
    rng = np.random.default_rng(seed)
    ctx = list(rng.integers(500, 3000, size=10)) + [0, 700]
    q = [1] * 10 + [200, 65]
    need = sum((c + k + 15) // 16 for c, k in zip(ctx, q))
    lay = W.build_layout(f"noalloc{seed}", ctx, q, num_q_heads=32, num_kv_heads=8, head_dim=128,
                         num_blocks=need + 9, seed=seed)
    return lay, W.make_values_numpy(lay)


def _noalloc_call(st, split):
    """The new entry point, called through the C ABI with raw device pointers."""
    lay = st.layout
    out = torch.full_like(st.q, float("nan"))
    lse = torch.full((lay.num_tokens, lay.num_q_heads), float("nan"), device="cuda")
    d = api.cache_desc(st.k_cache)
    o = api.AttnOptions()
    o.kv_split_tokens = split
    rc = api.lib().pa_attention_mixed_noalloc(
        st.q.data_ptr(), lay.num_q_heads, st.k_cache.data_ptr(), st.v_cache.data_ptr(), ctypes.byref(d),
        st.qsl.data_ptr(), st.seq_lens.data_ptr(), st.bt.data_ptr(), lay.bt_stride, lay.num_seqs, lay.num_tokens,
        lay.max_query_len, lay.max_seq_len, ctypes.c_float(1.0 / math.sqrt(lay.head_dim)), out.data_ptr(),
        lse.data_ptr(), ctypes.byref(o), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0, api.STATUS_NAMES.get(rc, rc)
    return out, lse


def test_noalloc_matches_workspace_entry_point_on_two_calls_in_a_row():
    assert torch.cuda.is_available()
    build.build()
    split = 256  # every decode request is split, so the partial states go through the scratch
    for seed in (31, 32):
        lay, vals = _batch(seed)
        st = DevStep(lay, vals)
        st.write()
        ref_out, ref_lse = st.attend(kv_split_tokens=split)       # caller-allocated workspace
        out, lse = _noalloc_call(st, split)                       # built-in scratch
        torch.cuda.synchronize()
        # same tolerance as every parity test, against the existing entry point ...
        assert_parity(out, bf16_to_f64(ref_out), lse, ref_lse.cpu().numpy().astype(np.float64),
                      what=f"noalloc vs workspace, call seed {seed}")
        # ... and against the oracle
        ref, oref_lse, _ = oracle_for_step(lay, vals)
        assert_parity(out, ref, lse, oref_lse, what=f"noalloc vs oracle, call seed {seed}")


def test_noalloc_rejects_bounds_beyond_its_scratch():
    build.build()
    d = api.CacheDesc(140_000, 8, 128, 16)
    need = api.lib().pa_workspace_size(4096, 4096, 64, ctypes.byref(d), 131072)
    assert need > api.NOALLOC_SCRATCH_BYTES
    rc = api.lib().pa_attention_mixed_noalloc(1 << 40, 64, 1 << 40, 1 << 40, ctypes.byref(d), 1 << 40, 1 << 40,
                                              1 << 40, 8192, 4096, 4096, 1, 131072, ctypes.c_float(0.08),
                                              (1 << 40) + (1 << 36), None, None, None)
    assert rc == 3  # PA_ERR_WORKSPACE_TOO_SMALL, nothing enqueued


def test_noalloc_status_word_is_readable():
    # the allocation-free call's device status word lives in the built-in scratch; the accessor copies
    # it out.  A block id outside the pool is read as zeros and flagged; the next clean call clears it.
    build.build()
    lay, vals = _batch(33)
    st = DevStep(lay, vals)
    st.write()
    good_bt = st.bt
    st.bt = good_bt.clone()
    st.bt[0, 0] = lay.num_blocks + 77
    _noalloc_call(st, 0)
    assert api.noalloc_device_status() & api.DEVICE_BAD_BLOCK
    st.bt = good_bt
    _noalloc_call(st, 0)
    assert api.noalloc_device_status() == 0
