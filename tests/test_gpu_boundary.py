"""The C ABI's promises about resources and bad metadata, on the GPU.

* The library creates no stream or event: a mixed step runs its prefill kernel beside its decode
  kernel on the side stream and fork/join events the caller passes in the options (the binding
  keeps one set per caller stream).  Two callers on two streams, each with its own workspace, get
  oracle-exact results; without a side stream the two kernels run one after the other on the
  caller's stream and give bit-identical outputs.
* Device metadata the host cannot check never makes a kernel read or write outside the host-sized
  buffers: requests whose query rows overlap (a query_start_loc that goes back) ask for more work
  items than the workspace holds, and the plan keeps what fits and flags the step; a request longer
  than the host's max_query_len is skipped and flagged rather than left unwritten.
* pa_kv_write_ex reports a slot outside the pool through its status word.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_461_b200 import api, build
from paged_kv_cache_461_b200 import workloads as W
from tests.gpu_util import DevStep, assert_parity, oracle_for_step, to_dev_bf16, to_host_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    build.build()
    api.lib()


def _mixed(seed, n_dec=24):
    rng = np.random.default_rng(seed)
    ctx = list(rng.integers(30, 1500, size=n_dec)) + [0, 300, 1100]
    q = [1] * n_dec + [400, 250, 90]
    need = sum((int(c) + int(k) + 15) // 16 for c, k in zip(ctx, q))
    return W.build_layout(f"boundary{seed}", ctx, q, num_q_heads=32, num_kv_heads=8, head_dim=128,
                          num_blocks=need + 11, seed=seed)


def test_two_caller_streams_with_their_own_workspaces_match_the_oracle():
    lays = [_mixed(41), _mixed(42)]
    vals = [W.make_values_numpy(x) for x in lays]
    steps = [DevStep(x, v) for x, v in zip(lays, vals)]
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    outs, lses, wss = [], [], []
    for st, s in zip(steps, streams):
        lay = st.layout
        wss.append(api.alloc_workspace(lay.num_seqs, lay.num_tokens, lay.num_q_heads, st.k_cache, lay.max_seq_len))
        outs.append(torch.full_like(st.q, float("nan")))
        lses.append(torch.full((lay.num_tokens, lay.num_q_heads), float("nan"), device="cuda"))
    torch.cuda.synchronize()
    # both steps in flight at once, each on its own caller stream (each gets its own side stream)
    for st, s, out, lse, ws in zip(steps, streams, outs, lses, wss):
        with torch.cuda.stream(s):
            st.write()
            lay = st.layout
            api.attention_mixed(st.q, st.k_cache, st.v_cache, st.qsl, st.seq_lens, st.bt, lay.max_query_len,
                                lay.max_seq_len, out=out, lse=lse, workspace=ws)
    torch.cuda.synchronize()
    for st, v, out, lse, ws in zip(steps, vals, outs, lses, wss):
        ref, ref_lse, _ = oracle_for_step(st.layout, v)
        assert_parity(out, ref, lse, ref_lse, what=f"caller stream, {st.layout.name}")
        assert api.read_device_status(ws) == 0
    assert len({(k[0], k[1]) for k in api._SIDE}) >= 2     # one side stream per caller stream


def test_serial_step_without_a_side_stream_is_bit_identical():
    lay = _mixed(43)
    st = DevStep(lay, W.make_values_numpy(lay))
    st.write()
    ws = api.alloc_workspace(lay.num_seqs, lay.num_tokens, lay.num_q_heads, st.k_cache, lay.max_seq_len)
    side = torch.empty_like(st.q)
    serial = torch.empty_like(st.q)
    api.attention_mixed(st.q, st.k_cache, st.v_cache, st.qsl, st.seq_lens, st.bt, lay.max_query_len,
                        lay.max_seq_len, out=side, workspace=ws)
    pf_split = ws[16:20].view(torch.int32).item()
    api.attention_mixed(st.q, st.k_cache, st.v_cache, st.qsl, st.seq_lens, st.bt, lay.max_query_len,
                        lay.max_seq_len, out=serial, workspace=ws, concurrent=False)
    pf_serial = ws[16:20].view(torch.int32).item()
    torch.cuda.synchronize()
    assert torch.equal(side.view(torch.int16), serial.view(torch.int16))
    # beside decode the plan keeps part of the SMs for it; alone, prefill may take them all
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert pf_split < sms and pf_serial >= pf_split


def test_overlapping_query_rows_stay_inside_the_workspace():
    # query_start_loc = [0, T, 0, T, ...]: every even request owns rows [0, T), every odd one has a
    # negative length.  The good requests together ask for more prefill work items than the host-sized
    # list holds; the plan must keep to the list, flag the step, and never touch the bytes after it.
    T, R = 512, 8
    lay = W.build_layout("overlap", [0] * R, [T // R] * R, num_q_heads=32, num_kv_heads=8, head_dim=128,
                         num_blocks=80, seed=44)
    st = DevStep(lay, W.make_values_numpy(lay))
    st.write()
    qsl = torch.tensor([0 if i % 2 == 0 else T for i in range(R + 1)], dtype=torch.int32, device="cuda")
    seq_lens = torch.full((R,), T, dtype=torch.int32, device="cuda")
    bt = torch.zeros((R, (T + 15) // 16), dtype=torch.int32, device="cuda")
    bt[:] = torch.arange(bt.shape[1], dtype=torch.int32, device="cuda")
    d = api.cache_desc(st.k_cache)
    need = api.lib().pa_workspace_size(R, T, 32, ctypes.byref(d), T)
    assert need > 0
    tail = 1 << 16
    buf = torch.full((need + tail,), 0xAB, dtype=torch.uint8, device="cuda")
    out = torch.zeros((T, 32, 128), dtype=torch.bfloat16, device="cuda")
    rc = api.lib().pa_attention_mixed(
        st.q.data_ptr(), 32, st.k_cache.data_ptr(), st.v_cache.data_ptr(), ctypes.byref(d), qsl.data_ptr(),
        seq_lens.data_ptr(), bt.data_ptr(), bt.shape[1], R, T, T, T, ctypes.c_float(1 / math.sqrt(128)),
        out.data_ptr(), None, buf.data_ptr(), need, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0
    torch.cuda.synchronize()
    assert bool((buf[need:] == 0xAB).all()), "bytes past the workspace were written"
    assert api.read_device_status(buf) & api.DEVICE_BAD_SEQ


def test_request_longer_than_max_query_len_is_skipped_and_flagged():
    # the host says every request is decode-shaped (max_query_len 1, so no prefill kernel runs); one
    # device-side request has 3 query tokens.  It must be skipped and flagged, the others computed.
    ctx = [40, 300, 77, 500]
    q = [1, 3, 1, 1]
    lay = W.build_layout("qlong", ctx, q, num_q_heads=32, num_kv_heads=8, head_dim=128, num_blocks=80, seed=45)
    vals = W.make_values_numpy(lay)
    st = DevStep(lay, vals)
    st.write()
    out = torch.full_like(st.q, float("nan"))
    ws = api.alloc_workspace(lay.num_seqs, lay.num_tokens, lay.num_q_heads, st.k_cache, lay.max_seq_len)
    api.attention_mixed(st.q, st.k_cache, st.v_cache, st.qsl, st.seq_lens, st.bt, 1, lay.max_seq_len, out=out,
                        workspace=ws)
    torch.cuda.synchronize()
    assert api.read_device_status(ws) & api.DEVICE_BAD_SEQ
    qsl = lay.query_start_loc
    assert torch.isnan(out[qsl[1]:qsl[2]].float()).all()                    # untouched
    rows = np.concatenate([np.arange(qsl[r], qsl[r + 1]) for r in (0, 2, 3)])
    ref, _, _ = oracle_for_step(lay, vals, token_list=rows.astype(np.int32))
    assert_parity(out, ref, rows=rows, what="requests beside the skipped one")


def test_kv_write_ex_reports_slots_outside_the_pool():
    T = 64
    rng = np.random.default_rng(46)
    lay = W.build_layout("slots", rng.integers(0, 60, size=T), np.ones(T, np.int32), num_q_heads=8,
                         num_kv_heads=8, head_dim=128, num_blocks=T * 5, seed=46)
    vals = W.make_values_numpy(lay, sentinel="pattern")
    slots = lay.slot_mapping.copy()
    pool_slots = lay.num_blocks * 16
    slots[5] = pool_slots            # the first slot past the pool
    slots[17] = pool_slots + 12345
    slots[30] = -1                   # padding, skipped without a report
    kc, vc = to_dev_bf16(vals.k_cache), to_dev_bf16(vals.v_cache)
    kn, vn = to_dev_bf16(vals.k_new), to_dev_bf16(vals.v_new)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    api.kv_write(kn, vn, torch.from_numpy(slots).cuda(), kc, vc, status=status)
    torch.cuda.synchronize()
    assert status.item() == api.DEVICE_BAD_SLOT
    # a slot outside the pool is skipped like a padding slot (the oracle takes only slots inside the pool)
    skipped = np.where((slots >= 0) & (slots < pool_slots), slots, -1)
    ek, ev = oracle.kv_write(vals.k_new, vals.v_new, skipped, vals.k_cache, vals.v_cache)
    assert np.array_equal(to_host_bits(kc), ek) and np.array_equal(to_host_bits(vc), ev)
    # good slots only: nothing reported
    status.zero_()
    good = slots.copy()
    good[[5, 17]] = -1
    api.kv_write(kn, vn, torch.from_numpy(good).cuda(), kc, vc, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
