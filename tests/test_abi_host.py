"""The C-ABI library on a machine without a GPU: it loads, exports every entry
point include/pa.h declares, and rejects bad arguments on the host before any
CUDA call (no compute is launched in these tests)."""
import ctypes
import os
import re
import subprocess

import pytest

from paged_kv_cache_461_b200 import api, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pa.h")


@pytest.fixture(scope="module")
def L():
    build.build()
    return api.lib()


def declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(pa_[a-z_0-9]+)\s*\(", text)))


def test_header_and_binding_agree():
    assert sorted(api.EXPORTED) == declared_symbols()


def test_library_exports_every_declared_symbol(L):
    out = subprocess.run(["nm", "-D", "--defined-only", api.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\s(pa_[a-z_0-9]+)$", out, flags=re.M))
    for sym in declared_symbols():
        assert sym in exported, f"{sym} declared in pa.h but not exported"
        assert getattr(L, sym) is not None


def test_library_exports_nothing_else(L):
    out = subprocess.run(["nm", "-D", "--defined-only", api.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    ours = set(re.findall(r"\s(pa_[a-z_0-9]+)$", out, flags=re.M))
    assert ours == set(declared_symbols())


def test_version_and_status_strings(L):
    assert L.pa_abi_version() == 4
    for code, name in api.STATUS_NAMES.items():
        assert L.pa_status_string(code).decode() == name


def _desc(nb=64, hkv=8, d=128, bs=16):
    return api.CacheDesc(nb, hkv, d, bs)


def test_workspace_size_rules(L):
    d = _desc()
    ws = lambda *a: L.pa_workspace_size(*a)
    base = ws(4, 4, 32, ctypes.byref(d), 1000)
    assert base > 0
    # grows (never shrinks) with every bound
    assert ws(8, 4, 32, ctypes.byref(d), 1000) >= base
    assert ws(4, 400, 32, ctypes.byref(d), 1000) >= base
    assert ws(4, 4, 32, ctypes.byref(d), 100000) >= base
    # invalid / unsupported -> 0
    assert ws(4, 4, 30, ctypes.byref(d), 1000) == 0          # Hq % Hkv != 0
    assert ws(-1, 4, 32, ctypes.byref(d), 1000) == 0
    assert ws(4, 4, 32, ctypes.byref(_desc(d=96)), 1000) == 0
    assert ws(4, 4, 32, ctypes.byref(_desc(bs=32)), 1000) == 0
    assert ws(4, 4, 3 * 8, ctypes.byref(d), 1000) == 0       # G = 3 does not divide 128
    # a split size must be a multiple of 16
    o = api.AttnOptions()
    o.kv_split_tokens = 24
    assert L.pa_workspace_size_ex(4, 4, 32, ctypes.byref(d), 1000, ctypes.byref(o)) == 0
    o.kv_split_tokens = 32
    assert L.pa_workspace_size_ex(4, 4, 32, ctypes.byref(d), 1000, ctypes.byref(o)) > base
    o.reserved[0] = 1
    assert L.pa_workspace_size_ex(4, 4, 32, ctypes.byref(d), 1000, ctypes.byref(o)) == 0
    # decode path for speculative-verify shapes: q_len * G must fit 16 packed rows
    o = api.AttnOptions()
    o.decode_max_query_len = 4                      # G = 4: 16 rows
    assert L.pa_workspace_size_ex(4, 4, 32, ctypes.byref(d), 1000, ctypes.byref(o)) > 0
    o.decode_max_query_len = 5                      # 20 rows
    assert L.pa_workspace_size_ex(4, 4, 32, ctypes.byref(d), 1000, ctypes.byref(o)) == 0
    o.decode_max_query_len = -2
    assert L.pa_workspace_size_ex(4, 4, 32, ctypes.byref(d), 1000, ctypes.byref(o)) == 0
    o.decode_max_query_len = -1                     # prefill kernel only: no split partials needed
    assert 0 < L.pa_workspace_size_ex(4, 4, 32, ctypes.byref(d), 100000, ctypes.byref(o)) < \
        L.pa_workspace_size(4, 4, 32, ctypes.byref(d), 100000)


FAKE = 1 << 40  # a non-null pointer value; never dereferenced by host validation paths below


def test_kv_write_host_validation(L):
    d = _desc()
    call = lambda *a: L.pa_kv_write(*a)
    assert call(FAKE, FAKE, 1024, FAKE, 0, FAKE, FAKE, ctypes.byref(d), None) == 0          # nothing to do
    assert call(None, FAKE, 1024, FAKE, 4, FAKE, FAKE, ctypes.byref(d), None) == 1          # null k_new
    assert call(FAKE, FAKE, 1024, None, 4, FAKE, FAKE, ctypes.byref(d), None) == 1          # null slots
    assert call(FAKE, FAKE, 1000, FAKE, 4, FAKE, FAKE, ctypes.byref(d), None) == 1          # row stride < Hkv*D
    assert call(FAKE, FAKE, 1024, FAKE, -1, FAKE, FAKE, ctypes.byref(d), None) == 1
    assert call(FAKE, FAKE, 1024, FAKE, 4, FAKE, FAKE, None, None) == 1                     # no descriptor
    assert call(FAKE, FAKE, 1024, FAKE, 4, FAKE, FAKE, ctypes.byref(_desc(d=80)), None) == 2
    assert call(FAKE, FAKE, 1024, FAKE, 4, FAKE, FAKE, ctypes.byref(_desc(bs=8)), None) == 2
    assert call(FAKE, FAKE, 1024, FAKE, 4, FAKE, FAKE, ctypes.byref(_desc(nb=1 << 30)), None) == 2


def _attn(L, **kw):
    a = dict(q=FAKE, hq=32, k=FAKE, v=FAKE, desc=_desc(), qsl=FAKE, sl=FAKE, bt=FAKE, bts=64, R=4, T=4, mq=1,
             ms=1000, scale=0.088, out=FAKE + (1 << 30), lse=None, ws=FAKE + (1 << 32), wsb=1 << 30)
    a.update(kw)
    return L.pa_attention_mixed(a["q"], a["hq"], a["k"], a["v"], ctypes.byref(a["desc"]), a["qsl"], a["sl"], a["bt"],
                                a["bts"], a["R"], a["T"], a["mq"], a["ms"], ctypes.c_float(a["scale"]), a["out"],
                                a["lse"], a["ws"], a["wsb"], None)


def test_attention_host_validation(L):
    assert _attn(L, R=0) == 0 and _attn(L, T=0) == 0       # empty step: nothing enqueued
    assert _attn(L, q=None) == 1
    assert _attn(L, bt=None) == 1
    assert _attn(L, hq=30) == 1                            # Hq % Hkv
    assert _attn(L, bts=10) == 1                           # bt_stride < ceil(max_seq_len / 16)
    assert _attn(L, R=-1) == 1
    assert _attn(L, mq=-1) == 1
    assert _attn(L, scale=float("nan")) == 1
    assert _attn(L, out=FAKE) == 1                         # out aliases q
    assert _attn(L, out=FAKE + 100) == 1                   # partial overlap
    assert _attn(L, lse=FAKE + 64) == 1                    # lse inside q
    assert _attn(L, lse=FAKE + (1 << 30) + 16) == 1        # lse inside out
    assert _attn(L, ws=FAKE - 256) == 1                    # workspace running into q
    assert _attn(L, ws=FAKE + (1 << 30)) == 1              # workspace over out
    assert _attn(L, desc=_desc(d=256)) == 2
    assert _attn(L, hq=8 * 3) == 2                         # G = 3
    assert _attn(L, q=FAKE + 2) == 2                       # q not 16-byte aligned
    assert _attn(L, wsb=16) == 3                           # workspace too small


def test_merge_and_gather_host_validation(L):
    assert L.pa_merge_attn_states(FAKE, FAKE, None, 4, 8, 3, 96, FAKE, None, None) == 2
    assert L.pa_merge_attn_states(FAKE, FAKE, None, -1, 8, 3, 128, FAKE, None, None) == 1
    assert L.pa_merge_attn_states(FAKE, FAKE, None, 0, 8, 3, 128, FAKE, None, None) == 0
    assert L.pa_merge_attn_states(None, FAKE, None, 4, 8, 3, 128, FAKE, None, None) == 1
    assert L.pa_debug_gather_kv(FAKE, ctypes.byref(_desc()), FAKE, -3, FAKE, None) == 1
    assert L.pa_debug_gather_kv(FAKE, ctypes.byref(_desc()), FAKE, 0, FAKE, None) == 0
    assert L.pa_build_slot_mapping(None, FAKE, FAKE, 4, 2, 8, FAKE, None) == 1


def test_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    monkeypatch.setattr(api, "_lib", None)
    monkeypatch.setattr(api, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="missing"):
        api.lib()


def test_cache_layout_field(L):
    d = _desc()
    assert ctypes.sizeof(api.CacheDesc) == 24          # the layout field sits in what was padding
    bad = api.CacheDesc(64, 8, 128, 16, 2)
    assert L.pa_workspace_size(4, 4, 32, ctypes.byref(bad), 1000) == 0
    assert L.pa_kv_write(FAKE, FAKE, 1024, FAKE, 4, FAKE, FAKE, ctypes.byref(bad), None) == 1
    nhd = api.CacheDesc(64, 8, 128, 16, api.LAYOUT_NHD)
    assert L.pa_workspace_size(4, 4, 32, ctypes.byref(nhd), 1000) == L.pa_workspace_size(4, 4, 32, ctypes.byref(d), 1000)


def test_pack_unpack_host_validation(L):
    d = _desc()
    big = 1 << 34                                       # far from the (fake) caches
    assert L.pa_kv_pack(FAKE, FAKE + (1 << 30), ctypes.byref(d), FAKE, 0, FAKE + big, None) == 0
    assert L.pa_kv_pack(FAKE, FAKE + (1 << 30), ctypes.byref(d), FAKE, -1, FAKE + big, None) == 1
    assert L.pa_kv_pack(None, FAKE + (1 << 30), ctypes.byref(d), FAKE, 3, FAKE + big, None) == 1
    assert L.pa_kv_pack(FAKE, FAKE + (1 << 30), ctypes.byref(d), None, 3, FAKE + big, None) == 1
    assert L.pa_kv_pack(FAKE, FAKE + (1 << 30), ctypes.byref(d), FAKE, 3, FAKE + 64, None) == 1   # staging in k_cache
    assert L.pa_kv_pack(FAKE, FAKE + (1 << 30), ctypes.byref(d), FAKE, 3, FAKE + big + 8, None) == 2
    assert L.pa_kv_pack(FAKE, FAKE + (1 << 30), ctypes.byref(_desc(d=96)), FAKE, 3, FAKE + big, None) == 2
    assert L.pa_kv_unpack(FAKE + big, FAKE, -1, FAKE, FAKE + (1 << 30), ctypes.byref(d), None) == 1
    assert L.pa_kv_unpack(FAKE + big, FAKE, 0, FAKE, FAKE + (1 << 30), ctypes.byref(d), None) == 0
    assert L.pa_kv_unpack(FAKE + (1 << 30) + 32, FAKE, 2, FAKE, FAKE + (1 << 30), ctypes.byref(d), None) == 1
    assert L.pa_kv_unpack(FAKE + big, FAKE, 2, FAKE + 2, FAKE + (1 << 30), ctypes.byref(d), None) == 2


def _fused(L, **kw):
    a = dict(q=FAKE, hq=32, kn=FAKE + (1 << 33), vn=FAKE + (1 << 33) + (1 << 28), stride=1024, k=FAKE + (1 << 31),
             v=FAKE + (1 << 31) + (1 << 29), desc=_desc(), qsl=FAKE, sl=FAKE, bt=FAKE, bts=64, R=4, T=4, mq=1,
             ms=1000, scale=0.088, out=FAKE + (1 << 30), lse=None, ws=FAKE + (1 << 32), wsb=1 << 30, opt=None)
    a.update(kw)
    return L.pa_attention_decode_fused(a["q"], a["hq"], a["kn"], a["vn"], a["stride"], a["k"], a["v"],
                                       ctypes.byref(a["desc"]), a["qsl"], a["sl"], a["bt"], a["bts"], a["R"], a["T"],
                                       a["mq"], a["ms"], ctypes.c_float(a["scale"]), a["out"], a["lse"], a["ws"],
                                       a["wsb"], a["opt"], None)


def _mixed(L, **kw):
    a = dict(q=FAKE, hq=32, k=FAKE + (1 << 31), v=FAKE + (1 << 31) + (1 << 29), desc=_desc(), qsl=FAKE, sl=FAKE,
             bt=FAKE, bts=64, R=4, T=4, mq=1, ms=1000, scale=0.088, out=FAKE + (1 << 30), lse=None,
             ws=FAKE + (1 << 32), wsb=1 << 30, opt=None, stream=None)
    a.update(kw)
    return L.pa_attention_mixed_ex(a["q"], a["hq"], a["k"], a["v"], ctypes.byref(a["desc"]), a["qsl"], a["sl"],
                                   a["bt"], a["bts"], a["R"], a["T"], a["mq"], a["ms"], ctypes.c_float(a["scale"]),
                                   a["out"], a["lse"], a["ws"], a["wsb"], a["opt"], a["stream"])


def test_side_stream_and_events_come_all_or_none(L):
    # the caller's side stream and fork/join events for a mixed step: all three or none, and the side
    # stream differs from the call's stream; the library never creates them itself
    def opts(side=None, fork=None, join=None):
        o = api.AttnOptions()
        o.side_stream, o.fork_event, o.join_event = side, fork, join
        return ctypes.byref(o)
    assert _mixed(L, opt=opts(side=FAKE)) == 1
    assert _mixed(L, opt=opts(side=FAKE, fork=FAKE + 64)) == 1
    assert _mixed(L, opt=opts(fork=FAKE + 64, join=FAKE + 128)) == 1
    assert _mixed(L, opt=opts(side=FAKE, fork=FAKE + 64, join=FAKE + 64)) == 1       # one event for both
    assert _mixed(L, opt=opts(side=FAKE, fork=FAKE + 64, join=FAKE + 128), stream=FAKE) == 1   # side == stream
    # all three given (or none): passes these checks and stops only at the (absent) driver
    assert _mixed(L, opt=opts(side=FAKE, fork=FAKE + 64, join=FAKE + 128)) in (0, 4)
    assert _mixed(L, opt=opts()) in (0, 4)
    assert ctypes.sizeof(api.AttnOptions) == 32 + 3 * ctypes.sizeof(ctypes.c_void_p)


def test_fused_decode_host_validation(L):
    assert _fused(L, R=0) == 0
    assert _fused(L, mq=3) == 2                          # G = 4: 12 rows > the default 8 decode rows
    o = api.AttnOptions()
    o.decode_max_query_len = 3
    # 12 rows allowed with the option: passes validation, then fails only at the (absent) driver
    assert _fused(L, mq=3, opt=ctypes.byref(o)) in (0, 4)
    assert _fused(L, kn=None) == 1
    assert _fused(L, stride=1000) == 1                   # < Hkv * D
    assert _fused(L, stride=1028) == 2                   # not a multiple of 8 elements
    assert _fused(L, kn=FAKE + (1 << 33) + 2) == 2       # k_new not 16-byte aligned
    assert _fused(L, hq=8 * 3) == 2


def _mixed_write(L, **kw):
    a = dict(q=FAKE, hq=32, kn=FAKE + (1 << 33), vn=FAKE + (1 << 33) + (1 << 28), stride=1024,
             slots=FAKE + (1 << 34), k=FAKE + (1 << 31), v=FAKE + (1 << 31) + (1 << 29), desc=_desc(), qsl=FAKE,
             sl=FAKE, bt=FAKE, bts=64, R=4, T=4, mq=300, ms=1000, scale=0.088, out=FAKE + (1 << 30), lse=None,
             ws=FAKE + (1 << 32), wsb=1 << 30, opt=None)
    a.update(kw)
    return L.pa_attention_mixed_write(a["q"], a["hq"], a["kn"], a["vn"], a["stride"], a["slots"], a["k"], a["v"],
                                      ctypes.byref(a["desc"]), a["qsl"], a["sl"], a["bt"], a["bts"], a["R"], a["T"],
                                      a["mq"], a["ms"], ctypes.c_float(a["scale"]), a["out"], a["lse"], a["ws"],
                                      a["wsb"], a["opt"], None)


def test_mixed_write_host_validation(L):
    # the write-and-plan entry point takes any step shape (here prefill-shaped requests), and checks
    # its write arguments before anything is enqueued
    assert _mixed_write(L, slots=None) == 1
    assert _mixed_write(L, kn=None) == 1
    assert _mixed_write(L, stride=1000) == 1             # < Hkv * D
    assert _mixed_write(L, wsb=16) == 3                  # workspace too small
    assert _mixed_write(L, R=0) == 0


def test_binding_rejects_host_tensors_before_the_library(L):
    # every GPU entry point of the binding refuses host (CPU) tensors with a TypeError: there is
    # no CPU fallback, and nothing reaches the library
    import torch
    bf = torch.bfloat16
    q = torch.zeros(4, 2, 64, dtype=bf)
    kc = torch.zeros(8, 2, 16, 64, dtype=bf)
    vc = torch.zeros_like(kc)
    kn = torch.zeros(4, 2, 64, dtype=bf)
    qsl = torch.arange(5, dtype=torch.int32)
    sl = torch.full((4,), 5, dtype=torch.int32)
    bt = torch.zeros(4, 2, dtype=torch.int32)
    slots = torch.zeros(4, dtype=torch.int64)
    ids = torch.zeros(3, dtype=torch.int32)
    calls = [
        lambda: api.kv_write(kn, kn, slots, kc, vc),
        lambda: api.build_slot_mapping(qsl, sl, bt, 4),
        lambda: api.attention_mixed(q, kc, vc, qsl, sl, bt, 1, 5),
        lambda: api.attention_mixed_noalloc(q, kc, vc, qsl, sl, bt, 1, 5),
        lambda: api.attention_decode_fused(q, kn, kn, kc, vc, qsl, sl, bt, 1, 5),
        lambda: api.kv_pack(kc, vc, ids),
        lambda: api.kv_unpack(torch.zeros(3, 2, 2048, dtype=bf), ids, kc, vc),
        lambda: api.merge_attn_states(torch.zeros(2, 2, 3, 64), torch.zeros(2, 2, 3)),
        lambda: api.debug_gather_kv(kc, bt[0], 5),
    ]
    for call in calls:
        with pytest.raises(TypeError, match="CUDA"):
            call()


def test_binding_checks_dtype_before_device(L):
    import torch
    with pytest.raises(TypeError, match="int32"):
        api._need(torch.zeros(3, dtype=torch.int64), torch.int32, "seq_lens")
    with pytest.raises(TypeError, match="bfloat16"):
        api._need(torch.zeros(3, 2, 64), torch.bfloat16, "q")
    with pytest.raises(TypeError, match="torch tensor"):
        api._need([1, 2, 3], torch.int32, "seq_lens")
    c = api.PrefixCache()
    h = api.prefix_block_hashes(list(range(32)))
    with pytest.raises(ValueError, match="block ids"):
        c.insert(h, [1])
    c.close()


def test_boundary_from_plain_c(L, tmp_path):
    # a C99 program includes pa.h, links libpa_b200.so and calls the host-only entry points;
    # its chained FNV-1a digests must equal the oracle's restatement of the same definition
    import shutil
    from oracle import prefix as P
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    libdir = os.path.dirname(build.LIB)
    exe = str(tmp_path / "abi_from_c")
    subprocess.check_call([cc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", os.path.join(ROOT, "include"),
                           os.path.join(ROOT, "tests", "abi_from_c.c"), "-o", exe, "-L", libdir, "-lpa_b200",
                           f"-Wl,-rpath,{libdir}"])
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stderr
    got = r.stdout.split()
    import numpy as np
    want = [d.hex() for d in P.block_hashes(np.arange(48, dtype=np.int32), "fnv1a64")]
    assert got == want


def test_binding_launches_only_on_the_tensors_device(monkeypatch):
    # the library launches on the current CUDA device: tensors (or a given stream) on another device
    # are refused before the call; stand-ins replace torch.cuda's device and stream queries
    import torch

    class Stream:
        def __init__(self, dev, handle):
            self.device, self.cuda_stream = dev, handle

    monkeypatch.setattr(torch.cuda, "current_device", lambda: 0)
    monkeypatch.setattr(torch.cuda, "current_stream", lambda: Stream(torch.device("cuda", 0), 1234))
    cuda0, cuda1 = torch.device("cuda", 0), torch.device("cuda", 1)
    assert api._stream(None, cuda0).value == 1234
    assert api._stream(Stream(cuda0, 99), cuda0).value == 99
    with pytest.raises(ValueError, match="current CUDA device"):
        api._stream(None, cuda1)
    with pytest.raises(ValueError, match="stream is on"):
        api._stream(Stream(cuda1, 5), cuda0)
