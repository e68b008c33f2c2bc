"""Source-level guards for rules the CUDA code keeps so that it can never hang or fault a shared GPU:
every open-ended loop is the one time-bounded mbarrier wait, every barrier wait goes through it, no
kernel traps or asserts, and none of the calls that are closed on the target machines appears.
Host only: the sources are read as text."""
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "paged_kv_cache_461_b200", "csrc")


def _sources():
    out = {}
    for f in sorted(os.listdir(CSRC)):
        if f.endswith((".cu", ".cuh", ".cpp", ".h")):
            with open(os.path.join(CSRC, f)) as fh:
                out[f] = fh.read()
    with open(os.path.join(ROOT, "include", "pa.h")) as fh:
        out["pa.h"] = fh.read()
    return out


def _code(text):
    """The text without comments (string literals in these sources hold no comment markers)."""
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    return re.sub(r"//[^\n]*", " ", text)


def test_the_only_open_loop_is_the_time_bounded_mbarrier_wait():
    found = []
    for f, text in _sources().items():
        if not f.endswith((".cu", ".cuh")):
            continue                                     # host C++ (terminating searches) runs no kernel
        code = _code(text)
        for m in re.finditer(r"\bfor\s*\(\s*;\s*;\s*\)|\bwhile\s*\(|\bdo\s*\{", code):
            found.append((f, code[:m.start()].count("\n") + 1))
    assert [f for f, _ in found] == ["ptx.cuh"], found
    code = _code(_sources()["ptx.cuh"])
    body = code[code.index("bool mbar_wait("):]
    body = body[:body.index("\n}\n")]
    assert "for (;;)" in body and "kWaitLimitNs" in body and "global_timer_ns()" in body
    assert re.search(r"if \(abort && \*abort\)\s*return false;", body)


def test_barrier_waits_go_through_the_bounded_helper():
    for f, text in _sources().items():
        code = _code(text)
        if f != "ptx.cuh":
            assert "mbarrier.try_wait" not in code and "mbarrier.test_wait" not in code, f
        # every wait on an mbarrier in a kernel is mbar_wait / mbar_wait_warp (bounded) or a single test
        for m in re.finditer(r"\bmbar_(\w+)\(", code):
            assert m.group(1) in ("wait", "wait_warp", "test", "try_wait", "init", "arrive", "arrive_tx",
                                  "expect_tx", "arrive_expect_tx", "fence_init"), (f, m.group(0))


def test_no_trap_assert_or_closed_call():
    closed = ["Memcpy" + "Batch", "Memcpy3D" + "Batch", "multicast" + "::cluster"]
    for f, text in _sources().items():
        code = _code(text)
        assert "__trap" not in code and "trap;" not in code, f
        if f.endswith((".cu", ".cuh")):
            assert not re.search(r"\bassert\s*\(", code), f
        for name in closed:
            assert name not in text, (f, name)
