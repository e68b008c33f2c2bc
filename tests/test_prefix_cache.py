"""Prefix-cache hashing and the longest cached prefix (host C++ in the library)
against the plain-Python oracle in oracle/prefix.py, which is itself pinned to
published hash test vectors and to a brute-force search.  No GPU is needed."""
import json
import os
import threading

import numpy as np
import pytest

from oracle import prefix as P
from paged_kv_cache_461_b200 import api, build
from paged_kv_cache_461_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hash_vectors.json")


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    api.lib()


# ----------------------------------------------------------------------------- oracle pins

def test_oracle_hashes_match_published_vectors():
    g = json.load(open(GOLDEN))
    for msg, want in g["fnv1a64"]["vectors"]:
        assert P.fnv1a64(msg.encode()) == int(want, 16)
    import hashlib
    for msg, want in g["sha256"]["vectors"]:
        assert hashlib.sha256(msg.encode()).hexdigest() == want


def test_oracle_chaining_and_whole_blocks_only():
    rng = np.random.default_rng(1)
    toks = rng.integers(0, 128000, size=16 * 6 + 9).astype(np.int32)
    for algo in ("fnv1a64", "sha256"):
        h = P.block_hashes(toks, algo)
        assert len(h) == 6                                   # the 9 trailing tokens form no block
        assert P.block_hashes(toks[:16 * 6], algo) == h
        t2 = toks.copy()
        t2[16 * 3 + 5] += 1                                  # a change in block 3 ...
        h2 = P.block_hashes(t2, algo)
        assert h2[:3] == h[:3] and all(a != b for a, b in zip(h2[3:], h[3:]))   # ... moves blocks 3.. only
        h3 = P.block_hashes(toks, algo, root=b"\x01" + bytes(31))
        assert all(a != b for a, b in zip(h3, h))          # a different root moves every block
        # the same 16 tokens under different parents give different digests
        rep = np.tile(toks[:16], 3)
        hr = P.block_hashes(rep, algo)
        assert len(set(hr)) == 3
    # FNV digests are 8 significant bytes, zero padded
    assert all(d[8:] == bytes(24) for d in P.block_hashes(toks, "fnv1a64"))


def test_oracle_longest_hit_brute_force_definition():
    cached = {b"a": 1, b"b": 2, b"d": 4}
    assert P.longest_hit_brute(cached, [b"a", b"b", b"c", b"d"]) == [1, 2]
    assert P.longest_hit_brute(cached, [b"x", b"a"]) == []
    assert P.longest_hit_brute(cached, []) == []


# ----------------------------------------------------------------------------- library vs oracle

@pytest.mark.parametrize("algo", ["fnv1a64", "sha256"])
@pytest.mark.parametrize("n", [0, 15, 16, 17, 160, 1003])
def test_block_hashes_match_oracle(algo, n):
    rng = np.random.default_rng(n + len(algo))
    toks = rng.integers(-5, 1 << 31, size=n, dtype=np.int64).astype(np.int32)
    for root in (None, bytes(rng.integers(0, 256, 32, dtype=np.uint8))):
        lib_h = api.prefix_block_hashes(toks, algo, root)
        ref = P.block_hashes(toks, algo, root)
        assert len(lib_h) == len(ref) == n // 16
        for a, b in zip(lib_h, ref):
            assert bytes(a) == b


def test_sha256_block_digest_many_random_blocks():
    rng = np.random.default_rng(9)
    toks = rng.integers(0, 1 << 31, size=16 * 400, dtype=np.int64).astype(np.int32)
    lib_h = api.prefix_block_hashes(toks, "sha256")
    ref = P.block_hashes(toks, "sha256")
    assert [bytes(x) for x in lib_h] == ref


def test_longest_hit_matches_brute_force_under_inserts_and_removals():
    rng = np.random.default_rng(3)
    base = rng.integers(0, 32000, size=16 * 40).astype(np.int32)
    prompts = []
    for k in range(12):
        cut = int(rng.integers(0, 40)) * 16
        tail = rng.integers(0, 32000, size=int(rng.integers(0, 200))).astype(np.int32)
        prompts.append(np.concatenate([base[:cut], tail]))
    for algo in ("fnv1a64", "sha256"):
        cache = api.PrefixCache()
        ref = {}
        next_block = 0
        for i, pr in enumerate(prompts):
            h = api.prefix_block_hashes(pr, algo)
            if i % 3 != 2 and len(h):                          # some prompts are cached, some only looked up
                ids = np.arange(next_block, next_block + len(h), dtype=np.int32)
                next_block += len(h)
                cache.insert(h, ids)
                for d, b in zip((bytes(x) for x in h), ids.tolist()):
                    if d not in ref and b not in ref.values():
                        ref[d] = b
            if i == 6:                                         # recycle a few blocks
                for b in rng.choice(next_block, 5, replace=False).tolist():
                    cache.remove_block(b)
                    ref = {d: v for d, v in ref.items() if v != b}
        assert len(cache) == len(ref)
        for pr in prompts:
            h = api.prefix_block_hashes(pr, algo)
            got = cache.longest_hit(h).tolist()
            assert got == P.longest_hit_brute(ref, [bytes(x) for x in h])
        cache.close()


def test_insert_keeps_first_mapping_and_rejects_negative_ids():
    h = api.prefix_block_hashes(np.arange(48, dtype=np.int32))
    c = api.PrefixCache()
    c.insert(h[:2], [10, 11])
    c.insert(h[:3], [20, 21, 22])                             # digests 0, 1 already mapped: kept
    assert c.longest_hit(h).tolist() == [10, 11, 22]
    with pytest.raises(api.PaError):
        c.insert(h[:1], [-1])
    c.remove_block(11)
    assert c.longest_hit(h).tolist() == [10]
    assert len(c) == 2


def test_shared_prefix_workload_hits_the_shared_blocks():
    # requests that share a 2048-token prompt prefix (128 whole blocks) find the first request's
    # blocks for all of it, and nothing beyond (their suffixes differ)
    lay = W.workload_layout("prefix_sharing")
    rng = np.random.default_rng(11)
    shared = rng.integers(0, 128256, size=2048).astype(np.int32)
    cache = api.PrefixCache()
    for r in range(8):
        L = int(lay.seq_lens[r])
        toks = np.concatenate([shared, rng.integers(0, 128256, size=L - 2048).astype(np.int32)])
        h = api.prefix_block_hashes(toks)
        hit = cache.longest_hit(h)
        if r == 0:
            assert len(hit) == 0
        else:
            assert len(hit) == 128
            assert np.array_equal(hit, lay.block_table[0, :128])
            assert np.array_equal(lay.block_table[r, :128], lay.block_table[0, :128])
        nfull = L // 16
        cache.insert(h[:nfull], lay.block_table[r, :nfull])
    cache.close()


def test_concurrent_inserts_and_lookups():
    c = api.PrefixCache()
    toks = [np.random.default_rng(i).integers(0, 1000, size=16 * 50).astype(np.int32) for i in range(8)]
    hs = [api.prefix_block_hashes(t) for t in toks]

    def work(i):
        c.insert(hs[i], np.arange(i * 50, i * 50 + 50, dtype=np.int32))
        assert len(c.longest_hit(hs[i])) == 50

    th = [threading.Thread(target=work, args=(i,)) for i in range(8)]
    for t in th:
        t.start()
    for t in th:
        t.join()
    assert len(c) == 400
    c.close()


def test_prefix_hash_argument_checks():
    L = api.lib()
    import ctypes
    n = ctypes.c_int64(0)
    assert L.pa_prefix_block_hashes(None, -1, None, 0, None, ctypes.byref(n)) == 1
    assert L.pa_prefix_block_hashes(None, 5, None, 0, None, ctypes.byref(n)) == 1
    toks = np.zeros(32, np.int32)
    assert L.pa_prefix_block_hashes(toks.ctypes.data, 32, None, 7, None, ctypes.byref(n)) == 1
    assert L.pa_prefix_block_hashes(toks.ctypes.data, 15, None, 0, None, ctypes.byref(n)) == 0 and n.value == 0
    assert L.pa_prefix_cache_longest_hit(None, None, 0, None) == -1
    assert L.pa_prefix_cache_size(None) == -1


# ----------------------------------------------------------------------------- random operation sequences

from hypothesis import settings as _settings
from hypothesis import strategies as _st
from hypothesis.stateful import RuleBasedStateMachine, invariant, rule


class PrefixCacheMachine(RuleBasedStateMachine):
    """Random inserts, block removals and lookups against a plain model: a dict from digest to block
    where the first mapping of a digest wins and a block holds at most one digest."""

    def __init__(self):
        super().__init__()
        self.cache = api.PrefixCache()
        self.model = {}
        # three prompts that share prefixes of different lengths, hashed once
        base = np.arange(16 * 6, dtype=np.int32)
        self.prompts = [api.prefix_block_hashes(base),
                        api.prefix_block_hashes(np.concatenate([base[:48], base[48:] + 1000])),
                        api.prefix_block_hashes(np.concatenate([base[:16], base[16:] + 2000]))]

    def teardown(self):
        self.cache.close()

    @rule(p=_st.integers(0, 2), n=_st.integers(0, 6), first=_st.integers(0, 40))
    def insert(self, p, n, first):
        h = self.prompts[p][:n]
        ids = np.arange(first, first + len(h), dtype=np.int32)
        self.cache.insert(h, ids)
        for d, b in zip((bytes(x) for x in h), ids.tolist()):
            if d not in self.model and b not in self.model.values():
                self.model[d] = b

    @rule(b=_st.integers(0, 46))
    def remove(self, b):
        self.cache.remove_block(b)
        self.model = {d: v for d, v in self.model.items() if v != b}

    @rule(p=_st.integers(0, 2))
    def lookup(self, p):
        h = self.prompts[p]
        assert self.cache.longest_hit(h).tolist() == P.longest_hit_brute(self.model, [bytes(x) for x in h])

    @invariant()
    def same_size(self):
        assert len(self.cache) == len(self.model)


TestPrefixCacheMachine = PrefixCacheMachine.TestCase
TestPrefixCacheMachine.settings = _settings(max_examples=60, stateful_step_count=30, deadline=None,
                                            derandomize=True)
