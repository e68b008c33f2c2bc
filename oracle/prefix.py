"""Prefix-cache hashing and the longest cached prefix, in plain Python -- TEST
INFRASTRUCTURE ONLY (tests/ and bench.py's CPU leg may use it; the library never does).

What it follows: the scheduler hashes each request in 16-token blocks -- a
built-in hash by default, SHA-256 against collisions -- and walks the hashes in
order through the map from block hash to cached block, reusing each hit's KV
block; only whole blocks are reused (shengyayun.com 关键实现细节, items 1 and 2;
hn.213312.xyz section 二, item 2).  Reading taken where the pages are silent: a
block's digest covers its parent's digest and its own 16 token ids, so equal
digests name equal whole prefixes (the same key the library computes):
    digest(b) = H(parent (32 bytes) || tokens[16b .. 16b+15] as little-endian int32)
with parent = digest(b-1), or the root (32 zero bytes by default) for b = 0.
H is 64-bit FNV-1a (value little-endian in bytes 0..7, zero padded to 32) or
SHA-256.  FNV-1a is written out from its published definition; SHA-256 is
hashlib's.
"""
from __future__ import annotations

import hashlib
import struct

FNV64_OFFSET = 0xCBF29CE484222325
FNV64_PRIME = 0x100000001B3


def fnv1a64(data: bytes) -> int:
    """FNV-1a, 64-bit: for each byte, xor it into the state, then multiply by the FNV prime mod 2^64."""
    h = FNV64_OFFSET
    for b in data:
        h ^= b
        h = (h * FNV64_PRIME) & 0xFFFFFFFFFFFFFFFF
    return h


def block_digest(parent: bytes, tokens, algo: str) -> bytes:
    assert len(parent) == 32 and len(tokens) == 16
    msg = parent + b"".join(struct.pack("<i", int(t)) for t in tokens)
    if algo == "sha256":
        return hashlib.sha256(msg).digest()
    if algo == "fnv1a64":
        return struct.pack("<Q", fnv1a64(msg)) + bytes(24)
    raise ValueError(algo)


def block_hashes(tokens, algo: str = "fnv1a64", root: bytes | None = None) -> list:
    """Digests of the len(tokens) // 16 full blocks, each chained to the one before."""
    parent = bytes(32) if root is None else bytes(root)
    out = []
    for b in range(len(tokens) // 16):
        parent = block_digest(parent, list(tokens[16 * b:16 * b + 16]), algo)
        out.append(parent)
    return out


def longest_hit_brute(cached: dict, hashes: list) -> list:
    """Brute force: the longest k such that every one of the first k digests is cached;
    returns their cached blocks."""
    best = 0
    for k in range(len(hashes) + 1):
        if all(h in cached for h in hashes[:k]):
            best = k
    return [cached[h] for h in hashes[:best]]
