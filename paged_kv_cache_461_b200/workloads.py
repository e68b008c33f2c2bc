"""Seeded synthetic workloads for one engine step over a paged KV cache.

This module only *builds inputs*: request lengths, a block allocator's
assignment of physical 16-token blocks (block tables and the per-token slot
mapping that the allocator hands out), and random bf16 values.  It holds none
of the arithmetic of the KV write or of attention, so both the fp64 oracle and
the CUDA path can consume what it produces.

Shapes follow the vLLM V1 description in "Inside vLLM: Anatomy of a
High-Throughput LLM Inference System" (restated on hn.213312.xyz, section 一,
"前向传播": positions and slot mapping are built before the forward pass, and
all sequences are flattened into one super-sequence) and the 16-token default
block size (shengyayun.com blog, 关键实现细节 1-2).

Recipe (same order every time, so a seed fixes everything):
  lengths -> block permutation -> Q -> cached K -> cached V -> new K -> new V.
Values are N(0, 1) in fp32 rounded to bf16 (round to nearest even).  Cache
slots that hold no token are filled with a bf16 quiet NaN (0x7FC0), so a kernel
that reads a slot it should not read produces NaN in its output.
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace
from typing import Optional, Sequence

import numpy as np

BLOCK_SIZE = 16
BF16_QNAN = 0x7FC0


# ----------------------------------------------------------------------------
# bf16 helpers (storage only)
# ----------------------------------------------------------------------------

def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (nearest even) and return the uint16 bit patterns.
    Works through the array in pieces so that the 64-bit temporaries stay small for multi-GB pools."""
    flat = np.ascontiguousarray(x, dtype=np.float32).reshape(-1).view(np.uint32)
    out = np.empty(flat.shape, dtype=np.uint16)
    step = 1 << 23
    for s in range(0, flat.size, step):
        u = flat[s:s + step].astype(np.uint64)
        bias = ((u >> np.uint64(16)) & np.uint64(1)) + np.uint64(0x7FFF)
        out[s:s + step] = ((u + bias) >> np.uint64(16)).astype(np.uint16)
    return out.reshape(np.shape(x))


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to fp32."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


# ----------------------------------------------------------------------------
# Step layout: lengths, block tables, slot mapping
# ----------------------------------------------------------------------------

@dataclass
class StepLayout:
    """Metadata of one mixed step (everything except the tensor values)."""

    name: str
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    num_blocks: int
    q_lens: np.ndarray            # int32 [R]   tokens of this step per request
    ctx_lens: np.ndarray          # int32 [R]   tokens already cached before this step
    block_table: np.ndarray       # int32 [R, bt_stride]; entries past the used blocks are -1
    block_size: int = BLOCK_SIZE
    shared_prefix_blocks: int = 0  # leading blocks shared by every request (prefix caching)
    seed: int = 0
    extra: dict = field(default_factory=dict)

    # derived -------------------------------------------------------------
    @property
    def num_seqs(self) -> int:
        return int(self.q_lens.shape[0])

    @property
    def seq_lens(self) -> np.ndarray:
        return (self.ctx_lens.astype(np.int64) + self.q_lens).astype(np.int32)

    @property
    def query_start_loc(self) -> np.ndarray:
        qsl = np.zeros(self.num_seqs + 1, dtype=np.int32)
        np.cumsum(self.q_lens, out=qsl[1:])
        return qsl

    @property
    def num_tokens(self) -> int:
        return int(self.q_lens.sum())

    @property
    def max_query_len(self) -> int:
        return int(self.q_lens.max()) if self.num_seqs else 0

    @property
    def max_seq_len(self) -> int:
        return int(self.seq_lens.max()) if self.num_seqs else 0

    @property
    def bt_stride(self) -> int:
        return int(self.block_table.shape[1])

    def token_slot(self, r: int, pos: int) -> int:
        """Slot the block allocator assigned to position `pos` of request `r`."""
        blk = int(self.block_table[r, pos // self.block_size])
        return blk * self.block_size + pos % self.block_size

    @property
    def slot_mapping(self) -> np.ndarray:
        """int64 [T]: the slot handed out for every token of this step."""
        out = np.empty(self.num_tokens, dtype=np.int64)
        t = 0
        for r in range(self.num_seqs):
            c, q = int(self.ctx_lens[r]), int(self.q_lens[r])
            if q == 0:
                continue
            pos = np.arange(c, c + q)
            blocks = self.block_table[r, pos // self.block_size].astype(np.int64)
            out[t:t + q] = blocks * self.block_size + pos % self.block_size
            t += q
        return out

    @property
    def ctx_slots(self) -> np.ndarray:
        """int64: every slot that holds a cached-context token (each slot once)."""
        parts = []
        shared_tok = self.shared_prefix_blocks * self.block_size
        for r in range(self.num_seqs):
            c = int(self.ctx_lens[r])
            lo = 0 if r == 0 else min(shared_tok, c)
            if lo >= c:
                continue
            pos = np.arange(lo, c)
            blocks = self.block_table[r, pos // self.block_size].astype(np.int64)
            parts.append(blocks * self.block_size + pos % self.block_size)
        if not parts:
            return np.zeros(0, dtype=np.int64)
        return np.concatenate(parts)

    def kv_bytes(self) -> int:
        """Algorithmic K+V bytes one attention pass reads (exact tokens)."""
        return int(self.seq_lens.astype(np.int64).sum()) * self.num_kv_heads * self.head_dim * 2 * 2

    def describe(self) -> dict:
        return {
            "workload": self.name,
            "num_seqs": self.num_seqs,
            "num_tokens": self.num_tokens,
            "num_q_heads": self.num_q_heads,
            "num_kv_heads": self.num_kv_heads,
            "head_dim": self.head_dim,
            "block_size": self.block_size,
            "num_blocks": self.num_blocks,
            "max_seq_len": self.max_seq_len,
            "max_query_len": self.max_query_len,
            "seed": self.seed,
        }


def _blocks_needed(seq_len: int, bs: int = BLOCK_SIZE) -> int:
    return (int(seq_len) + bs - 1) // bs


def build_layout(name: str, ctx_lens: Sequence[int], q_lens: Sequence[int], *,
                 num_q_heads: int, num_kv_heads: int, head_dim: int,
                 num_blocks: Optional[int] = None, rng: Optional[np.random.Generator] = None,
                 seed: int = 0, shuffle: bool = True, shared_prefix_tokens: int = 0,
                 bt_stride: Optional[int] = None) -> StepLayout:
    """Allocate physical blocks for every request the way a block pool would.

    Physical ids come from a random permutation of the pool (``shuffle``) so
    that neighbouring logical blocks are never neighbours in memory.  With
    ``shared_prefix_tokens`` (a multiple of 16) every request's first blocks
    point at the same physical ids, as a prefix-cache hit would arrange.
    """
    ctx = np.asarray(ctx_lens, dtype=np.int32)
    ql = np.asarray(q_lens, dtype=np.int32)
    assert ctx.shape == ql.shape
    if rng is None:
        rng = np.random.default_rng(seed)
    bs = BLOCK_SIZE
    assert shared_prefix_tokens % bs == 0
    n_shared = shared_prefix_tokens // bs
    seq = ctx.astype(np.int64) + ql
    need = np.array([_blocks_needed(s) for s in seq], dtype=np.int64)
    if n_shared:
        assert (ctx >= shared_prefix_tokens).all(), "shared prefix must be fully cached"
    total_private = int((need - n_shared).sum()) + n_shared
    if num_blocks is None:
        num_blocks = max(total_private, 1)
    assert total_private <= num_blocks, f"pool of {num_blocks} blocks too small for {total_private}"
    perm = rng.permutation(num_blocks).astype(np.int32) if shuffle else np.arange(num_blocks, dtype=np.int32)
    max_blocks = int(need.max()) if len(need) else 1
    stride = max(bt_stride or 0, max_blocks, 1)
    bt = np.full((len(seq), stride), -1, dtype=np.int32)
    off = 0
    shared_ids = perm[:n_shared]
    off = n_shared
    for r in range(len(seq)):
        n = int(need[r])
        if n_shared:
            bt[r, :n_shared] = shared_ids
            k = n - n_shared
            bt[r, n_shared:n] = perm[off:off + k]
            off += k
        else:
            bt[r, :n] = perm[off:off + n]
            off += n
    return StepLayout(name=name, num_q_heads=num_q_heads, num_kv_heads=num_kv_heads,
                      head_dim=head_dim, num_blocks=int(num_blocks), q_lens=ql, ctx_lens=ctx,
                      block_table=bt, shared_prefix_blocks=n_shared, seed=seed)


# ----------------------------------------------------------------------------
# The five workloads (tiny decode, Llama-3-8B decode, mixed 8192-token step,
# prefix sharing, long-context decode)
# ----------------------------------------------------------------------------

WORKLOAD_NAMES = (
    "tiny_decode",          # 4 requests, ctx {17,33,64,100}, 4/4 heads, D 64, 64 blocks, seed 0
    "llama3_8b_decode",     # 256 requests, ctx U[512,4096], 32/8 heads, D 128, 70k blocks
    "mixed_step_8192",      # 192 decodes + prefill chunks up to 8000 tokens, 32/8 heads, D 128
    "prefix_sharing",       # 128 decodes sharing a 2048-token prefix, 32/8 heads, D 128
    "long_context_decode",  # 16 requests, ctx U[32768,131072], 64/8 heads, D 128
)


def workload_layout(name: str, seed: Optional[int] = None) -> StepLayout:
    """Build the metadata of one of the named workloads (lengths drawn first)."""
    if name == "tiny_decode":
        seed = 0 if seed is None else seed
        rng = np.random.default_rng(seed)
        return build_layout(name, [17, 33, 64, 100], [1, 1, 1, 1], num_q_heads=4, num_kv_heads=4,
                            head_dim=64, num_blocks=64, rng=rng, seed=seed)
    if name == "llama3_8b_decode":
        seed = 2 if seed is None else seed
        rng = np.random.default_rng(seed)
        ctx = rng.integers(512, 4096, size=256, endpoint=True)
        return build_layout(name, ctx, np.ones(256, dtype=np.int32), num_q_heads=32, num_kv_heads=8,
                            head_dim=128, num_blocks=70_000, rng=rng, seed=seed)
    if name == "mixed_step_8192":
        seed = 3 if seed is None else seed
        rng = np.random.default_rng(seed)
        dec_ctx = rng.integers(256, 4096, size=192, endpoint=True)
        chunks, cached = [], []
        budget = 8000
        while budget > 0:
            n = int(rng.integers(256, 2048, endpoint=True))
            c = int(rng.integers(0, 2048, endpoint=True))
            n = min(n, budget)
            chunks.append(n)
            cached.append(c)
            budget -= n
        ctx = np.concatenate([dec_ctx, np.asarray(cached)])
        ql = np.concatenate([np.ones(192, dtype=np.int64), np.asarray(chunks)])
        lay = build_layout(name, ctx, ql, num_q_heads=32, num_kv_heads=8, head_dim=128,
                           num_blocks=70_000, rng=rng, seed=seed)
        lay.extra["num_decode"] = 192
        return lay
    if name == "prefix_sharing":
        seed = 4 if seed is None else seed
        rng = np.random.default_rng(seed)
        suffix = rng.integers(64, 1024, size=128, endpoint=True)
        ctx = 2048 + suffix
        return build_layout(name, ctx, np.ones(128, dtype=np.int32), num_q_heads=32, num_kv_heads=8,
                            head_dim=128, num_blocks=32_768, rng=rng, seed=seed,
                            shared_prefix_tokens=2048)
    if name == "long_context_decode":
        seed = 5 if seed is None else seed
        rng = np.random.default_rng(seed)
        ctx = rng.integers(32768, 131072, size=16, endpoint=True)
        return build_layout(name, ctx, np.ones(16, dtype=np.int32), num_q_heads=64, num_kv_heads=8,
                            head_dim=128, num_blocks=140_000, rng=rng, seed=seed)
    raise KeyError(name)


# ----------------------------------------------------------------------------
# Layout transforms used by invariance tests (pure relabelling / copying)
# ----------------------------------------------------------------------------

def permute_physical_blocks(layout: StepLayout, perm: np.ndarray) -> StepLayout:
    """Relabel physical block b as perm[b] (the pool content must move the same way)."""
    bt = layout.block_table.copy()
    used = bt >= 0
    bt[used] = perm[bt[used]]
    return replace(layout, block_table=bt, extra=dict(layout.extra))


def privatize_shared_prefix(layout: StepLayout):
    """Give every request its own copy of the shared prefix blocks.

    Returns (new_layout, copies) where copies is an int64 [n, 2] array of
    (source block, destination block) pairs whose content must be duplicated.
    Destination ids are taken from blocks no request uses.
    """
    n_shared = layout.shared_prefix_blocks
    assert n_shared > 0
    used = np.zeros(layout.num_blocks, dtype=bool)
    used[layout.block_table[layout.block_table >= 0]] = True
    free = np.nonzero(~used)[0]
    R = layout.num_seqs
    assert len(free) >= (R - 1) * n_shared, "pool has no room for private copies"
    bt = layout.block_table.copy()
    copies = []
    k = 0
    for r in range(1, R):
        for b in range(n_shared):
            dst = int(free[k]); k += 1
            copies.append((int(bt[r, b]), dst))
            bt[r, b] = dst
    new = replace(layout, block_table=bt, shared_prefix_blocks=0, extra=dict(layout.extra))
    return new, np.asarray(copies, dtype=np.int64).reshape(-1, 2)


# ----------------------------------------------------------------------------
# Values
# ----------------------------------------------------------------------------

@dataclass
class StepValues:
    """bf16 tensors of one step.  numpy backend: uint16 bit patterns; torch: bfloat16."""

    q: object          # [T, Hq, D]
    k_new: object      # [T, Hkv, D]
    v_new: object      # [T, Hkv, D]
    k_cache: object    # [NB, Hkv, 16, D]  cached context filled, all else sentinel
    v_cache: object    # [NB, Hkv, 16, D]


def make_values_numpy(layout: StepLayout, seed: Optional[int] = None, *, q_scale: float = 1.0,
                      v_mean: float = 0.0, sentinel: str = "nan") -> StepValues:
    """Draw all values on the host with numpy (small workloads only)."""
    seed = layout.seed if seed is None else seed
    rng = np.random.default_rng([seed, 1])
    T, Hq, Hkv, D = layout.num_tokens, layout.num_q_heads, layout.num_kv_heads, layout.head_dim
    NB, bs = layout.num_blocks, layout.block_size
    ctx_slots = layout.ctx_slots
    n = len(ctx_slots)
    q = f32_to_bf16_bits(rng.standard_normal((T, Hq, D), dtype=np.float32) * np.float32(q_scale))
    kc_vals = f32_to_bf16_bits(rng.standard_normal((n, Hkv, D), dtype=np.float32))
    vc_vals = f32_to_bf16_bits(rng.standard_normal((n, Hkv, D), dtype=np.float32) + np.float32(v_mean))
    k_new = f32_to_bf16_bits(rng.standard_normal((T, Hkv, D), dtype=np.float32))
    v_new = f32_to_bf16_bits(rng.standard_normal((T, Hkv, D), dtype=np.float32) + np.float32(v_mean))
    if sentinel == "nan":
        k_cache = np.full((NB, Hkv, bs, D), BF16_QNAN, dtype=np.uint16)
        v_cache = np.full((NB, Hkv, bs, D), BF16_QNAN, dtype=np.uint16)
    elif sentinel == "pattern":
        # distinct finite-looking pattern per element (used by byte-exact write checks)
        pat = (np.arange(NB * Hkv * bs * D, dtype=np.uint64) * np.uint64(2654435761)) >> np.uint64(7)
        k_cache = (pat & np.uint64(0x3FFF)).astype(np.uint16).reshape(NB, Hkv, bs, D)
        v_cache = ((pat >> np.uint64(14)) & np.uint64(0x3FFF)).astype(np.uint16).reshape(NB, Hkv, bs, D)
    else:
        raise ValueError(sentinel)
    if n:
        blk = ctx_slots // bs
        off = ctx_slots % bs
        k_cache[blk, :, off, :] = kc_vals
        v_cache[blk, :, off, :] = vc_vals
    return StepValues(q=q, k_new=k_new, v_new=v_new, k_cache=k_cache, v_cache=v_cache)


def make_values_torch(layout: StepLayout, device, seed: Optional[int] = None, *, q_scale: float = 1.0,
                      v_mean: float = 0.0, chunk_tokens: int = 1 << 18) -> StepValues:
    """Draw values directly in device memory with a seeded torch generator.

    Used for the full-size workloads, whose pools (up to 9 GB) are too large to
    draw on the host.  Same order of draws as the numpy backend, but a
    different generator, so the two backends give different numbers.
    """
    import torch

    seed = layout.seed if seed is None else seed
    dev = torch.device(device)
    g = torch.Generator(device=dev)
    g.manual_seed(int(seed) * 7919 + 1)
    T, Hq, Hkv, D = layout.num_tokens, layout.num_q_heads, layout.num_kv_heads, layout.head_dim
    NB, bs = layout.num_blocks, layout.block_size
    bf = torch.bfloat16

    def randn(shape, scale=1.0, mean=0.0):
        x = torch.randn(shape, generator=g, device=dev, dtype=torch.float32)
        if scale != 1.0:
            x.mul_(scale)
        if mean != 0.0:
            x.add_(mean)
        return x.to(bf)

    q = randn((T, Hq, D), scale=q_scale)
    nan = torch.tensor(BF16_QNAN, dtype=torch.int16).view(bf).item()
    k_cache = torch.full((NB, Hkv, bs, D), float("nan"), dtype=bf, device=dev)
    v_cache = torch.full((NB, Hkv, bs, D), float("nan"), dtype=bf, device=dev)
    del nan
    ctx_slots = torch.from_numpy(layout.ctx_slots).to(dev)
    n = ctx_slots.numel()
    for cache, mean in ((k_cache, 0.0), (v_cache, v_mean)):
        for s in range(0, n, chunk_tokens):
            sl = ctx_slots[s:s + chunk_tokens]
            vals = randn((sl.numel(), Hkv, D), mean=mean)
            cache[sl // bs, :, sl % bs, :] = vals
    k_new = randn((T, Hkv, D))
    v_new = randn((T, Hkv, D), mean=v_mean)
    return StepValues(q=q, k_new=k_new, v_new=v_new, k_cache=k_cache, v_cache=v_cache)


def copy_blocks_numpy(values: StepValues, copies: np.ndarray) -> StepValues:
    """Duplicate whole blocks of both pools (src -> dst), e.g. for private prefix copies."""
    kc = values.k_cache.copy()
    vc = values.v_cache.copy()
    if len(copies):
        kc[copies[:, 1]] = kc[copies[:, 0]]
        vc[copies[:, 1]] = vc[copies[:, 0]]
    return replace(values, k_cache=kc, v_cache=vc)


def permute_pool_numpy(values: StepValues, perm: np.ndarray) -> StepValues:
    """Move block b of both pools to position perm[b]."""
    kc = np.empty_like(values.k_cache)
    vc = np.empty_like(values.v_cache)
    kc[perm] = values.k_cache
    vc[perm] = values.v_cache
    return replace(values, k_cache=kc, v_cache=vc)
