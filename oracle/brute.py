"""Pure-Python brute force (no numpy, no C) -- TEST INFRASTRUCTURE ONLY.

A second, independent statement of the same definition as oracle.c, written
with Python lists and the math module, used to pin the C oracle on tiny inputs.
It walks the block table key by key instead of gathering first.
"""
import math
import struct


def bf16_value(bits: int) -> float:
    """Exact value of a bf16 bit pattern."""
    return struct.unpack("<f", struct.pack("<I", (int(bits) & 0xFFFF) << 16))[0]


def attention(q, k_cache, v_cache, query_start_loc, seq_lens, block_table, num_q_heads, num_kv_heads,
              head_dim, scale, block_size=16):
    """q[t][h][d], k_cache[b][g][o][d] as nested lists of bf16 bit patterns.

    Returns (out[t][h][d], lse[t][h]) as nested lists of floats.
    """
    G = num_q_heads // num_kv_heads
    T = query_start_loc[-1]
    out = [[[0.0] * head_dim for _ in range(num_q_heads)] for _ in range(T)]
    lse = [[0.0] * num_q_heads for _ in range(T)]
    for r in range(len(seq_lens)):
        q_len = query_start_loc[r + 1] - query_start_loc[r]
        ctx = seq_lens[r] - q_len
        for i in range(q_len):
            t = query_start_loc[r] + i
            pos = ctx + i
            for h in range(num_q_heads):
                g = h // G
                scores = []
                for j in range(pos + 1):
                    blk = block_table[r][j // block_size]
                    krow = k_cache[blk][g][j % block_size]
                    s = 0.0
                    for d in range(head_dim):
                        s += bf16_value(q[t][h][d]) * bf16_value(krow[d])
                    scores.append(s * scale)
                m = max(scores)
                e = [math.exp(s - m) for s in scores]
                z = sum(e)
                for j in range(pos + 1):
                    blk = block_table[r][j // block_size]
                    vrow = v_cache[blk][g][j % block_size]
                    w = e[j] / z
                    for d in range(head_dim):
                        out[t][h][d] += w * bf16_value(vrow[d])
                lse[t][h] = m + math.log(z)
    return out, lse
