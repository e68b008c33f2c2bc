// kv_write.cuh -- the body of the KV-cache write (scatter of a step's new K/V rows into their 16-token
// blocks through the slot mapping), shared by the KV-write kernel and the kernel that writes the step's
// rows and plans its attention in one launch.  The write follows the model-runner step restated on
// hn.213312.xyz (section 一, "前向传播"): the forward pass writes each layer's new K/V into the cache
// before attention.
#pragma once

#include <type_traits>

#include "pa_internal.cuh"

namespace pa {

// What to write and where: new rows (token t's K at k_new + t*row_stride, [Hkv, D] contiguous, the same
// for V), one slot per token (negative: padding, nothing written), and the caches with their strides
// (element (token o, head h, dim d) of block b at b*Hkv*16*D + h*head_stride + o*tok_stride + d).
struct KvWriteArgs {
    const uint16_t *k_new, *v_new;
    int64_t row_stride;
    const int64_t *slots;
    int num_tokens;
    uint16_t *k_cache, *v_cache;
    int64_t num_blocks;
    int Hkv, D, head_stride, tok_stride;
};

// One warp per token, tokens cta, cta + n_ctas, ... of warp-sized groups; lanes stride over the token's
// Hkv*D/VEC vectors of K and V.  A slot outside the pool writes nothing and calls bad_slot() from lane 0.
template <int VEC, class BadSlot>
__device__ __forceinline__ void kv_write_tokens(const KvWriteArgs &a, int64_t cta, int64_t n_ctas, BadSlot bad_slot)
{
    using Vec = typename std::conditional<VEC == 8, uint4, uint16_t>::type;
    const int lane = threadIdx.x & 31;
    const int warps_per_cta = blockDim.x >> 5;
    const int64_t n_slots = a.num_blocks * kBlockSize;
    const int vec_per_row = a.D / VEC;
    const int vec_per_tok = a.Hkv * vec_per_row;
    for (int64_t t = cta * warps_per_cta + (threadIdx.x >> 5); t < a.num_tokens; t += n_ctas * warps_per_cta) {
        const int64_t slot = a.slots[t];
        const uint16_t *ks = a.k_new + t * a.row_stride;
        const uint16_t *vs = a.v_new + t * a.row_stride;
        // Up to four vectors of K and four of V per lane: the first group is loaded before the
        // slot is known (the token's rows are always readable), so the two loads overlap.
        Vec kv[4], vv[4];
        auto load = [&](int i0) {
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int i = i0 + u * 32;
                if (i < vec_per_tok) {
                    const int h = i / vec_per_row;
                    const int e = (i - h * vec_per_row) * VEC;
                    kv[u] = *reinterpret_cast<const Vec *>(ks + (int64_t)h * a.D + e);
                    vv[u] = *reinterpret_cast<const Vec *>(vs + (int64_t)h * a.D + e);
                }
            }
        };
        load(lane);
        if (slot < 0)
            continue; // padding token: nothing is written
        if (slot >= n_slots) { // a slot outside the pool: nothing is written, the caller is told
            if (lane == 0)
                bad_slot();
            continue;
        }
        const int64_t blk = slot / kBlockSize;
        const int off = (int)(slot % kBlockSize);
        for (int i0 = lane; i0 < vec_per_tok; i0 += 4 * 32) {
            if (i0 != lane)
                load(i0);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int i = i0 + u * 32;
                if (i < vec_per_tok) {
                    const int h = i / vec_per_row;
                    const int e = (i - h * vec_per_row) * VEC;
                    const int64_t dst =
                        blk * ((int64_t)a.Hkv * kBlockSize * a.D) + h * a.head_stride + off * a.tok_stride + e;
                    *reinterpret_cast<Vec *>(a.k_cache + dst) = kv[u];
                    *reinterpret_cast<Vec *>(a.v_cache + dst) = vv[u];
                }
            }
        }
    }
}

// Strides of a cache layout (HND: head-major blocks, NHD: token-major) and whether the rows and caches
// allow 16-byte vectors.
inline KvWriteArgs kv_write_args(const void *k_new, const void *v_new, int64_t row_stride, const int64_t *slots,
                                 int num_tokens, void *k_cache, void *v_cache, int64_t num_blocks, int Hkv, int D,
                                 int nhd, bool *vec_ok)
{
    KvWriteArgs a;
    a.k_new = static_cast<const uint16_t *>(k_new);
    a.v_new = static_cast<const uint16_t *>(v_new);
    a.row_stride = row_stride;
    a.slots = slots;
    a.num_tokens = num_tokens;
    a.k_cache = static_cast<uint16_t *>(k_cache);
    a.v_cache = static_cast<uint16_t *>(v_cache);
    a.num_blocks = num_blocks;
    a.Hkv = Hkv;
    a.D = D;
    a.head_stride = nhd ? D : kBlockSize * D;
    a.tok_stride = nhd ? Hkv * D : D;
    *vec_ok = ((reinterpret_cast<uintptr_t>(k_new) | reinterpret_cast<uintptr_t>(v_new) |
                reinterpret_cast<uintptr_t>(k_cache) | reinterpret_cast<uintptr_t>(v_cache)) % 16 == 0) &&
              (row_stride % 8 == 0) && (D % 8 == 0);
    return a;
}

// CTAs of 256 threads (8 tokens in flight each) for a write of num_tokens tokens
inline int64_t kv_write_ctas(int num_tokens)
{
    int64_t blocks = ((int64_t)num_tokens + 7) / 8;
    return blocks > 148 * 16 ? 148 * 16 : (blocks < 1 ? 1 : blocks);
}

} // namespace pa
