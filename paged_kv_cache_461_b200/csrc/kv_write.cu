// kv_write.cu -- the KV-cache write (scatter of this step's K/V rows into their
// 16-token blocks through the slot mapping), the slot-mapping builder, the
// debug gather and the whole-block pack / unpack to a staging buffer.  All are
// pure data movement, bound by HBM bandwidth: each warp moves whole (token,
// head) rows with 16-byte vector accesses, so every load and store is a full
// 32-byte sector run.
//
// Inside a block the element (token o, kv head h, dim d) sits at
// h*head_stride + o*tok_stride + d: HND (head-major) has head_stride = 16*D,
// tok_stride = D; NHD (token-major) has head_stride = D, tok_stride = Hkv*D.
//
// Semantics follow the model-runner step restated on hn.213312.xyz (section 一,
// "前向传播"): prepare-inputs builds positions and the slot mapping, then the
// forward pass writes each layer's new K/V into the cache before attention.
#include <type_traits>

#include "kv_write.cuh"
#include "pa_internal.cuh"

namespace pa {
namespace {

// One warp per token (kv_write.cuh); a slot outside the pool sets PA_DEVICE_BAD_SLOT in *status.
template <int VEC>
__global__ void __launch_bounds__(256) kv_write_kernel(const KvWriteArgs a, uint32_t *status)
{
    kv_write_tokens<VEC>(a, blockIdx.x, gridDim.x, [&]() {
        if (status != nullptr)
            atomicOr(status, PA_DEVICE_BAD_SLOT);
    });
}

// One CTA per request; threads stride over its query rows.
__global__ void slot_mapping_kernel(const int32_t *__restrict__ qsl, const int32_t *__restrict__ seq_lens,
                                    const int32_t *__restrict__ bt, int bt_stride, int num_tokens,
                                    int64_t *__restrict__ slots)
{
    const int r = blockIdx.x;
    const int qs = qsl[r], qe = qsl[r + 1];
    const int q_len = qe - qs;
    const int L = seq_lens[r];
    const int ctx = L - q_len;
    if (qs < 0 || qe > num_tokens || q_len <= 0)
        return;
    for (int i = threadIdx.x; i < q_len; i += blockDim.x) {
        const int64_t p = (int64_t)ctx + i;
        int64_t s = -1;
        if (ctx >= 0 && p / kBlockSize < bt_stride)
            s = (int64_t)bt[(int64_t)r * bt_stride + p / kBlockSize] * kBlockSize + p % kBlockSize;
        slots[qs + i] = s;
    }
}

// One warp per token of the request: copy its Hkv rows into out[j].
__global__ void gather_kernel(const uint16_t *__restrict__ cache, int64_t num_blocks, int Hkv, int D,
                              int head_stride, int tok_stride, const int32_t *__restrict__ bt_row, int seq_len,
                              uint16_t *__restrict__ out)
{
    const int lane = threadIdx.x & 31;
    const int j = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (j >= seq_len)
        return;
    const int64_t blk = bt_row[j / kBlockSize];
    const bool ok = blk >= 0 && blk < num_blocks;
    const int off = j % kBlockSize;
    const int n = Hkv * D;
    for (int i = lane; i < n; i += 32) {
        const int h = i / D, d = i - h * D;
        uint16_t v = 0;
        if (ok)
            v = cache[blk * ((int64_t)Hkv * kBlockSize * D) + h * head_stride + off * tok_stride + d];
        out[(int64_t)j * n + i] = v;
    }
}

// Whole-block copies between the caches and a staging buffer [num_ids][2][bv] of 16-byte
// vectors (bv vectors per block).  One unit = (entry i, cache kv) = staging row 2i+kv; CTAs
// stride over units and each CTA's threads over the unit's vectors, eight in flight per
// thread.  PACK: cache -> staging (an id outside the pool gives zeros); otherwise
// staging -> cache (an id outside the pool is skipped).
// Resident copy CTAs per SM: 4 x 256 threads x 8 vectors of 16 bytes = 128 KB of loads in flight per SM.
// Measured on B200 over 9,000 to 37,555 blocks: 6.26-6.53 TB/s read + written at 4 CTAs per SM against
// 5.80-6.05 at 3, 6 or 8 (more bytes in flight are not faster here; a plain contiguous copy of the same bytes
// runs at 6.66 TB/s).
constexpr int kCopyCtasPerSm = 4;

template <bool PACK>
__global__ void __launch_bounds__(256) kv_block_copy_kernel(uint4 *__restrict__ k_cache, uint4 *__restrict__ v_cache,
                                                            int64_t num_blocks, int bv,
                                                            const int32_t *__restrict__ ids, int64_t n_units,
                                                            uint4 *__restrict__ staging)
{
    constexpr int kU = 8;
    // the next unit's block id is loaded while this unit is copied
    int64_t bid_next = blockIdx.x < n_units ? ids[blockIdx.x >> 1] : 0;
    for (int64_t unit = blockIdx.x; unit < n_units; unit += gridDim.x) {
        const int64_t bid = bid_next;
        const int64_t nu = unit + gridDim.x;
        bid_next = nu < n_units ? ids[nu >> 1] : 0;
        const bool ok = bid >= 0 && bid < num_blocks;
        if (!PACK && !ok)
            continue;
        uint4 *cache = ((unit & 1) ? v_cache : k_cache) + (ok ? bid : 0) * (int64_t)bv;
        uint4 *stg = staging + unit * (int64_t)bv;
        for (int base = threadIdx.x; base < bv; base += blockDim.x * kU) {
            uint4 val[kU];
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                const int v = base + u * (int)blockDim.x;
                val[u] = make_uint4(0u, 0u, 0u, 0u);
                if (v < bv && (!PACK || ok))
                    val[u] = PACK ? cache[v] : stg[v];
            }
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                const int v = base + u * (int)blockDim.x;
                if (v < bv) {
                    if (PACK)
                        stg[v] = val[u];
                    else
                        cache[v] = val[u];
                }
            }
        }
    }
}

} // namespace

cudaError_t launch_kv_pack(const void *k_cache, const void *v_cache, int64_t num_blocks, int64_t block_elems,
                           const int32_t *ids, int num_ids, void *staging, int num_sms, cudaStream_t s)
{
    const int64_t units = 2 * (int64_t)num_ids;
    const unsigned grid = (unsigned)(units < (int64_t)num_sms * kCopyCtasPerSm ? units : (int64_t)num_sms * kCopyCtasPerSm);
    kv_block_copy_kernel<true><<<grid, 256, 0, s>>>(
        const_cast<uint4 *>(static_cast<const uint4 *>(k_cache)), const_cast<uint4 *>(static_cast<const uint4 *>(v_cache)),
        num_blocks, (int)(block_elems / 8), ids, units, static_cast<uint4 *>(staging));
    return cudaGetLastError();
}

cudaError_t launch_kv_unpack(const void *staging, const int32_t *ids, int num_ids, void *k_cache, void *v_cache,
                             int64_t num_blocks, int64_t block_elems, int num_sms, cudaStream_t s)
{
    const int64_t units = 2 * (int64_t)num_ids;
    const unsigned grid = (unsigned)(units < (int64_t)num_sms * kCopyCtasPerSm ? units : (int64_t)num_sms * kCopyCtasPerSm);
    kv_block_copy_kernel<false><<<grid, 256, 0, s>>>(static_cast<uint4 *>(k_cache), static_cast<uint4 *>(v_cache),
                                                     num_blocks, (int)(block_elems / 8), ids, units,
                                                     const_cast<uint4 *>(static_cast<const uint4 *>(staging)));
    return cudaGetLastError();
}

cudaError_t launch_kv_write(const void *k_new, const void *v_new, int64_t row_stride, const int64_t *slots,
                            int num_tokens, void *k_cache, void *v_cache, int64_t num_blocks, int Hkv, int D,
                            int nhd, uint32_t *status, cudaStream_t s)
{
    bool vec_ok = false;
    const KvWriteArgs a =
        kv_write_args(k_new, v_new, row_stride, slots, num_tokens, k_cache, v_cache, num_blocks, Hkv, D, nhd, &vec_ok);
    const unsigned blocks = (unsigned)kv_write_ctas(num_tokens);
    if (vec_ok)
        kv_write_kernel<8><<<blocks, 256, 0, s>>>(a, status);
    else
        kv_write_kernel<1><<<blocks, 256, 0, s>>>(a, status);
    return cudaGetLastError();
}

cudaError_t launch_slot_mapping(const int32_t *qsl, const int32_t *seq_lens, const int32_t *bt, int bt_stride,
                                int num_seqs, int num_tokens, int64_t *slots, cudaStream_t s)
{
    slot_mapping_kernel<<<num_seqs, 128, 0, s>>>(qsl, seq_lens, bt, bt_stride, num_tokens, slots);
    return cudaGetLastError();
}

cudaError_t launch_gather(const void *cache, int64_t num_blocks, int Hkv, int D, int nhd, const int32_t *bt_row,
                          int seq_len, void *out, cudaStream_t s)
{
    const int threads = 256;
    const int blocks = (seq_len + 7) / 8;
    gather_kernel<<<blocks, threads, 0, s>>>(static_cast<const uint16_t *>(cache), num_blocks, Hkv, D,
                                             nhd ? D : kBlockSize * D, nhd ? Hkv * D : D, bt_row, seq_len,
                                             static_cast<uint16_t *>(out));
    return cudaGetLastError();
}

} // namespace pa
