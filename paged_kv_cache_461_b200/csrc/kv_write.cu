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
#include <mutex>
#include <type_traits>

#include "pa_internal.cuh"
#include "ptx.cuh"

namespace pa {
namespace {

// One warp per token; lanes stride over the token's Hkv*D/VEC vectors of K and V.
template <int VEC>
__global__ void __launch_bounds__(256) kv_write_kernel(const uint16_t *__restrict__ k_new,
                                                       const uint16_t *__restrict__ v_new, int64_t row_stride,
                                                       const int64_t *__restrict__ slots, int num_tokens,
                                                       uint16_t *__restrict__ k_cache, uint16_t *__restrict__ v_cache,
                                                       int64_t num_blocks, int Hkv, int D, int head_stride,
                                                       int tok_stride, uint32_t *status)
{
    using Vec = typename std::conditional<VEC == 8, uint4, uint16_t>::type;
    const int lane = threadIdx.x & 31;
    const int warps_per_cta = blockDim.x >> 5;
    const int64_t n_slots = num_blocks * kBlockSize;
    const int vec_per_row = D / VEC;
    const int vec_per_tok = Hkv * vec_per_row;
    for (int64_t t = (int64_t)blockIdx.x * warps_per_cta + (threadIdx.x >> 5); t < num_tokens;
         t += (int64_t)gridDim.x * warps_per_cta) {
        const int64_t slot = slots[t];
        if (slot < 0)
            continue; // padding token: nothing is written
        if (slot >= n_slots) { // a slot outside the pool: nothing is written, the caller is told
            if (status != nullptr && lane == 0)
                atomicOr(status, PA_DEVICE_BAD_SLOT);
            continue;
        }
        const int64_t blk = slot / kBlockSize;
        const int off = (int)(slot % kBlockSize);
        const uint16_t *ks = k_new + t * row_stride;
        const uint16_t *vs = v_new + t * row_stride;
        const int64_t base = blk * ((int64_t)Hkv * kBlockSize * D) + off * tok_stride;
        auto dst_of = [&](int i) {
            const int h = i / vec_per_row;
            return base + h * head_stride + (i - h * vec_per_row) * VEC;
        };
        constexpr int kPer = 8; // vectors of K (and of V) per lane in flight at once
        if (VEC == 8 && vec_per_tok <= 32 * kPer) {
            // a token's rows in one go (Hkv * D <= 2048): every load of the lane first, then the stores
            Vec kv[kPer], vv[kPer];
#pragma unroll
            for (int u = 0; u < kPer; ++u) {
                const int i = lane + 32 * u;
                if (i < vec_per_tok) {
                    const int h = i / vec_per_row;
                    const int64_t src = (int64_t)h * D + (i - h * vec_per_row) * VEC;
                    kv[u] = *reinterpret_cast<const Vec *>(ks + src);
                    vv[u] = *reinterpret_cast<const Vec *>(vs + src);
                }
            }
#pragma unroll
            for (int u = 0; u < kPer; ++u) {
                const int i = lane + 32 * u;
                if (i < vec_per_tok) {
                    const int64_t dst = dst_of(i);
                    *reinterpret_cast<Vec *>(k_cache + dst) = kv[u];
                    *reinterpret_cast<Vec *>(v_cache + dst) = vv[u];
                }
            }
            continue;
        }
        for (int i = lane; i < vec_per_tok; i += 32) {
            const int h = i / vec_per_row;
            const int e = (i - h * vec_per_row) * VEC;
            const int64_t dst = dst_of(i);
            const Vec kv = *reinterpret_cast<const Vec *>(ks + (int64_t)h * D + e);
            const Vec vv = *reinterpret_cast<const Vec *>(vs + (int64_t)h * D + e);
            *reinterpret_cast<Vec *>(k_cache + dst) = kv;
            *reinterpret_cast<Vec *>(v_cache + dst) = vv;
        }
    }
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

// Whole-block copies between the caches and a staging buffer [num_ids][2][unit] (unit = one block of
// one cache, unit_bytes contiguous bytes in both).  Each copy goes global -> shared -> global with bulk
// copies issued by one thread: work item = (entry i, cache kv, chunk c) of at most kChunk bytes; a CTA
// keeps kStages - 1 loads in flight while the store of the previous item drains, and a stage is
// reloaded only once the store that read it is done reading.  PACK: cache -> staging (an id outside
// the pool stores zeros); otherwise staging -> cache (an id outside the pool is skipped).
constexpr int kCopyChunk = 16 * 1024;
constexpr int kCopyStages = 8;
constexpr int kCopySmem = kCopyStages * kCopyChunk + 1024 + kCopyStages * 8;

template <bool PACK>
__global__ void __launch_bounds__(32) kv_block_copy_kernel(uint8_t *__restrict__ k_cache, uint8_t *__restrict__ v_cache,
                                                           int64_t num_blocks, int64_t unit_bytes,
                                                           const int32_t *__restrict__ ids, int64_t n_units,
                                                           uint8_t *__restrict__ staging, uint32_t *status)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar0 = sbase + kCopyStages * kCopyChunk;
    const int lane = threadIdx.x;
    const int64_t chunks = (unit_bytes + kCopyChunk - 1) / kCopyChunk;
    const int64_t n_items = n_units * chunks;
    if (lane < kCopyStages)
        mbar_init(bar0 + lane * 8, 1);
    fence_barrier_init();
    __syncwarp();

    // the k-th item of this CTA: (global and shared addresses, size); bad = id outside the pool
    struct Item {
        const uint8_t *src;
        uint8_t *dst;
        uint32_t bytes;
        bool bad;
    };
    auto item = [&](int64_t k) {
        const int64_t it = (int64_t)blockIdx.x + k * gridDim.x;
        const int64_t unit = it / chunks, c = it - unit * chunks;
        const int64_t bid = ids[unit >> 1];
        Item x;
        x.bad = bid < 0 || bid >= num_blocks;
        uint8_t *cache = ((unit & 1) ? v_cache : k_cache) + (x.bad ? 0 : bid) * unit_bytes + c * kCopyChunk;
        uint8_t *stg = staging + unit * unit_bytes + c * kCopyChunk;
        x.src = PACK ? cache : stg;
        x.dst = PACK ? stg : cache;
        x.bytes = (uint32_t)min((int64_t)kCopyChunk, unit_bytes - c * kCopyChunk);
        return x;
    };
    const int64_t my_items = n_items > (int64_t)blockIdx.x ? (n_items - blockIdx.x + gridDim.x - 1) / gridDim.x : 0;
    auto load = [&](int64_t k) { // lane 0; a bad id loads nothing (its stage completes at once)
        const Item x = item(k);
        const int s = (int)(k % kCopyStages);
        mbar_arrive_expect_tx(bar0 + s * 8, x.bad ? 0u : x.bytes);
        if (!x.bad)
            bulk_load(sbase + s * kCopyChunk, x.src, x.bytes, bar0 + s * 8);
    };
    bool ok = true;
    int64_t issued = 0; // loads issued so far (lane 0)
    if (lane == 0)
        for (; issued < min(my_items, (int64_t)kCopyStages); ++issued)
            load(issued);
    int64_t k = 0;
    for (; k < my_items; ++k) {
        const int s = (int)(k % kCopyStages);
        const Item x = item(k);
        if (x.bad) {
            if (PACK) // zeros into the staging entry, by the whole warp
                for (uint32_t o = lane * 16; o < x.bytes; o += 32 * 16)
                    *reinterpret_cast<uint4 *>(x.dst + o) = make_uint4(0u, 0u, 0u, 0u);
        }
        if (lane == 0) {
            if (!mbar_wait(bar0 + s * 8, (uint32_t)((k / kCopyStages) & 1))) {
                ok = false;
            } else if (!x.bad) {
                bulk_store(x.dst, sbase + s * kCopyChunk, x.bytes);
            }
            bulk_commit();
            // the store of item k-1 has read its stage: refill that stage with item k-1+kCopyStages
            bulk_wait_read<1>();
            if (ok && k >= 1 && k - 1 + kCopyStages < my_items)
                load(issued++);
        }
        if (!__all_sync(0xffffffffu, ok))
            break;
    }
    if (lane == 0) {
        // on a timeout, let the loads still in flight into shared memory land (bounded) before exiting
        for (int64_t k2 = k; !ok && k2 < issued; ++k2)
            (void)mbar_wait(bar0 + (int)(k2 % kCopyStages) * 8, (uint32_t)((k2 / kCopyStages) & 1));
        bulk_wait_all();
        if (!ok && status != nullptr)
            atomicOr(status, PA_DEVICE_WAIT_TIMEOUT);
    }
}

} // namespace

namespace {

template <bool PACK>
cudaError_t launch_block_copy(void *k_cache, void *v_cache, int64_t num_blocks, int64_t block_elems,
                              const int32_t *ids, int num_ids, void *staging, int num_sms, uint32_t *status,
                              cudaStream_t s)
{
    constexpr int kMaxDev = 64;
    static std::once_flag once[kMaxDev];
    static cudaError_t attr_err[kMaxDev];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev)
        return cudaErrorInvalidDevice;
    std::call_once(once[dev], [dev] {
        attr_err[dev] =
            cudaFuncSetAttribute(kv_block_copy_kernel<PACK>, cudaFuncAttributeMaxDynamicSharedMemorySize, kCopySmem);
    });
    if (attr_err[dev] != cudaSuccess)
        return attr_err[dev];
    const int64_t unit_bytes = block_elems * 2;
    const int64_t items = 2 * (int64_t)num_ids * ((unit_bytes + kCopyChunk - 1) / kCopyChunk);
    const unsigned grid = (unsigned)(items < (int64_t)num_sms ? items : (int64_t)num_sms);
    kv_block_copy_kernel<PACK><<<grid, 32, kCopySmem, s>>>(static_cast<uint8_t *>(k_cache),
                                                          static_cast<uint8_t *>(v_cache), num_blocks, unit_bytes,
                                                          ids, 2 * (int64_t)num_ids, static_cast<uint8_t *>(staging),
                                                          status);
    return cudaGetLastError();
}

} // namespace

cudaError_t launch_kv_pack(const void *k_cache, const void *v_cache, int64_t num_blocks, int64_t block_elems,
                           const int32_t *ids, int num_ids, void *staging, int num_sms, uint32_t *status,
                           cudaStream_t s)
{
    return launch_block_copy<true>(const_cast<void *>(k_cache), const_cast<void *>(v_cache), num_blocks, block_elems,
                                   ids, num_ids, staging, num_sms, status, s);
}

cudaError_t launch_kv_unpack(const void *staging, const int32_t *ids, int num_ids, void *k_cache, void *v_cache,
                             int64_t num_blocks, int64_t block_elems, int num_sms, uint32_t *status, cudaStream_t s)
{
    return launch_block_copy<false>(k_cache, v_cache, num_blocks, block_elems, ids, num_ids,
                                    const_cast<void *>(staging), num_sms, status, s);
}

cudaError_t launch_kv_write(const void *k_new, const void *v_new, int64_t row_stride, const int64_t *slots,
                            int num_tokens, void *k_cache, void *v_cache, int64_t num_blocks, int Hkv, int D,
                            int nhd, uint32_t *status, cudaStream_t s)
{
    const int head_stride = nhd ? D : kBlockSize * D;
    const int tok_stride = nhd ? Hkv * D : D;
    const bool vec_ok = ((reinterpret_cast<uintptr_t>(k_new) | reinterpret_cast<uintptr_t>(v_new) |
                          reinterpret_cast<uintptr_t>(k_cache) | reinterpret_cast<uintptr_t>(v_cache)) % 16 == 0) &&
                        (row_stride % 8 == 0) && (D % 8 == 0);
    const int threads = 256;
    const int warps = threads / 32;
    int64_t blocks = ((int64_t)num_tokens + warps - 1) / warps;
    if (blocks > 148 * 16)
        blocks = 148 * 16;
    if (blocks < 1)
        blocks = 1;
    if (vec_ok)
        kv_write_kernel<8><<<(unsigned)blocks, threads, 0, s>>>(
            static_cast<const uint16_t *>(k_new), static_cast<const uint16_t *>(v_new), row_stride, slots, num_tokens,
            static_cast<uint16_t *>(k_cache), static_cast<uint16_t *>(v_cache), num_blocks, Hkv, D, head_stride,
            tok_stride, status);
    else
        kv_write_kernel<1><<<(unsigned)blocks, threads, 0, s>>>(
            static_cast<const uint16_t *>(k_new), static_cast<const uint16_t *>(v_new), row_stride, slots, num_tokens,
            static_cast<uint16_t *>(k_cache), static_cast<uint16_t *>(v_cache), num_blocks, Hkv, D, head_stride,
            tok_stride, status);
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
