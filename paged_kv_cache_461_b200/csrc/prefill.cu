// prefill.cu -- chunked-prefill attention over the paged cache on the 5th-gen
// tensor cores (tcgen05.mma, accumulators in TMEM).
//
// Prefill is compute bound (hn.213312.xyz section 一 "调度器"; shengyayun.com
// 适用场景).  A chunk of q_len tokens at positions c_r .. c_r+q_len-1 attends
// causally to its request's cached context plus the chunk itself; chunking
// must not change the result (hn.213312.xyz section 二.1), which holds here
// because every row's result depends only on its own position.
//
// Work unit = one CTA = (request r, q-tile, kv head h).  A tile is 128 query
// rows: 128/G tokens x the G query heads that share kv head h (rows ordered
// token-major), so one K/V tile feeds all heads of the group.
//
// Warp roles (192 threads, one CTA per SM):
//   warp 0      TMA producer: the Q tile once (3-D box {64 d, G heads,
//               128/G tokens}, 128-byte swizzle), then K and V tiles of 128
//               keys = 8 paged blocks, each block one 2-D box per 64-column
//               half, into a 2-stage ring;
//   warp 1      TMEM allocation (512 columns) and the single MMA-issuing
//               thread: S_j = Q K_j^T (M=128, N=128, K=head_dim) into one of
//               two TMEM S buffers, then O += P_{j-1} V_{j-1} (M=128, N=head_dim,
//               K=16 per paged block) -- S for tile j+1 runs on the tensor core
//               while the softmax warps work on tile j;
//   warps 2..5  softmax: thread = query row = TMEM lane; tcgen05.ld its S row,
//               causal mask by select, running max in the exp2 domain, P as
//               bf16 into shared memory (128-byte swizzled, K-major) for the
//               PV MMA; O is rescaled in TMEM only when a row's max grows by
//               more than 2^8 (otherwise the stale max is kept, which leaves
//               the normalised result unchanged); epilogue O / l -> bf16.
// V rows past the end of the sequence in the last block (unused slots) are
// zeroed in shared memory before the last PV MMA, so 0 * NaN never enters O.
#include <math_constants.h>

#include "ptx.cuh"
#include "pa_internal.cuh"

namespace pa {
namespace {

template <int D>
struct PfCfg {
    static constexpr int kHalves = D / 64;
    static constexpr int kHalfBytes = 128 * 128;        // 128 rows x 128 B
    static constexpr int kQ = 128 * D * 2;              // Q tile
    static constexpr int kKV = kPrefillKeys * D * 2;    // one K or V tile (8 blocks)
    static constexpr int kStages = 2;
    static constexpr int kP = 128 * kPrefillKeys * 2;   // P tile
    static constexpr int kOffQ = 0;
    static constexpr int kOffK = kOffQ + kQ;
    static constexpr int kOffV = kOffK + kStages * kKV;
    static constexpr int kOffP = kOffV + kStages * kKV;
    static constexpr int kOffBar = kOffP + kP;
    static constexpr int kBarBytes = 256;
    static constexpr int kUsed = kOffBar + kBarBytes + 1024;
    // keep one CTA per SM (each CTA allocates all 512 TMEM columns)
    static constexpr int kSmem = kUsed > 120 * 1024 ? kUsed : 120 * 1024;
};

enum PfBar { B_Q = 0, B_KF = 1, B_VF = 3, B_KVE = 5, B_SF = 7, B_SFREE = 9, B_PF = 11, B_PVD = 12, B_FIN = 13, B_NUM = 14 };

constexpr uint32_t kTmemCols = 512;
constexpr int kColS = 0;   // two S buffers: columns [0,128) and [128,256)
constexpr int kColO = 256; // O: columns [256, 256+D)

template <int D>
__global__ void __launch_bounds__(192, 1) prefill_kernel(const __grid_constant__ CUtensorMap tm_q,
                                                         const __grid_constant__ CUtensorMap tm_k,
                                                         const __grid_constant__ CUtensorMap tm_v,
                                                         const AttnParams p)
{
    using Cfg = PfCfg<D>;
    constexpr int kKS = D / 16; // k-steps of Q K^T
    const int u = (int)(blockIdx.x / (unsigned)p.Hkv);
    const int h = (int)(blockIdx.x % (unsigned)p.Hkv);
    if (u >= (int)p.hdr->n_pf_tiles || (p.hdr->status & PA_DEVICE_WAIT_TIMEOUT))
        return; // past the work list, or an earlier CTA of this call already gave up

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t sQ = sbase + Cfg::kOffQ;
    const uint32_t sK0 = sbase + Cfg::kOffK;
    const uint32_t sV0 = sbase + Cfg::kOffV;
    const uint32_t sP = sbase + Cfg::kOffP;
    const uint32_t bar = sbase + Cfg::kOffBar;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + Cfg::kOffBar + B_NUM * 8);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + Cfg::kOffBar + B_NUM * 8 + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // ---- tile geometry (same in every thread)
    const int2 tile = p.pf_tiles[u];
    const int r = tile.x, qt = tile.y;
    const int G = p.G;
    const int TQ = kPrefillRows / G;
    const int qs = p.qsl[r];
    const int q_len = p.qsl[r + 1] - qs;
    const int L = p.seq_lens[r];
    const int ctx = L - q_len;
    const int tok0 = qt * TQ;                 // first token of the tile within the request
    const int n_tok = min(TQ, q_len - tok0);
    const int rows = n_tok * G;
    const int p_min = ctx + tok0;             // position of the tile's first token
    const int p_max = p_min + n_tok - 1;      // position of its last token
    const int n_keys = p_max + 1;
    const int nkt = (n_keys + kPrefillKeys - 1) / kPrefillKeys;
    const int32_t *bt_row = p.bt + (int64_t)r * p.bt_stride;

    // ---- setup: barriers, TMEM
    if (threadIdx.x == 0) {
        mbar_init(bar + B_Q * 8, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(bar + (B_KF + s) * 8, 1);
            mbar_init(bar + (B_VF + s) * 8, 1);
            mbar_init(bar + (B_KVE + s) * 8, 1);
            mbar_init(bar + (B_SF + s) * 8, 1);
            mbar_init(bar + (B_SFREE + s) * 8, 128);
        }
        mbar_init(bar + B_PF * 8, 128);
        mbar_init(bar + B_PVD * 8, 1);
        mbar_init(bar + B_FIN * 8, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    auto fail = [&]() {
        *abort_flag = 1;
        atomicOr(&p.hdr->status, PA_DEVICE_WAIT_TIMEOUT);
    };

    if (warp == 0) {
        // ================= TMA producer
        if (lane == 0) {
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            mbar_arrive_expect_tx(bar + B_Q * 8, Cfg::kQ);
#pragma unroll
            for (int hf = 0; hf < Cfg::kHalves; ++hf)
                tma_load_3d(sQ + hf * Cfg::kHalfBytes, &tm_q, hf * 64, h * G, qs + tok0, bar + B_Q * 8);
        }
        int issued = 0;
        for (int kt = 0; kt < nkt; ++kt) {
            const int st = kt & 1;
            if (kt >= 2 && !mbar_wait_warp(bar + (B_KVE + st) * 8, ((kt - 2) >> 1) & 1, abort_flag)) {
                if (lane == 0)
                    fail();
                break;
            }
            const int key0 = kt * kPrefillKeys;
            const int nblk = (min(kPrefillKeys, n_keys - key0) + kBlockSize - 1) / kBlockSize;
            const uint32_t tx = (uint32_t)(nblk * kBlockSize * D * 2);
            if (lane == 0) {
                mbar_arrive_expect_tx(bar + (B_KF + st) * 8, tx);
                mbar_arrive_expect_tx(bar + (B_VF + st) * 8, tx);
            }
            __syncwarp();
            if (lane < nblk) {
                const int bid = bt_row[kt * (kPrefillKeys / kBlockSize) + lane];
                int y = -kBlockSize;
                if ((unsigned)bid < (unsigned long long)p.num_blocks)
                    y = (bid * p.Hkv + h) * kBlockSize;
                else
                    atomicOr(&p.hdr->status, PA_DEVICE_BAD_BLOCK);
#pragma unroll
                for (int hf = 0; hf < Cfg::kHalves; ++hf) {
                    const uint32_t o = hf * Cfg::kHalfBytes + lane * (kBlockSize * 128);
                    tma_load_2d(sK0 + st * Cfg::kKV + o, &tm_k, hf * 64, y, bar + (B_KF + st) * 8);
                    tma_load_2d(sV0 + st * Cfg::kKV + o, &tm_v, hf * 64, y, bar + (B_VF + st) * 8);
                }
            }
            issued = kt + 1;
        }
        if (*abort_flag && lane == 0) {
            // let loads already issued land before the CTA exits
            for (int kt = max(0, issued - 2); kt < issued; ++kt) {
                (void)mbar_wait(bar + (B_KF + (kt & 1)) * 8, (kt >> 1) & 1);
                (void)mbar_wait(bar + (B_VF + (kt & 1)) * 8, (kt >> 1) & 1);
            }
            (void)mbar_wait(bar + B_Q * 8, 0);
        }
    } else if (warp == 1) {
        // ================= MMA issuer (one thread)
        if (lane == 0) {
            constexpr uint32_t idesc_s = idesc_bf16_f32(128, kPrefillKeys, 0, 0);
            constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, 0, 1);
            bool ok = mbar_wait(bar + B_Q * 8, 0, abort_flag);
            auto issue_pv = [&](int j) -> bool {
                const int st = j & 1;
                if (!mbar_wait(bar + (B_VF + st) * 8, (j >> 1) & 1, abort_flag))
                    return false;
                if (!mbar_wait(bar + B_PF * 8, j & 1, abort_flag))
                    return false;
                tc_fence_after();
                const int key0 = j * kPrefillKeys;
                const int nblk = (min(kPrefillKeys, n_keys - key0) + kBlockSize - 1) / kBlockSize;
                const uint32_t sV = sV0 + st * Cfg::kKV;
                for (int kk = 0; kk < nblk; ++kk) {
                    const uint64_t a = smem_desc_sw128(sP + (kk >> 2) * Cfg::kHalfBytes + (kk & 3) * 32, 16, 1024);
                    const uint64_t b = smem_desc_sw128(sV + kk * (kBlockSize * 128), Cfg::kHalfBytes, 1024);
                    umma_f16(tmem + kColO, a, b, idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
                }
                umma_commit(bar + (B_KVE + st) * 8);
                umma_commit(bar + B_PVD * 8);
                return true;
            };
            for (int kt = 0; ok && kt < nkt; ++kt) {
                const int st = kt & 1;
                if (!mbar_wait(bar + (B_KF + st) * 8, (kt >> 1) & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                if (kt >= 2 && !mbar_wait(bar + (B_SFREE + st) * 8, ((kt - 2) >> 1) & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t sK = sK0 + st * Cfg::kKV;
#pragma unroll
                for (int ks = 0; ks < kKS; ++ks) {
                    const uint32_t off = (ks >> 2) * Cfg::kHalfBytes + (ks & 3) * 32;
                    umma_f16(tmem + kColS + st * kPrefillKeys, smem_desc_sw128(sQ + off, 16, 1024),
                             smem_desc_sw128(sK + off, 16, 1024), idesc_s, ks > 0 ? 1u : 0u);
                }
                umma_commit(bar + (B_SF + st) * 8);
                if (kt >= 1 && !issue_pv(kt - 1)) {
                    ok = false;
                    break;
                }
            }
            if (ok && !issue_pv(nkt - 1))
                ok = false;
            if (!ok)
                fail();
            // drain: nothing of ours may still be running on the tensor core at dealloc
            umma_commit(bar + B_FIN * 8);
            (void)mbar_wait(bar + B_FIN * 8, 0);
        }
    } else {
        // ================= softmax / correction / epilogue (warps 2..5)
        const int quad = warp & 3;                // TMEM lane quadrant this warp may access
        const int row = quad * 32 + lane;         // query row of the tile = TMEM lane
        const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
        const int p_row = row < rows ? p_min + row / G : p_max;
        const float sl2 = p.scale_log2;
        // l_sum: row sum of the bf16-rounded weights (normalises O); l_ex: exact fp32 sum (for the LSE)
        float m_ref = -CUDART_INF_F, l_sum = 0.f, l_ex = 0.f;
        bool ok = true;
        const bool tail_fix = (L % kBlockSize) != 0 && (p_max / kBlockSize) == ((L - 1) / kBlockSize);
        for (int kt = 0; kt < nkt; ++kt) {
            const int buf = kt & 1;
            if (!mbar_wait_warp(bar + (B_SF + buf) * 8, (kt >> 1) & 1, abort_flag)) {
                ok = false;
                break;
            }
            tc_fence_after();
            uint32_t sv[kPrefillKeys];
#pragma unroll
            for (int c = 0; c < kPrefillKeys / 32; ++c) {
                uint32_t tmp[32];
                tmem_ld32(tmem + lane_addr + kColS + buf * kPrefillKeys + c * 32, tmp);
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    sv[c * 32 + i] = tmp[i];
            }
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(bar + (B_SFREE + buf) * 8);

            const int key0 = kt * kPrefillKeys;
            const bool masked = key0 + kPrefillKeys - 1 > p_min;
            float mx = -CUDART_INF_F;
#pragma unroll
            for (int c = 0; c < kPrefillKeys; ++c) {
                float x = __uint_as_float(sv[c]) * sl2;
                if (masked && key0 + c > p_row)
                    x = -CUDART_INF_F;
                sv[c] = __float_as_uint(x);
                mx = fmaxf(mx, x);
            }
            float alpha = 1.f;
            if (kt == 0) {
                m_ref = mx;
            } else if (mx > m_ref + 8.f) {
                alpha = fast_exp2(m_ref - mx);
                m_ref = mx;
            }
            // P buffer is free and O is stable once the previous PV has completed
            if (kt > 0 && !mbar_wait_warp(bar + B_PVD * 8, (kt - 1) & 1, abort_flag)) {
                ok = false;
                break;
            }
            if (__any_sync(0xffffffffu, alpha != 1.f)) {
                tc_fence_after();
#pragma unroll 1
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t o[32];
                    tmem_ld32(tmem + lane_addr + kColO + c * 32, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
                    tmem_st32(tmem + lane_addr + kColO + c * 32, o);
                }
                tmem_wait_st();
            }
            l_sum *= alpha;
            l_ex *= alpha;
            // P row -> shared memory, K-major with the 128-byte swizzle: [key half][128 rows][64 keys]
#pragma unroll
            for (int ch = 0; ch < kPrefillKeys / 8; ++ch) {
                float pv[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    pv[i] = fast_exp2(__uint_as_float(sv[ch * 8 + i]) - m_ref);
                    l_ex += pv[i];
                }
                const uint32_t addr = sP + (ch >> 3) * Cfg::kHalfBytes + row * 128 + (((ch & 7) ^ (row & 7)) << 4);
                const uint32_t w0 = pack_bf16x2(pv[0], pv[1]), w1 = pack_bf16x2(pv[2], pv[3]);
                const uint32_t w2 = pack_bf16x2(pv[4], pv[5]), w3 = pack_bf16x2(pv[6], pv[7]);
                // the row sum uses the bf16-rounded weights the PV MMA sees
                l_sum += (__uint_as_float(w0 << 16) + __uint_as_float(w0 & 0xffff0000u)) +
                         (__uint_as_float(w1 << 16) + __uint_as_float(w1 & 0xffff0000u)) +
                         (__uint_as_float(w2 << 16) + __uint_as_float(w2 & 0xffff0000u)) +
                         (__uint_as_float(w3 << 16) + __uint_as_float(w3 & 0xffff0000u));
                asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(w0), "r"(w1), "r"(w2),
                             "r"(w3)
                             : "memory");
            }
            fence_proxy_async_smem();
            if (kt == nkt - 1 && tail_fix) {
                // zero V rows past the end of the sequence in the block holding key p_max
                const int st = kt & 1;
                if (!mbar_wait_warp(bar + (B_VF + st) * 8, (kt >> 1) & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                const int lb = (p_max / kBlockSize) - kt * (kPrefillKeys / kBlockSize);
                const int first = L % kBlockSize;
                const int nz = (kBlockSize - first) * Cfg::kHalves * 8; // 16-byte chunks
                const uint32_t sV = sV0 + st * Cfg::kKV;
                for (int i = row; i < nz; i += 128) {
                    const int chunk = i & 7;
                    const int rr = (i >> 3) % (kBlockSize - first);
                    const int hf = (i >> 3) / (kBlockSize - first);
                    const uint32_t addr = sV + hf * Cfg::kHalfBytes + (lb * kBlockSize + first + rr) * 128 + chunk * 16;
                    asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(addr), "r"(0u) : "memory");
                }
                fence_proxy_async_smem();
            }
            tc_fence_before();
            mbar_arrive(bar + B_PF * 8);
        }
        // ---- epilogue: O / l -> bf16
        if (ok && !mbar_wait_warp(bar + B_PVD * 8, (nkt - 1) & 1, abort_flag))
            ok = false;
        if (!ok) {
            if (lane == 0)
                fail();
        } else {
            tc_fence_after();
            const float inv = l_sum > 0.f ? 1.f / l_sum : 0.f;
            const bool store = row < rows;
            const int t = qs + tok0 + row / G;
            const int hq = h * G + row % G;
            __nv_bfloat16 *dst = p.out + ((int64_t)t * p.Hq + hq) * D;
#pragma unroll 1
            for (int c = 0; c < D / 32; ++c) {
                uint32_t o[32];
                tmem_ld32(tmem + lane_addr + kColO + c * 32, o);
                tmem_wait_ld();
                if (store) {
#pragma unroll
                    for (int i = 0; i < 32; i += 8) {
                        uint4 v;
                        v.x = pack_bf16x2(__uint_as_float(o[i]) * inv, __uint_as_float(o[i + 1]) * inv);
                        v.y = pack_bf16x2(__uint_as_float(o[i + 2]) * inv, __uint_as_float(o[i + 3]) * inv);
                        v.z = pack_bf16x2(__uint_as_float(o[i + 4]) * inv, __uint_as_float(o[i + 5]) * inv);
                        v.w = pack_bf16x2(__uint_as_float(o[i + 6]) * inv, __uint_as_float(o[i + 7]) * inv);
                        *reinterpret_cast<uint4 *>(dst + c * 32 + i) = v;
                    }
                }
            }
            if (store && p.lse)
                p.lse[(int64_t)t * p.Hq + hq] =
                    l_ex > 0.f ? (m_ref + log2f(l_ex)) * 0.69314718055994531f : -CUDART_INF_F;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

template <int D>
cudaError_t launch_prefill_t(const AttnParams &p, const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                             int64_t grid_tiles, cudaStream_t s)
{
    constexpr int smem = PfCfg<D>::kSmem;
    static bool attr_done[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !attr_done[dev]) {
        cudaError_t e = cudaFuncSetAttribute(prefill_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess)
            return e;
        attr_done[dev] = true;
    }
    const unsigned grid = (unsigned)(grid_tiles * p.Hkv);
    prefill_kernel<D><<<grid, 192, smem, s>>>(tq, tk, tv, p);
    return cudaGetLastError();
}

} // namespace

cudaError_t launch_prefill(const AttnParams &p, const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                           int64_t grid_tiles, cudaStream_t s)
{
    if (grid_tiles <= 0)
        return cudaSuccess;
    if (p.D == 128)
        return launch_prefill_t<128>(p, tq, tk, tv, grid_tiles, s);
    return launch_prefill_t<64>(p, tq, tk, tv, grid_tiles, s);
}

} // namespace pa
