// decode.cu -- paged attention for decode-shaped requests (q_len * G <= 8*NT
// query rows per kv head), the HBM-bound part of a mixed step.  Decode is
// memory-bandwidth bound (hn.213312.xyz section 一 "调度器"; shengyayun.com
// 适用场景 and 关键实现细节 4), so the design goal is to stream every needed
// K/V byte from HBM exactly once per kv head, with enough bytes in flight.
//
// Work unit = one CTA = (request r, kv head h, split s): keys
// [s*S, min((s+1)*S, L_r)) of kv head h, S the step's split size (the
// caller's, or 1024 / 2048 / 4096 as the plan kernel chose it; read from the
// workspace header).  All G query heads of the group (and
// all query tokens of a short multi-token request) are packed as the N columns
// of one warp MMA, so each K/V byte is read once per kv head.
//
// Data path per CTA (4 warps):
//   * each warp owns every 4th 16-token block of the split and a private ring
//     of 2 stages (so 3 CTAs, 12 warps, fit per SM); lane 0
//     fetches one (block, kv head) K tile and V tile with TMA loads (128-byte
//     swizzled, 2 KiB per 64-column half) that complete on the stage's
//     mbarrier, one ring ahead of use;
//   * S^T = K Q^T on mma.sync m16n8k16 (keys are the M=16 rows: one paged
//     block per MMA), bf16 in, fp32 accumulate; Q^T fragments stay in
//     registers for the whole split;
//   * online softmax in the exp2 domain with warp shuffles over the 8 lanes
//     that share a query column; P^T is re-laid out for the PV MMA in
//     registers with movmatrix (no shared-memory round trip);
//   * O^T += V^T P^T on mma.sync with V^T fragments from ldmatrix.trans;
//   * at the end the 4 warps' (m, l, O) are merged through shared memory and
//     written as bf16 output (single split) or as an fp32 partial state; the
//     last split CTA of a (request, kv head) to finish -- counted with one
//     atomic per (request, kv head) -- merges all the splits' states into the
//     output (flash-decoding's second pass without a second launch).
// Keys beyond L_r in the last block (unused slots, possibly NaN) are masked by
// select, and their V rows are zeroed in registers, so 0 * NaN never reaches
// an accumulator.
#include <math_constants.h>

#include <mutex>

#include "merge.cuh"
#include "pa_internal.cuh"
#include "ptx.cuh"

namespace pa {
namespace {

constexpr int kDecWarps = 4;

// Ring depth per warp: 2 blocks, so 3 CTAs (12 warps, 24 blocks = 192 KB of loads in flight)
// fit per SM; the extra warps hide the per-block MMA and softmax latency better than a third
// stage per warp with 2 CTAs per SM (same bytes in flight).
template <int D, int NT>
struct DecCfg {
    static constexpr int kStages = 2;
    static constexpr int kHalves = D / 64;
    static constexpr int kBox = 16 * 64 * 2;           // one TMA box: 16 rows x 64 bf16
    static constexpr int kTile = kHalves * kBox;       // one (block, kv head) of K or V
    static constexpr int kStage = 2 * kTile;           // K + V
    static constexpr int kData = kDecWarps * kStages * kStage;
    static constexpr int kSmem = kData + 64 * 8 + 1024; // + barriers + alignment slack
};

// byte offset of (row, 16-byte chunk) inside a K/V tile laid out as
// [half][16 rows][64 bf16] with the 128-byte TMA swizzle
__device__ __forceinline__ uint32_t tile_off(int row, int chunk)
{
    return (uint32_t)((chunk >> 3) * 2048 + row * 128 + (((chunk & 7) ^ (row & 7)) << 4));
}

template <int D, int NT>
__global__ void __launch_bounds__(kDecWarps * 32) decode_kernel(const __grid_constant__ CUtensorMap tm_k,
                                                                const __grid_constant__ CUtensorMap tm_v,
                                                                const AttnParams p)
{
    using Cfg = DecCfg<D, NT>;
    constexpr int kDecStages = Cfg::kStages;
    constexpr int kKS = D / 16; // k-steps of S^T over the head dim
    constexpr int kMT = D / 16; // m-tiles of O^T over the head dim
    constexpr int kRows = 8 * NT;

    const int u = (int)(blockIdx.x / (unsigned)p.Hkv);
    const int h = (int)(blockIdx.x % (unsigned)p.Hkv);
    if (blockIdx.x == 0 && threadIdx.x == 0)
        p.hdr->write_epoch = kWriteEpochIdle; // the step's write launch (if any) has finished
    if (u >= (int)p.hdr->n_dec_units || (p.hdr->status & PA_DEVICE_WAIT_TIMEOUT))
        return; // past the work list, or an earlier CTA of this call already gave up

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t bar0 = smem_u32(smem + Cfg::kData);

    const int2 unit = p.dec_units[u];
    const int r = unit.x, split = unit.y;
    const int qs = p.qsl[r];
    const int q_len = p.qsl[r + 1] - qs;
    const int L = p.seq_lens[r];
    const int ctx = L - q_len;
    const int rows = q_len * p.G;
    const int split_tokens = (int)p.hdr->split_tokens; // the plan's choice for this step
    const int k_begin = split * split_tokens;
    const int k_end = min(L, k_begin + split_tokens);
    const int n_splits = (L + split_tokens - 1) / split_tokens;
    const int nb = (k_end - k_begin + kBlockSize - 1) / kBlockSize;
    const int blk0 = k_begin / kBlockSize;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x < kDecWarps * kDecStages)
        mbar_init(bar0 + threadIdx.x * 8, 1);
    fence_barrier_init();
    __syncthreads();

    const int cw = nb > warp ? (nb - warp + kDecWarps - 1) / kDecWarps : 0; // this warp's blocks
    uint8_t *wbase = smem + warp * kDecStages * Cfg::kStage;
    const uint32_t wbase_s = smem_u32(wbase);
    const uint32_t wbar = bar0 + warp * kDecStages * 8;
    const int32_t *bt_row = p.bt + (int64_t)r * p.bt_stride;

    // block ids of this warp's blocks, 32 at a time: lane i holds block (32c + i)
    int bid_reg = 0;
    auto load_bids = [&](int c) {
        const int k = c * 32 + lane;
        bid_reg = k < cw ? bt_row[blk0 + warp + kDecWarps * k] : 0;
    };
    auto issue = [&](int k) { // whole warp calls; lane 0 issues the copies for block k into stage k % kDecStages
        if ((k & 31) == 0 && k > 0)
            load_bids(k >> 5);
        const int bid = __shfl_sync(0xffffffffu, bid_reg, k & 31);
        if (lane == 0) {
            const int stage = k % kDecStages;
            const uint32_t bar = wbar + stage * 8;
            // HND: 2-D map {D, blocks*Hkv*16}, row (bid*Hkv + h)*16;  NHD: 3-D map {D, Hkv, blocks*16},
            // (head h, token row bid*16).  Either way the box is 16 rows x 64 columns.
            int y = -kBlockSize; // fully out of bounds: TMA fills zeros
            if ((unsigned)bid < (unsigned long long)p.num_blocks)
                y = (p.nhd ? bid : bid * p.Hkv + h) * kBlockSize;
            else
                atomicOr(&p.hdr->status, PA_DEVICE_BAD_BLOCK);
            mbar_arrive_expect_tx(bar, Cfg::kStage);
            const uint32_t sk = wbase_s + stage * Cfg::kStage;
            // read once: first out of L2, so that a concurrent prefill keeps its re-read K/V tiles there
            const uint64_t pol = l2_policy_evict_first();
            if (p.nhd) {
#pragma unroll
                for (int hf = 0; hf < Cfg::kHalves; ++hf) {
                    tma_load_3d_hint(sk + hf * Cfg::kBox, &tm_k, hf * 64, h, y, bar, pol);
                    tma_load_3d_hint(sk + Cfg::kTile + hf * Cfg::kBox, &tm_v, hf * 64, h, y, bar, pol);
                }
            } else {
#pragma unroll
                for (int hf = 0; hf < Cfg::kHalves; ++hf) {
                    tma_load_2d_hint(sk + hf * Cfg::kBox, &tm_k, hf * 64, y, bar, pol);
                    tma_load_2d_hint(sk + Cfg::kTile + hf * Cfg::kBox, &tm_v, hf * 64, y, bar, pol);
                }
            }
        }
    };

    if (cw > 0) {
        load_bids(0);
        const int pro = min(cw, kDecStages);
        for (int k = 0; k < pro; ++k)
            issue(k);
    }

    // Q^T fragments (B operand): column n = query row (token i, head g) = 8*nt + lane/4
    uint32_t qf[NT][kKS][2];
    int lim[NT][2]; // last visible key of the lane's two columns
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const int n = nt * 8 + (lane >> 2);
        const bool valid = n < rows;
        const int t = qs + (valid ? n / p.G : 0);
        const int hq = h * p.G + (valid ? n % p.G : 0);
        const uint32_t *qrow = reinterpret_cast<const uint32_t *>(p.q + ((int64_t)t * p.Hq + hq) * D);
#pragma unroll
        for (int ks = 0; ks < kKS; ++ks) {
            qf[nt][ks][0] = valid ? qrow[(ks * 16 + 2 * (lane & 3)) >> 1] : 0u;
            qf[nt][ks][1] = valid ? qrow[(ks * 16 + 8 + 2 * (lane & 3)) >> 1] : 0u;
        }
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int nn = nt * 8 + 2 * (lane & 3) + e;
            lim[nt][e] = nn < rows ? ctx + nn / p.G : L - 1;
        }
    }

    // l_run: row sum of the bf16-rounded weights (normalises O); l_ex: exact fp32 sum (for the LSE)
    float m_run[NT][2], l_run[NT][2], l_ex[NT][2], acc[NT][kMT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            m_run[nt][e] = -CUDART_INF_F;
            l_run[nt][e] = 0.f;
            l_ex[nt][e] = 0.f;
        }
#pragma unroll
        for (int mt = 0; mt < kMT; ++mt)
#pragma unroll
            for (int c = 0; c < 4; ++c)
                acc[nt][mt][c] = 0.f;
    }

    const float sl2 = p.scale_log2;
    const int mi = lane >> 3;
    bool aborted = false;
    int k = 0;
    for (; k < cw; ++k) {
        const int stage = k % kDecStages;
        if (!mbar_wait_warp(wbar + stage * 8, (uint32_t)((k / kDecStages) & 1))) {
            aborted = true;
            break;
        }
        const int j0 = k_begin + (warp + kDecWarps * k) * kBlockSize;
        const uint32_t sK = wbase_s + stage * Cfg::kStage;
        const uint32_t sV = sK + Cfg::kTile;
        if (p.k_new != nullptr) {
            // fused KV write: this block's rows at positions ctx..L-1 are the step's new tokens.
            // Store them into the cache and over the (stale) rows the TMA just brought in.
            const int lo = max(j0, ctx), hi = min(j0 + kBlockSize, L);
            if (lo < hi) {
                const int64_t bidw = bt_row[j0 / kBlockSize];
                if (bidw >= 0 && bidw < p.num_blocks) {
                    constexpr int kCh = D / 8; // 16-byte chunks per row
                    uint8_t *tile = wbase + stage * Cfg::kStage;
                    for (int i = lane; i < (hi - lo) * 2 * kCh; i += 32) {
                        const int c = i % kCh, kv = (i / kCh) & 1, pos = lo + i / (2 * kCh);
                        const int64_t t = qs + (pos - ctx);
                        const int row = pos - j0;
                        const uint4 val = *reinterpret_cast<const uint4 *>((kv ? p.v_new : p.k_new) +
                                                                            t * p.new_row_stride + h * D + c * 8);
                        *reinterpret_cast<uint4 *>(tile + kv * Cfg::kTile + tile_off(row, c)) = val;
                        const int64_t e = p.nhd ? ((bidw * kBlockSize + row) * p.Hkv + h) * D + c * 8
                                                : ((bidw * p.Hkv + h) * kBlockSize + row) * D + c * 8;
                        *reinterpret_cast<uint4 *>((kv ? p.v_cache_w : p.k_cache_w) + e) = val;
                    }
                    // the stage is refilled by TMA (async proxy) after these generic writes
                    fence_proxy_async_smem();
                }
            }
            __syncwarp();
        }

        // ---- S^T[16 keys x 8NT cols] = K . Q^T
        float s[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int c = 0; c < 4; ++c)
                s[nt][c] = 0.f;
        {
            const int row = (lane & 7) + 8 * (mi & 1);
#pragma unroll
            for (int ks = 0; ks < kKS; ++ks) {
                uint32_t a0, a1, a2, a3;
                ldmatrix_x4(sK + tile_off(row, 2 * ks + (mi >> 1)), a0, a1, a2, a3);
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
                    mma_bf16_16816(s[nt], a0, a1, a2, a3, qf[nt][ks][0], qf[nt][ks][1]);
            }
        }

        // ---- mask, online softmax (exp2 domain)
        const int jl = j0 + (lane >> 2), jh = jl + 8;
        uint32_t bp[NT][2];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            float x[4];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                x[e] = jl <= lim[nt][e] ? s[nt][e] * sl2 : -CUDART_INF_F;
                x[2 + e] = jh <= lim[nt][e] ? s[nt][2 + e] * sl2 : -CUDART_INF_F;
            }
            float pr[4], alpha[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                float mx = fmaxf(x[e], x[2 + e]);
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
                const float m_new = fmaxf(m_run[nt][e], mx);
                const float m_use = m_new == -CUDART_INF_F ? 0.f : m_new;
                alpha[e] = fast_exp2(m_run[nt][e] - m_use);
                pr[e] = fast_exp2(x[e] - m_use);
                pr[2 + e] = fast_exp2(x[2 + e] - m_use);
                l_ex[nt][e] = l_ex[nt][e] * alpha[e] + pr[e] + pr[2 + e];
                m_run[nt][e] = m_new;
#pragma unroll
                for (int mt = 0; mt < kMT; ++mt) {
                    acc[nt][mt][e] *= alpha[e];
                    acc[nt][mt][2 + e] *= alpha[e];
                }
            }
            // P is rounded to bf16 for the PV MMA; the row sums use the same rounded
            // weights, so the output is an exact convex combination of the V rows
            const uint32_t w_lo = pack_bf16x2(pr[0], pr[1]), w_hi = pack_bf16x2(pr[2], pr[3]);
            l_run[nt][0] = l_run[nt][0] * alpha[0] + __uint_as_float(w_lo << 16) + __uint_as_float(w_hi << 16);
            l_run[nt][1] = l_run[nt][1] * alpha[1] + __uint_as_float(w_lo & 0xffff0000u) +
                           __uint_as_float(w_hi & 0xffff0000u);
            bp[nt][0] = movmatrix_trans(w_lo);
            bp[nt][1] = movmatrix_trans(w_hi);
        }

        // ---- O^T[D x 8NT] += V^T . P^T
        const int nvalid = L - j0; // keys of this block that exist (>= 16 except the last block)
        uint32_t mask_lo = 0xffffffffu, mask_hi = 0xffffffffu;
        if (nvalid < kBlockSize) {
            const int jlo = 2 * (lane & 3);
            mask_lo = (jlo < nvalid ? 0x0000ffffu : 0u) | (jlo + 1 < nvalid ? 0xffff0000u : 0u);
            mask_hi = (jlo + 8 < nvalid ? 0x0000ffffu : 0u) | (jlo + 9 < nvalid ? 0xffff0000u : 0u);
        }
        {
            const int row = (lane & 7) + 8 * (mi >> 1);
#pragma unroll
            for (int mt = 0; mt < kMT; ++mt) {
                uint32_t a0, a1, a2, a3;
                ldmatrix_x4_trans(sV + tile_off(row, 2 * mt + (mi & 1)), a0, a1, a2, a3);
                a0 &= mask_lo;
                a1 &= mask_lo;
                a2 &= mask_hi;
                a3 &= mask_hi;
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
                    mma_bf16_16816(acc[nt][mt], a0, a1, a2, a3, bp[nt][0], bp[nt][1]);
            }
        }
        __syncwarp();
        if (k + kDecStages < cw)
            issue(k + kDecStages);
    }

    if (aborted) {
        if (lane == 0)
            atomicOr(&p.hdr->status, PA_DEVICE_WAIT_TIMEOUT);
        // let copies still in flight into this warp's ring land before the CTA exits
        for (int kk = k; kk < min(cw, k + kDecStages); ++kk)
            (void)mbar_wait(wbar + (kk % kDecStages) * 8, (uint32_t)((kk / kDecStages) & 1));
    }

    // ---- per-lane partial row sums -> row sums
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            float v = l_run[nt][e], w = l_ex[nt][e];
            v += __shfl_xor_sync(0xffffffffu, v, 4);
            v += __shfl_xor_sync(0xffffffffu, v, 8);
            v += __shfl_xor_sync(0xffffffffu, v, 16);
            w += __shfl_xor_sync(0xffffffffu, w, 4);
            w += __shfl_xor_sync(0xffffffffu, w, 8);
            w += __shfl_xor_sync(0xffffffffu, w, 16);
            l_run[nt][e] = v;
            l_ex[nt][e] = w;
        }

    // ---- this warp's state -> its own (now idle) ring
    constexpr int kLd = D + 4; // padded row stride in floats
    float *cbuf = reinterpret_cast<float *>(wbase);
    float *cml = cbuf + kRows * kLd; // m[kRows], l_rounded[kRows], l_exact[kRows]
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int mt = 0; mt < kMT; ++mt)
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int n = nt * 8 + 2 * (lane & 3) + (c & 1);
                const int d = mt * 16 + (lane >> 2) + 8 * (c >> 1);
                cbuf[n * kLd + d] = acc[nt][mt][c];
            }
    if (lane < 4) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int n = nt * 8 + 2 * lane + e;
                cml[n] = m_run[nt][e];
                cml[kRows + n] = l_run[nt][e];
                cml[2 * kRows + n] = l_ex[nt][e];
            }
    }
    __syncthreads();

    // ---- merge the 4 warps and write
    constexpr int kTpr = (kDecWarps * 32) / kRows; // threads per query row
    constexpr int kEpt = D / kTpr;                 // consecutive elements per thread
    const int n = threadIdx.x / kTpr;
    const int d0 = (threadIdx.x % kTpr) * kEpt;
    // one query row n (elements d0 .. d0+kEpt-1): merge the 4 warps' states, then write the output
    // (single split) or this split's partial state
    auto write_state = [&](int n, int d0) {
        float M = -CUDART_INF_F;
#pragma unroll
        for (int w = 0; w < kDecWarps; ++w) {
            const float *ml = reinterpret_cast<const float *>(smem + w * kDecStages * Cfg::kStage) + kRows * kLd;
            M = fmaxf(M, ml[n]);
        }
        float wgt[kDecWarps];
        float lt = 0.f, lx = 0.f;
#pragma unroll
        for (int w = 0; w < kDecWarps; ++w) {
            const float *ml = reinterpret_cast<const float *>(smem + w * kDecStages * Cfg::kStage) + kRows * kLd;
            const float mw = ml[n];
            wgt[w] = (mw == -CUDART_INF_F) ? 0.f : fast_exp2(mw - M);
            lt += ml[kRows + n] * wgt[w];
            lx += ml[2 * kRows + n] * wgt[w];
        }
        const float inv = lt > 0.f ? 1.f / lt : 0.f;
        float o[kEpt];
#pragma unroll
        for (int i = 0; i < kEpt; ++i)
            o[i] = 0.f;
#pragma unroll
        for (int w = 0; w < kDecWarps; ++w) {
            const float *cb = reinterpret_cast<const float *>(smem + w * kDecStages * Cfg::kStage) + n * kLd + d0;
#pragma unroll
            for (int i = 0; i < kEpt; i += 4) {
                const float4 v = *reinterpret_cast<const float4 *>(cb + i);
                o[i] += wgt[w] * v.x;
                o[i + 1] += wgt[w] * v.y;
                o[i + 2] += wgt[w] * v.z;
                o[i + 3] += wgt[w] * v.w;
            }
        }
        const float lse = lx > 0.f ? (M + log2f(lx)) * 0.69314718055994531f : -CUDART_INF_F;
        const int t = qs + n / p.G;
        const int hq = h * p.G + n % p.G;
        if (n_splits == 1) {
            __nv_bfloat16 *dst = p.out + ((int64_t)t * p.Hq + hq) * D + d0;
            if constexpr (kEpt % 8 == 0) {
#pragma unroll
                for (int i = 0; i < kEpt; i += 8) {
                    uint4 v;
                    v.x = pack_bf16x2(o[i] * inv, o[i + 1] * inv);
                    v.y = pack_bf16x2(o[i + 2] * inv, o[i + 3] * inv);
                    v.z = pack_bf16x2(o[i + 4] * inv, o[i + 5] * inv);
                    v.w = pack_bf16x2(o[i + 6] * inv, o[i + 7] * inv);
                    *reinterpret_cast<uint4 *>(dst + i) = v;
                }
            } else {
                static_assert(kEpt == 4, "output vector width");
                uint2 v;
                v.x = pack_bf16x2(o[0] * inv, o[1] * inv);
                v.y = pack_bf16x2(o[2] * inv, o[3] * inv);
                *reinterpret_cast<uint2 *>(dst) = v;
            }
            if (p.lse && d0 == 0)
                p.lse[(int64_t)t * p.Hq + hq] = lse;
        } else {
            const int64_t idx = (((int64_t)r * p.QD + n / p.G) * p.Hq + hq) * p.max_splits + split;
            float *dst = p.part_o + idx * D + d0;
#pragma unroll
            for (int i = 0; i < kEpt; i += 4)
                *reinterpret_cast<float4 *>(dst + i) =
                    make_float4(o[i] * inv, o[i + 1] * inv, o[i + 2] * inv, o[i + 3] * inv);
            if (d0 == 0)
                p.part_lse[idx] = lse;
        }
    };
    if (n < rows)
        write_state(n, d0);
    if (n_splits == 1)
        return;
    // Split request: the last of its split CTAs for this kv head merges all the splits' states.
    // Release: the CTA barrier orders every thread's partial stores before thread 0's fence and
    // arrival (fences are cumulative); acquire: thread 0 fences after seeing the last arrival and
    // the barrier orders the other threads' reads (past L1) after it.
    __shared__ int s_last;
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        s_last = atomicAdd(&p.split_arrivals[(int64_t)r * p.Hkv + h], 1u) == (unsigned)(n_splits - 1);
        if (s_last)
            __threadfence();
    }
    __syncthreads();
    if (!s_last)
        return;
    for (int rr = warp; rr < rows; rr += kDecWarps) {
        const int t = qs + rr / p.G;
        const int hq = h * p.G + rr % p.G;
        const int64_t idx = (((int64_t)r * p.QD + rr / p.G) * p.Hq + hq) * p.max_splits;
        const int64_t orow = (int64_t)t * p.Hq + hq;
        merge_one<D, true>(p.part_o + idx * D, D, p.part_lse + idx, 1, n_splits, p.out + orow * D,
                           p.lse ? p.lse + orow : nullptr);
    }
}

template <int D, int NT>
cudaError_t launch_decode_t(const AttnParams &p, const CUtensorMap &tk, const CUtensorMap &tv, int64_t grid_units,
                            cudaStream_t s)
{
    constexpr int smem = DecCfg<D, NT>::kSmem;
    // the shared-memory attribute, once per device (host threads may call concurrently)
    constexpr int kMaxDev = 64;
    static std::once_flag once[kMaxDev];
    static cudaError_t attr_err[kMaxDev];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev)
        return cudaErrorInvalidDevice;
    std::call_once(once[dev], [dev] {
        attr_err[dev] = cudaFuncSetAttribute(decode_kernel<D, NT>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    });
    if (attr_err[dev] != cudaSuccess)
        return attr_err[dev];
    const unsigned grid = (unsigned)(grid_units * p.Hkv); // (unit, kv head), heads of a unit adjacent
    decode_kernel<D, NT><<<grid, kDecWarps * 32, smem, s>>>(tk, tv, p);
    return cudaGetLastError();
}

} // namespace

cudaError_t launch_decode(const AttnParams &p, const CUtensorMap &tk, const CUtensorMap &tv, int NT,
                          int64_t grid_units, cudaStream_t s)
{
    if (grid_units <= 0)
        return cudaSuccess;
    if (p.D == 128)
        return NT == 1 ? launch_decode_t<128, 1>(p, tk, tv, grid_units, s)
                       : launch_decode_t<128, 2>(p, tk, tv, grid_units, s);
    return NT == 1 ? launch_decode_t<64, 1>(p, tk, tv, grid_units, s) : launch_decode_t<64, 2>(p, tk, tv, grid_units, s);
}

} // namespace pa
