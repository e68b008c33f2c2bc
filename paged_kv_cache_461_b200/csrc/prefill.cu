// prefill.cu -- chunked-prefill attention over the paged cache on the 5th-gen
// tensor cores (tcgen05.mma, accumulators and P in TMEM).
//
// Prefill is compute bound (hn.213312.xyz section 一, scheduler paragraph;
// shengyayun.com 适用场景).  A chunk of q_len tokens at positions
// c_r .. c_r+q_len-1 attends causally to its request's cached context plus the
// chunk itself; chunking does not change any row's result (hn.213312.xyz
// section 二.1) because every row depends only on its own position.
//
// Work unit = one CTA = (request r, q-pair, kv head h).  A q-pair is two tiles
// A and B of 128 query rows each; a tile is 128/G tokens x the G query heads
// that share kv head h (token-major), so one K/V tile feeds every head of the
// group and both tiles.
//
// Warp roles (576 threads, one CTA per SM):
//   warp 0      TMA producer: both Q tiles once (3-D boxes {64 d, G heads,
//               128/G tokens}, 128-byte swizzle), then per 128-key step the K
//               tile and the V tile (8 paged blocks x 64-column halves, 2-D
//               boxes) into separate 2-stage rings;
//   warp 1      TMEM allocation (512 columns: S_A, O_A, S_B, O_B) and the
//               single MMA-issuing thread.  Order per key step j:
//                 PV_A(j-1), S_A(j), PV_B(j-1), S_B(j)   (ping-pong)
//               so the tensor core works on one tile while the other tile's
//               softmax runs.  S = Q K^T is SS (both operands in smem);
//               O += P V reads P from TMEM (written over S by the softmax)
//               and V from smem as an MN-major operand;
//   warps 2..9  softmax of tile A, warps 10..17 softmax of tile B: each
//               query row (= TMEM lane) is shared by two threads in two warps
//               of the same TMEM lane quadrant, one per 64-key half, so a
//               thread holds its 64 scores in registers after one tcgen05.ld
//               pass.  Causal mask by select, row max exchanged between the
//               two halves through shared memory (64-thread named barrier),
//               P = exp2(s*c - m*c) with packed fp32x2 FMAs, bf16 P back into
//               TMEM over S with tcgen05.st; O is rescaled in TMEM only when a
//               row's max grows by more than 2^8 (a stale max leaves the
//               normalised result unchanged); the epilogue writes O / l as
//               bf16, each thread half of the head dimension.
// Ordering facts the pipeline relies on: the commit after S_X(j) fires only
// once every earlier MMA of the issuing thread is done, so when the softmax
// sees S_X(j) the previous PV_X(j-1) has finished with P_X and O_X; and MMAs
// issued by one thread run in issue order, so S_X(j) (which overwrites the TMEM
// columns holding P_X(j-1)) runs after PV_X(j-1) has read them.
// V rows past the end of the sequence in its last block (unused slots) are
// zeroed in shared memory by the producer before any PV reads them, so 0 * NaN
// never enters O.
#include <math_constants.h>

#include "ptx.cuh"
#include "pa_internal.cuh"

namespace pa {
namespace {

template <int D>
struct PfCfg {
    static constexpr int kHalves = D / 64;
    static constexpr int kHalfBytes = 128 * 128;       // 128 rows x 128 B
    static constexpr int kTile = 128 * D * 2;          // one 128-row Q tile, or one 128-key K or V tile
    static constexpr int kStages = 2;
    static constexpr int kOffQ = 0;                    // Q_A, Q_B
    static constexpr int kOffK = 2 * kTile;            // K ring
    static constexpr int kOffV = kOffK + kStages * kTile; // V ring
    static constexpr int kOffBar = kOffV + kStages * kTile;
    static constexpr int kBarBytes = 256;
    static constexpr int kOffX = kOffBar + kBarBytes;   // row-max / row-sum exchange: [tile][parity][half][128] fp32
    static constexpr int kXBytes = 2 * 2 * 2 * 128 * 4;
    static constexpr int kUsed = kOffX + kXBytes + 1024;
    // keep one CTA per SM (each CTA allocates all 512 TMEM columns)
    static constexpr int kSmem = kUsed > 120 * 1024 ? kUsed : 120 * 1024;
};

// TMEM columns of the two tiles' S (P aliases its first 64 columns) and O
__device__ __forceinline__ int col_s(int x) { return x * 256; }
__device__ __forceinline__ int col_o(int x) { return x * 256 + 128; }

enum PfBar {
    B_Q = 0,
    B_KF = 1,    // 2: K stage full
    B_KE = 3,    // 2: K stage consumed
    B_VF = 5,    // 2: V stage full
    B_VE = 7,    // 2: V stage consumed
    B_SF = 9,    // 2: S_X ready (per tile)
    B_PF = 11,   // 2: P_X written (per tile, 256 arrivals)
    B_OF = 13,   // 2: O_X final (per tile)
    B_VFIX = 15, // V tail zeroed
    B_FIN = 16,
    B_NUM = 17
};

constexpr uint32_t kTmemCols = 512;
constexpr int kThreads = 576;
constexpr int kSoftmaxThreads = 256; // per tile: 128 rows x 2 halves

struct TileGeo {
    int rows;  // valid query rows (0 = tile absent)
    int p_min; // position of the first token
    int p_max; // position of the last token
    int nkt;   // 128-key steps the tile needs
};

__device__ __forceinline__ int blocks_in_step(int n_keys, int j)
{
    return (min(kPrefillKeys, n_keys - j * kPrefillKeys) + kBlockSize - 1) / kBlockSize;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1) prefill_kernel(const __grid_constant__ CUtensorMap tm_q,
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
    const uint32_t bar = sbase + Cfg::kOffBar;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + Cfg::kOffBar + B_NUM * 8);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + Cfg::kOffBar + B_NUM * 8 + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // ---- geometry of the q-pair (identical in every thread)
    const int2 work = p.pf_tiles[u];
    const int r = work.x, qp = work.y;
    const int G = p.G;
    const int TQ = kPrefillRows / G; // tokens per 128-row tile
    const int qs = p.qsl[r];
    const int q_len = p.qsl[r + 1] - qs;
    const int L = p.seq_lens[r];
    const int ctx = L - q_len;
    TileGeo tg[2];
#pragma unroll
    for (int x = 0; x < 2; ++x) {
        const int tok0 = (2 * qp + x) * TQ;
        const int n_tok = max(0, min(TQ, q_len - tok0));
        tg[x].rows = n_tok * G;
        tg[x].p_min = ctx + tok0;
        tg[x].p_max = ctx + tok0 + n_tok - 1;
        tg[x].nkt = n_tok ? (tg[x].p_max + kPrefillKeys) / kPrefillKeys : 0;
    }
    const int n_steps = max(tg[0].nkt, tg[1].nkt);
    const int n_keys_all = (tg[1].rows ? tg[1].p_max : tg[0].p_max) + 1; // keys the CTA loads
    const bool tail_fix = (L % kBlockSize) != 0 && (n_keys_all - 1) / kBlockSize == (L - 1) / kBlockSize;
    const int32_t *bt_row = p.bt + (int64_t)r * p.bt_stride;

    // ---- setup: barriers, TMEM
    if (threadIdx.x == 0) {
        mbar_init(bar + B_Q * 8, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(bar + (B_KF + s) * 8, 1);
            mbar_init(bar + (B_KE + s) * 8, 1);
            mbar_init(bar + (B_VF + s) * 8, 1);
            mbar_init(bar + (B_VE + s) * 8, 1);
            mbar_init(bar + (B_SF + s) * 8, 1);
            mbar_init(bar + (B_PF + s) * 8, kSoftmaxThreads);
            mbar_init(bar + (B_OF + s) * 8, 1);
        }
        mbar_init(bar + B_VFIX * 8, 1);
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
        // ===================================================== TMA producer
        if (lane == 0) {
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            const int ntiles = tg[1].rows ? 2 : 1;
            mbar_arrive_expect_tx(bar + B_Q * 8, ntiles * Cfg::kTile);
            for (int x = 0; x < ntiles; ++x)
#pragma unroll
                for (int hf = 0; hf < Cfg::kHalves; ++hf)
                    tma_load_3d(sQ + x * Cfg::kTile + hf * Cfg::kHalfBytes, &tm_q, hf * 64, h * G,
                                qs + (2 * qp + x) * TQ, bar + B_Q * 8);
        }
        bool ok = true;
        for (int j = 0; j < n_steps; ++j) {
            const int st = j & 1;
            const int nblk = blocks_in_step(n_keys_all, j);
            int y = -kBlockSize; // out-of-bounds box: TMA fills zeros
            if (lane < nblk) {
                const int bid = bt_row[j * (kPrefillKeys / kBlockSize) + lane];
                if ((unsigned)bid < (unsigned long long)p.num_blocks)
                    y = (bid * p.Hkv + h) * kBlockSize;
                else
                    atomicOr(&p.hdr->status, PA_DEVICE_BAD_BLOCK);
            }
            const uint32_t tx = (uint32_t)(nblk * kBlockSize * D * 2);
            // K(j) into stage st once K(j-2) is consumed
            if (j >= 2 && !mbar_wait_warp(bar + (B_KE + st) * 8, ((j - 2) >> 1) & 1, abort_flag)) {
                ok = false;
                break;
            }
            if (lane == 0)
                mbar_arrive_expect_tx(bar + (B_KF + st) * 8, tx);
            __syncwarp();
            if (lane < nblk)
#pragma unroll
                for (int hf = 0; hf < Cfg::kHalves; ++hf)
                    tma_load_2d(sK0 + st * Cfg::kTile + hf * Cfg::kHalfBytes + lane * (kBlockSize * 128), &tm_k,
                                hf * 64, y, bar + (B_KF + st) * 8);
            // V(j) into stage st once V(j-2) is consumed
            if (j >= 2 && !mbar_wait_warp(bar + (B_VE + st) * 8, ((j - 2) >> 1) & 1, abort_flag)) {
                ok = false;
                break;
            }
            if (lane == 0)
                mbar_arrive_expect_tx(bar + (B_VF + st) * 8, tx);
            __syncwarp();
            if (lane < nblk)
#pragma unroll
                for (int hf = 0; hf < Cfg::kHalves; ++hf)
                    tma_load_2d(sV0 + st * Cfg::kTile + hf * Cfg::kHalfBytes + lane * (kBlockSize * 128), &tm_v,
                                hf * 64, y, bar + (B_VF + st) * 8);
            if (tail_fix && j == n_steps - 1) {
                // zero the V rows past the end of the sequence in its last block
                if (!mbar_wait_warp(bar + (B_VF + st) * 8, (j >> 1) & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                const int lb = (L - 1) / kBlockSize - j * (kPrefillKeys / kBlockSize);
                const int first = L % kBlockSize;
                const int nrow = kBlockSize - first;
                const int nz = nrow * Cfg::kHalves * 8; // 16-byte chunks
                for (int i = lane; i < nz; i += 32) {
                    const int chunk = i & 7;
                    const int rr = (i >> 3) % nrow;
                    const int hf = (i >> 3) / nrow;
                    const uint32_t addr = sV0 + st * Cfg::kTile + hf * Cfg::kHalfBytes +
                                          (lb * kBlockSize + first + rr) * 128 + chunk * 16;
                    asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(addr), "r"(0u) : "memory");
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(bar + B_VFIX * 8);
            }
        }
        if (!ok && lane == 0)
            fail();
    } else if (warp == 1) {
        // ===================================================== MMA issuer (one thread)
        if (lane == 0) {
            constexpr uint32_t idesc_s = idesc_bf16_f32(128, kPrefillKeys, 0, 0);
            constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, 0, 1);
            bool ok = mbar_wait(bar + B_Q * 8, 0, abort_flag);
            // Descriptors are built once; per MMA only the 14-bit start-address field moves, by a
            // constant number of 16-byte units (shared addresses stay below 2^18, so no carry).
            const uint64_t dq = smem_desc_sw128(sQ, 16, 1024);
            const uint64_t dk = smem_desc_sw128(sK0, 16, 1024);
            const uint64_t dv = smem_desc_sw128(sV0, Cfg::kHalfBytes, 1024);
            const int pmax0 = tg[0].p_max, pmax1 = tg[1].p_max;
            auto issue_s = [&](int x, int j) {
                const uint64_t bq = dq + (uint64_t)((x * Cfg::kTile) >> 4);
                const uint64_t bk = dk + (uint64_t)(((j & 1) * Cfg::kTile) >> 4);
                const uint32_t d_tmem = tmem + col_s(x);
                if constexpr (D == 128) {
                    // k-steps 0..7: +32 B inside a 128-byte swizzle row, +16 KB to the second 64-column half
                    constexpr uint32_t H = Cfg::kHalfBytes >> 4;
                    umma_f16_x8_ss<0, 2, 4, 6, H, H + 2, H + 4, H + 6>(d_tmem, bq, bk, idesc_s, 0u);
                } else {
#pragma unroll
                    for (int ks = 0; ks < kKS; ++ks) {
                        const uint64_t off = (uint64_t)(((ks >> 2) * Cfg::kHalfBytes + (ks & 3) * 32) >> 4);
                        umma_f16(d_tmem, bq + off, bk + off, idesc_s, ks > 0 ? 1u : 0u);
                    }
                }
                umma_commit(bar + (B_SF + x) * 8);
            };
            auto issue_pv = [&](int x, int j) {
                const uint64_t bv = dv + (uint64_t)(((j & 1) * Cfg::kTile) >> 4);
                const int nblk = blocks_in_step((x ? pmax1 : pmax0) + 1, j);
                const uint32_t d_tmem = tmem + col_o(x);
                const uint32_t a_tmem = tmem + col_s(x);
                if (nblk == kPrefillKeys / kBlockSize) {
                    umma_f16_x8_ts<((kBlockSize * 128) >> 4)>(d_tmem, a_tmem, bv, idesc_pv, j > 0 ? 1u : 0u);
                } else {
                    for (int kk = 0; kk < nblk; ++kk)
                        umma_f16_ts(d_tmem, a_tmem + kk * 8, bv + (uint64_t)((kk * kBlockSize * 128) >> 4),
                                    idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
                }
            };
            // prologue: S(0) for both tiles
            if (ok && !mbar_wait(bar + B_KF * 8, 0, abort_flag))
                ok = false;
            if (ok) {
                tc_fence_after();
                for (int x = 0; x < 2; ++x)
                    if (tg[x].nkt > 0)
                        issue_s(x, 0);
                umma_commit(bar + B_KE * 8); // K(0) consumed
            }
            for (int j = 0; ok && j < n_steps; ++j) {
                const int st = j & 1;
                bool v_ready = false, k_ready = false;
                for (int x = 0; x < 2; ++x) {
                    if (j >= tg[x].nkt)
                        continue;
                    if (!mbar_wait(bar + (B_PF + x) * 8, j & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    if (!v_ready) {
                        const bool fix = tail_fix && j == n_steps - 1;
                        if (!mbar_wait(bar + (fix ? B_VFIX : (B_VF + st)) * 8, fix ? 0u : (uint32_t)((j >> 1) & 1),
                                       abort_flag)) {
                            ok = false;
                            break;
                        }
                        v_ready = true;
                    }
                    tc_fence_after();
                    issue_pv(x, j);
                    if (j + 1 < tg[x].nkt) {
                        if (!k_ready) {
                            if (!mbar_wait(bar + (B_KF + (st ^ 1)) * 8, ((j + 1) >> 1) & 1, abort_flag)) {
                                ok = false;
                                break;
                            }
                            k_ready = true;
                            tc_fence_after();
                        }
                        issue_s(x, j + 1);
                    } else {
                        umma_commit(bar + (B_OF + x) * 8);
                    }
                }
                if (!ok)
                    break;
                umma_commit(bar + (B_VE + st) * 8); // V(j) consumed
                if (j + 1 < n_steps)
                    umma_commit(bar + (B_KE + (st ^ 1)) * 8); // K(j+1) consumed
            }
            if (!ok)
                fail();
            // drain: nothing of ours may still be running on the tensor core at dealloc
            umma_commit(bar + B_FIN * 8);
            (void)mbar_wait(bar + B_FIN * 8, 0);
        }
    } else {
        // ===================================================== softmax / epilogue (warps 2..9: A, 10..17: B)
        const int x = (warp - 2) >> 3;          // tile
        const int half = ((warp - 2) >> 2) & 1; // 64-key half of the row (and half of the head dim)
        const TileGeo g = x ? tg[1] : tg[0];
        if (g.rows > 0) {
            const int quad = warp & 3;        // TMEM lane quadrant this warp may access
            const int row = quad * 32 + lane; // query row of the tile = TMEM lane
            const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
            const uint32_t tS = tmem + lane_addr + col_s(x);
            const uint32_t tO = tmem + lane_addr + col_o(x) + half * (D / 2);
            const int bar_id = 1 + x * 4 + quad; // named barrier of the two warps sharing these rows
            float *xch = reinterpret_cast<float *>(smem + Cfg::kOffX) + x * (2 * 2 * 128);
            const int p_row = row < g.rows ? g.p_min + row / G : g.p_max;
            const float c = p.scale_log2;
            const float thresh = 8.f / c;      // 2^8 growth, in raw score units
            float m_ref = -CUDART_INF_F;       // reference max, raw score units (same in both halves)
            uint64_t l2 = f2_pack(0.f, 0.f);   // exact fp32 partial row sum of this half
            bool ok = true;
            for (int j = 0; j < g.nkt; ++j) {
                if (!mbar_wait_warp(bar + (B_SF + x) * 8, j & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const int key0 = j * kPrefillKeys + half * 64;
                const bool diag = j * kPrefillKeys + kPrefillKeys - 1 > g.p_min; // causal mask needed
                uint32_t sv[64];
                tmem_ld32p(tS + half * 64, sv);
                tmem_ld32p(tS + half * 64 + 32, sv + 32);
                tmem_wait_ld();
                if (diag) {
#pragma unroll
                    for (int i = 0; i < 64; ++i)
                        if (key0 + i > p_row)
                            sv[i] = __float_as_uint(-CUDART_INF_F);
                }
                float mx = -CUDART_INF_F;
#pragma unroll
                for (int i = 0; i < 64; i += 2)
                    mx = fmax3(mx, __uint_as_float(sv[i]), __uint_as_float(sv[i + 1]));
                // combine with the other half of the row (double-buffered by step parity)
                float *slot = xch + (j & 1) * 256;
                slot[half * 128 + row] = mx;
                asm volatile("bar.sync %0, 64;" ::"r"(bar_id) : "memory");
                mx = fmaxf(mx, slot[(half ^ 1) * 128 + row]);
                float alpha = 1.f;
                if (j == 0) {
                    m_ref = mx;
                } else if (mx > m_ref + thresh) {
                    alpha = fast_exp2((m_ref - mx) * c);
                    m_ref = mx;
                }
                l2 = f2_mul(l2, f2_pack(alpha, alpha));
                // P = exp2(s*c - m*c) -> bf16 pairs -> TMEM columns [32*half, 32*half + 32) of S_X.
                // Both halves finished reading S before the barrier above.
                const uint64_t c2 = f2_pack(c, c);
                const float nm = -m_ref * c;
                const uint64_t nm2 = f2_pack(nm, nm);
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    uint32_t w[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        float e0, e1;
                        f2_unpack(f2_fma(f2_pack(__uint_as_float(sv[cc * 16 + 2 * i]),
                                                 __uint_as_float(sv[cc * 16 + 2 * i + 1])),
                                         c2, nm2),
                                  e0, e1);
                        const float p0 = fast_exp2(e0), p1 = fast_exp2(e1);
                        l2 = f2_add(l2, f2_pack(p0, p1));
                        w[i] = pack_bf16x2(p0, p1);
                    }
                    tmem_st8(tS + half * 32 + cc * 8, w);
                }
                if (__any_sync(0xffffffffu, alpha != 1.f)) {
                    // O_X is stable (S_X(j) completing implies PV_X(j-1) completed) and PV_X(j)
                    // cannot start before the arrive below: rescale this thread's half of the row
#pragma unroll 1
                    for (int cc = 0; cc < D / 32; ++cc) {
                        uint32_t o[16];
                        tmem_ld16(tO + cc * 16, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
                        tmem_st16(tO + cc * 16, o);
                    }
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(bar + (B_PF + x) * 8);
            }
            // ---- epilogue: O / l -> bf16 (this thread: half of the head dim)
            if (ok && !mbar_wait_warp(bar + (B_OF + x) * 8, 0, abort_flag))
                ok = false;
            float la, lb;
            f2_unpack(l2, la, lb);
            float l_half = la + lb;
            // full row sum = both halves' partial sums (exchange slot of parity nkt&1 is free)
            float *slot = xch + (g.nkt & 1) * 256;
            slot[half * 128 + row] = l_half;
            asm volatile("bar.sync %0, 64;" ::"r"(bar_id) : "memory");
            const float l_sum = l_half + slot[(half ^ 1) * 128 + row];
            if (!ok) {
                if (lane == 0)
                    fail();
            } else {
                tc_fence_after();
                const float inv = l_sum > 0.f ? 1.f / l_sum : 0.f;
                const bool store = row < g.rows;
                const int t = qs + (2 * qp + x) * TQ + row / G;
                const int hq = h * G + row % G;
                __nv_bfloat16 *dst = p.out + ((int64_t)t * p.Hq + hq) * D + half * (D / 2);
#pragma unroll 1
                for (int cc = 0; cc < D / 32; ++cc) {
                    uint32_t o[16];
                    tmem_ld16(tO + cc * 16, o);
                    tmem_wait_ld();
                    if (store) {
#pragma unroll
                        for (int i = 0; i < 16; i += 8) {
                            uint4 v;
                            v.x = pack_bf16x2(__uint_as_float(o[i]) * inv, __uint_as_float(o[i + 1]) * inv);
                            v.y = pack_bf16x2(__uint_as_float(o[i + 2]) * inv, __uint_as_float(o[i + 3]) * inv);
                            v.z = pack_bf16x2(__uint_as_float(o[i + 4]) * inv, __uint_as_float(o[i + 5]) * inv);
                            v.w = pack_bf16x2(__uint_as_float(o[i + 6]) * inv, __uint_as_float(o[i + 7]) * inv);
                            *reinterpret_cast<uint4 *>(dst + cc * 16 + i) = v;
                        }
                    }
                }
                if (store && p.lse && half == 0)
                    p.lse[(int64_t)t * p.Hq + hq] =
                        l_sum > 0.f ? (m_ref * c + log2f(l_sum)) * 0.69314718055994531f : -CUDART_INF_F;
            }
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
    prefill_kernel<D><<<grid, kThreads, smem, s>>>(tq, tk, tv, p);
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
