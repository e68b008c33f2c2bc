// prefill.cu -- chunked-prefill attention over the paged cache on the 5th-gen
// tensor cores (tcgen05.mma, accumulators and P in TMEM).
//
// Prefill is compute bound (hn.213312.xyz section 一, scheduler paragraph;
// shengyayun.com 适用场景).  A chunk of q_len tokens at positions
// c_r .. c_r+q_len-1 attends causally to its request's cached context plus the
// chunk itself; chunking does not change any row's result (hn.213312.xyz
// section 二.1) because every row depends only on its own position.
//
// Work item = (request r, q-pair, kv head h).  A q-pair is two tiles A and B of
// 128 query rows each; a tile is 128/G tokens x the G query heads that share
// kv head h (token-major), so one K/V tile feeds every head of the group and
// both tiles.  The kernel is persistent: one CTA per SM walks the cost-sorted work
// list in snake order, and every ring, barrier phase and counter carries over from one
// item to the next, so the next item's Q load and first QK^T overlap the
// previous item's last steps and epilogue.
//
// Warpgroup roles (512 threads, one CTA per SM; registers moved between the
// warpgroups with setmaxnreg so that a softmax thread can hold a whole row):
//   WG 0, WG 1  softmax of tile A and of tile B: one thread per query row
//               (= TMEM lane), all 128 scores of a key step in registers after
//               one tcgen05.ld pass.  Causal mask by select, P = exp2(s*c - m*c)
//               with packed fp32x2 FMAs, bf16 P back into TMEM over S with
//               tcgen05.st.  The reference max m moves (and O is rescaled in
//               TMEM) only when a row's max grows by more than 2^8 (a stale max
//               leaves the normalised result unchanged), so after an item's first
//               step the exponentials run against the current m with the step's
//               row max taken alongside, and a step is redone max-first only when
//               that max passed the threshold.  After a tile's last step the row
//               sum and max go to the epilogue warpgroup through shared memory
//               and the softmax moves straight on to its next item.
//   WG 2        epilogue of both tiles: waits for a tile's final O, writes O / l
//               as bf16 (and the LSE), then frees O for the next item's first PV.
//   WG 3        warp 12: TMA producer -- per item both Q tiles (3-D boxes
//               {64 d, G heads, 128/G tokens}, 128-byte swizzle) once the
//               previous item's last QK^T is done, then per 128-key step the K
//               tile and the V tile (8 paged blocks x 64-column halves, 2-D
//               boxes) into separate 2-stage rings;
//               warp 13: TMEM allocation (512 columns: S_A, O_A, S_B, O_B) and
//               the MMAs (one elected lane issues, the warp stays converged; it
//               reads each item's geometry one item ahead), in the order
//                 PV_A(j-1), S_A(j), PV_B(j-1), S_B(j)   (ping-pong)
//               so the tensor core works on one tile while the other tile's
//               softmax runs.  S = Q K^T is SS (both operands in smem);
//               O += P V reads P from TMEM (written over S by the softmax) and V
//               from smem as an MN-major operand.  Each group of 8 MMAs is
//               issued from one asm block with prebuilt descriptors.
// Ordering facts the pipeline relies on: a commit fires only once every
// earlier MMA of the issuing thread is done, so when the softmax sees S_X(j)
// the previous PV_X(j-1) has finished with P_X and O_X; and MMAs issued by one
// thread run in issue order, so S_X(j) (which overwrites the TMEM columns
// holding P_X(j-1)) runs after PV_X(j-1) has read them.
// V rows past the end of the sequence in its last block (unused slots) are
// zeroed in shared memory by the producer before any PV reads them, so 0 * NaN
// never enters O.
#include <math_constants.h>

#include <mutex>

#include "pa_internal.cuh"
#include "tcgen05.cuh"

namespace pa {
namespace {

constexpr int kStepKeys = 128;                     // keys per step (8 paged blocks)
constexpr int kStepBlocks = kStepKeys / kBlockSize;

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
    static constexpr int kOffLM = kOffBar + kBarBytes; // row sum and max for the epilogue: [tile][item parity][l|m][128] fp32
    static constexpr int kLMBytes = 2 * 2 * 2 * 128 * 4;
    static constexpr int kUsed = kOffLM + kLMBytes + 1024;
    // keep one CTA per SM (each CTA allocates all 512 TMEM columns)
    static constexpr int kSmem = kUsed > 120 * 1024 ? kUsed : 120 * 1024;
};

// TMEM columns of the two tiles' S (P aliases its first 64 columns) and O
__device__ __forceinline__ int col_s(int x) { return x * 256; }
__device__ __forceinline__ int col_o(int x) { return x * 256 + 128; }

enum PfBar {
    B_Q = 0,     // Q tiles of an item loaded
    B_QE = 1,    // Q tiles of an item consumed by its last QK^T
    B_KF = 2,    // 2: K stage full
    B_KE = 4,    // 2: K stage consumed
    B_VF = 6,    // 2: V stage full
    B_VE = 8,    // 2: V stage consumed
    B_SF = 10,   // 2: S_X ready (per tile)
    B_PF = 12,   // 2: P_X written (per tile, one arrival per row)
    B_OF = 14,   // 2: O_X of an item final (per tile)
    B_OE = 16,   // 2: O_X of an item read by the epilogue (per tile, one arrival per row)
    B_LF = 18,   // 2: row sums and maxima of an even item of tile X in shared memory (one arrival per row)
    B_VFIX = 20, // V tail of an even tail-fixed item zeroed
    B_FIN = 21,
    B_LF1 = 22,  // 2: as B_LF, odd items of tile X
    B_VFIX1 = 24, // as B_VFIX, odd tail-fixed items
    B_NUM = 25
};

// The two signals without a reply of their own (the row sums for the epilogue, the zeroed V tail
// for the MMA issuer) alternate between two barriers by item parity.  With one barrier a one-step
// item could complete the next phase before the waiter had seen the previous one, and the waiter,
// which tracks phases by parity, would then wait for good.  With two, the same barrier is reused two
// items later, and by then the waiter has provably passed: the epilogue releases O_X (which the MMA
// issuer waits for before the in-between item's first PV), and the V ring stage two steps back is
// released only after the issuer's wait.
__device__ __forceinline__ int bar_lf(int x, uint32_t item) { return ((item & 1) ? B_LF1 : B_LF) + x; }
__device__ __forceinline__ int bar_vfix(uint32_t n) { return (n & 1) ? B_VFIX1 : B_VFIX; }

constexpr uint32_t kTmemCols = 512;
constexpr int kThreads = 512;
constexpr int kRowThreads = 128; // one thread per query row of a tile
// Registers per thread of each warpgroup after the split (the launch gives every thread
// 65536 / 512 = 128): two softmax warpgroups hold a whole 128-key row of scores, the
// epilogue and control warpgroups need little.
constexpr int kRegSoftmax = 184;
constexpr int kRegEpilogue = 72;
constexpr int kRegControl = 72;
constexpr int kRegSplit = kRowThreads * (2 * kRegSoftmax + kRegEpilogue + kRegControl);
static_assert(kRegSplit <= 65536, "the warpgroup budgets must fit the CTA's register pool");

struct TileGeo {
    int rows;  // valid query rows (0 = tile absent)
    int p_min; // position of the first token
    int p_max; // position of the last token
    int nkt;   // 128-key steps the tile needs
};

struct ItemGeo {
    int r, qp, h, qs, L, tok0; // tok0: first token of tile A within the request
    TileGeo t0, t1;
    int n_steps, n_keys_all;
    bool tail_fix;
};

__device__ __forceinline__ ItemGeo item_geo(const AttnParams &p, int item)
{
    ItemGeo g;
    const int u = item / p.Hkv;
    g.h = item - u * p.Hkv;
    const int2 work = p.pf_tiles[u];
    g.r = work.x;
    g.qp = work.y;
    const int TQ = kPrefillRows / p.G;
    g.qs = p.qsl[g.r];
    const int q_len = p.qsl[g.r + 1] - g.qs;
    g.L = p.seq_lens[g.r];
    const int ctx = g.L - q_len;
    g.tok0 = 2 * g.qp * TQ;
    const int n0 = max(0, min(TQ, q_len - g.tok0));
    const int n1 = max(0, min(TQ, q_len - g.tok0 - TQ));
    g.t0.rows = n0 * p.G;
    g.t0.p_min = ctx + g.tok0;
    g.t0.p_max = g.t0.p_min + n0 - 1;
    g.t0.nkt = n0 ? (g.t0.p_max + kStepKeys) / kStepKeys : 0;
    g.t1.rows = n1 * p.G;
    g.t1.p_min = ctx + g.tok0 + TQ;
    g.t1.p_max = g.t1.p_min + n1 - 1;
    g.t1.nkt = n1 ? (g.t1.p_max + kStepKeys) / kStepKeys : 0;
    g.n_steps = max(g.t0.nkt, g.t1.nkt);
    g.n_keys_all = (n1 ? g.t1.p_max : g.t0.p_max) + 1;
    g.tail_fix = (g.L % kBlockSize) != 0 && (g.n_keys_all - 1) / kBlockSize == (g.L - 1) / kBlockSize;
    return g;
}

// What the MMA issuer needs of an item (read one item ahead: item_geo's loads are two dependent
// round trips to L2, which at an item boundary would stall the issuer while both tiles wait for S).
struct MmaGeo {
    int nkt[2], pmax[2], n_steps;
    bool tail_fix;
};

__device__ __forceinline__ MmaGeo mma_geo(const AttnParams &p, int item)
{
    const ItemGeo g = item_geo(p, item);
    MmaGeo m;
    m.nkt[0] = g.t0.nkt;
    m.nkt[1] = g.t1.nkt;
    m.pmax[0] = g.t0.p_max;
    m.pmax[1] = g.t1.p_max;
    m.n_steps = g.n_steps;
    m.tail_fix = g.tail_fix;
    return m;
}

// The k-th work item of this CTA.  The work list is sorted by cost, most expensive
// first; walking it in snake order (CTA b takes item b of even rounds and item
// n-1-b of odd rounds, n working CTAs) pairs heavy with light items, so the CTAs
// finish together.
__device__ __forceinline__ int snake_item(int k, int n_ctas)
{
    const int b = (k & 1) ? n_ctas - 1 - (int)blockIdx.x : (int)blockIdx.x;
    return k * n_ctas + b;
}

__device__ __forceinline__ int blocks_in_step(int n_keys, int j)
{
    return (min(kStepKeys, n_keys - j * kStepKeys) + kBlockSize - 1) / kBlockSize;
}

// P = exp2(s*c - m*c) of one thread's 128-score row -> bf16 pairs -> TMEM columns [0, 64) of its S (all of
// S was read before), the row's sum added into two packed chains s2a / s2b; with MAX the row max of the scores is
// taken alongside into m2 (two chains: few registers, and off the critical path behind the exponentials).
template <bool MAX>
__device__ __forceinline__ void softmax_exps(const uint32_t (&sv)[128], float c, float m_use, uint32_t tS,
                                             uint64_t &s2a, uint64_t &s2b, float (&m2)[2])
{
    const uint64_t c2 = f2_pack(c, c);
    const float nm = -m_use * c;
    const uint64_t nm2 = f2_pack(nm, nm);
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) {
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const float s0 = __uint_as_float(sv[cc * 32 + 2 * i]);
            const float s1 = __uint_as_float(sv[cc * 32 + 2 * i + 1]);
            float e0, e1;
            f2_unpack(f2_fma(f2_pack(s0, s1), c2, nm2), e0, e1);
            const float p0 = fast_exp2(e0), p1 = fast_exp2(e1);
            if (i & 1)
                s2b = f2_add(s2b, f2_pack(p0, p1));
            else
                s2a = f2_add(s2a, f2_pack(p0, p1));
            w[i] = pack_bf16x2(p0, p1);
            if constexpr (MAX)
                m2[i & 1] = fmax3(m2[i & 1], s0, s1);
        }
        tmem_st16(tS + cc * 16, w);
    }
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1) prefill_kernel(const __grid_constant__ CUtensorMap tm_q,
                                                              const __grid_constant__ CUtensorMap tm_k,
                                                              const __grid_constant__ CUtensorMap tm_v,
                                                              const AttnParams p)
{
    using Cfg = PfCfg<D>;
    if (blockIdx.x == 0 && threadIdx.x == 0)
        p.hdr->write_epoch = kWriteEpochIdle; // the step's write launch (if any) has finished
    const int n_items = (int)p.hdr->n_pf_tiles * p.Hkv;
    // CTAs that take work: the plan's share of the SMs for prefill (the rest go to decode)
    const int n_ctas = min(min((int)gridDim.x, n_items), max(1, (int)p.hdr->pf_ctas));
    if ((int)blockIdx.x >= n_ctas || (p.hdr->status & PA_DEVICE_WAIT_TIMEOUT))
        return; // no work for this CTA (its SM is left to decode), or an earlier CTA gave up

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t sQ = sbase + Cfg::kOffQ;
    const uint32_t sK0 = sbase + Cfg::kOffK;
    const uint32_t sV0 = sbase + Cfg::kOffV;
    const uint32_t bar = sbase + Cfg::kOffBar;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + Cfg::kOffBar + B_NUM * 8);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + Cfg::kOffBar + B_NUM * 8 + 4);
    float *lm_all = reinterpret_cast<float *>(smem + Cfg::kOffLM);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int wg = warp >> 2;
    const int G = p.G;
    const int TQ = kPrefillRows / G; // tokens per 128-row tile
    constexpr int kProducerWarp = 12, kMmaWarp = 13;

    // ---- setup: barriers, TMEM
    if (threadIdx.x == 0) {
        mbar_init(bar + B_Q * 8, 1);
        mbar_init(bar + B_QE * 8, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(bar + (B_KF + s) * 8, 1);
            mbar_init(bar + (B_KE + s) * 8, 1);
            mbar_init(bar + (B_VF + s) * 8, 1);
            mbar_init(bar + (B_VE + s) * 8, 1);
            mbar_init(bar + (B_SF + s) * 8, 1);
            mbar_init(bar + (B_PF + s) * 8, kRowThreads);
            mbar_init(bar + (B_OF + s) * 8, 1);
            mbar_init(bar + (B_OE + s) * 8, kRowThreads);
            mbar_init(bar + (B_LF + s) * 8, kRowThreads);
            mbar_init(bar + (B_LF1 + s) * 8, kRowThreads);
        }
        mbar_init(bar + B_VFIX * 8, 1);
        mbar_init(bar + B_VFIX1 * 8, 1);
        mbar_init(bar + B_FIN * 8, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == kMmaWarp) {
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

    if (wg == 3) {
        wg_reg_lower<kRegControl>();
        if (warp == kProducerWarp) {
            // ===================================================== TMA producer
            if (lane == 0) {
                tma_prefetch_desc(&tm_q);
                tma_prefetch_desc(&tm_k);
                tma_prefetch_desc(&tm_v);
            }
            bool ok = true;
            uint32_t gs = 0;   // K/V steps loaded so far by this CTA
            uint32_t nq = 0;   // items whose Q was loaded
            uint32_t nfix = 0; // items whose V tail was zeroed
            for (int k = 0, item = snake_item(0, n_ctas); ok && item < n_items; item = snake_item(++k, n_ctas)) {
                const ItemGeo g = item_geo(p, item);
                // Q of this item, once the previous item's last QK^T has read the old Q
                if (nq > 0 && !mbar_wait_warp(bar + B_QE * 8, (nq - 1) & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                if (lane == 0) {
                    const int ntiles = g.t1.rows ? 2 : 1;
                    const uint64_t pol = l2_policy_evict_first(); // each Q row is read by one item only
                    mbar_arrive_expect_tx(bar + B_Q * 8, ntiles * Cfg::kTile);
                    for (int x = 0; x < ntiles; ++x)
#pragma unroll
                        for (int hf = 0; hf < Cfg::kHalves; ++hf)
                            tma_load_3d_hint(sQ + x * Cfg::kTile + hf * Cfg::kHalfBytes, &tm_q, hf * 64, g.h * G,
                                             g.qs + g.tok0 + x * TQ, bar + B_Q * 8, pol);
                }
                ++nq;
                const int32_t *bt_row = p.bt + (int64_t)g.r * p.bt_stride;
                for (int j = 0; j < g.n_steps; ++j, ++gs) {
                    const int st = gs & 1;
                    const int nblk = blocks_in_step(g.n_keys_all, j);
                    // HND: 2-D map, row (bid*Hkv + h)*16;  NHD: 3-D map, (head h, token row bid*16)
                    int y = -kBlockSize; // out-of-bounds box: TMA fills zeros
                    if (lane < nblk) {
                        const int bid = bt_row[j * kStepBlocks + lane];
                        if ((unsigned)bid < (unsigned long long)p.num_blocks)
                            y = (p.nhd ? bid : bid * p.Hkv + g.h) * kBlockSize;
                        else
                            atomicOr(&p.hdr->status, PA_DEVICE_BAD_BLOCK);
                    }
                    const uint32_t tx = (uint32_t)(nblk * kBlockSize * D * 2);
                    const uint32_t ph_prev = ((gs >> 1) - 1) & 1; // phase of this stage's previous use
                    // K into stage st once the K two steps back is consumed
                    if (gs >= 2 && !mbar_wait_warp(bar + (B_KE + st) * 8, ph_prev, abort_flag)) {
                        ok = false;
                        break;
                    }
                    if (lane == 0)
                        mbar_arrive_expect_tx(bar + (B_KF + st) * 8, tx);
                    __syncwarp();
                    if (lane < nblk)
#pragma unroll
                        for (int hf = 0; hf < Cfg::kHalves; ++hf) {
                            const uint32_t dst = sK0 + st * Cfg::kTile + hf * Cfg::kHalfBytes + lane * (kBlockSize * 128);
                            if (p.nhd)
                                tma_load_3d(dst, &tm_k, hf * 64, g.h, y, bar + (B_KF + st) * 8);
                            else
                                tma_load_2d(dst, &tm_k, hf * 64, y, bar + (B_KF + st) * 8);
                        }
                    // V into stage st once the V two steps back is consumed
                    if (gs >= 2 && !mbar_wait_warp(bar + (B_VE + st) * 8, ph_prev, abort_flag)) {
                        ok = false;
                        break;
                    }
                    if (lane == 0)
                        mbar_arrive_expect_tx(bar + (B_VF + st) * 8, tx);
                    __syncwarp();
                    if (lane < nblk)
#pragma unroll
                        for (int hf = 0; hf < Cfg::kHalves; ++hf) {
                            const uint32_t dst = sV0 + st * Cfg::kTile + hf * Cfg::kHalfBytes + lane * (kBlockSize * 128);
                            if (p.nhd)
                                tma_load_3d(dst, &tm_v, hf * 64, g.h, y, bar + (B_VF + st) * 8);
                            else
                                tma_load_2d(dst, &tm_v, hf * 64, y, bar + (B_VF + st) * 8);
                        }
                    if (g.tail_fix && j == g.n_steps - 1) {
                        // zero the V rows past the end of the sequence in its last block
                        if (!mbar_wait_warp(bar + (B_VF + st) * 8, (gs >> 1) & 1, abort_flag)) {
                            ok = false;
                            break;
                        }
                        const int lb = (g.L - 1) / kBlockSize - j * kStepBlocks;
                        const int first = g.L % kBlockSize;
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
                            mbar_arrive(bar + bar_vfix(nfix) * 8);
                        ++nfix;
                    }
                }
            }
            if (!ok && lane == 0)
                fail();
        } else if (warp == kMmaWarp) {
            // ===================================================== MMA issuer (whole warp, one elected lane issues)
            constexpr uint32_t idesc_s = idesc_bf16_f32(128, kStepKeys, 0, 0);
            constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, 0, 1);
            // Descriptors are built once; per MMA only the 14-bit start-address field moves, by a
            // constant number of 16-byte units (shared addresses stay below 2^18, so no carry).
            const uint64_t dq = smem_desc_sw128(sQ, 16, 1024);
            const uint64_t dk = smem_desc_sw128(sK0, 16, 1024);
            const uint64_t dv = smem_desc_sw128(sV0, Cfg::kHalfBytes, 1024);
            auto issue_s = [&](int x, uint32_t gstep) {
                const uint64_t bq = dq + (uint64_t)((x * Cfg::kTile) >> 4);
                const uint64_t bk = dk + (uint64_t)(((gstep & 1) * Cfg::kTile) >> 4);
                const uint32_t d_tmem = tmem + col_s(x);
                if constexpr (D == 128) {
                    // k-steps 0..7: +32 B inside a 128-byte swizzle row, +16 KB to the second 64-column half
                    constexpr uint32_t H = Cfg::kHalfBytes >> 4;
                    umma_f16_x8_ss<0, 2, 4, 6, H, H + 2, H + 4, H + 6>(d_tmem, bq, bk, idesc_s, 0u);
                } else {
                    static_assert(D == 64, "head_dim 64 or 128");
                    umma_f16_x4_ss<2, 4, 6>(d_tmem, bq, bk, idesc_s); // k-steps 0..3: +32 B in the swizzle row
                }
                umma_commit(bar + (B_SF + x) * 8);
            };
            auto issue_pv = [&](int x, int j, uint32_t gstep, int p_max) {
                const uint64_t bv = dv + (uint64_t)(((gstep & 1) * Cfg::kTile) >> 4);
                const int nblk = blocks_in_step(p_max + 1, j);
                const uint32_t d_tmem = tmem + col_o(x);
                const uint32_t a_tmem = tmem + col_s(x);
                if (nblk == kStepBlocks) {
                    umma_f16_x8_ts<((kBlockSize * 128) >> 4)>(d_tmem, a_tmem, bv, idesc_pv, j > 0 ? 1u : 0u);
                } else {
                    for (int kk = 0; kk < nblk; ++kk)
                        umma_f16_ts(d_tmem, a_tmem + kk * 8, bv + (uint64_t)((kk * kBlockSize * 128) >> 4),
                                    idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
                }
            };
            bool ok = true;
            uint32_t gs = 0;            // K/V steps consumed so far
            uint32_t nq = 0;            // items started
            uint32_t nfix = 0;          // items with a zeroed V tail
            uint32_t tstep[2] = {0, 0}; // steps of tile X so far (phase of B_SF / B_PF)
            uint32_t titem[2] = {0, 0}; // items with tile X so far (phase of B_OF / B_OE)
            MmaGeo next = mma_geo(p, snake_item(0, n_ctas)); // the CTA has at least one item
            for (int k = 0, item = snake_item(0, n_ctas); ok && item < n_items; item = snake_item(++k, n_ctas)) {
                const MmaGeo g = next;
                const int nkt[2] = {g.nkt[0], g.nkt[1]};
                const int pmax[2] = {g.pmax[0], g.pmax[1]};
                if (!mbar_wait_warp(bar + B_Q * 8, nq & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                // prologue: S(0) for both tiles
                if (!mbar_wait_warp(bar + (B_KF + (gs & 1)) * 8, (gs >> 1) & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                // QK^T MMAs of this item still to issue: Q is released for the next item's load as soon
                // as the last one is done, while this item's last PV MMAs and softmax still run
                int s_left = nkt[0] + nkt[1];
                auto s_issued = [&]() {
                    if (--s_left == 0)
                        umma_commit(bar + B_QE * 8);
                };
                for (int x = 0; x < 2; ++x)
                    if (nkt[x] > 0) {
                        issue_s(x, gs);
                        s_issued();
                    }
                umma_commit(bar + (B_KE + (gs & 1)) * 8); // K of step 0 consumed
                // the next item's geometry, while this item's first softmax runs
                if (snake_item(k + 1, n_ctas) < n_items)
                    next = mma_geo(p, snake_item(k + 1, n_ctas));
                for (int j = 0; ok && j < g.n_steps; ++j) {
                    const uint32_t gj = gs + j;
                    // V of this step (loaded a step earlier, together with the K that S(j) used) and,
                    // if it has already landed, K of the next step are checked before P: the path from
                    // a softmax's arrive to its PV issue is then a single barrier wait.
                    {
                        const bool fix = g.tail_fix && j == g.n_steps - 1;
                        if (!mbar_wait_warp(bar + (fix ? bar_vfix(nfix) : (B_VF + (gj & 1))) * 8,
                                            fix ? ((nfix >> 1) & 1) : ((gj >> 1) & 1), abort_flag)) {
                            ok = false;
                            break;
                        }
                    }
                    bool k_ready = j + 1 < g.n_steps &&
                                   __all_sync(0xffffffffu, mbar_test(bar + (B_KF + ((gj + 1) & 1)) * 8,
                                                                     ((gj + 1) >> 1) & 1));
                    for (int x = 0; x < 2; ++x) {
                        if (j >= nkt[x])
                            continue;
                        if (!mbar_wait_warp(bar + (B_PF + x) * 8, tstep[x] & 1, abort_flag)) {
                            ok = false;
                            break;
                        }
                        // the first PV of an item overwrites O_X: the previous item's epilogue must be done
                        if (j == 0 && titem[x] > 0 &&
                            !mbar_wait_warp(bar + (B_OE + x) * 8, (titem[x] - 1) & 1, abort_flag)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        issue_pv(x, j, gj, pmax[x]);
                        ++tstep[x];
                        if (j + 1 < nkt[x]) {
                            if (!k_ready) {
                                if (!mbar_wait_warp(bar + (B_KF + ((gj + 1) & 1)) * 8, ((gj + 1) >> 1) & 1, abort_flag)) {
                                    ok = false;
                                    break;
                                }
                                k_ready = true;
                                tc_fence_after();
                            }
                            issue_s(x, gj + 1);
                            s_issued();
                        } else {
                            umma_commit(bar + (B_OF + x) * 8);
                        }
                    }
                    if (!ok)
                        break;
                    umma_commit(bar + (B_VE + (gj & 1)) * 8); // V of this step consumed
                    if (j + 1 < g.n_steps)
                        umma_commit(bar + (B_KE + ((gj + 1) & 1)) * 8); // K of the next step consumed
                }
                if (!ok)
                    break;
                if (g.tail_fix)
                    ++nfix;
                gs += g.n_steps;
                ++nq;
                for (int x = 0; x < 2; ++x)
                    if (nkt[x] > 0)
                        ++titem[x];
            }
            if (!ok && lane == 0)
                fail();
            // drain: nothing of ours may still be running on the tensor core at dealloc
            umma_commit(bar + B_FIN * 8);
            (void)mbar_wait_warp(bar + B_FIN * 8, 0);
        }
    } else if (wg == 2) {
        // ===================================================== epilogue of both tiles
        wg_reg_lower<kRegEpilogue>();
        const int quad = warp & 3;              // TMEM lane quadrant this warp may access
        const int row = threadIdx.x & 127;      // query row of the tile = TMEM lane
        const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
        const float c = p.scale_log2;
        bool ok = true;
        uint32_t titem[2] = {0, 0};
        for (int k = 0, item = snake_item(0, n_ctas); ok && item < n_items; item = snake_item(++k, n_ctas)) {
            const ItemGeo gi = item_geo(p, item);
            for (int x = 0; x < 2; ++x) {
                const TileGeo g = x ? gi.t1 : gi.t0;
                if (g.rows == 0)
                    continue;
                if (!mbar_wait_warp(bar + bar_lf(x, titem[x]) * 8, (titem[x] >> 1) & 1, abort_flag) ||
                    !mbar_wait_warp(bar + (B_OF + x) * 8, titem[x] & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const float *slot = lm_all + x * 512 + (titem[x] & 1) * 256;
                const float l_sum = slot[row], m_ref = slot[128 + row];
                const float inv = l_sum > 0.f ? 1.f / l_sum : 0.f;
                const bool store = row < g.rows;
                const int t = gi.qs + gi.tok0 + x * TQ + row / G;
                const int hq = gi.h * G + row % G;
                __nv_bfloat16 *dst = p.out + ((int64_t)t * p.Hq + hq) * D;
                const uint32_t tO = tmem + lane_addr + col_o(x);
#pragma unroll 1
                for (int cc = 0; cc < D / 32; ++cc) {
                    uint32_t o[32];
                    tmem_ld32p(tO + cc * 32, o);
                    tmem_wait_ld();
                    if (cc == D / 32 - 1) {
                        // O_X may now be overwritten by the next item's first PV
                        tc_fence_before();
                        mbar_arrive(bar + (B_OE + x) * 8);
                    }
                    if (store) {
#pragma unroll
                        for (int i = 0; i < 32; i += 8) {
                            uint4 v;
                            v.x = pack_bf16x2(__uint_as_float(o[i]) * inv, __uint_as_float(o[i + 1]) * inv);
                            v.y = pack_bf16x2(__uint_as_float(o[i + 2]) * inv, __uint_as_float(o[i + 3]) * inv);
                            v.z = pack_bf16x2(__uint_as_float(o[i + 4]) * inv, __uint_as_float(o[i + 5]) * inv);
                            v.w = pack_bf16x2(__uint_as_float(o[i + 6]) * inv, __uint_as_float(o[i + 7]) * inv);
                            *reinterpret_cast<uint4 *>(dst + cc * 32 + i) = v;
                        }
                    }
                }
                ++titem[x];
                if (store && p.lse)
                    p.lse[(int64_t)t * p.Hq + hq] =
                        l_sum > 0.f ? (m_ref * c + log2f(l_sum)) * 0.69314718055994531f : -CUDART_INF_F;
            }
        }
        if (!ok && lane == 0)
            fail();
    } else {
        // ===================================================== softmax (WG 0: tile A, WG 1: tile B)
        wg_reg_raise<kRegSoftmax>();
        const int x = wg;
        const int quad = warp & 3;              // TMEM lane quadrant this warp may access
        const int row = threadIdx.x & 127;      // query row of the tile = TMEM lane
        const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
        const uint32_t tS = tmem + lane_addr + col_s(x);
        const uint32_t tO = tmem + lane_addr + col_o(x);
        float *lm = lm_all + x * 512;
        const float c = p.scale_log2;
        const float thresh = 8.f / c; // 2^8 growth, in raw score units
        bool ok = true;
        uint32_t tstep = 0, titem = 0;
        for (int k = 0, item = snake_item(0, n_ctas); ok && item < n_items; item = snake_item(++k, n_ctas)) {
            const ItemGeo gi = item_geo(p, item);
            const TileGeo g = x ? gi.t1 : gi.t0;
            if (g.rows == 0)
                continue;
            const int p_row = row < g.rows ? g.p_min + row / G : g.p_max;
            float m_ref = -CUDART_INF_F;      // reference max, raw score units
            uint64_t l2 = f2_pack(0.f, 0.f);  // exact fp32 row sum, two packed partial sums
            for (int j = 0; j < g.nkt; ++j, ++tstep) {
                if (!mbar_wait_warp(bar + (B_SF + x) * 8, tstep & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const int key0 = j * kStepKeys;
                const bool diag = key0 + kStepKeys - 1 > g.p_min; // causal mask needed
                uint32_t sv[128];
                tmem_ld32p(tS, sv);
                tmem_ld32p(tS + 32, sv + 32);
                tmem_ld32p(tS + 64, sv + 64);
                tmem_ld32p(tS + 96, sv + 96);
                tmem_wait_ld();
                if (diag) {
#pragma unroll
                    for (int i = 0; i < 128; ++i)
                        if (key0 + i > p_row)
                            sv[i] = __float_as_uint(-CUDART_INF_F);
                }
                float alpha = 1.f;
                uint64_t s2a = f2_pack(0.f, 0.f), s2b = s2a; // this step's row sum (two packed chains)
                float m2[2] = {-CUDART_INF_F, -CUDART_INF_F};
                if (j > 0) {
                    // the exponentials against the reference max so far, with this step's row max taken
                    // alongside; only if that grew past the threshold (rare) is the step redone max-first
                    softmax_exps<true>(sv, c, m_ref, tS, s2a, s2b, m2);
                    const float mx = fmaxf(m2[0], m2[1]);
                    if (__any_sync(0xffffffffu, mx > m_ref + thresh)) {
                        if (mx > m_ref + thresh) {
                            alpha = fast_exp2((m_ref - mx) * c);
                            m_ref = mx;
                        }
                        s2a = s2b = f2_pack(0.f, 0.f);
                        tmem_wait_st(); // the first pass's P stores land before these replace them
                        softmax_exps<false>(sv, c, m_ref, tS, s2a, s2b, m2);
                    }
                } else {
                    // first step of the item: the row max first (eight independent chains, then combined)
                    float m8[8];
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        m8[q] = fmaxf(__uint_as_float(sv[2 * q]), __uint_as_float(sv[2 * q + 1]));
#pragma unroll
                    for (int i = 16; i < 128; i += 16)
#pragma unroll
                        for (int q = 0; q < 8; ++q)
                            m8[q] = fmax3(m8[q], __uint_as_float(sv[i + 2 * q]), __uint_as_float(sv[i + 2 * q + 1]));
                    m_ref = fmaxf(fmax3(m8[0], m8[1], m8[2]), fmax3(fmax3(m8[3], m8[4], m8[5]), m8[6], m8[7]));
                    softmax_exps<false>(sv, c, m_ref, tS, s2a, s2b, m2);
                }
                l2 = f2_add(f2_mul(l2, f2_pack(alpha, alpha)), f2_add(s2a, s2b));
                if (__any_sync(0xffffffffu, alpha != 1.f)) {
                    // O_X is stable (S_X(j) completing implies PV_X(j-1) completed) and PV_X(j)
                    // cannot start before the arrive below: rescale this thread's row
#pragma unroll 1
                    for (int cc = 0; cc < D / 32; ++cc) {
                        uint32_t o[32];
                        tmem_ld32p(tO + cc * 32, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
                        tmem_st32(tO + cc * 32, o);
                    }
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(bar + (B_PF + x) * 8);
            }
            if (!ok)
                break;
            // row sum and reference max -> the epilogue warpgroup (slot by item parity; the
            // epilogue reads it before it frees O_X, which this tile's next-but-one item waits for)
            float la, lb;
            f2_unpack(l2, la, lb);
            float *slot = lm + (titem & 1) * 256;
            slot[row] = la + lb;
            slot[128 + row] = m_ref;
            mbar_arrive(bar + bar_lf(x, titem) * 8);
            ++titem;
        }
        if (!ok && lane == 0)
            fail();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

template <int D>
cudaError_t launch_prefill_t(const AttnParams &p, const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                             int64_t grid_tiles, int num_sms, cudaStream_t s)
{
    constexpr int smem = PfCfg<D>::kSmem;
    // once per device (host threads may call concurrently): the shared-memory attribute, and the
    // registers per thread the kernel is launched with
    constexpr int kMaxDev = 64;
    static std::once_flag once[kMaxDev];
    static cudaError_t attr_err[kMaxDev];
    static int regs_per_thread[kMaxDev];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev)
        return cudaErrorInvalidDevice;
    std::call_once(once[dev], [dev] {
        attr_err[dev] = cudaFuncSetAttribute(prefill_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        cudaFuncAttributes fa;
        if (attr_err[dev] == cudaSuccess)
            attr_err[dev] = cudaFuncGetAttributes(&fa, prefill_kernel<D>);
        regs_per_thread[dev] = attr_err[dev] == cudaSuccess ? fa.numRegs : 0;
    });
    if (attr_err[dev] != cudaSuccess)
        return attr_err[dev];
    // The warpgroups' setmaxnreg budgets draw on the pool the CTA is launched with; a raise
    // beyond it would wait forever, so never launch a build whose pool is smaller.
    if (regs_per_thread[dev] * kThreads < kRegSplit)
        return cudaErrorInvalidConfiguration;
    // persistent: one CTA per SM, never more CTAs than the largest possible number of items
    const int64_t items = grid_tiles * p.Hkv;
    const unsigned grid = (unsigned)(items < num_sms ? items : num_sms);
    // launched at the device's highest priority: when the decode kernel of the same step runs
    // beside it on another stream, the persistent prefill CTAs are placed first and decode
    // fills the SMs they leave
    int lo = 0, hi = 0;
    cudaDeviceGetStreamPriorityRange(&lo, &hi);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributePriority;
    attr[0].val.priority = hi;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, prefill_kernel<D>, tq, tk, tv, p);
}

} // namespace

cudaError_t launch_prefill(const AttnParams &p, const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                           int64_t grid_tiles, int num_sms, cudaStream_t s)
{
    if (grid_tiles <= 0)
        return cudaSuccess;
    if (p.D == 128)
        return launch_prefill_t<128>(p, tq, tk, tv, grid_tiles, num_sms, s);
    return launch_prefill_t<64>(p, tq, tk, tv, grid_tiles, num_sms, s);
}

} // namespace pa
