// plan_merge.cu -- device-side work decomposition of a mixed step, and the
// stand-alone merge of attention states over disjoint key ranges.
//
// Plan: one CTA reads query_start_loc / seq_lens, classifies each request as
// decode (q_len * G small enough for the warp-MMA decode kernel) or prefill
// (tensor-core tiles of 128 query rows), and writes the work lists the next
// kernels index by blockIdx.  Nothing returns to the host, so the whole step
// stays asynchronous and capturable in a CUDA graph.  The V1 scheduler puts
// decodes first and prefill chunks after them (hn.213312.xyz section 一,
// "调度器"), but nothing here depends on that order.
//
// pa_merge_attn_states: the merge of attention states (merge.cuh) as a stand-alone call.
// Inside a step the split-KV merge runs at the end of the decode kernel itself.
#include <math_constants.h>

#include <atomic>
#include <type_traits>

#include "kv_write.cuh"
#include "merge.cuh"
#include "pa_internal.cuh"
#include "ptx.cuh"

namespace pa {
namespace {

__device__ __forceinline__ int warp_incl_scan(int v)
{
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o)
            v += n;
    }
    return v;
}

// Exclusive scan of three counters across a 1024-thread CTA.
__device__ __forceinline__ void cta_excl_scan3(int a, int b, int c, int &ea, int &eb, int &ec, int &ta, int &tb,
                                               int &tc)
{
    __shared__ int sa[32], sb[32], sc[32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int ia = warp_incl_scan(a), ib = warp_incl_scan(b), ic = warp_incl_scan(c);
    if (lane == 31) {
        sa[warp] = ia;
        sb[warp] = ib;
        sc[warp] = ic;
    }
    __syncthreads();
    if (warp == 0) {
        const int nw = blockDim.x >> 5;
        int xa = lane < nw ? sa[lane] : 0, xb = lane < nw ? sb[lane] : 0, xc = lane < nw ? sc[lane] : 0;
        xa = warp_incl_scan(xa);
        xb = warp_incl_scan(xb);
        xc = warp_incl_scan(xc);
        if (lane < nw) {
            sa[lane] = xa;
            sb[lane] = xb;
            sc[lane] = xc;
        }
    }
    __syncthreads();
    const int wa = warp ? sa[warp - 1] : 0, wb = warp ? sb[warp - 1] : 0, wc = warp ? sc[warp - 1] : 0;
    ea = wa + ia - a;
    eb = wb + ib - b;
    ec = wc + ic - c;
    const int nw = blockDim.x >> 5;
    ta = sa[nw - 1];
    tb = sb[nw - 1];
    tc = sc[nw - 1];
    __syncthreads();
}

// SM split of a mixed step.  The prefill kernel (tensor bound) and the decode kernel (HBM
// bound) run at the same time on disjoint SMs: the plan keeps pf_ctas persistent prefill CTAs
// busy and the decode CTAs take every other SM, and all of them once prefill is done.  Rates
// measured on B200 with this library's kernels running side by side (power-capped clocks):
//   prefill  ~6.2 TFLOP/s per SM (925 TFLOP/s over 148 SMs alone);
//   decode   ~80 GB/s per SM (three CTAs, ~190 KB of loads in flight per SM, so latency
//            bound when confined to part of the GPU), at most the HBM rate.
// (A forced sweep of the mixed 8192-token step put its optimum at 88-92 prefill SMs, where these
// two rates balance.)
constexpr float kPfFlopsPerSm = 6.2e12f;
constexpr int kDecCtasPerSm = 12; // decode CTAs per SM below which the plan keeps the shorter split
constexpr int kDecBuckets = 257;  // decode unit lengths in 128-key buckets (longer units share the last)
constexpr float kDecBytesPerSm = 80e9f;
constexpr float kDecBytesMax = 6.35e12f;

// Modelled step time (seconds) with pp prefill SMs out of num_sms: prefill lasts F / (pp f);
// decode runs at min(B, (S - pp) b) meanwhile and at B after that.
__device__ __forceinline__ float split_time(float pf_flops, float dec_bytes, int num_sms, int pp)
{
    const float t_pf = pf_flops / ((float)pp * kPfFlopsPerSm);
    const float r_dec = fminf(kDecBytesMax, (float)(num_sms - pp) * kDecBytesPerSm);
    const float done = r_dec * t_pf;
    return done >= dec_bytes ? t_pf : t_pf + (dec_bytes - done) / kDecBytesMax;
}

// Prefill CTAs that minimise the modelled step time: every thread of the CTA evaluates one
// candidate, then a block-wide argmin (ties go to the larger count).  Called by all threads.
__device__ int choose_pf_ctas(float pf_flops, float dec_bytes, int num_sms, int pf_items)
{
    __shared__ unsigned long long s_best[32];
    const int cap = max(1, min(num_sms, pf_items));
    if (pf_flops <= 0.f || dec_bytes <= 0.f)
        return cap;
    // key = (time bits, cap - pp): time is non-negative, so its float bits order like the value
    unsigned long long key = ~0ull;
    for (int pp = (int)threadIdx.x + 1; pp <= cap; pp += blockDim.x) {
        const float t = split_time(pf_flops, dec_bytes, num_sms, pp);
        const unsigned long long k = (unsigned long long)__float_as_uint(t) << 32 | (unsigned)(cap - pp);
        key = k < key ? k : key;
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) {
        const unsigned long long other = __shfl_xor_sync(0xffffffffu, key, o);
        key = other < key ? other : key;
    }
    if ((threadIdx.x & 31) == 0)
        s_best[threadIdx.x >> 5] = key;
    __syncthreads();
    unsigned long long best = ~0ull;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w)
        best = s_best[w] < best ? s_best[w] : best;
    return cap - (int)(best & 0xffffffffu);
}

// 128-key steps a prefill q-pair of request r needs: keys 0 .. position of its last token
__device__ __forceinline__ int pair_cost(int ctx, int q_len, int qp, int tq)
{
    const int last = min(q_len, (2 * qp + 2) * tq) - 1;
    return (ctx + last) / 128 + 1;
}

// Work lists of one step.  Decode units longest first (see pass 1b); prefill q-pairs sorted by
// cost (key steps), most expensive first -- a counting sort through a shared-memory
// histogram, so the persistent prefill CTAs, which walk the list in snake order, end
// at nearly the same time.  Pairs of equal cost land in any order; every pair is
// computed independently, so the order never changes a result.
// hist: [n_buckets] ints of dynamic shared memory (pair counts, then start offsets).  Called by every
// thread of one CTA.  reset_status: clear the status word first (the caller did otherwise).
__device__ __forceinline__ void plan_body(const AttnParams &p, int n_buckets, int *hist, bool reset_status)
{
    __shared__ unsigned long long s_sum[2][32];
    WsHeader *hdr = p.hdr;
    if (reset_status && threadIdx.x == 0)
        hdr->status = 0u;
    // work estimates, per thread then reduced once: keys read by its decode requests and
    // causal (query, key) pairs of its prefill requests
    unsigned long long my_dec_tokens = 0ull, my_pf_pairs = 0ull;
    for (int i = threadIdx.x; i < n_buckets; i += blockDim.x)
        hist[i] = 0;
    __syncthreads();
    const int tq = kPrefillRows / p.G;
    // n_dec: splits of a decode request at the host's split size (0 for every other request)
    auto classify = [&](int r, int &n_dec, int &n_pf, int &red, int &ctx, int &q_len) {
        n_dec = n_pf = red = 0;
        ctx = q_len = 0;
        if (r >= p.num_seqs)
            return;
        const int qs = p.qsl[r], qe = p.qsl[r + 1];
        q_len = qe - qs;
        const int L = p.seq_lens[r];
        const bool bad = qs < 0 || qe > p.num_tokens || q_len < 0 || q_len > p.max_query_len || L < q_len ||
                         L > p.max_seq_len;
        if (bad) {
            atomicOr(&hdr->status, PA_DEVICE_BAD_SEQ);
            q_len = 0;
            return;
        }
        ctx = L - q_len;
        if (q_len == 0)
            return;
        if (q_len * p.G <= p.dec_rows_cap) {
            n_dec = (L + p.split_tokens - 1) / p.split_tokens;
            red = n_dec > 1 ? 1 : 0;
        } else {
            n_pf = (q_len * p.G + kPrefillRowsPerCta - 1) / kPrefillRowsPerCta;
        }
    };
    // pass 1: classification, histogram of prefill pair costs, and the decode units the step would
    // have at two and four times the host's split size
    int carry_pf = 0, carry_u2 = 0, carry_u4 = 0;
    int kept_pf = 0, kept_ctx = 0, kept_q = 0, kept_L = 0; // this thread's request when one pass covers them all
    const int s2 = 2 * p.split_tokens, s4 = 4 * p.split_tokens;
    for (int base = 0; base < p.num_seqs; base += blockDim.x) {
        const int r = base + threadIdx.x;
        int n_dec, n_pf, red, ctx, q_len;
        classify(r, n_dec, n_pf, red, ctx, q_len);
        const int L = n_dec ? ctx + q_len : 0; // keys of a decode request
        kept_pf = n_pf;
        kept_ctx = ctx;
        kept_q = q_len;
        kept_L = L;
        for (int k = 0; k < n_pf; ++k)
            atomicAdd(&hist[min(pair_cost(ctx, q_len, k, tq), n_buckets - 1)], 1);
        if (n_dec)
            my_dec_tokens += (unsigned long long)L;
        if (n_pf)
            my_pf_pairs += (unsigned long long)q_len * ctx + (unsigned long long)q_len * (q_len + 1) / 2;
        int e0, e1, e2, tp, t2, t4;
        cta_excl_scan3(n_pf, (L + s2 - 1) / s2, (L + s4 - 1) / s4, e0, e1, e2, tp, t2, t4);
        carry_pf += tp;
        carry_u2 += t2;
        carry_u4 += t4;
    }
    // Split size of this step.  A decode CTA has a fixed cost (barrier setup, the first loads in
    // flight, the partial-state write and merge), so fewer, longer splits read HBM faster as long as
    // there are still about a dozen CTAs per SM to balance.  A step with prefill work keeps the short
    // split: its decode CTAs start on the SMs the prefill leaves free and spread over the others as
    // the prefill CTAs finish, which short units fill more evenly.  The caller's explicit split is kept.
    int split = p.split_tokens;
    if (p.auto_split && carry_pf == 0) {
        const int64_t want = (int64_t)kDecCtasPerSm * p.num_sms;
        if ((int64_t)carry_u4 * p.Hkv >= want)
            split = s4;
        else if ((int64_t)carry_u2 * p.Hkv >= want)
            split = s2;
    }
    // pass 1b: decode units at that split size, longest first: a counting sort over their key counts in
    // 128-key buckets, so that the CTAs of the longest units start first and the grid ends on short ones
    // (the decode grid is ragged: request lengths differ by up to 8x in one batch).  Split-arrival
    // counters zeroed.
    __shared__ int dec_hist[kDecBuckets];
    for (int i = threadIdx.x; i < kDecBuckets; i += blockDim.x)
        dec_hist[i] = 0;
    __syncthreads();
    auto dec_keys = [&](int r) { // keys of request r if it takes the decode kernel, else 0
        if (p.num_seqs <= (int)blockDim.x)
            return kept_L;
        int n_dec, n_pf, red, ctx, q_len;
        classify(r, n_dec, n_pf, red, ctx, q_len);
        return n_dec ? ctx + q_len : 0;
    };
    auto dec_bucket = [&](int L, int u) {
        const int len = min(split, L - u * split);
        return min((len + 127) >> 7, kDecBuckets - 1);
    };
    int carry_dec = 0, carry_red = 0;
    for (int base = 0; base < p.num_seqs; base += blockDim.x) {
        const int r = base + threadIdx.x;
        const int L = dec_keys(r);
        const int n_dec = (L + split - 1) / split;
        const int red = n_dec > 1 ? 1 : 0;
        int ed, er, e2, td, tr, t2;
        cta_excl_scan3(n_dec, red, 0, ed, er, e2, td, tr, t2);
        for (int u = 0; u < n_dec; ++u)
            atomicAdd(&dec_hist[dec_bucket(L, u)], 1);
        if (red)
            for (int h = 0; h < p.Hkv; ++h)
                p.split_arrivals[(int64_t)r * p.Hkv + h] = 0u; // counted by the decode kernel
        carry_dec += td;
        carry_red += tr;
    }
    __syncthreads();
    {
        int carry = 0; // bucket start offsets, longest bucket first
        for (int base = 0; base < kDecBuckets; base += blockDim.x) {
            const int b = kDecBuckets - 1 - (base + (int)threadIdx.x);
            const int cnt = b >= 0 ? dec_hist[b] : 0;
            int e0, e1, e2, t0, t1, t2;
            cta_excl_scan3(cnt, 0, 0, e0, e1, e2, t0, t1, t2);
            if (b >= 0)
                dec_hist[b] = carry + e0;
            carry += t0;
            __syncthreads();
        }
    }
    for (int base = 0; base < p.num_seqs; base += blockDim.x) {
        const int r = base + threadIdx.x;
        const int L = dec_keys(r);
        const int n_dec = (L + split - 1) / split;
        for (int u = 0; u < n_dec; ++u) {
            const int pos = atomicAdd(&dec_hist[dec_bucket(L, u)], 1);
            if (pos < p.max_dec_units)
                p.dec_units[pos] = make_int2(r, u);
        }
    }
    __syncthreads();
    if (carry_pf > 0) { // a step without prefill work skips the sort
        // bucket start offsets, most expensive bucket first
        int carry = 0;
        for (int base = 0; base < n_buckets; base += blockDim.x) {
            const int b = n_buckets - 1 - (base + (int)threadIdx.x); // descending cost
            const int cnt = b >= 0 ? hist[b] : 0;
            int e0, e1, e2, t0, t1, t2;
            cta_excl_scan3(cnt, 0, 0, e0, e1, e2, t0, t1, t2);
            if (b >= 0)
                hist[b] = carry + e0;
            carry += t0;
            __syncthreads();
        }
        // pass 2: scatter the prefill pairs into their cost buckets (requests re-read only when
        // there are more of them than threads)
        for (int base = 0; base < p.num_seqs; base += blockDim.x) {
            const int r = base + threadIdx.x;
            int n_dec, n_pf = kept_pf, red, ctx = kept_ctx, q_len = kept_q;
            if (p.num_seqs > (int)blockDim.x)
                classify(r, n_dec, n_pf, red, ctx, q_len);
            for (int k = 0; k < n_pf; ++k) {
                const int pos = atomicAdd(&hist[min(pair_cost(ctx, q_len, k, tq), n_buckets - 1)], 1);
                if (pos < p.max_pf_tiles) // only overlapping query rows can exceed the list (flagged below)
                    p.pf_tiles[pos] = make_int2(r, k);
            }
        }
    }
    // block sums of the two estimates (warp shuffles, then one warp over the warp partials)
#pragma unroll
    for (int o = 16; o; o >>= 1) {
        my_dec_tokens += __shfl_xor_sync(0xffffffffu, my_dec_tokens, o);
        my_pf_pairs += __shfl_xor_sync(0xffffffffu, my_pf_pairs, o);
    }
    if ((threadIdx.x & 31) == 0) {
        s_sum[0][threadIdx.x >> 5] = my_dec_tokens;
        s_sum[1][threadIdx.x >> 5] = my_pf_pairs;
    }
    __syncthreads();
    unsigned long long dec_tokens = 0ull, pf_pairs = 0ull;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) {
        dec_tokens += s_sum[0][w];
        pf_pairs += s_sum[1][w];
    }
    const float dec_bytes = (float)dec_tokens * (float)(p.Hkv * p.D * 4); // K + V, bf16
    const float pf_flops = (float)pf_pairs * (float)(4 * p.Hq * p.D);
    const int pf_ctas = p.pf_all_sms ? max(1, min(p.num_sms, carry_pf * p.Hkv))
                                     : choose_pf_ctas(pf_flops, dec_bytes, p.num_sms, carry_pf * p.Hkv);
    if (threadIdx.x == 0) {
        // Requests whose query rows overlap (a query_start_loc that decreases somewhere) can ask for more
        // work items than the host-sized lists hold: keep what fits, flag the step.
        if (carry_dec > p.max_dec_units || carry_pf > p.max_pf_tiles)
            atomicOr(&hdr->status, PA_DEVICE_BAD_SEQ);
        hdr->n_dec_units = (uint32_t)min((int64_t)carry_dec, p.max_dec_units);
        hdr->n_pf_tiles = (uint32_t)min((int64_t)carry_pf, p.max_pf_tiles);
        hdr->n_reduce = (uint32_t)carry_red;
        hdr->split_tokens = (uint32_t)split;
        hdr->pf_ctas = (uint32_t)pf_ctas;
    }
}

__global__ void __launch_bounds__(1024) plan_kernel(const AttnParams p, int n_buckets)
{
    extern __shared__ int hist[];
    plan_body(p, n_buckets, hist, true);
}

// One launch for the start of a step: CTA 0 plans the step's attention while the other CTAs write its new
// K/V rows into the cache (neither reads what the other writes).  A slot outside the pool sets
// PA_DEVICE_BAD_SLOT in the status word, which CTA 0 clears for this call first: a writer that meets one
// waits (bounded) until CTA 0 has published this call's epoch after the clear.  The step's attention
// kernels set the epoch word back to kWriteEpochIdle, so the same launch replayed from a CUDA graph (same
// epoch argument) waits for its own CTA 0 as well.
template <int VEC>
__global__ void __launch_bounds__(256) write_plan_kernel(const AttnParams p, int n_buckets, const KvWriteArgs w,
                                                         uint32_t epoch)
{
    extern __shared__ int hist[];
    WsHeader *hdr = p.hdr;
    if (blockIdx.x == 0) {
        if (threadIdx.x == 0) {
            hdr->status = 0u;
            __threadfence();
            atomicExch(&hdr->write_epoch, epoch);
        }
        plan_body(p, n_buckets, hist, false);
        return;
    }
    kv_write_tokens<VEC>(w, blockIdx.x - 1, gridDim.x - 1, [&]() {
        const uint64_t t0 = global_timer_ns();
        for (int it = 0; it < (1 << 20); ++it)
            if (atomicAdd(&hdr->write_epoch, 0u) == epoch || global_timer_ns() - t0 > kWaitLimitNs)
                break;
        atomicOr(&hdr->status, PA_DEVICE_BAD_SLOT);
    });
}

template <int D>
__global__ void __launch_bounds__(256) merge_states_kernel(const float *__restrict__ part_out,
                                                           const float *__restrict__ part_lse,
                                                           const int32_t *__restrict__ parts_per_row, int num_rows,
                                                           int num_heads, int num_parts, __nv_bfloat16 *out,
                                                           float *lse_out)
{
    const int64_t pair = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (pair >= (int64_t)num_rows * num_heads)
        return;
    const int row = (int)(pair / num_heads);
    int n = num_parts;
    if (parts_per_row)
        n = max(0, min(num_parts, parts_per_row[row]));
    merge_one<D>(part_out + pair * num_parts * D, D, part_lse + pair * num_parts, 1, n, out + pair * D,
                 lse_out ? lse_out + pair : nullptr);
}

} // namespace

cudaError_t launch_plan(const AttnParams &p, cudaStream_t s)
{
    // one bucket per possible cost (key steps), capped at 12k buckets (48 KB of shared memory);
    // costs beyond the last bucket share it
    int n_buckets = p.max_seq_len / 128 + 2;
    if (n_buckets > 12 * 1024)
        n_buckets = 12 * 1024;
    const int smem = n_buckets * (int)sizeof(int);
    // one thread per request (at least four warps, at most 1024 threads, which then loop): fewer warps make
    // the block-wide scans and reductions of this short, latency-bound kernel cheaper
    const int threads = min(1024, max(128, (p.num_seqs + 31) / 32 * 32));
    plan_kernel<<<1, threads, smem, s>>>(p, n_buckets);
    return cudaGetLastError();
}

cudaError_t launch_write_plan(const AttnParams &p, const KvWriteArgs &w, bool vec_ok, cudaStream_t s)
{
    int n_buckets = p.max_seq_len / 128 + 2;
    if (n_buckets > 12 * 1024)
        n_buckets = 12 * 1024;
    const int smem = n_buckets * (int)sizeof(int);
    static std::atomic<uint32_t> epoch_counter{0};
    uint32_t epoch = ++epoch_counter;
    if (epoch == kWriteEpochIdle)
        epoch = ++epoch_counter;
    const unsigned grid = 1u + (unsigned)kv_write_ctas(w.num_tokens);
    if (vec_ok)
        write_plan_kernel<8><<<grid, 256, smem, s>>>(p, n_buckets, w, epoch);
    else
        write_plan_kernel<1><<<grid, 256, smem, s>>>(p, n_buckets, w, epoch);
    return cudaGetLastError();
}

cudaError_t launch_merge_states(const float *part_out, const float *part_lse, const int32_t *parts_per_row,
                                int num_rows, int num_heads, int num_parts, int D, void *out, float *lse_out,
                                cudaStream_t s)
{
    const int64_t pairs = (int64_t)num_rows * num_heads;
    const unsigned blocks = (unsigned)((pairs + 7) / 8);
    auto *o = static_cast<__nv_bfloat16 *>(out);
    if (D == 128)
        merge_states_kernel<128><<<blocks, 256, 0, s>>>(part_out, part_lse, parts_per_row, num_rows, num_heads,
                                                         num_parts, o, lse_out);
    else
        merge_states_kernel<64><<<blocks, 256, 0, s>>>(part_out, part_lse, parts_per_row, num_rows, num_heads,
                                                        num_parts, o, lse_out);
    return cudaGetLastError();
}

} // namespace pa
