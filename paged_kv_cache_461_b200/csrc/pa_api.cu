// pa_api.cu -- the C ABI of libpa_b200.so (declared in include/pa.h): host-side
// validation, the workspace layout, TMA descriptor encoding and the launch
// sequence of one mixed step.  No function here allocates, frees or
// synchronises; everything is enqueued on the caller's stream.
#include <cudaTypedefs.h>
#include <nvtx3/nvToolsExt.h>

#include <cmath>
#include <cstring>
#include <mutex>

#include "kv_write.cuh"
#include "pa_internal.cuh"

using namespace pa;

namespace {

constexpr size_t kAlign = 256;
size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool cache_desc_ok(const pa_cache_desc_t *c, pa_status_t *why)
{
    if (!c || c->num_blocks <= 0 || c->num_kv_heads <= 0 || c->head_dim <= 0 || c->block_size <= 0) {
        *why = PA_ERR_INVALID_ARG;
        return false;
    }
    if (c->layout != PA_LAYOUT_HND && c->layout != PA_LAYOUT_NHD) {
        *why = PA_ERR_INVALID_ARG;
        return false;
    }
    if (c->block_size != kBlockSize || (c->head_dim != 64 && c->head_dim != 128)) {
        *why = PA_ERR_UNSUPPORTED;
        return false;
    }
    // TMA row coordinates of the caches are int32
    if ((double)c->num_blocks * c->num_kv_heads * kBlockSize >= 2147483647.0) {
        *why = PA_ERR_UNSUPPORTED;
        return false;
    }
    return true;
}

// Decomposition of a call from its host-side bounds only.
bool make_plan(int32_t num_seqs, int32_t num_tokens, int32_t num_q_heads, const pa_cache_desc_t *c,
               int32_t max_seq_len, const pa_attn_options_t *o, Plan &P, pa_status_t *why)
{
    *why = PA_OK;
    if (!cache_desc_ok(c, why))
        return false;
    if (num_seqs < 0 || num_tokens < 0 || max_seq_len < 0 || num_q_heads <= 0 ||
        num_q_heads % c->num_kv_heads != 0) {
        *why = PA_ERR_INVALID_ARG;
        return false;
    }
    if (o) {
        for (int i = 0; i < 6; ++i)
            if (o->reserved[i] != 0) {
                *why = PA_ERR_INVALID_ARG;
                return false;
            }
        if (o->kv_split_tokens < 0 || o->kv_split_tokens % kBlockSize != 0) {
            *why = PA_ERR_INVALID_ARG;
            return false;
        }
    }
    P.G = num_q_heads / c->num_kv_heads;
    if (P.G > kPrefillRows || kPrefillRows % P.G != 0) {
        *why = PA_ERR_UNSUPPORTED;
        return false;
    }
    // decode path: up to 8*NT packed (token, head) rows per kv head in one warp MMA
    const int dq = o ? o->decode_max_query_len : 0;
    if (dq < -1 || (dq > 0 && dq * P.G > 16)) {
        *why = dq < -1 ? PA_ERR_INVALID_ARG : PA_ERR_UNSUPPORTED;
        return false;
    }
    if (dq == -1) { // no decode kernel: every request takes the prefill kernel
        P.NT = 0;
        P.QD = 0;
        P.dec_rows_cap = 0;
    } else if (dq > 0) {
        P.NT = dq * P.G <= 8 ? 1 : 2;
        P.QD = dq;
        P.dec_rows_cap = dq * P.G;
    } else {
        P.NT = P.G <= 8 ? 1 : (P.G <= 16 ? 2 : 0);
        P.dec_rows_cap = 8 * P.NT;
        P.QD = P.NT ? P.dec_rows_cap / P.G : 0;
    }
    P.split_tokens = (o && o->kv_split_tokens) ? o->kv_split_tokens : kDefaultSplitTokens;
    const int64_t msl = max_seq_len > 0 ? max_seq_len : 1;
    P.max_splits = P.NT ? (int)((msl + P.split_tokens - 1) / P.split_tokens) : 0;
    P.max_dec_units = P.NT ? (int64_t)num_seqs * P.max_splits : 0;
    P.max_pf_tiles = (int64_t)num_tokens * P.G / kPrefillRows + num_seqs + 1;
    P.need_reduce = P.NT && P.max_splits > 1; // split partial states exist (the decode kernel merges them)
    const int64_t part_rows = P.need_reduce ? (int64_t)num_seqs * P.QD * num_q_heads * P.max_splits : 0;
    size_t off = align_up(sizeof(WsHeader));
    P.off_dec = off;
    off = align_up(off + sizeof(int2) * (size_t)P.max_dec_units);
    P.off_pf = off;
    off = align_up(off + sizeof(int2) * (size_t)P.max_pf_tiles);
    P.off_red = off;
    off = align_up(off + sizeof(uint32_t) * (size_t)num_seqs * (size_t)c->num_kv_heads);
    P.off_part_o = off;
    off = align_up(off + sizeof(float) * (size_t)c->head_dim * (size_t)part_rows);
    P.off_part_lse = off;
    off = align_up(off + sizeof(float) * (size_t)part_rows);
    P.total = off;
    return true;
}

// ------------------------------------------------------------- TMA descriptors
PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

struct MapKey {
    const void *ptr;
    uint64_t d0, d1, d2;
    uint32_t b1, b2, rank;
    bool operator==(const MapKey &o) const
    {
        return ptr == o.ptr && d0 == o.d0 && d1 == o.d1 && d2 == o.d2 && b1 == o.b1 && b2 == o.b2 && rank == o.rank;
    }
};

struct MapCache {
    static constexpr int kN = 16;
    MapKey key[kN];
    CUtensorMap map[kN];
    int used = 0, next = 0;
    std::mutex mu;
};

MapCache &map_cache()
{
    static MapCache c;
    return c;
}

// bf16 tensor map with 128-byte swizzle and a 64-element inner box.
// rank 2: dims {D, rows}, box {64, b1};  rank 3: dims {D, d1, d2}, box {64, b1, b2}.
bool get_map(const void *ptr, int rank, uint64_t D, uint64_t d1, uint64_t d2, uint32_t b1, uint32_t b2,
             CUtensorMap *out)
{
    MapCache &c = map_cache();
    MapKey k{ptr, D, d1, d2, b1, b2, (uint32_t)rank};
    std::lock_guard<std::mutex> g(c.mu);
    for (int i = 0; i < c.used; ++i)
        if (c.key[i] == k) {
            *out = c.map[i];
            return true;
        }
    auto fn = encode_fn();
    if (!fn)
        return false;
    CUtensorMap m;
    cuuint64_t dims[3] = {D, d1, d2};
    cuuint64_t strides[2] = {D * 2, D * 2 * d1};
    cuuint32_t box[3] = {64, b1, b2};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(&m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, const_cast<void *>(ptr), dims, strides, box,
                    estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
        return false;
    const int slot = c.used < MapCache::kN ? c.used++ : (c.next++ % MapCache::kN);
    c.key[slot] = k;
    c.map[slot] = m;
    *out = m;
    return true;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool ranges_overlap(const void *a, size_t na, const void *b, size_t nb)
{
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return na && nb && x < y + nb && y < x + na;
}

// SMs of the current device (looked up once per device)
int device_sms()
{
    constexpr int kMaxDev = 64;
    static std::once_flag once[kMaxDev];
    static int sms[kMaxDev];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev)
        return 148;
    std::call_once(once[dev], [dev] {
        int n = 0;
        sms[dev] = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && n > 0 ? n : 148;
    });
    return sms[dev];
}

pa_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? PA_OK : PA_ERR_CUDA; }

// An NVTX range around the launches of one entry point, so that a timeline (e.g. of a mixed step's
// concurrent kernels) shows which call they belong to.  Costs a branch when no tool is attached.
struct NvtxRange {
    explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
};

} // namespace

extern "C" {

int32_t pa_abi_version(void) { return 4; }

const char *pa_status_string(pa_status_t s)
{
    switch (s) {
    case PA_OK:
        return "PA_OK";
    case PA_ERR_INVALID_ARG:
        return "PA_ERR_INVALID_ARG";
    case PA_ERR_UNSUPPORTED:
        return "PA_ERR_UNSUPPORTED";
    case PA_ERR_WORKSPACE_TOO_SMALL:
        return "PA_ERR_WORKSPACE_TOO_SMALL";
    case PA_ERR_CUDA:
        return "PA_ERR_CUDA";
    }
    return "PA_ERR_UNKNOWN";
}

pa_status_t pa_kv_write_ex(const void *k_new, const void *v_new, int64_t new_row_stride, const int64_t *slot_mapping,
                           int32_t num_tokens, void *k_cache, void *v_cache, const pa_cache_desc_t *cache,
                           uint32_t *status, pa_stream_t stream)
{
    pa_status_t why;
    if (!cache_desc_ok(cache, &why))
        return why;
    if (num_tokens < 0 || new_row_stride < (int64_t)cache->num_kv_heads * cache->head_dim)
        return PA_ERR_INVALID_ARG;
    if (num_tokens == 0)
        return PA_OK;
    if (!k_new || !v_new || !slot_mapping || !k_cache || !v_cache)
        return PA_ERR_INVALID_ARG;
    if (status != nullptr && (reinterpret_cast<uintptr_t>(status) & 3u))
        return PA_ERR_INVALID_ARG;
    NvtxRange r("pa_kv_write");
    return cuda_status(launch_kv_write(k_new, v_new, new_row_stride, slot_mapping, num_tokens, k_cache, v_cache,
                                       cache->num_blocks, cache->num_kv_heads, cache->head_dim,
                                       cache->layout == PA_LAYOUT_NHD, status, reinterpret_cast<cudaStream_t>(stream)));
}

pa_status_t pa_kv_write(const void *k_new, const void *v_new, int64_t new_row_stride, const int64_t *slot_mapping,
                        int32_t num_tokens, void *k_cache, void *v_cache, const pa_cache_desc_t *cache,
                        pa_stream_t stream)
{
    return pa_kv_write_ex(k_new, v_new, new_row_stride, slot_mapping, num_tokens, k_cache, v_cache, cache, nullptr,
                          stream);
}

pa_status_t pa_build_slot_mapping(const int32_t *query_start_loc, const int32_t *seq_lens, const int32_t *block_table,
                                  int32_t bt_stride, int32_t num_seqs, int32_t num_tokens, int64_t *slot_mapping,
                                  pa_stream_t stream)
{
    if (num_seqs < 0 || num_tokens < 0 || bt_stride < 0)
        return PA_ERR_INVALID_ARG;
    if (num_seqs == 0 || num_tokens == 0)
        return PA_OK;
    if (!query_start_loc || !seq_lens || !block_table || !slot_mapping || bt_stride == 0)
        return PA_ERR_INVALID_ARG;
    NvtxRange r("pa_build_slot_mapping");
    return cuda_status(launch_slot_mapping(query_start_loc, seq_lens, block_table, bt_stride, num_seqs, num_tokens,
                                           slot_mapping, reinterpret_cast<cudaStream_t>(stream)));
}

size_t pa_workspace_size_ex(int32_t num_seqs, int32_t num_tokens, int32_t num_q_heads, const pa_cache_desc_t *cache,
                            int32_t max_seq_len, const pa_attn_options_t *options)
{
    Plan P;
    pa_status_t why;
    if (!make_plan(num_seqs, num_tokens, num_q_heads, cache, max_seq_len, options, P, &why))
        return 0;
    return P.total;
}

size_t pa_workspace_size(int32_t num_seqs, int32_t num_tokens, int32_t num_q_heads, const pa_cache_desc_t *cache,
                         int32_t max_seq_len)
{
    return pa_workspace_size_ex(num_seqs, num_tokens, num_q_heads, cache, max_seq_len, nullptr);
}

} // extern "C"

namespace {

// New K/V rows the decode kernel stores itself (pa_attention_decode_fused).
// The step's new K/V rows, written by the attention call itself: with slots == nullptr by the decode
// kernel (decode-shaped steps, slots from the block tables), else by the launch that also plans the step
// (any step, through the given slot mapping).
struct FusedWrite {
    const void *k_new, *v_new;
    int64_t row_stride;
    const int64_t *slots;
};

pa_status_t attention_impl(const void *q, int32_t num_q_heads, const void *k_cache, const void *v_cache,
                           const pa_cache_desc_t *cache, const int32_t *query_start_loc, const int32_t *seq_lens,
                           const int32_t *block_table, int32_t bt_stride, int32_t num_seqs, int32_t num_tokens,
                           int32_t max_query_len, int32_t max_seq_len, float softmax_scale, void *out, float *lse,
                           void *workspace, size_t workspace_bytes, const pa_attn_options_t *options,
                           const FusedWrite *fw, pa_stream_t stream)
{
    Plan P;
    pa_status_t why;
    if (!make_plan(num_seqs, num_tokens, num_q_heads, cache, max_seq_len, options, P, &why))
        return why;
    if (max_query_len < 0 || bt_stride < 0 || !std::isfinite(softmax_scale))
        return PA_ERR_INVALID_ARG;
    // the caller's side stream and fork/join events for running prefill beside decode: all or none
    cudaStream_t side = options ? reinterpret_cast<cudaStream_t>(options->side_stream) : nullptr;
    cudaEvent_t ev_fork = options ? reinterpret_cast<cudaEvent_t>(options->fork_event) : nullptr;
    cudaEvent_t ev_join = options ? reinterpret_cast<cudaEvent_t>(options->join_event) : nullptr;
    if ((side != nullptr) != (ev_fork != nullptr) || (side != nullptr) != (ev_join != nullptr) ||
        (side != nullptr && (side == reinterpret_cast<cudaStream_t>(stream) || ev_fork == ev_join)))
        return PA_ERR_INVALID_ARG;
    if ((int64_t)bt_stride * kBlockSize < (int64_t)max_seq_len)
        return PA_ERR_INVALID_ARG;
    if (num_seqs == 0 || num_tokens == 0)
        return PA_OK;
    if (!q || !k_cache || !v_cache || !query_start_loc || !seq_lens || !block_table || !out || !workspace)
        return PA_ERR_INVALID_ARG;
    const int D = cache->head_dim;
    const size_t q_bytes = (size_t)num_tokens * num_q_heads * D * 2;
    if (ranges_overlap(q, q_bytes, out, q_bytes))
        return PA_ERR_INVALID_ARG;
    const size_t lse_bytes = lse ? (size_t)num_tokens * num_q_heads * 4 : 0;
    if (ranges_overlap(lse, lse_bytes, out, q_bytes) || ranges_overlap(lse, lse_bytes, q, q_bytes))
        return PA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out) || !aligned16(workspace))
        return PA_ERR_UNSUPPORTED;
    if (workspace_bytes < P.total)
        return PA_ERR_WORKSPACE_TOO_SMALL;
    // the part of the workspace this call writes must not overlap its inputs or outputs
    if (ranges_overlap(workspace, P.total, q, q_bytes) || ranges_overlap(workspace, P.total, out, q_bytes) ||
        ranges_overlap(workspace, P.total, lse, lse_bytes))
        return PA_ERR_INVALID_ARG;

    const int Hkv = cache->num_kv_heads;
    const bool nhd = cache->layout == PA_LAYOUT_NHD;
    if (fw && !fw->slots) {
        // every request must be decode-shaped: the prefill kernel reads the new rows from the cache
        if ((int64_t)max_query_len * P.G > P.dec_rows_cap || P.NT == 0)
            return PA_ERR_UNSUPPORTED;
        if (!fw->k_new || !fw->v_new || fw->row_stride < (int64_t)Hkv * D)
            return PA_ERR_INVALID_ARG;
        if (!aligned16(fw->k_new) || !aligned16(fw->v_new) || fw->row_stride % 8 != 0)
            return PA_ERR_UNSUPPORTED;
    }
    if (fw && fw->slots && (!fw->k_new || !fw->v_new || fw->row_stride < (int64_t)Hkv * D))
        return PA_ERR_INVALID_ARG;
    // HND: 2-D {D, blocks*Hkv*16} with 16-row boxes;  NHD: 3-D {D, Hkv, blocks*16} with {64, 1, 16} boxes
    const uint64_t kv_rows = (uint64_t)cache->num_blocks * Hkv * kBlockSize;
    const uint64_t tok_rows = (uint64_t)cache->num_blocks * kBlockSize;
    CUtensorMap tk, tv;
    const bool maps_ok =
        nhd ? get_map(k_cache, 3, D, (uint64_t)Hkv, tok_rows, 1, kBlockSize, &tk) &&
                  get_map(v_cache, 3, D, (uint64_t)Hkv, tok_rows, 1, kBlockSize, &tv)
            : get_map(k_cache, 2, D, kv_rows, 1, kBlockSize, 1, &tk) && get_map(v_cache, 2, D, kv_rows, 1, kBlockSize, 1, &tv);
    if (!maps_ok)
        return PA_ERR_CUDA;

    uint8_t *ws = static_cast<uint8_t *>(workspace);
    AttnParams p;
    std::memset(&p, 0, sizeof p);
    p.q = static_cast<const __nv_bfloat16 *>(q);
    p.out = static_cast<__nv_bfloat16 *>(out);
    p.lse = lse;
    p.qsl = query_start_loc;
    p.seq_lens = seq_lens;
    p.bt = block_table;
    p.num_blocks = cache->num_blocks;
    p.bt_stride = bt_stride;
    p.num_seqs = num_seqs;
    p.num_tokens = num_tokens;
    p.max_seq_len = max_seq_len;
    p.max_query_len = max_query_len;
    p.max_dec_units = P.max_dec_units;
    p.max_pf_tiles = P.max_pf_tiles;
    p.Hq = num_q_heads;
    p.Hkv = Hkv;
    p.G = P.G;
    p.D = D;
    p.scale_log2 = softmax_scale * 1.4426950408889634f;
    p.hdr = reinterpret_cast<WsHeader *>(ws);
    p.dec_units = reinterpret_cast<int2 *>(ws + P.off_dec);
    p.pf_tiles = reinterpret_cast<int2 *>(ws + P.off_pf);
    p.split_arrivals = reinterpret_cast<uint32_t *>(ws + P.off_red);
    p.part_o = reinterpret_cast<float *>(ws + P.off_part_o);
    p.part_lse = reinterpret_cast<float *>(ws + P.off_part_lse);
    p.split_tokens = P.split_tokens;
    p.auto_split = (options && options->kv_split_tokens) ? 0 : 1;
    p.max_splits = P.max_splits;
    p.QD = P.QD;
    p.dec_rows_cap = P.dec_rows_cap;
    p.nhd = nhd;
    if (fw && !fw->slots) {
        p.k_new = static_cast<const uint16_t *>(fw->k_new);
        p.v_new = static_cast<const uint16_t *>(fw->v_new);
        p.new_row_stride = fw->row_stride;
        p.k_cache_w = static_cast<uint16_t *>(const_cast<void *>(k_cache));
        p.v_cache_w = static_cast<uint16_t *>(const_cast<void *>(v_cache));
    }

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    p.num_sms = device_sms();
    const bool prefill = (int64_t)max_query_len * P.G > P.dec_rows_cap;
    CUtensorMap tq;
    if (prefill && !get_map(q, 3, D, (uint64_t)num_q_heads, (uint64_t)num_tokens, (uint32_t)P.G,
                            (uint32_t)(kPrefillRows / P.G), &tq))
        return PA_ERR_CUDA;
    // A mixed step with a side stream forks after the plan: prefill (persistent, on the plan's share
    // of the SMs, at the highest priority) on the side stream, decode (with its split merge) on the
    // caller's stream, which then waits for prefill.  The two kernels never touch the same output
    // rows.  Without a side stream prefill takes every SM and decode follows it on `stream`.
    const bool fork = prefill && P.NT > 0 && side != nullptr;
    p.pf_all_sms = fork ? 0 : 1;
    NvtxRange range(!fw ? "pa_attention_mixed" : fw->slots ? "pa_attention_mixed_write" : "pa_attention_decode_fused");
    cudaError_t e;
    if (fw && fw->slots) {
        // the step's KV write and its plan in one launch (neither reads what the other writes)
        bool vec_ok = false;
        const KvWriteArgs w = kv_write_args(fw->k_new, fw->v_new, fw->row_stride, fw->slots, num_tokens,
                                            const_cast<void *>(k_cache), const_cast<void *>(v_cache),
                                            cache->num_blocks, Hkv, D, nhd, &vec_ok);
        e = launch_write_plan(p, w, vec_ok, s);
    } else {
        e = launch_plan(p, s);
    }
    if (e != cudaSuccess)
        return PA_ERR_CUDA;
    if (fork && (cudaEventRecord(ev_fork, s) != cudaSuccess || cudaStreamWaitEvent(side, ev_fork, 0) != cudaSuccess))
        return PA_ERR_CUDA;
    if (prefill) {
        e = launch_prefill(p, tq, tk, tv, P.max_pf_tiles, p.num_sms, fork ? side : s);
        if (e != cudaSuccess)
            return PA_ERR_CUDA;
    }
    if (fork && cudaEventRecord(ev_join, side) != cudaSuccess)
        return PA_ERR_CUDA;
    if (P.NT > 0) {
        e = launch_decode(p, tk, tv, P.NT, P.max_dec_units, s);
        if (e != cudaSuccess)
            return PA_ERR_CUDA;
    }
    if (fork && cudaStreamWaitEvent(s, ev_join, 0) != cudaSuccess)
        return PA_ERR_CUDA;
    return PA_OK;
}

} // namespace

extern "C" {

pa_status_t pa_attention_mixed_ex(const void *q, int32_t num_q_heads, const void *k_cache, const void *v_cache,
                                  const pa_cache_desc_t *cache, const int32_t *query_start_loc,
                                  const int32_t *seq_lens, const int32_t *block_table, int32_t bt_stride,
                                  int32_t num_seqs, int32_t num_tokens, int32_t max_query_len, int32_t max_seq_len,
                                  float softmax_scale, void *out, float *lse, void *workspace,
                                  size_t workspace_bytes, const pa_attn_options_t *options, pa_stream_t stream)
{
    return attention_impl(q, num_q_heads, k_cache, v_cache, cache, query_start_loc, seq_lens, block_table, bt_stride,
                          num_seqs, num_tokens, max_query_len, max_seq_len, softmax_scale, out, lse, workspace,
                          workspace_bytes, options, nullptr, stream);
}

pa_status_t pa_attention_decode_fused(const void *q, int32_t num_q_heads, const void *k_new, const void *v_new,
                                      int64_t new_row_stride, void *k_cache, void *v_cache,
                                      const pa_cache_desc_t *cache, const int32_t *query_start_loc,
                                      const int32_t *seq_lens, const int32_t *block_table, int32_t bt_stride,
                                      int32_t num_seqs, int32_t num_tokens, int32_t max_query_len,
                                      int32_t max_seq_len, float softmax_scale, void *out, float *lse,
                                      void *workspace, size_t workspace_bytes, const pa_attn_options_t *options,
                                      pa_stream_t stream)
{
    const FusedWrite fw{k_new, v_new, new_row_stride, nullptr};
    return attention_impl(q, num_q_heads, k_cache, v_cache, cache, query_start_loc, seq_lens, block_table, bt_stride,
                          num_seqs, num_tokens, max_query_len, max_seq_len, softmax_scale, out, lse, workspace,
                          workspace_bytes, options, &fw, stream);
}

pa_status_t pa_attention_mixed_write(const void *q, int32_t num_q_heads, const void *k_new, const void *v_new,
                                     int64_t new_row_stride, const int64_t *slot_mapping, void *k_cache,
                                     void *v_cache, const pa_cache_desc_t *cache, const int32_t *query_start_loc,
                                     const int32_t *seq_lens, const int32_t *block_table, int32_t bt_stride,
                                     int32_t num_seqs, int32_t num_tokens, int32_t max_query_len,
                                     int32_t max_seq_len, float softmax_scale, void *out, float *lse,
                                     void *workspace, size_t workspace_bytes, const pa_attn_options_t *options,
                                     pa_stream_t stream)
{
    if (!slot_mapping)
        return PA_ERR_INVALID_ARG;
    const FusedWrite fw{k_new, v_new, new_row_stride, slot_mapping};
    return attention_impl(q, num_q_heads, k_cache, v_cache, cache, query_start_loc, seq_lens, block_table, bt_stride,
                          num_seqs, num_tokens, max_query_len, max_seq_len, softmax_scale, out, lse, workspace,
                          workspace_bytes, options, &fw, stream);
}

pa_status_t pa_kv_pack(const void *k_cache, const void *v_cache, const pa_cache_desc_t *cache,
                       const int32_t *block_ids, int32_t num_ids, void *staging, pa_stream_t stream)
{
    pa_status_t why;
    if (!cache_desc_ok(cache, &why))
        return why;
    if (num_ids < 0)
        return PA_ERR_INVALID_ARG;
    if (num_ids == 0)
        return PA_OK;
    if (!k_cache || !v_cache || !block_ids || !staging)
        return PA_ERR_INVALID_ARG;
    const int64_t block_elems = (int64_t)cache->num_kv_heads * kBlockSize * cache->head_dim;
    const size_t cache_bytes = (size_t)cache->num_blocks * block_elems * 2;
    const size_t stage_bytes = (size_t)num_ids * 2 * block_elems * 2;
    if (ranges_overlap(staging, stage_bytes, k_cache, cache_bytes) ||
        ranges_overlap(staging, stage_bytes, v_cache, cache_bytes))
        return PA_ERR_INVALID_ARG;
    if (!aligned16(k_cache) || !aligned16(v_cache) || !aligned16(staging) || !aligned16(block_ids))
        return PA_ERR_UNSUPPORTED;
    NvtxRange r("pa_kv_pack");
    return cuda_status(launch_kv_pack(k_cache, v_cache, cache->num_blocks, block_elems, block_ids, num_ids, staging,
                                      device_sms(), reinterpret_cast<cudaStream_t>(stream)));
}

pa_status_t pa_kv_unpack(const void *staging, const int32_t *block_ids, int32_t num_ids, void *k_cache,
                         void *v_cache, const pa_cache_desc_t *cache, pa_stream_t stream)
{
    pa_status_t why;
    if (!cache_desc_ok(cache, &why))
        return why;
    if (num_ids < 0)
        return PA_ERR_INVALID_ARG;
    if (num_ids == 0)
        return PA_OK;
    if (!k_cache || !v_cache || !block_ids || !staging)
        return PA_ERR_INVALID_ARG;
    const int64_t block_elems = (int64_t)cache->num_kv_heads * kBlockSize * cache->head_dim;
    const size_t cache_bytes = (size_t)cache->num_blocks * block_elems * 2;
    const size_t stage_bytes = (size_t)num_ids * 2 * block_elems * 2;
    if (ranges_overlap(staging, stage_bytes, k_cache, cache_bytes) ||
        ranges_overlap(staging, stage_bytes, v_cache, cache_bytes))
        return PA_ERR_INVALID_ARG;
    if (!aligned16(k_cache) || !aligned16(v_cache) || !aligned16(staging) || !aligned16(block_ids))
        return PA_ERR_UNSUPPORTED;
    NvtxRange r("pa_kv_unpack");
    return cuda_status(launch_kv_unpack(staging, block_ids, num_ids, k_cache, v_cache, cache->num_blocks, block_elems,
                                        device_sms(), reinterpret_cast<cudaStream_t>(stream)));
}

pa_status_t pa_attention_mixed(const void *q, int32_t num_q_heads, const void *k_cache, const void *v_cache,
                               const pa_cache_desc_t *cache, const int32_t *query_start_loc, const int32_t *seq_lens,
                               const int32_t *block_table, int32_t bt_stride, int32_t num_seqs, int32_t num_tokens,
                               int32_t max_query_len, int32_t max_seq_len, float softmax_scale, void *out, float *lse,
                               void *workspace, size_t workspace_bytes, pa_stream_t stream)
{
    return pa_attention_mixed_ex(q, num_q_heads, k_cache, v_cache, cache, query_start_loc, seq_lens, block_table,
                                 bt_stride, num_seqs, num_tokens, max_query_len, max_seq_len, softmax_scale, out, lse,
                                 workspace, workspace_bytes, nullptr, stream);
}

pa_status_t pa_merge_attn_states(const float *part_out, const float *part_lse, const int32_t *parts_per_row,
                                 int32_t num_rows, int32_t num_heads, int32_t num_parts, int32_t head_dim, void *out,
                                 float *lse_out, pa_stream_t stream)
{
    if (num_rows < 0 || num_heads <= 0 || num_parts < 0)
        return PA_ERR_INVALID_ARG;
    if (head_dim != 64 && head_dim != 128)
        return PA_ERR_UNSUPPORTED;
    if (num_rows == 0)
        return PA_OK;
    if (!out || (num_parts > 0 && (!part_out || !part_lse)))
        return PA_ERR_INVALID_ARG;
    if (!aligned16(part_out) || (reinterpret_cast<uintptr_t>(out) & 7u))
        return PA_ERR_UNSUPPORTED;
    NvtxRange r("pa_merge_attn_states");
    return cuda_status(launch_merge_states(part_out, part_lse, parts_per_row, num_rows, num_heads, num_parts, head_dim,
                                           out, lse_out, reinterpret_cast<cudaStream_t>(stream)));
}

pa_status_t pa_debug_gather_kv(const void *cache_ptr, const pa_cache_desc_t *cache, const int32_t *bt_row,
                               int32_t seq_len, void *out, pa_stream_t stream)
{
    pa_status_t why;
    if (!cache_desc_ok(cache, &why))
        return why;
    if (seq_len < 0)
        return PA_ERR_INVALID_ARG;
    if (seq_len == 0)
        return PA_OK;
    if (!cache_ptr || !bt_row || !out)
        return PA_ERR_INVALID_ARG;
    return cuda_status(launch_gather(cache_ptr, cache->num_blocks, cache->num_kv_heads, cache->head_dim,
                                     cache->layout == PA_LAYOUT_NHD, bt_row, seq_len, out,
                                     reinterpret_cast<cudaStream_t>(stream)));
}

} // extern "C"
