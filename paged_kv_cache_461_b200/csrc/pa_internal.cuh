// pa_internal.cuh -- parameters, workspace layout and launchers shared by the
// host layer (pa_api.cu) and the kernels.  Not part of the public ABI.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "../../include/pa.h"

namespace pa {

constexpr int kBlockSize = 16;           // tokens per KV block
constexpr int kDefaultSplitTokens = 1024; // keys per split-KV partition of a decode request
constexpr int kPrefillRows = 128;        // query rows (tokens x grouped heads) per prefill tile
constexpr int kPrefillRowsPerCta = 256;  // a prefill work item is a pair of tiles

// Device-visible counters at the start of the workspace (one 256-byte header).
struct WsHeader {
    uint32_t status;      // PA_DEVICE_* bits
    uint32_t n_dec_units; // (request, split) decode work items
    uint32_t n_pf_tiles;  // (request, q-tile) prefill work items
    uint32_t n_reduce;    // decode requests with more than one split (merged by their last split CTA)
    uint32_t pf_ctas;     // persistent prefill CTAs that take work; the others leave their SM to decode
    uint32_t split_tokens; // keys per split-KV partition of this step's decode requests
    uint32_t write_epoch;  // call id published once the status word is cleared (write-and-plan launch);
                           // kWriteEpochIdle once the step's attention kernels have started
    uint32_t pad[57];
};

// write_epoch between calls: the attention kernels of a step (which start only after its write-and-plan
// launch has finished) set it to this value, which no call id takes.  A launch replayed from a CUDA graph
// keeps its call id, so without the reset its writers could take the previous replay's epoch for this one's.
constexpr uint32_t kWriteEpochIdle = 0xFFFFFFFFu;
static_assert(sizeof(WsHeader) == 256, "header is 256 bytes");

// How a call is decomposed (host side, from the host hints only).
struct Plan {
    int G = 1;              // q heads per kv head
    int NT = 0;             // 8-row query groups per decode warp (0: no decode path)
    int dec_rows_cap = 0;   // requests with q_len*G <= this take the decode kernel
    int QD = 0;             // max query tokens of a decode request
    int split_tokens = kDefaultSplitTokens;
    int max_splits = 1;
    int64_t max_dec_units = 0;
    int64_t max_pf_tiles = 0;
    bool need_prefill = false;
    bool need_reduce = false;
    // byte offsets inside the workspace
    size_t off_dec = 0, off_pf = 0, off_red = 0, off_part_o = 0, off_part_lse = 0, total = 0;
};

struct AttnParams {
    const __nv_bfloat16 *q;
    __nv_bfloat16 *out;
    float *lse;                 // nullable
    const int32_t *qsl;
    const int32_t *seq_lens;
    const int32_t *bt;
    int64_t num_blocks;
    int bt_stride;
    int num_seqs;
    int num_tokens;
    int max_seq_len;
    int max_query_len;          // host bound of q_len; a request above it is skipped (PA_DEVICE_BAD_SEQ)
    int64_t max_dec_units;      // room of the decode work list in the workspace
    int64_t max_pf_tiles;       // room of the prefill work list in the workspace
    int Hq, Hkv, G, D;
    float scale_log2;           // softmax_scale * log2(e)
    WsHeader *hdr;
    int2 *dec_units;            // (r, split)
    int2 *pf_tiles;             // (r, q-tile)
    uint32_t *split_arrivals;   // [num_seqs * Hkv] split CTAs of (request, kv head) done so far
    float *part_o;              // [num_seqs*QD*Hq*max_splits, D]
    float *part_lse;            // [num_seqs*QD*Hq*max_splits]
    int split_tokens, max_splits, QD, dec_rows_cap;
    int auto_split;             // 1: the plan may take 2x or 4x split_tokens (the caller left the split to the library)
    int nhd;                    // cache layout PA_LAYOUT_NHD (else HND)
    int num_sms;                // SMs of the device (the plan splits them between prefill and decode)
    int pf_all_sms;             // 1: prefill runs alone (every SM); 0: beside decode on the plan's share
    // fused KV write (pa_attention_decode_fused); k_new == nullptr otherwise
    const uint16_t *k_new, *v_new;
    int64_t new_row_stride;     // elements
    uint16_t *k_cache_w, *v_cache_w;
};

// launchers (return cudaGetLastError() of the launch)
cudaError_t launch_kv_write(const void *k_new, const void *v_new, int64_t row_stride, const int64_t *slots,
                            int num_tokens, void *k_cache, void *v_cache, int64_t num_blocks, int Hkv, int D,
                            int nhd, uint32_t *status, cudaStream_t s);
cudaError_t launch_kv_pack(const void *k_cache, const void *v_cache, int64_t num_blocks, int64_t block_elems,
                           const int32_t *ids, int num_ids, void *staging, int num_sms, cudaStream_t s);
cudaError_t launch_kv_unpack(const void *staging, const int32_t *ids, int num_ids, void *k_cache, void *v_cache,
                             int64_t num_blocks, int64_t block_elems, int num_sms, cudaStream_t s);
cudaError_t launch_slot_mapping(const int32_t *qsl, const int32_t *seq_lens, const int32_t *bt, int bt_stride,
                                int num_seqs, int num_tokens, int64_t *slots, cudaStream_t s);
cudaError_t launch_gather(const void *cache, int64_t num_blocks, int Hkv, int D, int nhd, const int32_t *bt_row,
                          int seq_len, void *out, cudaStream_t s);
cudaError_t launch_plan(const AttnParams &p, cudaStream_t s);
struct KvWriteArgs;
cudaError_t launch_write_plan(const AttnParams &p, const KvWriteArgs &w, bool vec_ok, cudaStream_t s);
cudaError_t launch_decode(const AttnParams &p, const CUtensorMap &tk, const CUtensorMap &tv, int NT,
                          int64_t grid_units, cudaStream_t s);
cudaError_t launch_merge_states(const float *part_out, const float *part_lse, const int32_t *parts_per_row,
                                int num_rows, int num_heads, int num_parts, int D, void *out, float *lse_out,
                                cudaStream_t s);
cudaError_t launch_prefill(const AttnParams &p, const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                           int64_t grid_tiles, int num_sms, cudaStream_t s);

} // namespace pa
