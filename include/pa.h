/*
 * pa.h -- C ABI of libpa_b200.so: paged attention over a block-managed KV
 * cache for NVIDIA B200 (sm_100a).
 *
 * The operations follow vLLM V1 as described in "Inside vLLM: Anatomy of a
 * High-Throughput LLM Inference System" (restated on hn.213312.xyz and
 * shengyayun.com):
 *   - the KV cache is a pool of fixed 16-token blocks handed out and taken back
 *     on demand, 16 tokens per block by default (hn.213312.xyz section 一,
 *     scheduler paragraph; shengyayun.com, 关键实现细节 1);
 *   - before the forward pass the runner copies metadata to the GPU and builds
 *     positions and the slot mapping; the forward pass then runs a custom
 *     paged-attention kernel over all sequences flattened into one
 *     "super-sequence" (hn.213312.xyz section 一, forward-pass paragraph);
 *   - one V1 step mixes prefill chunks and decode tokens (hn.213312.xyz
 *     section 一 "调度器"; shengyayun.com 适用场景); a chunk attends to its
 *     request's cached context and must give the same result as an unchunked
 *     prefill (hn.213312.xyz section 二.1); prefix-cache hits reuse cached
 *     blocks directly, so several block tables may name the same physical
 *     blocks (section 二.2; shengyayun.com 关键实现细节 2).
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller; only the
 *     pa_cache_desc_t / pa_attn_options_t structs are read from host memory,
 *     during the call (the prefix-cache functions are host-only, see there).
 *     The library never allocates device memory, creates a stream or an
 *     event, frees or synchronises: work is enqueued on `stream` (and, for a
 *     mixed step, on the caller's side stream given in pa_attn_options_t) and
 *     the call returns at once.
 *   - bf16 tensors are IEEE bfloat16 (2 bytes per element).
 *   - Host-side validation happens before anything is enqueued; a non-PA_OK
 *     status means nothing was enqueued, except PA_ERR_CUDA (a launch failed).
 *   - Metadata that lives on the device (seq_lens, block ids, slots) cannot be
 *     validated on the host.  The kernels never read or write outside the
 *     buffers described by the host-side sizes: a request whose lengths are
 *     inconsistent is skipped and a block id outside the pool reads zeros;
 *     both set a bit in the device status word (see pa_attention_mixed).
 */
#ifndef PA_B200_H
#define PA_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(PA_BUILD) && defined(__GNUC__)
#define PA_API __attribute__((visibility("default")))
#else
#define PA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* A cudaStream_t (the same handle type); NULL is the legacy default stream. */
typedef struct CUstream_st *pa_stream_t;
/* A cudaEvent_t (the same handle type). */
typedef struct CUevent_st *pa_event_t;

typedef enum pa_status {
    PA_OK = 0,
    PA_ERR_INVALID_ARG = 1,          /* null pointer, negative size, inconsistent shapes, aliasing */
    PA_ERR_UNSUPPORTED = 2,          /* valid but not implemented: head_dim, block_size, GQA ratio, alignment */
    PA_ERR_WORKSPACE_TOO_SMALL = 3,  /* workspace_bytes < pa_workspace_size_ex(...) */
    PA_ERR_CUDA = 4                  /* a CUDA launch or driver call failed */
} pa_status_t;

/* Layouts of one cache block (the pages fix only the block size, not the
 * order of the dimensions inside a block). */
#define PA_LAYOUT_HND 0 /* [num_blocks][num_kv_heads][block_size][head_dim]: one (block, kv head)
                           is block_size*head_dim*2 contiguous bytes (4 KiB at head_dim 128) */
#define PA_LAYOUT_NHD 1 /* [num_blocks][block_size][num_kv_heads][head_dim]: one token's rows of
                           all kv heads are contiguous */

/* K and V caches have the same shape: num_blocks blocks of block_size tokens x
 * num_kv_heads x head_dim bf16, contiguous, in the given layout.  A whole block
 * is num_kv_heads*block_size*head_dim*2 contiguous bytes in either layout.
 * Slot s is token s % block_size of block s / block_size. */
typedef struct pa_cache_desc {
    int64_t num_blocks;    /* > 0; num_blocks*num_kv_heads*block_size must be < 2^31 */
    int32_t num_kv_heads;  /* > 0 */
    int32_t head_dim;      /* 64 or 128 */
    int32_t block_size;    /* 16 (vLLM's default block size) */
    int32_t layout;        /* PA_LAYOUT_HND (0) or PA_LAYOUT_NHD (1); anything else is INVALID_ARG */
} pa_cache_desc_t;

/* Optional knobs of pa_attention_mixed_ex / pa_workspace_size_ex.  A NULL
 * options pointer, or a zero field, takes the default. */
typedef struct pa_attn_options {
    int32_t kv_split_tokens;       /* keys per split-KV partition of a decode request;
                                      a positive multiple of 16, used as given; 0 = the library
                                      chooses per step on the device: 1024, or, in a step without
                                      prefill work, 2048 / 4096 when the step's decode requests
                                      still give at least 12 split CTAs per SM at that size (the
                                      workspace is sized for 1024) */
    int32_t decode_max_query_len;  /* requests with q_len <= this take the memory-bound decode
                                      kernel instead of the tensor-core prefill kernel, e.g. k+1
                                      for speculative verification of k drafted tokens
                                      (shengyayun.com 关键实现细节 3: the target model checks the
                                      k candidates in one pass); 0 = default (8 / G query rows,
                                      at least 1).  Allowed up to 16 / G (G = num_q_heads /
                                      num_kv_heads), else PA_ERR_UNSUPPORTED.  -1: no decode
                                      kernel, every request takes the prefill kernel -- for
                                      batches known to hold only prefill work (a prefill
                                      instance under prefill/decode disaggregation); such a
                                      call never runs a decode grid beside prefill. */
    int32_t reserved[6];           /* must be zero */
    /* How the two kernels of a step that holds both prefill-shaped and decode-shaped requests
     * run.  The pages' V1 scheduler puts both kinds of work in one step (hn.213312.xyz section
     * 一, "调度器"); prefill is bound by the tensor cores and decode by HBM, so they run best side
     * by side.  side_stream: a second stream of the caller's, on the same device as `stream`,
     * for the prefill kernel; fork_event / join_event: two events the call records and waits on
     * to fork from `stream` and join back to it, so that the call stays one ordered unit on
     * `stream` (and can be captured into a CUDA graph with `stream`).  All three NULL: the
     * kernels run one after the other on `stream`.  Either all three or none (else
     * INVALID_ARG); side_stream must differ from `stream`.  The caller owns them: the library
     * creates no stream or event.  Calls that can be issued at the same time (other host
     * threads, or other streams) need their own three. */
    pa_stream_t side_stream;
    pa_event_t fork_event;
    pa_event_t join_event;
} pa_attn_options_t;

/* Bits of the device status word (uint32 at byte 0 of the workspace). */
#define PA_DEVICE_BAD_SEQ 1u      /* a request had q_len < 0, q_len > max_query_len, seq_len < q_len,
                                     seq_len > max_seq_len or query rows outside [0, num_tokens); it was
                                     skipped.  Also set when requests' query rows overlap (query_start_loc
                                     decreasing somewhere) so far that their work does not fit the
                                     workspace: the work that fits is done, the rest is dropped */
#define PA_DEVICE_BAD_BLOCK 2u    /* a block id outside [0, num_blocks) was read (as zeros) */
#define PA_DEVICE_WAIT_TIMEOUT 4u /* a kernel gave up waiting on a copy or a tensor-core result */
#define PA_DEVICE_BAD_SLOT 8u     /* pa_kv_write_ex: a slot >= num_blocks*block_size was skipped */

PA_API int32_t pa_abi_version(void); /* 4 */
PA_API const char *pa_status_string(pa_status_t status);

/*
 * pa_kv_write -- scatter this step's new K and V rows into their cache slots.
 * (hn.213312.xyz section 一: the slot mapping is built while inputs are
 * prepared, and the KV tensors are allocated and bound once at start-up.)
 *
 *   k_cache[s / bs][h][s % bs][:] = k_new row t, head h   (same for V)
 * for every token t < num_tokens with s = slot_mapping[t] >= 0 and every
 * h < num_kv_heads.
 *
 * k_new, v_new: bf16; token t's row starts at element t*new_row_stride and
 *   holds num_kv_heads*head_dim contiguous elements ([T, Hkv, D] when
 *   new_row_stride == Hkv*D; larger strides read rows out of a fused QKV).
 * slot_mapping: int64 [num_tokens]; < 0 marks a padding token (skipped).  A
 *   slot >= num_blocks*block_size is skipped too.  Two tokens with the same
 *   non-negative slot in one call leave that slot undefined.
 * The copy is bit-exact; no other cache byte is written.
 */
PA_API pa_status_t pa_kv_write(const void *k_new, const void *v_new, int64_t new_row_stride,
                        const int64_t *slot_mapping, int32_t num_tokens, void *k_cache, void *v_cache,
                        const pa_cache_desc_t *cache, pa_stream_t stream);

/*
 * pa_kv_write_ex -- pa_kv_write that also reports slots outside the pool.
 * (The pages' block manager hands out and takes back whole blocks on demand,
 * shengyayun.com 关键实现细节 1, and the runner builds the slot mapping from
 * those blocks while preparing inputs, hn.213312.xyz section 一; a slot past
 * the pool therefore means corrupt metadata, which this call makes visible.)
 * status: NULL, or a device uint32 (4-byte aligned, else INVALID_ARG) into
 * which the kernel ORs PA_DEVICE_BAD_SLOT when a token's slot is >=
 * num_blocks*block_size (that token is skipped as in pa_kv_write).  The call
 * never clears it: the caller zeroes it before the calls it wants to check.
 */
PA_API pa_status_t pa_kv_write_ex(const void *k_new, const void *v_new, int64_t new_row_stride,
                                  const int64_t *slot_mapping, int32_t num_tokens, void *k_cache, void *v_cache,
                                  const pa_cache_desc_t *cache, uint32_t *status, pa_stream_t stream);

/*
 * pa_build_slot_mapping -- the slot of every token of the step.
 * (hn.213312.xyz section 一, forward-pass paragraph: positions and the slot
 * mapping are prepared on the way into the forward pass.)
 * Token i of request r (row query_start_loc[r] + i) sits at position
 * p = seq_lens[r] - q_len_r + i and gets
 *   slot = block_table[r*bt_stride + p / 16] * 16 + p % 16.
 * query_start_loc int32 [num_seqs+1] (non-decreasing, last <= num_tokens),
 * seq_lens int32 [num_seqs], block_table int32 [num_seqs, bt_stride],
 * slot_mapping int64 [num_tokens] out.  Rows of a request with
 * seq_len < q_len, or whose block index would reach bt_stride, get -1.
 * Rows not covered by any request are left untouched.
 */
PA_API pa_status_t pa_build_slot_mapping(const int32_t *query_start_loc, const int32_t *seq_lens,
                                  const int32_t *block_table, int32_t bt_stride, int32_t num_seqs,
                                  int32_t num_tokens, int64_t *slot_mapping, pa_stream_t stream);

/*
 * pa_workspace_size[_ex] -- bytes of device workspace pa_attention_mixed[_ex]
 * needs for these host-side bounds (0 on invalid arguments).  The value only
 * grows with each argument, so one workspace sized for the largest step of a
 * run serves every smaller step.
 * (The pages' runner captures the forward pass in CUDA graphs when a worker
 * starts, hn.213312.xyz section 一, and its KV tensors are allocated once up
 * front; a step replayed from a graph cannot allocate, so the scratch a call
 * needs -- work lists, split-KV partial states, the status word -- is sized
 * here from host bounds alone and owned by the caller.)
 */
PA_API size_t pa_workspace_size(int32_t num_seqs, int32_t num_tokens, int32_t num_q_heads,
                         const pa_cache_desc_t *cache, int32_t max_seq_len);
PA_API size_t pa_workspace_size_ex(int32_t num_seqs, int32_t num_tokens, int32_t num_q_heads,
                            const pa_cache_desc_t *cache, int32_t max_seq_len,
                            const pa_attn_options_t *options);

/*
 * pa_attention_mixed[_ex] -- causal attention of one mixed prefill/decode
 * step over the paged cache.
 * (hn.213312.xyz section 一 forward-pass paragraph and sections 二.1/二.2;
 *  shengyayun.com 适用场景: the V1 scheduler puts prefill and decode work in
 *  the same step.)
 *
 * Request r owns query rows [query_start_loc[r], query_start_loc[r+1]) of q;
 * q_len_r is their count, seq_lens[r] = L_r counts its tokens in the cache
 * including this step's (pa_kv_write must already have run on this stream),
 * and c_r = L_r - q_len_r tokens were cached before the step.  Row i of the
 * request is at position p = c_r + i; query head h uses kv head
 * h / (num_q_heads / num_kv_heads) and attends keys 0..p of its request:
 *   out[row][h] = sum_j softmax_j(softmax_scale * q . K_j) V_j.
 * Key j of request r lives at block block_table[r*bt_stride + j/16], row j%16.
 * Requests may appear in any order and may share physical blocks.
 *
 * q: bf16 [num_tokens, num_q_heads, head_dim], 16-byte aligned.
 * k_cache, v_cache: per `cache`, 16-byte aligned.
 * query_start_loc: int32 [num_seqs+1]; seq_lens: int32 [num_seqs];
 * block_table: int32 [num_seqs, bt_stride] with bt_stride >= ceil(max_seq_len/16);
 *   entries past ceil(L_r/16) are never read.
 * max_query_len, max_seq_len: host-side upper bounds of q_len_r and L_r.
 * out: bf16 [num_tokens, num_q_heads, head_dim]; must not overlap q.  Rows
 *   that belong to no request are not written.
 * lse: fp32 [num_tokens, num_q_heads] natural-log log-sum-exp of the scaled
 *   scores, or NULL; must not overlap q or out.
 * workspace: device memory of at least pa_workspace_size_ex(...) bytes,
 *   16-byte aligned, not overlapping q, out or lse, used only while the
 *   enqueued work runs; calls that can run concurrently need distinct
 *   workspaces.  Byte 0 holds the device status
 *   word (PA_DEVICE_* bits), reset by every call and readable after it.
 *
 * Supported: head_dim 64 or 128, block_size 16, num_q_heads/num_kv_heads a
 * divisor of 128.  Errors: INVALID_ARG (null pointer, negative size,
 * num_q_heads % num_kv_heads != 0, bt_stride too small, q / out / lse /
 * workspace overlapping, nonzero reserved option), UNSUPPORTED,
 * WORKSPACE_TOO_SMALL, CUDA.
 *
 * Concurrency inside a call: when a step can hold both prefill-shaped and
 * decode-shaped requests and options name a side stream and two events, the
 * prefill kernel runs on the side stream beside the decode kernel on
 * `stream`, on an SM share the device plan picks; `stream` waits for it
 * before the call's work is complete (an event fork/join, so the call is
 * still one ordered unit on `stream` and can be captured into a CUDA graph).
 * Without them (and always for pa_attention_mixed) the prefill kernel takes
 * every SM and the decode kernel runs after it on `stream`.  `stream` (and the
 * side stream) must belong to the current device: every launch goes to the
 * current device (the call does not query a stream's device, which is not
 * allowed while the stream is being captured).
 */
PA_API pa_status_t pa_attention_mixed(const void *q, int32_t num_q_heads, const void *k_cache,
                               const void *v_cache, const pa_cache_desc_t *cache,
                               const int32_t *query_start_loc, const int32_t *seq_lens,
                               const int32_t *block_table, int32_t bt_stride, int32_t num_seqs,
                               int32_t num_tokens, int32_t max_query_len, int32_t max_seq_len,
                               float softmax_scale, void *out, float *lse, void *workspace,
                               size_t workspace_bytes, pa_stream_t stream);
PA_API pa_status_t pa_attention_mixed_ex(const void *q, int32_t num_q_heads, const void *k_cache,
                                  const void *v_cache, const pa_cache_desc_t *cache,
                                  const int32_t *query_start_loc, const int32_t *seq_lens,
                                  const int32_t *block_table, int32_t bt_stride, int32_t num_seqs,
                                  int32_t num_tokens, int32_t max_query_len, int32_t max_seq_len,
                                  float softmax_scale, void *out, float *lse, void *workspace,
                                  size_t workspace_bytes, const pa_attn_options_t *options,
                                  pa_stream_t stream);

/*
 * pa_attention_mixed_noalloc -- pa_attention_mixed_ex for callers that cannot
 * allocate device memory.  (No counterpart in the paper: an addition of this
 * library.)
 *
 * Some callers cannot call cudaMalloc or any allocator at the point where
 * attention runs: code inside a stream that is being captured by another
 * framework, a plugin host that owns every allocation, or a runtime whose
 * memory is fully reserved up front.  This entry point needs no workspace
 * argument: it uses a scratch array compiled into the library, of
 * PA_NOALLOC_SCRATCH_BYTES bytes, which every GPU that loads the library
 * holds until the process exits.  The caller still passes q, the caches, the
 * metadata, out and lse exactly as for pa_attention_mixed_ex, and the results
 * are the same.
 *
 *  - The first call on a device looks up that device's copy of the array
 *    (cudaGetSymbolAddress) with the device current; make that first call
 *    before any stream capture on that device.  As with every attention
 *    entry point, the first launch of each kernel shape on a device (head
 *    dim 64 or 128; decode-only, prefill-only or mixed) also sets that
 *    kernel's shared-memory size attribute (cudaFuncSetAttribute) once.
 *    Beyond those one-time calls a call does only its launches (and, for a
 *    mixed step with the options' side stream, the event record / wait
 *    pairs).
 *  - Bounds that need more than PA_NOALLOC_SCRATCH_BYTES of workspace
 *    (pa_workspace_size_ex(...) > PA_NOALLOC_SCRATCH_BYTES) are rejected with
 *    PA_ERR_WORKSPACE_TOO_SMALL before anything is enqueued; a larger
 *    kv_split_tokens shrinks the need of long-context decode batches.
 *  - Every call on a device shares the one array.  Calls whose work can
 *    overlap on the GPU (different streams, no ordering between them) race on
 *    it and give undefined results; calls ordered on one stream are safe.
 *    The array keeps the previous call's contents; each call re-initialises
 *    everything it reads (status word included) before reading it.
 *  - The device status word (PA_DEVICE_* bits) sits in the array too; read
 *    it with pa_noalloc_device_status after the call.
 *  - Nothing here calls cudaMalloc, cudaFree or any allocating routine.
 */
#define PA_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)
PA_API pa_status_t pa_attention_mixed_noalloc(const void *q, int32_t num_q_heads, const void *k_cache,
                                              const void *v_cache, const pa_cache_desc_t *cache,
                                              const int32_t *query_start_loc, const int32_t *seq_lens,
                                              const int32_t *block_table, int32_t bt_stride, int32_t num_seqs,
                                              int32_t num_tokens, int32_t max_query_len, int32_t max_seq_len,
                                              float softmax_scale, void *out, float *lse,
                                              const pa_attn_options_t *options, pa_stream_t stream);

/*
 * pa_noalloc_device_status -- the device status word of the last
 * pa_attention_mixed_noalloc call on the current device.  (No counterpart in
 * the paper: the status word normally sits at byte 0 of the caller's
 * workspace, and callers of the allocation-free entry point have none.)
 * Enqueues one 4-byte copy on `stream` from the built-in array to status_out
 * (host or device memory; a host pointer can be read once `stream` has
 * synchronised).  Order it after the call on the same stream.  INVALID_ARG
 * for a NULL status_out.
 */
PA_API pa_status_t pa_noalloc_device_status(uint32_t *status_out, pa_stream_t stream);

/*
 * pa_merge_attn_states -- the split-KV reduce on its own.
 * Given attention states of num_parts disjoint key sets for each (row, head):
 * normalised outputs part_out fp32 [num_rows, num_heads, num_parts, head_dim]
 * and log-sum-exps part_lse fp32 [num_rows, num_heads, num_parts] (natural
 * log; -inf marks an empty part), write
 *   LSE = ln sum_s exp(lse_s),  out = sum_s exp(lse_s - LSE) * o_s
 * as bf16 out [num_rows, num_heads, head_dim] and, if lse_out is not NULL,
 * fp32 lse_out [num_rows, num_heads].  parts_per_row (int32 [num_rows], may be
 * NULL) limits row i to its first parts_per_row[i] parts.  A row whose parts
 * are all empty gets out = 0, lse = -inf.  head_dim 64 or 128.
 */
PA_API pa_status_t pa_merge_attn_states(const float *part_out, const float *part_lse, const int32_t *parts_per_row,
                                 int32_t num_rows, int32_t num_heads, int32_t num_parts, int32_t head_dim,
                                 void *out, float *lse_out, pa_stream_t stream);

/*
 * pa_attention_decode_fused -- KV write and decode attention of a decode step
 * in one pass.  (hn.213312.xyz section 一, forward-pass paragraph: each step
 * writes the new tokens' K/V into their slots, then attends over the cache.)
 *
 * Same arguments, rules and results as pa_attention_mixed_ex, plus this
 * step's new rows k_new/v_new (bf16, token t's row at element
 * t*new_row_stride, [Hkv, head_dim] contiguous, as for pa_kv_write).  The
 * new rows of every request -- positions c_r .. L_r-1, slot taken from the
 * block table as pa_build_slot_mapping does -- are stored into k_cache /
 * v_cache by the attention kernel itself, which also places them straight
 * into the tile it attends over instead of reading them back.  The cache
 * bytes afterwards equal those of pa_kv_write with that slot mapping, and
 * out / lse are bit-identical to pa_kv_write followed by
 * pa_attention_mixed_ex.  Requests skipped for bad metadata (device status
 * bit PA_DEVICE_BAD_SEQ) and rows in a block whose id is outside the pool
 * are not written.
 *
 * Every request must take the decode kernel: max_query_len * G must not
 * exceed the decode row limit (8 rows per kv head by default, 16 with
 * options->decode_max_query_len), else PA_ERR_UNSUPPORTED.  k_new, v_new
 * 16-byte aligned with new_row_stride a multiple of 8, else UNSUPPORTED.
 * The workspace is sized by pa_workspace_size_ex as for the unfused call.
 */
PA_API pa_status_t pa_attention_decode_fused(const void *q, int32_t num_q_heads, const void *k_new,
                                             const void *v_new, int64_t new_row_stride, void *k_cache,
                                             void *v_cache, const pa_cache_desc_t *cache,
                                             const int32_t *query_start_loc, const int32_t *seq_lens,
                                             const int32_t *block_table, int32_t bt_stride, int32_t num_seqs,
                                             int32_t num_tokens, int32_t max_query_len, int32_t max_seq_len,
                                             float softmax_scale, void *out, float *lse, void *workspace,
                                             size_t workspace_bytes, const pa_attn_options_t *options,
                                             pa_stream_t stream);

/*
 * pa_attention_mixed_write -- a whole step's KV write and attention, any
 * step shape.  (hn.213312.xyz section 一, forward-pass paragraph: each step
 * writes the new tokens' K/V into their slots, then attends over the cache.)
 *
 * Same arguments, rules and results as pa_attention_mixed_ex, plus this
 * step's new rows k_new/v_new (bf16, token t's row at element
 * t*new_row_stride, [Hkv, head_dim] contiguous) and slot_mapping (int64
 * [num_tokens], as for pa_kv_write).  The rows are written by the same
 * launch that plans the step (its first kernel: one CTA plans while the
 * others write; neither reads what the other writes), so the plan costs no
 * time of its own.  Cache bytes afterwards equal those of pa_kv_write with
 * that slot mapping; out / lse are bit-identical to pa_kv_write followed by
 * pa_attention_mixed_ex.  A slot outside the pool writes nothing and sets
 * PA_DEVICE_BAD_SLOT in the status word at byte 0 of the workspace, beside
 * the attention's own bits.  The workspace is sized by pa_workspace_size_ex.
 * PA_ERR_INVALID_ARG for a NULL slot_mapping / k_new / v_new or
 * new_row_stride < Hkv*head_dim.  (No counterpart on the pages: an engine
 * entry point that folds the plan into the step's first kernel.)
 */
PA_API pa_status_t pa_attention_mixed_write(const void *q, int32_t num_q_heads, const void *k_new,
                                            const void *v_new, int64_t new_row_stride, const int64_t *slot_mapping,
                                            void *k_cache, void *v_cache, const pa_cache_desc_t *cache,
                                            const int32_t *query_start_loc, const int32_t *seq_lens,
                                            const int32_t *block_table, int32_t bt_stride, int32_t num_seqs,
                                            int32_t num_tokens, int32_t max_query_len, int32_t max_seq_len,
                                            float softmax_scale, void *out, float *lse, void *workspace,
                                            size_t workspace_bytes, const pa_attn_options_t *options,
                                            pa_stream_t stream);

/*
 * pa_kv_pack / pa_kv_unpack -- copy whole cache blocks to and from a
 * contiguous staging buffer, e.g. to move a request's KV between a prefill
 * instance and a decode instance (hn.213312.xyz section 二, item 5, and
 * shengyayun.com 关键实现细节 item 4: with prefill/decode disaggregation the
 * prefill side hands its finished KV blocks to the decode side through a
 * transfer connector).
 *
 * staging: bf16 [num_ids][2][block_elems], block_elems =
 *   num_kv_heads*block_size*head_dim; entry i holds block block_ids[i] of
 *   k_cache (index 0) then of v_cache (index 1), byte for byte in the cache's
 *   own layout (a receiver must use the same layout and head_dim).
 * pack:   staging[i][0] = k_cache block block_ids[i], staging[i][1] = v block;
 *         an id outside [0, num_blocks) packs zeros.
 * unpack: the inverse, k_cache block block_ids[i] = staging[i][0] (same for
 *         V); an id outside the pool is skipped, no other cache byte is
 *         written.  Duplicate ids in one unpack leave those blocks undefined.
 * block_ids: device int32 [num_ids].  Every pointer 16-byte aligned, else
 * PA_ERR_UNSUPPORTED; staging must not overlap the caches.
 */
PA_API pa_status_t pa_kv_pack(const void *k_cache, const void *v_cache, const pa_cache_desc_t *cache,
                              const int32_t *block_ids, int32_t num_ids, void *staging, pa_stream_t stream);
PA_API pa_status_t pa_kv_unpack(const void *staging, const int32_t *block_ids, int32_t num_ids, void *k_cache,
                                void *v_cache, const pa_cache_desc_t *cache, pa_stream_t stream);

/*
 * Prefix caching on the host: chained block hashes and the longest cached
 * prefix.  (shengyayun.com 关键实现细节 item 2: the scheduler hashes each
 * request in 16-token blocks -- a built-in hash by default, SHA-256 against
 * collisions -- and find_longest_cache_hit walks the hashes in order through
 * the map from block hash to cached block, reusing every hit's KV block as it
 * is; item 1: only whole blocks are reused, a trailing partial block is not.
 * hn.213312.xyz section 二, item 2.)
 *
 * All pointers of these functions are HOST pointers; nothing touches the GPU.
 *
 * Block b (tokens 16b .. 16b+15) gets the digest of the byte string
 *   parent (32 bytes) || its 16 token ids as little-endian int32,
 * where parent is block b-1's digest, or *root for block 0 (32 zero bytes if
 * root is NULL; a caller may fold extra keys into it).  Equal digests thus
 * stand for equal whole prefixes.  PA_HASH_FNV1A64: 64-bit FNV-1a, stored
 * little-endian in bytes 0..7, bytes 8..31 zero.  PA_HASH_SHA256: SHA-256
 * (FIPS 180-4), all 32 bytes.
 */
#define PA_HASH_FNV1A64 0
#define PA_HASH_SHA256 1
typedef struct pa_block_hash {
    uint8_t bytes[32];
} pa_block_hash_t;

/* Digests of the num_tokens / 16 full blocks of token_ids (host int32
 * [num_tokens]) into out_hashes (host, room for num_tokens / 16 entries);
 * *num_blocks receives that count.  INVALID_ARG on a negative count, a null
 * pointer that is needed, or an unknown algo. */
PA_API pa_status_t pa_prefix_block_hashes(const int32_t *token_ids, int64_t num_tokens, const pa_block_hash_t *root,
                                          int32_t algo, pa_block_hash_t *out_hashes, int64_t *num_blocks);

/* A map from block digest to physical block id, and back (one digest per
 * block).  Safe to call from several host threads. */
typedef struct pa_prefix_cache pa_prefix_cache_t;
PA_API pa_prefix_cache_t *pa_prefix_cache_create(void); /* NULL if out of host memory */
PA_API void pa_prefix_cache_destroy(pa_prefix_cache_t *cache);
/* Record that block block_ids[i] holds the KV of the prefix hashes[i] names.
 * A digest or a block already present keeps its first mapping.  Block ids
 * must be >= 0 (else INVALID_ARG, nothing recorded). */
PA_API pa_status_t pa_prefix_cache_insert(pa_prefix_cache_t *cache, const pa_block_hash_t *hashes,
                                          const int32_t *block_ids, int32_t n);
/* Forget block_id (when the allocator hands it out for other tokens). */
PA_API pa_status_t pa_prefix_cache_remove_block(pa_prefix_cache_t *cache, int32_t block_id);
/* Longest cached prefix: walks hashes[0..n) in order, writes the cached block
 * of each hit to out_block_ids and stops at the first miss.  Returns the
 * number of hits, or -1 on invalid arguments. */
PA_API int32_t pa_prefix_cache_longest_hit(pa_prefix_cache_t *cache, const pa_block_hash_t *hashes, int32_t n,
                                           int32_t *out_block_ids);
PA_API int64_t pa_prefix_cache_size(pa_prefix_cache_t *cache); /* digests held, -1 for NULL */

/*
 * pa_debug_gather_kv -- test helper: contiguous copy of one request's first
 * seq_len tokens of a cache, following its block table row (device int32
 * [ceil(seq_len/16)]).  out: bf16 [seq_len, num_kv_heads, head_dim].  A block
 * id outside the pool gives zero rows.
 * (Token j of a request lives in block block_table[j / 16] at row j % 16 --
 * the pages' fixed 16-token blocks handed out by the block manager,
 * shengyayun.com 关键实现细节 1, indexed through the per-request block table,
 * hn.213312.xyz section 一.  This copy lets tests check that index handling
 * byte for byte against a plain walk of the table.)
 */
PA_API pa_status_t pa_debug_gather_kv(const void *cache_ptr, const pa_cache_desc_t *cache, const int32_t *bt_row,
                               int32_t seq_len, void *out, pa_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* PA_B200_H */
