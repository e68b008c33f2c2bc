// pa_noalloc.cu -- pa_attention_mixed_noalloc: the mixed-step attention for
// callers that cannot allocate device memory.  Its workspace is a file-scope
// __device__ array of PA_NOALLOC_SCRATCH_BYTES (64 MiB) compiled into the
// library; each device that loads the library holds its own copy until exit.
//
// In host code `g_pa_noalloc_scratch` names a host-side stand-in, not device
// memory, so its device address is looked up once per device with
// cudaGetSymbolAddress (that device current) and cached here.  Calls share the
// array: ones that overlap on the GPU race; ones ordered on a stream do not.
// The plan kernel that starts every call rewrites all state the later kernels
// read (status word, work lists), so no clearing is needed between calls.
#include <mutex>

#include "pa_internal.cuh"

namespace {

static __device__ __align__(256) uint8_t g_pa_noalloc_scratch[PA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void *g_scratch_ptr[kMaxDevices] = {};

// Device address of this device's copy of the scratch array (nullptr on failure).
void *scratch_for_current_device()
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return nullptr;
    std::lock_guard<std::mutex> g(g_scratch_mu);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_pa_noalloc_scratch) != cudaSuccess || !p)
            return nullptr;
        g_scratch_ptr[dev] = p;
    }
    return g_scratch_ptr[dev];
}

} // namespace

extern "C" PA_API pa_status_t pa_attention_mixed_noalloc(const void *q, int32_t num_q_heads, const void *k_cache,
                                                         const void *v_cache, const pa_cache_desc_t *cache,
                                                         const int32_t *query_start_loc, const int32_t *seq_lens,
                                                         const int32_t *block_table, int32_t bt_stride,
                                                         int32_t num_seqs, int32_t num_tokens, int32_t max_query_len,
                                                         int32_t max_seq_len, float softmax_scale, void *out,
                                                         float *lse, const pa_attn_options_t *options,
                                                         pa_stream_t stream)
{
    const size_t need = pa_workspace_size_ex(num_seqs, num_tokens, num_q_heads, cache, max_seq_len, options);
    if (need == 0)
        return pa_attention_mixed_ex(q, num_q_heads, k_cache, v_cache, cache, query_start_loc, seq_lens, block_table,
                                     bt_stride, num_seqs, num_tokens, max_query_len, max_seq_len, softmax_scale, out,
                                     lse, nullptr, 0, options, stream); // reports the argument error
    if (need > PA_NOALLOC_SCRATCH_BYTES)
        return PA_ERR_WORKSPACE_TOO_SMALL;
    void *scratch = scratch_for_current_device();
    if (!scratch)
        return PA_ERR_CUDA;
    return pa_attention_mixed_ex(q, num_q_heads, k_cache, v_cache, cache, query_start_loc, seq_lens, block_table,
                                 bt_stride, num_seqs, num_tokens, max_query_len, max_seq_len, softmax_scale, out, lse,
                                 scratch, PA_NOALLOC_SCRATCH_BYTES, options, stream);
}

extern "C" PA_API pa_status_t pa_noalloc_device_status(uint32_t *status_out, pa_stream_t stream)
{
    if (!status_out)
        return PA_ERR_INVALID_ARG;
    void *scratch = scratch_for_current_device();
    if (!scratch)
        return PA_ERR_CUDA;
    // the status word is the first field of the workspace header, at byte 0
    return cudaMemcpyAsync(status_out, scratch, sizeof(uint32_t), cudaMemcpyDefault,
                           reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
               ? PA_OK
               : PA_ERR_CUDA;
}
