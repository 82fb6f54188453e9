// paged_decode_attention_noalloc: the decode attention of decode.cu for
// callers that cannot allocate device memory.
//
// Some callers of this library cannot call cudaMalloc: a host program that
// reserved all of the GPU's memory for its own allocator at start-up (so a
// fresh cudaMalloc fails or fragments that reservation), or a latency-critical
// serving loop where cudaMalloc's implicit device-wide synchronisation is not
// acceptable. They cannot provide the split-K workspace that
// paged_decode_attention asks for, so this entry point brings its own: a
// fixed array in the library's device memory, reserved on every GPU that
// loads the library and kept until the process exits.
#include <mutex>

#include "common.cuh"

namespace {

// The workspace lives here. Device memory of this size is reserved on every
// GPU that loads the library; calls needing more are refused.
static __device__ __align__(256) unsigned char g_decode_scratch[KVP_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_scratch_addr[kMaxDevices];  // device address of g_decode_scratch, per device

// Looks up (once per device, with that device current) the device address
// of the scratch array. In host code the array's name is only a host-side
// stand-in, never an address a kernel may use.
int scratch_address(int dev, void **out)
{
    if (dev < 0 || dev >= kMaxDevices) return kvp::set_error(KVP_EINVAL, "device %d out of range", dev);
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        const int rc = kvp::check_cuda(cudaGetSymbolAddress(&p, g_decode_scratch), "cudaGetSymbolAddress(scratch)");
        if (rc) return rc;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return KVP_OK;
}

}  // namespace

extern "C" int paged_decode_attention_noalloc(kvp_pool *pool, int layer, const kvp_attn_config *attn, int B,
                                              const float *q, const int32_t *block_tables, int max_blocks_per_seq,
                                              const int32_t *ctx_lens, int max_ctx_len, int split_tokens, float *out,
                                              void *stream)
{
    int rc = kvp::check_pool(pool, layer);
    if (rc) return rc;
    if (B == 0) return KVP_OK;
    int Hq, Hkv, G;
    if ((rc = kvp::resolve_attn(pool, attn, &Hq, &Hkv, &G))) return rc;
    const size_t need = paged_decode_workspace_size(pool, attn, B, max_ctx_len, split_tokens);
    if (need == 0) return KVP_EINVAL;  // message already set
    if (need > KVP_NOALLOC_SCRATCH_BYTES)
        return kvp::set_error(KVP_EINVAL,
                              "paged_decode_attention_noalloc: this call needs %zu bytes of workspace, above the "
                              "library's fixed %u bytes (use fewer sequences, a shorter max_ctx_len, a larger "
                              "split_tokens, or paged_decode_attention with your own workspace)",
                              need, (unsigned)KVP_NOALLOC_SCRATCH_BYTES);
    void *ws = nullptr;
    if ((rc = scratch_address(pool->cfg.device, &ws))) return rc;
    // The workspace starts with one int32 split counter per (sequence, kv
    // head), which must be zero when the kernel starts. The array keeps
    // whatever the previous call left, so clear the counters every time.
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    rc = kvp::check_cuda(cudaMemsetAsync(ws, 0, static_cast<size_t>(B) * Hkv * sizeof(int32_t), s),
                         "clear scratch counters");
    if (rc) return rc;
    return paged_decode_attention(pool, layer, attn, B, q, block_tables, max_blocks_per_seq, ctx_lens, max_ctx_len,
                                  split_tokens, out, ws, KVP_NOALLOC_SCRATCH_BYTES, stream);
}
