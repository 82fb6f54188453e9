// paged_prefill_attention: chunked-prefill attention over the paged cache on
// the tcgen05 tensor cores (see the kernel below).
#include "common.cuh"

using namespace kvp;

extern "C" size_t paged_prefill_workspace_size(const kvp_pool *pool, const kvp_attn_config *attn, int S,
                                               int total_q, int max_q_len)
{
    (void)pool, (void)attn, (void)S, (void)total_q, (void)max_q_len;
    return 0;
}

extern "C" int paged_prefill_attention(kvp_pool *pool, int layer, const kvp_attn_config *attn, int S,
                                       const float *q, const int32_t *cu_q, const int32_t *ctx_lens,
                                       const int32_t *block_tables, int max_blocks_per_seq, int total_q,
                                       int max_q_len, float *out, void *workspace, size_t ws_bytes, void *stream)
{
    (void)pool, (void)layer, (void)attn, (void)S, (void)q, (void)cu_q, (void)ctx_lens, (void)block_tables;
    (void)max_blocks_per_seq, (void)total_q, (void)max_q_len, (void)out, (void)workspace, (void)ws_bytes;
    (void)stream;
    return set_error(KVP_EUNSUPPORTED, "paged_prefill_attention is not built yet");
}
