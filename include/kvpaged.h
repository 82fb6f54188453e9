/*
 * kvpaged.h -- C ABI of libkvpaged.so, the B200 (sm_100a) paged KV cache.
 *
 * The library implements the per-layer hot path of a block-pooled KV cache:
 *
 *   kv_append               new tokens' q/k/v -> optional per-head RMSNorm ->
 *                           RoPE -> fp32->fp16/bf16 (nearest, ties to even) ->
 *                           scatter into the block slot of each token
 *   paged_decode_attention  one query token per sequence, GQA attention over
 *                           the sequence's blocks, online softmax in fp32,
 *                           split-K over the context with an fp32
 *                           log-sum-exp combine
 *   paged_prefill_attention several query tokens per sequence (chunked
 *                           prefill), causal over the paged cache, QK^T and PV
 *                           on the tcgen05 tensor cores
 *
 * Page citations name the page title and the function on it:
 *   makarna/pkg/kvcache/paged_cache.go        (PagedKVCache, Append, ...)
 *   makarna/pkg/model/arch/hybrid_decoder.go  (runHybridAttentionBlock, ...)
 *   soft3/glia/run/arch/decoder/forward.rs    (forward_layer)
 *
 * Conventions shared by every entry point:
 *   - Every pointer argument except the config structs and handles is a
 *     DEVICE pointer on the pool's device; the caller owns all memory (the
 *     library allocates only the pool handle and its 8-byte status word).
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream) unless stated otherwise. Kernels are launched with a
 *     programmatic dependency on the stream's previous kernel: a grid may be
 *     placed on the SMs while that kernel runs, but it touches no global
 *     memory before that kernel has completed, so stream order holds exactly
 *     as for plain launches.
 *   - Errors that the host can see (bad shapes, unsupported sizes, NULL
 *     pointers) are returned before anything is launched, with a message
 *     available from kvp_last_error().
 *   - Errors that only the device can see (a block id outside the pool, a
 *     position past MaxSeqLen, a context longer than the block table) never
 *     trap: the affected work is skipped, the first such error code is stored
 *     in the pool's status word, and kv_pool_sync_status() reports it.
 *   - Pool layout, per layer: K and V each [num_blocks][Hkv][block_size][D]
 *     16-bit words (head-major inside a block, the packed layout of
 *     writePackedBlockU32 in makarna/pkg/kvcache/paged_cache.go); layer l
 *     starts l * num_blocks*Hkv*block_size*D words after the base.
 */
#ifndef KVPAGED_H
#define KVPAGED_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes. The device-side codes mirror the Go errors of
 * makarna/pkg/kvcache/paged_cache.go: "KV cache overflow" (Append, AppendKV)
 * is KVP_EOVERFLOW, "block index out of range" (AppendKV) is KVP_ERANGE. */
enum {
    KVP_OK = 0,
    KVP_EINVAL = -1,        /* bad argument, NULL pointer, unknown sequence */
    KVP_ERANGE = -2,        /* block id / block index / context out of range */
    KVP_EOVERFLOW = -3,     /* position past max_seq_len or the rope table */
    KVP_EUNSUPPORTED = -4,  /* head_dim, group size or block size not built */
    KVP_ECUDA = -5,         /* a CUDA runtime call failed */
    KVP_EDEVICE = -6,       /* kv_pool_sync_status: the device stored an error */
    KVP_ETIMEOUT = -7       /* a bounded wait inside a kernel ran out */
};

/* KV element types of the pool. */
enum { KVP_F16 = 1, KVP_BF16 = 2 };

/* Pool shape: the fields of PagedCacheConfig (NumLayers, NumKVHeads,
 * HeadDim, BlockSize, MaxSeqLen, GPU) in makarna/pkg/kvcache/paged_cache.go,
 * plus the pool's block count and element type.
 *   head_dim   64, 128 or 256
 *   block_size a power of two from 1 to 256
 *   max_seq_len positions accepted by kv_append are [0, max_seq_len) */
typedef struct {
    int32_t num_layers;
    int32_t num_kv_heads;
    int32_t head_dim;
    int32_t block_size;
    int32_t max_seq_len;
    int32_t num_blocks;   /* blocks per layer */
    int32_t kv_dtype;     /* KVP_F16 or KVP_BF16 */
    int32_t device;       /* CUDA ordinal holding k_base / v_base */
} kvp_cache_config;

/* Attention shape: the subset of HybridDecoderConfig (NumHeads, NumKVHeads,
 * HeadDim, RopeTheta) of makarna/pkg/model/arch/hybrid_decoder.go plus the
 * q/k RMSNorm epsilon. num_kv_heads == 0 means num_heads
 * (normalizeHybridDecoderConfig). num_heads / num_kv_heads (the GQA group)
 * must be 1, 2, 4 or 8 for the decode path.
 *
 * The last three fields are those of a per-layer RoPE and cache (the
 * layer_rope_dim / layer_kv_cache_seq of forward_layer in
 * soft3/glia/run/arch/decoder/forward.rs); zero-filled they give full
 * rotate-half RoPE and unlimited attention:
 *   rope_dim   rotated leading dims: 0 = head_dim, else even and <= head_dim;
 *              the rest of the row passes through unrotated
 *   rope_style KVP_ROPE_HALF: pairs (i, i + rope_dim/2);
 *              KVP_ROPE_INTERLEAVED: pairs (2i, 2i + 1)
 *   window     0, or a sliding window: the query at position p sees keys
 *              max(0, p - window + 1) .. p only, and every block-table row is
 *              a RING of max_blocks_per_seq entries -- position p lives in
 *              entry (p / block_size) mod max_blocks_per_seq, slot
 *              p % block_size (the paged form of a sliding layer's
 *              window-sized ring cache, kv_slot = past_seq_len % cache_seq).
 *              Calls refuse max_blocks_per_seq * block_size < window with
 *              KVP_EINVAL. A position's slot is reused once the position has
 *              left every window, so positions past
 *              max_blocks_per_seq * block_size are accepted (up to
 *              max_seq_len). */
enum { KVP_ROPE_HALF = 0, KVP_ROPE_INTERLEAVED = 1 };
typedef struct {
    int32_t num_heads;
    int32_t num_kv_heads;
    int32_t head_dim;
    float rope_theta;
    float rms_eps;
    int32_t rope_dim;
    int32_t rope_style;
    int32_t window;
} kvp_attn_config;

typedef struct kvp_pool kvp_pool; /* opaque host handle */

/* ---------------------------------------------------------------- pool */

/* Wraps caller-owned device memory as a pool. k_base / v_base hold
 * num_layers * num_blocks * Hkv * block_size * head_dim 16-bit words each,
 * 256-byte aligned, and must outlive the handle. Allocates the handle and an
 * 8-byte device status word (zeroed). Returns KVP_OK and *out, or an error. */
int kv_pool_create(const kvp_cache_config *cfg, void *k_base, void *v_base, kvp_pool **out);

/* Frees the handle and its status word (not the pool memory). NULL is a no-op. */
int kv_pool_destroy(kvp_pool *pool);

/* Device addresses of layer `layer`'s K and V pools. */
int kv_pool_layer_ptrs(const kvp_pool *pool, int layer, void **k, void **v);

/* Synchronises `stream`, then reads and clears the pool's device status
 * word. Returns KVP_OK, or KVP_EDEVICE when a kernel stored an error (the
 * stored code -- KVP_ERANGE, KVP_EOVERFLOW, KVP_EINVAL or KVP_ETIMEOUT -- is
 * written to *device_code when that pointer is not NULL, and named in
 * kvp_last_error()). */
int kv_pool_sync_status(kvp_pool *pool, void *stream, int *device_code);

/* Thread-local message describing the last error returned on this thread. */
const char *kvp_last_error(void);

/* ---------------------------------------------------------------- rope */

/* Size in bytes of a RoPE table covering positions [0, max_pos). */
size_t kvp_rope_table_bytes(const kvp_attn_config *attn, int max_pos);

/* Fills a caller-owned DEVICE table [max_pos][R/2] of (cos, sin) float
 * pairs, R = the config's rotary width (rope_dim, or head_dim when 0): pair i
 * at position p rotates by the angle p * theta^(-2i/R), evaluated in fp64 and
 * rounded to fp32. The pages leave HybridRoPE's formula unstated; by default
 * this is the rotate-half convention of the Llama-3 / Qwen3 shapes they
 * serve (rope_style picks the dims a pair turns). Computed once at set-up
 * time on the host and copied with a blocking cudaMemcpy: call it outside
 * any stream capture. theta must be > 0, head_dim even and <= 256 (the
 * fused-RoPE limits of runHybridAttentionBlock). */
int kvp_rope_table_fill(const kvp_attn_config *attn, int max_pos, float *table);

/* ------------------------------------------------------------ kv_append */

/* Appends T new tokens of layer `layer` (Append / AppendKV in
 * makarna/pkg/kvcache/paged_cache.go, preceded by the QNorm/KNorm and RoPE
 * steps of runHybridAttentionBlock in makarna/pkg/model/arch/hybrid_decoder.go).
 *
 * For token t of sequence r = tok_req[t] at position p = positions[t]:
 *   q' = rope(norm(q[t], q_norm_w)),  k' = rope(norm(k[t], k_norm_w)),  v' = v[t]
 *   the K/V slot is (block_tables[r][p / block_size], p % block_size), or
 *   with a window entry (p / block_size) mod max_blocks_per_seq (the ring);
 *   K and V receive cvt(k'), cvt(v') with cvt = nearest 16-bit value, ties to
 *   even (float32ToFloat16Bits / float32ToBFloat16Bits; a NaN becomes a quiet
 *   NaN keeping its top payload bits); q_out[t] = q'.
 * norm(x, w) = (x * (1 / sqrt(sum_d x_d^2 * (1/D) + eps))) * w with the sum
 * taken in order d = 0..D-1 in fp32 (the per-head RMS form of forward_layer in
 * soft3/glia/run/arch/decoder/forward.rs); skipped when the weight is NULL.
 * rope uses the table of kvp_rope_table_fill (built for the same rope_dim)
 * on the first rope_dim dims, paired as rope_style says; skipped when
 * rope_table is NULL.
 * Every float step is one IEEE operation, so results are reproducible bit for
 * bit.
 *
 *   q          [T][Hq][D] float32      k, v  [T][Hkv][D] float32
 *   q_norm_w, k_norm_w  [D] float32 or NULL (one weight shared by all heads)
 *   rope_table [rope_max_pos][D/2][2] float32 or NULL
 *   tok_req, positions  [T] int32;  block_tables [num_seqs][max_blocks_per_seq]
 *   q_out      [T][Hq][D] float32 (written for every accepted token)
 * Device errors: tok_req outside [0, num_seqs) -> KVP_EINVAL; position outside
 * [0, max_seq_len) or past the rope table -> KVP_EOVERFLOW (q_out row zeroed);
 * p / block_size >= max_blocks_per_seq (without a window) or a block id
 * outside [0, num_blocks) -> KVP_ERANGE (q_out still written, no store). Two
 * tokens aimed at the same slot in one call race (with a ring: two positions
 * of one sequence max_blocks_per_seq * block_size apart). T == 0 is a no-op. */
int kv_append(kvp_pool *pool, int layer, const kvp_attn_config *attn, int T, const float *q, const float *k,
              const float *v, const float *q_norm_w, const float *k_norm_w, const float *rope_table,
              int rope_max_pos, const int32_t *tok_req, const int32_t *positions, int num_seqs,
              const int32_t *block_tables, int max_blocks_per_seq, float *q_out, void *stream);

/* ------------------------------------------------------- decode attention */

/* Workspace bytes paged_decode_attention needs for B sequences of at most
 * max_ctx_len keys with the given split size (0 = automatic, as the call
 * itself chooses). Returns 0 on a bad argument. */
size_t paged_decode_workspace_size(const kvp_pool *pool, const kvp_attn_config *attn, int B, int max_ctx_len,
                                   int split_tokens);

/* One query token per sequence (the batch kernel of
 * runHybridAttentionBlockBatch in makarna/pkg/model/arch/hybrid_decoder.go;
 * the attention of forward_layer in soft3/glia/run/arch/decoder/forward.rs).
 * Query head g of sequence r reads KV head g / (Hq/Hkv) and the keys
 * 0 .. ctx_lens[r]-1 (with a window, the last `window` of them, through the
 * ring), i.e. ctx_lens[r] counts the keys INCLUDING the token kv_append just
 * wrote:
 *   out[r][g] = sum_j softmax_j(q[r][g] . K_j * scale) V_j,
 *   scale = float32(1/sqrt(float64(D))),
 * accumulated in fp32 with an online softmax over 16-key tiles. The tiles of
 * all (sequence, kv head) contexts are divided evenly among the GPU's warps;
 * a context shared by several warps is combined from their (max, sum,
 * unnormalised output) partials by log-sum-exp in fp32 (by the last of them
 * to finish, or by a second small grid). With 4 or 8 query heads per kv head
 * and block_size >= 16 the tile products run on tensor cores with 16-bit
 * inputs: K and V exactly, q and the softmax weights each as a 16-bit high
 * part plus the 16-bit rounding of the remainder (about 16 more bits). split_tokens is the fewest keys one warp takes (0 = automatic;
 * otherwise a multiple of 16): a large value keeps each context on one warp.
 *
 *   q, out        [B][Hq][D] float32
 *   block_tables  [B][max_blocks_per_seq] int32 (entries past the context are
 *                 never read)
 *   ctx_lens      [B] int32 in [0, max_ctx_len]; 0 gives an all-zero row
 *   B             at most 2048
 *   workspace     >= paged_decode_workspace_size(...) bytes, 256-byte
 *                 aligned, ZERO-FILLED before its first use; every call leaves
 *                 its counters at zero again. Calls sharing a workspace must
 *                 not overlap on the device.
 * Device errors: ctx_lens[r] above max_ctx_len, max_seq_len or (without a
 * window) max_blocks_per_seq*block_size -> KVP_ERANGE and a zero row; a block
 * id outside the pool -> KVP_ERANGE and that block is left out. */
int paged_decode_attention(kvp_pool *pool, int layer, const kvp_attn_config *attn, int B, const float *q,
                           const int32_t *block_tables, int max_blocks_per_seq, const int32_t *ctx_lens,
                           int max_ctx_len, int split_tokens, float *out, void *workspace, size_t ws_bytes,
                           void *stream);

/* Size of the fixed workspace of paged_decode_attention_noalloc: 16 MiB. */
#define KVP_NOALLOC_SCRATCH_BYTES (16u * 1024u * 1024u)

/* paged_decode_attention for callers that cannot allocate device memory.
 * The pages have no counterpart of this entry point. It serves callers that
 * cannot call cudaMalloc: a host program that reserved all of the GPU's memory
 * for its own allocator at start-up, or a latency-critical serving loop that
 * cannot afford cudaMalloc's device-wide synchronisation. Instead of a
 * caller-provided workspace it uses a fixed array of
 * KVP_NOALLOC_SCRATCH_BYTES inside the library's device memory, reserved on
 * every GPU that loads the library and held until the process exits. It
 * allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 *   - Arguments, results and device errors are those of
 *     paged_decode_attention without workspace / ws_bytes.
 *   - A call whose workspace (paged_decode_workspace_size with the same B,
 *     max_ctx_len and split_tokens) exceeds KVP_NOALLOC_SCRATCH_BYTES is
 *     refused with KVP_EINVAL and a message naming the sizes.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture.
 *   - All calls on a device share the one array, which keeps the previous
 *     call's contents; each call clears the split counters on `stream` before
 *     its launch. Calls that overlap on the GPU (another stream, another
 *     thread) race on the array and must be serialised by the caller. */
int paged_decode_attention_noalloc(kvp_pool *pool, int layer, const kvp_attn_config *attn, int B, const float *q,
                                   const int32_t *block_tables, int max_blocks_per_seq, const int32_t *ctx_lens,
                                   int max_ctx_len, int split_tokens, float *out, void *stream);

/* ------------------------------------------------------ prefill attention */

/* Workspace bytes paged_prefill_attention needs (0 on a bad argument). */
size_t paged_prefill_workspace_size(const kvp_pool *pool, const kvp_attn_config *attn, int S, int total_q,
                                    int max_q_len);

/* Chunked prefill over the paged cache (the single-request kernel of
 * runHybridAttentionBlock for seqLen > 1, with kvLen = startPos + seqLen).
 * Sequence s has q_len_s = cu_q[s+1] - cu_q[s] >= 1 new queries whose K/V
 * kv_append already wrote; its query i sits at position
 * ctx_lens[s] - q_len_s + i and sees keys 0 .. that position (causal), or
 * with a window the last `window` of them. With a window the chunk must not
 * have overwritten, in its ring, a key one of its own queries needs: a
 * sequence whose smallest needed key max(0, ctx - q_len - window + 1) is at
 * or below ctx - 1 - max_blocks_per_seq * block_size is refused (append such a
 * chunk in pieces of at most max_blocks_per_seq * block_size - window + 1
 * tokens, attending after each).
 *   q, out   [total_q][Hq][D] float32 (rows cu_q[s] .. cu_q[s+1]-1 belong to s)
 *   cu_q     [S+1] int32, cu_q[0] = 0, cu_q[S] = total_q; max_q_len bounds q_len_s
 *   ctx_lens [S] int32; block_tables [S][max_blocks_per_seq]
 * QK^T and PV run on the tensor cores with 16-bit operands of the pool's type
 * (q and the softmax weights rounded to it; K and V exact) and fp32
 * accumulation; the softmax is fp32. With an fp16 pool the outputs agree with
 * exact attention within 1e-3 + 1e-3*|x|; with a bf16 pool (8 significant
 * bits) within about 1e-2 + 1e-2*|x|.
 * Device errors as paged_decode_attention, plus KVP_ERANGE for a refused
 * sequence (its rows are left unwritten). */
int paged_prefill_attention(kvp_pool *pool, int layer, const kvp_attn_config *attn, int S, const float *q,
                            const int32_t *cu_q, const int32_t *ctx_lens, const int32_t *block_tables,
                            int max_blocks_per_seq, int total_q, int max_q_len, float *out, void *workspace,
                            size_t ws_bytes, void *stream);

/* ---------------------------------------------------------- conversions */

/* The 16-bit conversion kv_append applies (float32ToFloat16Bits /
 * float32ToBFloat16Bits of makarna/pkg/kvcache/paged_cache.go, NaN quieted),
 * exposed for verification: out[i] = cvt(x[i]) for n floats. */
int kvp_convert_f32(const float *x, uint16_t *out, int64_t n, int kv_dtype, void *stream);

/* Same conversion applied to the float32 BIT PATTERNS start .. start+count-1
 * (no input buffer), so all 2^32 patterns can be checked. */
int kvp_convert_bits(uint64_t start, int64_t count, int kv_dtype, uint16_t *out, void *stream);

/* Library version: major * 10000 + minor * 100 + patch. */
int kvp_version(void);

/* -------------------------------------------- host block manager (prefix cache)
 *
 * Host-only bookkeeping that turns requests' token streams into block ids:
 * per-layer block allocation with rollback and prefix caching, after
 * PagedKVCache (ensureCapacityLocked, AppendToken, AllocateForTokens, Commit,
 * Free, LayerBlockIDs) in makarna/pkg/kvcache/paged_cache.go. The page does
 * not show the BlockPool it calls; the reading taken:
 *   - a block is free, held (one reference per sequence holding it: its owner
 *     and every borrower), or cached and unheld (findable by its hash until
 *     evicted);
 *   - allocation takes free blocks first, then evicts the least recently
 *     released cached blocks; it takes all it needs or nothing;
 *   - a block whose last reference goes is cached if it has a hash, else freed;
 *   - a full block's hash is 64-bit FNV-1a over (a parent flag, the parent
 *     block's hash, the block's token ids as little-endian int32); a prompt's
 *     cached prefix is the longest run of its chained hashes present in every
 *     layer, and its blocks are borrowed (never to be written: kv_append must
 *     not target them);
 *   - Commit publishes the blocks it completes, the first block per hash wins.
 * All calls are host calls (no CUDA); calls on one kvp_blocks are serialised
 * by its mutex. Errors: KVP_EINVAL (bad argument), KVP_ERANGE (not enough
 * free blocks: nothing is taken), KVP_EOVERFLOW (beyond max_seq_len). The
 * block ids index the pool of kv_pool_create (num_blocks must match). */
typedef struct kvp_blocks kvp_blocks;
typedef struct kvp_seq kvp_seq;

/* A manager of num_blocks blocks per layer. max_seq_len = 0: no limit. */
int kvp_blocks_create(int num_layers, int num_blocks, int block_size, int max_seq_len, kvp_blocks **out);
int kvp_blocks_destroy(kvp_blocks *blocks); /* sequences must be destroyed first */

/* Free, cached-unheld and held block counts of one layer (any may be NULL). */
int kvp_blocks_count(kvp_blocks *blocks, int layer, int *free_blocks, int *cached_blocks, int *held_blocks);

/* References held on one block (>= 0), or an error code. */
int kvp_blocks_refs(kvp_blocks *blocks, int layer, int block);

/* The chained hash of one full block of n token ids (parent NULL for the
 * first block of a sequence). */
uint64_t kvp_block_hash(const int32_t *tokens, int n, const uint64_t *parent);

/* A sequence (request) with no blocks; destroy releases its blocks. */
int kvp_seq_create(kvp_blocks *blocks, kvp_seq **out);
int kvp_seq_destroy(kvp_seq *seq);

/* Releases every block the sequence holds and forgets its tokens (Free). */
int kvp_seq_free(kvp_seq *seq);

/* A prompt of n tokens (AllocateForTokens): releases what the sequence held,
 * borrows the cached prefix, allocates blocks for the rest of the prompt's
 * full blocks in every layer (all or nothing), and sets *computed to the
 * tokens whose K/V are already cached -- never all n: the last prompt token
 * is always computed. */
int kvp_seq_allocate_for_tokens(kvp_seq *seq, const int32_t *tokens, int n, int *computed);

/* One more token (AppendToken): when it completes a block, the block is
 * allocated if needed and hashed. */
int kvp_seq_append_token(kvp_seq *seq, int32_t token);

/* Blocks for num_tokens positions in every layer (ensureCapacityLocked; new
 * blocks are owned; on failure nothing is kept from this call). */
int kvp_seq_reserve(kvp_seq *seq, int num_tokens);

/* new_tokens more tokens are computed (Commit): completed blocks with hashes
 * are published to the prefix cache. */
int kvp_seq_commit(kvp_seq *seq, int new_tokens);

/* Computed tokens, and blocks held per layer. */
int kvp_seq_len(const kvp_seq *seq);
int kvp_seq_num_blocks(const kvp_seq *seq);

/* One layer's block-table row (LayerBlockIDs): out[0..max_blocks) gets the
 * block ids and -1 past them; owned (may be NULL) gets 1 for owned, 0 for
 * borrowed. Returns the number of blocks, or KVP_ERANGE when max_blocks is
 * too small. */
int kvp_seq_block_table(const kvp_seq *seq, int layer, int32_t *out, int max_blocks, uint8_t *owned);

/* The entries of layer `layer`'s block-table row that changed since this
 * sequence's previous call for that layer, for a caller that keeps the row in
 * device memory and uploads only what changed (the rule of
 * LayerDevicePtrTables in makarna/pkg/kvcache/paged_cache.go: a layer's
 * device tables are rebuilt only when its number of blocks grows). Blocks
 * only ever grow at the end of a row, except when they are replaced
 * (kvp_seq_allocate_for_tokens, kvp_seq_free). So:
 *   - first call for the layer, or blocks replaced since the last one: writes
 *     the whole row (entries past the blocks = -1); *first = 0,
 *     *end = max_blocks;
 *   - blocks grew: writes only the new entries; [*first, *end) is their range;
 *   - otherwise: writes nothing; *first = *end = 0.
 * `row` is the caller's host copy of the row (max_blocks int32), the same
 * buffer on every call; entries outside [*first, *end) are left as they are,
 * so after the call the copy equals kvp_seq_block_table's row.
 * Errors: KVP_EINVAL for bad arguments; KVP_ERANGE when the sequence holds
 * more than max_blocks blocks (nothing written, the state unchanged). */
int kvp_seq_block_table_delta(kvp_seq *seq, int layer, int32_t *row, int max_blocks, int *first, int *end);

#ifdef __cplusplus
}
#endif

#endif /* KVPAGED_H */
