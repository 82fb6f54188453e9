"""B200-native paged KV cache: kv_append and paged attention over a
block-pooled cache, as hand-written sm_100a kernels behind a C ABI
(include/kvpaged.h, libkvpaged.so). This package is the thin Python binding;
PyTorch provides device memory and streams only."""

from ._native import (  # noqa: F401
    EXPORTS,
    KVP_BF16,
    KVP_EDEVICE,
    KVP_EINVAL,
    KVP_EOVERFLOW,
    KVP_ERANGE,
    KVP_ETIMEOUT,
    KVP_EUNSUPPORTED,
    KVP_F16,
    KVP_OK,
    KVP_ROPE_HALF,
    KVP_ROPE_INTERLEAVED,
    AttnConfig,
    Blocks,
    CacheConfig,
    KvpError,
    Pool,
    Sequence,
    attn_config,
    block_hash,
    convert_bits,
    convert_f32,
    decode_workspace_size,
    kv_append,
    lib,
    paged_decode_attention,
    paged_decode_attention_noalloc,
    NOALLOC_SCRATCH_BYTES,
    paged_prefill_attention,
    prefill_workspace_size,
    rope_table_bytes,
    rope_table_fill,
)
