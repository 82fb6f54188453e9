"""ctypes binding of libkvpaged.so (argument marshalling only).

Every computation happens in the CUDA kernels behind the C ABI declared in
include/kvpaged.h; this module only turns torch tensors into device pointers,
fills the config structs and raises on error codes. There is no fallback: if
the shared library is missing the import fails.
"""

from __future__ import annotations

import ctypes as C
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkvpaged.so")

KVP_OK, KVP_EINVAL, KVP_ERANGE, KVP_EOVERFLOW = 0, -1, -2, -3
KVP_EUNSUPPORTED, KVP_ECUDA, KVP_EDEVICE, KVP_ETIMEOUT = -4, -5, -6, -7
KVP_F16, KVP_BF16 = 1, 2
DTYPE_CODES = {"f16": KVP_F16, "bf16": KVP_BF16}
STATUS_NAMES = {0: "KVP_OK", -1: "KVP_EINVAL", -2: "KVP_ERANGE", -3: "KVP_EOVERFLOW", -4: "KVP_EUNSUPPORTED",
                -5: "KVP_ECUDA", -6: "KVP_EDEVICE", -7: "KVP_ETIMEOUT"}

# every entry point declared in include/kvpaged.h
EXPORTS = (
    "kv_pool_create", "kv_pool_destroy", "kv_pool_layer_ptrs", "kv_pool_sync_status", "kvp_last_error",
    "kvp_rope_table_bytes", "kvp_rope_table_fill", "kv_append", "paged_decode_workspace_size",
    "paged_decode_attention", "paged_decode_attention_noalloc", "paged_prefill_workspace_size", "paged_prefill_attention", "kvp_convert_f32",
    "kvp_convert_bits", "kvp_version",
    "kvp_blocks_create", "kvp_blocks_destroy", "kvp_blocks_count", "kvp_blocks_refs", "kvp_block_hash",
    "kvp_seq_create", "kvp_seq_destroy", "kvp_seq_free", "kvp_seq_allocate_for_tokens", "kvp_seq_append_token",
    "kvp_seq_reserve", "kvp_seq_commit", "kvp_seq_len", "kvp_seq_num_blocks", "kvp_seq_block_table",
    "kvp_seq_block_table_delta",
)


class KvpError(RuntimeError):
    def __init__(self, code: int, msg: str, device_code: int = 0):
        super().__init__(f"{STATUS_NAMES.get(code, code)}: {msg}")
        self.code = code
        self.device_code = device_code


class CacheConfig(C.Structure):
    _fields_ = [("num_layers", C.c_int32), ("num_kv_heads", C.c_int32), ("head_dim", C.c_int32),
                ("block_size", C.c_int32), ("max_seq_len", C.c_int32), ("num_blocks", C.c_int32),
                ("kv_dtype", C.c_int32), ("device", C.c_int32)]


class AttnConfig(C.Structure):
    _fields_ = [("num_heads", C.c_int32), ("num_kv_heads", C.c_int32), ("head_dim", C.c_int32),
                ("rope_theta", C.c_float), ("rms_eps", C.c_float), ("rope_dim", C.c_int32),
                ("rope_style", C.c_int32), ("window", C.c_int32)]


KVP_ROPE_HALF, KVP_ROPE_INTERLEAVED = 0, 1


_lib = None


def lib() -> C.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with paged_kv_cache_321_b200.build.build()")
        L = C.CDLL(LIB_PATH)
        P, i32, i64, u64, sz = C.c_void_p, C.c_int, C.c_int64, C.c_uint64, C.c_size_t
        CP, AP = C.POINTER(CacheConfig), C.POINTER(AttnConfig)
        sig = {
            "kv_pool_create": (i32, [CP, P, P, C.POINTER(P)]),
            "kv_pool_destroy": (i32, [P]),
            "kv_pool_layer_ptrs": (i32, [P, i32, C.POINTER(P), C.POINTER(P)]),
            "kv_pool_sync_status": (i32, [P, P, C.POINTER(i32)]),
            "kvp_last_error": (C.c_char_p, []),
            "kvp_rope_table_bytes": (sz, [AP, i32]),
            "kvp_rope_table_fill": (i32, [AP, i32, P]),
            "kv_append": (i32, [P, i32, AP, i32, P, P, P, P, P, P, i32, P, P, i32, P, i32, P, P]),
            "paged_decode_workspace_size": (sz, [P, AP, i32, i32, i32]),
            "paged_decode_attention": (i32, [P, i32, AP, i32, P, P, i32, P, i32, i32, P, P, sz, P]),
            "paged_decode_attention_noalloc": (i32, [P, i32, AP, i32, P, P, i32, P, i32, i32, P, P]),
            "paged_prefill_workspace_size": (sz, [P, AP, i32, i32, i32]),
            "paged_prefill_attention": (i32, [P, i32, AP, i32, P, P, P, P, i32, i32, i32, P, P, sz, P]),
            "kvp_convert_f32": (i32, [P, P, i64, i32, P]),
            "kvp_convert_bits": (i32, [u64, i64, i32, P, P]),
            "kvp_version": (i32, []),
            "kvp_blocks_create": (i32, [i32, i32, i32, i32, C.POINTER(P)]),
            "kvp_blocks_destroy": (i32, [P]),
            "kvp_blocks_count": (i32, [P, i32, C.POINTER(i32), C.POINTER(i32), C.POINTER(i32)]),
            "kvp_blocks_refs": (i32, [P, i32, i32]),
            "kvp_block_hash": (u64, [P, i32, C.POINTER(u64)]),
            "kvp_seq_create": (i32, [P, C.POINTER(P)]),
            "kvp_seq_destroy": (i32, [P]),
            "kvp_seq_free": (i32, [P]),
            "kvp_seq_allocate_for_tokens": (i32, [P, P, i32, C.POINTER(i32)]),
            "kvp_seq_append_token": (i32, [P, C.c_int32]),
            "kvp_seq_reserve": (i32, [P, i32]),
            "kvp_seq_commit": (i32, [P, i32]),
            "kvp_seq_len": (i32, [P]),
            "kvp_seq_num_blocks": (i32, [P]),
            "kvp_seq_block_table": (i32, [P, i32, P, i32, P]),
            "kvp_seq_block_table_delta": (i32, [P, i32, P, i32, P, P]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype, fn.argtypes = res, args
        _lib = L
    return _lib


def _check(rc: int):
    if rc != KVP_OK:
        raise KvpError(rc, lib().kvp_last_error().decode(errors="replace"))


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return C.c_void_p(t.data_ptr())


def _stream(stream) -> C.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return C.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def attn_config(num_heads: int, num_kv_heads: int, head_dim: int, rope_theta: float = 0.0,
                rms_eps: float = 1e-6, rope_dim: int = 0, rope_style: int = KVP_ROPE_HALF,
                window: int = 0) -> AttnConfig:
    """rope_dim: rotated leading dims (0: all); rope_style: KVP_ROPE_HALF or
    KVP_ROPE_INTERLEAVED; window > 0: sliding window, block-table rows are
    rings of their length."""
    return AttnConfig(num_heads, num_kv_heads, head_dim, rope_theta, rms_eps, rope_dim, rope_style, window)


class Pool:
    """A per-layer block pool: K and V tensors [num_layers, num_blocks, Hkv,
    block_size, D] of 16-bit words, owned by torch, wrapped by a C handle."""

    def __init__(self, num_layers: int, num_kv_heads: int, head_dim: int, block_size: int, max_seq_len: int,
                 num_blocks: int, kv_dtype: str, device: Optional[torch.device] = None,
                 k: Optional[torch.Tensor] = None, v: Optional[torch.Tensor] = None):
        device = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
        shape = (num_layers, num_blocks, num_kv_heads, block_size, head_dim)
        self.k = torch.empty(shape, dtype=torch.int16, device=device) if k is None else k
        self.v = torch.empty(shape, dtype=torch.int16, device=device) if v is None else v
        if tuple(self.k.shape) != shape or tuple(self.v.shape) != shape:
            raise ValueError(f"pool tensors must have shape {shape}")
        self.cfg = CacheConfig(num_layers, num_kv_heads, head_dim, block_size, max_seq_len, num_blocks,
                               DTYPE_CODES[kv_dtype], device.index if device.index is not None else 0)
        self.kv_dtype = kv_dtype
        h = C.c_void_p()
        _check(lib().kv_pool_create(C.byref(self.cfg), _ptr(self.k), _ptr(self.v), C.byref(h)))
        self.handle = h

    def close(self):
        if getattr(self, "handle", None):
            lib().kv_pool_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def layer_ptrs(self, layer: int):
        k, v = C.c_void_p(), C.c_void_p()
        _check(lib().kv_pool_layer_ptrs(self.handle, layer, C.byref(k), C.byref(v)))
        return k.value, v.value

    def sync_status(self, stream=None) -> int:
        """Synchronises the stream; raises KvpError if a kernel stored a device
        error since the last call."""
        code = C.c_int(0)
        rc = lib().kv_pool_sync_status(self.handle, _stream(stream), C.byref(code))
        if rc != KVP_OK:
            raise KvpError(rc, lib().kvp_last_error().decode(errors="replace"), code.value)
        return 0


def rope_table_bytes(attn: AttnConfig, max_pos: int) -> int:
    return lib().kvp_rope_table_bytes(C.byref(attn), max_pos)


def rope_table_fill(attn: AttnConfig, max_pos: int, table: torch.Tensor):
    if table.numel() * table.element_size() < rope_table_bytes(attn, max_pos):
        raise ValueError("rope table buffer too small")
    _check(lib().kvp_rope_table_fill(C.byref(attn), max_pos, _ptr(table)))


def kv_append(pool: Pool, layer: int, attn: AttnConfig, q, k, v, tok_req, positions, block_tables, q_out,
              q_norm_w=None, k_norm_w=None, rope_table=None, rope_max_pos: int = 0, stream=None):
    T = tok_req.numel()
    _check(lib().kv_append(pool.handle, layer, C.byref(attn), T, _ptr(q), _ptr(k), _ptr(v), _ptr(q_norm_w),
                           _ptr(k_norm_w), _ptr(rope_table), rope_max_pos, _ptr(tok_req), _ptr(positions),
                           block_tables.shape[0], _ptr(block_tables), block_tables.shape[1], _ptr(q_out),
                           _stream(stream)))


def decode_workspace_size(pool: Pool, attn: AttnConfig, B: int, max_ctx_len: int, split_tokens: int = 0) -> int:
    n = lib().paged_decode_workspace_size(pool.handle, C.byref(attn), B, max_ctx_len, split_tokens)
    if n == 0 and B > 0:
        raise KvpError(KVP_EINVAL, lib().kvp_last_error().decode(errors="replace"))
    return n


def paged_decode_attention(pool: Pool, layer: int, attn: AttnConfig, q, block_tables, ctx_lens, max_ctx_len: int,
                           out, workspace, split_tokens: int = 0, stream=None):
    B = ctx_lens.numel()
    _check(lib().paged_decode_attention(pool.handle, layer, C.byref(attn), B, _ptr(q), _ptr(block_tables),
                                        block_tables.shape[1], _ptr(ctx_lens), max_ctx_len, split_tokens, _ptr(out),
                                        _ptr(workspace), workspace.numel() * workspace.element_size(),
                                        _stream(stream)))


NOALLOC_SCRATCH_BYTES = 16 * 1024 * 1024  # KVP_NOALLOC_SCRATCH_BYTES


def paged_decode_attention_noalloc(pool: Pool, layer: int, attn: AttnConfig, q, block_tables, ctx_lens,
                                   max_ctx_len: int, out, split_tokens: int = 0, stream=None):
    """paged_decode_attention using the library's fixed device workspace, for
    callers that cannot allocate device memory (see include/kvpaged.h)."""
    B = ctx_lens.numel()
    _check(lib().paged_decode_attention_noalloc(pool.handle, layer, C.byref(attn), B, _ptr(q), _ptr(block_tables),
                                                block_tables.shape[1], _ptr(ctx_lens), max_ctx_len, split_tokens,
                                                _ptr(out), _stream(stream)))


def prefill_workspace_size(pool: Pool, attn: AttnConfig, S: int, total_q: int, max_q_len: int) -> int:
    return lib().paged_prefill_workspace_size(pool.handle, C.byref(attn), S, total_q, max_q_len)


def paged_prefill_attention(pool: Pool, layer: int, attn: AttnConfig, q, cu_q, ctx_lens, block_tables,
                            max_q_len: int, out, workspace=None, stream=None):
    S = ctx_lens.numel()
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().paged_prefill_attention(pool.handle, layer, C.byref(attn), S, _ptr(q), _ptr(cu_q),
                                         _ptr(ctx_lens), _ptr(block_tables), block_tables.shape[1], q.shape[0],
                                         max_q_len, _ptr(out), _ptr(workspace), ws_bytes, _stream(stream)))


def convert_f32(x: torch.Tensor, out: torch.Tensor, kv_dtype: str, stream=None):
    _check(lib().kvp_convert_f32(_ptr(x), _ptr(out), x.numel(), DTYPE_CODES[kv_dtype], _stream(stream)))


def convert_bits(start: int, count: int, kv_dtype: str, out: torch.Tensor, stream=None):
    _check(lib().kvp_convert_bits(start, count, DTYPE_CODES[kv_dtype], _ptr(out), _stream(stream)))


# ------------------------------------------------------- host block manager
class Blocks:
    """Per-layer block allocator with a prefix cache (host only; see
    include/kvpaged.h). Block ids index a Pool of the same num_blocks."""

    def __init__(self, num_layers: int, num_blocks: int, block_size: int, max_seq_len: int = 0):
        self.num_layers, self.num_blocks, self.block_size = num_layers, num_blocks, block_size
        h = C.c_void_p()
        _check(lib().kvp_blocks_create(num_layers, num_blocks, block_size, max_seq_len, C.byref(h)))
        self.handle = h

    def counts(self, layer: int = 0):
        """(free, cached and unheld, held) blocks of a layer."""
        f, c, h = C.c_int(), C.c_int(), C.c_int()
        _check(lib().kvp_blocks_count(self.handle, layer, C.byref(f), C.byref(c), C.byref(h)))
        return f.value, c.value, h.value

    def refs(self, layer: int, block: int) -> int:
        rc = lib().kvp_blocks_refs(self.handle, layer, block)
        if rc < 0:
            _check(rc)
        return rc

    def sequence(self) -> "Sequence":
        return Sequence(self)

    def close(self):
        if self.handle:
            lib().kvp_blocks_destroy(self.handle)
            self.handle = None


def block_hash(tokens, parent: Optional[int] = None) -> int:
    arr = (C.c_int32 * len(tokens))(*[int(t) for t in tokens])
    par = C.c_uint64(parent) if parent is not None else None
    return lib().kvp_block_hash(arr, len(tokens), C.byref(par) if par is not None else None)


class Sequence:
    """One request's blocks in every layer (PagedKVCache's per-request state)."""

    def __init__(self, blocks: Blocks):
        self.blocks = blocks
        h = C.c_void_p()
        _check(lib().kvp_seq_create(blocks.handle, C.byref(h)))
        self.handle = h

    def allocate_for_tokens(self, tokens) -> int:
        arr = (C.c_int32 * len(tokens))(*[int(t) for t in tokens])
        computed = C.c_int()
        _check(lib().kvp_seq_allocate_for_tokens(self.handle, arr, len(tokens), C.byref(computed)))
        return computed.value

    def append_token(self, token: int):
        _check(lib().kvp_seq_append_token(self.handle, int(token)))

    def reserve(self, num_tokens: int):
        _check(lib().kvp_seq_reserve(self.handle, num_tokens))

    def commit(self, new_tokens: int):
        _check(lib().kvp_seq_commit(self.handle, new_tokens))

    def free(self):
        _check(lib().kvp_seq_free(self.handle))

    def __len__(self) -> int:
        return lib().kvp_seq_len(self.handle)

    def num_blocks(self) -> int:
        return lib().kvp_seq_num_blocks(self.handle)

    def block_table(self, layer: int = 0, max_blocks: Optional[int] = None):
        """(block ids, owned flags) of one layer; ids padded with -1 to max_blocks."""
        n = self.num_blocks() if max_blocks is None else max_blocks
        ids = (C.c_int32 * max(n, 1))()
        owned = (C.c_uint8 * max(n, 1))()
        rc = lib().kvp_seq_block_table(self.handle, layer, ids, n, owned)
        if rc < 0:
            _check(rc)
        return list(ids)[:n], [bool(x) for x in list(owned)[:n]]

    def block_table_delta(self, layer: int, row) -> tuple:
        """Updates `row` (a host int32 numpy array, the same one every call)
        with the entries that changed since the last call for this layer and
        returns their range (first, end); first == end: nothing changed."""
        import numpy as np

        assert isinstance(row, np.ndarray) and row.dtype == np.int32 and row.flags.c_contiguous
        first, end = C.c_int(), C.c_int()
        _check(lib().kvp_seq_block_table_delta(self.handle, layer, row.ctypes.data_as(C.c_void_p), row.size,
                                               C.byref(first), C.byref(end)))
        return first.value, end.value

    def sync_block_table(self, layer: int, row, device_row: torch.Tensor, stream=None) -> tuple:
        """Keeps a device-resident row equal to the layer's block table,
        uploading only the entries that changed (growth: the new ones; a
        replaced prompt: the whole row). `row` is this row's host copy.
        Returns the uploaded range."""
        first, end = self.block_table_delta(layer, row)
        if end > first:
            src = torch.from_numpy(row[first:end])
            if stream is not None:
                with torch.cuda.stream(stream):
                    device_row[first:end].copy_(src, non_blocking=False)
            else:
                device_row[first:end].copy_(src)
        return first, end

    def close(self):
        if self.handle:
            lib().kvp_seq_destroy(self.handle)
            self.handle = None
