"""The C-ABI library loads without a GPU and exports every function that
include/kvpaged.h declares (no compute calls: those need a GPU)."""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    text = open(os.path.join(ROOT, "include", "kvpaged.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\**\s*([a-z_][a-z0-9_]*)\s*\(", text, flags=re.M)
    return sorted(set(n for n in names if n not in ("if", "while")))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("kv_pool_create", "kv_append", "paged_decode_attention", "paged_prefill_attention"):
        assert required in names
    assert len(names) >= 15


def test_library_exports_every_declared_symbol():
    from paged_kv_cache_321_b200 import build

    lib_path = build.build()
    lib = ctypes.CDLL(lib_path)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing
    lib.kvp_version.restype = ctypes.c_int
    assert lib.kvp_version() >= 100


def test_binding_lists_every_export():
    import paged_kv_cache_321_b200 as K

    assert sorted(K.EXPORTS) == declared_functions()


def test_host_side_errors_need_no_gpu():
    # argument validation happens before any CUDA call
    import paged_kv_cache_321_b200 as K

    lib = K.lib()
    out = ctypes.c_void_p()
    rc = lib.kv_pool_create(None, None, None, ctypes.byref(out))
    assert rc == K.KVP_EINVAL
    assert b"NULL" in lib.kvp_last_error()
    assert lib.kv_pool_destroy(None) == K.KVP_OK
    cfg = K.AttnConfig(32, 8, 128, 5e5, 1e-6)
    assert lib.kvp_rope_table_bytes(ctypes.byref(cfg), 100) == 100 * 128 * 4
    assert lib.kvp_rope_table_fill(ctypes.byref(K.AttnConfig(32, 8, 127, 5e5, 1e-6)), 10, None) != 0


def test_rope_table_size_follows_the_rotary_width():
    # the table holds rope_dim/2 (cos, sin) pairs per position; invalid
    # widths (odd, wider than the head) size to 0
    import paged_kv_cache_321_b200 as K

    lib = K.lib()
    size = lambda **kw: lib.kvp_rope_table_bytes(ctypes.byref(K.attn_config(32, 8, 128, 1e4, 1e-6, **kw)), 100)
    assert size() == 100 * 128 * 4
    assert size(rope_dim=32) == 100 * 32 * 4
    assert size(rope_dim=64, rope_style=K.KVP_ROPE_INTERLEAVED) == 100 * 64 * 4
    assert size(rope_dim=33) == 0 and size(rope_dim=130) == 0
    assert lib.kvp_rope_table_fill(ctypes.byref(K.attn_config(32, 8, 128, 1e4, 1e-6, rope_dim=31)), 10, None) != 0


def test_attn_config_layout_matches_the_header():
    # eight 4-byte fields in the header's order; zero-filled extras mean
    # full rotate-half RoPE and no window
    import paged_kv_cache_321_b200 as K

    c = K.attn_config(32, 8, 128, 5e5, 1e-6)
    assert ctypes.sizeof(c) == 32
    assert (c.rope_dim, c.rope_style, c.window) == (0, K.KVP_ROPE_HALF, 0)
    assert [f[0] for f in K.AttnConfig._fields_] == ["num_heads", "num_kv_heads", "head_dim", "rope_theta",
                                                      "rms_eps", "rope_dim", "rope_style", "window"]


@pytest.mark.parametrize("field,value,code", [
    ("num_layers", 0, "KVP_EINVAL"), ("num_blocks", -1, "KVP_EINVAL"), ("max_seq_len", 0, "KVP_EINVAL"),
    ("head_dim", 96, "KVP_EUNSUPPORTED"), ("block_size", 24, "KVP_EUNSUPPORTED"),
    ("block_size", 512, "KVP_EUNSUPPORTED"), ("kv_dtype", 3, "KVP_EINVAL"),
])
def test_pool_config_checked_before_any_device_call(field, value, code):
    # PagedCacheConfig's shape rules are host checks: refused with no GPU
    import paged_kv_cache_321_b200 as K

    lib = K.lib()
    cfg = K.CacheConfig(1, 8, 128, 16, 4096, 64, K.KVP_F16, 0)
    setattr(cfg, field, value)
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: the check comes first
    out = ctypes.c_void_p()
    assert lib.kv_pool_create(ctypes.byref(cfg), fake, fake, ctypes.byref(out)) == getattr(K, code)
    assert not out.value
