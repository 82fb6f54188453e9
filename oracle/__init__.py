"""CPU oracle for the paged KV cache hot path -- TEST INFRASTRUCTURE ONLY.

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. The product (the CUDA library and its
Python binding) never imports, links or calls it, and shares no code with it.

The arithmetic lives in ``oracle.c`` (plain C, fp64 accumulation for
attention, IEEE single operations in written order for norm and rotation);
this module compiles it with gcc and marshals numpy arrays into it.
"""

from __future__ import annotations

import ctypes as C
import os
import subprocess
import threading
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
# no FMA contraction, no fast-math; sin/cos/pow stay separate glibc calls
CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fno-builtin-sin",
          "-fno-builtin-cos", "-fno-builtin-pow", "-fopenmp", "-Wall", "-shared", "-fPIC"]

F16, BF16, F32 = 1, 2, 3
DTYPES = {"f16": F16, "bf16": BF16, "f32": F32}
POOL_NP = {"f16": np.uint16, "bf16": np.uint16, "f32": np.uint32}  # pool element storage
OK, EINVAL, ERANGE, EOVERFLOW, EUNSUPPORTED = 0, -1, -2, -3, -4

_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so next to it (if stale)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    with _lock:
        if _lib is None:
            build()
            L = C.CDLL(_LIB)
            P = C.c_void_p
            i32, i64, u64, f32, f64 = C.c_int, C.c_int64, C.c_uint64, C.c_float, C.c_double
            sig = {
                "orc_f16_value": (f64, [C.c_uint16]),
                "orc_bf16_value": (f64, [C.c_uint16]),
                "orc_f32_to_f16": (C.c_uint16, [C.c_uint32]),
                "orc_f32_to_bf16": (C.c_uint16, [C.c_uint32]),
                "orc_convert_range": (None, [u64, u64, i32, P]),
                "orc_convert_array": (None, [P, i64, i32, P]),
                "orc_rmsnorm_row": (None, [P, P, i32, f32, P]),
                "orc_rope_table": (None, [f64, i32, i32, P]),
                "orc_rope_row": (None, [P, i32, P, P]),
                "orc_rope_row_ex": (None, [P, i32, i32, i32, P, P]),
                "orc_kv_append": (i32, [i32, i32, i32, i32, i32, i32, i32, i32, i32,
                                        P, P, P, P, P, f32, P, i32, i32, i32, i32, P, P, P, i32, P, P, P]),
                "orc_paged_attention": (i32, [i32, i32, i32, i32, i32, i32, i32, P, P, P, P, i32,
                                              P, P, P, P, i32, i32, i32]),
                "orc_gather_contiguous": (i32, [i32, i32, i32, i32, i32, P, i32, P, P, i32]),
                "orc_dense_attention": (i32, [i32, i32, i32, i32, P, i32, P, P, P]),
                "orc_softmax_scale": (f64, [i32]),
            }
            for name, (res, args) in sig.items():
                fn = getattr(L, name)
                fn.restype = res
                fn.argtypes = args
            _lib = L
    return _lib


def _p(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


# --------------------------------------------------------------------------
# conversions
# --------------------------------------------------------------------------
def convert(x: np.ndarray, kv_dtype: str) -> np.ndarray:
    """float32 array -> 16-bit patterns (nearest, ties to even; NaN reading)."""
    x = _c(x, np.float32)
    out = np.empty(x.shape, dtype=np.uint16)
    lib().orc_convert_array(_p(x), x.size, DTYPES[kv_dtype], _p(out))
    return out


def convert_range(start: int, count: int, kv_dtype: str) -> np.ndarray:
    out = np.empty(count, dtype=np.uint16)
    lib().orc_convert_range(start, count, DTYPES[kv_dtype], _p(out))
    return out


def value16(bits: np.ndarray, kv_dtype: str) -> np.ndarray:
    f = lib().orc_f16_value if kv_dtype == "f16" else lib().orc_bf16_value
    b = np.asarray(bits, dtype=np.uint16).ravel()
    return np.array([f(int(x)) for x in b], dtype=np.float64).reshape(np.shape(bits))


def softmax_scale(D: int) -> float:
    return lib().orc_softmax_scale(D)


# --------------------------------------------------------------------------
# norm / rope
# --------------------------------------------------------------------------
def rmsnorm_row(x: np.ndarray, w: Optional[np.ndarray], eps: float) -> np.ndarray:
    x = _c(x, np.float32)
    w = _c(w, np.float32)
    y = np.empty_like(x)
    lib().orc_rmsnorm_row(_p(x), _p(w), x.size, eps, _p(y))
    return y


def rope_table(theta: float, D: int, max_pos: int, rope_dim: int = 0) -> np.ndarray:
    """[max_pos, R/2, 2] float32 (cos, sin) for the rotary width R = rope_dim
    (0: D)."""
    R = rope_dim or D
    t = np.empty((max_pos, R // 2, 2), dtype=np.float32)
    lib().orc_rope_table(float(theta), R, max_pos, _p(t))
    return t


def rope_row(x: np.ndarray, cs: np.ndarray, rope_dim: int = 0, style: int = 0) -> np.ndarray:
    """Rotates the first rope_dim dims (0: all) of one row; style 0 pairs
    (i, i + rope_dim/2), style 1 pairs (2i, 2i + 1)."""
    x = _c(x, np.float32)
    cs = _c(cs, np.float32)
    y = np.empty_like(x)
    lib().orc_rope_row_ex(_p(x), x.size, rope_dim or x.size, style, _p(cs), _p(y))
    return y


# --------------------------------------------------------------------------
# kv_append / attention
# --------------------------------------------------------------------------
def kv_append(*, Hq, Hkv, D, bs, kv_dtype, q, k, v, tok_req, positions, block_tables, pool_k, pool_v,
              max_seq_len, q_norm_w=None, k_norm_w=None, eps=1e-6, rope=None, S=None, rope_dim=0,
              rope_style=0, window=0):
    """Appends T tokens into ONE layer's pools (modified in place).

    pool_k / pool_v: [num_blocks, Hkv, bs, D], C-contiguous, uint16 for the
    16-bit types and uint32 (float32 bit patterns) for "f32".
    rope: [max_pos, R/2, 2] float32 table (R = rope_dim or D) or None.
    window > 0: block-table rows are rings (entry (p / bs) mod row length).
    Returns (status, q_out)."""
    q, k, v = _c(q, np.float32), _c(k, np.float32), _c(v, np.float32)
    T = len(tok_req)
    bt = _c(block_tables, np.int32)
    S = bt.shape[0] if S is None else S
    assert pool_k.flags.c_contiguous and pool_v.flags.c_contiguous
    assert pool_k.dtype == POOL_NP[kv_dtype] and pool_v.dtype == POOL_NP[kv_dtype]
    nb = pool_k.shape[0]
    rope = _c(rope, np.float32)
    q_out = np.zeros((T, Hq * D), dtype=np.float32)
    st = lib().orc_kv_append(
        T, S, Hq, Hkv, D, bs, nb, max_seq_len, DTYPES[kv_dtype], _p(q), _p(k), _p(v),
        _p(_c(q_norm_w, np.float32)), _p(_c(k_norm_w, np.float32)), eps,
        _p(rope), 0 if rope is None else rope.shape[0], rope_dim, rope_style, window,
        _p(_c(tok_req, np.int32)), _p(_c(positions, np.int32)), _p(bt), bt.shape[1],
        _p(pool_k), _p(pool_v), _p(q_out))
    return st, q_out


def paged_attention(*, Hq, Hkv, D, bs, kv_dtype, q, q_seq, q_pos, block_tables, pool_k, pool_v,
                    want_weights=False, threads=0, window=0):
    """q: [NQ, Hq, D] float32; query i of sequence q_seq[i] at position q_pos[i]
    sees keys 0..q_pos[i] (window > 0: the last `window` of them, through the
    ring). Returns (status, out [NQ,Hq,D] float32, weights)."""
    q = _c(q, np.float32).reshape(-1, Hq, D)
    NQ = q.shape[0]
    q_seq, q_pos = _c(q_seq, np.int32), _c(q_pos, np.int32)
    bt = _c(block_tables, np.int32)
    out = np.empty((NQ, Hq, D), dtype=np.float32)
    maxk = int(q_pos.max(initial=-1)) + 1
    w = np.zeros((NQ, Hq, max(maxk, 1)), dtype=np.float64) if want_weights else None
    assert pool_k.dtype == POOL_NP[kv_dtype] and pool_v.dtype == POOL_NP[kv_dtype]
    assert pool_k.flags.c_contiguous and pool_v.flags.c_contiguous
    st = lib().orc_paged_attention(NQ, Hq, Hkv, D, bs, pool_k.shape[0], DTYPES[kv_dtype], _p(q), _p(q_seq),
                                   _p(q_pos), _p(bt), bt.shape[1], _p(pool_k), _p(pool_v), _p(out), _p(w),
                                   max(maxk, 1), window, threads)
    return st, out, w


def gather_contiguous(*, nk, Hkv, D, bs, bt_row, pool) -> np.ndarray:
    """Keys (or values) 0..nk-1 of one sequence as a contiguous [nk, Hkv, D]
    copy, in the pool's element type (uint16, or uint32 for an f32 pool)."""
    bt_row = _c(bt_row, np.int32)
    assert pool.dtype in (np.uint16, np.uint32) and pool.flags.c_contiguous
    dst = np.empty((max(nk, 0), Hkv, D), dtype=pool.dtype)
    dt = F32 if pool.dtype == np.uint32 else F16  # only the element size matters here
    st = lib().orc_gather_contiguous(nk, Hkv, D, bs, pool.shape[0], _p(bt_row), bt_row.size, _p(pool), _p(dst), dt)
    if st:
        raise ValueError(f"gather failed with status {st}")
    return dst


def dense_attention(*, Hq, Hkv, D, kv_dtype, q, ck, cv) -> np.ndarray:
    q = _c(q, np.float32).reshape(Hq, D)
    out = np.empty((Hq, D), dtype=np.float32)
    st = lib().orc_dense_attention(Hq, Hkv, D, DTYPES[kv_dtype], _p(q), ck.shape[0], _p(_c(ck, POOL_NP[kv_dtype])),
                                   _p(_c(cv, POOL_NP[kv_dtype])), _p(out))
    if st:
        raise ValueError(f"dense attention failed with status {st}")
    return out


# --------------------------------------------------------------------------
# whole-step helpers over a generated workload
# --------------------------------------------------------------------------
def workload_append(wl, pool_k=None, pool_v=None):
    """Runs the oracle's kv_append for every new token of a workload on its
    layer. Returns (status, q_out, pool_k_layer, pool_v_layer) with the pools
    copied unless given."""
    sp = wl.spec
    pk = wl.pool_k[sp.layer].copy() if pool_k is None else pool_k
    pv = wl.pool_v[sp.layer].copy() if pool_v is None else pool_v
    rope = rope_table(sp.theta, sp.D, wl.max_seq_len, sp.rope_dim) if sp.theta else None
    st, q_out = kv_append(Hq=sp.Hq, Hkv=sp.Hkv, D=sp.D, bs=sp.bs, kv_dtype=sp.kv_dtype, q=wl.q, k=wl.k, v=wl.v,
                          tok_req=wl.tok_req, positions=wl.positions, block_tables=wl.block_tables,
                          pool_k=pk, pool_v=pv, max_seq_len=wl.max_seq_len, q_norm_w=wl.q_norm_w,
                          k_norm_w=wl.k_norm_w, eps=sp.eps, rope=rope, rope_dim=sp.rope_dim,
                          rope_style=sp.rope_style, window=sp.window)
    return st, q_out, pk, pv


def workload_queries(wl, q_out, token_ids):
    """Attention inputs for the given new-token indices: (q, q_seq, q_pos)."""
    sp = wl.spec
    t = np.asarray(token_ids, dtype=np.int64)
    return q_out[t].reshape(-1, sp.Hq, sp.D), wl.tok_req[t], wl.positions[t]
