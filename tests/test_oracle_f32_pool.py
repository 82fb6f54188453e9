"""Pins for the oracle's float32 pool (the float32 K/V blocks the pages'
paged attention also reads; runHybridAttentionBlock's f32 path in
makarna/pkg/model/arch/hybrid_decoder.go): kv_append stores the float32
values themselves, and attention reads them exactly.

Checks: the same step appended into an fp16 pool and into a float32 pool
stores, slot for slot, the fp16 conversion of what the float32 pool holds
(the conversion is pinned exhaustively elsewhere) and leaves every other
slot alone; attention over a float32 pool holding fp16-representable values
equals attention over that fp16 pool bit for bit; the contiguous unpaged
twin; a constant V that fp16 cannot represent comes back exactly.
"""

import numpy as np
import pytest

from workloads import NAN_BITS, Segment, Spec, make_workload

f32 = np.float32


def spec(kv_dtype, **kw):
    base = dict(name="f32-pool", Hq=8, Hkv=2, D=64, bs=16, kv_dtype=kv_dtype, theta=1e4, qk_norm=True,
                segments=(Segment(q_len=1, count=5, prior_lo=0, prior_hi=120), Segment(q_len=20, fixed=(33,))),
                seed_offset=950)
    base.update(kw)
    return Spec(**base)


def test_f32_pool_holds_what_the_16bit_pool_converts(orc):
    w32, w16 = make_workload(spec("f32")), make_workload(spec("f16"))
    assert w32.pool_k.dtype == np.uint32 and np.array_equal(w32.block_tables, w16.block_tables)
    st32, q32, pk32, pv32 = orc.workload_append(w32)
    st16, q16, pk16, pv16 = orc.workload_append(w16)
    assert st32 == 0 and st16 == 0
    assert np.array_equal(q32.view(np.uint32), q16.view(np.uint32))  # q' does not depend on the pool type
    sp = w32.spec
    touched = np.zeros(pk32.shape[:3], dtype=bool)
    for t in range(w32.T):
        r, p = w32.tok_req[t], w32.positions[t]
        blk, slot = w32.block_tables[r, p // sp.bs], p % sp.bs
        touched[blk, :, slot] = True
        for pool32, pool16 in ((pk32, pk16), (pv32, pv16)):
            vals = pool32[blk, :, slot].view(f32)
            assert np.array_equal(orc.convert(vals, "f16"), pool16[blk, :, slot])
    # v is stored as given (never normed or rotated)
    t = 0
    r, p = w32.tok_req[t], w32.positions[t]
    assert np.array_equal(pv32[w32.block_tables[r, p // sp.bs], :, p % sp.bs].view(f32).ravel(), w32.v[t])
    assert np.array_equal(pk32[~touched], w32.pool_k[0][~touched])
    assert np.array_equal(pv32[~touched], w32.pool_v[0][~touched])


def _widen(orc, pool16):
    """A float32 pool holding exactly the fp16 pool's values."""
    return orc.value16(pool16, "f16").astype(f32).view(np.uint32).reshape(pool16.shape)


def test_f32_pool_attention_equals_16bit_on_the_same_values(orc):
    w16 = make_workload(spec("f16", segments=(Segment(q_len=1, count=4, prior_lo=0, prior_hi=60),)))
    sp = w16.spec
    st, q_out, pk16, pv16 = orc.workload_append(w16)
    pk32, pv32 = _widen(orc, pk16), _widen(orc, pv16)
    kw = dict(Hq=sp.Hq, Hkv=sp.Hkv, D=sp.D, bs=sp.bs, q=q_out.reshape(-1, sp.Hq, sp.D), q_seq=w16.tok_req,
              q_pos=w16.positions, block_tables=w16.block_tables)
    st16, a, wa = orc.paged_attention(kv_dtype="f16", pool_k=pk16, pool_v=pv16, want_weights=True, **kw)
    st32, b, wb = orc.paged_attention(kv_dtype="f32", pool_k=pk32, pool_v=pv32, want_weights=True, **kw)
    assert st16 == 0 and st32 == 0
    assert np.array_equal(a, b) and np.array_equal(wa, wb)


def test_f32_pool_dense_twin_and_constant_values(orc):
    w = make_workload(spec("f32", segments=(Segment(q_len=1, count=5, prior_lo=0, prior_hi=150),)))
    sp = w.spec
    st, q_out, pk, pv = orc.workload_append(w)
    q = q_out.reshape(-1, sp.Hq, sp.D)
    st, out, _ = orc.paged_attention(Hq=sp.Hq, Hkv=sp.Hkv, D=sp.D, bs=sp.bs, kv_dtype="f32", q=q, q_seq=w.tok_req,
                                     q_pos=w.positions, block_tables=w.block_tables, pool_k=pk, pool_v=pv)
    assert st == 0 and np.all(np.isfinite(out))
    for i in range(w.T):
        nk = int(w.positions[i]) + 1
        r = w.tok_req[i]
        ck = orc.gather_contiguous(nk=nk, Hkv=sp.Hkv, D=sp.D, bs=sp.bs, bt_row=w.block_tables[r], pool=pk)
        cv = orc.gather_contiguous(nk=nk, Hkv=sp.Hkv, D=sp.D, bs=sp.bs, bt_row=w.block_tables[r], pool=pv)
        assert ck.dtype == np.uint32
        dense = orc.dense_attention(Hq=sp.Hq, Hkv=sp.Hkv, D=sp.D, kv_dtype="f32", q=q[i], ck=ck, cv=cv)
        assert np.array_equal(dense, out[i])
    # a constant value fp16 cannot hold comes back exactly
    c = f32(1.2345678)
    pv_c = np.where(pv == NAN_BITS["f32"], pv, np.array([c], f32).view(np.uint32)[0])
    st, out, _ = orc.paged_attention(Hq=sp.Hq, Hkv=sp.Hkv, D=sp.D, bs=sp.bs, kv_dtype="f32", q=q, q_seq=w.tok_req,
                                     q_pos=w.positions, block_tables=w.block_tables, pool_k=pk, pool_v=pv_c)
    assert np.all(out == c)


def test_pool_element_type_is_checked(orc):
    w = make_workload(spec("f16", segments=(Segment(q_len=1, fixed=(5,)),)))
    sp = w.spec
    with pytest.raises(AssertionError):
        orc.paged_attention(Hq=sp.Hq, Hkv=sp.Hkv, D=sp.D, bs=sp.bs, kv_dtype="f32", q=np.zeros((1, sp.Hq, sp.D), f32),
                            q_seq=[0], q_pos=[5], block_tables=w.block_tables, pool_k=w.pool_k[0], pool_v=w.pool_v[0])
