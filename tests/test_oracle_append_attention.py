"""Pins for the oracle's kv_append scatter and paged attention.

Scatter: position p of a sequence lives in block block_tables[r][p / bs] at
slot p % bs (makarna/pkg/kvcache/paged_cache.go: GetBlockForPosition,
GetBlockOffset, Append). Attention: the textbook form of
soft3/glia/run/arch/decoder/forward.rs (forward_layer) with causal visibility
kvLen = startPos + seqLen (makarna/pkg/model/arch/hybrid_decoder.go).
Pins: hand-indexed slots, closed forms (two keys, constant values, zero
query, one key), GQA head mapping, block-ID permutation invariance and a
contiguous unpaged twin.
"""

import math

import numpy as np
import pytest

from workloads import NAN16, Segment, Spec, make_workload

f32 = np.float32


def small_spec(**kw):
    base = dict(name="t", Hq=4, Hkv=2, D=64, bs=16, kv_dtype="f16", theta=1e4,
                segments=(Segment(q_len=1, count=5, prior_lo=0, prior_hi=90),), seed_offset=900)
    base.update(kw)
    return Spec(**base)


# ------------------------------------------------------------------ append
def test_append_hand_indexed_slot(orc):
    wl = make_workload(small_spec(segments=(Segment(q_len=1, fixed=(100,)),), theta=0.0))
    sp = wl.spec
    st, q_out, pk, pv = orc.workload_append(wl)
    assert st == 0
    # position 100 with 16-slot blocks: table entry 6, slot 4
    blk = wl.block_tables[0, 6]
    for h in range(sp.Hkv):
        k_row = wl.k[0, h * sp.D:(h + 1) * sp.D]
        v_row = wl.v[0, h * sp.D:(h + 1) * sp.D]
        assert np.array_equal(pk[blk, h, 4], orc.convert(k_row, "f16"))
        assert np.array_equal(pv[blk, h, 4], orc.convert(v_row, "f16"))
    # nothing else changed
    mask = np.ones(pk.shape[:3], dtype=bool)
    mask[blk, :, 4] = False
    assert np.array_equal(pk[mask], wl.pool_k[0][mask]) and np.array_equal(pv[mask], wl.pool_v[0][mask])
    # without norm and rope, q passes through unchanged
    assert np.array_equal(q_out, wl.q)


def test_append_applies_norm_then_rope(orc):
    wl = make_workload(small_spec(qk_norm=True, kv_dtype="bf16"))
    sp = wl.spec
    st, q_out, pk, _ = orc.workload_append(wl)
    assert st == 0
    table = orc.rope_table(sp.theta, sp.D, wl.max_seq_len)
    for t in range(wl.T):
        p, r = wl.positions[t], wl.tok_req[t]
        for g in range(sp.Hq):
            x = wl.q[t, g * sp.D:(g + 1) * sp.D]
            want = orc.rope_row(orc.rmsnorm_row(x, wl.q_norm_w, sp.eps), table[p])
            assert np.array_equal(q_out[t, g * sp.D:(g + 1) * sp.D], want)
        blk = wl.block_tables[r, p // sp.bs]
        for h in range(sp.Hkv):
            x = wl.k[t, h * sp.D:(h + 1) * sp.D]
            want = orc.convert(orc.rope_row(orc.rmsnorm_row(x, wl.k_norm_w, sp.eps), table[p]), "bf16")
            assert np.array_equal(pk[blk, h, p % sp.bs], want)


def test_append_errors(orc):
    wl = make_workload(small_spec(theta=0.0))
    sp = wl.spec
    base = dict(Hq=sp.Hq, Hkv=sp.Hkv, D=sp.D, bs=sp.bs, kv_dtype=sp.kv_dtype, q=wl.q, k=wl.k, v=wl.v,
                tok_req=wl.tok_req, block_tables=wl.block_tables, max_seq_len=wl.max_seq_len)
    # position past MaxSeqLen: "KV cache overflow"; q_out row zeroed, pool untouched
    pos = wl.positions.copy(); pos[0] = wl.max_seq_len
    pk, pv = wl.pool_k[0].copy(), wl.pool_v[0].copy()
    st, q_out = orc.kv_append(positions=pos, pool_k=pk, pool_v=pv, **base)
    assert st == orc.EOVERFLOW and not q_out[0].any()
    # block id outside the pool: "block index out of range"; q_out still written
    bt = wl.block_tables.copy(); r0 = wl.tok_req[0]; bt[r0, wl.positions[0] // sp.bs] = wl.num_blocks
    pk, pv = wl.pool_k[0].copy(), wl.pool_v[0].copy()
    st, q_out = orc.kv_append(positions=wl.positions, pool_k=pk, pool_v=pv, **{**base, "block_tables": bt})
    assert st == orc.ERANGE and np.array_equal(q_out[0], wl.q[0])
    # unknown sequence
    tr = wl.tok_req.copy(); tr[0] = wl.S
    pk, pv = wl.pool_k[0].copy(), wl.pool_v[0].copy()
    st, _ = orc.kv_append(positions=wl.positions, pool_k=pk, pool_v=pv, **{**base, "tok_req": tr})
    assert st == orc.EINVAL


# --------------------------------------------------------------- attention
def _pool(nb, Hkv, bs, D, fill):
    return np.full((nb, Hkv, bs, D), fill, dtype=np.uint16)


def test_attention_two_keys_closed_form(orc):
    # D = 4, scale = float32(1/2). keys (2,0,0,0) and 0, query (1,0,0,0):
    # scores 1 and 0 -> weights sigmoid(1), 1 - sigmoid(1); values e0 and e1.
    D, bs = 4, 16
    one, two = 0x3C00, 0x4000  # fp16 1.0 and 2.0
    pk, pv = _pool(3, 1, bs, D, 0), _pool(3, 1, bs, D, 0)
    pk[2, 0, 0, 0] = two
    pv[2, 0, 0, 0] = one
    pv[2, 0, 1, 1] = one
    q = np.array([[[1, 0, 0, 0]]], dtype=f32)
    st, out, w = orc.paged_attention(Hq=1, Hkv=1, D=D, bs=bs, kv_dtype="f16", q=q, q_seq=[0], q_pos=[1],
                                     block_tables=np.array([[2]]), pool_k=pk, pool_v=pv, want_weights=True)
    s = 1 / (1 + math.exp(-1.0))
    assert st == 0
    assert np.allclose(out[0, 0], [s, 1 - s, 0, 0], rtol=0, atol=1e-7)
    assert abs(w[0, 0, 0] - s) < 1e-15


def test_attention_gqa_head_mapping(orc):
    # kv head 0 holds values 1, kv head 1 values 2: query heads 0,1 read head 0
    D, bs, Hq, Hkv = 8, 4, 4, 2
    rng = np.random.default_rng(8)
    pk = orc.convert(rng.standard_normal((2, Hkv, bs, D)).astype(f32), "f16")
    pv = np.empty((2, Hkv, bs, D), dtype=np.uint16)
    pv[:, 0], pv[:, 1] = 0x3C00, 0x4000
    q = rng.standard_normal((1, Hq, D)).astype(f32)
    st, out, _ = orc.paged_attention(Hq=Hq, Hkv=Hkv, D=D, bs=bs, kv_dtype="f16", q=q, q_seq=[0], q_pos=[6],
                                     block_tables=np.array([[1, 0]]), pool_k=pk, pool_v=pv)
    assert st == 0
    assert np.all(out[0, :2] == 1.0) and np.all(out[0, 2:] == 2.0)


@pytest.fixture(scope="module")
def wl_small():
    return make_workload(small_spec(Hq=8, Hkv=2, segments=(Segment(q_len=1, count=6, prior_lo=0, prior_hi=150),)))


def _decode(orc, wl, pk, pv, q=None):
    sp = wl.spec
    q = wl.q.reshape(-1, sp.Hq, sp.D) if q is None else q
    return orc.paged_attention(Hq=sp.Hq, Hkv=sp.Hkv, D=sp.D, bs=sp.bs, kv_dtype=sp.kv_dtype, q=q,
                               q_seq=wl.tok_req, q_pos=wl.positions, block_tables=wl.block_tables,
                               pool_k=pk, pool_v=pv, want_weights=True, window=sp.window)


def test_attention_weights_sum_to_one_and_match_dense_twin(orc, wl_small):
    wl = wl_small
    sp = wl.spec
    st, q_out, pk, pv = orc.workload_append(wl)
    st, out, w = _decode(orc, wl, pk, pv, q_out.reshape(-1, sp.Hq, sp.D))
    assert st == 0 and np.all(np.isfinite(out))
    for i in range(wl.T):
        nk = wl.positions[i] + 1
        assert np.allclose(w[i, :, :nk].sum(axis=1), 1.0, atol=1e-12)
        assert not w[i, :, nk:].any()
        r = wl.tok_req[i]
        ck = orc.gather_contiguous(nk=nk, Hkv=sp.Hkv, D=sp.D, bs=sp.bs, bt_row=wl.block_tables[r], pool=pk)
        cv = orc.gather_contiguous(nk=nk, Hkv=sp.Hkv, D=sp.D, bs=sp.bs, bt_row=wl.block_tables[r], pool=pv)
        dense = orc.dense_attention(Hq=sp.Hq, Hkv=sp.Hkv, D=sp.D, kv_dtype=sp.kv_dtype,
                                    q=q_out[i].reshape(sp.Hq, sp.D), ck=ck, cv=cv)
        assert np.array_equal(dense, out[i])


def test_attention_special_cases(orc, wl_small):
    wl = wl_small
    sp = wl.spec
    st, q_out, pk, pv = orc.workload_append(wl)
    # constant values: output equals that constant
    pv_c = np.where(pv == NAN16["f16"], pv, np.uint16(0x3E00))  # 1.5 in every written slot
    st, out, _ = _decode(orc, wl, pk, pv_c, q_out.reshape(-1, sp.Hq, sp.D))
    assert np.all(out == 1.5)
    # zero query: uniform weights, output = mean of visible values
    st, out, w = _decode(orc, wl, pk, pv, np.zeros((wl.T, sp.Hq, sp.D), f32))
    for i in range(wl.T):
        nk = wl.positions[i] + 1
        assert np.allclose(w[i, :, :nk], 1.0 / nk, rtol=1e-14)
        r = wl.tok_req[i]
        cv = orc.gather_contiguous(nk=nk, Hkv=sp.Hkv, D=sp.D, bs=sp.bs, bt_row=wl.block_tables[r], pool=pv)
        mean = orc.value16(cv, "f16").mean(axis=0)  # [Hkv, D]
        grp = sp.Hq // sp.Hkv
        assert np.allclose(out[i], np.repeat(mean, grp, axis=0), rtol=0, atol=2e-7)
    # a single visible key: output is exactly that key's value row
    one = [i for i in range(wl.T) if wl.positions[i] == 0]
    if one:
        i = one[0]
        blk = wl.block_tables[wl.tok_req[i], 0]
        vals = orc.value16(pv[blk, :, 0], "f16").astype(f32)
        assert np.array_equal(out[i], np.repeat(vals, sp.Hq // sp.Hkv, axis=0))


def test_attention_block_permutation_invariance(orc, wl_small):
    wl = wl_small
    sp = wl.spec
    st, q_out, pk, pv = orc.workload_append(wl)
    q = q_out.reshape(-1, sp.Hq, sp.D)
    _, base, _ = _decode(orc, wl, pk, pv, q)
    rng = np.random.default_rng(11)
    perm = rng.permutation(wl.num_blocks)  # block b moves to perm[b]
    pk2, pv2 = np.empty_like(pk), np.empty_like(pv)
    pk2[perm], pv2[perm] = pk, pv
    bt2 = np.where(wl.block_tables >= 0, perm[np.maximum(wl.block_tables, 0)], -1).astype(np.int32)
    st, out2, _ = orc.paged_attention(Hq=sp.Hq, Hkv=sp.Hkv, D=sp.D, bs=sp.bs, kv_dtype=sp.kv_dtype, q=q,
                                      q_seq=wl.tok_req, q_pos=wl.positions, block_tables=bt2,
                                      pool_k=pk2, pool_v=pv2)
    assert st == 0 and np.array_equal(out2, base)


def test_attention_causal_visibility(orc):
    # a prefill chunk: query at position p sees keys 0..p only; later keys
    # poisoned with NaN would otherwise make the output NaN
    spec = small_spec(segments=(Segment(q_len=40, fixed=(25,)),), theta=5e4)
    wl = make_workload(spec)
    sp = wl.spec
    st, q_out, pk, pv = orc.workload_append(wl)
    # the last 10 tokens' slots are re-poisoned: earlier queries must not see them
    for t in range(30, 40):
        p = wl.positions[t]
        pk[wl.block_tables[0, p // sp.bs], :, p % sp.bs] = NAN16["f16"]
        pv[wl.block_tables[0, p // sp.bs], :, p % sp.bs] = NAN16["f16"]
    st, out, _ = orc.paged_attention(Hq=sp.Hq, Hkv=sp.Hkv, D=sp.D, bs=sp.bs, kv_dtype="f16",
                                     q=q_out[:30].reshape(-1, sp.Hq, sp.D), q_seq=wl.tok_req[:30],
                                     q_pos=wl.positions[:30], block_tables=wl.block_tables, pool_k=pk, pool_v=pv)
    assert st == 0 and np.all(np.isfinite(out))


def test_attention_bad_block_id(orc, wl_small):
    wl = wl_small
    sp = wl.spec
    bt = wl.block_tables.copy()
    bt[wl.tok_req[0], 0] = -5
    st, out, _ = orc.paged_attention(Hq=sp.Hq, Hkv=sp.Hkv, D=sp.D, bs=sp.bs, kv_dtype="f16",
                                     q=wl.q.reshape(-1, sp.Hq, sp.D), q_seq=wl.tok_req, q_pos=wl.positions,
                                     block_tables=bt, pool_k=wl.pool_k[0], pool_v=wl.pool_v[0])
    assert st == orc.ERANGE and not out[0].any()


def test_empty_query_gives_zeros(orc, wl_small):
    wl = wl_small
    sp = wl.spec
    st, out, _ = orc.paged_attention(Hq=sp.Hq, Hkv=sp.Hkv, D=sp.D, bs=sp.bs, kv_dtype="f16",
                                     q=wl.q[:1].reshape(-1, sp.Hq, sp.D), q_seq=[0], q_pos=[-1],
                                     block_tables=wl.block_tables, pool_k=wl.pool_k[0], pool_v=wl.pool_v[0])
    assert st == 0 and not out.any()
