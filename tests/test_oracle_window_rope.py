"""Pins for the oracle's partial / interleaved RoPE and sliding-window ring.

RoPE of a partial-rotary layer turns only the first rope_dim dims (Op::Rope's
rope_dim in the per-layer RoPE step of forward_layer,
soft3/glia/run/arch/decoder/forward.rs), with the frequencies of that width;
the interleaved convention pairs dims (2i, 2i+1) instead of (i, i + rope_dim/2).
A sliding layer keeps a ring of window-many slots and attends over the last
`window` positions (kv_slot = past_seq_len % cache_seq, read_start =
total_seq - cache_seq in the same function); the paged form keeps a ring of
block-table entries. The checks are closed forms (basis vectors against
math.cos / math.sin, a window of one key), exact identities between the two
pairings, the relative-position property, and equality with independent
paths (attention over a contiguous copy of the last keys; a full, unwrapped
block table; a brute-force slot census).
"""

import math

import numpy as np
import pytest

from workloads import Segment, Spec, make_workload

f32 = np.float32


@pytest.fixture(scope="module")
def wl_small():
    return make_workload(Spec(name="w", Hq=8, Hkv=2, D=64, bs=16, kv_dtype="f16", theta=1e4,
                              segments=(Segment(q_len=1, count=6, prior_lo=0, prior_hi=150),), seed_offset=902))


# ------------------------------------------------------------------ RoPE
@pytest.mark.parametrize("R,style", [(32, 0), (64, 1), (128, 1), (16, 0)])
def test_partial_rope_leaves_tail_untouched(orc, R, style):
    rng = np.random.default_rng(21)
    D = 128
    t = orc.rope_table(1e4, D, 300, R)
    assert t.shape == (300, R // 2, 2)
    for p in (0, 1, 77, 299):
        x = rng.standard_normal(D).astype(f32)
        y = orc.rope_row(x, t[p], R, style)
        assert np.array_equal(y[R:], x[R:])
        if p == 0:
            assert np.array_equal(y, x)


@pytest.mark.parametrize("style", [0, 1])
def test_partial_rope_basis_vectors_use_rotary_width(orc, style):
    # pair i rotates by p * theta^(-2i/R) with R the rotary width, not D
    D, R, theta = 64, 16, 1e4
    t = orc.rope_table(theta, D, 400, R)
    for i in (0, 3, R // 2 - 1):
        a, b = (2 * i, 2 * i + 1) if style else (i, i + R // 2)
        for p in (1, 5, 399):
            ea = np.zeros(D, f32)
            ea[a] = 1
            y = orc.rope_row(ea, t[p], R, style).astype(np.float64)
            ang = p * theta ** (-2.0 * i / R)
            want = np.zeros(D)
            want[a], want[b] = math.cos(ang), math.sin(ang)
            assert np.all(np.abs(y - want) <= 1.2e-7), (i, p)
            eb = np.zeros(D, f32)
            eb[b] = 1
            y = orc.rope_row(eb, t[p], R, style).astype(np.float64)
            want = np.zeros(D)
            want[a], want[b] = -math.sin(ang), math.cos(ang)
            assert np.all(np.abs(y - want) <= 1.2e-7), (i, p)


@pytest.mark.parametrize("R", [8, 32, 128])
def test_interleaved_is_rotate_half_of_deinterleaved_row(orc, R):
    # interleaved pair i = (2i, 2i+1) is rotate-half pair i of the row whose
    # first R dims are reordered evens-then-odds: an exact identity
    rng = np.random.default_rng(22)
    D = 128
    perm = np.concatenate([np.arange(0, R, 2), np.arange(1, R, 2), np.arange(R, D)])
    inv = np.argsort(perm)
    t = orc.rope_table(5e5, D, 2000, R)
    for p in rng.integers(0, 2000, size=20):
        x = rng.standard_normal(D).astype(f32)
        inter = orc.rope_row(x, t[p], R, 1)
        half = orc.rope_row(x[perm], t[p], R, 0)
        assert np.array_equal(inter, half[inv])


def test_two_dim_rotary_pairings_agree(orc):
    # with a rotary width of 2 both conventions pair dims (0, 1)
    rng = np.random.default_rng(23)
    t = orc.rope_table(1e4, 64, 100, 2)
    for p in (3, 50, 99):
        x = rng.standard_normal(64).astype(f32)
        assert np.array_equal(orc.rope_row(x, t[p], 2, 0), orc.rope_row(x, t[p], 2, 1))


@pytest.mark.parametrize("R,style", [(32, 1), (64, 0), (128, 1)])
def test_partial_rope_relative_position_and_norm(orc, R, style):
    rng = np.random.default_rng(24)
    D = 128
    t = orc.rope_table(1e4, D, 4000, R)
    q = rng.standard_normal(D).astype(f32)
    k = rng.standard_normal(D).astype(f32)
    for _ in range(20):
        p, pp, sh = (int(v) for v in rng.integers(0, 1300, size=3))
        rq = orc.rope_row(q, t[p], R, style).astype(np.float64)
        a = float(np.dot(rq, orc.rope_row(k, t[pp], R, style).astype(np.float64)))
        b = float(np.dot(orc.rope_row(q, t[p + sh], R, style).astype(np.float64),
                         orc.rope_row(k, t[pp + sh], R, style).astype(np.float64)))
        assert abs(a - b) < 2e-4 * (1 + abs(a))
        assert abs(np.linalg.norm(rq) - np.linalg.norm(q.astype(np.float64))) < 1e-5


# ------------------------------------------------------- sliding window
def _stream(orc, *, N, W, bs, mbps, Hq=4, Hkv=2, D=64, kv_dtype="f16", theta=1e4, rope_dim=0, style=0, seed=30):
    """Appends positions 0..N-1 of one sequence one step at a time (block
    ids drawn without replacement) and returns the windowed decode output
    of every step, the final pools and the step inputs."""
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((N, Hq * D)).astype(f32)
    k = rng.standard_normal((N, Hkv * D)).astype(f32)
    v = rng.standard_normal((N, Hkv * D)).astype(f32)
    nb = mbps + 3
    ids = rng.permutation(nb)[:mbps].astype(np.int32)
    bt = ids.reshape(1, mbps)
    pk = np.full((nb, Hkv, bs, D), 0x7E00, np.uint16)
    pv = pk.copy()
    rope = orc.rope_table(theta, D, N, rope_dim) if theta else None
    outs = []
    for p in range(N):
        st, qo = orc.kv_append(Hq=Hq, Hkv=Hkv, D=D, bs=bs, kv_dtype=kv_dtype, q=q[p:p + 1], k=k[p:p + 1],
                               v=v[p:p + 1], tok_req=[0], positions=[p], block_tables=bt, pool_k=pk, pool_v=pv,
                               max_seq_len=N, rope=rope, rope_dim=rope_dim, rope_style=style, window=W)
        assert st == 0
        st, out, _ = orc.paged_attention(Hq=Hq, Hkv=Hkv, D=D, bs=bs, kv_dtype=kv_dtype, q=qo.reshape(1, Hq, D),
                                         q_seq=[0], q_pos=[p], block_tables=bt, pool_k=pk, pool_v=pv, window=W)
        assert st == 0
        outs.append(out[0])
    return np.array(outs), pk, pv, bt, (q, k, v)


@pytest.mark.parametrize("W,bs,ring", [(20, 4, 5), (20, 4, 7), (16, 16, 1), (33, 8, 6)])
def test_ring_matches_full_table(orc, W, bs, ring):
    # the same token stream through a ring of `ring` entries and through a
    # table long enough never to wrap gives bitwise equal outputs at every step
    N = 90
    a, _, _, _, _ = _stream(orc, N=N, W=W, bs=bs, mbps=ring, rope_dim=32, style=1)
    b, _, _, _, _ = _stream(orc, N=N, W=W, bs=bs, mbps=-(-N // bs), rope_dim=32, style=1)
    assert np.all(np.isfinite(a)) and np.array_equal(a, b)


def test_ring_slots_hold_latest_positions(orc):
    # brute-force census: slot s of entry e holds the last position p < N with
    # (p // bs) % ring == e and p % bs == s
    N, W, bs, ring = 61, 18, 4, 5
    _, pk, pv, bt, (q, k, v) = _stream(orc, N=N, W=W, bs=bs, mbps=ring, theta=0.0)
    Hkv, D = pk.shape[1], pk.shape[3]
    for e in range(ring):
        for s in range(bs):
            ps = [p for p in range(N) if (p // bs) % ring == e and p % bs == s]
            if not ps:
                assert np.all(pk[bt[0, e], :, s] == 0x7E00)
                continue
            p = ps[-1]
            assert np.array_equal(pk[bt[0, e], :, s], orc.convert(k[p].reshape(Hkv, D), "f16"))
            assert np.array_equal(pv[bt[0, e], :, s], orc.convert(v[p].reshape(Hkv, D), "f16"))


def test_window_is_attention_over_the_last_keys(orc, wl_small):
    # windowed paged attention == plain attention over a contiguous copy of
    # the last W keys only (an unpaged path with no window logic)
    wl = wl_small
    sp = wl.spec
    st, q_out, pk, pv = orc.workload_append(wl)
    q = q_out.reshape(-1, sp.Hq, sp.D)
    for W in (1, 5, 16, 37):
        st, out, w = orc.paged_attention(Hq=sp.Hq, Hkv=sp.Hkv, D=sp.D, bs=sp.bs, kv_dtype=sp.kv_dtype, q=q,
                                         q_seq=wl.tok_req, q_pos=wl.positions, block_tables=wl.block_tables,
                                         pool_k=pk, pool_v=pv, want_weights=True, window=W)
        assert st == 0
        for i in range(wl.T):
            nk = int(wl.positions[i]) + 1
            lo = max(0, nk - W)
            r = wl.tok_req[i]
            ck = orc.gather_contiguous(nk=nk, Hkv=sp.Hkv, D=sp.D, bs=sp.bs, bt_row=wl.block_tables[r], pool=pk)
            cv = orc.gather_contiguous(nk=nk, Hkv=sp.Hkv, D=sp.D, bs=sp.bs, bt_row=wl.block_tables[r], pool=pv)
            dense = orc.dense_attention(Hq=sp.Hq, Hkv=sp.Hkv, D=sp.D, kv_dtype=sp.kv_dtype, q=q[i],
                                        ck=ck[lo:], cv=cv[lo:])
            assert np.array_equal(dense, out[i]), (W, i)
            assert not w[i, :, :lo].any() and np.allclose(w[i, :, lo:nk].sum(axis=1), 1.0, atol=1e-12)


def test_window_of_one_key_is_its_value(orc, wl_small):
    wl = wl_small
    sp = wl.spec
    st, q_out, pk, pv = orc.workload_append(wl)
    st, out, _ = orc.paged_attention(Hq=sp.Hq, Hkv=sp.Hkv, D=sp.D, bs=sp.bs, kv_dtype=sp.kv_dtype,
                                     q=q_out.reshape(-1, sp.Hq, sp.D), q_seq=wl.tok_req, q_pos=wl.positions,
                                     block_tables=wl.block_tables, pool_k=pk, pool_v=pv, window=1)
    grp = sp.Hq // sp.Hkv
    for i in range(wl.T):
        v = orc.value16(orc.convert(wl.v[i].reshape(sp.Hkv, sp.D), sp.kv_dtype), sp.kv_dtype).astype(f32)
        assert np.array_equal(out[i], np.repeat(v, grp, axis=0))


def test_window_covering_the_context_changes_nothing(orc, wl_small):
    wl = wl_small
    sp = wl.spec
    st, q_out, pk, pv = orc.workload_append(wl)
    kw = dict(Hq=sp.Hq, Hkv=sp.Hkv, D=sp.D, bs=sp.bs, kv_dtype=sp.kv_dtype, q=q_out.reshape(-1, sp.Hq, sp.D),
              q_seq=wl.tok_req, q_pos=wl.positions, block_tables=wl.block_tables, pool_k=pk, pool_v=pv)
    W = int(wl.positions.max()) + 1
    assert W <= wl.max_blocks_per_seq * sp.bs
    _, a, _ = orc.paged_attention(**kw)
    _, b, _ = orc.paged_attention(**kw, window=W)
    assert np.array_equal(a, b)


def test_ring_shorter_than_window_is_refused(orc):
    pk = np.zeros((4, 1, 4, 64), np.uint16)
    bt = np.arange(3, dtype=np.int32).reshape(1, 3)
    st, _, _ = orc.paged_attention(Hq=1, Hkv=1, D=64, bs=4, kv_dtype="f16", q=np.zeros((1, 1, 64), f32),
                                   q_seq=[0], q_pos=[5], block_tables=bt, pool_k=pk, pool_v=pk, window=13)
    assert st == orc.EINVAL
    st, _ = orc.kv_append(Hq=1, Hkv=1, D=64, bs=4, kv_dtype="f16", q=np.zeros((1, 64), f32),
                          k=np.zeros((1, 64), f32), v=np.zeros((1, 64), f32), tok_req=[0], positions=[5],
                          block_tables=bt, pool_k=pk, pool_v=pk.copy(), max_seq_len=64, window=13)
    assert st == orc.EINVAL


def test_swa_workload_rings(orc):
    # the sliding-window workload generator: rings of ceil(W/bs) entries, the
    # resident prior positions at their ring slots (a slot census of NaNs)
    sp = Spec(name="swa-t", Hq=4, Hkv=2, D=64, bs=8, kv_dtype="bf16", theta=1e4, window=40,
              segments=(Segment(q_len=1, fixed=(0, 7, 39, 40, 41, 200)),), seed_offset=901)
    wl = make_workload(sp)
    ring = 5
    assert wl.max_blocks_per_seq == ring and wl.max_seq_len >= 201
    for r, prior in enumerate(wl.prior):
        written = {((p // 8) % ring, p % 8) for p in range(max(0, prior - ring * 8), prior)}
        nb = min(ring, -(-(int(prior) + 1) // 8))
        for e in range(nb):
            blk = wl.block_tables[r, e]
            for s in range(8):
                nan = np.all(wl.pool_k[0, blk, :, s] == 0x7FC0)
                assert nan == ((e, s) not in written), (r, e, s)


@pytest.mark.parametrize("n,same", [(5, True), (6, False)])
def test_ring_chunk_limit(orc, n, same):
    # Why a chunk appended at once must not exceed ring tokens - window + 1:
    # appending its tokens one at a time and attending after each is the
    # sliding layer's meaning; appending the whole chunk first gives the same
    # result while the chunk's later keys have not overwritten a ring slot
    # an earlier query of it still needs (W 20, ring 6 x 4 = 24 tokens:
    # a limit of 5 tokens), and a different one beyond
    W, bs, ring, prior, Hq, Hkv, D = 20, 4, 6, 40, 4, 2, 64
    rng = np.random.default_rng(60)
    N = prior + n
    q = rng.standard_normal((N, Hq * D)).astype(f32)
    k = rng.standard_normal((N, Hkv * D)).astype(f32)
    v = rng.standard_normal((N, Hkv * D)).astype(f32)
    bt = np.arange(ring, dtype=np.int32).reshape(1, ring)
    kw = dict(Hq=Hq, Hkv=Hkv, D=D, bs=bs, kv_dtype="f16", block_tables=bt, max_seq_len=N, window=W)
    akw = dict(Hq=Hq, Hkv=Hkv, D=D, bs=bs, kv_dtype="f16", block_tables=bt, window=W)

    def fresh():
        return np.full((ring, Hkv, bs, D), 0x7E00, np.uint16), np.full((ring, Hkv, bs, D), 0x7E00, np.uint16)

    # streamed: each query attends right after its own token is appended
    pk, pv = fresh()
    want = []
    for p in range(N):
        st, qo = orc.kv_append(q=q[p:p + 1], k=k[p:p + 1], v=v[p:p + 1], tok_req=[0], positions=[p],
                               pool_k=pk, pool_v=pv, **kw)
        if p >= prior:
            st, o, _ = orc.paged_attention(q=qo.reshape(1, Hq, D), q_seq=[0], q_pos=[p], pool_k=pk, pool_v=pv, **akw)
            want.append(o[0])
    # chunked: the prior streamed, then the n chunk tokens appended at once
    pk, pv = fresh()
    for p in range(prior):
        orc.kv_append(q=q[p:p + 1], k=k[p:p + 1], v=v[p:p + 1], tok_req=[0], positions=[p], pool_k=pk, pool_v=pv,
                      **kw)
    st, qo = orc.kv_append(q=q[prior:], k=k[prior:], v=v[prior:], tok_req=[0] * n,
                           positions=list(range(prior, N)), pool_k=pk, pool_v=pv, **kw)
    st, got, _ = orc.paged_attention(q=qo.reshape(n, Hq, D), q_seq=[0] * n, q_pos=list(range(prior, N)),
                                     pool_k=pk, pool_v=pv, **akw)
    assert np.array_equal(got, np.array(want)) == same
    # the refusal rule of the prefill kernel, evaluated here, agrees
    ctx, need = N, max(0, N - n - W + 1)
    assert (need + ring * bs <= ctx - 1) == (not same)
