"""GPU parity of the per-layer RoPE variants and the sliding-window ring
against the oracle.

kv_append with partial rotary (only the first rope_dim dims turn) and with
interleaved pairs (2i, 2i+1): the cache bytes and q_out are compared bit for
bit over the whole pool. Sliding-window decode and prefill read the last
`window` keys of each sequence through a ring of block-table entries
(position p in entry (p / block_size) mod ring length): outputs within
1e-3 + 1e-3*|oracle| on both decode kernels (tensor-core groups of 4 and 8,
CUDA-core groups of 1 and 2 and blocks smaller than a tile) and on the
tensor-core prefill, with contexts below the window, at its edge and many
rings long, and every unused slot a NaN sentinel."""

import numpy as np
import pytest
import torch

import paged_kv_cache_321_b200 as K
from gpu_harness import GpuRun, assert_close, oracle_decode, oracle_rows
from workloads import Segment, Spec, make_workload

pytestmark = pytest.mark.gpu


def spec(name, **kw):
    base = dict(name=name, Hq=32, Hkv=8, D=128, bs=16, kv_dtype="bf16", theta=1e4,
                segments=(Segment(q_len=1, count=12, prior_lo=0, prior_hi=1500),), seed_offset=300)
    base.update(kw)
    return Spec(**base)


ROPE_CASES = {
    "partial-half-32": spec("partial-half-32", rope_dim=32, qk_norm=True, kv_dtype="f16"),
    "partial-inter-64": spec("partial-inter-64", rope_dim=64, rope_style=1, seed_offset=301),
    "interleaved-full": spec("interleaved-full", rope_style=1, Hq=8, Hkv=2, D=64, seed_offset=302),
    "partial-inter-d256": spec("partial-inter-d256", D=256, Hq=8, Hkv=2, rope_dim=64, rope_style=1,
                               qk_norm=True, seed_offset=303),
    "prefill-partial": spec("prefill-partial", rope_dim=48, rope_style=1,
                            segments=(Segment(q_len=70, fixed=(0, 33)),), seed_offset=304),
}


@pytest.mark.parametrize("name", sorted(ROPE_CASES))
def test_append_rope_variants_bit_exact(orc, name):
    wl = make_workload(ROPE_CASES[name])
    run = GpuRun(wl, torch.device("cuda", 0))
    run.append()
    run.pool.sync_status()
    st, q_ref, pk, pv = orc.workload_append(wl)
    assert st == 0
    gk, gv = run.layer_pools()
    assert np.array_equal(run.q_out.cpu().numpy().view(np.uint32), q_ref.view(np.uint32)), "q_out"
    assert np.array_equal(gk, pk), "K pool"
    assert np.array_equal(gv, pv), "V pool"


WINDOW_CASES = {
    # tensor-core kernel, groups of 4, ring of 256 blocks
    "tc-g4-w4096": spec("tc-g4-w4096", window=4096, segments=(Segment(q_len=1, count=16, prior_lo=3000, prior_hi=20000),
                                                              Segment(q_len=1, fixed=(0, 15, 4095, 4096, 4111))),
                        seed_offset=310),
    # window not a multiple of the tile, a ring longer than the window
    "tc-g4-w1000-ring70": spec("tc-g4-w1000-ring70", window=1000, ring_blocks=70, kv_dtype="f16",
                               segments=(Segment(q_len=1, count=10, prior_lo=0, prior_hi=9000),), seed_offset=311),
    "tc-g8-bs32-w777": spec("tc-g8-bs32-w777", Hq=64, window=777, bs=32,
                            segments=(Segment(q_len=1, count=9, prior_lo=500, prior_hi=5000),), seed_offset=312),
    # CUDA-core kernel: groups of 1 and 2, and blocks smaller than a tile
    "cc-g1-w300": spec("cc-g1-w300", Hq=8, Hkv=8, window=300, kv_dtype="f16",
                       segments=(Segment(q_len=1, count=10, prior_lo=0, prior_hi=2000),), seed_offset=313),
    "cc-g2-w129": spec("cc-g2-w129", Hq=16, Hkv=8, D=64, window=129,
                       segments=(Segment(q_len=1, count=10, prior_lo=0, prior_hi=2000),), seed_offset=314),
    "cc-g4-bs8-w100": spec("cc-g4-bs8-w100", Hq=16, Hkv=4, bs=8, window=100,
                           segments=(Segment(q_len=1, count=10, prior_lo=0, prior_hi=900),), seed_offset=315),
    "window-one": spec("window-one", Hq=16, Hkv=4, window=1, segments=(Segment(q_len=1, count=6, prior_lo=0, prior_hi=90),),
                       seed_offset=316),
}


@pytest.mark.parametrize("name", sorted(WINDOW_CASES))
def test_window_decode_matches_oracle(orc, name):
    wl = make_workload(WINDOW_CASES[name])
    run = GpuRun(wl, torch.device("cuda", 0))
    run.append()
    out = run.decode()
    run.pool.sync_status()
    st, q_ref, pk, pv = orc.workload_append(wl)
    assert st == 0
    gk, gv = run.layer_pools()
    assert np.array_equal(gk, pk) and np.array_equal(gv, pv), "ring slots"
    st, ref = oracle_decode(orc, wl, q_ref, pk, pv)
    assert st == 0
    assert_close(out.cpu().numpy(), ref, name)


@pytest.mark.parametrize("name", ["tc-g4-w1000-ring70", "cc-g1-w300"])
def test_window_decode_splits_agree(orc, name):
    # every split size gives the oracle's result
    wl = make_workload(WINDOW_CASES[name])
    run = GpuRun(wl, torch.device("cuda", 0))
    run.append()
    st, q_ref, pk, pv = orc.workload_append(wl)
    st, ref = oracle_decode(orc, wl, q_ref, pk, pv)
    for split in (16, 64, 4096):
        out = run.decode(split_tokens=split)
        run.pool.sync_status()
        assert_close(out.cpu().numpy(), ref, f"{name} split {split}")


def test_ring_stream_token_by_token(orc):
    # one sequence appended a token at a time through a 4-block ring (the
    # ring wraps 12 times) and decoded after every step
    Hq, Hkv, D, bs, W, ring, N = 8, 2, 128, 16, 50, 4, 800
    dev = torch.device("cuda", 0)
    attn = K.attn_config(Hq, Hkv, D, 1e4, 1e-6, 0, 0, W)
    nb = ring + 2
    pool = K.Pool(1, Hkv, D, bs, N, nb, "f16", device=dev)
    pool.k.fill_(0x7E00)
    pool.v.fill_(0x7E00)
    rope = torch.empty(N * D, dtype=torch.float32, device=dev)
    K.rope_table_fill(attn, N, rope)
    rng = np.random.default_rng(40)
    q = rng.standard_normal((N, Hq * D)).astype(np.float32)
    k = rng.standard_normal((N, Hkv * D)).astype(np.float32)
    v = rng.standard_normal((N, Hkv * D)).astype(np.float32)
    bt_np = np.array([[4, 1, 5, 2]], np.int32)
    bt = torch.from_numpy(bt_np).to(dev)
    qd, kd, vd = (torch.from_numpy(a).to(dev) for a in (q, k, v))
    qo = torch.empty((N, Hq * D), dtype=torch.float32, device=dev)
    outs = torch.empty((N, Hq, D), dtype=torch.float32, device=dev)
    zero = torch.zeros(1, dtype=torch.int32, device=dev)
    ws = torch.zeros(K.decode_workspace_size(pool, attn, 1, N) // 4 + 64, dtype=torch.float32, device=dev)
    for p in range(N):
        pos = torch.tensor([p], dtype=torch.int32, device=dev)
        K.kv_append(pool, 0, attn, qd[p:p + 1], kd[p:p + 1], vd[p:p + 1], zero, pos, bt, qo[p:p + 1], None, None,
                    rope, N)
        K.paged_decode_attention(pool, 0, attn, qo[p:p + 1].view(1, Hq, D), bt, pos + 1, N, outs[p:p + 1], ws)
    pool.sync_status()
    pk = np.full((nb, Hkv, bs, D), 0x7E00, np.uint16)
    pv = pk.copy()
    tab = orc.rope_table(np.float32(1e4), D, N)
    ref = np.empty((N, Hq, D), np.float32)
    for p in range(N):
        st, q_ref = orc.kv_append(Hq=Hq, Hkv=Hkv, D=D, bs=bs, kv_dtype="f16", q=q[p:p + 1], k=k[p:p + 1],
                                  v=v[p:p + 1], tok_req=[0], positions=[p], block_tables=bt_np, pool_k=pk, pool_v=pv,
                                  max_seq_len=N, rope=tab, window=W)
        assert st == 0
        st, o, _ = orc.paged_attention(Hq=Hq, Hkv=Hkv, D=D, bs=bs, kv_dtype="f16", q=q_ref.reshape(1, Hq, D),
                                       q_seq=[0], q_pos=[p], block_tables=bt_np, pool_k=pk, pool_v=pv, window=W)
        ref[p] = o[0]
    assert np.array_equal(pool.k[0].cpu().numpy().view(np.uint16), pk)
    assert_close(outs.cpu().numpy(), ref, "ring stream")
    pool.close()


PREFILL_CASES = {
    # no wrap during the chunk: the ring holds the whole context
    "pf-w200-nowrap": spec("pf-w200-nowrap", kv_dtype="f16", window=200, ring_blocks=40,
                           segments=(Segment(q_len=300, fixed=(0, 150)), Segment(q_len=1, fixed=(77,))),
                           seed_offset=320),
    # a wrapped ring: chunk of 441 = ring tokens - window + 1, the longest allowed
    "pf-w200-wrap": spec("pf-w200-wrap", kv_dtype="f16", window=200, ring_blocks=40, Hq=16, Hkv=4,
                         segments=(Segment(q_len=441, fixed=(900,)), Segment(q_len=37, fixed=(2000,))),
                         seed_offset=321),
    # window smaller than a KV tile, groups of 8, bs 32
    "pf-w64-g8-bs32": spec("pf-w64-g8-bs32", Hq=16, Hkv=2, bs=32, window=64, ring_blocks=8, kv_dtype="f16",
                           segments=(Segment(q_len=150, fixed=(10, 1000)),), seed_offset=322),
    # groups of 1, a window at the first chunk's start
    "pf-w40-g1": spec("pf-w40-g1", Hq=4, Hkv=4, window=40, ring_blocks=10, kv_dtype="f16",
                      segments=(Segment(q_len=90, fixed=(0, 41, 500)),), seed_offset=324),
}


@pytest.mark.parametrize("name", sorted(PREFILL_CASES))
def test_window_prefill_matches_oracle(orc, name):
    wl = make_workload(PREFILL_CASES[name])
    run = GpuRun(wl, torch.device("cuda", 0))
    run.append()
    run.pool.sync_status()
    out, rows = run.prefill()
    run.pool.sync_status()
    st, q_ref, pk, pv = orc.workload_append(wl)
    st, ref = oracle_rows(orc, wl, q_ref, pk, pv, rows)
    assert st == 0
    assert_close(out.cpu().numpy(), ref, name)


def test_window_prefill_refuses_overwritten_chunk(orc):
    # a chunk one token longer than the ring allows: reported, rows untouched
    sp = spec("pf-too-long", kv_dtype="f16", window=200, ring_blocks=40, Hq=16, Hkv=4,
              segments=(Segment(q_len=442, fixed=(900,)),), seed_offset=323)
    wl = make_workload(sp)
    run = GpuRun(wl, torch.device("cuda", 0))
    run.append()
    run.pool.sync_status()
    out, _ = run.prefill()
    with pytest.raises(K.KvpError) as e:
        run.pool.sync_status()
    assert e.value.code == K.KVP_EDEVICE
    assert torch.isnan(out).all()


def test_ring_shorter_than_window_refused_on_host():
    dev = torch.device("cuda", 0)
    pool = K.Pool(1, 2, 64, 16, 256, 8, "f16", device=dev)
    attn = K.attn_config(4, 2, 64, 1e4, 1e-6, 0, 0, 100)
    bt = torch.zeros((1, 6), dtype=torch.int32, device=dev)  # 96 tokens < 100
    q = torch.zeros((1, 4, 64), dtype=torch.float32, device=dev)
    ctx = torch.ones(1, dtype=torch.int32, device=dev)
    ws = torch.zeros(1 << 20, dtype=torch.float32, device=dev)
    with pytest.raises(K.KvpError) as e:
        K.paged_decode_attention(pool, 0, attn, q, bt, ctx, 1, torch.empty_like(q), ws)
    assert e.value.code == K.KVP_EINVAL
    pool.close()


@pytest.mark.parametrize("kw", [dict(rope_dim=33), dict(rope_dim=130), dict(rope_dim=-2), dict(rope_style=2),
                                dict(window=-1)])
def test_bad_rope_or_window_fields_refused_on_host(kw):
    dev = torch.device("cuda", 0)
    pool = K.Pool(1, 2, 128, 16, 256, 8, "f16", device=dev)
    attn = K.attn_config(4, 2, 128, 1e4, 1e-6, **kw)
    T = 1
    f = lambda n: torch.zeros((T, n), dtype=torch.float32, device=dev)
    i = torch.zeros(T, dtype=torch.int32, device=dev)
    bt = torch.zeros((1, 4), dtype=torch.int32, device=dev)
    with pytest.raises(K.KvpError) as e:
        K.kv_append(pool, 0, attn, f(4 * 128), f(2 * 128), f(2 * 128), i, i, bt, f(4 * 128))
    assert e.value.code == K.KVP_EINVAL
    pool.close()
