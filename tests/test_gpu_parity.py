"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

kv_append: the written cache (the WHOLE layer pool, NaN sentinels included)
and q_out must match the oracle bit for bit. Decode attention: every output
element within 1e-3 absolute + 1e-3 relative of the oracle's fp64 result.
Small workloads are compared completely; the full-size workloads run in the
launch configuration the benchmark times and are compared on sampled
sequences.
"""

import numpy as np
import pytest
import torch

from gpu_harness import GpuRun, assert_close, oracle_decode
from workloads import NAN16, SPECS, Segment, Spec, make_workload

pytestmark = pytest.mark.gpu

RAGGED = (0, 1, 15, 16, 17, 255, 256, 257, 700, 1500)


def spec(name, **kw):
    base = dict(name=name, Hq=32, Hkv=8, D=128, bs=16, kv_dtype="bf16", theta=5e5,
                segments=(Segment(q_len=1, fixed=RAGGED),), seed_offset=100)
    base.update(kw)
    return Spec(**base)


SMALL = {
    "llama-ragged": spec("llama-ragged"),
    "qwen3-norm-shared": spec("qwen3-norm-shared", bs=32, kv_dtype="f16", theta=1e6, qk_norm=True,
                              segments=(Segment(q_len=1, count=8, prior_lo=100, prior_hi=900),),
                              share_group=4, share_tokens=256, seed_offset=101),
    "gqa8-long": spec("gqa8-long", Hq=64, value_scale=0.5, theta=1e6,
                      segments=(Segment(q_len=1, fixed=(3000, 4100, 33)),), seed_offset=102),
    "d64-g2-f16": spec("d64-g2-f16", Hq=4, Hkv=2, D=64, kv_dtype="f16", theta=1e4, qk_norm=True,
                       segments=(Segment(q_len=1, count=6, prior_lo=0, prior_hi=300),), seed_offset=103),
    "d256-g4": spec("d256-g4", Hq=8, Hkv=2, D=256, segments=(Segment(q_len=1, fixed=(5, 130, 611)),),
                    seed_offset=104),
    "d256-g8": spec("d256-g8", Hq=16, Hkv=2, D=256, kv_dtype="f16",
                    segments=(Segment(q_len=1, fixed=(47, 520)),), seed_offset=105),
    "d64-g8": spec("d64-g8", Hq=16, Hkv=2, D=64, segments=(Segment(q_len=1, fixed=(9, 333)),), seed_offset=106),
    "mha-g1": spec("mha-g1", Hq=4, Hkv=4, D=128, kv_dtype="f16", segments=(Segment(q_len=1, fixed=(1, 77, 400)),),
                   seed_offset=107),
    "bs8": spec("bs8", bs=8, Hq=8, Hkv=2, segments=(Segment(q_len=1, fixed=(3, 8, 9, 100, 301)),), seed_offset=108),
    "bs1": spec("bs1", bs=1, Hq=4, Hkv=1, D=64, kv_dtype="f16", segments=(Segment(q_len=1, fixed=(0, 5, 40)),),
                seed_offset=109),
    "bs128": spec("bs128", bs=128, Hq=8, Hkv=2, segments=(Segment(q_len=1, fixed=(127, 128, 129, 600)),),
                  seed_offset=110),
    "no-rope": spec("no-rope", theta=0.0, Hq=8, Hkv=2, seed_offset=111),
    "two-layers": spec("two-layers", num_layers=2, layer=1, Hq=8, Hkv=2, qk_norm=True, seed_offset=112),
}


@pytest.fixture(scope="module")
def dev():
    assert torch.cuda.is_available(), "GPU tests need CUDA"
    return torch.device("cuda", 0)


def _check_append(orc, run):
    wl = run.wl
    st, q_ref, pk_ref, pv_ref = orc.workload_append(wl)
    assert st == 0
    run.append()
    run.pool.sync_status()
    pk, pv = run.layer_pools()
    q_gpu = run.q_out.cpu().numpy()
    assert np.array_equal(q_gpu.view(np.uint32), q_ref.view(np.uint32)), "q_out differs"
    for name, got, ref in (("K", pk, pk_ref), ("V", pv, pv_ref)):
        if not np.array_equal(got, ref):
            bad = np.argwhere(got != ref)
            raise AssertionError(f"{name} pool differs at {len(bad)} words, first {bad[0].tolist()}: "
                                 f"gpu {got[tuple(bad[0])]:#06x} oracle {ref[tuple(bad[0])]:#06x}")
    # other layers untouched
    for l in range(wl.spec.num_layers):
        if l != wl.spec.layer:
            assert np.array_equal(run.pool.k[l].cpu().numpy().view(np.uint16), wl.pool_k[l])
    return q_ref, pk_ref, pv_ref


@pytest.mark.parametrize("name", ["tiny"] + sorted(SMALL))
def test_append_and_decode_small(orc, dev, name):
    wl = make_workload(SPECS[name] if name == "tiny" else SMALL[name])
    run = GpuRun(wl, dev)
    q_ref, pk, pv = _check_append(orc, run)
    st, ref = oracle_decode(orc, wl, q_ref, pk, pv)
    assert st == 0
    # split_tokens = the fewest keys a warp takes: 16 spreads contexts over
    # many warps (many partials), a huge value puts everything on one warp
    for split in (0, 16, 96, 1 << 20):
        out = run.decode(split_tokens=split)
        run.pool.sync_status()
        assert_close(out.cpu().numpy(), ref, f"{name} split={split}")


@pytest.mark.parametrize("name", ["llama3-8b-b32", "qwen3-shared-b64", "long-32k-b8", "mixed-prefill"])
def test_full_size_append_exact_and_sampled_decode(orc, dev, name):
    wl = make_workload(SPECS[name])
    run = GpuRun(wl, dev)
    q_ref, pk, pv = _check_append(orc, run)
    out = run.decode()  # the benchmark's launch configuration (automatic split)
    run.pool.sync_status()
    dseq = wl.decode_seqs
    rng = np.random.default_rng(5)
    pick = np.sort(rng.choice(len(dseq), size=min(4, len(dseq)), replace=False))
    pick = np.union1d(pick, [int(np.argmax(wl.ctx[dseq])), int(np.argmin(wl.ctx[dseq]))])
    st, ref = oracle_decode(orc, wl, q_ref, pk, pv, seqs=dseq[pick])
    assert st == 0
    assert_close(out.cpu().numpy()[pick], ref, name)


def test_split_invariance_and_single_split_identity(orc, dev):
    wl = make_workload(SMALL["gqa8-long"])
    run = GpuRun(wl, dev)
    run.append()
    one = run.decode(split_tokens=1 << 20)  # one warp takes every context: no partials
    run.pool.sync_status()
    for split in (16, 48, 256, 0):
        out = run.decode(split_tokens=split)
        run.pool.sync_status()
        assert_close(out.cpu().numpy(), one.cpu().numpy(), f"split {split} vs 1")


@pytest.mark.parametrize("name", ["gqa8-long", "llama-ragged"])
def test_workspace_reuse_is_bitwise_stable(orc, dev, name):
    # a zero-filled workspace reused by calls of different split sizes and
    # batch sizes gives the same bits as a fresh one each time: every call
    # leaves its split counters (the first B*Hkv int32 words) at zero
    import paged_kv_cache_321_b200 as K
    wl = make_workload(SMALL[name])
    run = GpuRun(wl, dev)
    run.append()
    q, bt, ctx, mx = run.decode_inputs()
    B, Hkv = ctx.numel(), wl.spec.Hkv
    n = max(K.decode_workspace_size(run.pool, run.attn, B, mx, sp) for sp in (16, 0))
    shared = torch.zeros(n // 4 + 64, dtype=torch.float32, device=dev)
    one = (q[:1].contiguous(), bt[:1].contiguous(), ctx[:1].contiguous(), int(wl.ctx[wl.decode_seqs[0]]))
    calls = [((q, bt, ctx, mx), 16), ((q, bt, ctx, mx), 16), ((q, bt, ctx, mx), 0), (one, 16), ((q, bt, ctx, mx), 16)]
    for args, split in calls:
        out = torch.empty_like(args[0])
        K.paged_decode_attention(run.pool, 0, run.attn, *args, out, shared, split)
        fresh = torch.zeros_like(shared)
        ref = torch.empty_like(args[0])
        K.paged_decode_attention(run.pool, 0, run.attn, *args, ref, fresh, split)
        run.pool.sync_status()
        assert np.array_equal(out.cpu().numpy().view(np.uint32), ref.cpu().numpy().view(np.uint32)), split
        assert not shared.view(torch.int32)[:B * Hkv].any().item(), "split counters not reset"


def test_decode_special_cases(orc, dev):
    wl = make_workload(SMALL["llama-ragged"])
    run = GpuRun(wl, dev)
    run.append()
    sp = wl.spec
    # constant values in every written slot -> output equals the constant
    nan = NAN16[sp.kv_dtype]
    const = 0x3FC0  # bf16 1.5
    v_np = wl.pool_v[0].copy()
    pv_gpu = run.pool.v[0].cpu().numpy().view(np.uint16)
    v_np = np.where(pv_gpu == nan, pv_gpu, np.uint16(const))
    saved = run.pool.v[0].clone()
    run.pool.v[0].copy_(torch.from_numpy(v_np.view(np.int16)))
    out = run.decode().cpu().numpy()
    ctx = wl.ctx[wl.decode_seqs]
    assert np.all(np.abs(out - 1.5) <= 1e-6)
    run.pool.v[0].copy_(saved)
    # zero query -> mean of the visible values; ctx == 1 -> exactly v_0
    q0 = torch.zeros((len(ctx), sp.Hq, sp.D), dtype=torch.float32, device=dev)
    out = run.decode(q=q0).cpu().numpy()
    st, q_ref, pk, pv = orc.workload_append(wl)
    st, ref = orc.paged_attention(Hq=sp.Hq, Hkv=sp.Hkv, D=sp.D, bs=sp.bs, kv_dtype=sp.kv_dtype,
                                  q=np.zeros((len(ctx), sp.Hq, sp.D), np.float32), q_seq=wl.decode_seqs,
                                  q_pos=ctx - 1, block_tables=wl.block_tables, pool_k=pk, pool_v=pv)[:2]
    assert_close(out, ref, "zero query")
    i1 = int(np.nonzero(ctx == 1)[0][0])
    blk = wl.block_tables[wl.decode_seqs[i1], 0]
    v0 = orc.value16(pv[blk, :, 0], sp.kv_dtype).astype(np.float32)
    got = run.decode().cpu().numpy()[i1]
    assert np.array_equal(got, np.repeat(v0, sp.Hq // sp.Hkv, axis=0))


def test_block_permutation_is_bitwise_invariant(orc, dev):
    wl = make_workload(SMALL["llama-ragged"])
    run = GpuRun(wl, dev)
    run.append()
    base = run.decode().cpu().numpy()
    perm = np.random.default_rng(3).permutation(wl.num_blocks)
    ip = torch.from_numpy(np.argsort(perm)).to(dev)
    run.pool.k[0].copy_(run.pool.k[0].index_select(0, ip))
    run.pool.v[0].copy_(run.pool.v[0].index_select(0, ip))
    bt = wl.block_tables
    run.bt = torch.from_numpy(np.where(bt >= 0, perm[np.maximum(bt, 0)], -1).astype(np.int32)).to(dev)
    out = run.decode().cpu().numpy()
    assert np.array_equal(out.view(np.uint32), base.view(np.uint32))


def test_shared_prefix_requests_give_identical_outputs(orc, dev):
    # four requests: identical block tables (fully shared blocks) and identical q
    spec_ = spec("dup", Hq=8, Hkv=2, segments=(Segment(q_len=1, fixed=(700,)),), seed_offset=120)
    wl = make_workload(spec_)
    run = GpuRun(wl, dev)
    run.append()
    q, bt, ctx, mx = run.decode_inputs()
    B = 4
    q4 = q.repeat(B, 1, 1).contiguous()
    bt4 = bt.repeat(B, 1).contiguous()
    ctx4 = ctx.repeat(B).contiguous()
    import paged_kv_cache_321_b200 as K
    out = torch.empty_like(q4)
    n = K.decode_workspace_size(run.pool, run.attn, B, mx)
    ws = torch.zeros(n // 4 + 64, dtype=torch.float32, device=dev)
    K.paged_decode_attention(run.pool, 0, run.attn, q4, bt4, ctx4, mx, out, ws)
    o = out.cpu().numpy().view(np.uint32)
    for b in range(1, B):
        assert np.array_equal(o[b], o[0])


def test_device_errors_are_reported(orc, dev):
    import paged_kv_cache_321_b200 as K
    wl = make_workload(SMALL["llama-ragged"])
    run = GpuRun(wl, dev)
    # position past max_seq_len -> KVP_EOVERFLOW, q_out row zeroed
    pos = run.positions.clone()
    pos[0] = wl.max_seq_len
    run.q_out.fill_(7.0)
    K.kv_append(run.pool, 0, run.attn, run.q, run.k, run.v, run.tok_req, pos, run.bt, run.q_out, None, None,
                run.rope, wl.max_seq_len)
    with pytest.raises(K.KvpError) as e:
        run.pool.sync_status()
    assert e.value.device_code == K.KVP_EOVERFLOW
    assert not run.q_out[0].any()
    # a block id outside the pool -> KVP_ERANGE
    bt = run.bt.clone()
    bt[0, 0] = wl.num_blocks
    q, _, ctx, mx = run.decode_inputs()
    out = torch.empty_like(q)
    n = K.decode_workspace_size(run.pool, run.attn, ctx.numel(), mx)
    ws = torch.zeros(n // 4 + 64, dtype=torch.float32, device=dev)
    K.paged_decode_attention(run.pool, 0, run.attn, q, bt, ctx, mx, out, ws)
    with pytest.raises(K.KvpError) as e:
        run.pool.sync_status()
    assert e.value.device_code == K.KVP_ERANGE
    # a context longer than max_ctx_len -> KVP_ERANGE and a zero row
    K.paged_decode_attention(run.pool, 0, run.attn, q, run.bt.index_select(0, torch.arange(len(ctx), device=dev)),
                             ctx, int(ctx.max()) - 1, out, ws)
    with pytest.raises(K.KvpError) as e:
        run.pool.sync_status()
    assert e.value.device_code == K.KVP_ERANGE
    assert not out[int(torch.argmax(ctx))].any()
    # host-visible errors raise before any launch
    with pytest.raises(K.KvpError):
        K.paged_decode_attention(run.pool, 5, run.attn, q, bt, ctx, mx, out, ws)
    run.pool.sync_status()
