"""GPU parity of chunked-prefill attention (tcgen05 tensor cores) against the
oracle: every query row of a chunk attends causally over the paged cache
(keys 0..its own position). Tolerance as for decode: 1e-3 + 1e-3*|oracle|
(the tensor-core operands are fp16: q rounded after scaling, P rounded)."""

import numpy as np
import pytest
import torch

from gpu_harness import GpuRun, assert_close, oracle_rows
from workloads import SPECS, Segment, Spec, make_workload

pytestmark = pytest.mark.gpu


def spec(name, **kw):
    base = dict(name=name, Hq=32, Hkv=8, D=128, bs=16, kv_dtype="f16", theta=5e5,
                segments=(Segment(q_len=50, fixed=(0, 37)), Segment(q_len=200, fixed=(130,)),
                          Segment(q_len=1, fixed=(300,))),
                seed_offset=200)
    base.update(kw)
    return Spec(**base)


CASES = {
    "g4-bs16": spec("g4-bs16"),
    "g4-bs32": spec("g4-bs32", bs=32, seed_offset=201),
    "g1": spec("g1", Hq=4, Hkv=4, seed_offset=202),
    "g2": spec("g2", Hq=8, Hkv=4, seed_offset=203),
    "g8": spec("g8", Hq=16, Hkv=2, seed_offset=204),
    "long-chunk": spec("long-chunk", Hq=8, Hkv=2, segments=(Segment(q_len=300, fixed=(700,)),),
                       seed_offset=205),
    "one-token-chunks": spec("one-token-chunks", Hq=8, Hkv=2, segments=(Segment(q_len=2, fixed=(0, 5, 127, 128)),),
                             seed_offset=206),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_prefill_matches_oracle(orc, name):
    wl = make_workload(CASES[name])
    run = GpuRun(wl, torch.device("cuda", 0))
    run.append()
    run.pool.sync_status()
    out, rows = run.prefill()
    run.pool.sync_status()
    st, q_ref, pk, pv = orc.workload_append(wl)
    st, ref = oracle_rows(orc, wl, q_ref, pk, pv, rows)
    assert st == 0
    assert_close(out.cpu().numpy(), ref, name)


def test_prefill_last_row_equals_decode(orc):
    # the last query of a chunk sees the same keys as a decode at that position
    wl = make_workload(CASES["g4-bs16"])
    run = GpuRun(wl, torch.device("cuda", 0))
    run.append()
    out, rows = run.prefill()
    last = [int(np.nonzero(rows == wl.cu_q[r + 1] - 1)[0][0]) for r in wl.prefill_seqs]
    import paged_kv_cache_321_b200 as K
    seqs = wl.prefill_seqs
    q = out.new_empty((len(seqs), wl.spec.Hq, wl.spec.D))
    q.copy_(run.q_out.index_select(0, torch.tensor(rows[last], device=q.device)).view(len(seqs), wl.spec.Hq, wl.spec.D))
    dec = run.decode(seqs=seqs, q=q)
    run.pool.sync_status()
    assert_close(out.cpu().numpy()[last], dec.cpu().numpy(), "prefill last row vs decode")


def test_prefill_full_size_sampled(orc):
    wl = make_workload(SPECS["mixed-prefill"])
    run = GpuRun(wl, torch.device("cuda", 0))
    run.append()
    out, rows = run.prefill()
    run.pool.sync_status()
    st, q_ref, pk, pv = orc.workload_append(wl)
    rng = np.random.default_rng(9)
    pick = np.sort(rng.choice(len(rows), size=96, replace=False))
    pick = np.union1d(pick, [0, len(rows) - 1])
    st, ref = oracle_rows(orc, wl, q_ref, pk, pv, rows[pick])
    assert st == 0
    assert_close(out.cpu().numpy()[pick], ref, "mixed-prefill sampled rows")


def test_prefill_bf16_pool_within_its_bound(orc):
    # With a bf16 pool the tensor-core operands are bf16 (A and B of one MMA
    # share a type): q and the softmax weights are rounded to 8 significant
    # bits (relative error up to 2^-8) instead of fp16's 11, so the error is
    # about 8x fp16's and the 1e-3 bar does not hold; this pins the bound that
    # does, 1e-2 + 1e-2*|oracle| (about 2x the largest error seen).
    wl = make_workload(spec("bf16-pool", kv_dtype="bf16", Hq=16, Hkv=2, bs=32,
                            segments=(Segment(q_len=150, fixed=(10, 1000)),), seed_offset=207))
    run = GpuRun(wl, torch.device("cuda", 0))
    run.append()
    out, rows = run.prefill()
    run.pool.sync_status()
    st, q_ref, pk, pv = orc.workload_append(wl)
    st, ref = oracle_rows(orc, wl, q_ref, pk, pv, rows)
    g = out.cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(g))
    assert np.all(np.abs(g - ref) <= 1e-2 + 1e-2 * np.abs(ref))
