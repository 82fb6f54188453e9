"""The allocation-free decode entry point.

paged_decode_attention_noalloc exists for callers that cannot allocate
device memory -- a host that reserved all GPU memory for its own allocator,
or a latency-critical loop that cannot afford cudaMalloc's device-wide
synchronisation -- so it uses a fixed workspace inside the library instead of
one the caller passes in. This test calls it through the C ABI twice in a row
and checks both results against the ordinary entry point with a
caller-provided workspace, within the tolerance the parity tests use. It
sits in a file pytest collects last and builds everything it needs itself,
so it passes both alone in a fresh process and after the other tests.
"""

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


def test_noalloc_decode_matches_the_workspace_entry_point():
    import paged_kv_cache_321_b200 as K
    from gpu_harness import GpuRun, assert_close
    from workloads import Segment, Spec, make_workload

    spec = Spec(name="noalloc", Hq=32, Hkv=8, D=128, bs=16, kv_dtype="bf16", theta=5e5,
                segments=(Segment(q_len=1, fixed=(1, 17, 300, 1500, 2500)),), seed_offset=300)
    wl = make_workload(spec)
    run = GpuRun(wl, torch.device("cuda", 0))
    run.append()
    q, bt, ctx, mx = run.decode_inputs()
    ref = run.decode()  # caller-provided workspace
    run.pool.sync_status()
    ref = ref.cpu().numpy()
    for _ in range(2):  # the fixed workspace keeps the previous call's contents
        out = torch.full_like(q, float("nan"))
        K.paged_decode_attention_noalloc(run.pool, 0, run.attn, q, bt, ctx, mx, out)
        run.pool.sync_status()
        assert_close(out.cpu().numpy(), ref, "noalloc vs workspace")


def test_noalloc_refuses_calls_above_its_fixed_size():
    import paged_kv_cache_321_b200 as K
    from gpu_harness import GpuRun
    from workloads import Segment, Spec, make_workload

    spec = Spec(name="noalloc-big", Hq=32, Hkv=8, D=128, bs=16, kv_dtype="f16", theta=0.0,
                segments=(Segment(q_len=1, fixed=(40,)),), seed_offset=301)
    wl = make_workload(spec)
    run = GpuRun(wl, torch.device("cuda", 0))
    q, bt, ctx, mx = run.decode_inputs()
    B = 2048  # partials of 2048 sequences x 8 kv heads need far more than 16 MiB
    big = K.decode_workspace_size(run.pool, run.attn, B, 20000)
    assert big > K.NOALLOC_SCRATCH_BYTES
    qq = q.expand(B, -1, -1).contiguous()
    bb = torch.zeros((B, 2000), dtype=torch.int32, device=q.device)
    cc = torch.zeros(B, dtype=torch.int32, device=q.device)
    out = torch.empty_like(qq)
    with pytest.raises(K.KvpError, match="fixed"):
        K.paged_decode_attention_noalloc(run.pool, 0, run.attn, qq, bb, cc, 20000, out)
