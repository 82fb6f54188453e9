"""Host-side checks of the seeded workload generator (no arithmetic of the
method lives there; these check shapes, block-table structure and sentinels)."""

import numpy as np
import pytest

from workloads import NAN16, SPECS, Segment, Spec, make_workload


@pytest.mark.parametrize("name", ["tiny", "llama3-8b-b32", "qwen3-shared-b64", "mixed-prefill"])
def test_block_tables_and_sentinels(name):
    wl = make_workload(SPECS[name])
    sp = wl.spec
    bs = sp.bs
    nan = NAN16[sp.kv_dtype]
    used = {}
    for r in range(wl.S):
        nb = (wl.ctx[r] + bs - 1) // bs
        row = wl.block_tables[r]
        assert np.all(row[:nb] >= 0) and np.all(row[:nb] < wl.num_blocks)
        assert np.all(row[nb:] == -1)
        for j, b in enumerate(row[:nb]):
            used.setdefault(int(b), set()).add((r, j))
    # a block is owned by one sequence unless it is a shared prefix block,
    # and shared blocks sit at the same table index for every sharer
    for b, owners in used.items():
        if len(owners) > 1:
            assert sp.share_group and len({j for _, j in owners}) == 1
            assert max(j for _, j in owners) < sp.share_tokens // bs
    # the slot every new token is appended to holds the sentinel
    pk = wl.pool_k[sp.layer]
    for t in range(wl.T):
        r, p = wl.tok_req[t], wl.positions[t]
        assert np.all(pk[wl.block_tables[r, p // bs], :, p % bs] == nan)
    # prior tokens hold finite values
    for r in range(min(wl.S, 8)):
        for p in (0, wl.prior[r] - 1):
            if p >= 0 and wl.prior[r] > 0:
                assert np.all(pk[wl.block_tables[r, p // bs], :, p % bs] != nan)
    # unowned blocks are all sentinel
    free = np.setdiff1d(np.arange(wl.num_blocks), np.array(list(used.keys())))
    assert np.all(pk[free] == nan)
    assert wl.num_blocks >= len(used)


def test_shared_prefix_structure():
    wl = make_workload(SPECS["qwen3-shared-b64"])
    bt = wl.block_tables
    for g in range(8):
        rows = bt[g * 8:(g + 1) * 8]
        pri = wl.prior[g * 8:(g + 1) * 8]
        for a in range(8):
            ns = min(64, pri[a] // 32)
            assert np.array_equal(rows[a, :ns], rows[np.argmax(pri)][:ns])
            # the appended token's block is private
            assert pri[a] // 32 >= ns


def test_seeded_and_deterministic():
    a = make_workload(SPECS["tiny"])
    b = make_workload(SPECS["tiny"])
    assert np.array_equal(a.q, b.q) and np.array_equal(a.pool_k, b.pool_k)
    assert np.array_equal(a.block_tables, b.block_tables)
    c = make_workload(SPECS["tiny"], seed_offset=99)
    assert not np.array_equal(a.q, c.q)


def test_tiny_matches_its_description():
    wl = make_workload(SPECS["tiny"])
    assert wl.S == 1 and wl.prior[0] == 100 and wl.positions[0] == 100 and wl.ctx[0] == 101
    assert wl.num_blocks == 32 and wl.block_tables[0, :7].min() >= 0
    assert wl.q_norm_w is not None and wl.spec.theta == 1e4


def test_truncated_draws_are_on_the_16bit_grid():
    spec = Spec(name="g", Hq=2, Hkv=1, D=16, bs=8, kv_dtype="f16", theta=0.0,
                segments=(Segment(q_len=1, fixed=(64,)),))
    wl = make_workload(spec)
    vals = wl.pool_k[0][wl.pool_k[0] != NAN16["f16"]].view(np.float16).astype(np.float32)
    assert np.all(np.isfinite(vals)) and 0.5 < np.std(vals) < 1.5
