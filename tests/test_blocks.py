"""Host block manager (prefix cache): the library against the plain Python
model in oracle/blocks.py, on the CPU. The model's hash is pinned to the
published FNV-1a 64-bit test vectors; its behaviour to scenarios that follow
PagedKVCache in makarna/pkg/kvcache/paged_cache.go (prefix hits borrow
blocks, the last prompt token is never reported cached, allocation rolls back,
Commit publishes completed blocks)."""

import random

import numpy as np
import pytest

import paged_kv_cache_321_b200 as K
from oracle import blocks as OB


def test_fnv1a64_published_vectors():
    assert OB.fnv1a64(b"") == 0xCBF29CE484222325
    assert OB.fnv1a64(b"a") == 0xAF63DC4C8601EC8C
    assert OB.fnv1a64(b"foobar") == 0x85944171F73967E8


def test_block_hash_matches_model_and_chains():
    rng = random.Random(1)
    for n in (0, 1, 16, 32):
        toks = [rng.randrange(-5, 50000) for _ in range(n)]
        assert K.block_hash(toks) == OB.block_hash(toks)
        parent = rng.getrandbits(64)
        assert K.block_hash(toks, parent) == OB.block_hash(toks, parent)
    a = [1, 2, 3, 4]
    # the chain: equal tokens under different parents (or none) hash apart
    assert len({OB.block_hash(a), OB.block_hash(a, 0), OB.block_hash(a, 1)}) == 3


def _state(seq, nl):
    return [seq.block_table(l) for l in range(nl)], len(seq)


def _mstate(m, nl):
    return [(list(m.ids[l]), list(m.owned[l])) for l in range(nl)], m.computed


def test_prefix_hit_borrows_committed_blocks():
    b = K.Blocks(2, 16, 4)
    s1 = b.sequence()
    prompt = list(range(100, 110))            # 2 full blocks + 2 tokens
    assert s1.allocate_for_tokens(prompt) == 0
    ids1, own1 = s1.block_table(0)
    assert len(ids1) == 2 and all(own1)
    s1.commit(len(prompt))                    # both full blocks published
    s2 = b.sequence()
    assert s2.allocate_for_tokens(prompt) == 8  # 2 cached blocks
    ids2, own2 = s2.block_table(0)
    assert ids2 == ids1 and own2 == [False, False]
    assert b.refs(0, ids1[0]) == 2
    # a prompt that is exactly the cached blocks still computes its last token
    s3 = b.sequence()
    assert s3.allocate_for_tokens(prompt[:8]) == 7
    # a different second block: only the first one hits
    s4 = b.sequence()
    assert s4.allocate_for_tokens(prompt[:4] + [7, 7, 7, 7, 1]) == 4
    ids4, own4 = s4.block_table(1)
    assert own4 == [False, True]
    for s in (s1, s2, s3, s4):
        s.close()
    assert b.counts(0)[2] == 0 and b.counts(1)[2] == 0
    b.close()


def test_allocation_rolls_back_when_blocks_run_out():
    b = K.Blocks(3, 4, 2)
    s1, s2 = b.sequence(), b.sequence()
    s1.allocate_for_tokens([1] * 6)           # 3 blocks per layer
    before = [b.counts(l) for l in range(3)]
    with pytest.raises(K.KvpError) as e:
        s2.allocate_for_tokens([2] * 6)       # needs 3 more, 1 left
    assert e.value.code == K.KVP_ERANGE
    assert [b.counts(l) for l in range(3)] == before
    assert s2.num_blocks() == 0
    with pytest.raises(K.KvpError):
        s1.reserve(12)                        # 6 blocks: 3 more needed
    assert [b.counts(l) for l in range(3)] == before and s1.num_blocks() == 3
    s1.reserve(8)                             # 4 blocks: the last free one
    assert b.counts(0)[0] == 0
    s1.close(), s2.close(), b.close()


def test_released_cached_blocks_are_evicted_oldest_first():
    b = K.Blocks(1, 5, 2)
    a, c, d = b.sequence(), b.sequence(), b.sequence()
    a.allocate_for_tokens([1, 1, 2, 2, 9])    # blocks 0, 1
    a.commit(5)
    a.free()                                  # both cached; 0 released first
    assert b.counts(0) == (3, 2, 0)
    c.allocate_for_tokens([3, 3, 4, 4, 5, 5, 6, 6, 9])  # 4 blocks: 3 free + evict block 0
    assert sorted(c.block_table(0)[0]) == [0, 2, 3, 4]
    assert b.counts(0) == (0, 1, 4)           # block 1 is still cached
    c.free()                                  # never committed: back to the free list
    # the chain starts at the evicted [1, 1] block, so nothing hits now
    assert d.allocate_for_tokens([1, 1, 2, 2, 9]) == 0
    assert d.block_table(0)[1] == [True, True]
    for s in (a, c, d):
        s.close()
    b.close()


@pytest.mark.parametrize("seed", range(6))
def test_library_matches_model_on_random_request_streams(seed):
    rng = random.Random(seed)
    nl, nb, bs = rng.choice([1, 2, 3]), rng.choice([6, 12, 24]), rng.choice([1, 2, 4])
    b = K.Blocks(nl, nb, bs, 64)
    m = OB.PoolModel(nl, nb, bs, 64)
    seqs = [b.sequence() for _ in range(3)]
    mseqs = [OB.SeqModel(m) for _ in range(3)]
    mirrors = {(j, l): np.full(nb, 7777, np.int32) for j in range(3) for l in range(nl)}
    prefixes = [[rng.randrange(5) for _ in range(rng.randrange(1, 20))] for _ in range(3)]
    for _ in range(300):
        i = rng.randrange(3)
        s, ms = seqs[i], mseqs[i]
        op = rng.random()
        if op < 0.3:
            toks = list(rng.choice(prefixes)) + [rng.randrange(5) for _ in range(rng.randrange(0, 6))]
            want = ms.allocate_for_tokens(toks)
            if want is None:
                with pytest.raises(K.KvpError):
                    s.allocate_for_tokens(toks)
            else:
                assert s.allocate_for_tokens(toks) == want
        elif op < 0.55:
            t = rng.randrange(5)
            ok = ms.append_token(t)
            if ok:
                s.append_token(t)
            else:
                with pytest.raises(K.KvpError):
                    s.append_token(t)
        elif op < 0.75:
            n = rng.randrange(0, 5)
            ms.commit(n)
            s.commit(n)
        elif op < 0.85:
            n = rng.randrange(0, 40)
            if ms.reserve(n):
                s.reserve(n)
            else:
                with pytest.raises(K.KvpError):
                    s.reserve(n)
        else:
            ms.free_all()
            s.free()
        for j in range(3):
            assert _state(seqs[j], nl) == _mstate(mseqs[j], nl), (seed, j)
            for l in range(nl):
                if rng.random() < 0.5:  # device rows synced at random moments
                    got = seqs[j].block_table_delta(l, mirrors[j, l])
                    assert got == mseqs[j].table_delta(l, nb), (seed, j, l)
                    ids = seqs[j].block_table(l, nb)[0]
                    assert mirrors[j, l].tolist() == ids
        for l in range(nl):
            assert b.counts(l) == m.counts(l)
            for blk in range(nb):
                assert b.refs(l, blk) == m.refs[l][blk]
    for s in seqs:
        s.close()
    for l in range(nl):
        assert b.counts(l)[2] == 0
    b.close()


def test_bad_arguments_are_refused():
    with pytest.raises(K.KvpError):
        K.Blocks(0, 4, 2)
    b = K.Blocks(1, 4, 2, max_seq_len=4)
    s = b.sequence()
    with pytest.raises(K.KvpError) as e:
        s.allocate_for_tokens([1] * 5)
    assert e.value.code == K.KVP_EOVERFLOW
    s.allocate_for_tokens([1] * 4)
    with pytest.raises(K.KvpError) as e:
        s.block_table(0, max_blocks=1)
    assert e.value.code == K.KVP_ERANGE
    s.close(), b.close()


def test_block_table_delta_uploads_only_growth():
    # LayerDevicePtrTables' rule: a row changes only when its blocks grow
    # (then only the new entries) or are replaced (then all of it)
    b = K.Blocks(2, 16, 4)
    s = b.sequence()
    row = np.full(10, 99, np.int32)
    s.allocate_for_tokens(list(range(9)))          # 2 full blocks (the 9th token's block comes later)
    assert s.block_table_delta(0, row) == (0, 10)  # first call: the whole row
    assert row.tolist() == s.block_table(0, 10)[0] and row[2:].tolist() == [-1] * 8
    assert s.block_table_delta(0, row) == (0, 0)   # nothing changed
    for t in (9, 10, 11):                           # completes block 2: a third block
        s.append_token(t)
    assert s.block_table_delta(0, row) == (2, 3)
    s.reserve(20)                                    # 5 blocks
    assert s.block_table_delta(0, row) == (3, 5)
    assert row.tolist() == s.block_table(0, 10)[0]
    # layer 1 keeps its own state: its first call is the whole row
    row1 = np.zeros(10, np.int32)
    assert s.block_table_delta(1, row1) == (0, 10) and row1.tolist() == s.block_table(1, 10)[0]
    s.free()                                         # replaced: the whole row again, all -1
    assert s.block_table_delta(0, row) == (0, 10) and row.tolist() == [-1] * 10
    s.allocate_for_tokens([5] * 4)
    assert s.block_table_delta(0, row) == (0, 10) and row.tolist() == s.block_table(0, 10)[0]
    with pytest.raises(K.KvpError) as e:
        s.block_table_delta(0, np.zeros(0, np.int32))
    assert e.value.code == K.KVP_ERANGE
    assert s.block_table_delta(0, row) == (0, 0)     # a refused call leaves the state alone
    s.close(), b.close()
