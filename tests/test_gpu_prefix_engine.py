"""The host block manager driving the kernels: a request whose prompt shares
a prefix with a committed one borrows its blocks, appends only its uncached
tokens, and its chunked-prefill and decode outputs match the oracle computed
from scratch on private blocks (tolerance 1e-3 + 1e-3*|oracle|); the borrowed
blocks are never written. Each token's q/k/v are a fixed function of (token
id, position), as they are for a real model, so a shared prefix has the same
cached K/V whichever request wrote it."""

import numpy as np
import pytest
import torch

import paged_kv_cache_321_b200 as K
from gpu_harness import assert_close

pytestmark = pytest.mark.gpu

HQ, HKV, D, BS, THETA, MAXLEN, NBLK = 8, 2, 128, 16, 1e4, 512, 64
F16_NAN = 0x7E00


def qkv_of(tokens, positions):
    """Deterministic q, k, v rows for (token, position) pairs."""
    q = np.empty((len(tokens), HQ * D), np.float32)
    k = np.empty((len(tokens), HKV * D), np.float32)
    v = np.empty((len(tokens), HKV * D), np.float32)
    for i, (t, p) in enumerate(zip(tokens, positions)):
        rng = np.random.default_rng(int(t) * 1_000_003 + int(p))
        q[i], k[i], v[i] = rng.standard_normal(HQ * D), rng.standard_normal(HKV * D), rng.standard_normal(HKV * D)
    return q, k, v


def test_prefix_borrowing_request_matches_oracle(orc):
    dev = torch.device("cuda", 0)
    attn = K.attn_config(HQ, HKV, D, THETA, 1e-6)
    pool = K.Pool(1, HKV, D, BS, MAXLEN, NBLK, "f16", device=dev)
    pool.k.fill_(F16_NAN)  # never-written slots read as NaN (fp16 quiet NaN bits)
    pool.v.fill_(F16_NAN)
    rope = torch.empty(MAXLEN * D, dtype=torch.float32, device=dev)
    K.rope_table_fill(attn, MAXLEN, rope)
    blocks = K.Blocks(1, NBLK, BS, MAXLEN)
    mbps = MAXLEN // BS
    rng = np.random.default_rng(7)
    shared = rng.integers(0, 1000, 48).tolist()          # 3 full blocks
    prompt_a = shared + rng.integers(0, 1000, 22).tolist()
    prompt_b = shared + rng.integers(0, 1000, 30).tolist()

    def append(seq, tokens, positions, out_q):
        q, k, v = qkv_of(tokens, positions)
        bt = torch.tensor([seq.block_table(0, mbps)[0]], dtype=torch.int32, device=dev)
        T = len(tokens)
        K.kv_append(pool, 0, attn, torch.from_numpy(q).to(dev), torch.from_numpy(k).to(dev),
                    torch.from_numpy(v).to(dev), torch.zeros(T, dtype=torch.int32, device=dev),
                    torch.tensor(positions, dtype=torch.int32, device=dev), bt, out_q, None, None, rope, MAXLEN)
        pool.sync_status()
        return bt

    # request A: nothing cached, all 70 tokens appended, then committed
    a = blocks.sequence()
    assert a.allocate_for_tokens(prompt_a) == 0
    a.reserve(len(prompt_a))
    qa = torch.empty((len(prompt_a), HQ * D), dtype=torch.float32, device=dev)
    append(a, prompt_a, list(range(len(prompt_a))), qa)
    a.commit(len(prompt_a))

    # request B: the 3 shared blocks are borrowed, 30 tokens appended
    b = blocks.sequence()
    computed = b.allocate_for_tokens(prompt_b)
    assert computed == 48
    b.reserve(len(prompt_b) + 1)
    ids_a, _ = a.block_table(0)
    ids_b, owned_b = b.block_table(0)
    assert ids_b[:3] == ids_a[:3] and owned_b[:3] == [False] * 3 and all(owned_b[3:])
    borrowed_before = pool.k[0, ids_a[:3]].clone(), pool.v[0, ids_a[:3]].clone()
    new_pos = list(range(computed, len(prompt_b)))
    qb = torch.empty((len(new_pos), HQ * D), dtype=torch.float32, device=dev)
    bt_b = append(b, prompt_b[computed:], new_pos, qb)
    assert torch.equal(pool.k[0, ids_a[:3]], borrowed_before[0])
    assert torch.equal(pool.v[0, ids_a[:3]], borrowed_before[1])

    # chunked prefill of B's new tokens over its whole context
    out = torch.full((len(new_pos), HQ, D), float("nan"), dtype=torch.float32, device=dev)
    ctx = torch.tensor([len(prompt_b)], dtype=torch.int32, device=dev)
    cu = torch.tensor([0, len(new_pos)], dtype=torch.int32, device=dev)
    K.paged_prefill_attention(pool, 0, attn, qb.view(-1, HQ, D), cu, ctx, bt_b, len(new_pos), out)
    pool.sync_status()

    # one decode step of B
    pos_d = len(prompt_b)
    qd = torch.empty((1, HQ * D), dtype=torch.float32, device=dev)
    append(b, [123], [pos_d], qd)
    ctx_d = torch.tensor([pos_d + 1], dtype=torch.int32, device=dev)
    outd = torch.empty((1, HQ, D), dtype=torch.float32, device=dev)
    n = K.decode_workspace_size(pool, attn, 1, pos_d + 1)
    ws = torch.zeros(n // 4 + 64, dtype=torch.float32, device=dev)
    K.paged_decode_attention(pool, 0, attn, qd.view(1, HQ, D), bt_b, ctx_d, pos_d + 1, outd, ws)
    pool.sync_status()

    # the oracle: B from scratch on private blocks 0.., nothing borrowed
    toks = prompt_b + [123]
    pos = list(range(len(toks)))
    q, k, v = qkv_of(toks, pos)
    pk = np.full((NBLK, HKV, BS, D), F16_NAN, np.uint16)
    pv = np.full((NBLK, HKV, BS, D), F16_NAN, np.uint16)
    bt_o = np.full((1, mbps), -1, np.int32)
    bt_o[0, : (len(toks) + BS - 1) // BS] = np.arange((len(toks) + BS - 1) // BS)
    st, q_out = orc.kv_append(Hq=HQ, Hkv=HKV, D=D, bs=BS, kv_dtype="f16", q=q, k=k, v=v,
                              tok_req=np.zeros(len(toks), np.int32), positions=np.array(pos, np.int32),
                              block_tables=bt_o, pool_k=pk, pool_v=pv, max_seq_len=MAXLEN,
                              rope=orc.rope_table(THETA, D, MAXLEN))
    assert st == 0
    rows = np.array(new_pos + [pos_d])
    st, ref, _ = orc.paged_attention(Hq=HQ, Hkv=HKV, D=D, bs=BS, kv_dtype="f16",
                                     q=q_out[rows].reshape(-1, HQ, D), q_seq=np.zeros(len(rows), np.int32),
                                     q_pos=rows.astype(np.int32), block_tables=bt_o, pool_k=pk, pool_v=pv)
    assert st == 0
    # the roped queries the kernels used are the oracle's, bit for bit
    assert np.array_equal(qb.cpu().numpy().view(np.uint32), q_out[new_pos].view(np.uint32))
    assert_close(out.cpu().numpy(), ref[:-1], "prefill with a borrowed prefix")
    assert_close(outd.cpu().numpy(), ref[-1:], "decode with a borrowed prefix")
    for s in (a, b):
        s.close()
    blocks.close()
    pool.close()


def test_device_block_tables_follow_growth():
    # device-resident rows kept equal to the block tables by uploading only
    # the entries that changed (the new ones on growth, all after a new prompt)
    dev = torch.device("cuda", 0)
    blocks = K.Blocks(2, 32, 4, 64)
    seqs = [blocks.sequence(), blocks.sequence()]
    M = 16
    dev_rows = torch.full((2, 2, M), 12345, dtype=torch.int32, device=dev)  # [layer][seq][entry]
    host = {(l, i): np.zeros(M, np.int32) for l in range(2) for i in range(2)}

    def sync_and_check():
        for l in range(2):
            for i, s in enumerate(seqs):
                s.sync_block_table(l, host[l, i], dev_rows[l, i])
        torch.cuda.synchronize()
        for l in range(2):
            for i, s in enumerate(seqs):
                assert dev_rows[l, i].cpu().tolist() == s.block_table(l, M)[0]

    seqs[0].allocate_for_tokens(list(range(10)))
    seqs[1].allocate_for_tokens(list(range(100, 105)))
    sync_and_check()
    for t in range(30):
        seqs[t % 2].append_token(t)
        sync_and_check()
    seqs[0].allocate_for_tokens([1, 2, 3, 4, 5])  # a new prompt replaces the row
    sync_and_check()
    for s in seqs:
        s.close()
    blocks.close()
