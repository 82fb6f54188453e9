"""Helpers that run a generated workload through the CUDA library (C ABI via
the package's binding) and through the oracle, for the parity tests."""

from __future__ import annotations

import numpy as np
import torch

import paged_kv_cache_321_b200 as K

TOL_ABS = 1e-3
TOL_REL = 1e-3


class GpuRun:
    """A workload's inputs resident on the GPU, plus a pool holding its cache."""

    def __init__(self, wl, device="cuda"):
        sp = wl.spec
        self.wl = wl
        dev = torch.device(device)
        self.dev = dev
        self.pool = K.Pool(sp.num_layers, sp.Hkv, sp.D, sp.bs, wl.max_seq_len, wl.num_blocks, sp.kv_dtype,
                           device=dev)
        self.pool.k.copy_(torch.from_numpy(wl.pool_k.view(np.int16)))
        self.pool.v.copy_(torch.from_numpy(wl.pool_v.view(np.int16)))
        self.attn = K.attn_config(sp.Hq, sp.Hkv, sp.D, float(np.float32(sp.theta)), sp.eps, sp.rope_dim,
                                  sp.rope_style, sp.window)
        t = lambda a, dt=None: None if a is None else torch.from_numpy(np.ascontiguousarray(a)).to(dev)
        self.q, self.k, self.v = t(wl.q), t(wl.k), t(wl.v)
        self.qn, self.kn = t(wl.q_norm_w), t(wl.k_norm_w)
        self.tok_req, self.positions = t(wl.tok_req), t(wl.positions)
        self.bt = t(wl.block_tables)
        self.ctx = t(wl.ctx)
        self.q_out = torch.zeros((wl.T, sp.Hq * sp.D), dtype=torch.float32, device=dev)
        self.rope = None
        if sp.theta:
            self.rope = torch.empty(wl.max_seq_len * (sp.rope_dim or sp.D), dtype=torch.float32, device=dev)
            K.rope_table_fill(self.attn, wl.max_seq_len, self.rope)

    def append(self):
        sp = self.wl.spec
        K.kv_append(self.pool, sp.layer, self.attn, self.q, self.k, self.v, self.tok_req, self.positions, self.bt,
                    self.q_out, self.qn, self.kn, self.rope, self.wl.max_seq_len if self.rope is not None else 0)

    def decode_inputs(self, seqs=None):
        """(q [B,Hq,D], block tables, ctx lens, max ctx) of the decode sequences."""
        wl = self.wl
        sp = wl.spec
        seqs = wl.decode_seqs if seqs is None else np.asarray(seqs)
        tok = wl.cu_q[seqs]  # each decode sequence's single new token
        idx = torch.from_numpy(tok.astype(np.int64)).to(self.dev)
        q = self.q_out.index_select(0, idx).view(len(seqs), sp.Hq, sp.D).contiguous()
        s = torch.from_numpy(seqs.astype(np.int64)).to(self.dev)
        bt = self.bt.index_select(0, s).contiguous()
        ctx = self.ctx.index_select(0, s).contiguous()
        return q, bt, ctx, int(wl.ctx[seqs].max(initial=0))

    def decode(self, seqs=None, split_tokens=0, q=None, out=None):
        sp = self.wl.spec
        qd, bt, ctx, mx = self.decode_inputs(seqs)
        q = qd if q is None else q
        B = ctx.numel()
        out = torch.empty((B, sp.Hq, sp.D), dtype=torch.float32, device=self.dev) if out is None else out
        n = K.decode_workspace_size(self.pool, self.attn, B, mx, split_tokens)
        ws = torch.zeros(max(n, 256) // 4 + 64, dtype=torch.float32, device=self.dev)
        K.paged_decode_attention(self.pool, sp.layer, self.attn, q, bt, ctx, mx, out, ws, split_tokens)
        return out

    def prefill(self, seqs=None, out=None):
        """Prefill attention for the given sequences' new tokens (default: all
        sequences with more than one new token). Returns (out [n, Hq, D], rows)
        where rows are the new-token indices in order."""
        wl = self.wl
        sp = wl.spec
        seqs = wl.prefill_seqs if seqs is None else np.asarray(seqs)
        rows = np.concatenate([np.arange(wl.cu_q[r], wl.cu_q[r + 1]) for r in seqs]).astype(np.int64)
        cu = np.zeros(len(seqs) + 1, dtype=np.int32)
        cu[1:] = np.cumsum(wl.q_lens[seqs])
        dev = self.dev
        q = self.q_out.index_select(0, torch.from_numpy(rows).to(dev)).view(-1, sp.Hq, sp.D).contiguous()
        s = torch.from_numpy(seqs.astype(np.int64)).to(dev)
        bt = self.bt.index_select(0, s).contiguous()
        ctx = self.ctx.index_select(0, s).contiguous()
        out = torch.full_like(q, float("nan")) if out is None else out
        K.paged_prefill_attention(self.pool, sp.layer, self.attn, q, torch.from_numpy(cu).to(dev), ctx, bt,
                                  int(wl.q_lens[seqs].max()), out)
        return out, rows

    def layer_pools(self):
        sp = self.wl.spec
        return (self.pool.k[sp.layer].cpu().numpy().view(np.uint16),
                self.pool.v[sp.layer].cpu().numpy().view(np.uint16))


def oracle_decode(orc, wl, q_out, pk, pv, seqs=None, threads=0):
    """Oracle attention for the decode sequences' new tokens."""
    sp = wl.spec
    seqs = wl.decode_seqs if seqs is None else np.asarray(seqs)
    tok = wl.cu_q[seqs]
    q = q_out[tok].reshape(-1, sp.Hq, sp.D)
    st, out, _ = orc.paged_attention(Hq=sp.Hq, Hkv=sp.Hkv, D=sp.D, bs=sp.bs, kv_dtype=sp.kv_dtype, q=q,
                                     q_seq=seqs, q_pos=wl.ctx[seqs] - 1, block_tables=wl.block_tables,
                                     pool_k=pk, pool_v=pv, threads=threads, window=sp.window)
    return st, out


def oracle_rows(orc, wl, q_out, pk, pv, rows, threads=0):
    """Oracle attention for arbitrary new-token rows (query at its position)."""
    sp = wl.spec
    rows = np.asarray(rows)
    st, out, _ = orc.paged_attention(Hq=sp.Hq, Hkv=sp.Hkv, D=sp.D, bs=sp.bs, kv_dtype=sp.kv_dtype,
                                     q=q_out[rows].reshape(-1, sp.Hq, sp.D), q_seq=wl.tok_req[rows],
                                     q_pos=wl.positions[rows], block_tables=wl.block_tables, pool_k=pk, pool_v=pv,
                                     threads=threads, window=sp.window)
    return st, out


def assert_close(gpu, ref, what=""):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert gpu.shape == ref.shape, (gpu.shape, ref.shape)
    assert np.all(np.isfinite(gpu)), f"{what}: non-finite GPU output"
    err = np.abs(gpu - ref)
    bound = TOL_ABS + TOL_REL * np.abs(ref)
    bad = err > bound
    if bad.any():
        i = np.unravel_index(np.argmax(err - bound), err.shape)
        raise AssertionError(f"{what}: {bad.sum()} elements out of tolerance; worst at {i}: gpu {gpu[i]} "
                             f"oracle {ref[i]} (max abs err {err.max():.3e})")
    return float(err.max())
