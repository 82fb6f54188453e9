"""Seeded workload generator (numpy PCG64).

Every input of a hot-path step is drawn here, in a fixed order, from
``numpy.random.Generator(PCG64(SEED_BASE + spec.seed_offset))``:

1. prior context length of every sequence (integers, inclusive bounds);
2. one permutation of the pool's block IDs (blocks are taken from it in
   order: first each sharing group's prefix blocks, then each sequence's
   private blocks, so IDs are non-contiguous and drawn without replacement);
3. prior K then V contents: each sharing group's prefix first, then every
   sequence's private prior tokens, each as ``[tokens, Hkv, D]`` N(0,1) draws
   times ``value_scale``;
4. the new tokens' q ``[T, Hq*D]``, k ``[T, Hkv*D]``, v ``[T, Hkv*D]``
   (N(0,1) times ``value_scale``), float32;
5. the per-head norm weights for q then k, ``1 + 0.1*N(0,1)`` of shape ``[D]``
   (only when the spec has q/k norm).

Prior cache contents stand for keys and values that earlier steps already
wrote. They are drawn directly as 16-bit values (an f32 pool keeps the
float32 draws as they are): the float32 draw is
TRUNCATED onto the 16-bit grid (bf16: the upper half of the float32 word;
fp16: exponent re-biased and the low 13 mantissa bits dropped, magnitudes
below the fp16 normal range set to zero). Truncation is a way of drawing
values, not the round-to-nearest-even conversion the method performs on new
tokens, which lives only in the oracle and in the CUDA kernels.

Every cache slot that holds no prior token -- including the slot each new
token is about to be appended to, the unused tail of a sequence's last block
and every block no sequence owns -- is filled with a quiet-NaN
sentinel of the pool's type, so any stray read turns an attention output into NaN and any stray
write shows up as a changed sentinel.

Pool layout (per layer): ``[num_blocks][Hkv][block_size][D]`` 16-bit words,
head-major inside a block, so one (block, head) tile is contiguous.

Sliding-window specs (``window > 0``) give every sequence a ring of
``ring_blocks`` block-table entries (default ``ceil(window / block_size)``):
position p lives in entry ``(p // block_size) % ring_blocks``, so only the
last ``ring_blocks * block_size`` prior tokens are resident and drawn (in
position order), each at its ring slot.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional, Sequence

import numpy as np

SEED_BASE = 20261202
NAN16 = {"f16": 0x7E00, "bf16": 0x7FC0}
NAN_BITS = {**NAN16, "f32": 0x7FC00000}  # unused-slot sentinel of each pool type
POOL_NP = {"f16": np.uint16, "bf16": np.uint16, "f32": np.uint32}


@dataclass(frozen=True)
class Segment:
    """A run of sequences with the same new-token count.

    ``fixed`` gives the prior lengths explicitly; otherwise ``count`` priors
    are drawn uniformly from ``[prior_lo, prior_hi]`` (inclusive).
    """

    q_len: int
    count: int = 0
    prior_lo: int = 0
    prior_hi: int = 0
    fixed: tuple = ()


@dataclass(frozen=True)
class Spec:
    name: str
    Hq: int
    Hkv: int
    D: int
    bs: int
    kv_dtype: str  # "f16", "bf16" or "f32" (float32 pool)
    theta: float
    segments: tuple
    eps: float = 1e-6
    qk_norm: bool = False
    value_scale: float = 1.0
    share_group: int = 0  # consecutive sequences per prefix-sharing group
    share_tokens: int = 0  # tokens covered by the shared prefix blocks
    pool_blocks: int = 0  # 0: ceil(pool_margin * blocks needed)
    pool_margin: float = 1.1
    num_layers: int = 1
    layer: int = 0
    seed_offset: int = 0
    rope_dim: int = 0  # rotated leading dims (0: all D)
    rope_style: int = 0  # 0: pairs (i, i + rope_dim/2); 1: pairs (2i, 2i + 1)
    window: int = 0  # sliding window in keys (0: none); block-table rows become rings
    ring_blocks: int = 0  # ring length in blocks (0: ceil(window / bs))
    description: str = ""


@dataclass
class Workload:
    spec: Spec
    S: int
    prior: np.ndarray  # int32 [S] tokens already cached
    q_lens: np.ndarray  # int32 [S] new tokens this step
    ctx: np.ndarray  # int32 [S] prior + q_lens (keys visible after the append)
    cu_q: np.ndarray  # int32 [S+1] offsets of each sequence's new tokens
    max_blocks_per_seq: int
    block_tables: np.ndarray  # int32 [S, max_blocks_per_seq], -1 = unused
    num_blocks: int
    max_seq_len: int
    T: int
    tok_req: np.ndarray  # int32 [T]
    positions: np.ndarray  # int32 [T]
    q: np.ndarray  # float32 [T, Hq*D]
    k: np.ndarray  # float32 [T, Hkv*D]
    v: np.ndarray  # float32 [T, Hkv*D]
    q_norm_w: Optional[np.ndarray]  # float32 [D] or None
    k_norm_w: Optional[np.ndarray]
    pool_k: np.ndarray  # uint16 (uint32 for f32) [num_layers, num_blocks, Hkv, bs, D]
    pool_v: np.ndarray
    shared_blocks: int = 0  # blocks shared inside each group (0: none)
    extra: dict = field(default_factory=dict)

    # convenience views -------------------------------------------------
    @property
    def decode_seqs(self) -> np.ndarray:
        return np.nonzero(self.q_lens == 1)[0].astype(np.int32)

    @property
    def prefill_seqs(self) -> np.ndarray:
        return np.nonzero(self.q_lens > 1)[0].astype(np.int32)

    @property
    def elem_bytes(self) -> int:
        return 4 if self.spec.kv_dtype == "f32" else 2

    def visible_keys(self, seqs: Optional[Sequence[int]] = None) -> np.ndarray:
        """Keys the decode query of each sequence sees: its context, or the
        last `window` of it."""
        s = self.decode_seqs if seqs is None else np.asarray(seqs)
        n = self.ctx[s].astype(np.int64)
        return np.minimum(n, self.spec.window) if self.spec.window > 0 else n

    def kv_read_bytes(self, seqs: Optional[Sequence[int]] = None) -> int:
        """Algorithmic K+V bytes one decode pass reads: every visible key and
        value element once, for every KV head."""
        sp = self.spec
        return int(self.visible_keys(seqs).sum()) * sp.Hkv * sp.D * 2 * self.elem_bytes

    def unique_kv_read_bytes(self, seqs: Optional[Sequence[int]] = None) -> int:
        """Like kv_read_bytes but counting each physical block slot once
        (shared prefix blocks are read by several sequences)."""
        s = self.decode_seqs if seqs is None else np.asarray(seqs)
        sp = self.spec
        if sp.window > 0:  # rings are private
            return self.kv_read_bytes(s)
        seen = {}
        for r in s:
            n = int(self.ctx[r])
            nb = (n + sp.bs - 1) // sp.bs
            for j in range(nb):
                bid = int(self.block_tables[r, j])
                used = min(sp.bs, n - j * sp.bs)
                seen[bid] = max(seen.get(bid, 0), used)
        return sum(seen.values()) * sp.Hkv * sp.D * 2 * self.elem_bytes


def _normal(rng: np.random.Generator, shape, scale: float) -> np.ndarray:
    x = rng.standard_normal(size=shape, dtype=np.float32)
    if scale != 1.0:
        x *= np.float32(scale)
    return x


def _truncate_to_16(x: np.ndarray, kv_dtype: str) -> np.ndarray:
    """Draw 16-bit values by truncating float32 draws (see module doc); an
    f32 pool keeps the float32 draws as they are (their bit patterns)."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    if kv_dtype == "f32":
        return b.copy()
    if kv_dtype == "bf16":
        return (b >> 16).astype(np.uint16)
    a = b & np.uint32(0x7FFFFFFF)
    small = a < np.uint32(0x38800000)  # below 2^-14, the fp16 normal range
    a >>= np.uint32(13)
    a -= np.uint32((127 - 15) << 10)  # re-bias the exponent field
    a[small] = 0  # -> signed zero (N(0,1) draws never exceed the fp16 range)
    a |= (b >> np.uint32(16)) & np.uint32(0x8000)
    return a.astype(np.uint16)


def _draw_priors(rng: np.random.Generator, spec: Spec):
    priors, qls = [], []
    for seg in spec.segments:
        if seg.fixed:
            p = np.asarray(seg.fixed, dtype=np.int64)
        else:
            p = rng.integers(seg.prior_lo, seg.prior_hi + 1, size=seg.count, dtype=np.int64)
        priors.append(p)
        qls.append(np.full(len(p), seg.q_len, dtype=np.int64))
    return np.concatenate(priors).astype(np.int32), np.concatenate(qls).astype(np.int32)


def make_workload(spec: Spec, seed_offset: Optional[int] = None) -> Workload:
    rng = np.random.Generator(np.random.PCG64(SEED_BASE + (spec.seed_offset if seed_offset is None else seed_offset)))
    bs, Hkv, D, Hq = spec.bs, spec.Hkv, spec.D, spec.Hq
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")

    # 1. prior lengths
    prior, q_lens = _draw_priors(rng, spec)
    S = len(prior)
    ctx = prior + q_lens
    nblk = (ctx.astype(np.int64) + bs - 1) // bs
    mbps = int(max(1, nblk.max(initial=1)))
    ring = 0
    if spec.window > 0:
        if spec.share_group:
            raise ValueError("sliding-window rings are private: no prefix sharing")
        ring = spec.ring_blocks or -(-spec.window // bs)
        if ring * bs < spec.window:
            raise ValueError("the ring must hold the window")
        nblk = np.minimum(nblk, ring)
        mbps = ring

    # sharing groups: sequence r shares its first n_shared[r] blocks
    share_blocks = spec.share_tokens // bs if spec.share_group else 0
    group_of = np.arange(S) // spec.share_group if spec.share_group else np.full(S, -1)
    n_groups = int(group_of.max()) + 1 if spec.share_group else 0
    n_shared = np.minimum(share_blocks, prior // bs) if spec.share_group else np.zeros(S, dtype=np.int64)

    need = n_groups * share_blocks + int((nblk - n_shared).sum())
    num_blocks = spec.pool_blocks or int(math.ceil(spec.pool_margin * need))
    if num_blocks < need:
        raise ValueError(f"pool of {num_blocks} blocks cannot hold {need}")

    # 2. block IDs
    perm = rng.permutation(num_blocks).astype(np.int32)
    cursor = 0
    group_blocks = []
    for _ in range(n_groups):
        group_blocks.append(perm[cursor:cursor + share_blocks])
        cursor += share_blocks
    bt = np.full((S, mbps), -1, dtype=np.int32)
    for r in range(S):
        ns = int(n_shared[r])
        if ns:
            bt[r, :ns] = group_blocks[group_of[r]][:ns]
        npriv = int(nblk[r]) - ns
        bt[r, ns:ns + npriv] = perm[cursor:cursor + npriv]
        cursor += npriv

    # 3. prior cache contents
    L = spec.num_layers
    nan = NAN_BITS[spec.kv_dtype]
    pool_k = np.full((L, num_blocks, Hkv, bs, D), nan, dtype=POOL_NP[spec.kv_dtype])
    pool_v = np.full((L, num_blocks, Hkv, bs, D), nan, dtype=POOL_NP[spec.kv_dtype])
    pk, pv = pool_k[spec.layer], pool_v[spec.layer]

    def _place(block_ids, start, kvals, vvals):
        """Writes tokens start .. start+n-1 ([n, Hkv, D] values) of a sequence
        whose j-th block is block_ids[j]; start is a multiple of bs."""
        n = kvals.shape[0]
        full = n // bs
        if full:
            ids = block_ids[start // bs:start // bs + full]
            pk[ids] = kvals[:full * bs].reshape(full, bs, Hkv, D).transpose(0, 2, 1, 3)
            pv[ids] = vvals[:full * bs].reshape(full, bs, Hkv, D).transpose(0, 2, 1, 3)
        rest = n - full * bs
        if rest:
            b = block_ids[start // bs + full]
            pk[b, :, :rest, :] = kvals[full * bs:].transpose(1, 0, 2)
            pv[b, :, :rest, :] = vvals[full * bs:].transpose(1, 0, 2)

    for g in range(n_groups):
        toks = share_blocks * bs
        kx = _truncate_to_16(_normal(rng, (toks, Hkv, D), spec.value_scale), spec.kv_dtype)
        vx = _truncate_to_16(_normal(rng, (toks, Hkv, D), spec.value_scale), spec.kv_dtype)
        # members with shorter priors use a prefix of the group's blocks
        _place(group_blocks[g], 0, kx, vx)
    for r in range(S):
        if ring:
            # the resident positions [max(0, prior - ring*bs), prior) at their ring slots
            first = max(0, int(prior[r]) - ring * bs)
            n = int(prior[r]) - first
            if n <= 0:
                continue
            kx = _truncate_to_16(_normal(rng, (n, Hkv, D), spec.value_scale), spec.kv_dtype)
            vx = _truncate_to_16(_normal(rng, (n, Hkv, D), spec.value_scale), spec.kv_dtype)
            pos = np.arange(first, first + n)
            ids = bt[r, (pos // bs) % ring]
            pk[ids, :, pos % bs, :] = kx
            pv[ids, :, pos % bs, :] = vx
            continue
        start = int(n_shared[r]) * bs
        n = int(prior[r]) - start
        if n <= 0:
            continue
        kx = _truncate_to_16(_normal(rng, (n, Hkv, D), spec.value_scale), spec.kv_dtype)
        vx = _truncate_to_16(_normal(rng, (n, Hkv, D), spec.value_scale), spec.kv_dtype)
        _place(bt[r], start, kx, vx)
    # a group member whose prior stops inside the shared region must not see
    # slots past its own prior as valid: those live in private blocks, so the
    # shared content there is simply never addressed by it.

    # 4. new tokens
    T = int(q_lens.sum())
    cu_q = np.zeros(S + 1, dtype=np.int32)
    cu_q[1:] = np.cumsum(q_lens)
    tok_req = np.repeat(np.arange(S, dtype=np.int32), q_lens)
    positions = np.concatenate([np.arange(prior[r], prior[r] + q_lens[r], dtype=np.int32) for r in range(S)]) if T else np.zeros(0, np.int32)
    q = _normal(rng, (T, Hq * D), spec.value_scale)
    k = _normal(rng, (T, Hkv * D), spec.value_scale)
    v = _normal(rng, (T, Hkv * D), spec.value_scale)

    # 5. norm weights
    qn = kn = None
    if spec.qk_norm:
        qn = (1.0 + 0.1 * rng.standard_normal(D)).astype(np.float32)
        kn = (1.0 + 0.1 * rng.standard_normal(D)).astype(np.float32)

    return Workload(
        spec=spec, S=S, prior=prior, q_lens=q_lens, ctx=ctx.astype(np.int32), cu_q=cu_q,
        max_blocks_per_seq=mbps, block_tables=bt, num_blocks=num_blocks,
        max_seq_len=max(mbps * bs, int(ctx.max(initial=0))), T=T, tok_req=tok_req, positions=positions.astype(np.int32),
        q=q, k=k, v=v, q_norm_w=qn, k_norm_w=kn, pool_k=pool_k, pool_v=pool_v,
        shared_blocks=share_blocks,
    )


# --------------------------------------------------------------------------
# The five workloads of the hot path, with the shapes of the models they copy.
# --------------------------------------------------------------------------
SPECS = {
    "tiny": Spec(
        name="tiny", Hq=4, Hkv=2, D=64, bs=16, kv_dtype="f16", theta=1e4,
        segments=(Segment(q_len=1, fixed=(100,)),), qk_norm=True, pool_blocks=32,
        seed_offset=1,
        description="1 layer, batch 1, GQA 2:1, D=64, bs=16, fp16 pool of 32 blocks; "
                    "100 cached tokens, append at position 100, attend over 101",
    ),
    "llama3-8b-b32": Spec(
        name="llama3-8b-b32", Hq=32, Hkv=8, D=128, bs=16, kv_dtype="bf16", theta=5e5,
        segments=(Segment(q_len=1, count=32, prior_lo=512, prior_hi=4096),), seed_offset=2,
        description="Llama-3-8B-shaped decode, batch 32, Hq=32, Hkv=8, D=128, bs=16, bf16, "
                    "context U[512,4096]",
    ),
    "qwen3-shared-b64": Spec(
        name="qwen3-shared-b64", Hq=32, Hkv=8, D=128, bs=32, kv_dtype="f16", theta=1e6,
        segments=(Segment(q_len=1, count=64, prior_lo=1024, prior_hi=8192),), qk_norm=True,
        share_group=8, share_tokens=2048, seed_offset=3,
        description="Qwen3-style decode with q/k norm, batch 64, bs=32, fp16, context "
                    "U[1024,8192], groups of 8 share their first 2048 tokens' blocks",
    ),
    "long-32k-b8": Spec(
        name="long-32k-b8", Hq=64, Hkv=8, D=128, bs=16, kv_dtype="bf16", theta=1e6,
        segments=(Segment(q_len=1, fixed=(32768,) * 8),), value_scale=0.5, seed_offset=4,
        description="long-context decode, batch 8, GQA 8:1, D=128, bs=16, bf16, 32768 cached "
                    "tokens each, values x0.5",
    ),
    "mistral-swa-b32": Spec(
        name="mistral-swa-b32", Hq=32, Hkv=8, D=128, bs=16, kv_dtype="bf16", theta=1e4,
        segments=(Segment(q_len=1, count=32, prior_lo=2048, prior_hi=32768),), window=4096,
        seed_offset=6,
        description="Mistral-7B-shaped sliding-window decode, batch 32, Hq=32, Hkv=8, D=128, "
                    "bs=16, bf16, context U[2048,32768], window 4096 over a ring of 256 blocks",
    ),
    "mixed-prefill": Spec(
        name="mixed-prefill", Hq=32, Hkv=8, D=128, bs=16, kv_dtype="f16", theta=5e5,
        segments=(Segment(q_len=512, fixed=(0, 512, 1024, 2048)),
                  Segment(q_len=1, count=128, prior_lo=256, prior_hi=4096)),
        seed_offset=5,
        description="mixed chunked prefill: 4 chunks of 512 new tokens on caches of "
                    "0/512/1024/2048 tokens plus 128 decodes with context U[256,4096], fp16",
    ),
}


def spec_by_name(name: str) -> Spec:
    return SPECS[name]
