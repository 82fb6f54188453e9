"""Plain Python model of the host block manager (test infrastructure only).

Follows PagedKVCache in makarna/pkg/kvcache/paged_cache.go step by step:
ensureCapacityLocked (allocate the missing blocks in every layer, give back
what this call took on a failure), AppendToken (hash a block when it fills),
AllocateForTokens (hash the prompt's full blocks, borrow the cached prefix,
allocate the rest, never report the last prompt token as cached), Commit
(publish completed blocks) and Free. The page does not show the BlockPool
those functions call; this model takes the same reading as the library:
free blocks are handed out last-released-first from a stack initialised so
that block 0 goes first, then cached blocks with no holder are evicted
least recently released first; a block whose last holder lets go is kept as
cached if it has a hash, else freed; the first block published under a hash
keeps it. A block's hash is 64-bit FNV-1a over the byte string
[1 if there is a parent else 0] + parent hash (8 bytes, little-endian, if
any) + the block's token ids (4 bytes each, little-endian, two's complement).

Only tests/ use this module.
"""

from __future__ import annotations

import struct
from collections import OrderedDict

FNV_OFFSET = 0xCBF29CE484222325
FNV_PRIME = 0x100000001B3


def fnv1a64(data: bytes) -> int:
    """64-bit FNV-1a of a byte string."""
    h = FNV_OFFSET
    for b in data:
        h ^= b
        h = (h * FNV_PRIME) & 0xFFFFFFFFFFFFFFFF
    return h


def block_hash(tokens, parent=None) -> int:
    data = bytes([1 if parent is not None else 0])
    if parent is not None:
        data += struct.pack("<Q", parent)
    data += b"".join(struct.pack("<i", int(t)) for t in tokens)
    return fnv1a64(data)


class PoolModel:
    """One BlockPool per the reading above, for every layer."""

    def __init__(self, num_layers, num_blocks, block_size, max_seq_len=0):
        self.num_layers, self.num_blocks, self.block_size = num_layers, num_blocks, block_size
        self.max_seq_len = max_seq_len
        self.refs = [[0] * num_blocks for _ in range(num_layers)]
        self.hash_of = [dict() for _ in range(num_layers)]      # block -> hash
        self.by_hash = [dict() for _ in range(num_layers)]      # hash -> block
        self.free = [list(range(num_blocks - 1, -1, -1)) for _ in range(num_layers)]  # stack, top = end
        self.cached = [OrderedDict() for _ in range(num_layers)]  # unheld hashed blocks, oldest first

    # BlockPool.AllocateBlocks
    def allocate(self, layer, n):
        if n > len(self.free[layer]) + len(self.cached[layer]):
            return None
        out = []
        for _ in range(n):
            if self.free[layer]:
                b = self.free[layer].pop()
            else:
                b, _ = self.cached[layer].popitem(last=False)
                del self.by_hash[layer][self.hash_of[layer].pop(b)]
            self.refs[layer][b] = 1
            out.append(b)
        return out

    # BlockPool.FreeBlocks
    def release(self, layer, ids):
        for b in ids:
            if self.refs[layer][b] <= 0:
                continue
            self.refs[layer][b] -= 1
            if self.refs[layer][b] == 0:
                if b in self.hash_of[layer]:
                    self.cached[layer][b] = True
                else:
                    self.free[layer].append(b)

    # BlockPool.FindCachedBlocks
    def find(self, layer, hashes, limit):
        out = []
        for h in hashes[:limit]:
            if h not in self.by_hash[layer]:
                break
            out.append(self.by_hash[layer][h])
        return out

    # BlockPool.TouchBlocks
    def touch(self, layer, ids):
        for b in ids:
            self.cached[layer].pop(b, None)
            self.refs[layer][b] += 1

    # BlockPool.CacheBlocks
    def cache(self, layer, ids, hashes):
        for b, h in zip(ids, hashes):
            if b in self.hash_of[layer] or h in self.by_hash[layer]:
                continue
            self.hash_of[layer][b] = h
            self.by_hash[layer][h] = b

    def counts(self, layer):
        held = sum(1 for r in self.refs[layer] if r > 0)
        return len(self.free[layer]), len(self.cached[layer]), held


class SeqModel:
    """PagedKVCache's per-request state."""

    def __init__(self, pool: PoolModel):
        self.pool = pool
        self.epoch = 0
        self.synced = {}  # layer -> (epoch, entries) of the last table delta
        self.free_all()

    def free_all(self):
        p = getattr(self, "pool", None)
        if p is not None and hasattr(self, "ids"):
            for l in range(p.num_layers):
                p.release(l, self.ids[l])
        self.ids = [[] for _ in range(self.pool.num_layers)]
        self.owned = [[] for _ in range(self.pool.num_layers)]
        self.tokens, self.hashes = [], []
        self.computed = self.written = 0
        self.epoch = getattr(self, "epoch", 0) + 1

    # LayerDevicePtrTables' rule: device rows change only when the number of
    # blocks grows, or when the sequence's blocks are replaced
    def table_delta(self, layer, max_blocks):
        n = len(self.ids[layer])
        if n > max_blocks:
            return None
        ep, done = self.synced.get(layer, (None, 0))
        if ep != self.epoch:
            rng = (0, max_blocks)
        elif n > done:
            rng = (done, n)
        else:
            rng = (0, 0)
        self.synced[layer] = (self.epoch, n)
        return rng

    def _ensure(self, required):
        p = self.pool
        cur = len(self.ids[0])
        if required <= cur:
            return True
        taken = []
        for l in range(p.num_layers):
            got = p.allocate(l, required - cur)
            if got is None:
                for k, g in enumerate(taken):
                    p.release(k, g)
                    del self.ids[k][cur:]
                    del self.owned[k][cur:]
                return False
            taken.append(got)
            self.ids[l] += got
            self.owned[l] += [True] * len(got)
        return True

    def allocate_for_tokens(self, tokens):
        p = self.pool
        if p.max_seq_len and len(tokens) > p.max_seq_len:
            return None
        self.free_all()
        bs = p.block_size
        self.tokens = list(tokens)
        self.hashes = []
        for i in range(len(tokens) // bs):
            self.hashes.append(block_hash(tokens[i * bs:(i + 1) * bs], self.hashes[-1] if i else None))
        if self.hashes:
            hit = len(self.hashes)
            cached = []
            for l in range(p.num_layers):
                c = p.find(l, self.hashes, hit)
                cached.append(c)
                hit = len(c)
            for l in range(p.num_layers):
                c = cached[l][:hit]
                p.touch(l, c)
                self.ids[l] = list(c)
                self.owned[l] = [False] * hit
            fresh = len(self.hashes) - hit
            if fresh > 0:
                for l in range(p.num_layers):
                    got = p.allocate(l, fresh)
                    if got is None:
                        for k in range(p.num_layers):
                            p.release(k, self.ids[k])
                        self.ids = [[] for _ in range(p.num_layers)]
                        self.owned = [[] for _ in range(p.num_layers)]
                        self.tokens, self.hashes = [], []
                        return None
                    self.ids[l] += got
                    self.owned[l] += [True] * fresh
            self.computed = hit * bs
        if self.computed >= len(tokens):
            self.computed = max(len(tokens) - 1, 0)
        self.written = self.computed
        return self.computed

    def append_token(self, t):
        bs = self.pool.block_size
        self.tokens.append(int(t))
        n = len(self.tokens)
        if n % bs:
            return True
        bi = n // bs - 1
        ok = self._ensure(bi + 1)
        parent = self.hashes[bi - 1] if 0 < bi <= len(self.hashes) else None
        h = block_hash(self.tokens[bi * bs:(bi + 1) * bs], parent)
        if bi < len(self.hashes):
            self.hashes[bi] = h
        else:
            self.hashes.append(h)
        return ok

    def reserve(self, num_tokens):
        bs = self.pool.block_size
        return self._ensure((num_tokens + bs - 1) // bs)

    def commit(self, n):
        p = self.pool
        old = self.computed
        self.computed += n
        self.written = max(self.written, self.computed)
        ob, nb = old // p.block_size, min(self.computed // p.block_size, len(self.hashes))
        if nb > ob:
            for l in range(p.num_layers):
                upto = min(nb, len(self.ids[l]))
                if upto > ob:
                    p.cache(l, self.ids[l][ob:upto], self.hashes[ob:upto])
