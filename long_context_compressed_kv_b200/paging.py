"""Host-side management of paged compressed caches.

[deep-read] "异构 KV cache 与磁盘前缀复用": next to a fixed-size state cache
(the window ring and the uncompressed tail, per sequence) the compressed
history lives in a classical block cache whose block covers lcm(4, 128) = 128
raw tokens, i.e. 32 CSA entries and 32 indexer keys, or 1 HCA entry.  The
kernels read such pools through a block table (``block_table`` in
``index_topk``, ``sparse_mqa``, ``dense_mqa`` and ``decode``; see "Paged
caches" in include/v4attn.h); this module keeps the table and the free list
on the host:

* ``BlockPool`` - ids of the pool's blocks, handed out and taken back;
* ``BlockTable`` - per sequence the blocks that cover its tokens so far, grown
  as the sequence extends, released when it ends; ``tensor()`` gives the int32
  [B][blocks_per_seq] table the calls take (-1 marks a block not allocated);
* ``pool_rows`` / ``scatter_to_pool`` - the pool row of an entry, and a
  per-sequence cache copied into a pool (for moving existing caches over).

One table can serve every layer of a sequence: each layer keeps its own pools,
all indexed by the same block ids (32 rows a block in a CSA layer's entry and
key pools, 1 row in an HCA layer's).
"""
from __future__ import annotations

from typing import List, Optional

import numpy as np
import torch

BLOCK_TOKENS = 128          # raw tokens a block covers: lcm(4, 128)


def entries_per_block(m: int) -> int:
    """Rows a block holds in the pools of a layer with compression ratio m."""
    if m < 1 or BLOCK_TOKENS % m:
        raise ValueError(f"compression ratio {m} does not divide a {BLOCK_TOKENS}-token block")
    return BLOCK_TOKENS // m


class BlockPool:
    """The ids 0 .. n_blocks-1 of a pool's blocks; lowest free ids first."""

    def __init__(self, n_blocks: int):
        if n_blocks < 1:
            raise ValueError("a pool needs at least one block")
        self.n_blocks = n_blocks
        self._free = list(range(n_blocks - 1, -1, -1))     # pop() yields the lowest id

    @property
    def n_free(self) -> int:
        return len(self._free)

    def alloc(self, n: int) -> List[int]:
        if n < 0:
            raise ValueError("negative block count")
        if n > len(self._free):
            raise MemoryError(f"{n} blocks asked for, {len(self._free)} free")
        return [self._free.pop() for _ in range(n)]

    def free(self, ids) -> None:
        for i in ids:
            if not 0 <= i < self.n_blocks:
                raise ValueError(f"block {i} is not in the pool")
        taken = set(self._free)
        for i in ids:
            if i in taken:
                raise ValueError(f"block {i} is already free")
            taken.add(i)
        self._free.extend(ids)
        self._free.sort(reverse=True)


class BlockTable:
    """Blocks of B sequences: sequence b's logical block i (raw tokens
    128 i .. 128 i + 127) is physical block table[b][i], -1 while not
    allocated.  blocks_per_seq bounds a sequence's length to
    128 * blocks_per_seq tokens."""

    def __init__(self, B: int, blocks_per_seq: int, pool: BlockPool):
        if B < 1 or blocks_per_seq < 1:
            raise ValueError("a table needs at least one sequence and one block each")
        self.B, self.blocks_per_seq, self.pool = B, blocks_per_seq, pool
        self.table = np.full((B, blocks_per_seq), -1, dtype=np.int32)
        self.n_blocks = np.zeros(B, dtype=np.int64)          # allocated blocks per sequence

    def ensure(self, b: int, n_tokens: int) -> None:
        """Allocate the blocks that tokens 0 .. n_tokens-1 of sequence b need."""
        need = -(-n_tokens // BLOCK_TOKENS)
        if need > self.blocks_per_seq:
            raise ValueError(f"{n_tokens} tokens need {need} blocks, the table holds "
                             f"{self.blocks_per_seq}")
        have = int(self.n_blocks[b])
        if need > have:
            self.table[b, have:need] = self.pool.alloc(need - have)
            self.n_blocks[b] = need

    def release(self, b: int) -> None:
        """Give sequence b's blocks back to the pool (the sequence ended)."""
        have = int(self.n_blocks[b])
        self.pool.free([int(x) for x in self.table[b, :have]])
        self.table[b, :] = -1
        self.n_blocks[b] = 0

    def tensor(self, device="cuda") -> torch.Tensor:
        """The int32 [B][blocks_per_seq] table the library's calls take."""
        return torch.from_numpy(self.table.copy()).to(device)


def pool_rows(table: np.ndarray, m: int, b: int, e) -> np.ndarray:
    """Pool row of entry (or indexer key) e of sequence b in a layer of ratio m."""
    epb = entries_per_block(m)
    e = np.asarray(e, dtype=np.int64)
    return table[b, e // epb].astype(np.int64) * epb + e % epb


def scatter_to_pool(rows: torch.Tensor, table: np.ndarray, m: int,
                    n_blocks: int, pool: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Copy per-sequence cache rows [B][n][...] into a pool of n_blocks * epb
    rows: sequence b's rows of logical block i land in block table[b][i]
    (blocks whose table entry is -1 are skipped).  n must cover the table's
    allocated blocks, i.e. n >= epb * (last allocated block + 1)."""
    epb = entries_per_block(m)
    B = rows.shape[0]
    rest = tuple(rows.shape[2:])
    if pool is None:
        pool = torch.zeros((n_blocks * epb,) + rest, dtype=rows.dtype, device=rows.device)
    view = pool.view((n_blocks, epb) + rest)
    for b in range(B):
        ids = np.nonzero(table[b] >= 0)[0]
        if ids.size == 0:
            continue
        if (int(ids[-1]) + 1) * epb > rows.shape[1]:
            raise ValueError("the per-sequence rows do not cover the table's blocks")
        src = rows[b, : (int(ids[-1]) + 1) * epb].reshape((-1, epb) + rest)
        idx = torch.from_numpy(ids).to(rows.device)
        dst = torch.from_numpy(table[b, ids].astype(np.int64)).to(rows.device)
        view[dst] = src[idx]
    return pool
