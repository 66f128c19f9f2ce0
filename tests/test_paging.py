"""Host-side block management of paged compressed caches (CPU only): the pool's
free list, the per-sequence block table as sequences grow and end, the pool
row of an entry (row = table[b][e / epb] * epb + e mod epb, epb = 128 / m: the
layout the kernels read, see "Paged caches" in include/v4attn.h), and the copy
of per-sequence caches into a pool."""
import numpy as np
import pytest
import torch

from long_context_compressed_kv_b200 import paging


def test_entries_per_block_follow_the_128_token_block():
    assert paging.entries_per_block(4) == 32        # CSA: 32 entries and 32 indexer keys
    assert paging.entries_per_block(128) == 1       # HCA: one entry a block
    with pytest.raises(ValueError):
        paging.entries_per_block(3)


def test_pool_hands_out_lowest_ids_and_takes_them_back():
    pool = paging.BlockPool(6)
    assert pool.alloc(2) == [0, 1]
    assert pool.alloc(1) == [2]
    pool.free([1])
    assert pool.n_free == 4
    assert pool.alloc(2) == [1, 3]
    with pytest.raises(MemoryError):
        pool.alloc(3)
    with pytest.raises(ValueError):
        pool.free([4])                              # never handed out: still free
    with pytest.raises(ValueError):
        pool.free([6])                              # not in the pool
    with pytest.raises(ValueError):
        pool.free([0, 0])


def test_table_grows_with_the_sequence_and_releases_its_blocks():
    pool = paging.BlockPool(10)
    t = paging.BlockTable(2, 4, pool)
    t.ensure(0, 1)                                  # token 0: one block
    t.ensure(1, 128)                                # tokens 0..127: still one block
    t.ensure(0, 129)                                # token 128 opens block 1
    assert t.table.tolist() == [[0, 2, -1, -1], [1, -1, -1, -1]]
    t.ensure(0, 100)                                # shorter: nothing to do
    assert t.n_blocks.tolist() == [2, 1]
    with pytest.raises(ValueError):
        t.ensure(1, 4 * 128 + 1)                    # beyond blocks_per_seq
    t.release(0)
    assert t.table[0].tolist() == [-1] * 4 and pool.n_free == 9
    t.ensure(1, 3 * 128)
    assert t.table[1].tolist() == [1, 0, 2, -1]     # the freed ids come back first
    tt = t.tensor("cpu")
    assert tt.dtype == torch.int32 and tuple(tt.shape) == (2, 4)


@pytest.mark.parametrize("m", [4, 128])
def test_scatter_puts_every_entry_at_its_pool_row(m):
    rng = np.random.default_rng(m)
    epb = paging.entries_per_block(m)
    B, bps = 3, 5
    n_blocks = B * bps + 4
    table = rng.permutation(n_blocks)[: B * bps].reshape(B, bps).astype(np.int32)
    table[2, 3:] = -1                               # sequence 2 holds three blocks only
    rows = torch.from_numpy(rng.standard_normal((B, bps * epb, 6)).astype(np.float32))
    pool = paging.scatter_to_pool(rows, table, m, n_blocks)
    assert tuple(pool.shape) == (n_blocks * epb, 6)
    for b in range(B):
        n_ent = (3 if b == 2 else bps) * epb
        e = np.arange(n_ent)
        r = paging.pool_rows(table, m, b, e)
        assert np.array_equal(r, table[b, e // epb].astype(np.int64) * epb + e % epb)
        assert torch.equal(pool[torch.from_numpy(r)], rows[b, :n_ent])
    # the unused blocks stay zero
    used = set(table[table >= 0].tolist())
    free = [i for i in range(n_blocks) if i not in used]
    assert not pool.view(n_blocks, epb, 6)[free].any()
