"""Context-parallel compression layout on CPU gloo ranks ([deep-read]
"上下文并行必须理解压缩边界"): a sequence split over 3 ranks at chunk edges
that cut through compression blocks, the boundary exchange of raw rows, each
rank compressing the entries it owns, and the all-gather with select-and-pad
must give exactly the single-process compression of the whole sequence, for
CSA (m = 4, half-overlapping windows) and HCA (m = 128), with a partial last
block.  The oracle's pooling stands in for the GPU compression here (this is
a test of the data layout, which is the same code on NCCL and GPU tensors)."""
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from long_context_compressed_kv_b200 import cp

CASES = [(4, True, 1003), (128, False, 1003), (4, True, 48)]


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(m, overlap, L, c=8):
    rng = np.random.default_rng(m + L)
    arrs = {k: rng.standard_normal((L, c)) for k in (["Ca", "Za", "Cb", "Zb"] if overlap else ["Ca", "Za"])}
    bias = rng.standard_normal((2 * m if overlap else m, c)) * 0.1
    return arrs, bias


def _pool(entries, m, overlap, L, arrs, bias, base, n_rows):
    from oracle import compress as ocomp
    def f(name):
        a = arrs[name]
        return lambda t: a[np.clip(t - base, 0, n_rows - 1)]
    kw = dict(Cb=f("Cb"), Zb=f("Zb")) if overlap else {}
    return ocomp.pool(np.asarray(entries), m, overlap, L, f("Ca"), f("Za"), bias, **kw)


def _rank_main(rank, world, port, out):
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        res = {}
        for m, overlap, L in CASES:
            arrs, bias = _inputs(m, overlap, L)
            bounds = cp.chunk_bounds(L, world)
            if min(e - s for s, e in bounds[:-1]) < cp.tail_rows(m, overlap):
                continue                                   # too short to split this way
            cp.check_chunks(bounds, m, overlap)
            s, e = bounds[rank]
            n = cp.tail_rows(m, overlap)
            local = torch.from_numpy(np.stack([arrs[k][s:e] for k in sorted(arrs)], 1))
            prev = cp.boundary_exchange(local, n, dist)
            ext = torch.cat([prev, local], 0).numpy()     # rows of tokens s - n .. e - 1
            ext_arrs = {k: ext[:, j] for j, k in enumerate(sorted(arrs))}
            i0, i1 = cp.owned_entries(s, e, L, m)
            ent = _pool(np.arange(i0, i1), m, overlap, L, ext_arrs, bias, s - n, ext.shape[0])
            max_n = max(cp.owned_entries(a, b, L, m)[1] - cp.owned_entries(a, b, L, m)[0]
                        for a, b in bounds)
            full = cp.gather_entries(torch.from_numpy(np.ascontiguousarray(ent)).reshape(
                i1 - i0, -1), i1 - i0, max_n, dist)
            res[(m, overlap, L)] = full.numpy()
        out[rank] = res
    finally:
        dist.destroy_process_group()


def test_chunk_bounds_and_ownership_cover_every_entry_once():
    for m, L, world in [(4, 1003, 3), (128, 1003, 3), (4, 16, 2), (128, 256, 2), (4, 7, 1)]:
        bounds = cp.chunk_bounds(L, world)
        assert bounds[0][0] == 0 and bounds[-1][1] == L
        assert all(a[1] == b[0] for a, b in zip(bounds, bounds[1:]))
        owned = [cp.owned_entries(s, e, L, m) for s, e in bounds]
        got = [i for i0, i1 in owned for i in range(i0, i1)]
        assert got == list(range(-(-L // m)))
        for (s, e), (i0, i1) in zip(bounds, owned):
            for i in range(i0, i1):          # a complete block ends in the range
                assert s <= min(m * (i + 1) - 1, L - 1) < e


def test_three_gloo_ranks_compress_like_one_process():
    world = 3
    port = _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_rank_main, args=(world, port, out), nprocs=world, join=True,
                           start_method="spawn")
        res = dict(out)
    assert sorted(res) == [0, 1, 2]
    checked = 0
    for m, overlap, L in CASES:
        key = (m, overlap, L)
        if key not in res[0]:
            continue
        arrs, bias = _inputs(m, overlap, L)
        n_ent = -(-L // m)
        ref = _pool(np.arange(n_ent), m, overlap, L, arrs, bias, 0, L)
        for r in range(world):               # every rank holds the whole sequence's entries
            assert np.array_equal(res[r][key], ref)
        checked += 1
    assert checked >= 2
