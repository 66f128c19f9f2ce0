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


def _merge_main(rank, world, port, out):
    from oracle import indexer as oidx, mqa as omqa
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        rng = np.random.default_rng(11)           # the same draws on every rank
        nq, H, d, N, scale, k = 2, 3, 8, 20, 0.4, 8
        q = rng.standard_normal((nq, H, d))
        keys = rng.standard_normal((N, d))
        sink = rng.standard_normal(H)
        scores = np.round(rng.standard_normal((3, 50)) * 2) / 2   # many exact ties
        # this rank's contiguous slices of the keys and of the score rows
        a, b = cp.chunk_bounds(N, world)[rank]
        parts = [omqa.attend(q[i], keys[a:b], scale, sink if rank == 0 else None)
                 for i in range(nq)]
        o = torch.from_numpy(np.stack([p[0] for p in parts]))
        lse = torch.from_numpy(np.stack([p[1] for p in parts]))
        mo, ml = cp.merge_attention(o, lse, dist)
        sa, sb = cp.chunk_bounds(50, world)[rank]
        loc = [oidx.topk(scores[r, sa:sb], sb - sa, k) for r in range(3)]
        gidx = np.stack([np.where(l >= 0, l + sa, -1) for l in loc])
        gsc = np.stack([np.where(g >= 0, scores[r, np.maximum(g, 0)], -np.inf)
                        for r, g in enumerate(gidx)])
        sel = cp.merge_topk(torch.from_numpy(gsc), torch.from_numpy(gidx), k, dist)
        out[rank] = dict(o=mo.numpy(), lse=ml.numpy(), sel=sel.numpy())
    finally:
        dist.destroy_process_group()


def test_entry_sharded_decode_merges_match_one_process():
    """A history sharded by entries over 3 gloo ranks: the attention parts
    (sink on one rank) merge into the attention over all keys, and the local
    top-k selections (scores with many exact ties) into the global top-k
    (oracle attend / topk on each rank's slice stand in for the GPU calls)."""
    from oracle import indexer as oidx, mqa as omqa
    world = 3
    port = _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_merge_main, args=(world, port, out), nprocs=world, join=True,
                           start_method="spawn")
        res = dict(out)
    rng = np.random.default_rng(11)
    nq, H, d, N, scale, k = 2, 3, 8, 20, 0.4, 8
    q = rng.standard_normal((nq, H, d))
    keys = rng.standard_normal((N, d))
    sink = rng.standard_normal(H)
    scores = np.round(rng.standard_normal((3, 50)) * 2) / 2
    ref = [omqa.attend(q[i], keys, scale, sink) for i in range(nq)]
    ref_sel = np.stack([oidx.topk(scores[r], 50, k) for r in range(3)])
    for r in range(world):
        assert np.allclose(res[r]["o"], np.stack([x[0] for x in ref]), rtol=1e-12, atol=1e-12)
        assert np.allclose(res[r]["lse"], np.stack([x[1] for x in ref]), rtol=1e-12, atol=1e-12)
        assert np.array_equal(res[r]["sel"], ref_sel)
