"""Context parallelism for the compression step: the data layout across ranks.

[deep-read] "上下文并行必须理解压缩边界": context parallelism gives every
rank a contiguous run of a sequence's tokens, but a compression block of m
tokens (4 for CSA, 128 for HCA) can straddle two ranks and a packed
sequence's tail can fall short of a block.  The page's remedy is two
communication stages: each rank first sends its last raw KV rows to the next
rank so that the blocks at its boundary can be completed, then the ranks
all-gather their local compressed entries at a fixed length and select the
valid ones (select-and-pad).

Here (all collectives are ``torch.distributed`` calls, so the same code runs
over NCCL on GPU tensors and over gloo on CPU ones):

* ``chunk_bounds`` - the contiguous token range of each rank;
* ``owned_entries`` - the entries a rank produces: those whose block ends in
  its range (entry i's block ends at token m (i + 1) - 1), and on the last rank
  also the partial block at the sequence's end;
* ``tail_rows`` - how many raw rows a rank needs from its predecessor: the
  window of its first owned entry reaches back at most m - 1 tokens (HCA) or
  2 m - 1 (CSA, whose windows overlap the previous block by m); sending the
  last ring = m (HCA) or 2 m (CSA) rows, the size of the per-sequence tail
  ring, covers both, and for chunk starts on block edges the CSA case needs
  exactly the page's m rows of the previous block;
* ``boundary_exchange`` - stage one: rank r's last ``n`` rows to rank r + 1;
* ``gather_entries`` - stage two: every rank's entries, padded to one length,
  all-gathered, and the valid rows concatenated in rank (= entry) order.

Between the two stages each rank compresses its owned entries
(``v4attn_compress``) over its predecessor's tail rows followed by its own
rows, reading absolute token t at row t - (start - n_tail).

For decode over a history sharded by entries (each rank holding a contiguous
slice of a sequence's compressed entries and indexer keys) two merges close
the step:

* ``merge_topk`` - every rank's k best (score, global index) pairs of its
  slice merged into the sequence's k best (higher score first, ties to the
  lower index, ascending output, -1 padding): each global winner is among
  its own slice's k best, so the union of the local selections holds them;
* ``merge_attention`` - the attention of the same queries over the ranks'
  disjoint key sets (each normalised over its own keys, with its log
  denominator; the sink counted on one rank only) merged into the attention
  over their union: LSE = log sum_r exp(lse_r), o = sum_r exp(lse_r - LSE) o_r.
"""
from __future__ import annotations

from typing import List, Tuple

import torch


def chunk_bounds(L: int, world: int) -> List[Tuple[int, int]]:
    """[start, end) token range of every rank: L tokens split as evenly as
    possible, earlier ranks one longer when L is not divisible."""
    if world < 1 or L < 0:
        raise ValueError("bad world size or length")
    q, r = divmod(L, world)
    out, s = [], 0
    for k in range(world):
        e = s + q + (1 if k < r else 0)
        out.append((s, e))
        s = e
    return out


def owned_entries(start: int, end: int, L: int, m: int) -> Tuple[int, int]:
    """[i0, i1): the entries the rank holding tokens [start, end) produces -
    those whose block's last token m (i + 1) - 1 lies in the range, plus the
    sequence's partial last block (entry ceil(L / m) - 1 when m does not divide
    L) on the rank that holds token L - 1."""
    i0 = start // m                                         # first i with m(i+1)-1 >= start
    i1 = end // m                                           # first i with m(i+1)-1 >= end
    if end == L and L % m:
        i1 = -(-L // m)
    return i0, max(i0, i1)


def tail_rows(m: int, overlap: bool) -> int:
    """Raw rows a rank sends its successor: the tail ring's size."""
    return 2 * m if overlap else m


def check_chunks(bounds: List[Tuple[int, int]], m: int, overlap: bool) -> None:
    """Every rank after the first must hold at least the rows its successor
    needs from it (else a window would reach two ranks back)."""
    need = tail_rows(m, overlap)
    for k, (s, e) in enumerate(bounds[:-1]):
        if e - s < need:
            raise ValueError(f"rank {k} holds {e - s} tokens, fewer than the {need} its "
                             f"successor's boundary window needs")


def boundary_exchange(x_local: torch.Tensor, n: int, dist, group=None) -> torch.Tensor:
    """Stage one: send the last ``n`` rows of this rank's raw rows [rows, ...]
    to the next rank and receive the previous rank's; rank 0 gets zeros (no
    token precedes it; its windows' missing rows are left out of the softmax)."""
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    if x_local.shape[0] < n and rank < world - 1:
        raise ValueError("a rank holds fewer rows than its successor needs")
    prev = torch.zeros((n,) + tuple(x_local.shape[1:]), dtype=x_local.dtype,
                       device=x_local.device)
    ops = []
    if rank + 1 < world:
        ops.append(dist.P2POp(dist.isend, x_local[-n:].contiguous(),
                              dist.get_global_rank(group, rank + 1) if group else rank + 1,
                              group))
    if rank > 0:
        ops.append(dist.P2POp(dist.irecv, prev,
                              dist.get_global_rank(group, rank - 1) if group else rank - 1,
                              group))
    if ops:
        for req in dist.batch_isend_irecv(ops):
            req.wait()
    return prev


def gather_entries(local: torch.Tensor, n_valid: int, max_n: int, dist,
                   group=None) -> torch.Tensor:
    """Stage two: every rank's first ``n_valid`` rows of ``local`` [>= n_valid, ...]
    padded to ``max_n`` rows, all-gathered, and the valid rows of every rank
    concatenated in rank order (select-and-pad): the compressed entries of the
    whole sequence, entry i at row i."""
    world = dist.get_world_size(group)
    if n_valid > max_n:
        raise ValueError("more valid entries than the fixed length")
    rest = tuple(local.shape[1:])
    pad = torch.zeros((max_n,) + rest, dtype=local.dtype, device=local.device)
    pad[:n_valid] = local[:n_valid]
    counts = torch.tensor([n_valid], dtype=torch.int64, device=local.device)
    all_counts = [torch.zeros_like(counts) for _ in range(world)]
    dist.all_gather(all_counts, counts, group=group)
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad, group=group)
    return torch.cat([p[: int(c.item())] for p, c in zip(parts, all_counts)], 0)


def merge_topk(scores: torch.Tensor, idx: torch.Tensor, k: int, dist, group=None) -> torch.Tensor:
    """Global top-k from every rank's local selection.  scores [nq, kl] and
    idx [nq, kl] (int64 global entry indices, -1 for no entry) hold a rank's
    kl >= min(k, slice) best entries per query; returns int64 [nq, k]: the k
    best over all ranks, higher score first with ties to the lower index,
    in ascending index order, -1 padded (every rank gets it)."""
    world = dist.get_world_size(group)
    s_all = [torch.empty_like(scores) for _ in range(world)]
    i_all = [torch.empty_like(idx) for _ in range(world)]
    dist.all_gather(s_all, scores.contiguous(), group=group)
    dist.all_gather(i_all, idx.contiguous(), group=group)
    s = torch.cat(s_all, 1).to(torch.float64)
    i = torch.cat(i_all, 1)
    s = torch.where(i >= 0, s, torch.full_like(s, float("-inf")))
    out = torch.full((s.shape[0], k), -1, dtype=torch.int64, device=s.device)
    for q in range(s.shape[0]):
        valid = i[q] >= 0
        sq, iq = s[q][valid], i[q][valid]
        # by score descending, then by index ascending (a stable two-key sort)
        o1 = torch.argsort(iq, stable=True)
        o2 = torch.argsort(-sq[o1], stable=True)
        chosen = torch.sort(iq[o1][o2][:k]).values
        out[q, : chosen.numel()] = chosen
    return out


def merge_attention(o: torch.Tensor, lse: torch.Tensor, dist, group=None):
    """Attention over the union of the ranks' disjoint key sets from each
    rank's part: o [..., H, d] normalised over the rank's keys (zero for a
    rank with none), lse [..., H] the log of its denominator (-inf for none).
    Returns (o, lse) of the union (every rank gets them)."""
    world = dist.get_world_size(group)
    o_all = [torch.empty_like(o) for _ in range(world)]
    l_all = [torch.empty_like(lse) for _ in range(world)]
    dist.all_gather(o_all, o.contiguous(), group=group)
    dist.all_gather(l_all, lse.contiguous(), group=group)
    L = torch.stack(l_all, 0)                                  # [R, ..., H]
    top = torch.amax(L, 0)
    top = torch.where(torch.isfinite(top), top, torch.zeros_like(top))
    w = torch.exp(L - top)                                     # exp(-inf) = 0
    den = w.sum(0)
    lse_all = torch.log(den) + top
    frac = torch.where(den > 0, w / den, torch.zeros_like(w))
    out = sum(frac[r].unsqueeze(-1) * o_all[r] for r in range(world))
    return out, lse_all
