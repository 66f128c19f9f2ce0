"""Seeded synthetic inputs for the compressed-attention hot path.

This module only draws random numbers and lays them out in the shapes of the
workloads.  It holds none of the method's arithmetic: no pooling, no
normalisation, no RoPE, no quantisation and no projection.  The CPU oracle
(``oracle/``) and the CUDA path (``long_context_compressed_kv_b200``) both
consume exactly the arrays returned here and nothing else is shared between
them.

Every array is drawn from a counter-based Philox-4x64 stream (Salmon et al.,
"Parallel random numbers: as easy as 1, 2, 3", SC'11; numpy's
``np.random.Philox``) keyed by ``(seed, crc32(name), block)``, so any block of
rows can be regenerated on its own, in any order, on any machine.

The workload recipes (``workload(...)``) follow the five layer shapes of the
pages: a tiny fp32 CSA layer, HCA and CSA decode at the V4-Flash layer shape
at 128K context, a V4-Pro CSA+HCA pair at 1M context, and a chunked prefill of
a V4-Flash CSA+HCA pair.  Their statistics (N(0,1) token activations and
queries, Xavier projections, N(0,0.1) position biases, N(0,1) sink logits,
U(0,1) indexer head weights) are the ones those shapes are stated with.
"""
from __future__ import annotations

import dataclasses
import zlib
from typing import Optional

import numpy as np

ROWS_PER_BLOCK = 256


def _rng(seed: int, name: str, block: int = 0) -> np.random.Generator:
    key = (int(seed) & 0xFFFFFFFF) << 32 | zlib.crc32(name.encode())
    bitgen = np.random.Philox(key=[key, int(block)])
    return np.random.Generator(bitgen)


def _blocked(seed, name, shape, draw, rows: Optional[np.ndarray] = None):
    """Draw ``shape`` row-blockwise; ``rows`` selects leading-axis rows only."""
    shape = tuple(int(s) for s in shape)
    lead = shape[0]
    inner = shape[1:]
    if rows is None:
        out = np.empty(shape, dtype=np.float32)
        for blk in range((lead + ROWS_PER_BLOCK - 1) // ROWS_PER_BLOCK):
            r0 = blk * ROWS_PER_BLOCK
            r1 = min(lead, r0 + ROWS_PER_BLOCK)
            vals = draw(_rng(seed, name, blk), (ROWS_PER_BLOCK,) + inner)
            out[r0:r1] = vals[: r1 - r0]
        return out
    rows = np.asarray(rows, dtype=np.int64)
    out = np.empty((len(rows),) + inner, dtype=np.float32)
    cache = {}
    for i, r in enumerate(rows):
        blk = int(r) // ROWS_PER_BLOCK
        if blk not in cache:
            cache[blk] = draw(_rng(seed, name, blk), (ROWS_PER_BLOCK,) + inner)
        out[i] = cache[blk][int(r) % ROWS_PER_BLOCK]
    return out


def normal(seed, name, shape, std=1.0, rows=None) -> np.ndarray:
    """float32 N(0, std^2)."""
    return _blocked(seed, name, shape,
                    lambda g, s: (g.standard_normal(s, dtype=np.float32) * np.float32(std)),
                    rows)


def uniform(seed, name, shape, lo=0.0, hi=1.0, rows=None) -> np.ndarray:
    """float32 U(lo, hi)."""
    return _blocked(seed, name, shape,
                    lambda g, s: g.uniform(lo, hi, s).astype(np.float32), rows)


def xavier(seed, name, fan_in, fan_out) -> np.ndarray:
    """float32 [fan_in, fan_out] Xavier-normal weights, std sqrt(2/(in+out))."""
    return normal(seed, name, (fan_in, fan_out), std=float(np.sqrt(2.0 / (fan_in + fan_out))))


def bf16_values(x: np.ndarray) -> np.ndarray:
    """Round float32 data to bfloat16 with torch (an input-format step).

    Returns float32 holding bf16-representable values, so both sides read the
    same numbers whether they take the array as float32 or as bf16."""
    import torch
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16).to(
        torch.float32).numpy()


# ---------------------------------------------------------------------------
# workload recipes
# ---------------------------------------------------------------------------

@dataclasses.dataclass(frozen=True)
class Layer:
    """Shape of one attention layer (kind, ratio, heads, dims)."""
    kind: str            # "csa" (overlapped windows of 2m) or "hca" (windows of m)
    m: int               # compression ratio
    H: int               # query heads
    d: int               # head / entry dim
    d_rope: int          # RoPE dims at the end of d
    n_win: int = 128     # sliding window of raw tokens
    H_I: int = 0         # indexer heads (csa)
    d_I: int = 0         # indexer dim (csa)
    top_k: int = 0       # selected entries per query (csa)
    kv_fp8: bool = True  # FP8 e4m3 nope dims + BF16 rope dims; else fp32
    idx_fp4: bool = True  # MXFP4 indexer keys and queries; else fp32
    rope_theta: float = 160000.0


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    seed: int
    B: int
    L: int                      # context length (tokens 0..L-1); decode query at L-1
    layers: tuple               # of Layer
    d_model: int = 0            # raw-token width where a projection is part of the step
    n_queries: int = 0          # multi-query (tiny / prefill) workloads
    prefix: int = 0             # prefill: tokens already in the caches
    low_rank: int = 0           # tiny config: indexer query rank


FLASH_CSA = Layer("csa", 4, 64, 512, 64, 128, 64, 128, 512)
FLASH_HCA = Layer("hca", 128, 64, 512, 64, 128)
PRO_CSA = Layer("csa", 4, 128, 512, 64, 128, 64, 128, 1024)
PRO_HCA = Layer("hca", 128, 128, 512, 64, 128)
TINY_CSA = Layer("csa", 4, 16, 128, 32, 128, 4, 32, 64, kv_fp8=False, idx_fp4=False)

WORKLOADS = {
    # 1: tiny CSA layer, fp32 throughout, 32 decode queries at L-32..L-1
    "tiny_csa_fp32": Workload("tiny_csa_fp32", 0, 1, 8192, (TINY_CSA,), d_model=256,
                              n_queries=32, low_rank=64),
    # 2: HCA decode, V4-Flash layer shape, B=16 at 128K
    "hca_flash_128k": Workload("hca_flash_128k", 1, 16, 131072, (FLASH_HCA,)),
    # 3: CSA decode, V4-Flash layer shape, B=32 at 128K
    "csa_flash_128k": Workload("csa_flash_128k", 2, 32, 131072, (FLASH_CSA,)),
    # 4: V4-Pro CSA + HCA pair, B=4 at 1M
    "pro_pair_1m": Workload("pro_pair_1m", 3, 4, 1048576, (PRO_CSA, PRO_HCA)),
    # 5: chunked prefill of a V4-Flash CSA + HCA pair: 65536 new on a 65536 prefix
    "flash_prefill_64k": Workload("flash_prefill_64k", 4, 1, 131072, (FLASH_CSA, FLASH_HCA),
                                  d_model=4096, n_queries=65536, prefix=65536),
}


def scaled(w: Workload, B=None, L=None, top_k=None, H=None, n_queries=None, prefix=None,
           name=None) -> Workload:
    """Same recipe at a smaller size (parity cases the oracle finishes in seconds)."""
    layers = []
    for ly in w.layers:
        ly2 = ly
        if top_k is not None and ly.kind == "csa":
            ly2 = dataclasses.replace(ly2, top_k=top_k)
        if H is not None:
            ly2 = dataclasses.replace(ly2, H=H)
        layers.append(ly2)
    return dataclasses.replace(
        w, name=name or (w.name + "_scaled"), B=B or w.B, L=L or w.L, layers=tuple(layers),
        n_queries=n_queries if n_queries is not None else w.n_queries,
        prefix=prefix if prefix is not None else w.prefix)


def decode_layer_inputs(w: Workload, li: int) -> dict:
    """Inputs of one decode step (query at p = L-1 in every sequence) of layer ``li``.

    The history before the step is synthetic: every stored compressed entry
    and every SWA token entry is an N(0,1) vector per dim (unit RMS, as after
    RMSNorm), every indexer key and indexer query row is N(0,1) before MXFP4
    coding.  The raw compressor inputs of the incomplete block (the tail) and
    of the new token are N(0,1) values and N(0,1) gate logits; the position
    bias is N(0, 0.1).  Queries are N(0,1) (unit RMS per head, as after the
    per-head RMSNorm) rounded to bf16; sink logits are N(0,1); indexer head
    weights are U(0,1).
    """
    ly = w.layers[li]
    s = w.seed * 16 + li
    B, L, m = w.B, w.L, ly.m
    p = L - 1
    n_hist = (L // m) - 1 if (L % m == 0) else (L // m)
    ring = 2 * m if ly.kind == "csa" else m
    nb = 4 if ly.kind == "csa" else 2  # raw arrays per compressor (Ca,Za,Cb,Zb) or (C,Z)
    out = dict(p=p, n_hist=n_hist, ring=ring)
    out["hist_entries"] = normal(s, "hist_entries", (B * n_hist, ly.d)).reshape(B, n_hist, ly.d)
    out["swa_hist"] = normal(s, "swa_hist", (B * (ly.n_win - 1), ly.d)).reshape(
        B, ly.n_win - 1, ly.d)
    names = ["Ca", "Za", "Cb", "Zb"][:nb] if ly.kind == "csa" else ["C", "Z"]
    # tail: raw tokens p-ring+1 .. p-1 (ring-1 of them) + the new token p
    for nm in names:
        out["tail_" + nm] = normal(s, "tail_" + nm, (B * ring, ly.d)).reshape(B, ring, ly.d)
    bias_rows = 2 * m if ly.kind == "csa" else m
    out["bias"] = normal(s, "bias", (bias_rows, ly.d), std=0.1)
    out["Q"] = bf16_values(normal(s, "Q", (B * ly.H, ly.d))).reshape(B, ly.H, ly.d)
    out["sink"] = normal(s, "sink", (ly.H,))
    if ly.kind == "csa":
        out["hist_keys"] = normal(s, "hist_keys", (B * n_hist, ly.d_I)).reshape(B, n_hist, ly.d_I)
        for nm in names:
            out["itail_" + nm] = normal(s, "itail_" + nm, (B * ring, ly.d_I)).reshape(
                B, ring, ly.d_I)
        out["ibias"] = normal(s, "ibias", (bias_rows, ly.d_I), std=0.1)
        out["qI"] = normal(s, "qI", (B * ly.H_I, ly.d_I)).reshape(B, ly.H_I, ly.d_I)
        out["w"] = uniform(s, "w", (B, ly.H_I))
    return out


def tiny_inputs(w: Workload) -> dict:
    """Inputs of the tiny fp32 CSA layer: raw tokens and projection weights."""
    ly = w.layers[0]
    s = w.seed
    dm = w.d_model
    out = dict(
        x=normal(s, "x", (w.L, dm)),
        W_kv=xavier(s, "W_kv", dm, ly.d),
        W_z=xavier(s, "W_z", dm, ly.d),
        bias=normal(s, "bias", (2 * ly.m, ly.d), std=0.1),
        W_kvI=xavier(s, "W_kvI", dm, ly.d_I),
        W_zI=xavier(s, "W_zI", dm, ly.d_I),
        ibias=normal(s, "ibias", (2 * ly.m, ly.d_I), std=0.1),
        W_dq=xavier(s, "W_dq", dm, w.low_rank),
        W_uq=xavier(s, "W_uq", w.low_rank, ly.H_I * ly.d_I),
        W_w=xavier(s, "W_w", dm, ly.H_I),
        W_q=xavier(s, "W_q", dm, ly.H * ly.d),
        sink=normal(s, "sink", (ly.H,)),
    )
    out["positions"] = np.arange(w.L - w.n_queries, w.L, dtype=np.int64)
    return out


PREFILL_CSA_COLS = ("Ca", "Cb", "Za", "Zb")
PREFILL_IDX_COLS = ("ICa", "ICb", "IZa", "IZb")
PREFILL_HCA_COLS = ("C", "Z")


def prefill_weight(w: Workload) -> np.ndarray:
    """bf16-valued [d_model, 4*512 + 4*128 + 2*512] projection of the prefill pair."""
    csa, hca = w.layers
    ncol = 4 * csa.d + 4 * csa.d_I + 2 * hca.d
    return bf16_values(xavier(w.seed, "W_proj", w.d_model, ncol))


def prefill_x(w: Workload, rows=None) -> np.ndarray:
    """bf16-valued raw tokens x [L, d_model] ~ N(0,1) (or only ``rows``)."""
    return bf16_values(normal(w.seed, "x", (w.L, w.d_model), rows=rows))


def prefill_queries(w: Workload, li: int, rows=None) -> dict:
    """Per-query inputs of prefill layer ``li`` for query rows (0..n_queries-1)."""
    ly = w.layers[li]
    s = w.seed * 16 + li
    n = w.n_queries
    out = dict(
        Q=bf16_values(normal(s, "Q", (n, ly.H * ly.d), rows=rows)).reshape(-1, ly.H, ly.d),
        sink=normal(s, "sink", (ly.H,)),
    )
    if ly.kind == "csa":
        out["qI"] = normal(s, "qI", (n, ly.H_I * ly.d_I), rows=rows).reshape(-1, ly.H_I, ly.d_I)
        out["w"] = uniform(s, "w", (n, ly.H_I), rows=rows)
    out["bias"] = normal(s, "bias", (2 * ly.m if ly.kind == "csa" else ly.m, ly.d), std=0.1)
    if ly.kind == "csa":
        out["ibias"] = normal(s, "ibias", (2 * ly.m, ly.d_I), std=0.1)
    return out
