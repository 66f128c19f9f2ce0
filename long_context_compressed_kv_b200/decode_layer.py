"""Device state of one CSA or HCA layer for decode, and its decode step.

The state follows the split of "DeepSeek-V4 深读" (ricardokevins.github.io),
section "异构 KV cache 与磁盘前缀复用": a fixed-size state per sequence (the
sliding-window ring of raw-token KV and the uncompressed tail of the current
block) next to the compressed caches (main entries and, for CSA, indexer
keys).  Everything here allocates device tensors and marshals them into the
C ABI; all computation runs in libv4attn.
"""
from __future__ import annotations

from typing import Optional

import numpy as np
import torch

from . import (BF16, CSA, E4M3_BF16ROPE, F32, MXFP4, compress, decode, row_bytes, workspace)


def _t(x, dtype=torch.float32, device="cuda"):
    if isinstance(x, torch.Tensor):
        return x.to(device=device, dtype=dtype)
    return torch.from_numpy(np.ascontiguousarray(x)).to(device=device, dtype=dtype)


def code_rows(desc, vals: torch.Tensor, fmt: int, out: torch.Tensor, out_scale,
              first_row: int = 0, stream=None):
    """Store fp32 vectors vals [B, n, c] (device) in ``fmt`` at rows
    first_row .. first_row+n-1 (mod the row count of ``out``), unchanged
    (compress with m = 1, no RMSNorm, no RoPE)."""
    B, n, c = vals.shape
    if n == 0:
        return
    vals = vals.contiguous()
    lens = torch.full((B,), first_row + n, dtype=torch.int64, device=vals.device)
    eb = torch.full((B,), first_row, dtype=torch.int64, device=vals.device)
    compress(desc, m=1, overlap=False, c=c, Ca=vals, Za=None, in_rows=n, in_seq_stride=n * c,
             in_row_stride=c, seq_len=lens, entry_begin=eb, n_entries=n, out_dtype=fmt, out=out,
             out_scale=out_scale, out_rows=out.shape[1], apply_rmsnorm=False, apply_rope=False,
             stream=stream)


def _alloc_rows(B, rows, fmt, c, d_rope, device):
    out = torch.zeros(B, rows, row_bytes(fmt, c, d_rope), dtype=torch.uint8, device=device)
    if fmt == E4M3_BF16ROPE:
        sc = torch.zeros(B, rows, dtype=torch.float32, device=device)
    elif fmt == MXFP4:
        sc = torch.zeros(B, rows, c // 32, dtype=torch.uint8, device=device)
    else:
        sc = None
    return out, sc


class DecodeLayer:
    """Caches, state rings and per-step buffers of one layer for B sequences.

    kv_rows   capacity of the compressed caches (entries 0 .. kv_rows-1);
    swa_rows  rows of the window ring (token t at row t % swa_rows);
    in_dtype  dtype of the raw compressor inputs (float32 or bfloat16).
    """

    def __init__(self, desc, B: int, kv_rows: int, swa_rows: Optional[int] = None,
                 in_dtype=torch.float32, out_dtype=torch.bfloat16, device="cuda"):
        self.desc, self.B, self.device = desc, B, device
        self.csa = desc.kind == CSA
        self.m, self.d, self.d_rope = desc.m, desc.d, desc.d_rope
        self.ring = 2 * desc.m if self.csa else desc.m
        self.n_arr = 4 if self.csa else 2
        # capacity rounded up to whole 128-row tiles (aligned rows for the TMA paths)
        kv_rows = (kv_rows + 127) // 128 * 128
        self.kv_rows = kv_rows
        self.swa_rows = swa_rows or max(desc.n_win, 1)
        self.in_dtype = in_dtype
        self.fmt = desc.kv_dtype
        self.kv, self.kv_scale = _alloc_rows(B, kv_rows, self.fmt, desc.d, desc.d_rope, device)
        self.swa, self.swa_scale = _alloc_rows(B, self.swa_rows, self.fmt, desc.d, desc.d_rope,
                                               device)
        self.tail = torch.zeros(B, self.ring, self.n_arr, desc.d, dtype=in_dtype, device=device)
        self.x_main = torch.zeros(B, self.n_arr, desc.d, dtype=in_dtype, device=device)
        self.bias = torch.zeros(self.ring, desc.d, dtype=torch.float32, device=device)
        self.Q = torch.zeros(B, desc.H, desc.d, dtype=torch.bfloat16, device=device)
        self.sink: Optional[torch.Tensor] = None
        self.pos = torch.zeros(B, dtype=torch.int64, device=device)
        self.out = torch.zeros(B, desc.H, desc.d, dtype=out_dtype, device=device)
        self.lse = torch.zeros(B, desc.H, dtype=torch.float32, device=device)
        if self.csa:
            self.kfmt = desc.idx_dtype
            self.keys, self.keys_sf = _alloc_rows(B, kv_rows, self.kfmt, desc.d_I, 0, device)
            self.itail = torch.zeros(B, self.ring, 4, desc.d_I, dtype=in_dtype, device=device)
            self.x_idx = torch.zeros(B, 4, desc.d_I, dtype=in_dtype, device=device)
            self.ibias = torch.zeros(self.ring, desc.d_I, dtype=torch.float32, device=device)
            self.qI, self.qI_sf = _alloc_rows(1, B * desc.H_I, self.kfmt, desc.d_I, 0, device)
            self.qI = self.qI.reshape(B, desc.H_I, -1)
            self.qI_sf = None if self.qI_sf is None else self.qI_sf.reshape(B, desc.H_I, -1)
            self.w = torch.zeros(B, desc.H_I, dtype=torch.float32, device=device)
            self.idx = torch.full((B, desc.top_k), -1, dtype=torch.int32, device=device)
        self.ws = workspace(desc, B, kv_rows, device=device)

    # ------------------------------------------------------------ loading state
    def load_entries(self, vals, first_entry: int = 0):
        """Store precomputed entry vectors [B, n, d] (fp32) as entries first_entry.."""
        code_rows(self.desc, _t(vals, device=self.device), self.fmt, self.kv, self.kv_scale,
                  first_entry)

    def load_keys(self, vals, first_entry: int = 0):
        """Store precomputed indexer-key vectors [B, n, d_I] (fp32)."""
        code_rows(self.desc, _t(vals, device=self.device), self.kfmt, self.keys, self.keys_sf,
                  first_entry)

    def load_window(self, vals, first_token: int):
        """Store window KV vectors [B, n, d] of tokens first_token .. (ring rows)."""
        vals = _t(vals, device=self.device)
        n = vals.shape[1]
        for start in range(0, n, self.swa_rows):
            chunk = vals[:, start:start + self.swa_rows]
            t0 = first_token + start
            # rows t % swa_rows for t = t0 .. t0+len-1, split at the ring wrap
            r0 = t0 % self.swa_rows
            k = min(chunk.shape[1], self.swa_rows - r0)
            code_rows(self.desc, chunk[:, :k], self.fmt, self.swa, self.swa_scale, r0)
            if k < chunk.shape[1]:
                code_rows(self.desc, chunk[:, k:], self.fmt, self.swa, self.swa_scale, 0)

    def load_tail(self, arrays, first_token: int, itail_arrays=None):
        """Raw compressor inputs of tokens first_token .. into the tail rings:
        arrays [B, n, n_arr, d] (order Ca, Za, Cb, Zb for CSA; C, Z for HCA)."""
        arrays = _t(arrays, self.in_dtype, self.device)
        for j in range(arrays.shape[1]):
            self.tail[:, (first_token + j) % self.ring] = arrays[:, j]
        if itail_arrays is not None:
            it = _t(itail_arrays, self.in_dtype, self.device)
            for j in range(it.shape[1]):
                self.itail[:, (first_token + j) % self.ring] = it[:, j]

    def set_index_query(self, qI_vals):
        """Indexer queries [B, H_I, d_I] (fp32) -> the indexer's stored format."""
        v = _t(qI_vals, device=self.device).reshape(1, -1, self.desc.d_I)
        rows = self.qI.reshape(1, v.shape[1], -1)
        sf = None if self.qI_sf is None else self.qI_sf.reshape(1, v.shape[1], -1)
        code_rows(self.desc, v, self.kfmt, rows, sf, 0)

    # ------------------------------------------------------------ the step
    def step(self, max_vis: int, stream=None):
        """One decode step: new token self.x_main (+ self.x_idx) at self.pos."""
        kw = {}
        if self.csa:
            kw = dict(x_idx=self.x_idx, itail=self.itail, ibias=self.ibias, keys=self.keys,
                      keys_sf=self.keys_sf, key_rows=self.kv_rows, qI=self.qI, qI_sf=self.qI_sf,
                      w=self.w, idx_out=self.idx)
        decode(self.desc, pos=self.pos, x_main=self.x_main, tail=self.tail, bias=self.bias,
               kv=self.kv, kv_scale=self.kv_scale, kv_rows=self.kv_rows, swa=self.swa,
               swa_scale=self.swa_scale, swa_rows=self.swa_rows, Q=self.Q, out=self.out,
               ws=self.ws, max_vis=max_vis, sink=self.sink, lse=self.lse, stream=stream, **kw)
