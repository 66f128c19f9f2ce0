#!/usr/bin/env python
"""Decode throughput of DeepSeek-V4 CSA/HCA attention layers on B200.

One step = one decode step (one new token per sequence) through every layer
of the workload: new-token append + block compression, indexer + top-k (CSA),
MQA over selected / all entries + window + sink, split-K combine.  The
default workload is the V4-Pro CSA + HCA layer pair at 1M context, batch 4
(every decode step of the hot path); the Flash 128K HCA and CSA layers are
reported beside it under "also".

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

N > 1 runs as one process per GPU (torchrun); sequences are independent, so
every rank decodes its own batch (weak scaling, no collective on the data
path); the time is the max over ranks.  One JSON line is printed by rank 0.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

HEADLINE = "pro_pair_1m"
ALSO = ("hca_flash_128k", "csa_flash_128k")
METRIC = "CSA/HCA layer decode queries/s at 128K & 1M ctx; % of HBM/FP4-TC roofline"
L2_BYTES = 126 * 1024 * 1024
FLUSH_BYTES = 320 * 1024 * 1024


# ------------------------------------------------------------------ state from synthetic inputs

def desc_for(ly):
    import long_context_compressed_kv_b200 as v
    return v.layer_desc(v.CSA if ly.kind == "csa" else v.HCA, ly.m, ly.H, ly.d, ly.d_rope,
                        n_win=ly.n_win, rope_theta=ly.rope_theta, H_I=ly.H_I, d_I=ly.d_I,
                        top_k=ly.top_k, kv_dtype=v.E4M3_BF16ROPE if ly.kv_fp8 else v.F32,
                        idx_dtype=v.MXFP4 if ly.idx_fp4 else v.F32)


def build_decode_layer(w, li, inp, in_dtype=None, out_dtype=None):
    """A DecodeLayer holding the coded synthetic history of ``synth.decode_layer_inputs``
    and the new token's inputs, ready for ``step``."""
    import torch
    from long_context_compressed_kv_b200.decode_layer import DecodeLayer
    ly = w.layers[li]
    p, ring = inp["p"], inp["ring"]
    lay = DecodeLayer(desc_for(ly), w.B, kv_rows=inp["n_hist"] + 1, swa_rows=ly.n_win,
                      in_dtype=in_dtype or torch.float32, out_dtype=out_dtype or torch.bfloat16)
    lay.load_entries(inp["hist_entries"])
    lay.load_window(inp["swa_hist"], first_token=p - (ly.n_win - 1))
    names = ["Ca", "Za", "Cb", "Zb"] if ly.kind == "csa" else ["C", "Z"]
    tail = np.stack([inp["tail_" + nm][:, : ring - 1] for nm in names], 2)
    itail = None
    if ly.kind == "csa":
        itail = np.stack([inp["itail_" + nm][:, : ring - 1] for nm in names], 2)
    lay.load_tail(tail, p - ring + 1, itail)
    lay.x_main.copy_(torch.from_numpy(np.stack([inp["tail_" + nm][:, ring - 1] for nm in names], 1)))
    lay.bias.copy_(torch.from_numpy(inp["bias"]))
    lay.Q.copy_(torch.from_numpy(inp["Q"]))
    lay.sink = torch.from_numpy(inp["sink"]).cuda()
    lay.pos.fill_(p)
    if ly.kind == "csa":
        lay.load_keys(inp["hist_keys"])
        lay.x_idx.copy_(torch.from_numpy(
            np.stack([inp["itail_" + nm][:, ring - 1] for nm in names], 1)))
        lay.ibias.copy_(torch.from_numpy(inp["ibias"]))
        lay.set_index_query(inp["qI"])
        lay.w.copy_(torch.from_numpy(inp["w"]))
    lay.max_vis = (p + 1) // ly.m
    return lay


class PrefillPair:
    """Chunked prefill of a CSA + HCA layer pair (one sequence): ``w.n_queries``
    new tokens on a prefix of ``w.prefix`` tokens.  ``prefix_state()`` builds
    the caches of the prefix (untimed); ``step()`` is the timed chunk: the
    projection of the new tokens' raw activations into every compressor input
    (one GEMM), the CSA entries, CSA indexer keys and HCA entries their blocks
    complete, every new token's window KV in both layers, then for every new
    token the indexer + top-k, the sparse MQA (CSA) and the dense MQA (HCA).
    Every device buffer is allocated here; every computation runs in the
    library."""

    CHUNK = 4096                       # host-side generation chunk (rows)

    def __init__(self, w, out_dtype=None):
        import torch
        import long_context_compressed_kv_b200 as v
        self.v, self.w = v, w
        csa, hca = w.layers
        self.csa, self.hca = csa, hca
        L, P, n = w.L, w.prefix, w.n_queries
        assert P + n == L
        # projection columns: CSA (Ca, Cb, Za, Zb), CSA indexer (ICa, ICb, IZa, IZb), HCA (C, Z)
        names = list(synth.PREFILL_CSA_COLS) + list(synth.PREFILL_IDX_COLS) + \
            list(synth.PREFILL_HCA_COLS)
        widths = [csa.d] * 4 + [csa.d_I] * 4 + [hca.d] * 2
        self.cols, c0 = {}, 0
        for nm, wd in zip(names, widths):
            self.cols[nm] = (c0, c0 + wd)
            c0 += wd
        self.ncol = c0
        dev = "cuda"
        self.x = torch.empty(L, w.d_model, dtype=torch.bfloat16, device=dev)
        for r0 in range(0, L, self.CHUNK):
            rows = np.arange(r0, min(L, r0 + self.CHUNK))
            self.x[r0:r0 + len(rows)] = torch.from_numpy(synth.prefill_x(w, rows)).to(dev)
        self.W = torch.from_numpy(synth.prefill_weight(w)).to(dev).to(torch.bfloat16)
        self.Y = torch.empty(L, self.ncol, dtype=torch.float32, device=dev)
        self.dc, self.dh = desc_for(csa), desc_for(hca)
        self.rows_c = (L // csa.m + 127) // 128 * 128
        self.rows_h = max(128, (L // hca.m + 127) // 128 * 128)

        def rows_of(fmt, c, nr, d_rope=64):
            out = torch.zeros(1, nr, v.row_bytes(fmt, c, d_rope), dtype=torch.uint8, device=dev)
            sc = (torch.zeros(1, nr, dtype=torch.float32, device=dev) if fmt == v.E4M3_BF16ROPE
                  else torch.zeros(1, nr, c // 32, dtype=torch.uint8, device=dev))
            return out, sc
        self.kv_c, self.kvs_c = rows_of(v.E4M3_BF16ROPE, csa.d, self.rows_c)
        self.keys, self.keys_sf = rows_of(v.MXFP4, csa.d_I, self.rows_c, 0)
        self.kv_h, self.kvs_h = rows_of(v.E4M3_BF16ROPE, hca.d, self.rows_h)
        # window KV of every token (token t at row t)
        self.swa_c, self.swas_c = rows_of(v.E4M3_BF16ROPE, csa.d, L)
        self.swa_h, self.swas_h = rows_of(v.E4M3_BF16ROPE, hca.d, L)
        # per-query inputs of the new tokens
        self.Q_c = torch.empty(n, csa.H, csa.d, dtype=torch.bfloat16, device=dev)
        self.Q_h = torch.empty(n, hca.H, hca.d, dtype=torch.bfloat16, device=dev)
        self.qI = torch.zeros(n, csa.H_I, csa.d_I // 2, dtype=torch.uint8, device=dev)
        self.qI_sf = torch.zeros(n, csa.H_I, csa.d_I // 32, dtype=torch.uint8, device=dev)
        self.wI = torch.empty(n, csa.H_I, dtype=torch.float32, device=dev)
        for r0 in range(0, n, self.CHUNK):
            rows = np.arange(r0, min(n, r0 + self.CHUNK))
            q0 = synth.prefill_queries(w, 0, rows=rows)
            q1 = synth.prefill_queries(w, 1, rows=rows)
            sl = slice(r0, r0 + len(rows))
            self.Q_c[sl] = torch.from_numpy(q0["Q"]).to(dev)
            self.Q_h[sl] = torch.from_numpy(q1["Q"]).to(dev)
            self.wI[sl] = torch.from_numpy(q0["w"]).to(dev)
            vals = torch.from_numpy(q0["qI"]).to(dev).reshape(1, -1, csa.d_I)
            qrows = self.qI[sl].reshape(1, -1, csa.d_I // 2)
            qsf = self.qI_sf[sl].reshape(1, -1, csa.d_I // 32)
            from long_context_compressed_kv_b200.decode_layer import code_rows as _code_rows
            _code_rows(self.dc, vals, v.MXFP4, qrows, qsf, 0)
            self.qI[sl] = qrows.reshape(len(rows), csa.H_I, -1)
            self.qI_sf[sl] = qsf.reshape(len(rows), csa.H_I, -1)
        q0 = synth.prefill_queries(w, 0, rows=np.arange(1))
        q1 = synth.prefill_queries(w, 1, rows=np.arange(1))
        self.bias_c = torch.from_numpy(q0["bias"]).to(dev)
        self.ibias = torch.from_numpy(q0["ibias"]).to(dev)
        self.bias_h = torch.from_numpy(q1["bias"]).to(dev)
        self.sink_c = torch.from_numpy(q0["sink"]).to(dev)
        self.sink_h = torch.from_numpy(q1["sink"]).to(dev)
        self.pos = torch.arange(P, L, dtype=torch.int64, device=dev)
        self.seq = torch.zeros(n, dtype=torch.int32, device=dev)
        self.idx = torch.full((n, csa.top_k), -1, dtype=torch.int32, device=dev)
        od = out_dtype or torch.bfloat16
        self.out_c = torch.zeros(n, csa.H, csa.d, dtype=od, device=dev)
        self.lse_c = torch.zeros(n, csa.H, dtype=torch.float32, device=dev)
        self.out_h = torch.zeros(n, hca.H, hca.d, dtype=od, device=dev)
        self.lse_h = torch.zeros(n, hca.H, dtype=torch.float32, device=dev)
        self.ws_c = v.workspace(self.dc, n, self.rows_c)
        self.ws_h = v.workspace(self.dh, n, self.rows_h)
        self._one = lambda val: torch.full((1,), val, dtype=torch.int64, device=dev)
        self.L_t = self._one(L)

    def _col(self, nm):
        c0, _ = self.cols[nm]
        return self.Y[:, c0:]

    def _compress_tokens(self, t0, t1, seq_len):
        """Entries and keys whose blocks complete in tokens [t0, t1) (a block
        that straddles t0 was skipped as incomplete before), and the window
        rows of tokens [t0, t1)."""
        v, csa, hca, L = self.v, self.csa, self.hca, self.w.L
        common = dict(in_rows=L, in_seq_stride=L * self.ncol, in_row_stride=self.ncol,
                      seq_len=seq_len)
        e0, ne = t0 // csa.m, t1 // csa.m - t0 // csa.m
        v.compress(self.dc, m=csa.m, overlap=True, c=csa.d, Ca=self._col("Ca"),
                   Za=self._col("Za"), Cb=self._col("Cb"), Zb=self._col("Zb"), bias=self.bias_c,
                   entry_begin=self._one(e0), n_entries=ne, complete_only=True,
                   out_dtype=v.E4M3_BF16ROPE, out=self.kv_c, out_scale=self.kvs_c,
                   out_rows=self.rows_c, **common)
        v.compress(self.dc, m=csa.m, overlap=True, c=csa.d_I, Ca=self._col("ICa"),
                   Za=self._col("IZa"), Cb=self._col("ICb"), Zb=self._col("IZb"),
                   bias=self.ibias, entry_begin=self._one(e0), n_entries=ne, complete_only=True,
                   out_dtype=v.MXFP4, out=self.keys, out_scale=self.keys_sf, out_rows=self.rows_c,
                   apply_rmsnorm=False, apply_rope=False, **common)
        h0, nh = t0 // hca.m, t1 // hca.m - t0 // hca.m
        v.compress(self.dh, m=hca.m, overlap=False, c=hca.d, Ca=self._col("C"),
                   Za=self._col("Z"), bias=self.bias_h, entry_begin=self._one(h0), n_entries=nh,
                   complete_only=True, out_dtype=v.E4M3_BF16ROPE, out=self.kv_h,
                   out_scale=self.kvs_h, out_rows=self.rows_h, **common)
        for desc, col, out, sc in ((self.dc, "Ca", self.swa_c, self.swas_c),
                                   (self.dh, "C", self.swa_h, self.swas_h)):
            v.compress(desc, m=1, overlap=False, c=csa.d, Ca=self._col(col), Za=None,
                       entry_begin=self._one(t0), n_entries=t1 - t0, out_dtype=v.E4M3_BF16ROPE,
                       out=out, out_scale=sc, out_rows=L, **common)

    def prefix_state(self):
        """The caches of the prefix tokens (not part of the timed step)."""
        P = self.w.prefix
        if P:
            self.v.project(self.x[:P], self.W, self.Y[:P])
            self._compress_tokens(0, P, self._one(P))

    def step(self):
        """The timed chunked-prefill step of the new tokens."""
        for _, f in self.phases():
            f()

    def phases(self):
        """The step's calls as (name, callable), in step order."""
        v, csa, hca, w = self.v, self.csa, self.hca, self.w
        P, L = w.prefix, w.L
        return [
            ("project (a0)", lambda: v.project(self.x[P:], self.W, self.Y[P:])),
            ("compress (a1)", lambda: self._compress_tokens(P, L, self.L_t)),
            ("index_topk (a3, a4)", lambda: v.index_topk(
                self.dc, qI=self.qI, qI_sf=self.qI_sf, w=self.wI, q_pos=self.pos, q_seq=self.seq,
                B=1, keys=self.keys, keys_sf=self.keys_sf, key_rows=self.rows_c,
                max_vis=L // csa.m, idx_out=self.idx, ws=self.ws_c)),
            ("sparse_mqa (a2, a5-a7)", lambda: v.sparse_mqa(
                self.dc, Q=self.Q_c, q_pos=self.pos, q_seq=self.seq, B=1, kv=self.kv_c,
                kv_scale=self.kvs_c, kv_rows=self.rows_c, swa=self.swa_c, swa_scale=self.swas_c,
                swa_rows=L, idx=self.idx, out=self.out_c, ws=self.ws_c, sink=self.sink_c,
                lse=self.lse_c)),
            ("dense_mqa (a2, a5-a7)", lambda: v.dense_mqa(
                self.dh, Q=self.Q_h, q_pos=self.pos, q_seq=self.seq, B=1, kv=self.kv_h,
                kv_scale=self.kvs_h, kv_rows=self.rows_h, swa=self.swa_h, swa_scale=self.swas_h,
                swa_rows=L, max_vis=L // hca.m, out=self.out_h, ws=self.ws_h, sink=self.sink_h,
                lse=self.lse_h)),
        ]

    def flops(self):
        """Algorithmic FLOPs of one step by tensor-core format."""
        csa, hca, w = self.csa, self.hca, self.w
        P, L, n = w.prefix, w.L, w.n_queries
        pos = np.arange(P, L, dtype=np.float64)
        nv_c = np.floor((pos + 1) / csa.m)
        nv_h = np.floor((pos + 1) / hca.m)
        win = np.minimum(pos + 1, csa.n_win)
        proj = 2.0 * n * w.d_model * self.ncol
        idx = float(np.sum(nv_c)) * 2 * csa.H_I * csa.d_I
        mqa_c = float(np.sum(np.minimum(nv_c, csa.top_k) + win)) * 4 * csa.H * csa.d
        mqa_h = float(np.sum(nv_h + np.minimum(pos + 1, hca.n_win))) * 4 * hca.H * hca.d
        return {"bf16": proj, "fp4": idx, "fp8": mqa_c + mqa_h}


def algorithmic_bytes(w):
    """Bytes one decode step must move (per the method), per layer: visible or
    selected entries x 580 B, indexer keys x 68 B, window tokens x 580 B, Q in
    bf16, indexer q (MXFP4) + weights, the new token's inputs, the output."""
    out = {}
    for ly in w.layers:
        p = w.L - 1
        n_vis = (p + 1) // ly.m
        entry = (ly.d - ly.d_rope) + 2 * ly.d_rope + 4
        q_b = ly.H * ly.d * 2 + ly.H * ly.d * 2
        if ly.kind == "csa":
            key_b = ly.d_I // 2 + ly.d_I // 32
            idx = n_vis * key_b + ly.H_I * (key_b + 4)
            mqa = (ly.top_k + ly.n_win) * entry + q_b
            out["csa"] = dict(index=w.B * idx, mqa=w.B * mqa, entries=w.B * (ly.top_k + ly.n_win),
                              keys=w.B * n_vis)
        else:
            mqa = (n_vis + ly.n_win) * entry + q_b
            out["hca"] = dict(mqa=w.B * mqa, entries=w.B * (n_vis + ly.n_win))
    return out


def algorithmic_flops(w):
    out = 0
    for ly in w.layers:
        n_vis = (w.L) // ly.m
        if ly.kind == "csa":
            out += w.B * (n_vis * 2 * ly.H_I * ly.d_I + (ly.top_k + ly.n_win) * 4 * ly.H * ly.d)
        else:
            out += w.B * (n_vis + ly.n_win) * 4 * ly.H * ly.d
    return out


# ------------------------------------------------------------------ clocks

def graph_kernel_nodes(graph):
    """Number of kernel nodes in a captured torch CUDA graph (None if the
    runtime bindings are unavailable)."""
    try:
        from cuda.bindings import runtime as rt
        g = rt.cudaGraph_t(init_value=graph.raw_cuda_graph())
        err, _, n = rt.cudaGraphGetNodes(g, 0)
        if err != rt.cudaError_t.cudaSuccess:
            return None
        err, nodes, n = rt.cudaGraphGetNodes(g, n)
        if err != rt.cudaError_t.cudaSuccess:
            return None
        kern = 0
        for nd in nodes[:n]:
            err, ty = rt.cudaGraphNodeGetType(nd)
            if err == rt.cudaError_t.cudaSuccess and ty == rt.cudaGraphNodeType.cudaGraphNodeTypeKernel:
                kern += 1
        return kern
    except Exception:
        return None


def code_digest(paths):
    """sha256 of C/CUDA sources with comments and whitespace removed, so that a
    comment edit does not count as a change of the kernel."""
    import hashlib
    import re
    h = hashlib.sha256()
    for f in paths:
        text = open(os.path.join(ROOT, f), encoding="utf-8").read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
        text = re.sub(r"//[^\n]*", " ", text)
        h.update(" ".join(text.split()).encode())
    return h.hexdigest()


def _index_traffic():
    """DRAM bytes (read + write) per indexer launch from the committed ncu
    capture, or None when the kernel's code has changed since."""
    path = os.path.join(ROOT, "profiles", "index_tc_pro_pair_1m_counters.json")
    try:
        rec = json.load(open(path))
        same = code_digest(rec["sources"]) == rec["code_sha256"]
        return int(rec["dram_bytes_per_launch"]) if same else None
    except (OSError, KeyError, ValueError):
        return None


class ClockSampler:
    """SM clock and clock-event reasons sampled through NVML every few
    milliseconds from a host thread; only samples taken between ``start()``
    and ``stop()`` (the timed region) are kept."""

    PERIOD_S = 0.005

    def __init__(self, cuda_index: int):
        self.cuda_index = cuda_index
        self.samples = []
        self.max_mhz = None
        self._on = False
        self._quit = False
        self._thread = None
        self._nvml = None
        self._h = None

    def _handle(self):
        import pynvml
        import torch
        pynvml.nvmlInit()
        props = torch.cuda.get_device_properties(self.cuda_index)
        try:
            bus = "%08x:%02x:%02x.0" % (props.pci_domain_id, props.pci_bus_id, props.pci_device_id)
            return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.cuda_index)

    def _loop(self):
        nv, h = self._nvml, self._h
        while not self._quit:
            if self._on:
                try:
                    sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                    rs = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                    self.samples.append((sm, rs))
                except Exception:
                    pass
            time.sleep(self.PERIOD_S)

    def __enter__(self):
        try:
            self._nvml, self._h = self._handle()
            self.max_mhz = self._nvml.nvmlDeviceGetMaxClockInfo(self._h, self._nvml.NVML_CLOCK_SM)
            self._thread = threading.Thread(target=self._loop, daemon=True)
            self._thread.start()
        except Exception:
            self._nvml = None
        return self

    def start(self):
        self._on = True

    def stop(self):
        self._on = False

    def __exit__(self, *exc):
        self._quit = True
        if self._thread is not None:
            self._thread.join(timeout=2)
        if self._nvml is not None:
            try:
                self._nvml.nvmlShutdown()
            except Exception:
                pass

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0,
                    "source": "nvml"}
        nv = self._nvml
        names = {"hw_slowdown": getattr(nv, "nvmlClocksEventReasonHwSlowdown", 0x8),
                 "hw_thermal_slowdown": getattr(nv, "nvmlClocksEventReasonHwThermalSlowdown", 0x40),
                 "sw_thermal_slowdown": getattr(nv, "nvmlClocksEventReasonSwThermalSlowdown", 0x20),
                 "sw_power_cap": getattr(nv, "nvmlClocksEventReasonSwPowerCap", 0x4),
                 "hw_power_brake": getattr(nv, "nvmlClocksEventReasonHwPowerBrakeSlowdown", 0x80)}
        reasons = sorted({n for n, bit in names.items() for _, rs in self.samples if rs & bit})
        return {"sm_mhz": float(np.median([sm for sm, _ in self.samples])),
                "sm_max_mhz": self.max_mhz, "reasons": reasons, "samples": len(self.samples),
                "source": "nvml"}


# ------------------------------------------------------------------ timing helpers

def timed_device(run, flush, steps, stream):
    """Per-step CUDA-event durations (ms) of ``run`` with an L2 flush between
    steps (outside the timed intervals), all on ``stream``."""
    import torch
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps)]
    with torch.cuda.stream(stream):
        for a, b in evs:
            flush()
            a.record(stream)
            run()
            b.record(stream)
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in evs]


def capture_graph(fn):
    """Capture ``fn``'s launches into a CUDA graph (after one eager call)."""
    import torch
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    torch.cuda.synchronize()
    return g


def _dist_device(dist):
    import torch
    return "cuda" if torch.cuda.is_available() and dist.get_backend() == "nccl" else "cpu"


def max_over_ranks(x: float, dist):
    """The largest of the ranks' values (every rank gets it)."""
    if dist is None:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=_dist_device(dist))
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(dist):
    import torch
    if dist is not None:
        dist.barrier()
    if torch.cuda.is_available():
        torch.cuda.synchronize()


def rank_workload(name: str, rank: int):
    """Rank r's share of a weak-scaling run: the workload's recipe at its own
    batch size, drawn under a rank-specific seed, so that every rank holds
    different sequences (global sequences r*B .. r*B+B-1); rank 0's draws are
    those of a one-GPU run."""
    import dataclasses
    w = synth.WORKLOADS[name]
    return w if rank == 0 else dataclasses.replace(w, seed=w.seed + 7919 * rank)


def shard(rank: int, world: int, B: int):
    """Global sequence ids of rank ``rank`` (weak scaling: B per rank)."""
    assert 0 <= rank < world
    return range(rank * B, (rank + 1) * B)


def job_value(ms_max: float, B: int, world: int) -> float:
    """Whole-job queries/s: every rank's B sequences in the slowest rank's time."""
    return world * B / (ms_max / 1e3)


# ------------------------------------------------------------------ the GPU arm

class Workload:
    """The decode layers of one workload on this GPU, captured as one graph."""

    def __init__(self, name, rank: int = 0):
        import torch
        self.w = rank_workload(name, rank)
        self.inputs = [synth.decode_layer_inputs(self.w, li) for li in range(len(self.w.layers))]
        self.layers = [build_decode_layer(self.w, li, inp) for li, inp in enumerate(self.inputs)]
        torch.cuda.synchronize()
        self.graph = None

    def step(self):
        for lay in self.layers:
            lay.step(lay.max_vis)

    def capture(self):
        import torch
        self.step()                               # first launches outside the capture
        torch.cuda.synchronize()
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            self.step()
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        self.graph = torch.cuda.CUDAGraph(keep_graph=True)
        with torch.cuda.graph(self.graph):
            self.step()
        torch.cuda.synchronize()
        self.kernel_nodes = graph_kernel_nodes(self.graph)

    def replay(self):
        self.graph.replay()

    def capture_layers(self):
        """One graph per layer (the same calls as the step's graph), so that a
        serving loop can overlap one layer's copies with another's kernels."""
        import torch
        self.layer_graphs = []
        for lay in self.layers:
            g = torch.cuda.CUDAGraph(keep_graph=True)
            with torch.cuda.graph(g):
                lay.step(lay.max_vis)
            self.layer_graphs.append(g)
        torch.cuda.synchronize()

    def queries_per_step(self):
        return self.w.B

    def launches_per_step(self):
        """Kernel launches of one step: the kernel nodes of the captured graph
        (every one of them is a library kernel; the step makes no other call)."""
        if getattr(self, "kernel_nodes", None):
            return self.kernel_nodes
        n = 0
        for ly in self.w.layers:
            # fused append (+ index scores + top-k) (+ query coding when the
            # append cannot do it) + MQA + combine
            tc_mqa = ly.kv_fp8 and ly.d == 512
            coded_in_append = tc_mqa and self.w.B <= 1024
            n += 1 + (2 if ly.kind == "csa" else 0) + (1 if tc_mqa and not coded_in_append else 0) + 2
        return n

    # per-step host<->device traffic of the end-to-end measurement
    def host_io(self, per_layer=False):
        """(host, device) pairs of every layer's per-step inputs and outputs
        (pinned host copies); with ``per_layer`` grouped by layer."""
        import torch
        ins, outs = [], []
        for lay in self.layers:
            li, lo = [], []
            for t in ([lay.x_main, lay.Q, lay.pos] +
                      ([lay.x_idx, lay.qI, lay.qI_sf, lay.w] if lay.csa else [])):
                if t is None:
                    continue
                h = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
                h.copy_(t)
                li.append((h, t))
            h = torch.empty(lay.out.shape, dtype=lay.out.dtype, pin_memory=True)
            lo.append((h, lay.out))
            if per_layer:
                ins.append(li)
                outs.append(lo)
            else:
                ins += li
                outs += lo
        return ins, outs


def dominant_roofline(wl, flush, steps, stream, dist, peaks, abytes):
    """The workload's dominant kernel timed alone as a graph replay (CUDA events
    on its stream, L2 flushed between launches) against the HBM copy peak:
    the CSA indexer (scores only) when the workload has a CSA layer, else the
    HCA layer's dense MQA (query image + MQA).  Returns (roofline dict, ms)."""
    import torch
    import long_context_compressed_kv_b200 as v
    csa = [lay for lay in wl.layers if lay.csa]
    if csa:
        lay = csa[0]
        scores = torch.empty(lay.B, lay.max_vis, dtype=torch.float32, device="cuda")

        def run():
            v.index_topk(lay.desc, qI=lay.qI, qI_sf=lay.qI_sf, w=lay.w, q_pos=lay.pos,
                         keys=lay.keys, keys_sf=lay.keys_sf, key_rows=lay.kv_rows,
                         max_vis=lay.max_vis, idx_out=None, scores_out=scores, ws=lay.ws)
        name, nbytes = "index_scores (CSA indexer, MXFP4 keys)", abytes["csa"]["index"]
    else:
        lay = wl.layers[0]

        def run():
            v.dense_mqa(lay.desc, Q=lay.Q, q_pos=lay.pos, kv=lay.kv, kv_scale=lay.kv_scale,
                        kv_rows=lay.kv_rows, swa=lay.swa, swa_scale=lay.swa_scale,
                        swa_rows=lay.swa_rows, max_vis=lay.max_vis, out=lay.out, ws=lay.ws,
                        sink=lay.sink, lse=lay.lse)
        name, nbytes = "dense_mqa (HCA shared-KV MQA, E4M3 entries)", abytes["hca"]["mqa"]
    for _ in range(3):
        flush()
        run()
    # timed as a graph replay: a direct call would also time the host-side enqueue
    g = capture_graph(run)
    t = float(np.mean(timed_device(g.replay, flush, steps, stream)))
    t = max_over_ranks(t, dist)
    achieved = nbytes / (t / 1e3) / 1e9
    roof = {"kernel": name, "bound": "hbm", "achieved": round(achieved, 1),
            "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
            "traffic": _index_traffic() if csa and wl.w.name == HEADLINE else None,
            "peak_source": peaks["source"], "launch_us": round(t * 1e3, 2),
            "algorithmic_bytes": int(nbytes)}
    del g
    return roof, t


def run_gpu(args, dist, rank, world):
    import torch
    torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
    stream = torch.cuda.current_stream()
    flush_buf = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    flush_sink = torch.zeros(1, dtype=torch.int32, device="cuda")

    def flush():
        # write a buffer larger than L2, then read it back: the step starts with
        # nothing of its own in L2 and with no dirty line whose write-back it
        # would otherwise pay for
        flush_buf.zero_()
        flush_sink.copy_(flush_buf.view(torch.int32).amax().view(1))

    wl = Workload(args.workload, rank)
    wl.capture()
    launches = wl.launches_per_step()
    for _ in range(args.warmup):
        flush()
        wl.replay()
    barrier(dist)
    with ClockSampler(torch.cuda.current_device()) as clk:
        barrier(dist)
        clk.start()
        per_step = timed_device(wl.replay, flush, args.steps, stream)
        clk.stop()
        barrier(dist)
    ms = max_over_ranks(float(np.mean(per_step)), dist)
    if args.profile:
        return dict(profile=True, ms=ms, launches=launches)
    q_step = wl.queries_per_step()
    value = job_value(ms, q_step, world)

    # ---- dominant kernel, timed alone
    peaks = _peaks()
    abytes = algorithmic_bytes(wl.w)
    roof, t_idx = dominant_roofline(wl, flush, max(args.steps, 10), stream, dist, peaks, abytes)
    csa = [lay for lay in wl.layers if lay.csa]
    step_bytes = sum(sum(vv for kk, vv in d.items() if kk in ("index", "mqa"))
                     for d in abytes.values())
    step_roof = {"bytes": int(step_bytes), "us": round(ms * 1e3, 2),
                 "achieved_gbs": round(step_bytes / (ms / 1e3) / 1e9, 1),
                 "frac_hbm": round(step_bytes / (ms / 1e3) / 1e9 / peaks["hbm_gbs"], 4)}

    # ---- end to end through the public API with host buffers: every step
    # copies its inputs from pinned host memory, runs the step, and reads the
    # outputs back.  "graph": one captured graph per layer, as a serving loop
    # runs it, with the copies on their own streams: layer l + 1's inputs go
    # up while layer l runs and layer l's output comes back while layer l + 1
    # runs (the timed interval holds every copy: both side streams start
    # after its first event and the step stream waits for them before its
    # last).  "eager": the same copies and the layers' calls through the
    # Python binding, all on the one stream
    ins, outs = wl.host_io()
    ins_l, outs_l = wl.host_io(per_layer=True)
    h2d = sum(h.numel() * h.element_size() for h, _ in ins)
    d2h = sum(h.numel() * h.element_size() for h, _ in outs)
    wl.capture_layers()
    up, down = torch.cuda.Stream(), torch.cuda.Stream()

    def pipelined():
        main = torch.cuda.current_stream()
        start = torch.cuda.Event()
        start.record(main)
        up.wait_event(start)
        down.wait_event(start)
        landed = []
        with torch.cuda.stream(up):
            for pairs in ins_l:
                for h, d in pairs:
                    d.copy_(h, non_blocking=True)
                e = torch.cuda.Event()
                e.record(up)
                landed.append(e)
        for li, g in enumerate(wl.layer_graphs):
            main.wait_event(landed[li])
            g.replay()
            e = torch.cuda.Event()
            e.record(main)
            down.wait_event(e)
            with torch.cuda.stream(down):
                for h, d in outs_l[li]:
                    h.copy_(d, non_blocking=True)
        done = torch.cuda.Event()
        done.record(down)
        main.wait_event(done)

    def with_copies(run):
        def f():
            for h, d in ins:
                d.copy_(h, non_blocking=True)
            run()
            for h, d in outs:
                h.copy_(d, non_blocking=True)
        return f
    e2e = {}
    for name, f in (("graph", pipelined), ("eager", with_copies(wl.step))):
        for _ in range(args.warmup):
            flush()
            f()
        barrier(dist)
        e2e[name] = max_over_ranks(float(np.mean(timed_device(f, flush, args.steps, stream))), dist)
    e2e_ms = e2e["graph"]
    e2e_val = world * q_step / (e2e_ms / 1e3)
    e2e_eager = world * q_step / (e2e["eager"] / 1e3)
    peaks_tc = measure_tc_peaks(stream)
    if roof is not None and csa:
        fp4 = abytes["csa"]["keys"] * 2 * csa[0].desc.H_I * csa[0].desc.d_I
        ach_t = fp4 / (t_idx / 1e3) / 1e12
        roof["tensor"] = {"format": "mxfp4", "flops_per_launch": int(fp4),
                          "achieved_tflops": round(ach_t, 1),
                          "peak_tflops": peaks_tc["fp4_mxf4_tflops"],
                          "frac": round(ach_t / peaks_tc["fp4_mxf4_tflops"], 4),
                          "peak_source": "measured in this run (tcgen05 probe)"}

    # ---- the BF16-score selector variant on the same CSA layer: index + top-k
    # with fp32 scores against bf16 scores, and the recall of the bf16
    # selection against the fp32 one
    bf16_sel = None
    if csa and world == 1:
        import long_context_compressed_kv_b200 as v
        lay = csa[0]
        idx32 = torch.empty_like(lay.idx)
        idx16 = torch.empty_like(lay.idx)
        times = {}
        for name, out_idx, sd in (("fp32", idx32, v.F32), ("bf16", idx16, v.BF16)):
            def sel(out_idx=out_idx, sd=sd):
                v.index_topk(lay.desc, qI=lay.qI, qI_sf=lay.qI_sf, w=lay.w, q_pos=lay.pos,
                             keys=lay.keys, keys_sf=lay.keys_sf, key_rows=lay.kv_rows,
                             max_vis=lay.max_vis, idx_out=out_idx, ws=lay.ws, score_dtype=sd)
            for _ in range(3):
                flush()
                sel()
            g_sel = capture_graph(sel)
            times[name] = float(np.mean(timed_device(g_sel.replay, flush, max(args.steps, 10),
                                                     stream)))
            del g_sel
        a32, a16 = idx32.cpu().numpy(), idx16.cpu().numpy()
        rec = [len(np.intersect1d(a32[b][a32[b] >= 0], a16[b][a16[b] >= 0])) /
               max(1, int((a32[b] >= 0).sum())) for b in range(a32.shape[0])]
        bf16_sel = {"index_topk_us_fp32_scores": round(times["fp32"] * 1e3, 2),
                    "index_topk_us_bf16_scores": round(times["bf16"] * 1e3, 2),
                    "speedup": round(times["fp32"] / times["bf16"], 3),
                    "recall_of_fp32_selection": round(float(np.mean(rec)), 4),
                    "note": "synthetic N(0,1) keys and queries, not trained weights"}

    # ---- the same step on paged caches: every layer's compressed cache (and
    # the CSA indexer keys) scattered over a shuffled pool of 128-token blocks
    # behind a block table, the window and tails per sequence as before
    paged = None
    if world == 1:
        paged = paged_decode_measure(wl, flush, args.steps, stream)

    also = {}
    if not args.no_also and world == 1:
        del wl
        torch.cuda.empty_cache()
        for name in ALSO:
            w2 = Workload(name, rank)
            w2.capture()
            for _ in range(args.warmup):
                flush()
                w2.replay()
            t2 = float(np.mean(timed_device(w2.replay, flush, args.steps, stream)))
            b2 = algorithmic_bytes(w2.w)
            sb = sum(sum(vv for kk, vv in d.items() if kk in ("index", "mqa")) for d in b2.values())
            r2, _ = dominant_roofline(w2, flush, max(args.steps, 10), stream, None, peaks, b2)
            also[name] = {"queries_per_s": round(w2.queries_per_step() / (t2 / 1e3), 1),
                          "us_per_step": round(t2 * 1e3, 2),
                          "frac_hbm": round(sb / (t2 / 1e3) / 1e9 / peaks["hbm_gbs"], 4),
                          "roofline": r2}
            del w2
            torch.cuda.empty_cache()
    return dict(value=value, ms=ms, roof=roof, step_roof=step_roof, clocks=clk.summary(),
                paged=paged,
                e2e=dict(value=e2e_val, h2d=h2d, d2h=d2h, ms=e2e_ms, eager_value=e2e_eager,
                         eager_ms=e2e["eager"]), also=also, tc_peaks=peaks_tc,
                bf16_selector=bf16_sel,
                launches=launches, q_step=q_step,
                per_step=per_step)


def paged_decode_measure(wl, flush, steps, stream, spare_blocks=16, seed=1):
    """The workload's decode step with paged compressed caches: per layer a
    pool of B * blocks_per_seq + spare_blocks blocks (epb = 128 / m entries a
    block) holding each sequence's entries (and, for CSA, indexer keys) in a
    shuffled order, a block table, and one captured graph of every layer's
    v4attn_decode on them; timed like the step itself.  Also checks that the
    outputs equal the contiguous step's (CSA: bit for bit; HCA, whose paged
    entries are gathered rather than tiled and so split over other CTAs,
    within 5e-3 of the output's RMS, the f16 rounding of the split partials,
    plus one bf16 step of the element)."""
    import torch
    import long_context_compressed_kv_b200 as v
    rng = np.random.default_rng(seed)
    calls, outs = [], []
    for lay in wl.layers:
        epb = 128 // lay.m
        bps = lay.kv_rows // epb
        n = lay.B * bps + spare_blocks
        table = rng.permutation(n)[: lay.B * bps].astype(np.int64)
        sel = torch.from_numpy(table).cuda()
        bt = sel.to(torch.int32).view(lay.B, bps).contiguous()

        def scatter(rows, n=n, epb=epb, bps=bps, sel=sel, B=lay.B):
            pool = torch.zeros((n * epb,) + tuple(rows.shape[2:]), dtype=rows.dtype,
                               device=rows.device)
            pool.view((n, epb) + tuple(rows.shape[2:]))[sel] = \
                rows.reshape((B * bps, epb) + tuple(rows.shape[2:]))
            return pool
        pkv, psc = scatter(lay.kv), scatter(lay.kv_scale)
        out, lse = torch.zeros_like(lay.out), torch.zeros_like(lay.lse)
        kw = {}
        if lay.csa:
            pk, psf = scatter(lay.keys), scatter(lay.keys_sf)
            idx = torch.full_like(lay.idx, -1)
            kw = dict(x_idx=lay.x_idx, itail=lay.itail, ibias=lay.ibias, keys=pk, keys_sf=psf,
                      key_rows=n * epb, qI=lay.qI, qI_sf=lay.qI_sf, w=lay.w, idx_out=idx)

        def call(lay=lay, pkv=pkv, psc=psc, n=n, epb=epb, bt=bt, out=out, lse=lse, kw=kw):
            v.decode(lay.desc, pos=lay.pos, x_main=lay.x_main, tail=lay.tail, bias=lay.bias,
                     kv=pkv, kv_scale=psc, kv_rows=n * epb, swa=lay.swa,
                     swa_scale=lay.swa_scale, swa_rows=lay.swa_rows, Q=lay.Q, out=out,
                     ws=lay.ws, max_vis=lay.max_vis, sink=lay.sink, lse=lse, block_table=bt,
                     **kw)
        calls.append(call)
        outs.append((lay, out, lse))

    def step():
        for c in calls:
            c()
    step()
    torch.cuda.synchronize()
    wl.replay()                       # the contiguous step's outputs, to compare
    torch.cuda.synchronize()
    same = {}
    for lay, out, lse in outs:
        name = "csa" if lay.csa else "hca"
        if lay.csa:
            same[name] = bool(torch.equal(out, lay.out) and torch.equal(lse, lay.lse))
        else:
            # within 5e-3 of the RMS (the split partials' f16 rounding) plus one
            # bf16 step of the element (the output's own rounding may flip)
            ref = lay.out.float()
            rms = float(ref.pow(2).mean().sqrt())
            same[name] = bool(((out.float() - ref).abs() <= 5e-3 * rms + ref.abs() / 128).all())
    g = capture_graph(step)
    for _ in range(3):
        flush()
        g.replay()
    t = float(np.mean(timed_device(g.replay, flush, steps, stream)))
    for lay, _, _ in outs:
        v.device_status(lay.ws)       # raises on a device-side check (a bad table entry)
    del g
    return {"queries_per_s": round(wl.queries_per_step() / (t / 1e3), 1),
            "us_per_step": round(t * 1e3, 2),
            "outputs_match_contiguous": same,
            "how": "pools of 128-token blocks (32 CSA entries + 32 indexer keys, or 1 HCA "
                   "entry, a block) in shuffled order behind a block table; one graph of "
                   "both layers' decode calls; L2 flushed between steps"}


def measure_tc_peaks(stream, reps=5, n_iter=16384):
    """Dense MMA rate of the three tcgen05 kinds the kernels use (bf16, E4M3,
    block-scaled MXFP4), from the library's probe: one CTA per SM issuing
    128 x 256 MMAs over shared-memory operands; best of ``reps`` launches timed
    with CUDA events on ``stream``, with the SM clock sampled meanwhile."""
    import torch
    import long_context_compressed_kv_b200 as v
    out = {}
    narrow = {}
    with ClockSampler(torch.cuda.current_device()) as clk:
        for kind, name in ((0, "bf16"), (1, "fp8_e4m3"), (2, "fp4_mxf4")):
            for n_cols in (256, 128, 64):
                v.tc_peak_probe(kind, 64, n_cols, stream=stream)          # warm-up
                best = 0.0
                clk.start()
                for _ in range(reps):
                    a = torch.cuda.Event(enable_timing=True)
                    b = torch.cuda.Event(enable_timing=True)
                    a.record(stream)
                    flops, ctas = v.tc_peak_probe(kind, n_iter, n_cols, stream=stream)
                    b.record(stream)
                    b.synchronize()
                    best = max(best, flops / (a.elapsed_time(b) / 1e3) / 1e12)
                clk.stop()
                if n_cols == 256:
                    out[name + "_tflops"] = round(best, 1)
                else:
                    narrow[f"{name}_n{n_cols}_tflops"] = round(best, 1)
    out["ctas"] = ctas
    out["shape"] = "M=128 N=256 per instruction, 1 CTA per SM, operands in shared memory"
    out["narrow_n"] = narrow
    out["clocks"] = clk.summary()
    return out


def run_prefill(args, dist, rank, world):
    """The chunked-prefill workload: one step = the whole chunk of new tokens
    through both layers (bench.PrefillPair.step), tokens/s."""
    import torch
    torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
    stream = torch.cuda.current_stream()
    w = rank_workload(args.workload, rank)
    pp = PrefillPair(w)
    pp.prefix_state()
    flush_buf = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    flush_sink = torch.zeros(1, dtype=torch.int32, device="cuda")

    def flush():
        flush_buf.zero_()
        flush_sink.copy_(flush_buf.view(torch.int32).amax().view(1))
    steps = min(args.steps, 10)
    for _ in range(args.warmup):
        flush()
        pp.step()
    barrier(dist)
    with ClockSampler(torch.cuda.current_device()) as clk:
        barrier(dist)
        clk.start()
        per_step = timed_device(pp.step, flush, steps, stream)
        clk.stop()
        barrier(dist)
    ms = max_over_ranks(float(np.mean(per_step)), dist)
    n = w.n_queries
    value = world * n / (ms / 1e3)
    # per-phase device time (each phase alone, after an L2 flush)
    phases = {}
    for name, f in pp.phases():
        phases[name] = round(float(np.mean(timed_device(f, flush, 3, stream))), 4)
    peaks = measure_tc_peaks(stream)
    fl = pp.flops()
    pk = {"bf16": peaks["bf16_tflops"], "fp4": peaks["fp4_mxf4_tflops"],
          "fp8": peaks["fp8_e4m3_tflops"]}
    t_roof = sum(fl[k] / (pk[k] * 1e12) for k in fl)       # seconds at the measured peaks
    total = sum(fl.values())
    dom = max(phases, key=phases.get)
    dom_fl = {"project (a0)": ("bf16", fl["bf16"]), "index_topk (a3, a4)": ("fp4", fl["fp4"])}
    roof = {"bound": "tensor", "achieved": round(total / (ms / 1e3) / 1e12, 2),
            "peak": round(total / t_roof / 1e12, 1), "unit": "TFLOP/s",
            "frac": round(t_roof / (ms / 1e3), 5), "traffic": None,
            "note": "step FLOPs over the sum of each format's FLOPs at its measured tcgen05 "
                    "peak (bf16 projection, MXFP4 indexer, E4M3/bf16 MQA)",
            "flops": {k: float(v_) for k, v_ in fl.items()}, "dominant_phase": dom}
    if dom in dom_fl:
        fmt, f_ = dom_fl[dom]
        roof["dominant"] = {"phase": dom, "format": fmt,
                            "achieved_tflops": round(f_ / (phases[dom] / 1e3) / 1e12, 2),
                            "peak_tflops": pk[fmt],
                            "frac": round(f_ / (phases[dom] / 1e3) / 1e12 / pk[fmt], 5)}
    # end to end: the chunk's raw tokens and per-query inputs copied in from
    # pinned memory, the step, both layers' outputs and LSE read back
    e2e = None
    try:
        P = w.prefix
        ins = [(torch.empty(t.shape, dtype=t.dtype, pin_memory=True), t)
               for t in (pp.x[P:], pp.Q_c, pp.Q_h, pp.qI, pp.qI_sf, pp.wI)]
        outs = [(torch.empty(t.shape, dtype=t.dtype, pin_memory=True), t)
                for t in (pp.out_c, pp.out_h, pp.lse_c, pp.lse_h, pp.idx)]
        for h, d in ins:
            h.copy_(d)

        def e2e_step():
            for h, d in ins:
                d.copy_(h, non_blocking=True)
            pp.step()
            for h, d in outs:
                h.copy_(d, non_blocking=True)
        e2e_step()
        barrier(dist)
        e_ms = max_over_ranks(float(np.mean(timed_device(e2e_step, flush, min(steps, 3),
                                                         stream))), dist)
        e2e = {"value": round(world * n / (e_ms / 1e3), 1), "unit": "tokens/s",
               "h2d_bytes_per_step": int(sum(h.numel() * h.element_size() for h, _ in ins)),
               "d2h_bytes_per_step": int(sum(h.numel() * h.element_size() for h, _ in outs)),
               "ms_per_step": round(e_ms, 4)}
    except RuntimeError as ex:              # pinned host memory refused
        e2e = {"value": None, "unavailable": str(ex).splitlines()[0][:200]}
    return dict(value=value, ms=ms, roof=roof, phases=phases, clocks=clk.summary(), e2e=e2e,
                tc_peaks=peaks, steps=steps, w=w)


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(path))
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "source": "fallback"}


# ------------------------------------------------------------------ the oracle (CPU) arm

def _cpu_info():
    """(logical CPUs of this host, CPU model string)."""
    model = None
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                model = line.split(":", 1)[1].strip()
                break
    except OSError:
        pass
    return os.cpu_count(), model


def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info()]
        return max(n) if n else 1
    except Exception:  # noqa: BLE001
        return 1


def oracle_sample(name, seconds_target=12.0, max_seqs=None):
    """Time the CPU oracle's decode step on a bounded sample of the workload:
    whole sequences (every layer of the workload) until ~seconds_target of
    CPU work.  Returns (queries/s, sample description, seconds)."""
    from oracle import pipeline
    w = synth.WORKLOADS[name]
    inputs = [synth.decode_layer_inputs(w, li) for li in range(len(w.layers))]
    caches = [dict() for _ in w.layers]
    n = 0
    t_total = 0.0
    b = 0
    while t_total < seconds_target and (max_seqs is None or n < max_seqs):
        t0 = time.perf_counter()
        for li, ly in enumerate(w.layers):
            pipeline.decode_layer(inputs[li], ly, [b % w.B])
        t_total += time.perf_counter() - t0
        n += 1
        b += 1
    return n / t_total, f"{n} sequence(s) x {len(w.layers)} layer(s) of {name}", t_total


def oracle_prefill_sample(name, seconds_target=12.0):
    """Time the CPU oracle's per-token work of the chunked-prefill workload on
    a bounded sample: for consecutive new tokens at the end of the chunk, the
    token's projection row, its share of the pooling (one CSA entry + indexer
    key per 4 tokens, one HCA entry per 128), the indexer scores over every
    visible key, top-k, and both layers' attention.  The cached keys and
    entries it reads are synthetic stand-ins of the right shapes (the time of
    these steps does not depend on their values).  Returns (tokens/s,
    description, seconds)."""
    from oracle import compress as ocomp, indexer as oidx, mqa as omqa, pipeline
    w = synth.WORKLOADS[name]
    csa, hca = w.layers
    W = synth.prefill_weight(w).astype(np.float64)
    rng = np.random.default_rng(0)
    nk = w.L // csa.m
    keys = rng.standard_normal((nk, csa.d_I))
    ents_c = rng.standard_normal((nk, csa.d))
    ents_h = rng.standard_normal((w.L // hca.m, hca.d))
    win = rng.standard_normal((csa.n_win, csa.d))
    n, t_total, r = 0, 0.0, w.n_queries - 1
    blk = synth.ROWS_PER_BLOCK
    cache = {}
    while t_total < seconds_target and r >= 0:
        b0 = r // blk * blk
        if b0 not in cache:                # one generator block of rows at a time
            rows = np.arange(b0, min(w.n_queries, b0 + blk))
            cache = {b0: (synth.prefill_queries(w, 0, rows=rows),
                          synth.prefill_queries(w, 1, rows=rows),
                          synth.prefill_x(w, rows=rows + w.prefix).astype(np.float64))}
        Q0, Q1, X = cache[b0]
        j = r - b0
        q0 = {k: (v_[j:j + 1] if k in ("Q", "qI", "w") else v_) for k, v_ in Q0.items()}
        q1 = {k: (v_[j:j + 1] if k == "Q" else v_) for k, v_ in Q1.items()}
        x = X[j:j + 1]
        t0 = time.perf_counter()
        p = w.prefix + r
        y = x @ W                                             # a0
        if p % csa.m == 0:                                    # a1 (amortised shares)
            i = np.array([p // csa.m])
            ocomp.pool(i, csa.m, True, w.L, lambda t: np.repeat(y[:, :csa.d], t.size, 0).reshape(
                t.shape + (csa.d,)), lambda t: np.zeros(t.shape + (csa.d,)), q0["bias"],
                lambda t: np.zeros(t.shape + (csa.d,)), lambda t: np.zeros(t.shape + (csa.d,)))
        nv = (p + 1) // csa.m
        s = oidx.scores(pipeline.store_key(q0["qI"][0], csa)[1], q0["w"][0], keys[:nv])  # a3
        sel = oidx.topk(s, nv, csa.top_k)                     # a4
        kc = np.concatenate([ents_c[sel[sel >= 0]], win], 0)
        qc = omqa.prepare_query(q0["Q"][0], p, csa.d_rope, csa.rope_theta, True)
        omqa.attend(qc, kc, 1 / np.sqrt(csa.d), q0["sink"])   # a6 CSA
        kh = np.concatenate([ents_h[:(p + 1) // hca.m], win], 0)
        qh = omqa.prepare_query(q1["Q"][0], p, hca.d_rope, hca.rope_theta, True)
        omqa.attend(qh, kh, 1 / np.sqrt(hca.d), q1["sink"])   # a6 HCA
        t_total += time.perf_counter() - t0
        n += 1
        r -= 1
    return n / t_total, f"{n} consecutive new tokens at the end of the chunk of {name}", t_total


def run_reference(args):
    """The reference arm: the fp64 CPU oracle, as it stands, on host cores."""
    from oracle import pipeline
    w = synth.WORKLOADS[args.workload]
    inputs = [synth.decode_layer_inputs(w, li) for li in range(len(w.layers))]
    times = []
    for s in range(args.warmup + args.steps):
        b = s % w.B
        t0 = time.perf_counter()
        for li, ly in enumerate(w.layers):
            pipeline.decode_layer(inputs[li], ly, [b])
        dt = time.perf_counter() - t0
        if s >= args.warmup:
            times.append(dt)
    value = 1.0 / float(np.mean(times))
    cores = _blas_threads()
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 4),
            "unit": "queries/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(float(np.mean(times)) * 1e3, 2),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": args.workload, "batch": w.B, "context": w.L,
                       "layers": [ly.kind for ly in w.layers], "l2": "n/a (CPU)"},
            "cpu_baseline": {"value": round(value, 4), "unit": "queries/s", "cores": cores,
                             "nproc": _cpu_info()[0], "cpu_model": _cpu_info()[1],
                             "kind": "oracle",
                             "sample": f"per step: 1 sequence through every layer of {args.workload}"},
            "e2e": {"value": round(value, 4), "unit": "queries/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="v4attn", choices=["v4attn", "reference"])
    ap.add_argument("--workload", default=HEADLINE, choices=sorted(synth.WORKLOADS))
    ap.add_argument("--no-also", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile", action="store_true",
                    help="graph capture, warm-up and timed steps only (for a kernel launch list)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            run_reference(args)
        return
    dist = None
    if world > 1:
        import datetime
        import torch
        import torch.distributed as tdist
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        dist = tdist
    if synth.WORKLOADS[args.workload].prefix > 0:
        res = run_prefill(args, dist, rank, world)
        if rank == 0:
            w = res["w"]
            line = {
                "metric": "chunked-prefill tokens/s of a V4-Flash CSA + HCA layer pair; "
                          "% of FP4/FP8/BF16-TC roofline",
                "value": round(res["value"], 1), "unit": "tokens/s", "n_gpus": world,
                "steps": res["steps"], "warmup": args.warmup, "ms_per_step": round(res["ms"], 4),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "bf16 projection, e4m3+bf16 KV, mxfp4 indexer, f32 accumulate",
                "data": "synthetic",
                "config": {"workload": args.workload, "new_tokens": w.n_queries,
                           "prefix": w.prefix, "d_model": w.d_model,
                           "layers": [f"{ly.kind} m={ly.m} H={ly.H} d={ly.d}" +
                                      (f" top_k={ly.top_k} H_I={ly.H_I}x{ly.d_I}"
                                       if ly.kind == "csa" else "") for ly in w.layers],
                           "l2": "flushed between steps (320 MB write, then read back)"},
                "e2e": res["e2e"], "roofline": res["roof"], "phases_ms": res["phases"],
                "tc_peaks": res["tc_peaks"], "clocks": res["clocks"], "cpu_baseline": None,
            }
            if world == 1 and not args.no_cpu_baseline:
                val, sample, secs = oracle_prefill_sample(args.workload)
                ncpu, model = _cpu_info()
                line["cpu_baseline"] = {"value": round(val, 3), "unit": "tokens/s",
                                        "cores": _blas_threads(), "nproc": ncpu,
                                        "cpu_model": model, "kind": "oracle", "sample": sample,
                                        "seconds": round(secs, 1)}
            print(json.dumps(line), flush=True)
        if dist is not None:
            dist.barrier()
            dist.destroy_process_group()
        return
    res = run_gpu(args, dist, rank, world)
    if res.get("profile"):
        if rank == 0:
            print(json.dumps({"profile": args.workload, "ms_per_step": res["ms"],
                              "launches_per_step": res["launches"]}), flush=True)
        return
    if rank == 0:
        w = synth.WORKLOADS[args.workload]
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            val, sample, secs = oracle_sample(args.workload)
            ncpu, model = _cpu_info()
            cpu = {"value": round(val, 4), "unit": "queries/s", "cores": _blas_threads(),
                   "kind": "oracle", "sample": sample, "seconds": round(secs, 1),
                   "nproc": ncpu, "cpu_model": model,
                   "threads": "numpy/BLAS threads of the fp64 matrix products (cores)"}
        line = {
            "metric": METRIC, "value": round(res["value"], 1), "unit": "queries/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(res["ms"], 5), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "e4m3+bf16 KV, mxfp4 indexer, f32 accumulate",
            "data": "synthetic",
            "config": {"workload": args.workload, "batch_per_gpu": w.B, "context": w.L,
                       "layers": [f"{ly.kind} m={ly.m} H={ly.H} d={ly.d}" +
                                  (f" top_k={ly.top_k} H_I={ly.H_I}x{ly.d_I}" if ly.kind == "csa"
                                   else "") for ly in w.layers],
                       "l2": "flushed between steps (320 MB write, then read back: cold and clean)",
                       "parallelism": f"dp{world} (independent sequences)",
                       "graph": "one CUDA graph per step"},
            "e2e": {"value": round(res["e2e"]["value"], 1), "unit": "queries/s",
                    "h2d_bytes_per_step": int(res["e2e"]["h2d"]),
                    "d2h_bytes_per_step": int(res["e2e"]["d2h"]),
                    "ms_per_step": round(res["e2e"]["ms"], 5),
                    "how": "every step: pinned H2D of each layer's inputs on a copy stream, "
                           "one captured graph per layer, D2H of each layer's output on a "
                           "second copy stream (layer l+1's inputs up and layer l's output "
                           "down while the other layer runs)",
                    "eager": {"value": round(res["e2e"]["eager_value"], 1),
                              "ms_per_step": round(res["e2e"]["eager_ms"], 5),
                              "how": "the same copies around eager calls through the binding"}},
            "tc_peaks": res["tc_peaks"],
            "gpu_launches": res["launches"] * args.steps,
            "roofline": res["roof"],
            "step_roofline": res["step_roof"],
            "cpu_baseline": cpu,
            "clocks": res["clocks"],
            "also": res["also"],
            "bf16_score_selector": res.get("bf16_selector"),
            "paged_kv": res.get("paged"),
        }
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
