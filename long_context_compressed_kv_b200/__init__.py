"""Python binding of libv4attn: DeepSeek-V4 hybrid compressed attention
(CSA / HCA) on B200.

Argument marshalling only: every function turns torch tensors into the
pointers and sizes of the C ABI (include/v4attn.h) and calls the library on
the current CUDA stream.  Every step of the hot path runs in the library's
CUDA kernels; there is no CPU or PyTorch fallback, and importing this module
raises when the library has not been built.
"""
from __future__ import annotations

import ctypes
from typing import Optional

import torch

from . import _abi
from ._abi import (BF16, CSA, E4M3_BF16ROPE, F32, HCA, MXFP4, CompressArgs, DecodeArgs,
                   IndexArgs, LayerDesc, MqaArgs, ProjectArgs)

_lib = _abi.load()

__all__ = ["F32", "BF16", "E4M3_BF16ROPE", "MXFP4", "CSA", "HCA", "V4AttnError", "layer_desc",
           "workspace", "workspace_size", "workspace_init", "compress", "index_topk",
           "index_topk_noalloc", "noalloc_device_status", "debug_index_stall",
           "device_status_code", "tc_peak_probe",
           "sparse_mqa", "dense_mqa",
           "decode", "project", "device_status", "build_info", "row_bytes"]


class V4AttnError(RuntimeError):
    def __init__(self, fn: str, status: int):
        msg = _lib.v4attn_status_string(status).decode()
        if status == _abi.ERR_CUDA:
            msg += ": " + _lib.v4attn_last_cuda_error().decode()
        super().__init__(f"{fn}: {msg} (status {status})")
        self.status = status


def _check(fn: str, status: int):
    if status != _abi.OK:
        raise V4AttnError(fn, status)


def _p(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensor must live on the GPU")
    return t.data_ptr()


def _stream(stream=None) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.bfloat16:
        return BF16
    raise ValueError(f"unsupported dtype {t.dtype}")


def row_bytes(fmt: int, c: int, d_rope: int = 64) -> int:
    if fmt == F32:
        return 4 * c
    if fmt == E4M3_BF16ROPE:
        return (c - d_rope) + 2 * d_rope
    if fmt == MXFP4:
        return c // 2
    raise ValueError(fmt)


def layer_desc(kind: int, m: int, H: int, d: int, d_rope: int, n_win: int = 128,
               rope_theta: float = 160000.0, softmax_scale: float = 0.0, H_I: int = 0,
               d_I: int = 0, top_k: int = 0, kv_dtype: int = E4M3_BF16ROPE,
               idx_dtype: int = MXFP4, rms_eps: float = 1e-6) -> LayerDesc:
    return LayerDesc(kind, m, n_win, H, d, d_rope, rope_theta, softmax_scale, H_I, d_I, top_k,
                     kv_dtype, idx_dtype, rms_eps)


def workspace_size(desc: LayerDesc, n_q: int, max_vis: int) -> int:
    n = _lib.v4attn_workspace_size(ctypes.byref(desc), n_q, max_vis)
    if n == 0:
        raise V4AttnError("v4attn_workspace_size", _abi.ERR_INVALID_ARG)
    return n


def workspace(desc: LayerDesc, n_q: int, max_vis: int, device="cuda") -> torch.Tensor:
    """A zero-status workspace for calls on this layer with <= n_q queries."""
    ws = torch.empty(workspace_size(desc, n_q, max_vis), dtype=torch.uint8, device=device)
    _check("v4attn_workspace_init", _lib.v4attn_workspace_init(_p(ws), ws.numel(), _stream()))
    return ws


def compress(desc: LayerDesc, *, m: int, overlap: bool, c: int, Ca, Za, Cb=None, Zb=None,
             in_rows: int, in_seq_stride: int, in_row_stride: int, bias=None, seq_len,
             entry_begin, n_entries: int, out_dtype: int, out, out_scale=None, out_rows: int,
             complete_only=False, apply_rmsnorm=True, apply_rope=True, ws=None, stream=None):
    a = CompressArgs(m, int(overlap), c, int(seq_len.numel()), _p(Ca), _p(Za), _p(Cb), _p(Zb),
                     _dt(Ca), in_seq_stride, in_row_stride, in_rows, _p(bias), _p(seq_len),
                     _p(entry_begin), n_entries, int(complete_only), int(apply_rmsnorm),
                     int(apply_rope), out_dtype, _p(out), _p(out_scale), out_rows)
    _check("v4attn_compress", _lib.v4attn_compress(ctypes.byref(desc), ctypes.byref(a), _p(ws),
                                                   0 if ws is None else ws.numel(),
                                                   _stream(stream)))


def _bt(block_table):
    """(pointer, blocks per sequence) of an int32 [B][blocks_per_seq] block table, or (None, 0)."""
    if block_table is None:
        return None, 0
    assert block_table.dim() == 2 and block_table.is_contiguous()
    return _p(block_table), int(block_table.shape[1])


def index_topk(desc: LayerDesc, *, qI, w, q_pos, keys, key_rows: int, max_vis: int, idx_out, ws,
               qI_sf=None, keys_sf=None, q_seq=None, B: Optional[int] = None, scores_out=None,
               score_dtype: int = F32, block_table=None, stream=None):
    """Indexer scores + top-k (see include/v4attn.h); with ``block_table``
    (int32 [B][blocks_per_seq]) the keys are a paged pool of ``key_rows`` rows."""
    n_q = int(q_pos.numel())
    bt, bps = _bt(block_table)
    a = IndexArgs(n_q, B if B is not None else n_q, _p(qI), _p(qI_sf), _p(w), _p(q_seq),
                  _p(q_pos), _p(keys), _p(keys_sf), key_rows, max_vis, _p(idx_out),
                  _p(scores_out), score_dtype, bt, bps)
    _check("v4attn_index_topk", _lib.v4attn_index_topk(ctypes.byref(desc), ctypes.byref(a),
                                                       _p(ws), ws.numel(), _stream(stream)))


def index_topk_noalloc(desc: LayerDesc, *, qI, w, q_pos, keys, key_rows: int, max_vis: int,
                       idx_out, qI_sf=None, keys_sf=None, q_seq=None, B: Optional[int] = None,
                       scores_out=None, stream=None):
    """index_topk with the library's built-in scratch instead of a workspace,
    for callers that cannot allocate device memory (see include/v4attn.h)."""
    n_q = int(q_pos.numel())
    a = IndexArgs(n_q, B if B is not None else n_q, _p(qI), _p(qI_sf), _p(w), _p(q_seq),
                  _p(q_pos), _p(keys), _p(keys_sf), key_rows, max_vis, _p(idx_out),
                  _p(scores_out), F32)
    _check("v4attn_index_topk_noalloc",
           _lib.v4attn_index_topk_noalloc(ctypes.byref(desc), ctypes.byref(a), _stream(stream)))


def noalloc_device_status(stream=None) -> int:
    """Raw status word of the last index_topk_noalloc call on this device
    (synchronises); raises on a device-side error."""
    bits = ctypes.c_uint32(0)
    st = _lib.v4attn_noalloc_device_status(_stream(stream), ctypes.byref(bits))
    _check("v4attn_noalloc_device_status", st)
    return bits.value


def debug_index_stall(desc: LayerDesc, *, qI, w, q_pos, keys, key_rows: int, max_vis: int, ws,
                      wait_ns: int, qI_sf=None, keys_sf=None, q_seq=None, B=None,
                      scores_out=None, idx_out=None, stream=None):
    """Failure-detection hook: index_topk with one wait of the tensor-core
    indexer made to run out after ``wait_ns`` (see include/v4attn.h)."""
    n_q = int(q_pos.numel())
    a = IndexArgs(n_q, B if B is not None else n_q, _p(qI), _p(qI_sf), _p(w), _p(q_seq),
                  _p(q_pos), _p(keys), _p(keys_sf), key_rows, max_vis, _p(idx_out),
                  _p(scores_out), F32)
    _check("v4attn_debug_index_stall",
           _lib.v4attn_debug_index_stall(ctypes.byref(desc), ctypes.byref(a), _p(ws), ws.numel(),
                                         int(wait_ns), _stream(stream)))


def tc_peak_probe(kind: int, n_iter: int, n_cols: int = 256, ws=None, stream=None):
    """Launch the tensor-core throughput probe (see include/v4attn.h);
    returns (dense FLOPs of the launch, CTAs)."""
    n = ctypes.c_int32(0)
    f = ctypes.c_double(0.0)
    _check("v4attn_tc_peak_probe",
           _lib.v4attn_tc_peak_probe(int(kind), int(n_cols), int(n_iter), ctypes.byref(n),
                                     ctypes.byref(f), _p(ws), _stream(stream)))
    return f.value, n.value


def device_status_code(ws, stream=None):
    """(status code, raw word) of a workspace, without raising."""
    bits = ctypes.c_uint32(0)
    st = _lib.v4attn_device_status(_p(ws), _stream(stream), ctypes.byref(bits))
    return st, bits.value


def workspace_init(ws, stream=None):
    _check("v4attn_workspace_init", _lib.v4attn_workspace_init(_p(ws), ws.numel(),
                                                                _stream(stream)))


def _mqa(fn, desc, Q, q_pos, kv, kv_rows, swa, swa_rows, out, ws, kv_scale, swa_scale, q_seq, B,
         idx, n_sel, max_vis, sink, lse, q_rmsnorm, stream, block_table=None):
    n_q = int(q_pos.numel())
    bt, bps = _bt(block_table)
    a = MqaArgs(n_q, B if B is not None else n_q, _p(Q), _dt(Q), int(q_rmsnorm), _p(q_seq),
                _p(q_pos), _p(kv), _p(kv_scale), kv_rows, _p(swa), _p(swa_scale), swa_rows,
                _p(idx), n_sel, max_vis, _p(sink), _p(out), _dt(out), _p(lse), bt, bps)
    _check(fn, getattr(_lib, fn)(ctypes.byref(desc), ctypes.byref(a), _p(ws), ws.numel(),
                                 _stream(stream)))


def sparse_mqa(desc: LayerDesc, *, Q, q_pos, kv, kv_rows: int, swa, swa_rows: int, idx, out, ws,
               kv_scale=None, swa_scale=None, q_seq=None, B=None, sink=None, lse=None,
               q_rmsnorm=False, block_table=None, stream=None):
    _mqa("v4attn_sparse_mqa", desc, Q, q_pos, kv, kv_rows, swa, swa_rows, out, ws, kv_scale,
         swa_scale, q_seq, B, idx, int(idx.shape[-1]), 0, sink, lse, q_rmsnorm, stream,
         block_table)


def dense_mqa(desc: LayerDesc, *, Q, q_pos, kv, kv_rows: int, swa, swa_rows: int, max_vis: int,
              out, ws, kv_scale=None, swa_scale=None, q_seq=None, B=None, sink=None, lse=None,
              q_rmsnorm=False, block_table=None, stream=None):
    _mqa("v4attn_dense_mqa", desc, Q, q_pos, kv, kv_rows, swa, swa_rows, out, ws, kv_scale,
         swa_scale, q_seq, B, None, 0, max_vis, sink, lse, q_rmsnorm, stream, block_table)


def decode(desc: LayerDesc, *, pos, x_main, tail, bias, kv, kv_rows: int, swa, swa_rows: int,
           Q, out, ws, max_vis: int, kv_scale=None, swa_scale=None, x_idx=None, itail=None,
           ibias=None, keys=None, keys_sf=None, key_rows: int = 0, qI=None, qI_sf=None, w=None,
           sink=None, lse=None, idx_out=None, block_table=None, stream=None):
    bt, bps = _bt(block_table)
    a = DecodeArgs(int(pos.numel()), _p(pos), _dt(x_main), _p(x_main), _p(tail), _p(bias),
                   _p(x_idx), _p(itail), _p(ibias), _p(kv), _p(kv_scale), kv_rows, _p(keys),
                   _p(keys_sf), key_rows, _p(swa), _p(swa_scale), swa_rows, _p(Q), _dt(Q),
                   _p(qI), _p(qI_sf), _p(w), _p(sink), _p(out), _dt(out), _p(lse), _p(idx_out),
                   max_vis, bt, bps)
    _check("v4attn_decode", _lib.v4attn_decode(ctypes.byref(desc), ctypes.byref(a), _p(ws),
                                               ws.numel(), _stream(stream)))


def project(X, W, Y, stream=None):
    """Y = X @ W for 2-D row-major views (leading-dimension strides allowed)."""
    M, K = X.shape
    K2, N = W.shape
    assert K == K2 and tuple(Y.shape) == (M, N)
    for t in (X, W, Y):
        assert t.stride(1) == 1
    a = ProjectArgs(M, N, K, _p(X), _dt(X), X.stride(0), _p(W), _dt(W), W.stride(0), _p(Y), _dt(Y),
                    Y.stride(0))
    _check("v4attn_project", _lib.v4attn_project(ctypes.byref(a), _stream(stream)))


def device_status(ws, stream=None) -> int:
    """Synchronise and return the raw status word; raises on a device-side error."""
    bits = ctypes.c_uint32(0)
    st = _lib.v4attn_device_status(_p(ws), _stream(stream), ctypes.byref(bits))
    _check("v4attn_device_status", st)
    return bits.value


def build_info() -> str:
    return _lib.v4attn_build_info().decode()
