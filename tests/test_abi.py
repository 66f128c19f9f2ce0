"""The C-ABI library loads, exports every entry point include/v4attn.h
declares, its ctypes mirror matches the C struct layouts (checked against a
gcc-compiled probe of the header), and host-side argument checks reject bad
calls before anything is launched (no GPU needed)."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "v4attn.h")


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(v4attn_\w+)\s*\(", text)))


def test_library_exports_every_declared_entry_point():
    from long_context_compressed_kv_b200 import _abi
    lib = _abi.load()
    names = _declared_functions()
    assert len(names) >= 11
    for n in names:
        assert hasattr(lib, n), n
        assert n in _abi.SIGNATURES, n
    # and nothing in the binding is missing from the header
    assert set(_abi.SIGNATURES) <= set(names)


def test_struct_layouts_match_header(tmp_path):
    from long_context_compressed_kv_b200 import _abi
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "v4attn.h"', "int main(void){"]
    for cname, cls in _abi.STRUCTS.items():
        lines.append(f'printf("{cname} %zu\\n", sizeof({cname}));')
        for fname, _ in cls._fields_:
            lines.append(f'printf("{cname}.{fname} %zu\\n", offsetof({cname}, {fname}));')
    lines.append("return 0;}")
    src = tmp_path / "probe.c"
    src.write_text("\n".join(lines))
    exe = tmp_path / "probe"
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), "-I", "/usr/local/cuda/include",
                    str(src), "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout
    got = dict(line.split() for line in out.strip().splitlines())
    for cname, cls in _abi.STRUCTS.items():
        assert int(got[cname]) == ctypes.sizeof(cls), cname
        for fname, _ in cls._fields_:
            assert int(got[f"{cname}.{fname}"]) == getattr(cls, fname).offset, (cname, fname)


def test_host_side_validation_rejects_bad_calls():
    from long_context_compressed_kv_b200 import _abi
    lib = _abi.load()
    d = _abi.LayerDesc(_abi.HCA, 128, 128, 64, 512, 64, 160000.0, 0.0, 0, 0, 0,
                       _abi.E4M3_BF16ROPE, _abi.MXFP4, 1e-6)
    assert lib.v4attn_workspace_size(ctypes.byref(d), 16, 1024) > 0
    bad = _abi.LayerDesc.from_buffer_copy(d)
    bad.d = 100                                   # not a multiple of 32
    assert lib.v4attn_workspace_size(ctypes.byref(bad), 16, 1024) == 0
    assert lib.v4attn_dense_mqa(ctypes.byref(bad), None, None, 0, None) == _abi.ERR_UNSUPPORTED
    assert lib.v4attn_dense_mqa(ctypes.byref(d), None, None, 0, None) == _abi.ERR_INVALID_ARG
    a = _abi.MqaArgs()
    a.n_q = 1
    a.B = 1
    assert lib.v4attn_dense_mqa(ctypes.byref(d), ctypes.byref(a), None, 0, None) == \
        _abi.ERR_INVALID_ARG                      # null pointers
    fp8_other = _abi.LayerDesc.from_buffer_copy(d)
    fp8_other.d = 256
    assert lib.v4attn_workspace_size(ctypes.byref(fp8_other), 1, 1) == 0
    c = _abi.CompressArgs()
    assert lib.v4attn_compress(ctypes.byref(d), ctypes.byref(c), None, 0, None) == \
        _abi.ERR_INVALID_ARG
    p = _abi.ProjectArgs()
    p.M, p.N, p.K = 4, 4, 4
    assert lib.v4attn_project(ctypes.byref(p), None) == _abi.ERR_INVALID_ARG
    assert lib.v4attn_status_string(_abi.ERR_WORKSPACE) == b"workspace missing or too small"
    assert b"sm_100a" in lib.v4attn_build_info()


def test_csa_workspace_covers_index_and_sparse_mqa():
    from long_context_compressed_kv_b200 import _abi
    lib = _abi.load()
    d = _abi.LayerDesc(_abi.CSA, 4, 128, 128, 512, 64, 160000.0, 0.0, 64, 128, 1024,
                       _abi.E4M3_BF16ROPE, _abi.MXFP4, 1e-6)
    n = lib.v4attn_workspace_size(ctypes.byref(d), 4, 262144)
    assert n >= 4 * 262144 * 4                    # fp32 scores of every visible key


def _no_gpu():
    try:
        import torch
        return not torch.cuda.is_available()
    except Exception:
        return True


@pytest.mark.skipif(not _no_gpu(), reason="host-only check with fake device pointers")
def test_every_entry_point_rejects_a_short_workspace():
    """Each call checks its workspace on the host before launching: a decode
    step given one byte less than v4attn_workspace_size, an indexer call
    without room for its scores, an MQA call without room for its partials
    all return V4A_ERR_WORKSPACE.  The pointers are fake (never touched: every
    check here runs before a launch)."""
    from long_context_compressed_kv_b200 import _abi
    lib = _abi.load()
    fake = ctypes.c_void_p(1 << 20)          # 16-byte aligned, never dereferenced
    B, L = 4, 1 << 20
    for kind, m, kv, idx in ((_abi.CSA, 4, _abi.E4M3_BF16ROPE, _abi.MXFP4),
                             (_abi.HCA, 128, _abi.E4M3_BF16ROPE, _abi.MXFP4),
                             (_abi.CSA, 4, _abi.F32, _abi.F32)):
        csa = kind == _abi.CSA
        d = _abi.LayerDesc(kind, m, 128, 128, 512, 64, 160000.0, 0.0, 64 if csa else 0,
                           128 if csa else 0, 1024 if csa else 0, kv, idx, 1e-6)
        rows = L // m
        need = lib.v4attn_workspace_size(ctypes.byref(d), B, rows)
        assert need > 0
        a = _abi.DecodeArgs()
        a.B = B
        for f in ("pos", "x_main", "tail", "bias", "kv", "kv_scale", "swa", "swa_scale", "Q",
                  "sink", "out"):
            setattr(a, f, fake)
        if csa:
            for f in ("x_idx", "itail", "ibias", "keys", "keys_sf", "qI", "qI_sf", "w", "idx_out"):
                setattr(a, f, fake)
        a.in_dtype = _abi.BF16
        a.q_dtype = _abi.BF16
        a.out_dtype = _abi.BF16
        a.kv_rows = a.key_rows = rows
        a.swa_rows = 128
        a.max_vis = rows
        assert lib.v4attn_decode(ctypes.byref(d), ctypes.byref(a), fake, need - 1, None) == \
            _abi.ERR_WORKSPACE
        q = _abi.MqaArgs()
        q.n_q, q.B = B, B
        for f in ("Q", "q_pos", "kv", "kv_scale", "swa", "swa_scale", "sink", "out"):
            setattr(q, f, fake)
        q.q_dtype = q.out_dtype = _abi.BF16
        q.kv_rows, q.swa_rows, q.max_vis = rows, 128, rows
        if csa:
            q.idx, q.n_sel = fake, 1024
            assert lib.v4attn_sparse_mqa(ctypes.byref(d), ctypes.byref(q), fake, 1024,
                                         None) == _abi.ERR_WORKSPACE
            ix = _abi.IndexArgs()
            ix.n_q, ix.B = B, B
            for f in ("qI", "qI_sf", "w", "q_pos", "keys", "keys_sf", "idx_out"):
                setattr(ix, f, fake)
            ix.key_rows = ix.max_vis = rows
            # the scores of every visible key of every query do not fit in 4 MB - 1
            assert lib.v4attn_index_topk(ctypes.byref(d), ctypes.byref(ix), fake,
                                         4 * B * rows - 1, None) == _abi.ERR_WORKSPACE
        else:
            assert lib.v4attn_dense_mqa(ctypes.byref(d), ctypes.byref(q), fake, 1024,
                                        None) == _abi.ERR_WORKSPACE


@pytest.mark.skipif(not _no_gpu(), reason="host-only check with fake device pointers")
def test_tensor_core_formats_are_refused_not_downgraded():
    """An MXFP4 indexer or E4M3 MQA call that the tensor-core kernel does not
    take is refused before any launch (no slower fallback runs): an MXFP4
    indexer with d_I = 64 or a key row count not divisible by 4 ->
    V4A_ERR_UNSUPPORTED, a misaligned pointer -> V4A_ERR_INVALID_ARG; an E4M3
    MQA with an fp32 Q -> V4A_ERR_UNSUPPORTED; a decode step whose indexer is
    refused launches nothing either (fake pointers, never dereferenced)."""
    from long_context_compressed_kv_b200 import _abi
    lib = _abi.load()
    fake = ctypes.c_void_p(1 << 20)
    ws = ctypes.c_void_p(1 << 21)
    big = 1 << 40

    def index_call(d_I, key_rows, qI=fake):
        d = _abi.LayerDesc(_abi.CSA, 4, 128, 64, 512, 64, 160000.0, 0.0, 64, d_I, 512,
                           _abi.E4M3_BF16ROPE, _abi.MXFP4, 1e-6)
        ix = _abi.IndexArgs()
        ix.n_q = ix.B = 2
        for f in ("qI_sf", "w", "q_pos", "keys", "keys_sf", "idx_out"):
            setattr(ix, f, fake)
        ix.qI = qI
        ix.key_rows = ix.max_vis = key_rows
        return lib.v4attn_index_topk(ctypes.byref(d), ctypes.byref(ix), ws, big, None)
    assert index_call(64, 4096) == _abi.ERR_UNSUPPORTED
    assert index_call(128, 4098) == _abi.ERR_UNSUPPORTED
    assert index_call(128, 4096, ctypes.c_void_p((1 << 20) + 8)) == _abi.ERR_INVALID_ARG
    d = _abi.LayerDesc(_abi.HCA, 128, 128, 64, 512, 64, 160000.0, 0.0, 0, 0, 0,
                       _abi.E4M3_BF16ROPE, _abi.MXFP4, 1e-6)
    q = _abi.MqaArgs()
    q.n_q, q.B = 2, 2
    for f in ("Q", "q_pos", "kv", "kv_scale", "swa", "swa_scale", "sink", "out"):
        setattr(q, f, fake)
    q.q_dtype, q.out_dtype = _abi.F32, _abi.BF16
    q.kv_rows, q.swa_rows, q.max_vis = 1024, 128, 1024
    assert lib.v4attn_dense_mqa(ctypes.byref(d), ctypes.byref(q), ws, big, None) == \
        _abi.ERR_UNSUPPORTED
    q.q_dtype = _abi.BF16
    q.Q = ctypes.c_void_p((1 << 20) + 2)
    assert lib.v4attn_dense_mqa(ctypes.byref(d), ctypes.byref(q), ws, big, None) == \
        _abi.ERR_INVALID_ARG
    # decode: the indexer of this step is refused before the append launch
    dc = _abi.LayerDesc(_abi.CSA, 4, 128, 64, 512, 64, 160000.0, 0.0, 64, 64, 512,
                        _abi.E4M3_BF16ROPE, _abi.MXFP4, 1e-6)
    a = _abi.DecodeArgs()
    a.B = 2
    for f in ("pos", "x_main", "tail", "bias", "kv", "kv_scale", "swa", "swa_scale", "Q", "sink",
              "out", "x_idx", "itail", "ibias", "keys", "keys_sf", "qI", "qI_sf", "w", "idx_out"):
        setattr(a, f, fake)
    a.in_dtype = a.q_dtype = a.out_dtype = _abi.BF16
    a.kv_rows = a.key_rows = 4096
    a.swa_rows = 128
    a.max_vis = 4096
    assert lib.v4attn_decode(ctypes.byref(dc), ctypes.byref(a), ws, big, None) == \
        _abi.ERR_UNSUPPORTED


@pytest.mark.skipif(not _no_gpu(), reason="host-only check with fake device pointers")
def test_block_table_arguments_are_checked():
    """Paged caches (include/v4attn.h, "Paged caches"): a block table needs at
    least one block per sequence, a 4-byte aligned table, a pool of whole blocks
    (32 CSA entries / indexer keys or 1 HCA entry a block), a visible bound
    within the table, and the tensor-core formats; each violation is refused
    before any launch (fake pointers, never dereferenced)."""
    from long_context_compressed_kv_b200 import _abi
    lib = _abi.load()
    fake = ctypes.c_void_p(1 << 20)
    ws = ctypes.c_void_p(1 << 21)
    big = 1 << 40

    def mqa(kind, m, kv_fmt, kv_rows, bps, max_vis, bt=fake):
        d = _abi.LayerDesc(kind, m, 128, 64, 512, 64, 160000.0, 0.0, 64, 128, 64, kv_fmt,
                           _abi.MXFP4, 1e-6)
        q = _abi.MqaArgs()
        q.n_q, q.B = 2, 2
        for f in ("Q", "q_pos", "kv", "kv_scale", "swa", "swa_scale", "sink", "out"):
            setattr(q, f, fake)
        q.q_dtype, q.out_dtype = _abi.BF16, _abi.BF16
        q.kv_rows, q.swa_rows, q.max_vis = kv_rows, 128, max_vis
        q.block_table, q.blocks_per_seq = bt, bps
        if kind == _abi.CSA:
            q.idx, q.n_sel = fake, 64
            return lib.v4attn_sparse_mqa(ctypes.byref(d), ctypes.byref(q), ws, big, None)
        return lib.v4attn_dense_mqa(ctypes.byref(d), ctypes.byref(q), ws, big, None)
    assert mqa(_abi.HCA, 128, _abi.E4M3_BF16ROPE, 1024, 0, 16) == _abi.ERR_INVALID_ARG
    assert mqa(_abi.HCA, 128, _abi.E4M3_BF16ROPE, 1024, 8, 16,
               ctypes.c_void_p((1 << 20) + 2)) == _abi.ERR_INVALID_ARG
    assert mqa(_abi.HCA, 128, _abi.F32, 1024, 8, 8) == _abi.ERR_UNSUPPORTED
    assert mqa(_abi.HCA, 128, _abi.E4M3_BF16ROPE, 1024, 8, 9) == _abi.ERR_INVALID_ARG
    assert mqa(_abi.CSA, 4, _abi.E4M3_BF16ROPE, 1000, 8, 256) == _abi.ERR_INVALID_ARG

    def index(idx_fmt, key_rows, bps, max_vis):
        d = _abi.LayerDesc(_abi.CSA, 4, 128, 64, 512, 64, 160000.0, 0.0, 64, 128, 512,
                           _abi.E4M3_BF16ROPE, idx_fmt, 1e-6)
        ix = _abi.IndexArgs()
        ix.n_q = ix.B = 2
        for f in ("qI", "qI_sf", "w", "q_pos", "keys", "keys_sf", "idx_out"):
            setattr(ix, f, fake)
        ix.key_rows, ix.max_vis = key_rows, max_vis
        ix.block_table, ix.blocks_per_seq = fake, bps
        return lib.v4attn_index_topk(ctypes.byref(d), ctypes.byref(ix), ws, big, None)
    assert index(_abi.F32, 4096, 16, 512) == _abi.ERR_UNSUPPORTED
    assert index(_abi.MXFP4, 4096 + 16, 16, 512) == _abi.ERR_INVALID_ARG
    assert index(_abi.MXFP4, 4096, 16, 513) == _abi.ERR_INVALID_ARG
