"""The no-allocation indexer entry point (v4attn_index_topk_noalloc) against
the oracle, and against v4attn_index_topk with a caller-allocated workspace.

The entry point exists for callers that cannot call cudaMalloc: code inside a
framework that owns the device allocator, or a serving loop that may not
allocate once it has started.  Its scratch is an array built into the
library, shared by every call.  The test makes two calls in a row, the second
over fewer visible keys than the first, so that scores the first call left in
the shared array past the second call's range would show up in its selection.
This file is collected last so that a run stopping at the first failure has
already run every other test.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import indexer as oidx
from tests.gpu_util import check_topk, code_rows, desc_for, dev, read_keys, v4

pytestmark = pytest.mark.gpu


def _case(seed, B, N, H_I, d_I, lo, hi):
    rng = np.random.default_rng(seed)
    keys = rng.standard_normal((B, N, d_I)).astype(np.float32)
    positions = 4 * rng.integers(lo, hi, B) + rng.integers(0, 4, B)
    qI = rng.standard_normal((B, H_I, d_I)).astype(np.float32)
    w = rng.uniform(0, 1, (B, H_I)).astype(np.float32)
    return keys, positions, qI, w


def test_noalloc_matches_oracle_and_workspace_call_twice():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    v = v4()
    B, N, H_I, d_I, k = 8, 20000, 64, 128, 512
    ly = synth.Layer("csa", 4, 64, 512, 64, 128, H_I, d_I, k)
    desc = desc_for(ly)
    # first call: 10000..20000 visible keys per query; second: 600..5000
    for call, (seed, lo, hi) in enumerate(((101, N // 2, N), (202, 150, 1250))):
        keys, positions, qI, w = _case(seed, B, N, H_I, d_I, lo, hi)
        max_vis = int(max((positions + 1) // 4))
        krows, ksf = code_rows(desc, dev(keys), v.MXFP4)
        qrows, qsf = code_rows(desc, dev(qI.reshape(1, B * H_I, d_I)), v.MXFP4)
        qrows, qsf = qrows.reshape(B, H_I, -1), qsf.reshape(B, H_I, -1)
        kw = dict(qI=qrows, qI_sf=qsf, w=dev(w), q_pos=dev(positions, torch.int64), keys=krows,
                  keys_sf=ksf, key_rows=N, max_vis=max_vis, B=B)
        got = torch.full((B, k), -7, dtype=torch.int32, device="cuda")
        v.index_topk_noalloc(desc, idx_out=got, **kw)
        assert v.noalloc_device_status() == 0
        ref = torch.full((B, k), -5, dtype=torch.int32, device="cuda")
        ws = v.workspace(desc, B, max_vis)
        v.index_topk(desc, idx_out=ref, ws=ws, **kw)
        torch.cuda.synchronize()
        g, r = got.cpu().numpy(), ref.cpu().numpy()
        # the oracle scores the keys and queries as stored (stage-wise)
        kd = read_keys(krows, ksf, v.MXFP4)
        qd = read_keys(qrows, qsf, v.MXFP4)
        for b in range(B):
            nv = (int(positions[b]) + 1) // 4
            s = oidx.scores(qd[b], w[b], kd[b, :nv])
            check_topk(g[b], s, nv, k)
            # both entry points run the same kernels on the same data
            assert np.array_equal(g[b], r[b]), (call, b)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    v = v4()
    ly = synth.Layer("csa", 4, 64, 512, 64, 128, 64, 128, 512)
    desc = desc_for(ly)

    def call(n_q, N):
        keys = torch.zeros(1, N, 64, dtype=torch.uint8, device="cuda")
        ksf = torch.zeros(1, N, 4, dtype=torch.uint8, device="cuda")
        q = torch.zeros(n_q, 64, 64, dtype=torch.uint8, device="cuda")
        qsf = torch.zeros(n_q, 64, 4, dtype=torch.uint8, device="cuda")
        idx = torch.zeros(n_q, 512, dtype=torch.int32, device="cuda")
        with pytest.raises(v.V4AttnError) as e:
            v.index_topk_noalloc(desc, qI=q, qI_sf=qsf, w=torch.ones(n_q, 64, device="cuda"),
                                 q_pos=torch.full((n_q,), 4 * N - 1, dtype=torch.int64,
                                                  device="cuda"),
                                 q_seq=torch.zeros(n_q, dtype=torch.int32, device="cuda"), B=1,
                                 keys=keys, keys_sf=ksf, key_rows=N, max_vis=N, idx_out=idx)
        assert e.value.status == 2          # V4A_ERR_UNSUPPORTED, nothing launched
    call(16, 200000)                        # 3.2M scores > the built-in scratch
    call(1366, 4)                           # more queries than the stated limit
