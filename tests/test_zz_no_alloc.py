"""The no-allocation indexer entry point (v4attn_index_topk_noalloc) gives the
same selection as v4attn_index_topk with a caller-allocated workspace.

It exists for callers that cannot call cudaMalloc (code inside a framework
that owns the device allocator, or a serving loop that may not allocate after
start-up); its scratch is an array built into the library.  The test makes two
calls in a row with different queries, since every call shares that array and
the second must not see the first's leftovers.  This file is collected last
so that a run stopping at the first failure has already run every other test.
"""
import numpy as np
import pytest
import torch

import synth
from tests.gpu_util import check_topk, code_rows, desc_for, dev, v4

pytestmark = pytest.mark.gpu


def _case(seed, B=8, N=20000, H_I=64, d_I=128):
    rng = np.random.default_rng(seed)
    keys = rng.standard_normal((B, N, d_I)).astype(np.float32)
    positions = 4 * rng.integers(N // 2, N, B) + rng.integers(0, 4, B)
    qI = rng.standard_normal((B, H_I, d_I)).astype(np.float32)
    w = rng.uniform(0, 1, (B, H_I)).astype(np.float32)
    return keys, positions, qI, w


def test_noalloc_matches_workspace_call_twice():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    v = v4()
    B, N, H_I, d_I, k = 8, 20000, 64, 128, 512
    ly = synth.Layer("csa", 4, 64, 512, 64, 128, H_I, d_I, k)
    desc = desc_for(ly)
    for call, seed in enumerate((101, 202)):
        keys, positions, qI, w = _case(seed, B, N, H_I, d_I)
        krows, ksf = code_rows(desc, dev(keys), v.MXFP4)
        qrows, qsf = code_rows(desc, dev(qI.reshape(1, B * H_I, d_I)), v.MXFP4)
        qrows, qsf = qrows.reshape(B, H_I, -1), qsf.reshape(B, H_I, -1)
        kw = dict(qI=qrows, qI_sf=qsf, w=dev(w), q_pos=dev(positions, torch.int64), keys=krows,
                  keys_sf=ksf, key_rows=N, max_vis=N, B=B)
        ref = torch.full((B, k), -5, dtype=torch.int32, device="cuda")
        ref_scores = torch.zeros(B, N, dtype=torch.float32, device="cuda")
        ws = v.workspace(desc, B, N)
        v.index_topk(desc, idx_out=ref, scores_out=ref_scores, ws=ws, **kw)
        got = torch.full((B, k), -7, dtype=torch.int32, device="cuda")
        v.index_topk_noalloc(desc, idx_out=got, **kw)
        torch.cuda.synchronize()
        g, r, s = got.cpu().numpy(), ref.cpu().numpy(), ref_scores.cpu().numpy()
        for b in range(B):
            nv = (int(positions[b]) + 1) // 4
            # the same selection as the workspace call, within the top-k tolerance
            check_topk(g[b], s[b], nv, k)
            assert set(g[b].tolist()) == set(r[b].tolist()), (call, b)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    v = v4()
    ly = synth.Layer("csa", 4, 64, 512, 64, 128, 64, 128, 512)
    desc = desc_for(ly)
    n_q, N = 16, 200000                     # 3.2M scores > the built-in scratch
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
    assert e.value.status == 2              # V4A_ERR_UNSUPPORTED
